// bwd_scalarA.cuh -- gradients of the scalar-A (Mamba-2 / SSD) scan, sm_100a.
//
// Training differentiates the recurrence of the forward pass ("03 -- Modelos
// de espacio de estados", sections "Discretizacion" and "Parallel scan";
// "P20 -- Mamba", section 5).  With a scalar transition per head ("Mamba-3",
// first section) the forward pass over a chunk of Q tokens has the matrix
// form of structured state-space duality ("Mamba-2 y state-space models",
// section 4.2); this file differentiates that form chunk by chunk, from the
// last chunk to the first.
//
// Per head (state h: N x P), chunk tokens t, s = 0 .. Q-1, cs_t = A sum_{r<=t}
// delta_r (from the chunk start), L[t,s] = e^(cs_t - cs_s) for s <= t, else 0,
// G = C^T B (G[t,s] = C_t . B_s), h_0 the state entering the chunk, and dh_Q
// the gradient of the state leaving it:
//   forward   y~_t = sum_s L[t,s] G[t,s] delta_s x_s + e^cs_t C_t^T h_0
//             y_t  = (y~_t + D x_t) silu(z_t)
//             h_Q  = e^cs_Q h_0 + sum_s e^(cs_Q - cs_s) delta_s B_s x_s^T
//   backward  dout = dy silu(z),  dz = dy (y~ + D x) silu'(z)
//             u_s  = sum_t L[t,s] G[t,s] dout_t + e^(cs_Q - cs_s) B_s^T dh_Q   (P)
//             dx_s = delta_s u_s + D dout_s
//             dC_t = sum_s L[t,s] delta_s (dout_t . x_s) B_s + e^cs_t h_0 dout_t
//             dB_s = delta_s (sum_t L[t,s] (dout_t . x_s) C_t + e^(cs_Q - cs_s) dh_Q x_s)
//             dh_0 = e^cs_Q dh_Q + sum_t e^cs_t C_t dout_t^T
//             dcs_t = dout_t . y~_t - delta_t (x_t . u_t)  [+ <dh_Q, h_Q> for t = Q-1]
//             ddelta_s = x_s . u_s + A sum_{t>=s} dcs_t,   dA += sum_t dcs_t S_t
// (S_t = sum_{r<=t} delta_r), then d(dt) = ddelta sigmoid(dt + bias) under the
// softplus.  Every term is the chain rule of one factor of the forward form:
// the exponentials carry cs_t with a plus sign where t is the output token
// and a minus sign where it is the source token, which is what dcs collects.
//
// Two kernels, one CTA per (batch, head):
//   ssd_bwd_states_kernel (256 threads) runs the forward state recurrence
//     chunk by chunk and stores h at every chunk start (and the final state)
//     in scratch;
//   ssd_bwd_kernel (512 threads) walks the chunks backwards with dh in
//     accumulator fragments and evaluates the products above from shared
//     memory (32-token chunks keep every product's operands on chip).
// Every product runs on the tensor cores as warp-level m16n8k8 tiles with
// tf32 operands and fp32 accumulation.  In the products whose results feed
// the step-size gradients (differences of nearly equal sums) and in the two
// state recurrences, every operand that is not a bf16 input is split into two
// tf32 parts (one extra product each), which keeps about 21 bits of it; bf16
// inputs are exact in tf32.
// dB and dC sum over the heads of a group: each head adds its chunk terms
// with 16-byte atomics into one of kSbCopies partial copies ([t][n] rows),
// and ssd_bwd_reduce_bc sums the copies into (batch, G, N, L).  dA, dD and
// the bias gradient sum over batch rows: one atomic per CTA.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "f32x2.cuh"
#include "ptx.cuh"

namespace selscan {

constexpr int kSbN = 128;       // state size built
constexpr int kSbP = 64;        // head dimension built
constexpr int kSbQ = 32;        // tokens per chunk
constexpr int kSbThreads = 256;
constexpr int kSbCopies = 8;    // partial copies of dB / dC (head h adds into copy h % 8)

struct SsdBwdParams {
    int batch, H, L, nchunks, heads_per_group, G;
    const __nv_bfloat16 *x, *dy, *z;  // (batch, H*P, L), time stride 1
    int64_t x_bs, x_cs, dy_bs, dy_cs, z_bs, z_cs;
    const float *dt;                  // (batch, H, L), time stride 1
    int64_t dt_bs, dt_hs;
    const float *dt_bias;             // (H) or null
    int softplus;
    const float *A, *Dskip;           // (H); Dskip may be null
    const __nv_bfloat16 *B, *C;       // (batch, G, N, L), time stride 1
    int64_t B_bs, B_gs, B_ns, C_bs, C_gs, C_ns;
    const float *h0, *dlast;          // (batch, H, P, N) contiguous, or null
    __nv_bfloat16 *dx, *dz;           // like x; dz null without gate
    int64_t dx_bs, dx_cs, dz_bs, dz_cs;
    float *ddt;                       // (batch, H, L), time stride 1
    int64_t ddt_bs, ddt_hs;
    float *dA, *dD, *ddt_bias;        // (H), accumulated; dD / ddt_bias may be null
    float *dh0;                       // (batch, H, P, N) or null
    float *pB, *pC;                   // [kSbCopies][batch][G][L][N], zeroed
    float *states;                    // [batch*H][nchunks+1][256 threads][32] (sb_state_coord)
};

__device__ __forceinline__ float sb_bf(__nv_bfloat16 v) { return __bfloat162float(v); }

// Tokens t .. t + 7 (t .. t + 3) of a bf16 row as fp32, zero from token
// `valid` on: one 16-byte (8-byte) load when all of them are in the
// sequence (rows are 16-byte aligned and t a multiple of 8 (4)).
__device__ __forceinline__ void sb_ld8(const __nv_bfloat16 *src, int t, int valid,
                                       float (&v)[8])
{
    if (t + 8 <= valid) {
        unpack8_bf16(*reinterpret_cast<const uint4 *>(src), v);
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
            v[k] = t + k < valid ? sb_bf(src[k]) : 0.f;
    }
}

__device__ __forceinline__ void sb_ld4(const __nv_bfloat16 *src, int t, int valid,
                                       float (&v)[4])
{
    if (t + 4 <= valid) {
        const uint2 q = *reinterpret_cast<const uint2 *>(src);
        v[0] = __uint_as_float(q.x << 16);
        v[1] = __uint_as_float(q.x & 0xffff0000u);
        v[2] = __uint_as_float(q.y << 16);
        v[3] = __uint_as_float(q.y & 0xffff0000u);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            v[k] = t + k < valid ? sb_bf(src[k]) : 0.f;
    }
}

// Step sizes of a chunk (one warp, lane = token): delta, the raw argument
// (for the softplus derivative) and the prefix sum S (inclusive).
__device__ __forceinline__ void sb_steps(const SsdBwdParams &p, int b, int hh, int t0, int valid,
                                         int lane, float bias, float &raw, float &dl, float &S)
{
    raw = 0.f;
    dl = 0.f;
    if (lane < valid) {
        raw = p.dt[int64_t(b) * p.dt_bs + int64_t(hh) * p.dt_hs + t0 + lane] + bias;
        dl = p.softplus ? (raw > 20.f ? raw : log1pf(expf(raw))) : raw;
    }
    S = dl;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, S, o);
        if (lane >= o)
            S += v;
    }
}

// ---- warp-level tensor-core products (mma.sync m16n8k8, tf32 inputs, fp32
// accumulators).  Fragment coordinates, with g = lane / 4 and q = lane % 4:
// A (16 x 8): a0 (g, q), a1 (g + 8, q), a2 (g, q + 4), a3 (g + 8, q + 4);
// B (8 x 8):  b0 (q, g), b1 (q + 4, g);
// D (16 x 8): d0 (g, 2q), d1 (g, 2q + 1), d2 (g + 8, 2q), d3 (g + 8, 2q + 1).
// x rounded to tf32 (10 mantissa bits), to nearest with ties away from
// zero: add half a unit of the 13 dropped bits to the magnitude, then clear
// them (a carry into the exponent gives the next power of two, or infinity).
__device__ __forceinline__ uint32_t sb_tf32(float x)
{
    return (__float_as_uint(x) + 0x1000u) & 0xffffe000u;
}

__device__ __forceinline__ void sb_mma(float (&d)[4], const uint32_t (&a)[4],
                                       const uint32_t (&b)[2])
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// x = hi + lo with hi, lo both tf32 (hi the rounded value, lo the rounded rest).
__device__ __forceinline__ void sb_split(float x, uint32_t &hi, uint32_t &lo)
{
    hi = sb_tf32(x);
    lo = sb_tf32(x - __uint_as_float(hi));
}

// How an operand enters a product: kSbRound rounds it to tf32; kSbExact
// passes its bits as they are (values of bf16 inputs: x, B, C, ungated dy,
// which tf32 holds exactly); kSbSplit takes it as the sum of two tf32
// numbers, with one extra product (hi hi, then lo hi and / or hi lo), which
// keeps about 21 bits of it.
constexpr int kSbRound = 0, kSbExact = 1, kSbSplit = 2;

template <int MODE>
__device__ __forceinline__ void sb_operand(float x, uint32_t &hi, uint32_t &lo)
{
    if (MODE == kSbSplit)
        sb_split(x, hi, lo);
    else if (MODE == kSbExact)
        hi = __float_as_uint(x);
    else
        hi = sb_tf32(x);
}

// D[NT tiles] += sum_{k < K} A(m0 + row, k) B(k, n0 + 8 t + col): one A
// fragment per k step serves NT output tiles.  fa(m, k) and fb(k, n) read
// the operands from shared memory in whatever layout they are kept; MA / MB
// say how each enters the products (kSbRound / kSbExact / kSbSplit).
template <int K, int NT, int MA, int MB, typename FA, typename FB>
__device__ __forceinline__ void sb_gemm(float (&d)[NT][4], int m0, int n0, FA fa, FB fb,
                                        int lane)
{
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        const float av[4] = {fa(m0 + g, k0 + q), fa(m0 + g + 8, k0 + q), fa(m0 + g, k0 + q + 4),
                             fa(m0 + g + 8, k0 + q + 4)};
        uint32_t ah[4], al[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            sb_operand<MA>(av[i], ah[i], al[i]);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float bv[2] = {fb(k0 + q, n0 + 8 * t + g), fb(k0 + q + 4, n0 + 8 * t + g)};
            uint32_t bh[2], bl[2];
#pragma unroll
            for (int i = 0; i < 2; ++i)
                sb_operand<MB>(bv[i], bh[i], bl[i]);
            if (MA == kSbSplit)
                sb_mma(d[t], al, bh);
            if (MB == kSbSplit)
                sb_mma(d[t], ah, bl);
            sb_mma(d[t], ah, bh);
        }
    }
}

template <int NT>
__device__ __forceinline__ void sb_zero(float (&d)[NT][4])
{
#pragma unroll
    for (int t = 0; t < NT; ++t)
        d[t][0] = d[t][1] = d[t][2] = d[t][3] = 0.f;
}

// ------------------------------------------------------------ forward states
// Scratch layout of the stored states: per (batch, head) and chunk entry, 256
// threads x 32 floats, thread-contiguous.  Thread u = 32 w + l holds the
// accumulator fragments of rows 16 w .. 16 w + 15 (n) and all 64 columns (p)
// in eight 16 x 8 tiles: float 4 t + e is element e of tile t, at row
// n = 16 w + l / 4 + 8 (e / 2) and column p = 8 t + 2 (l % 4) + e % 2.
__device__ __forceinline__ void sb_state_coord(int u, int f, int &n, int &pp)
{
    const int w = u >> 5, l = u & 31, t = f >> 2, e = f & 3;
    n = 16 * w + (l >> 2) + 8 * (e >> 1);
    pp = 8 * t + 2 * (l & 3) + (e & 1);
}

__global__ void __launch_bounds__(kSbThreads, 1) ssd_bwd_states_kernel(const SsdBwdParams p)
{
    constexpr int Q = kSbQ, N = kSbN, P = kSbP;
    __shared__ __align__(16) float Bs[Q][N + 4];
    __shared__ __align__(16) float xs[Q][P + 4];
    __shared__ __align__(16) float ws[Q];
    __shared__ float s_decay;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = blockIdx.x, b = bh / p.H, hh = bh - b * p.H;
    const int g = hh / p.heads_per_group;
    const float A = p.A[hh];
    const float bias = p.dt_bias ? p.dt_bias[hh] : 0.f;

    float hs[8][4];
    {
        const float *h0 = p.h0 ? p.h0 + (int64_t(b) * p.H + hh) * P * N : nullptr;
#pragma unroll
        for (int f = 0; f < 32; ++f) {
            int n, pp;
            sb_state_coord(tid, f, n, pp);
            hs[f >> 2][f & 3] = h0 ? h0[int64_t(pp) * N + n] : 0.f;
        }
    }
    float4 *st = reinterpret_cast<float4 *>(p.states) +
                 (int64_t(bh) * (p.nchunks + 1) * kSbThreads + tid) * 8;
    const int64_t chunk_stride = int64_t(kSbThreads) * 8;  // float4 per chunk entry
    const __nv_bfloat16 *Brow = p.B + int64_t(b) * p.B_bs + int64_t(g) * p.B_gs;
    const __nv_bfloat16 *xrow = p.x + int64_t(b) * p.x_bs + int64_t(hh) * P * p.x_cs;

    // the next chunk's B and x values and raw step sizes are read into
    // registers while the current chunk's products run
    const int bn = tid >> 1, bhalf = tid & 1;  // B row n, tokens 16 bhalf .. + 15
    const int xp = tid >> 2, xq = tid & 3;     // x row p, tokens 8 xq .. + 7
    float bv[16], xv[8], dtv = 0.f;
    auto fetch = [&](int c) {
        const int t0 = c * Q, valid = min(Q, p.L - t0);
        const __nv_bfloat16 *bsrc = Brow + int64_t(bn) * p.B_ns + t0 + 16 * bhalf;
        float v8[8];
        sb_ld8(bsrc, 16 * bhalf, valid, v8);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            bv[k] = v8[k];
        sb_ld8(bsrc + 8, 16 * bhalf + 8, valid, v8);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            bv[8 + k] = v8[k];
        sb_ld8(xrow + int64_t(xp) * p.x_cs + t0 + 8 * xq, 8 * xq, valid, xv);
        dtv = (warp == 0 && lane < valid)
                  ? p.dt[int64_t(b) * p.dt_bs + int64_t(hh) * p.dt_hs + t0 + lane]
                  : 0.f;
    };
    if (p.nchunks > 0)
        fetch(0);
    for (int c = 0; c < p.nchunks; ++c) {
        float4 *sc = st + int64_t(c) * chunk_stride;
#pragma unroll
        for (int t = 0; t < 8; ++t)
            sc[t] = make_float4(hs[t][0], hs[t][1], hs[t][2], hs[t][3]);
        const int t0 = c * Q, valid = min(Q, p.L - t0);
#pragma unroll
        for (int k = 0; k < 16; ++k)
            Bs[16 * bhalf + k][bn] = bv[k];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            xs[8 * xq + k][xp] = xv[k];
        if (warp == 0) {
            // the same step sizes as sb_steps computes in the walk
            const float raw = lane < valid ? dtv + bias : 0.f;
            const float dl =
                lane < valid ? (p.softplus ? (raw > 20.f ? raw : log1pf(expf(raw))) : raw) : 0.f;
            float S = dl;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, S, o);
                if (lane >= o)
                    S += v;
            }
            const float SQ = __shfl_sync(0xffffffffu, S, 31);
            ws[lane] = expf(A * (SQ - S)) * dl;
            if (lane == 0)
                s_decay = expf(A * SQ);
        }
        __syncthreads();
        if (c + 1 < p.nchunks)
            fetch(c + 1);
        // h = e^cs_Q h + sum_s (w_s B_s) x_s^T on the tensor cores
        const float dec = s_decay;
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                hs[t][e] *= dec;
        sb_gemm<Q, 8, kSbSplit, kSbExact>(hs, 16 * warp, 0,
            [&](int m, int k) { return ws[k] * Bs[k][m]; },
                            [&](int k, int n) { return xs[k][n]; }, lane);
        __syncthreads();
    }
    float4 *sc = st + int64_t(p.nchunks) * chunk_stride;
#pragma unroll
    for (int t = 0; t < 8; ++t)
        sc[t] = make_float4(hs[t][0], hs[t][1], hs[t][2], hs[t][3]);
}

// ------------------------------------------------------------ chunk walk
// 512 threads (16 warps per SM to hide the shared-memory latency of the
// products).  Shared memory of the walk (fp32); rows are padded (68 / 132 /
// 36 floats) so that the column groups a warp reads at once fall in distinct
// banks and every row stays 16-byte aligned.
constexpr int kSbWalk = 512;
constexpr int kSbXS = kSbP + 4;   // x, dout, dy silu'(z): [t][p]
constexpr int kSbNS = kSbN + 4;   // B, C: [t][n]; h_0^T, dh^T: [p][n]
constexpr int kSbTS = kSbQ + 4;   // x^T, dout^T: [p][t]; the Q x Q matrices
struct SbSmem {
    float xs[kSbQ][kSbXS], dos[kSbQ][kSbXS], zf[kSbQ][kSbXS];
    float xsT[kSbP][kSbTS], dosT[kSbP][kSbTS];
    float Bs[kSbQ][kSbNS], Cs[kSbQ][kSbNS];
    float h0T[kSbP][kSbNS], dhT[kSbP][kSbNS];
    // L.G.delta_s [t][s], (L.G)^T [s][t], L.delta_s.(dout x^T) [t][s], (L.(dout x^T))^T [s][t]
    float Md[kSbQ][kSbTS], MmT[kSbQ][kSbTS], Wm[kSbQ][kSbTS], VmT[kSbQ][kSbTS];
    float raw[kSbQ], dl[kSbQ], S[kSbQ], ecs[kSbQ], ecq[kSbQ], ddd[kSbQ], dyy[kSbQ];
    float red[kSbWalk / 32];
    float hqdh, ecQ;
};

// Block sum of one value per thread (every thread gets the total).
__device__ __forceinline__ float sb_block_sum(float v, float *red, int tid)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();  // red is free
    if ((tid & 31) == 0)
        red[tid >> 5] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kSbWalk / 32; ++w)
        t += red[w];
    return t;
}

// Sum over the 16 consecutive lanes that share a row (lanes 16r .. 16r + 15).
__device__ __forceinline__ float sb_sum16(float v)
{
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    return v;
}

__device__ __forceinline__ float sb_dot4(float4 a, float4 b, float acc)
{
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
}

template <typename T>
__device__ __forceinline__ float4 sb_ld4(const T &ref)
{
    return *reinterpret_cast<const float4 *>(&ref);
}

template <bool GATE>
__global__ void __launch_bounds__(kSbWalk, 1) ssd_bwd_kernel(const SsdBwdParams p)
{
    constexpr int Q = kSbQ, N = kSbN, P = kSbP;
    extern __shared__ __align__(16) uint8_t sb_raw[];
    SbSmem &sm = *reinterpret_cast<SbSmem *>(sb_raw);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, q4 = lane & 3;  // fragment row / column of this lane
    const int bh = blockIdx.x, b = bh / p.H, hh = bh - b * p.H;
    const int g = hh / p.heads_per_group;
    const float A = p.A[hh];
    const float bias = p.dt_bias ? p.dt_bias[hh] : 0.f;
    const float dsk = p.Dskip ? p.Dskip[hh] : 0.f;

    // dh (N x P) in accumulator fragments: warp w holds rows 16 (w / 2) .. + 15,
    // columns 32 (w % 2) .. + 31 (four 16 x 8 tiles)
    const int dm0 = 16 * (warp >> 1), dn0 = 32 * (warp & 1);
    float dh[4][4];
    {
        const float *dl0 = p.dlast ? p.dlast + (int64_t(b) * p.H + hh) * P * N : nullptr;
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int n = dm0 + g8 + 8 * (e >> 1), pp = dn0 + 8 * t + 2 * q4 + (e & 1);
                dh[t][e] = dl0 ? dl0[int64_t(pp) * N + n] : 0.f;
            }
    }
    const float4 *st_base = reinterpret_cast<const float4 *>(p.states) +
                            int64_t(bh) * (p.nchunks + 1) * kSbThreads * 8;
    const int64_t chunk_stride = int64_t(kSbThreads) * 8;
    // <dlast, final state> for the last chunk: states-kernel layout, read by
    // thread halves (u = tid / 2 owns rows 4 (u % 32) + i, columns 8 (u / 32) + j)
    float hq_next = 0.f;
    if (p.dlast) {
        const int u = tid >> 1, ih = tid & 1;  // floats 16 ih .. 16 ih + 15 of thread u
        const float4 *sf = st_base + int64_t(p.nchunks) * chunk_stride + u * 8 + 4 * ih;
        const float *dl0 = p.dlast + (int64_t(b) * p.H + hh) * P * N;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const float4 a = sf[v];
            const float hv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                int n, pp;
                sb_state_coord(u, 16 * ih + 4 * v + e, n, pp);
                hq_next = fmaf(dl0[int64_t(pp) * N + n], hv[e], hq_next);
            }
        }
    }
    hq_next = sb_block_sum(hq_next, sm.red, tid);
    const __nv_bfloat16 *Brow = p.B + int64_t(b) * p.B_bs + int64_t(g) * p.B_gs;
    const __nv_bfloat16 *Crow = p.C + int64_t(b) * p.C_bs + int64_t(g) * p.C_gs;
    const __nv_bfloat16 *xrow = p.x + int64_t(b) * p.x_bs + int64_t(hh) * P * p.x_cs;
    const __nv_bfloat16 *dyrow = p.dy + int64_t(b) * p.dy_bs + int64_t(hh) * P * p.dy_cs;
    const __nv_bfloat16 *zrow =
        GATE ? p.z + int64_t(b) * p.z_bs + int64_t(hh) * P * p.z_cs : nullptr;
    float *pB = p.pB + ((int64_t(hh % kSbCopies) * p.batch + b) * p.G + g) * int64_t(p.L) * N;
    float *pC = p.pC + ((int64_t(hh % kSbCopies) * p.batch + b) * p.G + g) * int64_t(p.L) * N;
    float accD = 0.f, accA = 0.f, accBias = 0.f;

    for (int c = p.nchunks - 1; c >= 0; --c) {
        const int t0 = c * Q, valid = min(Q, p.L - t0);
        // ---- 1. chunk inputs (and transposed copies), h_0^T, dh_Q^T, step sizes
        {
            const int pp = tid >> 3, q = tid & 7;  // row p, tokens 4q .. 4q + 3
            const int64_t xo = int64_t(pp) * p.x_cs + t0 + 4 * q;
            const int64_t yo = int64_t(pp) * p.dy_cs + t0 + 4 * q;
            const int64_t zo = GATE ? int64_t(pp) * p.z_cs + t0 + 4 * q : 0;
            float xv4[4], dv4[4], xl[4], yl[4], zl[4];
            sb_ld4(xrow + xo, 4 * q, valid, xl);
            sb_ld4(dyrow + yo, 4 * q, valid, yl);
            if (GATE)
                sb_ld4(zrow + zo, 4 * q, valid, zl);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int t = 4 * q + k;
                const float xv = xl[k];
                const float dyv = yl[k];
                float dout = dyv, zfac = 0.f;
                if (GATE) {
                    const float zv = zl[k];
                    const float sg = 1.f / (1.f + expf(-zv));
                    dout = dyv * zv * sg;
                    zfac = dyv * (sg * (1.f + zv * (1.f - sg)));
                }
                sm.xs[t][pp] = xv;
                sm.dos[t][pp] = dout;
                if (GATE)
                    sm.zf[t][pp] = zfac;
                xv4[k] = xv;
                dv4[k] = dout;
            }
            *reinterpret_cast<float4 *>(&sm.xsT[pp][4 * q]) =
                make_float4(xv4[0], xv4[1], xv4[2], xv4[3]);
            *reinterpret_cast<float4 *>(&sm.dosT[pp][4 * q]) =
                make_float4(dv4[0], dv4[1], dv4[2], dv4[3]);
        }
        {
            const int n = tid >> 2, q = tid & 3;  // row n, tokens 8q .. 8q + 7
            float bv[8], cv[8];
            sb_ld8(Brow + int64_t(n) * p.B_ns + t0 + 8 * q, 8 * q, valid, bv);
            sb_ld8(Crow + int64_t(n) * p.C_ns + t0 + 8 * q, 8 * q, valid, cv);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                sm.Bs[8 * q + k][n] = bv[k];
                sm.Cs[8 * q + k][n] = cv[k];
            }
        }
        {
            const int u = tid >> 1, ih = tid & 1;  // floats 16 ih .. 16 ih + 15 of thread u
            const float4 *s0 = st_base + int64_t(c) * chunk_stride + u * 8 + 4 * ih;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 a = s0[v];
                const float hv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    int n, pp;
                    sb_state_coord(u, 16 * ih + 4 * v + e, n, pp);
                    sm.h0T[pp][n] = hv[e];
                }
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                sm.dhT[dn0 + 8 * t + 2 * q4 + (e & 1)][dm0 + g8 + 8 * (e >> 1)] = dh[t][e];
        if (warp == 0) {
            float rw, dl, S;
            sb_steps(p, b, hh, t0, valid, lane, bias, rw, dl, S);
            const float SQ = __shfl_sync(0xffffffffu, S, 31);
            sm.raw[lane] = rw;
            sm.dl[lane] = dl;
            sm.S[lane] = S;
            sm.ecs[lane] = expf(A * S);
            sm.ecq[lane] = expf(A * (SQ - S));
            sm.ddd[lane] = 0.f;
            sm.dyy[lane] = 0.f;
            if (lane == 0)
                sm.ecQ = expf(A * SQ);
        }
        __syncthreads();

        // ---- 2. Q x Q matrices: warps 0-7 G = C B^T, warps 8-15 dout x^T;
        //         one 16 x 8 tile each, then the mask and the step sizes
        {
            const int w8 = warp & 7, m0 = 16 * (w8 >> 2), n0 = 8 * (w8 & 3);
            float acc[1][4];
            sb_zero(acc);
            if (warp < 8)
                sb_gemm<N, 1, kSbExact, kSbExact>(acc, m0, n0,
                    [&](int m, int k) { return sm.Cs[m][k]; },
                              [&](int k, int n) { return sm.Bs[n][k]; }, lane);
            else
                sb_gemm<P, 1, (GATE ? kSbSplit : kSbExact), kSbExact>(acc, m0, n0,
                    [&](int m, int k) { return sm.dos[m][k]; },
                              [&](int k, int n) { return sm.xs[n][k]; }, lane);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = m0 + g8 + 8 * (e >> 1), s_ = n0 + 2 * q4 + (e & 1);
                const float Lts = s_ <= t ? expf(A * (sm.S[t] - sm.S[s_])) : 0.f;
                const float v = acc[0][e] * Lts, ds = sm.dl[s_];
                if (warp < 8) {
                    sm.Md[t][s_] = v * ds;
                    sm.MmT[s_][t] = v;
                } else {
                    sm.Wm[t][s_] = v * ds;
                    sm.VmT[s_][t] = v;
                }
            }
        }
        __syncthreads();

        // ---- 3a. y~ (rows t, warps 0-7) and u (rows s, warps 8-15), 32 x 64
        //          each; warp w holds rows 16 ((w / 4) % 2), columns 16 (w % 4) .. + 15
        {
            const bool isy = warp < 8;
            const int m0 = 16 * ((warp >> 2) & 1), n0 = 16 * (warp & 3);
            float v1[2][4], v2[2][4];
            sb_zero(v1);
            sb_zero(v2);
            if (isy) {
                sb_gemm<Q, 2, kSbSplit, kSbExact>(v1, m0, n0,
                    [&](int m, int k) { return sm.Md[m][k]; },
                                    [&](int k, int n) { return sm.xsT[n][k]; }, lane);
                sb_gemm<N, 2, kSbExact, kSbSplit>(v2, m0, n0,
                    [&](int m, int k) { return sm.Cs[m][k]; },
                                    [&](int k, int n) { return sm.h0T[n][k]; }, lane);
            } else {
                sb_gemm<Q, 2, kSbSplit, (GATE ? kSbSplit : kSbExact)>(v1, m0, n0,
                    [&](int m, int k) { return sm.MmT[m][k]; },
                                    [&](int k, int n) { return sm.dosT[n][k]; }, lane);
                sb_gemm<N, 2, kSbExact, kSbSplit>(v2, m0, n0,
                    [&](int m, int k) { return sm.Bs[m][k]; },
                                    [&](int k, int n) { return sm.dhT[n][k]; }, lane);
            }
            float rs[2] = {0.f, 0.f};  // x.u (u warps) or dout.y~ (y~ warps) per row
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int hr = e >> 1, r = m0 + g8 + 8 * hr;
                    const int pp = n0 + 8 * t + 2 * q4 + (e & 1);
                    const float xv = sm.xs[r][pp], dv = sm.dos[r][pp];
                    const int64_t col = int64_t(hh * P + pp);
                    if (isy) {
                        const float yt = fmaf(sm.ecs[r], v2[t][e], v1[t][e]);
                        rs[hr] = fmaf(dv, yt, rs[hr]);
                        accD = fmaf(dv, xv, accD);
                        if (GATE && r < valid)
                            p.dz[int64_t(b) * p.dz_bs + col * p.dz_cs + t0 + r] =
                                __float2bfloat16_rn(sm.zf[r][pp] * fmaf(dsk, xv, yt));
                    } else {
                        const float uu = fmaf(sm.ecq[r], v2[t][e], v1[t][e]);
                        rs[hr] = fmaf(xv, uu, rs[hr]);
                        if (r < valid)
                            p.dx[int64_t(b) * p.dx_bs + col * p.dx_cs + t0 + r] =
                                __float2bfloat16_rn(fmaf(sm.dl[r], uu, dsk * dv));
                    }
                }
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                rs[hr] += __shfl_xor_sync(0xffffffffu, rs[hr], 1);
                rs[hr] += __shfl_xor_sync(0xffffffffu, rs[hr], 2);
                if (q4 == 0)
                    atomicAdd(isy ? &sm.dyy[m0 + g8 + 8 * hr] : &sm.ddd[m0 + g8 + 8 * hr],
                              rs[hr]);
            }
        }
        // ---- 3b. dC (warps 0-7) and dB (warps 8-15): 32 x 128 each; warp
        //          holds rows 16 ((w / 4) % 2), columns 32 (w % 4) .. + 31
        {
            const int m0 = 16 * ((warp >> 2) & 1), n0 = 32 * (warp & 3);
            float a1[4][4], a2[4][4];
            sb_zero(a1);
            sb_zero(a2);
            if (warp < 8) {
                sb_gemm<Q, 4, kSbRound, kSbExact>(a1, m0, n0,
                    [&](int m, int k) { return sm.Wm[m][k]; },
                              [&](int k, int n) { return sm.Bs[k][n]; }, lane);
                sb_gemm<P, 4, (GATE ? kSbRound : kSbExact), kSbRound>(a2, m0, n0,
                    [&](int m, int k) { return sm.dos[m][k]; },
                              [&](int k, int n) { return sm.h0T[k][n]; }, lane);
            } else {
                sb_gemm<Q, 4, kSbRound, kSbExact>(a1, m0, n0,
                    [&](int m, int k) { return sm.VmT[m][k]; },
                              [&](int k, int n) { return sm.Cs[k][n]; }, lane);
                sb_gemm<P, 4, kSbExact, kSbRound>(a2, m0, n0,
                    [&](int m, int k) { return sm.xs[m][k]; },
                              [&](int k, int n) { return sm.dhT[k][n]; }, lane);
            }
            float *dst = warp < 8 ? pC : pB;
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = m0 + g8 + 8 * hr;
                if (r < valid) {
                    const float sc = warp < 8 ? sm.ecs[r] : sm.ecq[r];
                    const float pre = warp < 8 ? 1.f : sm.dl[r];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int n = n0 + 8 * t + 2 * q4;
                        const float2 v = make_float2(
                            pre * fmaf(sc, a2[t][2 * hr], a1[t][2 * hr]),
                            pre * fmaf(sc, a2[t][2 * hr + 1], a1[t][2 * hr + 1]));
                        atomicAdd(reinterpret_cast<float2 *>(dst + int64_t(t0 + r) * N + n), v);
                    }
                }
            }
        }
        // ---- 3c. dh_0 = e^cs_Q dh_Q + C^T (e^cs dout): rows n, columns p
        {
            const float eQ = sm.ecQ;
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dh[t][e] *= eQ;
            sb_gemm<Q, 4, kSbExact, kSbSplit>(dh, dm0, dn0,
                [&](int m, int k) { return sm.Cs[k][m]; },
                          [&](int k, int n) { return sm.ecs[k] * sm.dos[k][n]; }, lane);
        }
        // <dh_0, h_0> of this chunk: the <dh_Q, h_Q> term of the next one
        float hq = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                hq = fmaf(dh[t][e],
                          sm.h0T[dn0 + 8 * t + 2 * q4 + (e & 1)][dm0 + g8 + 8 * (e >> 1)], hq);
        const float hq_this = hq_next;
        hq_next = sb_block_sum(hq, sm.red, tid);  // (its barriers also order 3a-3c before 4)
        // ---- 4. per-token scalars (one warp, lane = token)
        if (warp == 0) {
            const bool in = lane < valid;
            const float ds = sm.dl[lane];
            float dcs = sm.dyy[lane] - ds * sm.ddd[lane];
            if (lane == valid - 1)
                dcs += hq_this;
            if (!in)
                dcs = 0.f;
            float R = dcs;  // sum over t >= lane
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float v = __shfl_down_sync(0xffffffffu, R, off);
                if (lane + off < 32)
                    R += v;
            }
            const float dd = sm.ddd[lane] + A * R;
            const float rw = sm.raw[lane];
            const float ddt = p.softplus ? dd / (1.f + expf(-rw)) : dd;
            if (in)
                p.ddt[int64_t(b) * p.ddt_bs + int64_t(hh) * p.ddt_hs + t0 + lane] = ddt;
            accA = fmaf(dcs, sm.S[lane], accA);
            accBias += in ? ddt : 0.f;
        }
        __syncthreads();
    }

    // ---- per-head sums (over this batch row), dh0
    if (p.dh0) {
        float *d0 = p.dh0 + (int64_t(b) * p.H + hh) * P * N;
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                d0[int64_t(dn0 + 8 * t + 2 * q4 + (e & 1)) * N + dm0 + g8 + 8 * (e >> 1)] =
                    dh[t][e];
    }
    const float sD = sb_block_sum(accD, sm.red, tid);
    const float sA = sb_block_sum(accA, sm.red, tid);
    const float sBias = sb_block_sum(accBias, sm.red, tid);
    if (tid == 0) {
        atomicAdd(p.dA + hh, sA);
        if (p.dD)
            atomicAdd(p.dD + hh, sD);
        if (p.ddt_bias)
            atomicAdd(p.ddt_bias + hh, sBias);
    }
}

// dB, dC (batch, G, N, L) = sum of the kSbCopies partial copies, each
// [batch][G][L][N].  A block transposes 32 tokens x 128 states through
// shared memory so that both the reads and the writes are row-contiguous.
__global__ void __launch_bounds__(256) ssd_bwd_reduce_bc(const float *pB, const float *pC,
                                                         float *dB, float *dC, int64_t rows,
                                                         int L)
{
    __shared__ float tile[2][32][kSbN + 1];
    const int64_t bg = blockIdx.y;             // (batch, group) row
    const int t0 = blockIdx.x * 32;
    const int64_t copy = rows * int64_t(L) * kSbN;  // floats per partial copy
    const int tid = threadIdx.x;
    for (int e = tid; e < 32 * kSbN; e += 256) {
        const int t = e / kSbN, n = e - t * kSbN;
        float sb = 0.f, sc = 0.f;
        if (t0 + t < L) {
            const int64_t off = (bg * L + t0 + t) * kSbN + n;
            for (int k = 0; k < kSbCopies; ++k) {
                sb += pB[k * copy + off];
                sc += pC[k * copy + off];
            }
        }
        tile[0][t][n] = sb;
        tile[1][t][n] = sc;
    }
    __syncthreads();
    for (int e = tid; e < 32 * kSbN; e += 256) {
        const int n = e / 32, t = e - n * 32;
        if (t0 + t < L) {
            const int64_t off = (bg * kSbN + n) * L + t0 + t;
            dB[off] = tile[0][t][n];
            dC[off] = tile[1][t][n];
        }
    }
}

}  // namespace selscan
