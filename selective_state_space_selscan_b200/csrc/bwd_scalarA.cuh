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
// tf32 operands and fp32 accumulation, read from shared-memory tiles laid out
// so that no fragment load meets a bank conflict (sb_off).  In the products
// whose results feed the step-size gradients (differences of nearly equal
// sums) and in the two state recurrences, every operand that is not a bf16
// input is split into two parts (one extra product each), which keeps about
// 20 bits of it; bf16 inputs are exact in tf32.
// dB and dC sum over the heads of a group: each head adds its chunk terms
// with 8-byte atomics into a token-major accumulation buffer ([t][n] rows),
// and ssd_bwd_reduce_bc transposes it into (batch, G, N, L).  dA, dD and
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
// Accumulation copies of dB / dC (head h adds into copy h % kSbCopies).  One
// copy measured fastest on B4 H32 G1 L4096 (1.493 ms; 2, 4, 8, 16 copies:
// 1.499, 1.506, 1.529, 1.607 ms): zeroing and summing more copies costs more
// than the contention of 32 heads' atomics on one.
constexpr int kSbCopies = 1;

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
    float *states;                    // [batch*H][nchunks+1][P][N]: h^T at every chunk start
};

// Tokens t .. t + 7 (t .. t + 3) of a bf16 row as raw bits, two tokens per
// word in token order, zero from token `valid` on: one 16-byte (8-byte) load
// when all of them are in the sequence (rows are 16-byte aligned and t a
// multiple of 8 (4)).
__device__ __forceinline__ uint4 sb_raw8(const __nv_bfloat16 *src, int t, int valid)
{
    if (t + 8 <= valid)
        return *reinterpret_cast<const uint4 *>(src);
    const unsigned short *s = reinterpret_cast<const unsigned short *>(src);
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t lo = t + 2 * k < valid ? s[2 * k] : 0u;
        const uint32_t hi = t + 2 * k + 1 < valid ? s[2 * k + 1] : 0u;
        w[k] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint2 sb_raw4(const __nv_bfloat16 *src, int t, int valid)
{
    if (t + 4 <= valid)
        return *reinterpret_cast<const uint2 *>(src);
    const unsigned short *s = reinterpret_cast<const unsigned short *>(src);
    uint32_t w[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint32_t lo = t + 2 * k < valid ? s[2 * k] : 0u;
        const uint32_t hi = t + 2 * k + 1 < valid ? s[2 * k + 1] : 0u;
        w[k] = lo | (hi << 16);
    }
    return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ void sb_unpack4(uint2 v, float (&f)[4])
{
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
}

// f[i] = token i ^ r of the eight packed in v (r = 0 .. 3): bit 0 of r swaps
// the two tokens of every word, bit 1 swaps neighbouring words.
__device__ __forceinline__ void sb_unpack8_xor(uint4 v, int r, float (&f)[8])
{
    const uint32_t sel = (r & 1) ? 0x1032u : 0x3210u;
    uint32_t w[4] = {__byte_perm(v.x, 0u, sel), __byte_perm(v.y, 0u, sel),
                     __byte_perm(v.z, 0u, sel), __byte_perm(v.w, 0u, sel)};
    if (r & 2) {
        const uint32_t a = w[0], c = w[2];
        w[0] = w[1];
        w[1] = a;
        w[2] = w[3];
        w[3] = c;
    }
    unpack8_bf16(make_uint4(w[0], w[1], w[2], w[3]), f);
}

// o[i] = v[i ^ r] (r = 0 .. 3)
__device__ __forceinline__ void sb_xor4(const float (&v)[4], int r, float (&o)[4])
{
    const bool b0 = r & 1, b1 = r & 2;
    const float a0 = b1 ? v[2] : v[0], a1 = b1 ? v[3] : v[1];
    const float a2 = b1 ? v[0] : v[2], a3 = b1 ? v[1] : v[3];
    o[0] = b0 ? a1 : a0;
    o[1] = b0 ? a0 : a1;
    o[2] = b0 ? a3 : a2;
    o[3] = b0 ? a2 : a3;
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

// ---- shared-memory tiles.  A tile of rows of R floats (R = 32, 64 or 128)
// has row stride R + 8 and keeps element (r, c) at r (R + 8) + (c ^ (r & 4)):
// bit 2 of the column flips with bit 2 of the row.  With m16n8k8 fragments
// two read patterns occur: rows 8 apart by lane / 4 and columns by lane % 4
// (an operand whose summed index runs along the row), and rows by lane % 4
// and columns by lane / 4 (summed index down the column).  The stride of 8
// mod 32 words spreads the first over all 32 banks; the flip keeps the
// second, whose rows 0-3 and 4-7 would otherwise share banks, conflict-free
// as well.  Column blocks of 4 stay contiguous and 16-byte aligned.
constexpr int kSbSX = kSbP + 8;   // rows of P floats
constexpr int kSbSN = kSbN + 8;   // rows of N floats
constexpr int kSbST = kSbQ + 8;   // rows of Q floats

__device__ __forceinline__ int sb_off(int S, int r, int c) { return r * S + (c ^ (r & 4)); }

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

// x = hi + lo: hi is x with its 13 low mantissa bits cleared (a tf32
// value), lo = x - hi exactly (an fp32 value below 2^-10 of |x|).  A tf32
// product reads only the top 19 bits of each operand, so lo enters it
// truncated to tf32, which leaves an error below 2^-20 |x|.
__device__ __forceinline__ void sb_split(float x, uint32_t &hi, uint32_t &lo)
{
    hi = __float_as_uint(x) & 0xffffe000u;
    lo = __float_as_uint(x - __uint_as_float(hi));
}

// How an operand enters a product: kSbRound rounds it to tf32; kSbExact
// passes its bits as they are (values of bf16 inputs: x, B, C, ungated dy,
// which tf32 holds exactly); kSbSplit takes it as the sum of two parts
// (sb_split), with one extra product (hi hi, then lo hi and / or hi lo),
// which keeps about 20 bits of it.
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

// Where an operand lives: kSbAlong, the summed index k runs along the tile's
// rows (A(m, k) at tile (m, k); B(k, n) at tile (n, k)); kSbDown, it runs
// down the columns (A(m, k) at tile (k, m); B(k, n) at tile (k, n)).
constexpr int kSbAlong = 0, kSbDown = 1;

// Offset of the element (i, k) of an operand (i = m for A, n for B) for the
// lanes' i = i0 + lane / 4 and k = lane % 4 + 4 h (h = 0, 1), relative to
// the k-step k0 and the tile i0 (i0 and k0 multiples of 8).
template <int O, int S>
__device__ __forceinline__ int sb_lane_off(int i0, int g, int q, int h)
{
    return O == kSbAlong ? (i0 + g) * S + ((q + 4 * h) ^ (g & 4))
                         : (q + 4 * h) * S + i0 + (g ^ (4 * h));
}

// Step between k-steps (8 k) and between row blocks 8 apart in i.
template <int O, int S> struct SbStep {
    static constexpr int k8 = O == kSbAlong ? 8 : 8 * S;
    static constexpr int i8 = O == kSbAlong ? 8 * S : 8;
};

// D[MT row blocks][NT tiles] += sum_{k < K} A(m0 + 16 mt + row, k)
// B(k, n0 + 8 t + col): per k step the B fragments of the NT tiles are read
// (and split) once and serve all MT row blocks, and each A fragment serves
// the NT tiles.  A and B are tiles in the sb_off layout with row strides SA,
// SB and orientations OA, OB; as / bs, when not null, scale A(., k) and
// B(k, .) by as[k], bs[k]; MA / MB say how each operand enters the products
// (kSbRound / kSbExact / kSbSplit).
template <int K, int MT, int NT, int MA, int OA, int SA, int MB, int OB, int SB>
__device__ __forceinline__ void sb_gemm_mt(float (&d)[MT][NT][4], int m0, int n0, const float *a,
                                           const float *as, const float *b, const float *bs,
                                           int lane)
{
    const int g = lane >> 2, q = lane & 3;
    const int ao0 = sb_lane_off<OA, SA>(m0, g, q, 0), ao1 = sb_lane_off<OA, SA>(m0, g, q, 1);
    const int bo0 = sb_lane_off<OB, SB>(n0, g, q, 0), bo1 = sb_lane_off<OB, SB>(n0, g, q, 1);
    constexpr int AK = SbStep<OA, SA>::k8, AI = SbStep<OA, SA>::i8;
    constexpr int BK = SbStep<OB, SB>::k8, BI = SbStep<OB, SB>::i8;
#pragma unroll
    for (int ks = 0; ks < K / 8; ++ks) {
        uint32_t bh[NT][2], bl[NT][2];
        {
            float s0 = 1.f, s1 = 1.f;
            if (bs) {
                s0 = bs[8 * ks + q];
                s1 = bs[8 * ks + q + 4];
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                float bv[2] = {b[bo0 + ks * BK + t * BI], b[bo1 + ks * BK + t * BI]};
                if (bs) {
                    bv[0] *= s0;
                    bv[1] *= s1;
                }
#pragma unroll
                for (int i = 0; i < 2; ++i)
                    sb_operand<MB>(bv[i], bh[t][i], bl[t][i]);
            }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int ro = 2 * mt * AI + ks * AK;
            float av[4] = {a[ao0 + ro], a[ao0 + ro + AI], a[ao1 + ro], a[ao1 + ro + AI]};
            if (as) {
                const float s0 = as[8 * ks + q], s1 = as[8 * ks + q + 4];
                av[0] *= s0;
                av[1] *= s0;
                av[2] *= s1;
                av[3] *= s1;
            }
            uint32_t ah[4], al[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                sb_operand<MA>(av[i], ah[i], al[i]);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (MA == kSbSplit)
                    sb_mma(d[mt][t], al, bh[t]);
                if (MB == kSbSplit)
                    sb_mma(d[mt][t], ah, bl[t]);
                sb_mma(d[mt][t], ah, bh[t]);
            }
        }
    }
}

// One row block (MT = 1).
template <int K, int NT, int MA, int OA, int SA, int MB, int OB, int SB>
__device__ __forceinline__ void sb_gemm(float (&d)[NT][4], int m0, int n0, const float *a,
                                        const float *as, const float *b, const float *bs,
                                        int lane)
{
    sb_gemm_mt<K, 1, NT, MA, OA, SA, MB, OB, SB>(reinterpret_cast<float(&)[1][NT][4]>(d), m0,
                                                 n0, a, as, b, bs, lane);
}

template <int NT>
__device__ __forceinline__ void sb_zero(float (&d)[NT][4])
{
#pragma unroll
    for (int t = 0; t < NT; ++t)
        d[t][0] = d[t][1] = d[t][2] = d[t][3] = 0.f;
}

template <int MT, int NT>
__device__ __forceinline__ void sb_zero(float (&d)[MT][NT][4])
{
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
        sb_zero(d[mt]);
}

// ------------------------------------------------------------ forward states
// The states are kept transposed, h^T (P x N), as accumulator fragments:
// warp w holds all 64 rows p and columns n = 16 w .. + 15 (four row blocks of
// two 16 x 8 tiles), so that each split operand (w_s B_s) is split by one warp.  Each chunk entry of the scratch is h^T at the chunk
// start, row-major [p][n], so the walk reads it back with contiguous loads.
//
// Loads of a chunk (shared by both kernels): B, C rows n as 8 tokens per
// thread (thread (n, qq), tokens 8 qq .. + 7) and x, dy, z rows p as 4 tokens
// per thread (thread (p, q), tokens 4 q .. + 3).  A warp stores them to the
// token-major tiles one token per thread per instruction; each thread takes
// its tokens in an order rotated by its lane (token 8 qq + (i ^ qq), resp.
// 4 q + (i ^ ((q / 2) % 4)), at store i), which puts the 32 stores of an
// instruction in 32 different banks.
__global__ void __launch_bounds__(kSbThreads, 1) ssd_bwd_states_kernel(const SsdBwdParams p)
{
    constexpr int Q = kSbQ, N = kSbN, P = kSbP;
    __shared__ __align__(16) float Bs[Q * kSbSN];
    __shared__ __align__(16) float xs[Q * kSbSX];
    __shared__ __align__(16) float ws[Q];
    __shared__ float s_decay;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g8 = lane >> 2, q4 = lane & 3;
    const int bh = blockIdx.x, b = bh / p.H, hh = bh - b * p.H;
    const int g = hh / p.heads_per_group;
    const float A = p.A[hh];
    const float bias = p.dt_bias ? p.dt_bias[hh] : 0.f;
    const int n0 = 16 * warp;

    float hs[4][2][4];
    {
        const float *h0 = p.h0 ? p.h0 + (int64_t(b) * p.H + hh) * P * N : nullptr;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int pp = 16 * mt + g8 + 8 * (e >> 1), n = n0 + 8 * t + 2 * q4 + (e & 1);
                    hs[mt][t][e] = h0 ? h0[pp * N + n] : 0.f;
                }
    }
    // h^T fragments to a [p][n] entry of the scratch
    auto store_state = [&](float *sc) {
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr)
                    *reinterpret_cast<float2 *>(sc + (16 * mt + g8 + 8 * hr) * N + n0 + 8 * t +
                                                2 * q4) =
                        make_float2(hs[mt][t][2 * hr], hs[mt][t][2 * hr + 1]);
    };
    float *st = p.states + int64_t(bh) * (p.nchunks + 1) * P * N;
    const __nv_bfloat16 *Brow = p.B + int64_t(b) * p.B_bs + int64_t(g) * p.B_gs;
    const __nv_bfloat16 *xrow = p.x + int64_t(b) * p.x_bs + int64_t(hh) * P * p.x_cs;

    // the next chunk's B and x values and raw step sizes are read into
    // registers while the current chunk's products run (two rows per thread)
    const int bn = tid >> 2, bq = tid & 3;  // B rows bn, bn + 64, tokens 8 bq .. + 7
    const int xp = tid >> 3, xq = tid & 7;  // x rows xp, xp + 32, tokens 4 xq .. + 3
    const int xr = (xq >> 1) & 3;
    uint4 bv[2];
    uint2 xv[2];
    float dtv = 0.f;
    auto fetch = [&](int c) {
        const int t0 = c * Q, valid = min(Q, p.L - t0);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            bv[j] = sb_raw8(Brow + int64_t(bn + 64 * j) * p.B_ns + t0 + 8 * bq, 8 * bq, valid);
            xv[j] = sb_raw4(xrow + int64_t(xp + 32 * j) * p.x_cs + t0 + 4 * xq, 4 * xq, valid);
        }
        dtv = (warp == 0 && lane < valid)
                  ? p.dt[int64_t(b) * p.dt_bs + int64_t(hh) * p.dt_hs + t0 + lane]
                  : 0.f;
    };
    if (p.nchunks > 0)
        fetch(0);
    for (int c = 0; c < p.nchunks; ++c) {
        store_state(st + int64_t(c) * P * N);
        const int t0 = c * Q, valid = min(Q, p.L - t0);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float f[8];
            sb_unpack8_xor(bv[j], bq, f);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                Bs[sb_off(kSbSN, 8 * bq + (i ^ bq), bn + 64 * j)] = f[i];
            float v[4], o[4];
            sb_unpack4(xv[j], v);
            sb_xor4(v, xr, o);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                xs[sb_off(kSbSX, 4 * xq + (i ^ xr), xp + 32 * j)] = o[i];
        }
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
        // h^T = e^cs_Q h^T + sum_s x_s (w_s B_s)^T on the tensor cores
        const float dec = s_decay;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    hs[mt][t][e] *= dec;
        sb_gemm_mt<Q, 4, 2, kSbExact, kSbDown, kSbSX, kSbSplit, kSbDown, kSbSN>(
            hs, 0, n0, xs, nullptr, Bs, ws, lane);
        __syncthreads();
    }
    store_state(st + int64_t(p.nchunks) * P * N);
}

// ------------------------------------------------------------ chunk walk
// 512 threads (16 warps per SM to hide the shared-memory latency of the
// products).  Shared memory of the walk (fp32), every tile in the sb_off
// layout.
constexpr int kSbWalk = 512;
struct SbSmem {
    float xs[kSbQ * kSbSX], dos[kSbQ * kSbSX], zf[kSbQ * kSbSX];  // x, dout, dy silu'(z): [t][p]
    float xsT[kSbP * kSbST], dosT[kSbP * kSbST];                  // x, dout: [p][t]
    float Bs[kSbQ * kSbSN], Cs[kSbQ * kSbSN];                     // [t][n]
    float h0T[kSbP * kSbSN], dhT[kSbP * kSbSN];                   // h_0^T, dh_Q^T: [p][n]
    // L.G.delta_s [t][s], (L.G)^T [s][t], L.delta_s.(dout x^T) [t][s], (L.(dout x^T))^T [s][t]
    float Md[kSbQ * kSbST], MmT[kSbQ * kSbST], Wm[kSbQ * kSbST], VmT[kSbQ * kSbST];
    float ecs[kSbQ], ecq[kSbQ];
    // per-token values read by the per-token pass, which runs one chunk late:
    // two copies, chunk c in copy c % 2
    float raw[2][kSbQ], dl[2][kSbQ], S[2][kSbQ], ddd[2][kSbQ], dyy[2][kSbQ];
    float hqp[2][kSbWalk / 32];  // per-warp parts of <dh_0, h_0>
    float red[kSbWalk / 32];
    float ecQ;
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

__device__ __forceinline__ float2 sb_ld2(const float *tile, int off)
{
    return *reinterpret_cast<const float2 *>(tile + off);
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

    // dh^T (P x N) in accumulator fragments: warp w holds rows p = 16 (w % 4) .. + 15,
    // columns n = 32 (w / 4) .. + 31 (four 16 x 8 tiles); element 2 hr + e of
    // tile t is (p, n) = (dm0 + g8 + 8 hr, dn0 + 8 t + 2 q4 + e)
    const int dm0 = 16 * (warp & 3), dn0 = 32 * (warp >> 2);
    float dh[4][4];
    {
        const float *dl0 = p.dlast ? p.dlast + (int64_t(b) * p.H + hh) * P * N : nullptr;
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int pp = dm0 + g8 + 8 * (e >> 1), n = dn0 + 8 * t + 2 * q4 + (e & 1);
                dh[t][e] = dl0 ? dl0[pp * N + n] : 0.f;
            }
    }
    const float *st_base = p.states + int64_t(bh) * (p.nchunks + 1) * P * N;
    // <dlast, final state> for the last chunk (both [p][n])
    float hq_next = 0.f;  // <dlast, final state>
    if (p.dlast) {
        const float *sf = st_base + int64_t(p.nchunks) * P * N;
        const float *dl0 = p.dlast + (int64_t(b) * p.H + hh) * P * N;
        for (int i = tid; i < P * N; i += kSbWalk)
            hq_next = fmaf(dl0[i], sf[i], hq_next);
    }
    const float hq_last = sb_block_sum(hq_next, sm.red, tid);
    const __nv_bfloat16 *Brow = p.B + int64_t(b) * p.B_bs + int64_t(g) * p.B_gs;
    const __nv_bfloat16 *Crow = p.C + int64_t(b) * p.C_bs + int64_t(g) * p.C_gs;
    const __nv_bfloat16 *xrow = p.x + int64_t(b) * p.x_bs + int64_t(hh) * P * p.x_cs;
    const __nv_bfloat16 *dyrow = p.dy + int64_t(b) * p.dy_bs + int64_t(hh) * P * p.dy_cs;
    const __nv_bfloat16 *zrow =
        GATE ? p.z + int64_t(b) * p.z_bs + int64_t(hh) * P * p.z_cs : nullptr;
    float *pB = p.pB + ((int64_t(hh % kSbCopies) * p.batch + b) * p.G + g) * int64_t(p.L) * N;
    float *pC = p.pC + ((int64_t(hh % kSbCopies) * p.batch + b) * p.G + g) * int64_t(p.L) * N;
    float accD = 0.f, accA = 0.f, accBias = 0.f;
    // chunk loads: x, dy, z row xp, tokens 4 xq .. + 3 (stored in the order
    // rotated by xr); B, C row bn, tokens 8 bq .. + 7 (rotated by bq)
    const int xp = tid >> 3, xq = tid & 7, xr = (xq >> 1) & 3;
    const int bn = tid >> 2, bq = tid & 3;

    // ---- 4. per-token scalars of chunk cc (one warp, lane = token), given
    //         <dh_Q, h_Q> of that chunk
    auto per_token = [&](int cc, float hq_this) {
        const int tt0 = cc * Q, vv = min(Q, p.L - tt0), cb = cc & 1;
        const bool in = lane < vv;
        const float ds = sm.dl[cb][lane];
        float dcs = sm.dyy[cb][lane] - ds * sm.ddd[cb][lane];
        if (lane == vv - 1)
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
        const float dd = sm.ddd[cb][lane] + A * R;
        const float rw = sm.raw[cb][lane];
        const float ddt = p.softplus ? dd / (1.f + expf(-rw)) : dd;
        if (in)
            p.ddt[int64_t(b) * p.ddt_bs + int64_t(hh) * p.ddt_hs + tt0 + lane] = ddt;
        accA = fmaf(dcs, sm.S[cb][lane], accA);
        accBias += in ? ddt : 0.f;
    };
    // <dh_0, h_0> of chunk cc + 1 (summed from its warps' parts), or of the end
    auto hq_after = [&](int cc) {
        if (cc + 1 >= p.nchunks)
            return hq_last;
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kSbWalk / 32; ++w)
            t += sm.hqp[(cc + 1) & 1][w];
        return t;
    };
    constexpr int kTokenWarp = 8;  // a warp with half a tile in phase 2

    for (int c = p.nchunks - 1; c >= 0; --c) {
        const int t0 = c * Q, valid = min(Q, p.L - t0), cb = c & 1;
        // ---- 1. chunk inputs (and transposed copies), h_0^T, dh_Q^T, step sizes
        {
            float xl[4], yl[4], zl[4], dv[4], zv[4];
            sb_unpack4(sb_raw4(xrow + int64_t(xp) * p.x_cs + t0 + 4 * xq, 4 * xq, valid), xl);
            sb_unpack4(sb_raw4(dyrow + int64_t(xp) * p.dy_cs + t0 + 4 * xq, 4 * xq, valid), yl);
            if (GATE)
                sb_unpack4(sb_raw4(zrow + int64_t(xp) * p.z_cs + t0 + 4 * xq, 4 * xq, valid), zl);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                dv[k] = yl[k];
                zv[k] = 0.f;
                if (GATE) {
                    const float sg = 1.f / (1.f + expf(-zl[k]));
                    dv[k] = yl[k] * zl[k] * sg;
                    zv[k] = yl[k] * (sg * (1.f + zl[k] * (1.f - sg)));
                }
            }
            *reinterpret_cast<float4 *>(&sm.xsT[sb_off(kSbST, xp, 4 * xq)]) =
                make_float4(xl[0], xl[1], xl[2], xl[3]);
            *reinterpret_cast<float4 *>(&sm.dosT[sb_off(kSbST, xp, 4 * xq)]) =
                make_float4(dv[0], dv[1], dv[2], dv[3]);
            float o[4];
            sb_xor4(xl, xr, o);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                sm.xs[sb_off(kSbSX, 4 * xq + (i ^ xr), xp)] = o[i];
            sb_xor4(dv, xr, o);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                sm.dos[sb_off(kSbSX, 4 * xq + (i ^ xr), xp)] = o[i];
            if (GATE) {
                sb_xor4(zv, xr, o);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    sm.zf[sb_off(kSbSX, 4 * xq + (i ^ xr), xp)] = o[i];
            }
        }
        {
            float f[8];
            sb_unpack8_xor(sb_raw8(Brow + int64_t(bn) * p.B_ns + t0 + 8 * bq, 8 * bq, valid), bq,
                           f);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                sm.Bs[sb_off(kSbSN, 8 * bq + (i ^ bq), bn)] = f[i];
            sb_unpack8_xor(sb_raw8(Crow + int64_t(bn) * p.C_ns + t0 + 8 * bq, 8 * bq, valid), bq,
                           f);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                sm.Cs[sb_off(kSbSN, 8 * bq + (i ^ bq), bn)] = f[i];
        }
        {
            // h_0^T: 64 rows of 128 floats in 16-byte pieces, consecutive threads
            // on consecutive pieces
            const float4 *s0 = reinterpret_cast<const float4 *>(st_base + int64_t(c) * P * N);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int f = tid + kSbWalk * i, pp = f >> 5, n = 4 * (f & 31);
                *reinterpret_cast<float4 *>(&sm.h0T[sb_off(kSbSN, pp, n)]) = s0[f];
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr)
                *reinterpret_cast<float2 *>(
                    &sm.dhT[sb_off(kSbSN, dm0 + g8 + 8 * hr, dn0 + 8 * t + 2 * q4)]) =
                    make_float2(dh[t][2 * hr], dh[t][2 * hr + 1]);
        if (warp == 0) {
            float rw, dl, S;
            sb_steps(p, b, hh, t0, valid, lane, bias, rw, dl, S);
            const float SQ = __shfl_sync(0xffffffffu, S, 31);
            sm.raw[cb][lane] = rw;
            sm.dl[cb][lane] = dl;
            sm.S[cb][lane] = S;
            sm.ecs[lane] = expf(A * S);
            sm.ecq[lane] = expf(A * (SQ - S));
            sm.ddd[cb][lane] = 0.f;
            sm.dyy[cb][lane] = 0.f;
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
                sb_gemm<N, 1, kSbExact, kSbAlong, kSbSN, kSbExact, kSbAlong, kSbSN>(
                    acc, m0, n0, sm.Cs, nullptr, sm.Bs, nullptr, lane);
            else
                sb_gemm<P, 1, (GATE ? kSbSplit : kSbExact), kSbAlong, kSbSX, kSbExact, kSbAlong,
                        kSbSX>(acc, m0, n0, sm.dos, nullptr, sm.xs, nullptr, lane);
            float *Mr = warp < 8 ? sm.Md : sm.Wm;    // [t][s], times delta_s
            float *Mc = warp < 8 ? sm.MmT : sm.VmT;  // [s][t]
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int t = m0 + g8 + 8 * hr, s_ = n0 + 2 * q4;
                float v[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float Lts = s_ + e <= t ? expf(A * (sm.S[cb][t] - sm.S[cb][s_ + e])) : 0.f;
                    v[e] = acc[0][2 * hr + e] * Lts;
                }
                float w0 = v[0] * sm.dl[cb][s_], w1 = v[1] * sm.dl[cb][s_ + 1];
                if (warp >= 8) {
                    // Wm and VmT enter their products rounded to tf32: round once here
                    v[0] = __uint_as_float(sb_tf32(v[0]));
                    v[1] = __uint_as_float(sb_tf32(v[1]));
                    w0 = __uint_as_float(sb_tf32(w0));
                    w1 = __uint_as_float(sb_tf32(w1));
                }
                Mc[sb_off(kSbST, s_, t)] = v[0];
                Mc[sb_off(kSbST, s_ + 1, t)] = v[1];
                *reinterpret_cast<float2 *>(&Mr[sb_off(kSbST, t, s_)]) = make_float2(w0, w1);
            }
            // the per-token pass of the chunk after this one: its products all
            // finished before the barrier above
            if (warp == kTokenWarp && c + 1 < p.nchunks)
                per_token(c + 1, hq_after(c + 1));
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
                sb_gemm<Q, 2, kSbSplit, kSbAlong, kSbST, kSbExact, kSbAlong, kSbST>(
                    v1, m0, n0, sm.Md, nullptr, sm.xsT, nullptr, lane);
                sb_gemm<N, 2, kSbExact, kSbAlong, kSbSN, kSbSplit, kSbAlong, kSbSN>(
                    v2, m0, n0, sm.Cs, nullptr, sm.h0T, nullptr, lane);
            } else {
                sb_gemm<Q, 2, kSbSplit, kSbAlong, kSbST, (GATE ? kSbSplit : kSbExact), kSbAlong,
                        kSbST>(v1, m0, n0, sm.MmT, nullptr, sm.dosT, nullptr, lane);
                sb_gemm<N, 2, kSbExact, kSbAlong, kSbSN, kSbSplit, kSbAlong, kSbSN>(
                    v2, m0, n0, sm.Bs, nullptr, sm.dhT, nullptr, lane);
            }
            float rs[2] = {0.f, 0.f};  // x.u (u warps) or dout.y~ (y~ warps) per row
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int r = m0 + g8 + 8 * hr, p0 = n0 + 8 * t + 2 * q4;
                    const int off = sb_off(kSbSX, r, p0);
                    const float2 x2 = sb_ld2(sm.xs, off), d2 = sb_ld2(sm.dos, off);
                    float2 z2 = make_float2(0.f, 0.f);
                    if (GATE && isy)
                        z2 = sb_ld2(sm.zf, off);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float xv = e ? x2.y : x2.x, dv = e ? d2.y : d2.x;
                        const float v1e = v1[t][2 * hr + e], v2e = v2[t][2 * hr + e];
                        const int64_t col = int64_t(hh * P + p0 + e);
                        if (isy) {
                            const float yt = fmaf(sm.ecs[r], v2e, v1e);
                            rs[hr] = fmaf(dv, yt, rs[hr]);
                            accD = fmaf(dv, xv, accD);
                            if (GATE && r < valid)
                                p.dz[int64_t(b) * p.dz_bs + col * p.dz_cs + t0 + r] =
                                    __float2bfloat16_rn((e ? z2.y : z2.x) * fmaf(dsk, xv, yt));
                        } else {
                            const float uu = fmaf(sm.ecq[r], v2e, v1e);
                            rs[hr] = fmaf(xv, uu, rs[hr]);
                            if (r < valid)
                                p.dx[int64_t(b) * p.dx_bs + col * p.dx_cs + t0 + r] =
                                    __float2bfloat16_rn(fmaf(sm.dl[cb][r], uu, dsk * dv));
                        }
                    }
                }
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                rs[hr] += __shfl_xor_sync(0xffffffffu, rs[hr], 1);
                rs[hr] += __shfl_xor_sync(0xffffffffu, rs[hr], 2);
                if (q4 == 0)
                    atomicAdd(isy ? &sm.dyy[cb][m0 + g8 + 8 * hr] : &sm.ddd[cb][m0 + g8 + 8 * hr],
                              rs[hr]);
            }
        }
        // ---- 3b. dC (warps 0-7) and dB (warps 8-15): 32 x 128 each; warp
        //          holds all 32 rows, columns 16 (w % 8) .. + 15
        {
            const int n0 = 16 * (warp & 7);
            float a1[2][2][4], a2[2][2][4];
            sb_zero(a1);
            sb_zero(a2);
            if (warp < 8) {
                sb_gemm_mt<Q, 2, 2, kSbExact, kSbAlong, kSbST, kSbExact, kSbDown, kSbSN>(
                    a1, 0, n0, sm.Wm, nullptr, sm.Bs, nullptr, lane);
                sb_gemm_mt<P, 2, 2, (GATE ? kSbRound : kSbExact), kSbAlong, kSbSX, kSbRound,
                           kSbDown, kSbSN>(a2, 0, n0, sm.dos, nullptr, sm.h0T, nullptr, lane);
            } else {
                sb_gemm_mt<Q, 2, 2, kSbExact, kSbAlong, kSbST, kSbExact, kSbDown, kSbSN>(
                    a1, 0, n0, sm.VmT, nullptr, sm.Cs, nullptr, lane);
                sb_gemm_mt<P, 2, 2, kSbExact, kSbAlong, kSbSX, kSbRound, kSbDown, kSbSN>(
                    a2, 0, n0, sm.xs, nullptr, sm.dhT, nullptr, lane);
            }
            float *dst = warp < 8 ? pC : pB;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int r = 16 * mt + g8 + 8 * hr;
                    if (r < valid) {
                        const float sc = warp < 8 ? sm.ecs[r] : sm.ecq[r];
                        const float pre = warp < 8 ? 1.f : sm.dl[cb][r];
#pragma unroll
                        for (int t = 0; t < 2; ++t) {
                            const int n = n0 + 8 * t + 2 * q4;
                            const float2 v = make_float2(
                                pre * fmaf(sc, a2[mt][t][2 * hr], a1[mt][t][2 * hr]),
                                pre * fmaf(sc, a2[mt][t][2 * hr + 1], a1[mt][t][2 * hr + 1]));
                            atomicAdd(reinterpret_cast<float2 *>(dst + int64_t(t0 + r) * N + n),
                                      v);
                        }
                    }
                }
        }
        // ---- 3c. dh_0^T = e^cs_Q dh_Q^T + sum_t (e^cs_t dout_t) C_t^T: rows p, columns n
        {
            const float eQ = sm.ecQ;
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dh[t][e] *= eQ;
            sb_gemm<Q, 4, kSbSplit, kSbDown, kSbSX, kSbExact, kSbDown, kSbSN>(
                dh, dm0, dn0, sm.dos, sm.ecs, sm.Cs, nullptr, lane);
        }
        // <dh_0, h_0> of this chunk: the <dh_Q, h_Q> term of the next one
        float hq = 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const float2 h2 =
                    sb_ld2(sm.h0T, sb_off(kSbSN, dm0 + g8 + 8 * hr, dn0 + 8 * t + 2 * q4));
                hq = fmaf(dh[t][2 * hr], h2.x, fmaf(dh[t][2 * hr + 1], h2.y, hq));
            }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            hq += __shfl_xor_sync(0xffffffffu, hq, o);
        if (lane == 0)
            sm.hqp[cb][warp] = hq;
        __syncthreads();  // the tiles are free for the next chunk
    }
    if (warp == kTokenWarp && p.nchunks > 0)
        per_token(0, hq_after(0));

    // ---- per-head sums (over this batch row), dh0
    if (p.dh0) {
        float *d0 = p.dh0 + (int64_t(b) * p.H + hh) * P * N;
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                d0[(dm0 + g8 + 8 * (e >> 1)) * N + dn0 + 8 * t + 2 * q4 + (e & 1)] = dh[t][e];
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
