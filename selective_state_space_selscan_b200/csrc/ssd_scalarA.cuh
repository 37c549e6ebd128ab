// ssd_scalarA.cuh -- scalar-A (Mamba-2) selective scan on the sm_100a tensor
// cores, in the chunked matrix form of structured state-space duality
// ("Mamba-2 y state-space models", section 4.2: the selective SSM computed
// with matrix products; "Mamba-3" blog, first section: Mamba-2's transition
// is a scalar times the identity).
//
// One CTA owns one (batch, head) and walks its chunks of Q = 128 tokens in
// order, carrying the head's state h (N x P = 128 x 64, fp32) in tensor
// memory.  With cs_t = A log2(e) S_t, S_t the inclusive sum of the step
// sizes from the chunk start:
//
//   G[t,s]   = sum_n C[n,t] B[n,s]                       (tcgen05, K = N)
//   M[t,s]   = G[t,s] 2^(cs_t - cs_s) delta_s, s <= t     (CUDA cores)
//   Yd[t,p]  = sum_s M[t,s] x[p,s]                        (tcgen05, K = Q)
//   Yo[t,p]  = sum_n C[n,t] h_prev[n,p]                   (tcgen05, K = N)
//   y[p,t]   = Yd[t,p] + 2^cs_t Yo[t,p] + D x[p,t]        (then the gate)
//   h[n,p]   = 2^cs_Q h_prev[n,p]
//            + sum_s B[n,s] 2^(cs_Q - cs_s) delta_s x[p,s]   (tcgen05)
//
// 2^(cs_t - cs_s) is the product of the per-token decays between s and t, so
// this is the recurrence of the diagonal scan with A[d,n] = A_head.  No
// factor exceeds 1: below the diagonal 16 x 16 pieces of M the decay is split
// at the last token e of the column piece, 2^(cs_t - cs_e) 2^(cs_e - cs_s)
// (one exponential per row and piece, one per column), and in the pieces
// that hold a warp's diagonal it is taken per element.
//
// Per chunk c, in order (all threads unless noted), each tensor-core product
// issued by one thread as soon as its inputs are in place and waited for as
// late as possible, so that it runs under the next CUDA-core phase:
//   1. x * w for the state product (needs chunk c's x); issue the state
//      product h += B (x w)^T, which runs during step 2;
//   2. the second warpgroup prepares the step sizes of chunk c + 1 (into the
//      other set of per-token arrays); M from G (tensor memory) and the
//      decays; issue Yd(c) and G(c + 1), which run during step 3;
//   3. state: h -> bf16 copy for Yo(c + 1), last_state, h *= 2^cs_Q(c + 1);
//      issue Yo(c + 1) (into the other Yo columns), which runs during step 4;
//   4. y = Yd + 2^cs_t Yo + D x (+ gate), staged in shared memory and written
//      back by one bulk tensor store; issue the loads of chunk c + 2.
//
// Operands (bf16, 128-byte swizzle) in shared memory:
//   C chunk [n][t] and B chunk [n][s] as loaded by the bulk tensor copy,
//   used MN-major (C^T as A of G and Yo; B as B of G) and K-major (B as A of
//   the state product); x chunk [p][s] (K-major B of Yd); x * w [p][s]
//   (K-major B of the state product); M [t][s] (K-major A of Yd); h_prev in
//   bf16 [n][p] (MN-major B of Yo), in the x * w buffer.  The y tile [p][t]
//   is staged in the M buffer once Yd has read it.  Accumulators in tensor
//   memory (fp32): G (128 columns), Yd (64), Yo (2 x 64), h (64).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "f32x2.cuh"
#include "ptx.cuh"
#include "umma.cuh"

namespace selscan {

constexpr int kSsdN = 128;  // state size built
constexpr int kSsdP = 64;   // head dimension built
constexpr int kSsdQ = 128;  // chunk length
constexpr int kSsdWG = 4;   // warpgroups per CTA

struct SsdParams {
    int batch, H, L, nchunks;
    int heads_per_group;       // head h reads B/C group h / heads_per_group
    const float *dt;           // (batch, H, L), time stride 1
    int64_t dt_bs, dt_hs;
    const float *dt_bias;      // (H) or null
    int softplus;
    const float *A;            // (H)
    const float *Dskip;        // (H) or null
    const __nv_bfloat16 *z;    // (batch, H*P, L) or null
    int64_t z_bs, z_cs;
    float *last_state;         // (batch, H, P, N) or null
    const float *h0;           // (batch, H, P, N) or null: initial state
    unsigned long long timeout_ns;
    unsigned int *err;
};

struct SsdLayout {
    static constexpr int kC = 0;                   // 2 buffers x [2 slabs][128 n][64 t]
    static constexpr int kB = kC + 2 * 32768;      // 2 buffers x [2 slabs][128 n][64 s]
    static constexpr int kX = kB + 2 * 32768;      // 2 buffers x [2 slabs][64 p][64 s]
    static constexpr int kXw = kX + 2 * 16384;     // [2 slabs][64 p][64 s]
    static constexpr int kM = kXw + 16384;         // [2 slabs][128 t][64 s]; y tile [2][64 p][64 t]
    // bf16 state [128 n][64 p] for Yo, in the x*w buffer: written once the
    // state product has read x*w, read by Yo(c+1), which completes before
    // the next chunk's x*w is written
    static constexpr int kHs = kXw;
    static constexpr int kBytes = kM + 32768;
    static constexpr int kAlloc = kBytes + 1024;
};

constexpr uint32_t kSsdTmemCols = 512;
constexpr uint32_t kColG = 0, kColYd = 128, kColH = 256;
// Yo of chunk c in columns kColYo + 128 (c % 2): Yo(c + 1) is issued once the
// state of chunk c is out, while chunk c's epilogue still reads Yo(c)
constexpr uint32_t kColYo = 192;

__device__ __forceinline__ float ssd_softplus(float x)
{
    return x > 20.f ? x : log1pf(__expf(x));
}

// 16 consecutive fp32 from shared memory (16-byte aligned).
__device__ __forceinline__ void lds16(const float *src, float (&v)[16])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 q = reinterpret_cast<const float4 *>(src)[i];
        v[4 * i] = q.x;
        v[4 * i + 1] = q.y;
        v[4 * i + 2] = q.z;
        v[4 * i + 3] = q.w;
    }
}

// 16 values -> bf16, stored as two 16-byte swizzle units at byte offsets o0, o1.
__device__ __forceinline__ void sts16_bf16(uint8_t *base, uint32_t o0, uint32_t o1,
                                           const float (&m)[16])
{
    uint4 a, c;
    a.x = pack2_bf16(m[0], m[1]);
    a.y = pack2_bf16(m[2], m[3]);
    a.z = pack2_bf16(m[4], m[5]);
    a.w = pack2_bf16(m[6], m[7]);
    c.x = pack2_bf16(m[8], m[9]);
    c.y = pack2_bf16(m[10], m[11]);
    c.z = pack2_bf16(m[12], m[13]);
    c.w = pack2_bf16(m[14], m[15]);
    *reinterpret_cast<uint4 *>(base + o0) = a;
    *reinterpret_cast<uint4 *>(base + o1) = c;
}

template <bool GATE>
__global__ void __launch_bounds__(kSsdWG * 128, 1)
ssd_scalarA_kernel(const __grid_constant__ CUtensorMap tm_C,
                   const __grid_constant__ CUtensorMap tm_B,
                   const __grid_constant__ CUtensorMap tm_X,
                   const __grid_constant__ CUtensorMap tm_Y, const SsdParams p)
{
    using Lay = SsdLayout;
    constexpr int Q = kSsdQ, P = kSsdP, N = kSsdN, NWG = kSsdWG, NT = NWG * 128;
    constexpr int PW = P / NWG;    // p columns per thread in the epilogue / state pass
    constexpr int QPW = 8 / NWG;   // 16-column pieces of M per thread
    static_assert(PW % 16 == 0 && QPW % 2 == 0, "column split");
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, offset from the shared array itself so that
    // every pointer derived from it stays in the shared address space
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    // per-token values of the chunk being prepared (see cumsum below)
    // (two sets, by chunk parity: the next chunk's are prepared while this
    // chunk's are read)
    __shared__ __align__(16) float s_cs2[2][Q], s_n22[2][Q], s_sg2[2][Q];
    __shared__ float s_wsum[4];
    __shared__ uint64_t bar_tma[2], bar_g, bar_yo, bar_yd, bar_st;
    __shared__ uint32_t s_tbase;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane: token t or state n of this thread
    const int b = blockIdx.x / p.H, hh = blockIdx.x - b * p.H;
    const float a_l2 = p.A[hh] * 1.4426950408889634f;  // A in log2 units
    const float bias = p.dt_bias ? p.dt_bias[hh] : 0.f;
    const float dsk = p.Dskip ? p.Dskip[hh] : 0.f;
    const uint32_t sbase = smem_addr(smem);
    const uint32_t aXw = sbase + Lay::kXw, aM = sbase + Lay::kM, aHs = sbase + Lay::kHs;
    const float *dt_row = p.dt + int64_t(b) * p.dt_bs + int64_t(hh) * p.dt_hs;

    auto issue_loads = [&](int c) {
        const int t0 = c * Q, buf = c & 1;
        mbar_arrive_expect_tx(&bar_tma[buf], 32768 + 32768 + 16384);
        uint8_t *cs = smem + Lay::kC + buf * 32768;
        uint8_t *bs = smem + Lay::kB + buf * 32768;
        uint8_t *xs = smem + Lay::kX + buf * 16384;
        const int grow = (hh / p.heads_per_group) * N;  // first row of this head's group
        tma_load_3d(cs, &tm_C, &bar_tma[buf], t0, grow, b);
        tma_load_3d(cs + 16384, &tm_C, &bar_tma[buf], t0 + 64, grow, b);
        tma_load_3d(bs, &tm_B, &bar_tma[buf], t0, grow, b);
        tma_load_3d(bs + 16384, &tm_B, &bar_tma[buf], t0 + 64, grow, b);
        tma_load_3d(xs, &tm_X, &bar_tma[buf], t0, hh * P, b);
        tma_load_3d(xs + 8192, &tm_X, &bar_tma[buf], t0 + 64, hh * P, b);
    };

    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(&bar_g, 1);
        mbar_init(&bar_yo, 1);
        mbar_init(&bar_yd, 1);
        mbar_init(&bar_st, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_C);
        prefetch_tmap(&tm_B);
        prefetch_tmap(&tm_X);
        prefetch_tmap(&tm_Y);
        issue_loads(0);
        if (p.nchunks > 1)
            issue_loads(1);
    }
    if (warp == 0)
        tmem_alloc(&s_tbase, kSsdTmemCols);

    // Step sizes of chunk cc (second warpgroup, token r, so that the thread
    // issuing the tensor-core work in warp 0 never delays it): delta, its inclusive
    // sum in log2-decay units cs, and per token
    //   s_n2[s] = log2(delta_s) - cs_s        (pieces on a warp's diagonal)
    //   s_sg[s] = 2^(cs_e - cs_s) delta_s     (e = last token of s's piece)
    auto cumsum = [&](int cc, float dtv) {
        if (wg != 1)
            return;
        float dl = dtv + bias;
        if (p.softplus)
            dl = ssd_softplus(dl);
        dl = (cc * Q + r < p.L) ? dl : 0.f;
        float S = dl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, S, o);
            if (lane >= o)
                S += v;
        }
        if (lane == 31)
            s_wsum[quarter] = S;
        named_bar_sync(1, 128);
        for (int w = 0; w < quarter; ++w)
            S += s_wsum[w];
        const float cs = a_l2 * S;
        const float cse = __shfl_sync(0xffffffffu, cs, lane | 15);
        s_cs2[cc & 1][r] = cs;
        s_n22[cc & 1][r] = lg2_approx(dl) - cs;  // -inf for delta = 0, and 2^-inf = 0
        s_sg2[cc & 1][r] = ex2_approx(cse - cs) * dl;
    };

    // initial state h[n][p] (zero unless given): row n = r, columns p of this
    // warpgroup's slice
    float h_init[PW];
    {
        const float *h0row = p.h0 ? p.h0 + (int64_t(b) * p.H + hh) * P * N + r : nullptr;
#pragma unroll
        for (int i = 0; i < PW; ++i)
            h_init[i] = h0row ? h0row[int64_t(wg * PW + i) * N] : 0.f;
    }
    cumsum(0, (wg == 1 && r < p.L) ? dt_row[r] : 0.f);
    float dt_next = (wg == 1 && Q + r < p.L) ? dt_row[Q + r] : 0.f;
    __syncthreads();  // s_cs of chunk 0, TMEM address
    tmem_fence_after_sync();
    const uint32_t tb = s_tbase;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;  // this warp's TMEM lanes
    {
        const float alpha0 = ex2_approx(s_cs2[0][Q - 1]);
        uint8_t *hs = smem + Lay::kHs;
#pragma unroll
        for (int cc = 0; cc < PW; cc += 16) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                v[i] = h_init[cc + i];
            const uint32_t col = uint32_t(wg * PW + cc);
            sts16_bf16(hs, sw128_offset(r, col), sw128_offset(r, col + 8), v);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                v[i] *= alpha0;
            tmem_st16(tb + lane_off + kColH + col, v);
        }
    }
    fence_proxy_async_smem();
    tmem_fence_before_sync();
    __syncthreads();

    constexpr uint32_t idG = umma_idesc_bf16(128, 128, true, true);
    constexpr uint32_t idYo = umma_idesc_bf16(128, 64, true, true);
    constexpr uint32_t idYd = umma_idesc_bf16(128, 64, false, false);
    auto issue_G = [&](int c) {
        const uint32_t aC = sbase + Lay::kC + (c & 1) * 32768;
        const uint32_t aB = sbase + Lay::kB + (c & 1) * 32768;
#pragma unroll
        for (int kk = 0; kk < N / 16; ++kk)
            umma_bf16(tb + kColG, umma_desc_mnmajor(aC, N, kk), umma_desc_mnmajor(aB, N, kk),
                      idG, kk > 0);
        umma_commit(&bar_g);
    };
    auto issue_Yo = [&](int c) {
        const uint32_t aC = sbase + Lay::kC + (c & 1) * 32768;
        const uint32_t col = kColYo + uint32_t(c & 1) * 128u;
#pragma unroll
        for (int kk = 0; kk < N / 16; ++kk)
            umma_bf16(tb + col, umma_desc_mnmajor(aC, N, kk), umma_desc_mnmajor(aHs, N, kk),
                      idYo, kk > 0);
        umma_commit(&bar_yo);
    };
    bool ok = true;
    if (tid == 0) {
        tmem_fence_after_sync();
        ok = mbar_wait(&bar_tma[0], 0u, p.timeout_ns) && ok;
        issue_Yo(0);
        issue_G(0);
    }

    // byte offsets of x[p][t] / y[p][t] (t = r) in a [2 slabs][64 p][64 t]
    // tile for p = 8k + j: slab + p*128 + ((t%64/8 ^ j) << 4) + (t%8)*2
    uint32_t off8[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        off8[j] = uint32_t(r >> 6) * 8192u + ((((uint32_t(r) & 63u) >> 3) ^ uint32_t(j)) << 4) +
                  (uint32_t(r) & 7u) * 2u;

    for (int c = 0; c < p.nchunks; ++c) {
        const int buf = c & 1;
        const uint32_t ph = uint32_t(c & 1);          // bar_g / bar_yo / bar_yd / bar_st
        const uint32_t tph = uint32_t((c >> 1) & 1);  // bar_tma[buf]
        const int t0 = c * Q;
        const uint32_t aB = sbase + Lay::kB + buf * 32768;
        const uint32_t aX = sbase + Lay::kX + buf * 16384;
        const uint8_t *xs = smem + Lay::kX + buf * 16384;

        // ---- 1. x * w for the state product, w_s = 2^(cs_Q - cs_s) delta_s
        //         = 2^(cs_Q - cs_e) s_sg[s]; units of (p, 8 tokens)
        const float *s_cs = s_cs2[c & 1], *s_n2 = s_n22[c & 1], *s_sg = s_sg2[c & 1];
        ok = mbar_wait(&bar_tma[buf], tph, p.timeout_ns) && ok;
        ok = mbar_wait(&bar_yo, ph, p.timeout_ns) && ok;  // Yo(c) has read the bf16 state
        {
            const float csQ = s_cs[Q - 1];
            uint8_t *xw = smem + Lay::kXw;
#pragma unroll
            for (int k = 0; k < 1024 / NT; ++k) {
                const int u = tid + k * NT;
                const int pp = u & 63, g = u >> 6;  // g: 8-token group 0..15
                const float pf = ex2_approx(csQ - s_cs[(g >> 1) * 16 + 15]);
                const float4 w0 = reinterpret_cast<const float4 *>(s_sg + g * 8)[0];
                const float4 w1 = reinterpret_cast<const float4 *>(s_sg + g * 8)[1];
                const uint32_t off = uint32_t(g >> 3) * 8192u + uint32_t(pp) * 128u +
                                     ((uint32_t(g & 7) ^ uint32_t(pp & 7)) << 4);
                const uint4 xv = *reinterpret_cast<const uint4 *>(xs + off);
                const uint64_t PF = pk2(pf, pf);
                const uint64_t s01 = mul2(pk2(w0.x, w0.y), PF), s23 = mul2(pk2(w0.z, w0.w), PF);
                const uint64_t s45 = mul2(pk2(w1.x, w1.y), PF), s67 = mul2(pk2(w1.z, w1.w), PF);
                const uint64_t x01 = mul2(bf2_to_f2(xv.x), s01), x23 = mul2(bf2_to_f2(xv.y), s23);
                const uint64_t x45 = mul2(bf2_to_f2(xv.z), s45), x67 = mul2(bf2_to_f2(xv.w), s67);
                uint4 o;
                o.x = pack2_bf16(lo2(x01), hi2(x01));
                o.y = pack2_bf16(lo2(x23), hi2(x23));
                o.z = pack2_bf16(lo2(x45), hi2(x45));
                o.w = pack2_bf16(lo2(x67), hi2(x67));
                *reinterpret_cast<uint4 *>(xw + off) = o;
            }
        }
        // the state product h += B (x w)^T runs while the mask is built
        fence_proxy_async_smem();
        tmem_fence_before_sync();
        if (tid == 0)
            bulk_wait_read<0>();  // the previous chunk's y tile has left the M buffer
        __syncthreads();
        if (tid == 0) {
            tmem_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < Q / 16; ++kk)
                umma_bf16(tb + kColH, umma_desc_kmajor(aB, N, kk), umma_desc_kmajor(aXw, P, kk),
                          idYd, 1u);
            umma_commit(&bar_st);
        }
        // ---- 2. the next chunk's step sizes (second warpgroup, into the other
        //         set), then M: row t = r, pieces q = wg + NWG * j of 16 columns
        if (c + 1 < p.nchunks) {
            cumsum(c + 1, dt_next);
            if (wg == 1)
                dt_next = (t0 + 2 * Q + r < p.L) ? dt_row[t0 + 2 * Q + r] : 0.f;
        }
        const float cs_t = s_cs[r];
        const float ey = ex2_approx(cs_t);  // Yo row scale, used in step 4
        ok = mbar_wait(&bar_g, ph, p.timeout_ns) && ok;
        tmem_fence_after_sync();
        {
            uint8_t *mt = smem + Lay::kM;
#pragma unroll
            for (int j0 = 0; j0 < QPW; j0 += 2) {
                float gv[2][16];
                tmem_ld16x2(tb + lane_off + kColG + (wg + NWG * j0) * 16, gv[0],
                            tb + lane_off + kColG + (wg + NWG * (j0 + 1)) * 16, gv[1]);
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const int q = wg + NWG * (j0 + jj);
                    float m[16];
                    if (q < 2 * quarter) {
                        // every row of this warp is past piece q: split decay
                        float sg[16];
                        lds16(s_sg + q * 16, sg);
                        const float fr = ex2_approx(cs_t - s_cs[q * 16 + 15]);
                        const uint64_t FR = pk2(fr, fr);
#pragma unroll
                        for (int i = 0; i < 16; i += 2) {
                            const uint64_t v = mul2(
                                mul2(pk2(gv[jj][i], gv[jj][i + 1]), pk2(sg[i], sg[i + 1])), FR);
                            m[i] = lo2(v);
                            m[i + 1] = hi2(v);
                        }
                    } else if (q <= 2 * quarter + 1) {
                        // pieces holding this warp's diagonal: per element, masked
                        float n2[16];
                        lds16(s_n2 + q * 16, n2);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float e = ex2_approx(cs_t + n2[i]);
                            m[i] = (q * 16 + i <= r) ? gv[jj][i] * e : 0.f;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            m[i] = 0.f;
                    }
                    const uint32_t slab = uint32_t(q >> 2) * 16384u;
                    const uint32_t col = uint32_t(q & 3) * 16u;
                    sts16_bf16(mt, slab + sw128_offset(r, col), slab + sw128_offset(r, col + 8),
                               m);
                }
            }
        }
        fence_proxy_async_smem();
        tmem_fence_before_sync();
        __syncthreads();
        // ---- Yd = M x^T; then the next chunk's C^T B
        if (tid == 0) {
            tmem_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < Q / 16; ++kk)
                umma_bf16(tb + kColYd, umma_desc_kmajor(aM, 128, kk), umma_desc_kmajor(aX, P, kk),
                          idYd, kk > 0);
            umma_commit(&bar_yd);
            if (c + 1 < p.nchunks) {
                ok = mbar_wait(&bar_tma[buf ^ 1], uint32_t(((c + 1) >> 1) & 1), p.timeout_ns) &&
                     ok;
                tmem_fence_after_sync();
                issue_G(c + 1);
            }
        }
        // ---- 3. state n = r (while Yd runs): bf16 copy for Yo(c+1) (over
        //         x*w, which the state product has read), final state, decay
        //         into chunk c+1
        ok = mbar_wait(&bar_st, ph, p.timeout_ns) && ok;
        tmem_fence_after_sync();
        {
            uint8_t *hs = smem + Lay::kHs;
            const bool last = c == p.nchunks - 1;
            // chunk c+1's decay (its step sizes were prepared in step 2)
            const float alpha = last ? 1.f : ex2_approx(s_cs2[(c + 1) & 1][Q - 1]);
            float *ls = (p.last_state && last)
                            ? p.last_state + (int64_t(b) * p.H + hh) * P * N + r
                            : nullptr;
#pragma unroll
            for (int cc = 0; cc < PW; cc += 16) {
                const uint32_t col = uint32_t(wg * PW + cc);
                float hv[16];
                tmem_ld16(tb + lane_off + kColH + col, hv);
                if (!last) {
                    sts16_bf16(hs, sw128_offset(r, col), sw128_offset(r, col + 8), hv);
                    const uint64_t AL = pk2(alpha, alpha);
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        const uint64_t v = mul2(pk2(hv[i], hv[i + 1]), AL);
                        hv[i] = lo2(v);
                        hv[i + 1] = hi2(v);
                    }
                    tmem_st16(tb + lane_off + kColH + col, hv);
                } else if (ls) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        ls[int64_t(col + i) * N] = hv[i];
                }
            }
        }
        fence_proxy_async_smem();
        tmem_fence_before_sync();
        __syncthreads();
        if (tid == 0 && c + 1 < p.nchunks) {
            tmem_fence_after_sync();
            issue_Yo(c + 1);  // runs during this chunk's epilogue
        }
        // ---- 4. y for token t = r, columns p of this warpgroup's slice
        ok = mbar_wait(&bar_yd, ph, p.timeout_ns) && ok;
        tmem_fence_after_sync();
        {
            uint8_t *ys = smem + Lay::kM;  // Yd has finished reading M
            const bool valid = t0 + r < p.L;
            const uint32_t colYo = kColYo + uint32_t(c & 1) * 128u;
            const __nv_bfloat16 *zrow =
                GATE ? p.z + int64_t(b) * p.z_bs + int64_t(hh * P) * p.z_cs + t0 + r : nullptr;
#pragma unroll
            for (int cc = 0; cc < PW; cc += 16) {
                const int pbase = wg * PW + cc;
                float yd[16], yo[16];
                tmem_ld16x2(tb + lane_off + kColYd + pbase, yd, tb + lane_off + colYo + pbase, yo);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint32_t off = off8[i & 7] + uint32_t(pbase + i) * 128u;
                    const float xv = __uint_as_float(
                        uint32_t(*reinterpret_cast<const uint16_t *>(xs + off)) << 16);
                    float v = fmaf(ey, yo[i], yd[i]);
                    v = fmaf(dsk, xv, v);
                    if (GATE) {
                        const float zv =
                            valid ? __bfloat162float(zrow[int64_t(pbase + i) * p.z_cs]) : 0.f;
                        v *= zv / (1.f + __expf(-zv));
                    }
                    *reinterpret_cast<__nv_bfloat16 *>(ys + off) = __float2bfloat16_rn(v);
                }
            }
        }
        fence_proxy_async_smem();
        tmem_fence_before_sync();
        __syncthreads();
        // ---- y out; chunk c+2 into this chunk's buffer (x, B and C of
        //      chunk c are no longer read: Yd, the state product and Yo(c) are done)
        if (tid == 0) {
            tma_store_3d(&tm_Y, smem + Lay::kM, t0, hh * P, b);
            if (t0 + 64 < p.L)
                tma_store_3d(&tm_Y, smem + Lay::kM + 8192, t0 + 64, hh * P, b);
            bulk_commit();
            if (c + 2 < p.nchunks) {
                fence_proxy_async_smem();
                issue_loads(c + 2);
            }
        }
    }
    if (tid == 0)
        bulk_wait_all<0>();
    if (!ok)
        atomicOr(p.err, 4u);
    tmem_fence_after_sync();
    if (warp == 0)
        tmem_dealloc(tb, kSsdTmemCols);
}

}  // namespace selscan
