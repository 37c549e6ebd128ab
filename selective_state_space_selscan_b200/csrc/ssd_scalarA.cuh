// ssd_scalarA.cuh -- scalar-A (Mamba-2) selective scan on the sm_100a tensor
// cores, in the chunked matrix form of structured state-space duality
// ("Mamba-2 y state-space models", section 4.2: the selective SSM computed
// with matrix products; "Mamba-3" blog, first section: Mamba-2's transition
// is a scalar times the identity).
//
// One CTA owns one (batch, head) and walks its chunks of Q = 128 tokens in
// order, carrying the head's state h (N x P = 128 x 64, fp32) in tensor
// memory.  For a chunk with cumulative step sum S_t (inclusive, from the
// chunk start):
//
//   G[t,s]   = sum_n C[n,t] B[n,s]                       (tcgen05, K = N)
//   M[t,s]   = G[t,s] exp(A (S_t - S_s)) delta_s, s <= t  (CUDA cores)
//   Yd[t,p]  = sum_s M[t,s] x[p,s]                        (tcgen05, K = Q)
//   Yo[t,p]  = sum_n C[n,t] h_prev[n,p]                   (tcgen05, K = N)
//   y[p,t]   = Yd[t,p] + exp(A S_t) Yo[t,p] + D x[p,t]    (then the gate)
//   h[n,p]   = exp(A S_Q) h_prev[n,p]
//            + sum_s B[n,s] exp(A (S_Q - S_s)) delta_s x[p,s]   (tcgen05)
//
// exp(A (S_t - S_s)) is the product of the per-token decays between s and
// t, so this is the recurrence of the diagonal scan with A[d,n] = A_head.
// The mask factors never overflow: inside a 32-token block the exponential
// is taken per element; across blocks it is split at the end of the earlier
// block, where both factors are <= 1.
//
// Operands (bf16, 128-byte swizzle) in shared memory:
//   C chunk [n][t] and B chunk [n][s] as loaded by the bulk tensor copy,
//   used MN-major (C^T as A of G and Yo; B as B of G) and K-major (B as A of
//   the state product); x chunk [p][s] (K-major B of Yd); x * w [p][s]
//   (K-major B of the state product); M [t][s] (K-major A of Yd); h_prev in
//   bf16 [n][p] (MN-major B of Yo).  Accumulators in tensor memory (fp32):
//   G (128 columns), Yd (64), Yo (64), h (64).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "umma.cuh"

namespace selscan {

constexpr int kSsdN = 128;  // state size built
constexpr int kSsdP = 64;   // head dimension built
constexpr int kSsdQ = 128;  // chunk length

struct SsdParams {
    int batch, H, L, nchunks;
    const float *dt;           // (batch, H, L), time stride 1
    int64_t dt_bs, dt_hs;
    const float *dt_bias;      // (H) or null
    int softplus;
    const float *A;            // (H)
    const float *Dskip;        // (H) or null
    const __nv_bfloat16 *z;    // (batch, H*P, L) or null
    int64_t z_bs, z_cs;
    __nv_bfloat16 *y;          // (batch, H*P, L)
    int64_t y_bs, y_cs;
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
    static constexpr int kM = kXw + 16384;         // [2 slabs][128 t][64 s]
    static constexpr int kHs = kM + 32768;         // [128 n][64 p]
    static constexpr int kBytes = kHs + 16384;
    static constexpr int kAlloc = kBytes + 1024;
};

constexpr uint32_t kSsdTmemCols = 512;
constexpr uint32_t kColG = 0, kColYd = 128, kColYo = 192, kColH = 256;

__device__ __forceinline__ uint32_t ssd_pack2(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float ssd_softplus(float x)
{
    return x > 20.f ? x : log1pf(__expf(x));
}

template <bool GATE>
__global__ void __launch_bounds__(256, 1)
ssd_scalarA_kernel(const __grid_constant__ CUtensorMap tm_C,
                   const __grid_constant__ CUtensorMap tm_B,
                   const __grid_constant__ CUtensorMap tm_X, const SsdParams p)
{
    using Lay = SsdLayout;
    constexpr int Q = kSsdQ, P = kSsdP, N = kSsdN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ float s_delta[Q], s_S[Q], s_g[Q], s_wsum[4];
    __shared__ uint64_t bar_tma[2], bar_g, bar_yo, bar_mma;
    __shared__ uint32_t s_tbase;

    // Two threads per row: r = row / token / state index, half = which half of
    // the columns this thread handles.  Warp w reaches TMEM lanes 32*(w%4).
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = tid & 127, half = tid >> 7;
    const int b = blockIdx.x / p.H, hh = blockIdx.x - b * p.H;
    const float a_l2 = p.A[hh] * 1.4426950408889634f;  // A in log2 units
    const float bias = p.dt_bias ? p.dt_bias[hh] : 0.f;
    const float dsk = p.Dskip ? p.Dskip[hh] : 0.f;
    const uint32_t sbase = smem_addr(smem);
    const uint32_t aXw = sbase + Lay::kXw, aM = sbase + Lay::kM, aHs = sbase + Lay::kHs;

    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(&bar_g, 1);
        mbar_init(&bar_yo, 1);
        mbar_init(&bar_mma, 1);
        fence_mbar_init();
        prefetch_tmap(&tm_C);
        prefetch_tmap(&tm_B);
        prefetch_tmap(&tm_X);
    }
    if (warp == 0)
        tmem_alloc(&s_tbase, kSsdTmemCols);
    // initial state h[n][p] (zero unless given): this thread's row n = r,
    // columns p of its half; kept in fp32 for TMEM and in bf16 for C^T h
    float h_init[32];
    {
        const float *h0row = p.h0 ? p.h0 + (int64_t(b) * p.H + hh) * P * N + r : nullptr;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            h_init[i] = h0row ? h0row[int64_t(half * 32 + i) * N] : 0.f;
        uint8_t *hs = smem + Lay::kHs;
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
            uint4 pk;
            pk.x = ssd_pack2(h_init[g8 * 8 + 0], h_init[g8 * 8 + 1]);
            pk.y = ssd_pack2(h_init[g8 * 8 + 2], h_init[g8 * 8 + 3]);
            pk.z = ssd_pack2(h_init[g8 * 8 + 4], h_init[g8 * 8 + 5]);
            pk.w = ssd_pack2(h_init[g8 * 8 + 6], h_init[g8 * 8 + 7]);
            *reinterpret_cast<uint4 *>(hs + sw128_offset(r, half * 32 + g8 * 8)) = pk;
        }
    }
    fence_proxy_async_smem();
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tb = s_tbase;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;  // this warp's TMEM lanes
    const uint32_t colh = uint32_t(half * 32);                   // this thread's column half
    {
        float v0[16], v1[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            v0[i] = h_init[i];
            v1[i] = h_init[16 + i];
        }
        tmem_st16(tb + lane_off + kColH + colh, v0);
        tmem_st16(tb + lane_off + kColH + colh + 16, v1);
    }

    const float *dt_row = p.dt + int64_t(b) * p.dt_bs + int64_t(hh) * p.dt_hs;
    auto issue_loads = [&](int c) {
        const int t0 = c * Q, buf = c & 1;
        mbar_arrive_expect_tx(&bar_tma[buf], 32768 + 32768 + 16384);
        uint8_t *cs = smem + Lay::kC + buf * 32768;
        uint8_t *bs = smem + Lay::kB + buf * 32768;
        uint8_t *xs = smem + Lay::kX + buf * 16384;
        tma_load_3d(cs, &tm_C, &bar_tma[buf], t0, 0, b);
        tma_load_3d(cs + 16384, &tm_C, &bar_tma[buf], t0 + 64, 0, b);
        tma_load_3d(bs, &tm_B, &bar_tma[buf], t0, 0, b);
        tma_load_3d(bs + 16384, &tm_B, &bar_tma[buf], t0 + 64, 0, b);
        tma_load_3d(xs, &tm_X, &bar_tma[buf], t0, hh * P, b);
        tma_load_3d(xs + 8192, &tm_X, &bar_tma[buf], t0 + 64, hh * P, b);
    };
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
    bool ok = true;
    if (tid == 0) {
        issue_loads(0);
        if (p.nchunks > 1)
            issue_loads(1);
        ok = mbar_wait(&bar_tma[0], 0u, p.timeout_ns) && ok;
        tmem_fence_after_sync();
        issue_G(0);
    }
    float dt_next = (half == 0 && r < p.L) ? dt_row[r] : 0.f;

    for (int c = 0; c < p.nchunks; ++c) {
        const int buf = c & 1;
        const uint32_t ph = uint32_t(c & 1);        // bar_g / bar_yo / bar_mma phase
        const uint32_t tph = uint32_t((c >> 1) & 1);  // bar_tma[buf] phase
        const int t0 = c * Q;
        const uint32_t aC = sbase + Lay::kC + buf * 32768;
        const uint32_t aB = sbase + Lay::kB + buf * 32768;
        const uint32_t aX = sbase + Lay::kX + buf * 16384;
        // ---- carried-in term Yo = C^T h_prev (h_prev in bf16 from the last chunk)
        if (tid == 0) {
            if (c > 0)
                ok = mbar_wait(&bar_tma[buf], tph, p.timeout_ns) && ok;
            tmem_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < N / 16; ++kk)
                umma_bf16(tb + kColYo, umma_desc_mnmajor(aC, N, kk),
                          umma_desc_mnmajor(aHs, N, kk), idYo, kk > 0);
            umma_commit(&bar_yo);
        }
        // ---- step sizes and their cumulative sum over the chunk (first 128 threads)
        const bool valid = t0 + r < p.L;
        float dl = dt_next + bias;
        if (p.softplus)
            dl = ssd_softplus(dl);
        dl = valid ? dl : 0.f;
        float S = dl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float v = __shfl_up_sync(0xffffffffu, S, o);
            if (lane >= o)
                S += v;
        }
        if (half == 0 && lane == 31)
            s_wsum[warp] = S;
        __syncthreads();
        for (int w = 0; w < (warp & 3); ++w)
            S += s_wsum[w];
        if (half == 0) {
            s_delta[r] = dl;
            s_S[r] = S;
        }
        __syncthreads();
        S = s_S[r];
        dl = s_delta[r];
        const float S_end = s_S[Q - 1];
        if (half == 0)
            s_g[r] = ex2_approx(a_l2 * (s_S[(r | 31)] - S)) * dl;
        const float w_state = ex2_approx(a_l2 * (S_end - S)) * dl;  // x scale for h
        const float e_row = ex2_approx(a_l2 * S);                     // Yo row scale
        if (half == 0 && c + 1 < p.nchunks)
            dt_next = (t0 + Q + r < p.L) ? dt_row[t0 + Q + r] : 0.f;
        __syncthreads();
        // every thread reads this chunk's x below
        ok = mbar_wait(&bar_tma[buf], tph, p.timeout_ns) && ok;
        // ---- x * w for the state product (rows p of this half), h *= exp(A S_end)
        {
            const uint8_t *xs = smem + Lay::kX + buf * 16384;
            uint8_t *xw = smem + Lay::kXw;
            const uint32_t slab = uint32_t(r >> 6) * 8192u;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int pp = half * 32 + i;
                const uint32_t off = slab + sw128_offset(pp, r & 63);
                const float xv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(xs + off));
                *reinterpret_cast<__nv_bfloat16 *>(xw + off) = __float2bfloat16_rn(xv * w_state);
            }
            const float dec = ex2_approx(a_l2 * S_end);
#pragma unroll
            for (int cc = 0; cc < 32; cc += 16) {
                float v[16];
                tmem_ld16(tb + lane_off + kColH + colh + cc, v);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    v[i] *= dec;
                tmem_st16(tb + lane_off + kColH + colh + cc, v);
            }
        }
        // ---- M = G masked by the decays: row t = r, pieces 4*half .. 4*half+3
        ok = mbar_wait(&bar_g, ph, p.timeout_ns) && ok;
        tmem_fence_after_sync();
        {
            const int bi = warp & 3;  // 32-token block of this row
            uint8_t *mrow = smem + Lay::kM;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const int q = half * 4 + qq;  // 16-column piece of the row
                float m[16];
                if (q < 2 * (bi + 1)) {       // warp-uniform
                    float gv[16];
                    tmem_ld16(tb + lane_off + kColG + q * 16, gv);
                    const int bj = q >> 1;
                    // exp(A (S_t - S_{end of block bj})) for a block before this row's
                    const float fr = (bj < bi) ? ex2_approx(a_l2 * (S - s_S[32 * bj + 31])) : 0.f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int s = q * 16 + i;
                        float v;
                        if (bj < bi)
                            v = gv[i] * fr * s_g[s];
                        else
                            v = (s <= r) ? gv[i] * ex2_approx(a_l2 * (S - s_S[s])) * s_delta[s]
                                         : 0.f;
                        m[i] = v;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        m[i] = 0.f;
                }
                const uint32_t slab = uint32_t(q >> 2) * 16384u;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int col = (q & 3) * 16 + h2 * 8;
                    uint4 pk;
                    pk.x = ssd_pack2(m[h2 * 8 + 0], m[h2 * 8 + 1]);
                    pk.y = ssd_pack2(m[h2 * 8 + 2], m[h2 * 8 + 3]);
                    pk.z = ssd_pack2(m[h2 * 8 + 4], m[h2 * 8 + 5]);
                    pk.w = ssd_pack2(m[h2 * 8 + 6], m[h2 * 8 + 7]);
                    *reinterpret_cast<uint4 *>(mrow + slab + sw128_offset(r, col)) = pk;
                }
            }
        }
        fence_proxy_async_smem();
        tmem_fence_before_sync();
        __syncthreads();
        // ---- Yd = M x^T, h += B (x w)^T, then the next chunk's C^T B
        if (tid == 0) {
            tmem_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < Q / 16; ++kk)
                umma_bf16(tb + kColYd, umma_desc_kmajor(aM, 128, kk), umma_desc_kmajor(aX, P, kk),
                          idYd, kk > 0);
#pragma unroll
            for (int kk = 0; kk < Q / 16; ++kk)
                umma_bf16(tb + kColH, umma_desc_kmajor(aB, N, kk), umma_desc_kmajor(aXw, P, kk),
                          idYd, 1u);
            umma_commit(&bar_mma);
            if (c + 1 < p.nchunks) {
                ok = mbar_wait(&bar_tma[buf ^ 1], uint32_t(((c + 1) >> 1) & 1), p.timeout_ns) && ok;
                tmem_fence_after_sync();
                issue_G(c + 1);
            }
        }
        ok = mbar_wait(&bar_yo, ph, p.timeout_ns) && ok;
        ok = mbar_wait(&bar_mma, ph, p.timeout_ns) && ok;
        tmem_fence_after_sync();
        // ---- outputs of token t = r, columns p of this half
        {
            const uint8_t *xs = smem + Lay::kX + buf * 16384;
            const uint32_t slab = uint32_t(r >> 6) * 8192u;
            __nv_bfloat16 *yrow = p.y + int64_t(b) * p.y_bs + int64_t(hh * P) * p.y_cs + t0 + r;
            const __nv_bfloat16 *zrow =
                GATE ? p.z + int64_t(b) * p.z_bs + int64_t(hh * P) * p.z_cs + t0 + r : nullptr;
#pragma unroll
            for (int cc = 0; cc < 32; cc += 16) {
                float yd[16], yo[16];
                tmem_ld16(tb + lane_off + kColYd + colh + cc, yd);
                tmem_ld16(tb + lane_off + kColYo + colh + cc, yo);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int pp = half * 32 + cc + i;
                    const float xv = __bfloat162float(
                        *reinterpret_cast<const __nv_bfloat16 *>(xs + slab + sw128_offset(pp, r & 63)));
                    float v = fmaf(e_row, yo[i], yd[i]);
                    v = fmaf(dsk, xv, v);
                    if (GATE && valid) {
                        const float zv = __bfloat162float(zrow[int64_t(pp) * p.z_cs]);
                        v *= zv / (1.f + __expf(-zv));
                    }
                    if (valid)
                        yrow[int64_t(pp) * p.y_cs] = __float2bfloat16_rn(v);
                }
            }
            // h (state n = r) -> bf16 copy for the next chunk's Yo; final state out
            uint8_t *hs = smem + Lay::kHs;
            float *ls = (p.last_state && c == p.nchunks - 1)
                            ? p.last_state + (int64_t(b) * p.H + hh) * P * N + r
                            : nullptr;
#pragma unroll
            for (int cc = 0; cc < 32; cc += 16) {
                float hv[16];
                tmem_ld16(tb + lane_off + kColH + colh + cc, hv);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint4 pk;
                    pk.x = ssd_pack2(hv[h2 * 8 + 0], hv[h2 * 8 + 1]);
                    pk.y = ssd_pack2(hv[h2 * 8 + 2], hv[h2 * 8 + 3]);
                    pk.z = ssd_pack2(hv[h2 * 8 + 4], hv[h2 * 8 + 5]);
                    pk.w = ssd_pack2(hv[h2 * 8 + 6], hv[h2 * 8 + 7]);
                    *reinterpret_cast<uint4 *>(hs + sw128_offset(r, colh + cc + h2 * 8)) = pk;
                }
                if (ls) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        ls[int64_t(colh + cc + i) * N] = hv[i];
                }
            }
        }
        fence_proxy_async_smem();
        tmem_fence_before_sync();
        __syncthreads();
        // this chunk's C, B, x buffers are free: bring in chunk c + 2
        if (tid == 0 && c + 2 < p.nchunks) {
            fence_proxy_async_smem();
            issue_loads(c + 2);
        }
    }
    if (!ok)
        atomicOr(p.err, 4u);
    tmem_fence_after_sync();
    if (warp == 0)
        tmem_dealloc(tb, kSsdTmemCols);
}

}  // namespace selscan
