// bwd_diag.cuh -- gradients of the diagonal-A selective scan (N = 16).
//
// Training differentiates the same recurrence the forward pass evaluates
// ("03 -- Modelos de espacio de estados", sections "Discretizacion" and
// "Parallel scan"; "P20 -- Mamba", section 5).  With g = dLoss/dh_t walked
// from the last token to the first (starting from the gradient of the final
// state, if any):
//
//   dout = dy silu(z)                  dz   = dy out silu'(z)
//   g   += dout C_t                    dC_t = sum_d dout h_t
//   du   = dout D + sum_n g delta B_t  dB_t = sum_d g delta u
//   ddelta = sum_n g (A abar h_{t-1} + B_t u)       dA += g delta abar h_{t-1}
//   g    = abar g;   dDelta = ddelta * sigmoid(Delta + bias) under softplus
//
// and dh0 = g after the first token.  The expanded states are never stored:
// pass A runs the forward recurrence once and keeps h every kBwdT tokens;
// pass B walks the chunks backwards, recomputes the chunk's states from its
// checkpoint into shared memory and runs the reverse recurrence over them.
//
// Work split: one warp per (batch row, 32 channels), one lane per channel
// holding all 16 states.  dB and dC sum over the channels of a batch row:
// each token's 32 per-lane values are reduced across the warp by a
// butterfly (31 shuffles leave lane i with the sum of value i), then added
// to global memory atomically (one add per lane and token).  dA, dD and the
// bias gradient sum over batch rows and tokens: registers, then atomics.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "scan_diag.cuh"

namespace selscan {

constexpr int kBwdN = 16;  // states per channel
constexpr int kBwdT = 16;  // tokens per checkpoint chunk

struct BwdParams {
    int batch, dim, L, nchunks;
    const void *u, *delta, *z, *dy;  // (batch, dim, L), time stride 1
    int64_t u_bs, u_ds, dl_bs, dl_ds, z_bs, z_ds, dy_bs, dy_ds;
    const void *B, *C;               // (batch, 16, L), time stride 1
    int64_t B_bs, B_ns, C_bs, C_ns;
    const float *A;                  // (dim, 16)
    const float *delta_bias, *Dskip; // (dim) or null
    const float *h0, *dlast;         // (batch, dim, 16) or null
    int softplus;
    void *du, *ddelta, *dz;          // (batch, dim, L) like u; dz null without gate
    int64_t du_bs, du_ds, dd_bs, dd_ds, dz_bs, dz_ds;
    float *dA;                       // (dim, 16), accumulated
    float *dB, *dC;                  // (batch, 16, L) contiguous, accumulated
    float *dD, *dbias;               // (dim) or null, accumulated
    float *dh0;                      // (batch, dim, 16) or null, written
    float *ckpt;                     // [batch][dim][nchunks][16] scratch
};

__device__ __forceinline__ float bwd_ld(const void *p, int64_t off, const float *)
{
    return static_cast<const float *>(p)[off];
}

__device__ __forceinline__ float bwd_ld(const void *p, int64_t off, const __nv_bfloat16 *)
{
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[off]);
}

__device__ __forceinline__ void bwd_st(void *p, int64_t off, float v, const float *)
{
    static_cast<float *>(p)[off] = v;
}

__device__ __forceinline__ void bwd_st(void *p, int64_t off, float v, const __nv_bfloat16 *)
{
    static_cast<__nv_bfloat16 *>(p)[off] = __float2bfloat16_rn(v);
}

// exp(delta * A[n]) for the 16 states: r^(n+1) for S4D-real A
// (A[n] = (n+1) A[0], checked per channel), else one exponential per state.
template <bool FAST>
__device__ __forceinline__ void bwd_decays(float dt, const float (&al)[kBwdN], bool pow_path,
                                           float (&a)[kBwdN])
{
    if (pow_path) {
        const float r = FAST ? ex2_approx(dt * al[0]) : exp2f(dt * al[0]);
        a[0] = r;
#pragma unroll
        for (int n = 1; n < kBwdN; ++n)
            a[n] = a[n - 1] * r;
    } else {
#pragma unroll
        for (int n = 0; n < kBwdN; ++n)
            a[n] = FAST ? ex2_approx(dt * al[n]) : exp2f(dt * al[n]);
    }
}

template <typename T>
__device__ __forceinline__ float bwd_step_size(const BwdParams &p, int64_t row_dl, int t,
                                               float bias, float *raw)
{
    constexpr bool FAST = !std::is_same<T, float>::value;
    const T *tag = nullptr;
    const float x = bwd_ld(p.delta, row_dl + t, tag) + bias;
    *raw = x;
    if (!p.softplus)
        return x;
    return FAST ? softplus_fast(x) : softplus_exact(x);
}

template <typename T>
__global__ void __launch_bounds__(32)
selscan_bwd_kernel(const BwdParams p)
{
    constexpr int N = kBwdN, TC = kBwdT;
    constexpr bool FAST = !std::is_same<T, float>::value;
    const T *tag = nullptr;
    __shared__ float s_h[TC][N][32];  // recomputed states of the chunk, lane-minor

    const int lane = threadIdx.x;
    const int b = blockIdx.y;
    const int d = blockIdx.x * 32 + lane;
    const bool live = d < p.dim;
    const int dd = live ? d : 0;  // dead lanes mirror channel 0 and contribute zeros

    const int64_t row_u = int64_t(b) * p.u_bs + int64_t(dd) * p.u_ds;
    const int64_t row_dl = int64_t(b) * p.dl_bs + int64_t(dd) * p.dl_ds;
    const int64_t row_z = int64_t(b) * p.z_bs + int64_t(dd) * p.z_ds;
    const int64_t row_dy = int64_t(b) * p.dy_bs + int64_t(dd) * p.dy_ds;
    const int64_t row_du = int64_t(b) * p.du_bs + int64_t(dd) * p.du_ds;
    const int64_t row_dd = int64_t(b) * p.dd_bs + int64_t(dd) * p.dd_ds;
    const int64_t row_dz = int64_t(b) * p.dz_bs + int64_t(dd) * p.dz_ds;
    const int64_t bB = int64_t(b) * p.B_bs, bC = int64_t(b) * p.C_bs;
    const float bias = p.delta_bias ? p.delta_bias[dd] : 0.f;
    const float dsk = p.Dskip ? p.Dskip[dd] : 0.f;
    float An[N], al[N];
    bool pow_path = true;
#pragma unroll
    for (int n = 0; n < N; ++n) {
        An[n] = p.A[int64_t(dd) * N + n];
        al[n] = An[n] * kLog2e;
        pow_path = pow_path && (An[n] == float(n + 1) * An[0]);
    }
    float *ck = p.ckpt + (int64_t(b) * p.dim + dd) * p.nchunks * N;

    // ---- pass A: forward recurrence, h at the start of every chunk
    float h[N];
#pragma unroll
    for (int n = 0; n < N; ++n)
        h[n] = (p.h0 && live) ? p.h0[(int64_t(b) * p.dim + dd) * N + n] : 0.f;
    for (int t = 0; t < p.L; ++t) {
        if (t % TC == 0 && live) {
            float4 *dst = reinterpret_cast<float4 *>(ck + (t / TC) * N);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                dst[q] = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        }
        float raw;
        const float dt = bwd_step_size<T>(p, row_dl, t, bias, &raw);
        const float dx = dt * bwd_ld(p.u, row_u + t, tag);
        float a[N];
        bwd_decays<FAST>(dt, al, pow_path, a);
#pragma unroll
        for (int n = 0; n < N; ++n)
            h[n] = fmaf(a[n], h[n], dx * bwd_ld(p.B, bB + int64_t(n) * p.B_ns + t, tag));
    }
    __syncwarp();

    // ---- pass B: chunks backwards
    float g[N], gA[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        g[n] = (p.dlast && live) ? p.dlast[(int64_t(b) * p.dim + dd) * N + n] : 0.f;
        gA[n] = 0.f;
    }
    float gD = 0.f, gbias = 0.f;
    for (int c = p.nchunks - 1; c >= 0; --c) {
        const int t0 = c * TC;
        const int tn = min(TC, p.L - t0);
        float hc[N];  // state before the chunk
        {
            const float4 *src = reinterpret_cast<const float4 *>(ck + c * N);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v = live ? src[q] : make_float4(0.f, 0.f, 0.f, 0.f);
                hc[4 * q] = v.x;
                hc[4 * q + 1] = v.y;
                hc[4 * q + 2] = v.z;
                hc[4 * q + 3] = v.w;
            }
        }
        // recompute the chunk's states
        {
#pragma unroll
            for (int n = 0; n < N; ++n)
                h[n] = hc[n];
            for (int i = 0; i < tn; ++i) {
                const int t = t0 + i;
                float raw;
                const float dt = bwd_step_size<T>(p, row_dl, t, bias, &raw);
                const float dx = dt * bwd_ld(p.u, row_u + t, tag);
                float a[N];
                bwd_decays<FAST>(dt, al, pow_path, a);
#pragma unroll
                for (int n = 0; n < N; ++n) {
                    h[n] = fmaf(a[n], h[n], dx * bwd_ld(p.B, bB + int64_t(n) * p.B_ns + t, tag));
                    s_h[i][n][lane] = h[n];
                }
            }
        }
        __syncwarp();
        // reverse recurrence over the chunk
        for (int i = tn - 1; i >= 0; --i) {
            const int t = t0 + i;
            float raw;
            const float dt = bwd_step_size<T>(p, row_dl, t, bias, &raw);
            const float x = bwd_ld(p.u, row_u + t, tag);
            float a[N];
            bwd_decays<FAST>(dt, al, pow_path, a);
            float Bv[N], Cv[N], ht[N], hp[N];
#pragma unroll
            for (int n = 0; n < N; ++n) {
                Bv[n] = bwd_ld(p.B, bB + int64_t(n) * p.B_ns + t, tag);
                Cv[n] = bwd_ld(p.C, bC + int64_t(n) * p.C_ns + t, tag);
                ht[n] = s_h[i][n][lane];
                hp[n] = i > 0 ? s_h[i - 1][n][lane] : hc[n];
            }
            float out = dsk * x;
#pragma unroll
            for (int n = 0; n < N; ++n)
                out = fmaf(Cv[n], ht[n], out);
            const float dyv = live ? bwd_ld(p.dy, row_dy + t, tag) : 0.f;
            float dout = dyv;
            if (p.z) {
                const float zv = bwd_ld(p.z, row_z + t, tag);
                const float sg = 1.f / (1.f + __expf(-zv));
                if (live)
                    bwd_st(p.dz, row_dz + t, dyv * out * (sg * (1.f + zv * (1.f - sg))), tag);
                dout = dyv * zv * sg;
            }
            float dx = dout * dsk, ddt = 0.f;
            gD = fmaf(dout, x, gD);
            float v[32];  // dB (states 0..15), dC (states 0..15) of this channel
#pragma unroll
            for (int n = 0; n < N; ++n) {
                g[n] = fmaf(dout, Cv[n], g[n]);
                v[N + n] = dout * ht[n];
                v[n] = g[n] * dt * x;
                dx = fmaf(g[n] * dt, Bv[n], dx);
                const float ah = a[n] * hp[n];
                ddt = fmaf(g[n], fmaf(An[n], ah, Bv[n] * x), ddt);
                gA[n] = fmaf(g[n] * dt, ah, gA[n]);
                g[n] *= a[n];
            }
            float dDelta = ddt;
            if (p.softplus)
                dDelta = ddt / (1.f + __expf(-raw));
            gbias += dDelta;
            if (live) {
                bwd_st(p.du, row_du + t, dx, tag);
                bwd_st(p.ddelta, row_dd + t, dDelta, tag);
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k)
                    v[k] = 0.f;  // lanes past the last channel add exact zeros
            }
            // sum the 32 values over the warp's channels: lane i gets value i
#pragma unroll
            for (int lv = 0; lv < 5; ++lv) {
                const int half = 16 >> lv;
                const bool up = (lane & half) != 0;
#pragma unroll
                for (int k = 0; k < half; ++k) {
                    const float send = up ? v[k] : v[k + half];
                    const float keep = up ? v[k + half] : v[k];
                    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, half);
                }
            }
            float *dst = lane < N ? p.dB + (int64_t(b) * N + lane) * p.L + t
                                  : p.dC + (int64_t(b) * N + (lane - N)) * p.L + t;
            atomicAdd(dst, v[0]);
        }
        __syncwarp();
    }
    if (live) {
        if (p.dh0) {
#pragma unroll
            for (int n = 0; n < N; ++n)
                p.dh0[(int64_t(b) * p.dim + d) * N + n] = g[n];
        }
#pragma unroll
        for (int n = 0; n < N; ++n)
            atomicAdd(p.dA + int64_t(d) * N + n, gA[n]);
        if (p.dD)
            atomicAdd(p.dD + d, gD);
        if (p.dbias)
            atomicAdd(p.dbias + d, gbias);
    }
}

}  // namespace selscan
