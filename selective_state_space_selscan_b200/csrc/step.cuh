// step.cuh -- one decode step of the selective scan, state updated in place.
//
// "03 -- Modelos de espacio de estados: RWKV, S4, Mamba y el selective
// scan", section "Coste de inferencia": at decode time the layer does
// constant work per token, h_t = Abar_t h_{t-1} + Bbar_t x_t and
// y_t = C_t h_t, over a fixed-size state (no cache that grows with the
// context).  "Mamba-3: un modelo de espacio de estados centrado en la
// inferencia" (first section): with a scalar transition this update moves
// far more bytes than it computes, so the kernel is written for HBM.
//
// Work split.  A channel (b, c) owns N fp32 states, contiguous in `state`.
// TPC = N / 8 consecutive threads share a channel; thread k holds the
// 16-byte vectors k and k + TPC of the channel's state, so each of the two
// vector loads (and stores) covers whole 32-byte sectors, and every thread
// keeps two loads in flight.  y = sum_n C_n h_n is a butterfly over the TPC
// lanes.  Grid: x over the channels of a row (of one head, in the scalar
// form), y over heads, z over batch rows, so no thread divides an index.
// Per channel the kernel moves 8 N bytes of state plus four scalars; A
// (diagonal form), B and C are shared across channels and come from L2.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "scan_diag.cuh"

namespace selscan {

struct StepParams {
    int dim;            // channels per row: D, or H * headdim
    int headdim;        // channels per head (scalar form); 1 for the diagonal form
    int units;          // D (diagonal) or H (scalar): owners of A, bias, D
    int per_group;      // units per group of B / C
    int bc_vec;         // B and C rows are contiguous and 4-element aligned
    const void *u;      // (batch, dim), element strides su0, su1
    int64_t su0, su1;
    const void *delta;  // diagonal: (batch, D) like u; scalar: (batch, H) fp32
    int64_t sd0, sd1;
    const void *z;      // (batch, dim) like u, or null
    int64_t sz0, sz1;
    void *y;            // (batch, dim) like u
    int64_t sy0, sy1;
    const void *B;      // (batch, G, N) like u
    int64_t sb0, sb1, sb2;
    const void *C;
    int64_t sc0, sc1, sc2;
    const float *A;           // (D, N) contiguous, or (H)
    const float *delta_bias;  // (units) or null
    const float *Dskip;       // (units) or null
    float *state;             // (batch, dim, N) contiguous, updated in place
    int softplus;
};

__device__ __forceinline__ float step_load(const void *base, int64_t off, const float *)
{
    return static_cast<const float *>(base)[off];
}

__device__ __forceinline__ float step_load(const void *base, int64_t off,
                                           const __nv_bfloat16 *)
{
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(base)[off]);
}

__device__ __forceinline__ void step_store(void *base, int64_t off, float v, const float *)
{
    static_cast<float *>(base)[off] = v;
}

__device__ __forceinline__ void step_store(void *base, int64_t off, float v,
                                           const __nv_bfloat16 *)
{
    static_cast<__nv_bfloat16 *>(base)[off] = __float2bfloat16_rn(v);
}

// Four consecutive elements of a B or C row starting at element `off`.
__device__ __forceinline__ void step_load4(const void *base, int64_t off, int64_t stride,
                                           bool vec, float (&v)[4], const float *)
{
    const float *p = static_cast<const float *>(base) + off;
    if (vec) {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            v[i] = p[i * stride];
    }
}

__device__ __forceinline__ void step_load4(const void *base, int64_t off, int64_t stride,
                                           bool vec, float (&v)[4], const __nv_bfloat16 *)
{
    const __nv_bfloat16 *p = static_cast<const __nv_bfloat16 *>(base) + off;
    if (vec) {
        const uint2 q = *reinterpret_cast<const uint2 *>(p);
        v[0] = __uint_as_float(q.x << 16);
        v[1] = __uint_as_float(q.x & 0xffff0000u);
        v[2] = __uint_as_float(q.y << 16);
        v[3] = __uint_as_float(q.y & 0xffff0000u);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            v[i] = __bfloat162float(p[i * stride]);
    }
}

// T: element type of u, z, y, B, C (and of delta in the diagonal form).
// TPC: threads per channel (N / 8).  SCALAR: Mamba-2 form.  The fp32
// instances use the accurate exp / log1p; the bf16 ones the special-function
// unit (its error is far below bf16 rounding).
template <typename T, int TPC, bool SCALAR>
__global__ void __launch_bounds__(256, SCALAR ? 8 : 6) step_kernel(StepParams p)
{
    constexpr int V = 2;  // 16-byte state vectors per thread
    constexpr int N = 4 * V * TPC;
    constexpr bool kFast = !std::is_same<T, float>::value;
    const T *tag = nullptr;
    const int inner = int(blockIdx.x) * 256 + int(threadIdx.x);
    const int cl = inner / TPC;  // channel within the row (head)
    const int k = inner % TPC;
    const int b = int(blockIdx.z);
    const int unit = SCALAR ? int(blockIdx.y) : cl;
    const int c = SCALAR ? unit * p.headdim + cl : cl;
    // TPC divides 32, so a channel's lanes are all live or all past the end
    // and the butterfly below stays inside one channel.
    const bool live = cl < (SCALAR ? p.headdim : p.dim);

    float acc = 0.f, x = 0.f;
    if (live) {
        const int g = p.per_group == p.units ? 0 : unit / p.per_group;
        const int64_t ch = int64_t(b) * p.dim + c;
        float4 *sp = reinterpret_cast<float4 *>(p.state + ch * N);
        float4 h[V];
#pragma unroll
        for (int v = 0; v < V; ++v)
            h[v] = __ldcs(sp + k + v * TPC);
        float dt = SCALAR ? static_cast<const float *>(p.delta)[b * p.sd0 + unit * p.sd1]
                          : step_load(p.delta, b * p.sd0 + unit * p.sd1, tag);
        x = step_load(p.u, b * p.su0 + c * p.su1, tag);
        if (p.delta_bias)
            dt += p.delta_bias[unit];
        if (p.softplus)
            dt = kFast ? softplus_fast(dt) : softplus_exact(dt);
        const float dx = dt * x;
        float rs = 0.f;
        if (SCALAR)
            rs = kFast ? ex2_approx(dt * p.A[unit] * kLog2e) : expf(dt * p.A[unit]);
        const int64_t bo = int64_t(b) * p.sb0 + int64_t(g) * p.sb1;
        const int64_t co = int64_t(b) * p.sc0 + int64_t(g) * p.sc1;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int q = k + v * TPC;  // 16-byte vector index within the channel
            float a[4];
            if (SCALAR) {
                a[0] = a[1] = a[2] = a[3] = rs;
            } else {
                const float4 av = reinterpret_cast<const float4 *>(p.A + int64_t(unit) * N)[q];
                const float e[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    a[i] = kFast ? ex2_approx(dt * e[i] * kLog2e) : expf(dt * e[i]);
            }
            float Bv[4], Cv[4];
            step_load4(p.B, bo + int64_t(4 * q) * p.sb2, p.sb2, p.bc_vec, Bv, tag);
            step_load4(p.C, co + int64_t(4 * q) * p.sc2, p.sc2, p.bc_vec, Cv, tag);
            h[v].x = fmaf(a[0], h[v].x, dx * Bv[0]);
            h[v].y = fmaf(a[1], h[v].y, dx * Bv[1]);
            h[v].z = fmaf(a[2], h[v].z, dx * Bv[2]);
            h[v].w = fmaf(a[3], h[v].w, dx * Bv[3]);
            __stcs(sp + q, h[v]);
            acc = fmaf(Cv[0], h[v].x, acc);
            acc = fmaf(Cv[1], h[v].y, acc);
            acc = fmaf(Cv[2], h[v].z, acc);
            acc = fmaf(Cv[3], h[v].w, acc);
        }
    }
#pragma unroll
    for (int off = TPC / 2; off > 0; off >>= 1)
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (live && k == 0) {
        float out = acc + (p.Dskip ? p.Dskip[unit] * x : 0.f);
        if (p.z) {
            const float zv = step_load(p.z, b * p.sz0 + c * p.sz1, tag);
            out *= kFast ? silu_fast(zv) : silu_exact(zv);
        }
        step_store(p.y, b * p.sy0 + c * p.sy1, out, tag);
    }
}

}  // namespace selscan
