// scan_diag.cuh -- diagonal-A selective scan (S6) forward for sm_100a.
//
// What it computes: for each (batch b, channel d) and token t
//   delta_t = softplus(Delta + bias)      h_t = exp(delta_t A) h_{t-1} + delta_t B_t u_t
//   y_t     = (C_t . h_t + D u_t) * silu(z_t)
// ("03 -- Modelos de espacio de estados", sections "El mecanismo selectivo
// de Mamba", "Discretizacion", "Parallel scan"; "P20 -- Mamba", section 5).
//
// Design (B200):
//  * Work unit = (tile of CH channels of one batch row, time segment).  A
//    persistent grid takes units from an atomic ticket in segment-major
//    order, so the unit a ticket depends on (same tile, previous segment)
//    was always handed out earlier: every wait eventually ends.
//  * One producer warp streams each unit's inputs chunk by chunk with bulk
//    tensor copies (TMA, 128-byte swizzle, no multicast) into a ring of
//    STAGES shared-memory stages guarded by full/empty mbarriers.
//  * Consumer threads come in lane pairs: one channel per pair, 8 of the 16
//    states per lane, all in registers.  The expanded state never leaves the
//    SM ("P20 -- Mamba", section 3).  Per-token work that does not depend on
//    the state index (softplus, delta*u, the decay base, the gate) is split
//    between the two lanes and exchanged with warp shuffles; partial outputs
//    are reduce-scattered the same way.
//  * Segments are linked by their carry: the last chunk of a unit publishes
//    the channel states (fp32) and a gpu-scope release flag; the first chunk
//    of the next segment acquires it.  This is the associative carry of the
//    "Parallel scan" section applied across segments.
//  * Output tiles go back through shared memory with TMA stores.
//  * When A has the S4D-real structure A[d,n] = (n+1) A[d,0] (checked per
//    channel, bit-exactly, inside the kernel), exp(delta A[d,n]) = r^(n+1)
//    with r = exp(delta A[d,0]): one exponential per token instead of 16.
//    Other A take the general path (one exponential per state).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace selscan {

constexpr int kDiagN = 16;   // states per channel
constexpr int kDiagSPT = 8;  // states held by one lane

struct DiagParams {
    int batch, dim, L;
    int tiles_per_batch;  // ceil(dim / CH)
    int num_tiles;        // batch * tiles_per_batch
    int seg_len;          // tokens per segment (multiple of the chunk)
    int num_segs;
    int total_units;      // num_tiles * num_segs
    const float *A;       // (dim, 16)
    const float *delta_bias;  // (dim) or null
    const float *Dskip;   // (dim) or null
    const float *h0;      // (batch, dim, 16) or null
    float *agg;           // two-pass form: [units][CH][parity][8] segment end states
    float *agg_sd;        // two-pass form: [units][CH] sums of step sizes
    float *last_state;    // (batch, dim, 16) or null
    int softplus;
    unsigned int *ticket;  // zeroed before launch
    unsigned int *flags;   // [total_units][consumer warps], zeroed
    float *carry;          // [total_units][CH][16]
    unsigned long long timeout_ns;
    unsigned int *err;     // device error word
    int dbg_skip_publish;  // unit whose carry flag is withheld (-1: none)
};

constexpr unsigned int kErrTimeoutPipe = 1u;
constexpr unsigned int kErrTimeoutCarry = 2u;

template <typename T>
struct DiagShape {
    static constexpr int kChunk = 128 / int(sizeof(T));  // tokens per stage
    static constexpr int kVec = 16 / int(sizeof(T));     // tokens per 16 B
    static constexpr int kHalf = kVec / 2;               // tokens per lane
};

__device__ __forceinline__ void unpack_half(uint2 v, float (&f)[4],
                                            const __nv_bfloat16 *)
{
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xffff0000u);
}

__device__ __forceinline__ void unpack_half(uint2 v, float (&f)[2], const float *)
{
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
}

__device__ __forceinline__ uint2 pack_half(const float (&f)[4], const __nv_bfloat16 *)
{
    __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
    return make_uint2(*reinterpret_cast<uint32_t *>(&a),
                      *reinterpret_cast<uint32_t *>(&b));
}

__device__ __forceinline__ uint2 pack_half(const float (&f)[2], const float *)
{
    return make_uint2(__float_as_uint(f[0]), __float_as_uint(f[1]));
}

__device__ __forceinline__ float load_elem(const uint8_t *p, const __nv_bfloat16 *)
{
    return __uint_as_float(uint32_t(*reinterpret_cast<const uint16_t *>(p)) << 16);
}

__device__ __forceinline__ float load_elem(const uint8_t *p, const float *)
{
    return *reinterpret_cast<const float *>(p);
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// softplus with the fast special-function unit (bf16 instances).  For
// exp(x) < 2^-6 the Taylor series of log1p keeps the small step sizes
// accurate (lg2.approx loses relative accuracy right next to 1).
__device__ __forceinline__ float softplus_fast(float x)
{
    const float e = ex2_approx(x * kLog2e);
    const float series = e * (1.f - e * (0.5f - e * (1.f / 3.f - 0.25f * e)));
    const float viaLog = kLn2 * lg2_approx(1.f + e);
    const float r = e < 0.015625f ? series : viaLog;
    return x > 20.f ? x : r;
}

__device__ __forceinline__ float softplus_exact(float x)
{
    return x > 20.f ? x + log1pf(expf(-x)) : log1pf(expf(x));
}

// exp(x) for the fp32 decay factors.  For small |x| (x is delta * A, often
// -1e-3) the factor sits just below 1, and a long product of them is only as
// good as the rounding of each: 1 + expm1f(x) is the correctly rounded value
// up to one unbiased rounding, so products over thousands of tokens do not
// drift.  Larger |x| take expf.
__device__ __forceinline__ float exp_decay(float x)
{
    return fabsf(x) < 0.5f ? 1.f + expm1f(x) : expf(x);
}

__device__ __forceinline__ float silu_fast(float v)
{
    return v * rcp_approx(1.f + ex2_approx(-v * kLog2e));
}

__device__ __forceinline__ float silu_exact(float v)
{
    return v / (1.f + expf(-v));
}

template <typename T, int CH, int STAGES, bool GATE>
struct DiagLayout {
    static constexpr int kChunk = DiagShape<T>::kChunk;
    static constexpr int kTile = CH * 128;             // one input tile
    static constexpr int kBCTile = kDiagN * 128;       // B or C tile
    static constexpr int kStage = (2 + (GATE ? 1 : 0)) * kTile + 2 * kBCTile;
    static constexpr int kStagesOff = 0;
    static constexpr int kBCOff = STAGES * kStage;                 // fp32 [2][chunk][32]
    static constexpr int kYOff = kBCOff + 2 * kChunk * 32 * 4;     // [2][tile]
    static constexpr int kBarOff = kYOff + 2 * kTile;
    static constexpr int kInfoOff = kBarOff + 2 * STAGES * 8;
    static constexpr int kAbortOff = kInfoOff + STAGES * 16;
    static constexpr int kBytes = kAbortOff + 16;
    static constexpr int kAlloc = kBytes + 1024;  // room to align the base
};

// Per-stage descriptor written by the producer before the stage's loads.
// x = unit (ticket), y = first token, z = flags.
constexpr int kInfoFirst = 1, kInfoLast = 2, kInfoEnd = 4;

template <typename T, bool POW, bool GATE, int CH>
__device__ __forceinline__ void diag_chunk_compute(
    const uint8_t *u_row, const uint8_t *dl_row, const uint8_t *z_row,
    const float *bcb, uint8_t *y_row, int swz, int pp, int t0, int L,
    float bias, float a0, const float (&a)[kDiagSPT], float dsk, int softplus,
    float (&h)[kDiagSPT])
{
    constexpr int VB = DiagShape<T>::kVec;
    constexpr int HV = DiagShape<T>::kHalf;
    constexpr int TC = DiagShape<T>::kChunk;
    constexpr bool kFast = sizeof(T) == 2;
    const T *tag = nullptr;

#pragma unroll 1
    for (int j = 0; j < TC / VB; ++j) {
        const int off = ((j ^ swz) << 4) + pp * 8;
        float uv[HV], dv[HV], zv[HV];
        unpack_half(*reinterpret_cast<const uint2 *>(u_row + off), uv, tag);
        unpack_half(*reinterpret_cast<const uint2 *>(dl_row + off), dv, tag);
        if (GATE)
            unpack_half(*reinterpret_cast<const uint2 *>(z_row + off), zv, tag);

        // token-wise prologue for this lane's half of the 16-byte block
        float w_own[HV], q_own[HV];
#pragma unroll
        for (int i = 0; i < HV; ++i) {
            const int t = t0 + j * VB + pp * HV + i;
            const float x = dv[i] + bias;
            float dt = softplus ? (kFast ? softplus_fast(x) : softplus_exact(x)) : x;
            if (t >= L)
                dt = 0.f;  // padding past the end: identity step
            w_own[i] = dt * uv[i];
            q_own[i] = POW ? ex2_approx(dt * a0) : dt;
        }
        float w_all[VB], q_all[VB];
#pragma unroll
        for (int i = 0; i < HV; ++i) {
            const float wo = __shfl_xor_sync(0xffffffffu, w_own[i], 1);
            const float qo = __shfl_xor_sync(0xffffffffu, q_own[i], 1);
            w_all[i] = pp ? wo : w_own[i];
            w_all[HV + i] = pp ? w_own[i] : wo;
            q_all[i] = pp ? qo : q_own[i];
            q_all[HV + i] = pp ? q_own[i] : qo;
        }

        float yp[VB];
#pragma unroll
        for (int i = 0; i < VB; ++i) {
            const float4 *bcp =
                reinterpret_cast<const float4 *>(bcb + (j * VB + i) * 32 + pp * 16);
            const float4 b0 = bcp[0], b1 = bcp[1], c0 = bcp[2], c1 = bcp[3];
            const float Bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            const float Cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            float dA[8];
            if (POW) {
                const float r = q_all[i];
                const float r2 = r * r, r4 = r2 * r2, r8 = r4 * r4;
                const float base = pp ? r8 * r : r;
                dA[0] = base;
                dA[1] = base * r;
                dA[2] = base * r2;
                dA[3] = dA[1] * r2;
                dA[4] = base * r4;
                dA[5] = dA[1] * r4;
                dA[6] = dA[2] * r4;
                dA[7] = dA[3] * r4;
            } else {
#pragma unroll
                for (int n = 0; n < 8; ++n)
                    dA[n] = kFast ? ex2_approx(q_all[i] * a[n]) : exp_decay(q_all[i] * a[n]);
            }
            float acc = 0.f;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                h[n] = fmaf(dA[n], h[n], w_all[i] * Bv[n]);
                acc = fmaf(Cv[n], h[n], acc);
            }
            yp[i] = acc;
        }

        // reduce-scatter: this lane finishes tokens pp*HV .. pp*HV+HV-1
        float yo[HV];
#pragma unroll
        for (int i = 0; i < HV; ++i) {
            const float send = pp ? yp[i] : yp[HV + i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
            float v = (pp ? yp[HV + i] : yp[i]) + recv;
            v = fmaf(dsk, uv[i], v);
            if (GATE)
                v *= kFast ? silu_fast(zv[i]) : silu_exact(zv[i]);
            yo[i] = v;
        }
        *reinterpret_cast<uint2 *>(y_row + off) = pack_half(yo, tag);
    }
}

template <typename T, int CH, int STAGES, bool GATE>
__global__ void __launch_bounds__(CH * 2 + 32, 1)
scan_diag_kernel(const __grid_constant__ CUtensorMap tm_u,
                 const __grid_constant__ CUtensorMap tm_delta,
                 const __grid_constant__ CUtensorMap tm_z,
                 const __grid_constant__ CUtensorMap tm_B,
                 const __grid_constant__ CUtensorMap tm_C,
                 const __grid_constant__ CUtensorMap tm_y,
                 const DiagParams p)
{
    using Lay = DiagLayout<T, CH, STAGES, GATE>;
    constexpr int TC = DiagShape<T>::kChunk;
    constexpr int CONS = CH * 2;
    constexpr int CW = CONS / 32;
    constexpr int TILE = Lay::kTile;
    constexpr bool kFast = sizeof(T) == 2;
    static_assert(CONS % 32 == 0, "consumer threads must fill warps");

    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, offset from the shared array itself so that
    // every pointer derived from it stays in the shared address space
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t *stages = smem + Lay::kStagesOff;
    float *bc = reinterpret_cast<float *>(smem + Lay::kBCOff);
    uint8_t *ytile = smem + Lay::kYOff;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Lay::kBarOff);
    uint64_t *empty = full + STAGES;
    int4 *info = reinterpret_cast<int4 *>(smem + Lay::kInfoOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::kAbortOff);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CW);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int G = p.num_tiles;

    if (warp == CW) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_u);
            prefetch_tmap(&tm_delta);
            if (GATE)
                prefetch_tmap(&tm_z);
            prefetch_tmap(&tm_B);
            prefetch_tmap(&tm_C);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            while (ok) {
                const unsigned int tk = atomicAdd(p.ticket, 1u);
                if (tk >= unsigned(p.total_units))
                    break;
                const int k = int(tk) / G, g = int(tk) - k * G;
                const int b = g / p.tiles_per_batch;
                const int d0 = (g - b * p.tiles_per_batch) * CH;
                const int tb = k * p.seg_len;
                const int te = min(p.L, tb + p.seg_len);
                const int nch = (te - tb + TC - 1) / TC;
                for (int c = 0; c < nch; ++c) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const int t0 = tb + c * TC;
                    info[s] = make_int4(int(tk), t0,
                                        (c == 0 ? kInfoFirst : 0) |
                                            (c == nch - 1 ? kInfoLast : 0),
                                        0);
                    uint8_t *st = stages + s * Lay::kStage;
                    mbar_arrive_expect_tx(&full[s], Lay::kStage);
                    tma_load_3d(st, &tm_u, &full[s], t0, d0, b);
                    tma_load_3d(st + TILE, &tm_delta, &full[s], t0, d0, b);
                    if (GATE)
                        tma_load_3d(st + 2 * TILE, &tm_z, &full[s], t0, d0, b);
                    uint8_t *bct = st + (GATE ? 3 : 2) * TILE;
                    tma_load_3d(bct, &tm_B, &full[s], t0, 0, b);
                    tma_load_3d(bct + Lay::kBCTile, &tm_C, &full[s], t0, 0, b);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (ok && mbar_wait(&empty[s], ph ^ 1u, p.timeout_ns)) {
                info[s] = make_int4(-1, 0, kInfoEnd, 0);
                mbar_arrive(&full[s]);
            } else {
                atomicOr(p.err, kErrTimeoutPipe);
                *abort_flag = 1;
                __nanosleep(100000);  // let copies already issued land
            }
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    const int c = tid >> 1;   // channel within the tile
    const int pp = tid & 1;   // which half of the 16 states
    const int swz = c & 7;    // 128-byte swizzle phase of this row
    float h[kDiagSPT];
#pragma unroll
    for (int n = 0; n < kDiagSPT; ++n)
        h[n] = 0.f;
    float a[kDiagSPT];
    float a0 = 0.f, bias = 0.f, dsk = 0.f;
    bool pow_path = false;
    int unit = -1, k = 0, b = 0, d0 = 0, d = 0;
    int prev_t0 = 0, prev_d0 = 0, prev_b = 0;
    int s = 0, it = 0;
    uint32_t ph = 0;

    for (;;) {
        const bool arrived = mbar_wait(&full[s], ph, p.timeout_ns) && !*abort_flag;
        int4 inf = make_int4(-1, 0, 0, 0);
        if (arrived) {
            inf = info[s];  // ordered after the barrier wait (acquire)
            if (inf.z & kInfoEnd)
                break;  // every consumer reads the same marker
        }

        if (arrived && (inf.z & kInfoFirst)) {
            unit = inf.x;
            k = unit / G;
            const int g = unit - k * G;
            b = g / p.tiles_per_batch;
            d0 = (g - b * p.tiles_per_batch) * CH;
            d = d0 + c;
            const bool live = d < p.dim;
            const float *arow = p.A + size_t(live ? d : 0) * kDiagN;
            const float A0 = arow[0];
            bool ok = true;
#pragma unroll
            for (int n = 0; n < kDiagSPT; ++n) {
                const float an = arow[pp * kDiagSPT + n];
                ok = ok && (an == float(pp * kDiagSPT + n + 1) * A0);
                a[n] = kFast ? an * kLog2e : an;
            }
            a0 = A0 * kLog2e;
            pow_path = kFast && __all_sync(0xffffffffu, ok);
            bias = (p.delta_bias && live) ? p.delta_bias[d] : 0.f;
            dsk = (p.Dskip && live) ? p.Dskip[d] : 0.f;
            if (k == 0) {
#pragma unroll
                for (int n = 0; n < kDiagSPT; ++n)
                    h[n] = (p.h0 && live)
                               ? p.h0[(size_t(b) * p.dim + d) * kDiagN + pp * kDiagSPT + n]
                               : 0.f;
            } else {
                const int prev = unit - G;
                const uint32_t *flag = p.flags + size_t(prev) * CW + warp;
                bool got = true;
                if (lane == 0)
                    got = spin_flag(flag, 1u, p.timeout_ns);
                got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
                if (!got) {
                    if (lane == 0)
                        atomicOr(p.err, kErrTimeoutCarry);
#pragma unroll
                    for (int n = 0; n < kDiagSPT; ++n)
                        h[n] = 0.f;
                } else {
                    (void)ld_acquire_gpu(flag);
                    const float4 *src = reinterpret_cast<const float4 *>(
                        p.carry + (size_t(prev) * CH + c) * kDiagN + pp * kDiagSPT);
                    const float4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
                    h[0] = x0.x; h[1] = x0.y; h[2] = x0.z; h[3] = x0.w;
                    h[4] = x1.x; h[5] = x1.y; h[6] = x1.z; h[7] = x1.w;
                }
            }
        }

        uint8_t *st = stages + s * Lay::kStage;
        const uint8_t *Bt = st + (GATE ? 3 : 2) * TILE;
        const uint8_t *Ct = Bt + Lay::kBCTile;
        float *bcb = bc + (it & 1) * TC * 32;
        // B, C of this chunk -> fp32, token-major [t][B0..7 C0..7 B8..15 C8..15]
        for (int idx = tid; arrived && idx < TC * 32; idx += CONS) {
            const int t = idx >> 5, q = idx & 31;
            const int w16 = q & 15;
            const int n = (q >> 4) * 8 + (w16 & 7);
            const int byte = t * int(sizeof(T));
            const uint8_t *src = (w16 < 8 ? Bt : Ct) + n * 128 +
                                 ((((byte >> 4) ^ (n & 7))) << 4) + (byte & 15);
            bcb[idx] = load_elem(src, static_cast<const T *>(nullptr));
        }
        if (tid == 0)
            bulk_wait_read<0>();  // y tile (it & 1) free again
        // all consumers leave together if any of them timed out
        if (named_bar_any(1, CONS, !arrived)) {
            if (tid == 0)
                atomicOr(p.err, kErrTimeoutPipe);
            *abort_flag = 1;
            break;
        }
        if (tid == 0 && it > 0) {
            tma_store_3d(&tm_y, ytile + ((it - 1) & 1) * TILE, prev_t0, prev_d0, prev_b);
            bulk_commit();
        }

        const uint8_t *u_row = st + c * 128;
        const uint8_t *dl_row = st + TILE + c * 128;
        const uint8_t *z_row = st + 2 * TILE + c * 128;
        uint8_t *y_row = ytile + (it & 1) * TILE + c * 128;
        if (pow_path)
            diag_chunk_compute<T, true, GATE, CH>(u_row, dl_row, z_row, bcb, y_row, swz,
                                                  pp, inf.y, p.L, bias, a0, a, dsk,
                                                  p.softplus, h);
        else
            diag_chunk_compute<T, false, GATE, CH>(u_row, dl_row, z_row, bcb, y_row, swz,
                                                   pp, inf.y, p.L, bias, a0, a, dsk,
                                                   p.softplus, h);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);

        if (inf.z & kInfoLast) {
            if (k < p.num_segs - 1) {
                float4 *dst = reinterpret_cast<float4 *>(
                    p.carry + (size_t(unit) * CH + c) * kDiagN + pp * kDiagSPT);
                dst[0] = make_float4(h[0], h[1], h[2], h[3]);
                dst[1] = make_float4(h[4], h[5], h[6], h[7]);
                __threadfence();
                __syncwarp();
                if (lane == 0 && unit != p.dbg_skip_publish)
                    st_release_gpu(p.flags + size_t(unit) * CW + warp, 1u);
            } else if (p.last_state && d < p.dim) {
                float4 *dst = reinterpret_cast<float4 *>(
                    p.last_state + (size_t(b) * p.dim + d) * kDiagN + pp * kDiagSPT);
                dst[0] = make_float4(h[0], h[1], h[2], h[3]);
                dst[1] = make_float4(h[4], h[5], h[6], h[7]);
            }
        }
        prev_t0 = inf.y;
        prev_d0 = d0;
        prev_b = b;
        ++it;
        if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
        }
    }

    // flush the last output tile
    named_bar_sync(1, CONS);
    if (tid == 0) {
        if (it > 0 && !*abort_flag) {
            tma_store_3d(&tm_y, ytile + ((it - 1) & 1) * TILE, prev_t0, prev_d0, prev_b);
            bulk_commit();
        }
        bulk_wait_all<0>();
    }
}

}  // namespace selscan
