// scan_diag_bf16.cuh -- fast diagonal-A selective scan for bf16 inputs
// (fp32 state), sm_100a.
//
// Same contract and work decomposition as scan_diag.cuh (persistent grid,
// atomic ticket in segment-major order, one producer warp streaming chunks
// with bulk tensor copies, carries linked by gpu-scope release/acquire
// flags), with an inner loop laid out for the B200 SM:
//
//  * Two consumer lanes per channel (a lane pair), 128 channels per CTA, so
//    that each scheduler runs two consumer warps.  Lane p keeps the states of
//    parity p (n = p, p+2, ..., p+14) in registers and prepares the per-token
//    values (softplus, w = delta*u, the decay base, 1/w) of half of each
//    8-token block; the pair swaps them with warp shuffles, runs the 8 steps,
//    and reduce-scatters the two partial outputs so each lane finishes four
//    tokens (D skip, gate, bf16 store).  B and C of a chunk are staged once
//    per CTA as fp32, token-major, parity-split, so every lane reads its 8 B
//    and 8 C values of a token with four 16-byte broadcast loads.
//  * The state is kept rescaled, g = h / w with w = delta * u, so that the
//    input term needs no multiply:  g_t = (w_{t-1}/w_t) exp(delta_t A) g_{t-1}
//    + B_t and y_t = w_t (C_t . g_t).  |w| is kept >= 2^-64 so that the
//    rescaling stays finite (a zero input then contributes 2^-64 * B, far
//    below fp32 resolution of any non-trivial state).
//  * For S4D-real A (A[d,n] = (n+1) A[d,0], checked per channel at run time)
//    the decays are powers r^(n+1) of r = exp(delta A[d,0]); lane p needs
//    the odd (p=0) or even (p=1) powers, i.e. base * s^j with s = r^2,
//    computed with packed f32x2 multiplies.  Other A use one ex2 per state.
//  * Packed f32x2 FMAs (sm_100) update two states per instruction.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "scan_diag.cuh"
#include "f32x2.cuh"

namespace selscan {

constexpr float kWMin = 5.421010862427522e-20f;  // 2^-64

template <int CH, int STAGES, bool GATE>
struct DiagFastLayout {
    static constexpr int kChunk = 64;                    // tokens per stage
    static constexpr int kTile = CH * 128;               // bf16 [CH][64]
    static constexpr int kBCTile = kDiagN * 128;         // bf16 [16][64]
    static constexpr int kStage = (2 + (GATE ? 1 : 0)) * kTile + 2 * kBCTile;
    static constexpr int kStagesOff = 0;
    static constexpr int kBCPOff = STAGES * kStage;      // fp32 B/C [2][64][128 B]
    static constexpr int kYOff = kBCPOff + 2 * kChunk * 128;
    static constexpr int kBarOff = kYOff + 2 * kTile;
    static constexpr int kInfoOff = kBarOff + 2 * STAGES * 8;
    static constexpr int kAbortOff = kInfoOff + STAGES * 16;
    static constexpr int kBytes = kAbortOff + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

template <bool POW>
__device__ __forceinline__ void decay_pairs(uint64_t (&V)[4], float r, float c, int p,
                                            const uint64_t (&apair)[4])
{
    if (POW) {
        // powers r^(n+1) for n = p, p+2, ..., p+14 : base * s^j, s = r^2
        const float s = r * r;
        const float base = c * (p ? s : r);
        V[0] = pk2(base, base * s);
        const float s2 = s * s;
        const uint64_t S2 = pk2(s2, s2);
        V[1] = mul2(V[0], S2);
        V[2] = mul2(V[1], S2);
        V[3] = mul2(V[2], S2);
    } else {
        // general A: r holds delta; apair holds A*log2(e) of this lane's states
        const uint64_t RR = pk2(r, r), CC = pk2(c, c);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const uint64_t X = mul2(RR, apair[jj]);
            V[jj] = mul2(CC, pk2(ex2_approx(lo2(X)), ex2_approx(hi2(X))));
        }
    }
}

// MODE 0: one pass, segments chained through published carries.
// MODE 1: aggregate pass of the two-pass form: every segment scans from a
//         zero state and records its end state and the sum of its step sizes
//         (reads u, delta and B only; writes no y).
// MODE 2: output pass of the two-pass form: every segment starts from the
//         state folded from the aggregates of the segments before it.
template <int CH, int STAGES, bool GATE, bool SOFTPLUS, int MODE = 0>
__global__ void __launch_bounds__(2 * CH + 32, 1)
scan_diag_bf16_kernel(const __grid_constant__ CUtensorMap tm_u,
                      const __grid_constant__ CUtensorMap tm_delta,
                      const __grid_constant__ CUtensorMap tm_z,
                      const __grid_constant__ CUtensorMap tm_B,
                      const __grid_constant__ CUtensorMap tm_C,
                      const __grid_constant__ CUtensorMap tm_y,
                      const DiagParams p)
{
    using Lay = DiagFastLayout<CH, STAGES, GATE>;
    constexpr int TC = Lay::kChunk;
    constexpr int CONS = 2 * CH;  // two consumer lanes per channel
    constexpr int CW = CONS / 32;
    constexpr int TILE = Lay::kTile;
    static_assert(CONS % 32 == 0, "consumer threads must fill warps");

    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, offset from the shared array itself so that
    // every pointer derived from it stays in the shared address space
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t *stages = smem + Lay::kStagesOff;
    float *bcp = reinterpret_cast<float *>(smem + Lay::kBCPOff);
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
            if (MODE != 1)
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
                    mbar_arrive_expect_tx(&full[s], MODE == 1 ? 2 * TILE + Lay::kBCTile
                                                              : Lay::kStage);
                    tma_load_3d(st, &tm_u, &full[s], t0, d0, b);
                    tma_load_3d(st + TILE, &tm_delta, &full[s], t0, d0, b);
                    if (GATE && MODE != 1)
                        tma_load_3d(st + 2 * TILE, &tm_z, &full[s], t0, d0, b);
                    uint8_t *bct = st + (GATE ? 3 : 2) * TILE;
                    tma_load_3d(bct, &tm_B, &full[s], t0, 0, b);
                    if (MODE != 1)
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
    const int ch = tid >> 1;     // channel within the tile
    const int pp = tid & 1;      // state parity held by this lane; token half it prepares
    const int swz = ch & 7;      // 128-byte swizzle phase of this row
    uint64_t g[4];               // rescaled states n = pp, pp+2, ..., pp+14 (pairs)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
        g[jj] = pk2(0.f, 0.f);
    uint64_t apair[4];           // A*log2e of this lane's states, paired (general path)
    float a0 = 0.f, bias = 0.f, dsk = 0.f, wprev = 1.f;
    float sdel = 0.f;            // this lane's sum of step sizes in the segment (MODE 1)
    bool pow_path = true;
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
            const int gg = unit - k * G;
            b = gg / p.tiles_per_batch;
            d0 = (gg - b * p.tiles_per_batch) * CH;
            d = d0 + ch;
            const bool live = d < p.dim;
            const float *arow = p.A + size_t(live ? d : 0) * kDiagN;
            const float A0 = arow[0];
            bool ok = true;
            float al[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int n = 2 * j + pp;  // this lane's states
                const float an = arow[n];
                ok = ok && (an == float(n + 1) * A0);
                al[j] = an * kLog2e;
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                apair[jj] = pk2(al[2 * jj], al[2 * jj + 1]);
            a0 = A0 * kLog2e;
            pow_path = __all_sync(0xffffffffu, ok);
            bias = (p.delta_bias && live) ? p.delta_bias[d] : 0.f;
            dsk = (p.Dskip && live) ? p.Dskip[d] : 0.f;
            wprev = 1.f;  // g starts as h_in (w_{-1} := 1)
            sdel = 0.f;
            float hv[8];
            if (MODE == 1) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    hv[j] = 0.f;
            } else if (k == 0 || MODE == 2) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    hv[j] = (p.h0 && live) ? p.h0[(size_t(b) * p.dim + d) * kDiagN + 2 * j + pp]
                                           : 0.f;
                if (MODE == 2) {
                    // h_in = fold over the earlier segments j of this tile:
                    // h = exp(A * sum(delta_j)) h + E_j
                    for (int jseg = 0; jseg < k; ++jseg) {
                        const size_t uj = size_t(jseg) * G + gg;
                        const float sd = __ldcg(p.agg_sd + uj * CH + ch);
                        const float4 *e = reinterpret_cast<const float4 *>(
                            p.agg + (uj * CH + ch) * kDiagN + pp * 8);
                        const float4 e0 = __ldcg(e), e1 = __ldcg(e + 1);
                        const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            hv[j] = fmaf(ex2_approx(al[j] * sd), hv[j], ev[j]);
                    }
                }
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
                    for (int j = 0; j < 8; ++j)
                        hv[j] = 0.f;
                } else {
                    (void)ld_acquire_gpu(flag);
                    // carry layout: [unit][channel][parity][8]
                    const float4 *so = reinterpret_cast<const float4 *>(
                        p.carry + (size_t(prev) * CH + ch) * kDiagN + pp * 8);
                    const float4 o0 = __ldcg(so), o1 = __ldcg(so + 1);
                    hv[0] = o0.x; hv[1] = o0.y; hv[2] = o0.z; hv[3] = o0.w;
                    hv[4] = o1.x; hv[5] = o1.y; hv[6] = o1.z; hv[7] = o1.w;
                }
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                g[jj] = pk2(hv[2 * jj], hv[2 * jj + 1]);
        }

        uint8_t *st = stages + s * Lay::kStage;
        const uint8_t *Bt = st + (GATE ? 3 : 2) * TILE;
        const uint8_t *Ct = Bt + Lay::kBCTile;
        float *bcb = bcp + (it & 1) * TC * 32;
        // B, C -> fp32, token-major: [t][parity p][B: X[p], X[p+2], ..., X[p+14]][C: same]
        for (int q2 = tid; arrived && q2 < TC * (MODE == 1 ? 16 : 32); q2 += CONS) {
            // MODE 1 stages B only: (token, parity, k8) -> its slot in the
            // [t][parity][B 8 | C 8] row
            const int q = MODE == 1
                              ? ((q2 >> 4) << 5) + (((q2 >> 3) & 1) << 4) + (q2 & 7)
                              : q2;
            const int t = q >> 5, rest = q & 31;
            const int par = rest >> 4, isC = (rest >> 3) & 1, k8 = rest & 7;
            const int n = 2 * k8 + par;
            const uint8_t *src = isC ? Ct : Bt;
            const int chunk = (t * 2) >> 4, within = (t * 2) & 15;
            const uint16_t v = *reinterpret_cast<const uint16_t *>(
                src + n * 128 + ((chunk ^ (n & 7)) << 4) + within);
            bcb[q] = __uint_as_float(uint32_t(v) << 16);
        }
        if (tid == 0)
            bulk_wait_read<0>();  // y tile (it & 1) free again
        if (named_bar_any(1, CONS, !arrived)) {
            if (tid == 0)
                atomicOr(p.err, kErrTimeoutPipe);
            *abort_flag = 1;
            break;
        }
        if (MODE != 1 && tid == 0 && it > 0) {
            tma_store_3d(&tm_y, ytile + ((it - 1) & 1) * TILE, prev_t0, prev_d0, prev_b);
            bulk_commit();
        }

        const uint8_t *u_row = st + ch * 128;
        const uint8_t *dl_row = st + TILE + ch * 128;
        const uint8_t *z_row = st + 2 * TILE + ch * 128;
        uint8_t *y_row = ytile + (it & 1) * TILE + ch * 128;
        const int t0 = inf.y;

        // The 8-token blocks are software-pipelined: while block j runs its
        // eight steps, the same basic block prepares block j + 1 (softplus,
        // w, 1/w, decay base: special-function latency) and finishes block
        // j - 1 (reduce-scatter, D skip, gate, store), so the latencies of
        // those two phases hide under the step arithmetic.
        auto run = [&](auto pow_tag) {
            constexpr bool POWC = decltype(pow_tag)::value;
            float rv[4], wv[4], rwv[4], uv[4];  // prepared block (this lane's 4 tokens)
            float dts[4];                       // its step sizes (aggregate pass)
            uint2 zq = make_uint2(0, 0);
            auto prep = [&](int jb) {
                const int off = ((jb ^ swz) << 4) + pp * 8;
                const uint2 uq = *reinterpret_cast<const uint2 *>(u_row + off);
                const uint2 dq = *reinterpret_cast<const uint2 *>(dl_row + off);
                if (GATE && MODE != 1)
                    zq = *reinterpret_cast<const uint2 *>(z_row + off);
                const int tmine = t0 + jb * 8 + pp * 4;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t uw = kk < 2 ? uq.x : uq.y, dw = kk < 2 ? dq.x : dq.y;
                    uv[kk] = __uint_as_float((kk & 1) ? (uw & 0xffff0000u) : (uw << 16));
                    const float dv = __uint_as_float((kk & 1) ? (dw & 0xffff0000u) : (dw << 16));
                    const float x = dv + bias;
                    float dt = SOFTPLUS ? softplus_fast(x) : x;
                    dt = (tmine + kk < p.L) ? dt : 0.f;  // padding past L: identity step
                    dts[kk] = dt;
                    const float wr = dt * uv[kk];
                    wv[kk] = copysignf(fmaxf(fabsf(wr), kWMin), wr);
                    rwv[kk] = rcp_approx(wv[kk]);
                    rv[kk] = POWC ? ex2_approx(dt * a0) : dt;
                }
            };
            // finished-block state carried into the next iteration
            float yp_prev[8], w_prev4[4], u_prev4[4];
            uint2 z_prev = make_uint2(0, 0);
            int off_prev = 0;
            auto finish = [&]() {
                // reduce-scatter: this lane finishes tokens 4pp .. 4pp+3
                float yo[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const float send = pp ? yp_prev[kk] : yp_prev[4 + kk];
                    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
                    float v = ((pp ? yp_prev[4 + kk] : yp_prev[kk]) + recv) * w_prev4[kk];
                    v = fmaf(dsk, u_prev4[kk], v);
                    if (GATE) {
                        const uint32_t zw = kk < 2 ? z_prev.x : z_prev.y;
                        const float zv = __uint_as_float((kk & 1) ? (zw & 0xffff0000u) : (zw << 16));
                        v *= silu_fast(zv);
                    }
                    yo[kk] = v;
                }
                *reinterpret_cast<uint2 *>(y_row + off_prev) =
                    make_uint2(pack2_bf16(yo[0], yo[1]), pack2_bf16(yo[2], yo[3]));
            };
            prep(0);
#pragma unroll 2
            for (int j = 0; j < TC / 8; ++j) {
                // both lanes need r, w, 1/w of all 8 tokens of block j
                float r8[8], w8[8], rw8[8];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const float ro = __shfl_xor_sync(0xffffffffu, rv[kk], 1);
                    const float wo = __shfl_xor_sync(0xffffffffu, wv[kk], 1);
                    const float rwo = __shfl_xor_sync(0xffffffffu, rwv[kk], 1);
                    r8[kk] = pp ? ro : rv[kk];
                    r8[4 + kk] = pp ? rv[kk] : ro;
                    w8[kk] = pp ? wo : wv[kk];
                    w8[4 + kk] = pp ? wv[kk] : wo;
                    rw8[kk] = pp ? rwo : rwv[kk];
                    rw8[4 + kk] = pp ? rwv[kk] : rwo;
                }
                float wmine[4], umine[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    wmine[kk] = wv[kk];
                    umine[kk] = uv[kk];
                }
                const uint2 zmine = zq;
                if (MODE == 1)
                    sdel += (dts[0] + dts[1]) + (dts[2] + dts[3]);
                if (MODE != 1 && j > 0)
                    finish();            // block j - 1
                prep((j + 1) & 7);       // block j + 1 (wraps harmlessly after the last)
                float yp[8];
                const float *bcb_blk = bcb + j * 8 * 32 + pp * 16;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float c = (i == 0 ? wprev : w8[i - 1]) * rw8[i];
                    const ulonglong2 *bq = reinterpret_cast<const ulonglong2 *>(bcb_blk + i * 32);
                    const ulonglong2 b01 = bq[0], b23 = bq[1];
                    uint64_t V[4];
                    decay_pairs<POWC>(V, r8[i], c, pp, apair);
                    g[0] = fma2(V[0], g[0], b01.x);
                    g[1] = fma2(V[1], g[1], b01.y);
                    g[2] = fma2(V[2], g[2], b23.x);
                    g[3] = fma2(V[3], g[3], b23.y);
                    if (MODE == 1) {
                        yp[i] = 0.f;
                        continue;
                    }
                    const ulonglong2 c01 = bq[2], c23 = bq[3];
                    uint64_t Ya = mul2(c01.x, g[0]);
                    uint64_t Yb = mul2(c01.y, g[1]);
                    Ya = fma2(c23.x, g[2], Ya);
                    Yb = fma2(c23.y, g[3], Yb);
                    const uint64_t Y = add2(Ya, Yb);
                    yp[i] = lo2(Y) + hi2(Y);
                }
                wprev = w8[7];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    yp_prev[i] = yp[i];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    w_prev4[kk] = wmine[kk];
                    u_prev4[kk] = umine[kk];
                }
                z_prev = zmine;
                off_prev = ((j ^ swz) << 4) + pp * 8;
            }
            if (MODE != 1)
                finish();  // last block
        };
        if (pow_path)
            run(std::true_type{});
        else
            run(std::false_type{});

        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);

        if (inf.z & kInfoLast) {
            // back to h = w_last * g; continue from h with w_{-1} := 1
            float hv[8];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                hv[2 * jj] = lo2(g[jj]) * wprev;
                hv[2 * jj + 1] = hi2(g[jj]) * wprev;
                g[jj] = pk2(hv[2 * jj], hv[2 * jj + 1]);
            }
            wprev = 1.f;
            if (MODE == 1) {
                // aggregate of this segment: end state from zero, sum of steps
                const size_t ua = size_t(unit) * CH + ch;
                float4 *dst = reinterpret_cast<float4 *>(p.agg + ua * kDiagN + pp * 8);
                __stcg(dst, make_float4(hv[0], hv[1], hv[2], hv[3]));
                __stcg(dst + 1, make_float4(hv[4], hv[5], hv[6], hv[7]));
                const float sd = sdel + __shfl_xor_sync(0xffffffffu, sdel, 1);
                if (pp == 0)
                    __stcg(p.agg_sd + ua, sd);
            } else if (MODE == 0 && k < p.num_segs - 1) {
                float4 *dst = reinterpret_cast<float4 *>(
                    p.carry + (size_t(unit) * CH + ch) * kDiagN + pp * 8);
                dst[0] = make_float4(hv[0], hv[1], hv[2], hv[3]);
                dst[1] = make_float4(hv[4], hv[5], hv[6], hv[7]);
                __threadfence();
                __syncwarp();
                if (lane == 0 && unit != p.dbg_skip_publish)
                    st_release_gpu(p.flags + size_t(unit) * CW + warp, 1u);
            } else if (p.last_state && d < p.dim && k == p.num_segs - 1) {
                float *dst = p.last_state + (size_t(b) * p.dim + d) * kDiagN;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    dst[2 * j + pp] = hv[j];
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

    named_bar_sync(1, CONS);
    if (tid == 0) {
        if (MODE != 1 && it > 0 && !*abort_flag) {
            tma_store_3d(&tm_y, ytile + ((it - 1) & 1) * TILE, prev_t0, prev_d0, prev_b);
            bulk_commit();
        }
        bulk_wait_all<0>();
    }
}

}  // namespace selscan
