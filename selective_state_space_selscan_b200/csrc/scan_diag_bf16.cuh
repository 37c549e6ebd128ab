// scan_diag_bf16.cuh -- fast diagonal-A selective scan for bf16 inputs
// (fp32 state), sm_100a.
//
// What it computes (per batch row b, channel d, token t; "03 -- Modelos de
// espacio de estados", sections "El mecanismo selectivo de Mamba",
// "Discretizacion", "Parallel scan"; "P20 -- Mamba", section 5):
//   delta_t = softplus(Delta + bias)     h_t = exp(delta_t A) h_{t-1} + delta_t B_t u_t
//   y_t     = (C_t . h_t + D u_t) * silu(z_t)
//
// Same contract and work decomposition as scan_diag.cuh (persistent grid,
// atomic ticket in segment-major order, one producer warp streaming 64-token
// chunks with bulk tensor copies, segments linked by gpu-scope
// release/acquire flags), with an inner loop laid out for the B200 SM:
//
//  * One consumer thread per channel, all 16 states in registers (eight
//    packed f32x2 pairs): no exchange between lanes at all.  128 channels per
//    CTA, so each of the four schedulers runs one consumer warp; the chains
//    of a channel are sequential in time, so what matters is how fast a
//    single warp can issue.
//  * The state is kept rescaled, g = h / s with s = delta * u * log2(e), so
//    that the input term needs no multiply per state:
//       g_t = (s_{t-1}/s_t) exp(delta_t A) g_{t-1} + ln2 * B_t,
//       y_t = s_t (C_t . g_t) + D u_t.
//    B is staged pre-multiplied by ln2.  When some |s_t| of an 8-token block
//    is below 2^-64 (u = 0 padding, a zero step size, ...) the whole warp
//    takes the exact form of that block instead: s_t is clamped to +-2^-64
//    and the input term is scaled by s_t / clamp(s_t), which is 0 for a zero
//    input, so no tiny or zero input is rounded up.
//  * Per-token work that does not depend on the state index (softplus in
//    log2 units, the decay base, 1/s, the D skip, the gate) runs on pairs of
//    tokens with packed f32x2 instructions, and is software-pipelined: the
//    next 8-token block is prepared and the previous one finished while the
//    current block's eight steps run, interleaved token by token in the
//    source (a pair of the next block's preparation before every even step,
//    a pair of the previous block's outputs after every odd one), which is
//    the order the scheduler keeps under full register pressure; with one
//    warp per scheduler that order decides how much of the special-function
//    and shared-memory latency hides under the step arithmetic.
//  * For S4D-real A (A[d,n] = (n+1) A[d,0], checked per channel at run time)
//    the decays are powers r^(n+1) of r = exp(delta A[d,0]): one ex2 per token
//    and seven packed multiplies.  Other A take one ex2 per state.
//  * B and C of a chunk are staged once per CTA as fp32, token-major
//    ([t][B 16 | C 16]), so a thread reads a token's 32 values with eight
//    16-byte broadcast loads.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "scan_diag.cuh"
#include "f32x2.cuh"

namespace selscan {

constexpr float kTau = 5.421010862427522e-20f;  // 2^-64: smallest |s| of the fast form
constexpr float kSmallE = 0.015625f;            // below 2^-6 the log1p series is used

constexpr int kFastLanesPerChannel = 1;  // consumer threads per channel

template <int CH, int STAGES, bool GATE>
struct DiagFastLayout {
    static constexpr int kChunk = 64;                    // tokens per stage
    static constexpr int kTile = CH * 128;               // bf16 [CH][64], 128-byte swizzled rows
    static constexpr int kBCTile = kDiagN * 128;         // bf16 [16][64]
    static constexpr int kStage = (2 + (GATE ? 1 : 0)) * kTile + 2 * kBCTile;
    static constexpr int kStagesOff = 0;
    static constexpr int kBCFOff = STAGES * kStage;      // fp32 [2][64][32]
    static constexpr int kYOff = kBCFOff + 2 * kChunk * 32 * 4;
    static constexpr int kBarOff = kYOff + 2 * kTile;
    static constexpr int kInfoOff = kBarOff + 2 * STAGES * 8;
    static constexpr int kAbortOff = kInfoOff + STAGES * 16;
    static constexpr int kBytes = kAbortOff + 16;
    static constexpr int kAlloc = kBytes + 1024;
};

// Per-token values of one 8-token block, as pairs (tokens 2k, 2k+1).
struct PrepBlock {
    uint64_t R[4];   // decay base r = exp(delta A0) (S4D-real) or delta*log2e (general A)
    uint64_t W[4];   // s = delta * log2e * u
    uint64_t RS[4];  // 1 / s (fast form only)
    uint64_t SD;     // sum of the block's step sizes, log2 units (aggregate pass)
    bool tiny;       // some |s| < 2^-64 in the block
};

// Preparation of token pair k (tokens 2k, 2k + 1) of a block, from the
// block's u and Delta words; `mn` and `SDa` accumulate over the pairs.
template <bool SOFTPLUS, bool POW, int MODE>
__device__ __forceinline__ void prep_pair(PrepBlock &pb, float &mn, uint64_t &SDa, uint32_t uw,
                                          uint32_t dw, int k, int tfirst, int L, uint64_t BL2E2,
                                          float a0)
{
    const uint64_t L2E2 = pk2(kLog2e, kLog2e);
    const uint64_t U = bf2_to_f2(uw);
    uint64_t D2 = fma2(bf2_to_f2(dw), L2E2, BL2E2);  // (Delta + bias) log2e
    if (SOFTPLUS) {
        // delta log2e = log2(1 + 2^x): lg2 of 1 + e, or the log1p series
        // (in log2 units) when e < 2^-6; x itself beyond 2^64.
        const float xa = lo2(D2), xb = hi2(D2);
        const uint64_t E = pk2(ex2_approx(fminf(xa, 64.f)), ex2_approx(fminf(xb, 64.f)));
        const uint64_t T = add2(E, pk2(1.f, 1.f));
        uint64_t Q = fma2(E, pk2(kLog2e / 3.f, kLog2e / 3.f), pk2(-0.5f * kLog2e, -0.5f * kLog2e));
        Q = fma2(E, Q, L2E2);
        Q = mul2(E, Q);
        float da = lo2(E) < kSmallE ? lo2(Q) : lg2_approx(lo2(T));
        float db = hi2(E) < kSmallE ? hi2(Q) : lg2_approx(hi2(T));
        D2 = pk2(fmaxf(da, xa), fmaxf(db, xb));
    }
    if (tfirst + 8 > L) {
        // tokens past the end of the sequence: identity steps
        const int t = tfirst + 2 * k;
        D2 = pk2(t < L ? lo2(D2) : 0.f, t + 1 < L ? hi2(D2) : 0.f);
    }
    if (MODE == 1)
        SDa = add2(SDa, D2);
    if (POW) {
        const uint64_t X = mul2(D2, pk2(a0, a0));
        pb.R[k] = pk2(ex2_approx(lo2(X)), ex2_approx(hi2(X)));
    } else {
        pb.R[k] = D2;
    }
    const uint64_t W = mul2(D2, U);
    pb.W[k] = W;
    mn = fminf(mn, fminf(fabsf(lo2(W)), fabsf(hi2(W))));
    pb.RS[k] = pk2(rcp_approx(lo2(W)), rcp_approx(hi2(W)));
}

// Preparation of a whole block (the first block of a chunk).
template <bool SOFTPLUS, bool POW, int MODE>
__device__ __forceinline__ void prep8(PrepBlock &pb, const uint8_t *u_row, const uint8_t *dl_row,
                                      int off, int tfirst, int L, uint64_t BL2E2, float a0)
{
    const uint4 uq = *reinterpret_cast<const uint4 *>(u_row + off);
    const uint4 dq = *reinterpret_cast<const uint4 *>(dl_row + off);
    const uint32_t uw[4] = {uq.x, uq.y, uq.z, uq.w};
    const uint32_t dw[4] = {dq.x, dq.y, dq.z, dq.w};
    float mn = 3.0e38f;
    uint64_t SD = pk2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 4; ++k)
        prep_pair<SOFTPLUS, POW, MODE>(pb, mn, SD, uw[k], dw[k], k, tfirst, L, BL2E2, a0);
    pb.SD = SD;
    pb.tiny = mn < kTau;
}

// Outputs of token pair k: y = s (C.g) + D u, times silu(z), packed to bf16.
template <bool GATE>
__device__ __forceinline__ uint32_t finish_pair(float y0, float y1, float s0, float s1, uint32_t uw,
                                                uint32_t zw, float dsk)
{
    const uint64_t DU = mul2(bf2_to_f2(uw), pk2(dsk, dsk));
    uint64_t Y = fma2(pk2(s0, s1), pk2(y0, y1), DU);
    if (GATE) {
        // silu(z) = z sigmoid(z) = (z/2) (1 + tanh(z/2))
        const uint64_t HZ = mul2(bf2_to_f2(zw), pk2(0.5f, 0.5f));
        const uint64_t TH = pk2(tanh_approx(lo2(HZ)), tanh_approx(hi2(HZ)));
        Y = mul2(Y, fma2(HZ, TH, HZ));
    }
    return pack2_bf16(lo2(Y), hi2(Y));
}

// Outputs of one block: y = s (C.g) + D u, times silu(z); bf16 into the y tile.
template <bool GATE>
__device__ __forceinline__ void finish8(const float (&yp)[8], const float (&se)[8],
                                        const uint8_t *u_row, const uint8_t *z_row,
                                        uint8_t *y_row, int off, float dsk)
{
    const uint4 uq = *reinterpret_cast<const uint4 *>(u_row + off);
    uint4 zq = make_uint4(0, 0, 0, 0);
    if (GATE)
        zq = *reinterpret_cast<const uint4 *>(z_row + off);
    const uint32_t uw[4] = {uq.x, uq.y, uq.z, uq.w};
    const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
        o[k] = finish_pair<GATE>(yp[2 * k], yp[2 * k + 1], se[2 * k], se[2 * k + 1], uw[k], zw[k],
                                 dsk);
    *reinterpret_cast<uint4 *>(y_row + off) = make_uint4(o[0], o[1], o[2], o[3]);
}

// One 8-token block with its neighbours' work interleaved token by token:
// step i of this block, the preparation of pair i/2 of the next block (even
// i) and the outputs of pair i/2 of the previous block (odd i, OUT only).
template <bool EXACT, bool POW, bool OUT, bool SOFTPLUS, bool GATE, int MODE>
__device__ __forceinline__ void block8(uint64_t (&g)[8], const PrepBlock &pb, PrepBlock &nx,
                                       float &s_prev, const float *bct, float (&yp)[8],
                                       float (&se)[8], const uint64_t (&apair)[8],
                                       const uint8_t *u_row, const uint8_t *dl_row,
                                       const uint8_t *z_row, uint8_t *y_row, int off_n,
                                       int tfirst_n, int L_n, uint64_t BL2E2, float a0,
                                       const float (&yq)[8], const float (&sq)[8], int off_p,
                                       float dsk)
{
    const uint4 uq = *reinterpret_cast<const uint4 *>(u_row + off_n);
    const uint4 dq = *reinterpret_cast<const uint4 *>(dl_row + off_n);
    const uint32_t uw[4] = {uq.x, uq.y, uq.z, uq.w};
    const uint32_t dw[4] = {dq.x, dq.y, dq.z, dq.w};
    uint32_t fu[4] = {0, 0, 0, 0}, fz[4] = {0, 0, 0, 0}, o[4];
    if (OUT) {
        const uint4 a = *reinterpret_cast<const uint4 *>(u_row + off_p);
        fu[0] = a.x; fu[1] = a.y; fu[2] = a.z; fu[3] = a.w;
        if (GATE) {
            const uint4 c = *reinterpret_cast<const uint4 *>(z_row + off_p);
            fz[0] = c.x; fz[1] = c.y; fz[2] = c.z; fz[3] = c.w;
        }
    }
    float mn = 3.0e38f;
    uint64_t SDa = pk2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int k = i >> 1;
        const bool hi = (i & 1) != 0;
        if (!hi)
            prep_pair<SOFTPLUS, POW, MODE>(nx, mn, SDa, uw[k], dw[k], k, tfirst_n, L_n, BL2E2, a0);
        const float w = hi ? hi2(pb.W[k]) : lo2(pb.W[k]);
        float s, rs;
        if (EXACT) {
            s = copysignf(fmaxf(fabsf(w), kTau), w);
            rs = rcp_approx(s);
        } else {
            s = w;
            rs = hi ? hi2(pb.RS[k]) : lo2(pb.RS[k]);
        }
        const float rho = s_prev * rs;
        s_prev = s;
        se[i] = s;
        const float rr = hi ? hi2(pb.R[k]) : lo2(pb.R[k]);
        uint64_t V[8];
        if (POW) {
            const float r2 = rr * rr;
            V[0] = pk2(rho * rr, rho * r2);
            const uint64_t SS = pk2(r2, r2);
#pragma unroll
            for (int kk = 1; kk < 8; ++kk)
                V[kk] = mul2(V[kk - 1], SS);
        } else {
            const uint64_t DD = pk2(rr, rr), RR = pk2(rho, rho);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t X = mul2(DD, apair[kk]);
                V[kk] = mul2(RR, pk2(ex2_approx(lo2(X)), ex2_approx(hi2(X))));
            }
        }
        const ulonglong2 *q = reinterpret_cast<const ulonglong2 *>(bct + i * 32);
        const ulonglong2 b01 = q[0], b23 = q[1], b45 = q[2], b67 = q[3];
        uint64_t Bp[8] = {b01.x, b01.y, b23.x, b23.y, b45.x, b45.y, b67.x, b67.y};
        if (EXACT) {
            const float kap = w * rs;
            const uint64_t KK = pk2(kap, kap);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                Bp[kk] = mul2(KK, Bp[kk]);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            g[kk] = fma2(V[kk], g[kk], Bp[kk]);
        if (OUT) {
            const ulonglong2 c01 = q[4], c23 = q[5], c45 = q[6], c67 = q[7];
            uint64_t acc = mul2(c01.x, g[0]);
            acc = fma2(c01.y, g[1], acc);
            acc = fma2(c23.x, g[2], acc);
            acc = fma2(c23.y, g[3], acc);
            acc = fma2(c45.x, g[4], acc);
            acc = fma2(c45.y, g[5], acc);
            acc = fma2(c67.x, g[6], acc);
            acc = fma2(c67.y, g[7], acc);
            yp[i] = lo2(acc) + hi2(acc);
            if (hi)
                o[k] = finish_pair<GATE>(yq[i - 1], yq[i], sq[i - 1], sq[i], fu[k], fz[k], dsk);
        }
    }
    nx.SD = SDa;
    nx.tiny = mn < kTau;
    if (OUT)
        *reinterpret_cast<uint4 *>(y_row + off_p) = make_uint4(o[0], o[1], o[2], o[3]);
}

// MODE 0: one pass, segments chained through published carries.
// MODE 1: aggregate pass of the two-pass form: every segment scans from a
//         zero state and records its end state and the sum of its step sizes
//         (reads u, delta and B only; writes no y).
// MODE 2: output pass of the two-pass form: every segment starts from the
//         state folded from the aggregates of the segments before it.
template <int CH, int STAGES, bool GATE, bool SOFTPLUS, int MODE = 0>
__global__ void __launch_bounds__(CH + 32, 1)
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
    constexpr int CONS = CH;  // one consumer thread per channel
    constexpr int CW = CONS / 32;
    constexpr int TILE = Lay::kTile;
    constexpr bool OUT = MODE != 1;
    static_assert(CONS % 32 == 0 && CW >= 1 && CW <= 8, "consumer threads must fill warps");

    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, offset from the shared array itself so that
    // every pointer derived from it stays in the shared address space
    uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t *stages = smem + Lay::kStagesOff;
    float *bcf = reinterpret_cast<float *>(smem + Lay::kBCFOff);
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
            if (OUT)
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
                    if (!mbar_wait_backoff(&empty[s], ph ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const int t0 = tb + c * TC;
                    info[s] = make_int4(int(tk), t0,
                                        (c == 0 ? kInfoFirst : 0) |
                                            (c == nch - 1 ? kInfoLast : 0),
                                        0);
                    uint8_t *st = stages + s * Lay::kStage;
                    mbar_arrive_expect_tx(&full[s], OUT ? Lay::kStage : 2 * TILE + Lay::kBCTile);
                    tma_load_3d(st, &tm_u, &full[s], t0, d0, b);
                    tma_load_3d(st + TILE, &tm_delta, &full[s], t0, d0, b);
                    if (GATE && OUT)
                        tma_load_3d(st + 2 * TILE, &tm_z, &full[s], t0, d0, b);
                    uint8_t *bct = st + (GATE ? 3 : 2) * TILE;
                    tma_load_3d(bct, &tm_B, &full[s], t0, 0, b);
                    if (OUT)
                        tma_load_3d(bct + Lay::kBCTile, &tm_C, &full[s], t0, 0, b);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (ok && mbar_wait_backoff(&empty[s], ph ^ 1u, p.timeout_ns)) {
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
    const int ch = tid;          // channel within the tile
    const int swz = ch & 7;      // 128-byte swizzle phase of this row
    uint64_t g[8];               // rescaled states (2k, 2k+1)
#pragma unroll
    for (int k = 0; k < 8; ++k)
        g[k] = pk2(0.f, 0.f);
    uint64_t apair[8];           // A of this channel, paired (general path)
    float a0 = 0.f, dsk = 0.f, s_prev = 1.f;
    uint64_t BL2E2 = 0;          // bias * log2e, paired
    uint64_t SD = 0;             // sum of step sizes (log2 units) in the segment (MODE 1)
    bool pow_path = true;
    bool live = false;           // this thread's channel exists (ragged last tile)
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
            live = d < p.dim;
            // A, h0 and last_state are caller buffers with 4-byte alignment:
            // scalar accesses only
            const float *arow = p.A + size_t(live ? d : 0) * kDiagN;
            float av[16];
#pragma unroll
            for (int n = 0; n < 16; ++n)
                av[n] = __ldg(arow + n);
            bool ok = true;
#pragma unroll
            for (int n = 0; n < 16; ++n)
                ok = ok && (av[n] == float(n + 1) * av[0]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                apair[kk] = pk2(av[2 * kk], av[2 * kk + 1]);
            a0 = av[0];
            pow_path = __all_sync(0xffffffffu, ok);
            const float bias = (p.delta_bias && live) ? p.delta_bias[d] : 0.f;
            BL2E2 = pk2(bias * kLog2e, bias * kLog2e);
            dsk = (p.Dskip && live) ? p.Dskip[d] : 0.f;
            s_prev = 1.f;  // g starts as h_in (s_{-1} := 1)
            SD = 0;
            float hv[16];
#pragma unroll
            for (int n = 0; n < 16; ++n)
                hv[n] = 0.f;
            if (MODE == 1) {
                // from zero
            } else if (k == 0 || MODE == 2) {
                if (p.h0 && live) {
                    const float *src = p.h0 + (size_t(b) * p.dim + d) * kDiagN;
#pragma unroll
                    for (int n = 0; n < 16; ++n)
                        hv[n] = src[n];
                }
                if (MODE == 2) {
                    // h_in = fold over the earlier segments j of this tile:
                    // h = exp(A sum(delta_j)) h + E_j
                    for (int jseg = 0; jseg < k; ++jseg) {
                        const size_t uj = size_t(jseg) * G + gg;
                        const float sd2 = __ldcg(p.agg_sd + uj * CH + ch);
                        const float4 *e = reinterpret_cast<const float4 *>(
                            p.agg + (uj * CH + ch) * kDiagN);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float4 ev = __ldcg(e + q4);
                            const float evv[4] = {ev.x, ev.y, ev.z, ev.w};
#pragma unroll
                            for (int m = 0; m < 4; ++m)
                                hv[4 * q4 + m] = fmaf(ex2_approx(av[4 * q4 + m] * sd2),
                                                      hv[4 * q4 + m], evv[m]);
                        }
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
                } else {
                    (void)ld_acquire_gpu(flag);
                    const float4 *src = reinterpret_cast<const float4 *>(
                        p.carry + (size_t(prev) * CH + ch) * kDiagN);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 v = __ldcg(src + q4);
                        hv[4 * q4] = v.x; hv[4 * q4 + 1] = v.y; hv[4 * q4 + 2] = v.z; hv[4 * q4 + 3] = v.w;
                    }
                }
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                g[kk] = pk2(hv[2 * kk], hv[2 * kk + 1]);
        }

        uint8_t *st = stages + s * Lay::kStage;
        const uint8_t *Bt = st + (GATE ? 3 : 2) * TILE;
        const uint8_t *Ct = Bt + Lay::kBCTile;
        float *bcb = bcf + (it & 1) * TC * 32;
        // B (times ln2) and C of this chunk -> fp32, token-major [t][B 16 | C 16].
        // Lane r converts row r (B rows 0..15, C rows 16..31), warp w the
        // 8-token vectors w, w + CW, ...: one 16-byte read, eight 4-byte writes
        // to consecutive words.
        if (arrived && (OUT || lane < 16)) {
            const int isC = lane >> 4, n = lane & 15;
            const uint8_t *src = (isC ? Ct : Bt) + n * 128;
            const float sc = isC ? 1.f : kLn2;
            for (int v = warp; v < 8; v += CW) {
                const uint4 q = *reinterpret_cast<const uint4 *>(src + ((v ^ (n & 7)) << 4));
                float f[8];
                unpack8_bf16(q, f);
                float *dst = bcb + v * 8 * 32 + lane;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i * 32] = f[i] * sc;
            }
        }
        if (OUT && tid == 0)
            bulk_wait_read<0>();  // y tile (it & 1) free again
        if (OUT)
            fence_proxy_async_smem();  // my y writes of the previous chunk -> its TMA store
        if (named_bar_any(1, CONS, !arrived)) {
            if (tid == 0)
                atomicOr(p.err, kErrTimeoutPipe);
            *abort_flag = 1;
            break;
        }
        if (OUT && tid == 0 && it > 0) {
            tma_store_3d(&tm_y, ytile + ((it - 1) & 1) * TILE, prev_t0, prev_d0, prev_b);
            bulk_commit();
        }

        const uint8_t *u_row = st + ch * 128;
        const uint8_t *dl_row = st + TILE + ch * 128;
        const uint8_t *z_row = st + 2 * TILE + ch * 128;
        uint8_t *y_row = ytile + (it & 1) * TILE + ch * 128;
        const int t0 = inf.y;

        // Block j's eight steps run in the same basic block as the
        // preparation of block j + 1 and the outputs of block j - 1, so the
        // special-function and shared-memory latencies of those phases hide
        // under the step arithmetic.
        auto run = [&](auto pow_tag) {
            constexpr bool POWC = decltype(pow_tag)::value;
            PrepBlock cur, nxt;
            float yp[8], se[8], yp_prev[8], se_prev[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                yp_prev[i] = 0.f;
                se_prev[i] = 0.f;
            }
            prep8<SOFTPLUS, POWC, MODE>(cur, u_row, dl_row, swz << 4, t0, p.L, BL2E2, a0);
#pragma unroll 2
            for (int j = 0; j < TC / 8; ++j) {
                // channels past dim (zero-filled rows) never ask for the exact form
                const bool exact = __any_sync(0xffffffffu, cur.tiny && live);
                if (MODE == 1)
                    SD = add2(SD, cur.SD);
                const int jn = (j + 1) & 7;  // wraps harmlessly after the last block
                // block j - 1's outputs; for j = 0 this writes block 7's slot,
                // which the last block's outputs overwrite below
                auto body = [&](auto exact_tag) {
                    constexpr bool EX = decltype(exact_tag)::value;
                    block8<EX, POWC, OUT, SOFTPLUS, GATE, MODE>(
                        g, cur, nxt, s_prev, bcb + j * 8 * 32, yp, se, apair, u_row, dl_row,
                        z_row, y_row, (jn ^ swz) << 4, t0 + jn * 8, j < 7 ? p.L : 0x7fffffff,
                        BL2E2, a0, yp_prev, se_prev, (((j - 1) & 7) ^ swz) << 4, dsk);
                };
                if (exact)
                    body(std::true_type{});
                else
                    body(std::false_type{});
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    yp_prev[i] = yp[i];
                    se_prev[i] = se[i];
                }
                cur = nxt;
            }
            if (OUT)
                finish8<GATE>(yp_prev, se_prev, u_row, z_row, y_row, (7 ^ swz) << 4, dsk);
        };
        if (pow_path)
            run(std::true_type{});
        else
            run(std::false_type{});

        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);

        if (inf.z & kInfoLast) {
            // back to h = s_last g; continue from h with s_{-1} := 1
            float hv[16];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                hv[2 * kk] = lo2(g[kk]) * s_prev;
                hv[2 * kk + 1] = hi2(g[kk]) * s_prev;
                g[kk] = pk2(hv[2 * kk], hv[2 * kk + 1]);
            }
            s_prev = 1.f;
            if (MODE == 1) {
                // aggregate of this segment: end state from zero, sum of steps
                const size_t ua = size_t(unit) * CH + ch;
                float4 *dst = reinterpret_cast<float4 *>(p.agg + ua * kDiagN);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    __stcg(dst + q4, make_float4(hv[4 * q4], hv[4 * q4 + 1], hv[4 * q4 + 2],
                                                 hv[4 * q4 + 3]));
                __stcg(p.agg_sd + ua, lo2(SD) + hi2(SD));
            } else if (MODE == 0 && k < p.num_segs - 1) {
                float4 *dst = reinterpret_cast<float4 *>(
                    p.carry + (size_t(unit) * CH + ch) * kDiagN);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    dst[q4] = make_float4(hv[4 * q4], hv[4 * q4 + 1], hv[4 * q4 + 2],
                                          hv[4 * q4 + 3]);
                __threadfence();
                __syncwarp();
                if (lane == 0 && unit != p.dbg_skip_publish)
                    st_release_gpu(p.flags + size_t(unit) * CW + warp, 1u);
            } else if (p.last_state && d < p.dim && k == p.num_segs - 1) {
                float *dst = p.last_state + (size_t(b) * p.dim + d) * kDiagN;
#pragma unroll
                for (int n = 0; n < 16; ++n)
                    dst[n] = hv[n];
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

    if (OUT)
        fence_proxy_async_smem();
    named_bar_sync(1, CONS);
    if (tid == 0) {
        if (OUT && it > 0 && !*abort_flag) {
            tma_store_3d(&tm_y, ytile + ((it - 1) & 1) * TILE, prev_t0, prev_d0, prev_b);
            bulk_commit();
        }
        bulk_wait_all<0>();
    }
}

}  // namespace selscan
