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
// and dh0 = g after the first token.
//
// Work units are (32 channels of one batch row, one time segment), one warp
// each, one lane per channel holding all 16 states.  Both recurrences are
// linear, so segments need not wait for one another:
//   * bwd_agg_kernel scans every segment forward from a zero state (its end
//     state E) and backward from a zero gradient (its start gradient G:
//     g_{t-1} = abar_t (g_t + dout_t C_t) needs no forward state), and sums
//     its step sizes S;
//   * selscan_bwd_kernel starts segment k from
//       h_in  = fold_{j<k}  h <- exp(A S_j) h + E_j      (from h0)
//       g_end = fold_{j>k, last first} g <- exp(A S_j) g + G_j  (from dlast)
//     then keeps h every 8 tokens (pass A), and walks the 8-token chunks
//     backwards (pass B): the chunk's states are recomputed from their
//     checkpoint into shared memory and the reverse step runs over them.
// The expanded states (batch, D, L, N) are never stored.
//
// dB and dC sum over the channels of a batch row.  Per chunk they are sums
// over the warp's lanes of shared memory: dC_t[n] of dout_t times the
// recomputed states (before the reverse walk), dB_t[n] of the terms
// g delta u that the walk writes over the states it has used.  Lane l sums
// states 4 (l % 4) .. 4 (l % 4) + 3 of token l / 4 and adds both results
// with one 16-byte atomic each into one of kBwdCopies partial copies
// (token-major, [batch][L][16]), which bwd_reduce_bc sums and transposes.
// dA, dD and the bias gradient sum over batch rows and tokens: registers,
// then atomics.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "f32x2.cuh"
#include "ptx.cuh"
#include "scan_diag.cuh"

namespace selscan {

constexpr int kBwdN = 16;  // states per channel
constexpr int kBwdT = 8;   // tokens per checkpoint chunk
// dB / dC are accumulated into this many partial copies (tile i adds into
// copy i % kBwdCopies) and summed afterwards: all tiles of a batch row walk
// the same tokens at nearly the same time, so one copy would take every
// tile's atomic add of a token at once.
constexpr int kBwdCopies = 8;

struct BwdParams {
    int batch, dim, L, nchunks;      // nchunks = ceil(L / kBwdT)
    int tiles, segs, seg_chunks;     // units = tiles * segs; tile = (batch row, 32 channels)
    int tiles_per_batch;
    const void *u, *delta, *z, *dy;  // (batch, dim, L), time stride 1, 16-byte aligned rows
    int64_t u_bs, u_ds, dl_bs, dl_ds, z_bs, z_ds, dy_bs, dy_ds;
    const void *B, *C;               // (batch, 16, L), same alignment
    int64_t B_bs, B_ns, C_bs, C_ns;
    const float *A;                  // (dim, 16)
    const float *delta_bias, *Dskip; // (dim) or null
    const float *h0, *dlast;         // (batch, dim, 16) or null
    int softplus;
    void *du, *ddelta, *dz;          // (batch, dim, L) like u; dz null without gate
    int64_t du_bs, du_ds, dd_bs, dd_ds, dz_bs, dz_ds;
    float *dA;                       // (dim, 16), accumulated
    float *dB, *dC;                  // (batch, 16, L) contiguous, written by bwd_reduce_bc
    float *pB, *pC;                  // kBwdCopies partial sums [batch][L][16] of dB, dC
    float *dD, *dbias;               // (dim) or null, accumulated
    float *dh0;                      // (batch, dim, 16) or null, written
    float *ckpt;                     // [batch][dim][nchunks][16] scratch
    float *aggE, *aggG, *aggS;       // [units][32][16], [units][32][16], [units][32]
};

__device__ __forceinline__ void bwd_st8(void *base, int64_t off, int valid, const float (&v)[8],
                                        const __nv_bfloat16 *)
{
    __nv_bfloat16 *p = static_cast<__nv_bfloat16 *>(base) + off;
    if (valid >= 8) {
        uint4 q;
        q.x = pack2_bf16(v[0], v[1]);
        q.y = pack2_bf16(v[2], v[3]);
        q.z = pack2_bf16(v[4], v[5]);
        q.w = pack2_bf16(v[6], v[7]);
        *reinterpret_cast<uint4 *>(p) = q;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < valid)
                p[i] = __float2bfloat16_rn(v[i]);
    }
}

__device__ __forceinline__ void bwd_st8(void *base, int64_t off, int valid, const float (&v)[8],
                                        const float *)
{
    float *p = static_cast<float *>(base) + off;
    if (valid >= 8) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < valid)
                p[i] = v[i];
    }
}

// exp(delta * A[n]) for the 16 states as 8 pairs: r^(n+1) for S4D-real A
// (A[n] = (n+1) A[0], checked per channel), else one exponential per state.
template <bool FAST>
__device__ __forceinline__ void bwd_decays(float dt, const float (&al)[kBwdN], bool pow_path,
                                           uint64_t (&a2)[8])
{
    if (pow_path) {
        // r^1 .. r^16 by a product tree (depth 4, not a chain of 7)
        const float r = FAST ? ex2_approx(dt * al[0]) : exp2f(dt * al[0]);
        const float r2 = r * r, r4 = r2 * r2, r8 = r4 * r4;
        const uint64_t R2 = pk2(r2, r2), R4 = pk2(r4, r4), R8 = pk2(r8, r8);
        a2[0] = pk2(r, r2);
        a2[1] = mul2(a2[0], R2);
        a2[2] = mul2(a2[0], R4);
        a2[3] = mul2(a2[1], R4);
#pragma unroll
        for (int j = 4; j < 8; ++j)
            a2[j] = mul2(a2[j - 4], R8);
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            a2[j] = FAST ? pk2(ex2_approx(dt * al[2 * j]), ex2_approx(dt * al[2 * j + 1]))
                         : pk2(exp2f(dt * al[2 * j]), exp2f(dt * al[2 * j + 1]));
    }
}

template <bool FAST>
__device__ __forceinline__ float bwd_step(float raw, int softplus)
{
    if (!softplus)
        return raw;
    return FAST ? softplus_fast(raw) : softplus_exact(raw);
}

// B and C of the chunk (fp32, [token][n]): all the aggregate kernel keeps
// in shared memory besides its copy stages, so it fits more warps per SM.
struct BwdBC {
    float bc[kBwdT][2][kBwdN];
};

// Per-warp shared memory of the gradient walk: B and C, the recomputed
// states of the chunk ([token][lane] rows of 16 states in four 16-byte
// pieces; the reverse walk puts each lane's dB terms in their place once it
// has used them) and the output gradient through the gate ([token][lane]).
// Piece c of lane l's row sits at position c ^ ((l >> 1) & 3): the eight
// lanes of a quarter warp that store or load the same piece of their own
// rows then hit eight distinct bank groups.
struct BwdSmem : BwdBC {
    float4 h[kBwdT][32][4];
    float dout[kBwdT][32];
};

__device__ __forceinline__ int bwd_piece(int l, int c) { return c ^ ((l >> 1) & 3); }

// This lane's 16 values of token i (8 pairs) into / out of sm.h.
__device__ __forceinline__ void bwd_put_row(BwdSmem &sm, int i, int lane, const uint64_t (&v)[8])
{
#pragma unroll
    for (int c = 0; c < 4; ++c)
        sm.h[i][lane][bwd_piece(lane, c)] =
            make_float4(lo2(v[2 * c]), hi2(v[2 * c]), lo2(v[2 * c + 1]), hi2(v[2 * c + 1]));
}

__device__ __forceinline__ void bwd_get_row(const BwdSmem &sm, int i, int lane, uint64_t (&v)[8])
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float4 q = sm.h[i][lane][bwd_piece(lane, c)];
        v[2 * c] = pk2(q.x, q.y);
        v[2 * c + 1] = pk2(q.z, q.w);
    }
}

// Sum over the warp's 32 lanes of piece c (states 4c .. 4c + 3) of token i,
// weighted by sm.dout[i] when WEIGHTED.  The lanes of token i start at row
// i: a quarter warp (two consecutive tokens, four pieces each) then reads
// eight distinct bank groups at every step, and the eight tokens' weights
// lie in eight distinct banks.
// Four partial sums per half-piece keep the dependent chains 8 long.
template <bool WEIGHTED>
__device__ __forceinline__ float4 bwd_piece_sum(const BwdSmem &sm, int i, int c)
{
    uint64_t s0[4], s1[4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
        s0[a] = s1[a] = pk2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const int l = (k + i) & 31;
        const float4 h = sm.h[i][l][bwd_piece(l, c)];
        const int a = k & 3;
        if (WEIGHTED) {
            const float w = sm.dout[i][l];
            const uint64_t W = pk2(w, w);
            s0[a] = fma2(W, pk2(h.x, h.y), s0[a]);
            s1[a] = fma2(W, pk2(h.z, h.w), s1[a]);
        } else {
            s0[a] = add2(pk2(h.x, h.y), s0[a]);
            s1[a] = add2(pk2(h.z, h.w), s1[a]);
        }
    }
    const uint64_t t0 = add2(add2(s0[0], s0[1]), add2(s0[2], s0[3]));
    const uint64_t t1 = add2(add2(s1[0], s1[1]), add2(s1[2], s1[3]));
    return make_float4(lo2(t0), hi2(t0), lo2(t1), hi2(t1));
}

// One chunk's raw inputs, copied asynchronously: per lane its channel's 8
// tokens of u, delta, dy, z (KV 16-byte vectors each), one row of B (lanes
// 0..15) or C (lanes 16..31), and its checkpoint.
template <int KV>
struct BwdStage {
    uint4 u[KV][32], dl[KV][32], dy[KV][32], z[KV][32], bc[KV][32];
    float4 ck[4][32];
};

constexpr int kLdU = 1, kLdDl = 2, kLdDy = 4, kLdZ = 8, kLdB = 16, kLdC = 32, kLdCk = 64;

template <typename T>
constexpr int bwd_kv() { return int(sizeof(T)) * kBwdT / 16; }

// Issue the copies of tokens [t0, t0 + valid) of this lane's rows (`what` is
// a mask of kLd*); the caller commits the group.
template <typename T, int KV>
__device__ __forceinline__ void bwd_issue(const BwdParams &p, BwdStage<KV> &st, int64_t row_u,
                                          int64_t row_dl, int64_t row_dy, int64_t row_z, int b,
                                          int t0, int valid, int lane, int what, const float *ck)
{
    constexpr int EPV = 16 / int(sizeof(T));  // elements per 16-byte vector
    const T *base;
#pragma unroll
    for (int k = 0; k < KV; ++k) {
        const int left = valid - k * EPV;
        const uint32_t bytes = uint32_t(left <= 0 ? 0 : (left >= EPV ? 16 : left * int(sizeof(T))));
        const int off = t0 + (left > 0 ? k * EPV : 0);
        if (what & kLdU) {
            base = static_cast<const T *>(p.u);
            cp_async16(&st.u[k][lane], base + row_u + off, bytes);
        }
        if (what & kLdDl) {
            base = static_cast<const T *>(p.delta);
            cp_async16(&st.dl[k][lane], base + row_dl + off, bytes);
        }
        if (what & kLdDy) {
            base = static_cast<const T *>(p.dy);
            cp_async16(&st.dy[k][lane], base + row_dy + off, bytes);
        }
        if ((what & kLdZ) && p.z) {
            base = static_cast<const T *>(p.z);
            cp_async16(&st.z[k][lane], base + row_z + off, bytes);
        }
        const bool isC = lane >= kBwdN;
        if ((what & (isC ? kLdC : kLdB))) {
            const int n = lane & 15;
            base = static_cast<const T *>(isC ? p.C : p.B);
            const int64_t row = int64_t(b) * (isC ? p.C_bs : p.B_bs) +
                                int64_t(n) * (isC ? p.C_ns : p.B_ns);
            cp_async16(&st.bc[k][lane], base + row + off, bytes);
        }
    }
    if (what & kLdCk) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            cp_async16(&st.ck[q][lane], ck + 4 * q, 16);
    }
}

__device__ __forceinline__ void bwd_unpack(const uint4 (&v)[1], float (&f)[8], const __nv_bfloat16 *)
{
    unpack8_bf16(v[0], f);
}

__device__ __forceinline__ void bwd_unpack(const uint4 (&v)[2], float (&f)[8], const float *)
{
    f[0] = __uint_as_float(v[0].x); f[1] = __uint_as_float(v[0].y);
    f[2] = __uint_as_float(v[0].z); f[3] = __uint_as_float(v[0].w);
    f[4] = __uint_as_float(v[1].x); f[5] = __uint_as_float(v[1].y);
    f[6] = __uint_as_float(v[1].z); f[7] = __uint_as_float(v[1].w);
}

// This lane's 8 values of a staged tensor.
template <typename T, int KV>
__device__ __forceinline__ void bwd_vals(const uint4 (&src)[KV][32], int lane, float (&f)[8])
{
    uint4 v[KV];
#pragma unroll
    for (int k = 0; k < KV; ++k)
        v[k] = src[k][lane];
    const T *tag = nullptr;
    bwd_unpack(v, f, tag);
}

// Staged B / C rows -> fp32 [token][n] for the whole warp.
template <typename T, int KV>
__device__ __forceinline__ void bwd_bc_to_smem(const BwdStage<KV> &st, BwdBC &sm, int lane,
                                               bool withC)
{
    if (lane < kBwdN || withC) {
        float v[8];
        bwd_vals<T, KV>(st.bc, lane, v);
        const int isC = lane >= kBwdN;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            sm.bc[i][isC][lane & 15] = v[i];
    }
    __syncwarp();
}

template <typename T>
struct BwdChannel {
    float al[kBwdN];
    uint64_t An2[8];
    bool pow_path;
    float bias, dsk;
    int64_t row_u, row_dl, row_z, row_dy, row_du, row_dd, row_dz;

    __device__ __forceinline__ void init(const BwdParams &p, int b, int dd)
    {
        float An[kBwdN];
        pow_path = true;
#pragma unroll
        for (int n = 0; n < kBwdN; ++n) {
            An[n] = p.A[int64_t(dd) * kBwdN + n];
            al[n] = An[n] * kLog2e;
            pow_path = pow_path && (An[n] == float(n + 1) * An[0]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
            An2[j] = pk2(An[2 * j], An[2 * j + 1]);
        bias = p.delta_bias ? p.delta_bias[dd] : 0.f;
        dsk = p.Dskip ? p.Dskip[dd] : 0.f;
        row_u = int64_t(b) * p.u_bs + int64_t(dd) * p.u_ds;
        row_dl = int64_t(b) * p.dl_bs + int64_t(dd) * p.dl_ds;
        row_z = int64_t(b) * p.z_bs + int64_t(dd) * p.z_ds;
        row_dy = int64_t(b) * p.dy_bs + int64_t(dd) * p.dy_ds;
        row_du = int64_t(b) * p.du_bs + int64_t(dd) * p.du_ds;
        row_dd = int64_t(b) * p.dd_bs + int64_t(dd) * p.dd_ds;
        row_dz = int64_t(b) * p.dz_bs + int64_t(dd) * p.dz_ds;
    }
};

// Forward over [t0, t0 + valid): h <- abar h + delta u B, token by token;
// when KEEP is set (SM = BwdSmem) the state after each token goes to shared
// memory and the step sizes to dts.
template <typename T, bool KEEP, typename SM>
__device__ __forceinline__ void bwd_forward_chunk(const BwdParams &p, const BwdChannel<T> &ch,
                                                  SM &sm, int valid, const float (&uv)[8],
                                                  const float (&dv)[8], uint64_t (&h2)[8],
                                                  int lane, float (&dts)[8])
{
    constexpr bool FAST = !std::is_same<T, float>::value;
#pragma unroll
    for (int i = 0; i < kBwdT; ++i) {
        if (i >= valid)
            break;
        const float dt = bwd_step<FAST>(dv[i] + ch.bias, p.softplus);
        if (KEEP)
            dts[i] = dt;
        const float dx = dt * uv[i];
        const uint64_t DX = pk2(dx, dx);
        uint64_t a2[8];
        bwd_decays<FAST>(dt, ch.al, ch.pow_path, a2);
        const float4 *bq = reinterpret_cast<const float4 *>(sm.bc[i][0]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 bb = bq[q];
            h2[2 * q] = fma2(a2[2 * q], h2[2 * q], mul2(DX, pk2(bb.x, bb.y)));
            h2[2 * q + 1] = fma2(a2[2 * q + 1], h2[2 * q + 1], mul2(DX, pk2(bb.z, bb.w)));
        }
        if constexpr (KEEP)
            bwd_put_row(sm, i, lane, h2);
    }
}

// Segment aggregates: E (end state from zero), G (start gradient from a zero
// end gradient), S (sum of step sizes) of every (tile, segment) unit but the
// ones that no other unit needs (E of the last segment, G of the first).
template <typename T>
__global__ void __launch_bounds__(32)
bwd_agg_kernel(const BwdParams p)
{
    constexpr bool FAST = !std::is_same<T, float>::value;
    __shared__ __align__(16) BwdBC sm;
    const int lane = threadIdx.x;
    const int unit = blockIdx.x;
    const int seg = unit / p.tiles, tile = unit - seg * p.tiles;
    const int b = tile / p.tiles_per_batch;
    const int d = (tile - b * p.tiles_per_batch) * 32 + lane;
    const bool live = d < p.dim;
    BwdChannel<T> ch;
    ch.init(p, b, live ? d : 0);
    const int c0 = seg * p.seg_chunks, c1 = min(p.nchunks, c0 + p.seg_chunks);

    constexpr int KV = bwd_kv<T>();
    __shared__ __align__(16) BwdStage<KV> st[2];

    // forward from zero: end state (not needed for the last segment) and the
    // sum of step sizes; chunk c+1's inputs are copied while c is computed
    uint64_t h2[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        h2[j] = pk2(0.f, 0.f);
    float ssum = 0.f;
    {
        const bool fwd = seg < p.segs - 1;
        const int what = fwd ? (kLdU | kLdDl | kLdB) : kLdDl;
        int buf = 0;
        bwd_issue<T, KV>(p, st[0], ch.row_u, ch.row_dl, ch.row_dy, ch.row_z, b, c0 * kBwdT,
                         min(kBwdT, p.L - c0 * kBwdT), lane, what, nullptr);
        cp_async_commit();
        for (int c = c0; c < c1; ++c) {
            const int t0 = c * kBwdT, valid = min(kBwdT, p.L - t0);
            if (c + 1 < c1)
                bwd_issue<T, KV>(p, st[buf ^ 1], ch.row_u, ch.row_dl, ch.row_dy, ch.row_z, b,
                                 t0 + kBwdT, min(kBwdT, p.L - t0 - kBwdT), lane, what, nullptr);
            cp_async_commit();
            cp_async_wait<1>();
            float uv[8], dv[8], dts[8];  // dts unused (KEEP off)
            bwd_vals<T, KV>(st[buf].dl, lane, dv);
#pragma unroll
            for (int i = 0; i < kBwdT; ++i)
                if (i < valid)
                    ssum += bwd_step<FAST>(dv[i] + ch.bias, p.softplus);
            if (fwd) {
                bwd_vals<T, KV>(st[buf].u, lane, uv);
                bwd_bc_to_smem<T, KV>(st[buf], sm, lane, false);
                if (valid == kBwdT)  // a constant token count for whole chunks
                    bwd_forward_chunk<T, false>(p, ch, sm, kBwdT, uv, dv, h2, lane, dts);
                else
                    bwd_forward_chunk<T, false>(p, ch, sm, valid, uv, dv, h2, lane, dts);
            }
            __syncwarp();
            buf ^= 1;
        }
        cp_async_wait<0>();
    }
    // backward from zero: g_{t-1} = abar_t (g_t + dout_t C_t)
    uint64_t g2[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        g2[j] = pk2(0.f, 0.f);
    if (seg > 0) {
        const int what = kLdDl | kLdDy | kLdZ | kLdC;
        int buf = 0;
        {
            const int cl = c1 - 1;
            bwd_issue<T, KV>(p, st[0], ch.row_u, ch.row_dl, ch.row_dy, ch.row_z, b, cl * kBwdT,
                             min(kBwdT, p.L - cl * kBwdT), lane, what, nullptr);
        }
        cp_async_commit();
        for (int c = c1 - 1; c >= c0; --c) {
            const int t0 = c * kBwdT, valid = min(kBwdT, p.L - t0);
            if (c > c0)
                bwd_issue<T, KV>(p, st[buf ^ 1], ch.row_u, ch.row_dl, ch.row_dy, ch.row_z, b,
                                 t0 - kBwdT, kBwdT, lane, what, nullptr);
            cp_async_commit();
            cp_async_wait<1>();
            bwd_bc_to_smem<T, KV>(st[buf], sm, lane, true);
            float dv[8], yv[8], zv[8];
            bwd_vals<T, KV>(st[buf].dl, lane, dv);
            bwd_vals<T, KV>(st[buf].dy, lane, yv);
            if (p.z)
                bwd_vals<T, KV>(st[buf].z, lane, zv);
            auto walk = [&](auto full_tag) {
                const int vld = decltype(full_tag)::value ? kBwdT : valid;
#pragma unroll
                for (int i = kBwdT - 1; i >= 0; --i) {
                    if (i >= vld)
                        continue;
                    const float dt = bwd_step<FAST>(dv[i] + ch.bias, p.softplus);
                    float dout = live ? yv[i] : 0.f;
                    if (p.z)
                        dout *= zv[i] / (1.f + __expf(-zv[i]));
                    const uint64_t DO = pk2(dout, dout);
                    uint64_t a2[8];
                    bwd_decays<FAST>(dt, ch.al, ch.pow_path, a2);
                    const float4 *cq = reinterpret_cast<const float4 *>(sm.bc[i][1]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 cc = cq[q];
                        g2[2 * q] = mul2(a2[2 * q], fma2(DO, pk2(cc.x, cc.y), g2[2 * q]));
                        g2[2 * q + 1] =
                            mul2(a2[2 * q + 1], fma2(DO, pk2(cc.z, cc.w), g2[2 * q + 1]));
                    }
                }
            };
            if (valid == kBwdT)  // a constant token count for whole chunks
                walk(std::true_type{});
            else
                walk(std::false_type{});
            __syncwarp();
            buf ^= 1;
        }
        cp_async_wait<0>();
    }
    if (live) {
        const int64_t o = (int64_t(unit) * 32 + lane) * kBwdN;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            p.aggE[o + 2 * j] = lo2(h2[j]);
            p.aggE[o + 2 * j + 1] = hi2(h2[j]);
            p.aggG[o + 2 * j] = lo2(g2[j]);
            p.aggG[o + 2 * j + 1] = hi2(g2[j]);
        }
        p.aggS[int64_t(unit) * 32 + lane] = ssum;
    }
}

template <typename T>
__global__ void __launch_bounds__(32)
selscan_bwd_kernel(const BwdParams p)
{
    constexpr int N = kBwdN, TC = kBwdT;
    constexpr bool FAST = !std::is_same<T, float>::value;
    const T *tag = nullptr;
    __shared__ __align__(16) BwdSmem sm;

    const int lane = threadIdx.x;
    const int unit = blockIdx.x;
    const int seg = unit / p.tiles, tile = unit - seg * p.tiles;
    const int b = tile / p.tiles_per_batch;
    const int d = (tile - b * p.tiles_per_batch) * 32 + lane;
    const bool live = d < p.dim;
    const int dd = live ? d : 0;  // lanes past the last channel mirror channel 0, add zeros
    BwdChannel<T> ch;
    ch.init(p, b, dd);
    const int c0 = seg * p.seg_chunks, c1 = min(p.nchunks, c0 + p.seg_chunks);
    float *ck = p.ckpt + (int64_t(b) * p.dim + dd) * p.nchunks * N;

    // ---- initial state of the segment and gradient at its end
    uint64_t h2[8], g2[8];
    {
        float hv[N], gv[N];
#pragma unroll
        for (int n = 0; n < N; ++n) {
            hv[n] = (p.h0 && live) ? p.h0[(int64_t(b) * p.dim + dd) * N + n] : 0.f;
            gv[n] = (p.dlast && live) ? p.dlast[(int64_t(b) * p.dim + dd) * N + n] : 0.f;
        }
        for (int j = 0; j < seg; ++j) {
            const int64_t o = (int64_t(j) * p.tiles + tile) * 32 + lane;
            const float s = __ldcg(p.aggS + o);
#pragma unroll
            for (int n = 0; n < N; ++n)
                hv[n] = fmaf(ex2_approx(ch.al[n] * s), hv[n], __ldcg(p.aggE + o * N + n));
        }
        for (int j = p.segs - 1; j > seg; --j) {
            const int64_t o = (int64_t(j) * p.tiles + tile) * 32 + lane;
            const float s = __ldcg(p.aggS + o);
#pragma unroll
            for (int n = 0; n < N; ++n)
                gv[n] = fmaf(ex2_approx(ch.al[n] * s), gv[n], __ldcg(p.aggG + o * N + n));
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            h2[j] = live ? pk2(hv[2 * j], hv[2 * j + 1]) : pk2(0.f, 0.f);
            g2[j] = live ? pk2(gv[2 * j], gv[2 * j + 1]) : pk2(0.f, 0.f);
        }
    }

    constexpr int KV = bwd_kv<T>();
    __shared__ __align__(16) BwdStage<KV> st[2];

    // ---- pass A: forward over the segment, h at the start of every chunk;
    //      chunk c+1's inputs are copied while c is computed
    {
        const int what = kLdU | kLdDl | kLdB;
        int buf = 0;
        bwd_issue<T, KV>(p, st[0], ch.row_u, ch.row_dl, ch.row_dy, ch.row_z, b, c0 * TC,
                         min(TC, p.L - c0 * TC), lane, what, nullptr);
        cp_async_commit();
        for (int c = c0; c < c1; ++c) {
            const int t0 = c * TC, valid = min(TC, p.L - t0);
            if (c + 1 < c1)
                bwd_issue<T, KV>(p, st[buf ^ 1], ch.row_u, ch.row_dl, ch.row_dy, ch.row_z, b,
                                 t0 + TC, min(TC, p.L - t0 - TC), lane, what, nullptr);
            cp_async_commit();
            if (live) {
                float4 *dst = reinterpret_cast<float4 *>(ck + c * N);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    dst[q] = make_float4(lo2(h2[2 * q]), hi2(h2[2 * q]), lo2(h2[2 * q + 1]),
                                         hi2(h2[2 * q + 1]));
            }
            cp_async_wait<1>();
            float uv[8], dv[8], dts[8];  // dts unused (KEEP off)
            bwd_vals<T, KV>(st[buf].u, lane, uv);
            bwd_vals<T, KV>(st[buf].dl, lane, dv);
            bwd_bc_to_smem<T, KV>(st[buf], sm, lane, false);
            if (valid == TC)  // a constant token count for whole chunks
                bwd_forward_chunk<T, false>(p, ch, sm, TC, uv, dv, h2, lane, dts);
            else
                bwd_forward_chunk<T, false>(p, ch, sm, valid, uv, dv, h2, lane, dts);
            __syncwarp();
            buf ^= 1;
        }
        cp_async_wait<0>();
        __syncwarp();
    }

    // ---- pass B: chunks backwards
    uint64_t gA2[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        gA2[j] = pk2(0.f, 0.f);
    float gD = 0.f, gbias = 0.f;
    const int whatB = kLdU | kLdDl | kLdDy | kLdZ | kLdB | kLdC | kLdCk;
    int bufB = 0;
    {
        const int cl = c1 - 1;
        bwd_issue<T, KV>(p, st[0], ch.row_u, ch.row_dl, ch.row_dy, ch.row_z, b, cl * TC,
                         min(TC, p.L - cl * TC), lane, whatB, ck + cl * N);
    }
    cp_async_commit();
    for (int c = c1 - 1; c >= c0; --c) {
        const int t0 = c * TC, valid = min(TC, p.L - t0);
        if (c > c0)
            bwd_issue<T, KV>(p, st[bufB ^ 1], ch.row_u, ch.row_dl, ch.row_dy, ch.row_z, b,
                             t0 - TC, TC, lane, whatB, ck + (c - 1) * N);
        cp_async_commit();
        cp_async_wait<1>();
        // whole chunks (all but a ragged last one) take a copy of the walk in
        // which the number of tokens is a constant, so the unrolled token loop
        // keeps its registers in place from one token to the next
        auto chunk = [&](auto full_tag) {
            constexpr bool FULL = decltype(full_tag)::value;
            const int vld = FULL ? TC : valid;
            const BwdStage<KV> &cur = st[bufB];
            uint64_t hc2[8];  // state before the chunk
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 v = live ? cur.ck[q][lane] : make_float4(0.f, 0.f, 0.f, 0.f);
                hc2[2 * q] = pk2(v.x, v.y);
                hc2[2 * q + 1] = pk2(v.z, v.w);
            }
            float uv[8], dv[8], yv[8], zv[8], dts[8];
            bwd_vals<T, KV>(cur.u, lane, uv);
            bwd_vals<T, KV>(cur.dl, lane, dv);
            bwd_vals<T, KV>(cur.dy, lane, yv);
            if (p.z)
                bwd_vals<T, KV>(cur.z, lane, zv);
            bwd_bc_to_smem<T, KV>(cur, sm, lane, true);
            {
                uint64_t hr[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    hr[j] = hc2[j];
                bwd_forward_chunk<T, true>(p, ch, sm, vld, uv, dv, hr, lane, dts);
            }
            __syncwarp();
            // output gradient through the gate and the factor of dz, per token
            float dov[8], fzv[8];
#pragma unroll
            for (int i = 0; i < TC; ++i) {
                const float dyv = (live && i < vld) ? yv[i] : 0.f;
                float dout = dyv, f = 0.f;
                if (p.z) {
                    const float zz = zv[i];
                    const float sg = 1.f / (1.f + __expf(-zz));
                    f = dyv * (sg * (1.f + zz * (1.f - sg)));
                    dout = dyv * zz * sg;
                }
                dov[i] = dout;
                fzv[i] = f;
                sm.dout[i][lane] = dout;
            }
            __syncwarp();
            // dC of the chunk: lane -> token ri, states 4 rc .. 4 rc + 3
            const int ri = lane >> 2, rc = lane & 3;
            const float4 dCv = bwd_piece_sum<true>(sm, ri, rc);
            __syncwarp();  // all rows read before the walk overwrites them
            float o_du[8], o_dd[8], o_dz[8];
#pragma unroll
            for (int i = 0; i < TC; ++i)
                o_du[i] = o_dd[i] = o_dz[i] = 0.f;
            uint64_t ht2[8];  // state after token i, carried down from token i + 1
#pragma unroll
            for (int j = 0; j < 8; ++j)
                ht2[j] = pk2(0.f, 0.f);
#pragma unroll
            for (int i = TC - 1; i >= 0; --i) {
                if (i >= vld)
                    continue;
                if (i == vld - 1)
                    bwd_get_row(sm, i, lane, ht2);
                uint64_t hp2[8];
                if (i > 0) {
                    bwd_get_row(sm, i - 1, lane, hp2);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        hp2[j] = hc2[j];
                }
                const float raw = dv[i] + ch.bias;
                const float dt = dts[i];
                const float x = uv[i];
                uint64_t a2[8];
                bwd_decays<FAST>(dt, ch.al, ch.pow_path, a2);
                uint64_t B2[8], C2[8];
                {
                    const float4 *bq = reinterpret_cast<const float4 *>(sm.bc[i][0]);
                    const float4 *cq = reinterpret_cast<const float4 *>(sm.bc[i][1]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 bb = bq[q], cc = cq[q];
                        B2[2 * q] = pk2(bb.x, bb.y);
                        B2[2 * q + 1] = pk2(bb.z, bb.w);
                        C2[2 * q] = pk2(cc.x, cc.y);
                        C2[2 * q + 1] = pk2(cc.z, cc.w);
                    }
                }
                if (p.z) {
                    uint64_t Y2 = mul2(C2[0], ht2[0]);
#pragma unroll
                    for (int j = 1; j < 8; ++j)
                        Y2 = fma2(C2[j], ht2[j], Y2);
                    o_dz[i] = fzv[i] * fmaf(ch.dsk, x, lo2(Y2) + hi2(Y2));
                }
                const float dout = dov[i];
                gD = fmaf(dout, x, gD);
                // with g after adding dout C:  du = dt sum g B + D dout,
                // ddelta = sum g A abar h_prev + u sum g B,  dA += dt g abar h_prev
                const uint64_t DO = pk2(dout, dout), DT = pk2(dt, dt);
                const uint64_t DTX = pk2(dt * x, dt * x);
                uint64_t gB2 = pk2(0.f, 0.f), gAh2 = pk2(0.f, 0.f), vb[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    g2[j] = fma2(DO, C2[j], g2[j]);
                    vb[j] = mul2(g2[j], DTX);
                    gB2 = fma2(g2[j], B2[j], gB2);
                    const uint64_t gah = mul2(g2[j], mul2(a2[j], hp2[j]));
                    gAh2 = fma2(ch.An2[j], gah, gAh2);
                    gA2[j] = fma2(DT, gah, gA2[j]);
                    g2[j] = mul2(g2[j], a2[j]);
                    ht2[j] = hp2[j];
                }
                bwd_put_row(sm, i, lane, vb);  // this lane's dB terms of token i
                const float gB = lo2(gB2) + hi2(gB2);
                const float dx = fmaf(dout, ch.dsk, dt * gB);
                const float ddt = fmaf(x, gB, lo2(gAh2) + hi2(gAh2));
                const float dDelta = p.softplus ? ddt / (1.f + __expf(-raw)) : ddt;
                gbias += dDelta;
                o_du[i] = dx;
                o_dd[i] = dDelta;
            }
            __syncwarp();
            const float4 dBv = bwd_piece_sum<false>(sm, ri, rc);
            if (live) {
                bwd_st8(p.du, ch.row_du + t0, vld, o_du, tag);
                bwd_st8(p.ddelta, ch.row_dd + t0, vld, o_dd, tag);
                if (p.z)
                    bwd_st8(p.dz, ch.row_dz + t0, vld, o_dz, tag);
            }
            if (ri < vld) {
                const int64_t off = ((int64_t(tile % kBwdCopies) * p.batch + b) * p.L + t0 + ri) * N +
                                    4 * rc;
                atomicAdd(reinterpret_cast<float4 *>(p.pB + off), dBv);
                atomicAdd(reinterpret_cast<float4 *>(p.pC + off), dCv);
            }
        };
        if (valid == TC)
            chunk(std::true_type{});
        else
            chunk(std::false_type{});
        __syncwarp();
        bufB ^= 1;
    }
    cp_async_wait<0>();
    if (live) {
        if (p.dh0 && seg == 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                p.dh0[(int64_t(b) * p.dim + d) * N + 2 * j] = lo2(g2[j]);
                p.dh0[(int64_t(b) * p.dim + d) * N + 2 * j + 1] = hi2(g2[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            atomicAdd(p.dA + int64_t(d) * N + 2 * j, lo2(gA2[j]));
            atomicAdd(p.dA + int64_t(d) * N + 2 * j + 1, hi2(gA2[j]));
        }
        if (p.dD)
            atomicAdd(p.dD + d, gD);
        if (p.dbias)
            atomicAdd(p.dbias + d, gbias);
    }
}

// dB, dC (batch, 16, L) = sum of the kBwdCopies partial copies, each
// [batch][L][16] (`rows` = batch * L rows of 16).  One thread per row: it
// reads its row's 64 bytes from every copy and writes state n to dB[b][n][t],
// consecutive threads writing consecutive tokens.
__global__ void __launch_bounds__(256)
bwd_reduce_bc(const float *pB, const float *pC, float *dB, float *dC, int64_t rows, int L)
{
    const int64_t copy = rows * kBwdN;  // floats per partial copy
    for (int64_t r = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; r < rows;
         r += int64_t(gridDim.x) * blockDim.x) {
        const int64_t b = r / L, t = r - b * L;
        float *ob = dB + b * kBwdN * L + t, *oc = dC + b * kBwdN * L + t;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 sb = make_float4(0.f, 0.f, 0.f, 0.f), sc = sb;
#pragma unroll
            for (int k = 0; k < kBwdCopies; ++k) {
                const float4 vb = reinterpret_cast<const float4 *>(pB + k * copy + r * kBwdN)[q];
                const float4 vc = reinterpret_cast<const float4 *>(pC + k * copy + r * kBwdN)[q];
                sb.x += vb.x; sb.y += vb.y; sb.z += vb.z; sb.w += vb.w;
                sc.x += vc.x; sc.y += vc.y; sc.z += vc.z; sc.w += vc.w;
            }
            ob[int64_t(4 * q) * L] = sb.x;
            ob[int64_t(4 * q + 1) * L] = sb.y;
            ob[int64_t(4 * q + 2) * L] = sb.z;
            ob[int64_t(4 * q + 3) * L] = sb.w;
            oc[int64_t(4 * q) * L] = sc.x;
            oc[int64_t(4 * q + 1) * L] = sc.y;
            oc[int64_t(4 * q + 2) * L] = sc.z;
            oc[int64_t(4 * q + 3) * L] = sc.w;
        }
    }
}

}  // namespace selscan
