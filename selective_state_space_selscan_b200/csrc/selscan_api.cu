// selscan_api.cu -- C ABI of libselscan (see include/selscan.h): argument
// validation, tensor-map encoding, stream-ordered scratch memory and kernel
// launch for the diagonal-A scan and the scalar-A (SSD) scan.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <mutex>
#include <algorithm>

#include "selscan.h"
#include "selscan_debug.h"
#include "scan_diag.cuh"
#include "scan_diag_bf16.cuh"
#include "ssd_scalarA.cuh"
#include "step.cuh"
#include "bwd_diag.cuh"
#include "bwd_scalarA.cuh"

using namespace selscan;

// Device-side error word: bounded waits that give up OR a bit in here.
__device__ unsigned int g_selscan_err = 0;

// Kernels launched by this library in this process (selscan_launch_count).
static std::atomic<unsigned long long> g_launches{0};

// Status of the launch just made; counts it when it succeeded.
static cudaError_t counted_launch()
{
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess)
        g_launches.fetch_add(1, std::memory_order_relaxed);
    return e;
}

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int sm_count = 0;
    unsigned int *err = nullptr;
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];
cudaMemPool_t g_pool[kMaxDevices] = {};  // scratch pools, created on first use
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

unsigned long long default_timeout_ns()
{
    // Upper bound for any single wait inside a kernel.  Normal waits last
    // microseconds; the bound only matters if something is broken.
    static unsigned long long v = [] {
        const char *e = std::getenv("SELSCAN_WAIT_TIMEOUT_MS");
        unsigned long long ms = e ? std::strtoull(e, nullptr, 10) : 2000ull;
        if (ms == 0)
            ms = 2000ull;
        return ms * 1000000ull;
    }();
    return v;
}

selscan_status device_setup(int *dev_out, DeviceInfo **info_out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return SELSCAN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &di = g_dev[dev];
    if (!di.ready) {
        if (cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess)
            return SELSCAN_ERR_CUDA;
        if (cudaGetSymbolAddress(reinterpret_cast<void **>(&di.err), g_selscan_err) !=
            cudaSuccess)
            return SELSCAN_ERR_CUDA;
        di.ready = true;
    }
    if (!g_encode) {
        cudaDriverEntryPointQueryResult q;
        void *fn = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return SELSCAN_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *dev_out = dev;
    *info_out = &di;
    return SELSCAN_OK;
}

// Stream-ordered scratch from a pool of the library's own on the current
// device.  Its release threshold keeps freed memory mapped: the device's
// default pool hands memory back to the driver at every synchronisation, so
// the next call would map the backward checkpoints (hundreds of MB) again.
// selscan_release_scratch() trims the pools.
cudaError_t scratch_alloc(void **p, size_t bytes, cudaStream_t stream)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    cudaMemPool_t pool = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!g_pool[dev]) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.handleTypes = cudaMemHandleTypeNone;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            cudaMemPool_t np = nullptr;
            if ((e = cudaMemPoolCreate(&np, &props)) != cudaSuccess)
                return e;
            uint64_t keep = UINT64_MAX;
            if ((e = cudaMemPoolSetAttribute(np, cudaMemPoolAttrReleaseThreshold, &keep)) !=
                cudaSuccess) {
                cudaMemPoolDestroy(np);
                return e;
            }
            g_pool[dev] = np;
        }
        pool = g_pool[dev];
    }
    return cudaMallocFromPoolAsync(p, bytes, pool, stream);
}

// Time segments per channel tile of the backward pass: `tiles` units of
// (batch row, 32 channels), `nchunks` checkpoint chunks, `slots` warps that
// can be resident at once.  At least 32 chunks per segment.  A wave of
// resident warps ends with its slowest unit, so the time goes as
// ceil(tiles * S / slots) / S: take S (at most four waves) within 2 % of the
// lowest such cost, the smallest that gives at least 1.5 waves (shorter
// units balance better over the SMs; more segments cost more aggregate
// work).  With 1184 slots (148 SMs) this picks 7 segments for B4 D5120
// L4096 (4.05 ms; 6 or 8: 4.25-4.45 ms) and 6 for B8 D1536 L2048 (1.30 ms;
// 3: 1.37 ms).
int64_t bwd_segments(int64_t tiles, int64_t nchunks, int64_t slots)
{
    if (tiles < 1 || nchunks < 1 || slots < 1)
        return 1;
    const int64_t max_segs = std::max<int64_t>(1, std::min<int64_t>(nchunks / 32, 4 * slots / tiles));
    auto waves = [&](int64_t s) { return (tiles * s + slots - 1) / slots; };
    double best = 1e30;
    for (int64_t s = 1; s <= max_segs; ++s)
        best = std::min(best, double(waves(s)) / double(s));
    int64_t S = 0, S_any = 0;
    for (int64_t s = 1; s <= max_segs && !S; ++s) {
        if (double(waves(s)) / double(s) > 1.02 * best)
            continue;
        if (!S_any)
            S_any = s;
        if (2 * tiles * s >= 3 * slots)
            S = s;
    }
    return S ? S : S_any;
}

// Time segments per channel tile of the forward pass: `tiles` tiles of CH
// channels, `chunks` 64-token chunks, `ctas` persistent CTAs (one per SM);
// `forced_mode` is the test hook's form (-1: automatic).  Returns the segment
// count before rounding to whole chunks per segment; *two_pass tells the
// form.  The spread rule gives about 8 units per CTA with at least 4 chunks
// per segment.
//  - Few tiles (2 tiles <= ctas) and a spread of more than one segment: the
//    two-pass form, whose segments do not wait for one another.  Its count
//    S (at most the spread, which bounds the scratch) minimises
//      2 ceil(tiles S / ctas) (ceil(chunks / S) + 0.6) + 0.144 S
//    in 64-token chunk times: two passes of whole waves of units, each a
//    segment plus its start, and the folds of the earlier segments' end
//    states that every output-pass unit runs before it starts (fitted on
//    B1 D256 L65536: 64, 128, 256 segments 0.168, 0.201, 0.290 ms).  Against
//    the spread: B1 D2048 L131072 37 segments 1.867 ms (74: 1.968), B2 D2048
//    L32768 9 segments 0.949 ms (37: 1.016), B1 D128 L303104 148 segments
//    0.327 ms (1184: 1.462), B1 D256 L65536 74 segments 0.155 ms (256: 0.291).
//  - The chained form with tiles <= ctas: one segment per tile.  A tile's
//    segments run one after another (each waits for its predecessor's
//    carry), so the call cannot be shorter than one tile's whole sequence,
//    and every extra segment adds its start and carry hand-off to that
//    chain: B8 D1536 L2048 1 segment 0.168 ms (2: 0.173, 8: 0.191), B4 D4096
//    L4096 0.327 ms (8: 0.350, 10: 0.371), B2 D5120 L4096 0.323 ms (15:
//    0.354).
//  - The chained form with more tiles than CTAs: the spread rule, which
//    balances the units over the CTAs (B4 D5120 L4096: 8 segments 0.388 ms,
//    4: 0.411, 16: 0.413; B16 D2560 L1024: 4 segments 0.215 ms, 1: 0.249).
//  A forced form keeps the spread rule, so that tests of either form cover
//  multi-segment chains and folds.
int64_t fwd_segments(int64_t tiles, int64_t chunks, int64_t ctas, int forced_mode,
                     bool can_two_pass, bool *two_pass)
{
    *two_pass = false;
    if (tiles < 1 || chunks < 1 || ctas < 1)
        return 1;
    const int64_t spread = std::max<int64_t>(
        1, std::min<int64_t>((8 * ctas + tiles - 1) / tiles, (chunks + 3) / 4));
    if (forced_mode >= 0) {
        *two_pass = can_two_pass && forced_mode == 1 && spread > 1;
        return spread;
    }
    if (can_two_pass && spread > 1 && 2 * tiles <= ctas) {
        *two_pass = true;
        double best = 1e300;
        int64_t S = spread;
        for (int64_t s = 2; s <= spread; ++s) {
            const int64_t seg = (chunks + s - 1) / s, se = (chunks + seg - 1) / seg;
            if (se != s)
                continue;  // the same split as a smaller count
            const double waves = double((tiles * se + ctas - 1) / ctas);
            const double t = 2.0 * waves * (double(seg) + 0.6) + 0.144 * double(se);
            if (t < best * (1.0 - 1e-9)) {
                best = t;
                S = se;
            }
        }
        return S;
    }
    return tiles <= ctas ? 1 : spread;
}

size_t elem_size(int32_t dt) { return dt == SELSCAN_BF16 ? 2 : 4; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t numel(const selscan_tensor *t)
{
    int64_t n = 1;
    for (int i = 0; i < t->ndim && i < 4; ++i)
        n *= t->shape[i];
    return n;
}

// Present: non-NULL descriptor whose data is non-NULL, or that holds no
// element at all (frameworks hand out NULL data for empty tensors).
bool present(const selscan_tensor *t)
{
    return t && (t->data || (t->ndim >= 1 && t->ndim <= 4 && numel(t) == 0));
}

// A "sequence" tensor: rank 3 (outer0, outer1, L) with time stride 1 and
// 16-byte aligned rows, as the bulk tensor copies need.
selscan_status check_seq(const selscan_tensor *t, int64_t d0, int64_t d1, int64_t L,
                         int32_t dtype)
{
    if (!present(t))
        return SELSCAN_ERR_NULL;
    if (t->ndim != 3 || t->shape[0] != d0 || t->shape[1] != d1 || t->shape[2] != L)
        return SELSCAN_ERR_SHAPE;
    if (t->dtype != dtype)
        return SELSCAN_ERR_DTYPE;
    if (d0 == 0 || d1 == 0 || L == 0)
        return SELSCAN_OK;  // nothing will be read or written
    if (L > 1 && t->stride[2] != 1)
        return SELSCAN_ERR_STRIDE;
    if (t->stride[0] < 0 || t->stride[1] < 0)
        return SELSCAN_ERR_STRIDE;
    const int64_t es = int64_t(elem_size(dtype));
    if (!aligned16(t->data) || ((t->stride[0] * es) & 15) || ((t->stride[1] * es) & 15))
        return SELSCAN_ERR_ALIGN;
    return SELSCAN_OK;
}

// A small fp32 parameter tensor with the given shape, contiguous.
selscan_status check_param(const selscan_tensor *t, int ndim, const int64_t *shape,
                           bool nullable)
{
    if (!t || !t->data) {
        if (nullable)
            return SELSCAN_OK;
        if (!present(t))
            return SELSCAN_ERR_NULL;
    }
    if (t->ndim != ndim)
        return SELSCAN_ERR_SHAPE;
    int64_t expect = 1, count = 1;
    for (int i = ndim - 1; i >= 0; --i) {
        if (t->shape[i] != shape[i])
            return SELSCAN_ERR_SHAPE;
        count *= shape[i];
    }
    for (int i = ndim - 1; i >= 0 && count > 0; --i) {
        if (shape[i] > 1 && t->stride[i] != expect)
            return SELSCAN_ERR_STRIDE;
        expect *= shape[i];
    }
    if (t->dtype != SELSCAN_F32)
        return SELSCAN_ERR_DTYPE;
    if ((reinterpret_cast<uintptr_t>(t->data) & 3u) != 0)
        return SELSCAN_ERR_ALIGN;
    return SELSCAN_OK;
}

const void *opt_data(const selscan_tensor *t) { return (t && t->data) ? t->data : nullptr; }

// 3-D tiled map over (L, rows, outer): box (box_t, box_rows, 1), 128-byte
// swizzle, zero fill outside the tensor.
bool encode_3d(CUtensorMap *m, const void *ptr, int32_t dtype, int64_t L, int64_t rows,
               int64_t outer, int64_t row_stride, int64_t outer_stride, int box_t,
               int box_rows)
{
    const size_t es = elem_size(dtype);
    cuuint64_t dims[3] = {cuuint64_t(L), cuuint64_t(rows), cuuint64_t(outer)};
    // strides must be non-zero multiples of 16 even where the extent is 1
    int64_t rs = row_stride * int64_t(es), os = outer_stride * int64_t(es);
    if (rows <= 1 && rs == 0)
        rs = 16 * ((L * int64_t(es) + 15) / 16);
    if (outer <= 1 && os == 0)
        os = 16 * ((rows * rs + 15) / 16);
    cuuint64_t strides[2] = {cuuint64_t(rs), cuuint64_t(os)};
    cuuint32_t box[3] = {cuuint32_t(box_t), cuuint32_t(box_rows), 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = g_encode(m,
                          dtype == SELSCAN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                          3, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int g_dbg_skip_publish = -1;  // test hook, see selscan_debug_withhold_carry

// ----------------------------------------------------- diagonal-A launch
// Kernel variants share one launcher: KIND 0 = portable kernel (fp32 and
// bf16, one lane pair per channel); KIND 1 = fast bf16 kernel (its own
// threads-per-channel constant, kFastLanesPerChannel).
template <int KIND, typename T, int CH, int STAGES, bool GATE, bool SOFTPLUS>
struct DiagVariant;

template <typename T, int CH, int STAGES, bool GATE, bool SOFTPLUS>
struct DiagVariant<0, T, CH, STAGES, GATE, SOFTPLUS> {
    static constexpr int kChunk = DiagShape<T>::kChunk;
    static constexpr int kThreads = CH * 2 + 32;
    static constexpr int kConsWarps = CH * 2 / 32;
    static constexpr int kSmem = DiagLayout<T, CH, STAGES, GATE>::kAlloc;
    static constexpr auto kernel() { return scan_diag_kernel<T, CH, STAGES, GATE>; }
};

template <int CH, int STAGES, bool GATE, bool SOFTPLUS>
struct DiagVariant<1, __nv_bfloat16, CH, STAGES, GATE, SOFTPLUS> {
    static constexpr int kChunk = 64;
    static constexpr int kThreads = kFastLanesPerChannel * CH + 32;
    static constexpr int kConsWarps = kFastLanesPerChannel * CH / 32;
    static constexpr int kSmem = DiagFastLayout<CH, STAGES, GATE>::kAlloc;
    static constexpr auto kernel() { return scan_diag_bf16_kernel<CH, STAGES, GATE, SOFTPLUS>; }
    // two-pass form: MODE 1 reads no z, MODE 2 is the full output pass
    template <int MODE>
    static constexpr auto kernel_mode()
    {
        return scan_diag_bf16_kernel<CH, STAGES, GATE && MODE != 1, SOFTPLUS, MODE>;
    }
    template <int MODE>
    static constexpr int smem_mode()
    {
        return DiagFastLayout<CH, STAGES, GATE && MODE != 1>::kAlloc;
    }
};

// Dynamic shared memory limit of a kernel, raised once per device.
template <typename K>
bool ensure_smem(K kern, int bytes, int dev, bool (&done)[kMaxDevices])
{
    if (done[dev])
        return true;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return false;
    done[dev] = true;
    return true;
}

int g_dbg_diag_mode = -1;  // test hook, see selscan_debug_diag_mode
int g_dbg_bwd_segs = 0;     // test hook, see selscan_debug_bwd_segments
int g_dbg_fwd_segs = 0;     // test hook, see selscan_debug_fwd_segments

template <int KIND, typename T, int CH, int STAGES, bool GATE, bool SOFTPLUS>
selscan_status launch_diag(const selscan_tensor *u, const selscan_tensor *delta,
                           const selscan_tensor *B, const selscan_tensor *C,
                           const selscan_tensor *z, selscan_tensor *y, DiagParams prm,
                           int sm_count, cudaStream_t stream)
{
    using V = DiagVariant<KIND, T, CH, STAGES, GATE, SOFTPLUS>;
    constexpr int TC = V::kChunk;
    constexpr int CW = V::kConsWarps;
    const int32_t dt = u->dtype;
    const int64_t batch = prm.batch, dim = prm.dim, L = prm.L;
    const int64_t Bn = kDiagN;
    // B/C may be rank 3 (batch, N, L) or rank 4 (batch, 1, N, L)
    auto bc_strides = [](const selscan_tensor *t, int64_t &rs, int64_t &bs) {
        if (t->ndim == 3) {
            rs = t->stride[1];
            bs = t->stride[0];
        } else {
            rs = t->stride[2];
            bs = t->stride[0];
        }
    };
    CUtensorMap tm_u, tm_d, tm_z, tm_B, tm_C, tm_y;
    int64_t brs, bbs, crs, cbs;
    bc_strides(B, brs, bbs);
    bc_strides(C, crs, cbs);
    bool ok = encode_3d(&tm_u, u->data, dt, L, dim, batch, u->stride[1], u->stride[0], TC, CH) &&
              encode_3d(&tm_d, delta->data, dt, L, dim, batch, delta->stride[1],
                        delta->stride[0], TC, CH) &&
              encode_3d(&tm_B, B->data, dt, L, Bn, batch, brs, bbs, TC, kDiagN) &&
              encode_3d(&tm_C, C->data, dt, L, Bn, batch, crs, cbs, TC, kDiagN) &&
              encode_3d(&tm_y, y->data, dt, L, dim, batch, y->stride[1], y->stride[0], TC, CH);
    if (ok && GATE)
        ok = encode_3d(&tm_z, z->data, dt, L, dim, batch, z->stride[1], z->stride[0], TC, CH);
    else
        tm_z = tm_u;
    if (!ok)
        return SELSCAN_ERR_ALIGN;

    // Work decomposition: tiles of CH channels, segments of seg_len tokens.
    const int tpb = int((dim + CH - 1) / CH);
    const int G = int(batch) * tpb;
    const int ctas_max = sm_count;  // one persistent CTA per SM
    const int64_t chunks = (L + TC - 1) / TC;
    bool two_pass_plan = false;
    int64_t S = fwd_segments(G, chunks, ctas_max, g_dbg_diag_mode, KIND == 1, &two_pass_plan);
    if (g_dbg_fwd_segs > 0)
        S = std::min<int64_t>(g_dbg_fwd_segs, std::max<int64_t>(1, chunks));
    int64_t seg_chunks = (chunks + S - 1) / S;
    S = (chunks + seg_chunks - 1) / seg_chunks;
    prm.tiles_per_batch = tpb;
    prm.num_tiles = G;
    prm.seg_len = int(seg_chunks * TC);
    prm.num_segs = int(S);
    const int64_t units = int64_t(G) * S;
    if (units > 0x7fffffffll)
        return SELSCAN_ERR_UNSUPPORTED;
    prm.total_units = int(units);

    // Few tiles and several segments: a chain of carries would leave most
    // SMs waiting, so use the two-pass form (aggregates, then output).
    if constexpr (KIND == 1) {
    const bool two_pass = two_pass_plan && S > 1;
    if (two_pass) {
        int dev = 0;
        cudaGetDevice(&dev);
        const int64_t agg_units = int64_t(G) * (S - 1);  // the last segment needs none
        // scratch: 2 tickets | agg[agg_units][CH][16] | agg_sd[agg_units][CH] | h0 copy
        // Every output-pass segment reads the initial state, and segments no
        // longer wait for one another, so they read a copy: the caller's h0
        // may be the last_state buffer that the last segments overwrite.
        const size_t head = 256;
        const size_t agg_bytes = size_t(agg_units) * CH * kDiagN * 4;
        const size_t sd_bytes = ((size_t(agg_units) * CH * 4 + 255) / 256) * 256;
        const size_t h0_bytes = prm.h0 ? size_t(batch) * dim * kDiagN * 4 : 0;
        void *ws = nullptr;
        if (scratch_alloc(&ws, head + agg_bytes + sd_bytes + h0_bytes, stream) != cudaSuccess)
            return SELSCAN_ERR_CUDA;
        uint8_t *wsb = static_cast<uint8_t *>(ws);
        if (cudaMemsetAsync(wsb, 0, head, stream) != cudaSuccess ||
            (prm.h0 && cudaMemcpyAsync(wsb + head + agg_bytes + sd_bytes, prm.h0, h0_bytes,
                                       cudaMemcpyDeviceToDevice, stream) != cudaSuccess)) {
            cudaFreeAsync(ws, stream);
            return SELSCAN_ERR_CUDA;
        }
        if (prm.h0)
            prm.h0 = reinterpret_cast<const float *>(wsb + head + agg_bytes + sd_bytes);
        prm.flags = nullptr;
        prm.carry = nullptr;
        prm.agg = reinterpret_cast<float *>(wsb + head);
        prm.agg_sd = reinterpret_cast<float *>(wsb + head + agg_bytes);
        prm.dbg_skip_publish = -1;
        DiagParams p1 = prm, p2 = prm;
        p1.ticket = reinterpret_cast<unsigned int *>(wsb);
        p1.total_units = int(agg_units);
        p2.ticket = reinterpret_cast<unsigned int *>(wsb + 64);
        auto k1 = V::template kernel_mode<1>();
        auto k2 = V::template kernel_mode<2>();
        static bool done1[kMaxDevices] = {}, done2[kMaxDevices] = {};
        if (!ensure_smem(k1, V::template smem_mode<1>(), dev, done1) ||
            !ensure_smem(k2, V::template smem_mode<2>(), dev, done2)) {
            cudaFreeAsync(ws, stream);
            return SELSCAN_ERR_CUDA;
        }
        k1<<<int(std::min<int64_t>(ctas_max, agg_units)), V::kThreads,
             V::template smem_mode<1>(), stream>>>(tm_u, tm_d, tm_z, tm_B, tm_C, tm_y, p1);
        cudaError_t le = counted_launch();
        if (le == cudaSuccess) {
            k2<<<int(std::min<int64_t>(ctas_max, units)), V::kThreads,
                 V::template smem_mode<2>(), stream>>>(tm_u, tm_d, tm_z, tm_B, tm_C, tm_y, p2);
            le = counted_launch();
        }
        cudaFreeAsync(ws, stream);
        return le == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
    }
    }

    // scratch: ticket | flags[units][CW] | carry[units][CH][16]
    const size_t head = 256;
    const size_t flag_bytes = ((size_t(units) * CW * 4 + 255) / 256) * 256;
    const size_t carry_bytes = size_t(units) * CH * kDiagN * 4;
    const size_t ws_bytes = head + flag_bytes + carry_bytes;
    void *ws = nullptr;
    if (scratch_alloc(&ws, ws_bytes, stream) != cudaSuccess)
        return SELSCAN_ERR_CUDA;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    if (cudaMemsetAsync(wsb, 0, head + flag_bytes, stream) != cudaSuccess) {
        cudaFreeAsync(ws, stream);
        return SELSCAN_ERR_CUDA;
    }
    prm.ticket = reinterpret_cast<unsigned int *>(wsb);
    prm.flags = reinterpret_cast<unsigned int *>(wsb + head);
    prm.carry = reinterpret_cast<float *>(wsb + head + flag_bytes);
    prm.dbg_skip_publish = g_dbg_skip_publish;

    auto kern = V::kernel();
    static bool attr_set[kMaxDevices] = {};  // per instantiation and device
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 V::kSmem) != cudaSuccess) {
            cudaFreeAsync(ws, stream);
            return SELSCAN_ERR_CUDA;
        }
        attr_set[dev] = true;
    }
    const int grid = int(std::min<int64_t>(ctas_max, units));
    kern<<<grid, V::kThreads, V::kSmem, stream>>>(tm_u, tm_d, tm_z, tm_B, tm_C, tm_y, prm);
    const cudaError_t le = counted_launch();
    cudaFreeAsync(ws, stream);
    return le == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
}

}  // namespace

extern "C" {

const char *selscan_strerror(selscan_status s)
{
    switch (s) {
    case SELSCAN_OK: return "ok";
    case SELSCAN_ERR_NULL: return "required pointer is NULL";
    case SELSCAN_ERR_SHAPE: return "tensor ranks or sizes disagree";
    case SELSCAN_ERR_STRIDE: return "unsupported strides (time stride must be 1)";
    case SELSCAN_ERR_DTYPE: return "unsupported element type";
    case SELSCAN_ERR_ALIGN: return "pointer or row stride not 16-byte aligned";
    case SELSCAN_ERR_UNSUPPORTED: return "valid arguments, but this size is not built";
    case SELSCAN_ERR_CUDA: return "CUDA runtime error";
    case SELSCAN_ERR_TIMEOUT: return "a device-side wait timed out";
    }
    return "unknown status";
}

int selscan_version(void) { return SELSCAN_VERSION; }

unsigned long long selscan_launch_count(void)
{
    return g_launches.load(std::memory_order_relaxed);
}

selscan_status selscan_release_scratch(void)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    for (int d = 0; d < kMaxDevices; ++d)
        if (g_pool[d] && cudaMemPoolTrimTo(g_pool[d], 0) != cudaSuccess)
            return SELSCAN_ERR_CUDA;
    return SELSCAN_OK;
}

// Test hook (not part of the public header's stable surface): withhold the
// carry flag of one work unit so that its successor's bounded wait expires.
// -1 switches it off.
void selscan_debug_diag_mode(int mode) { g_dbg_diag_mode = mode; }

void selscan_debug_bwd_segments(int segs) { g_dbg_bwd_segs = segs < 0 ? 0 : segs; }
void selscan_debug_fwd_segments(int segs) { g_dbg_fwd_segs = segs < 0 ? 0 : segs; }

long long selscan_debug_bwd_plan(long long tiles, long long nchunks, long long slots)
{
    return bwd_segments(tiles, nchunks, slots);
}

long long selscan_debug_fwd_plan(long long tiles, long long chunks, long long ctas)
{
    bool two_pass = false;
    const int64_t S = fwd_segments(tiles, chunks, ctas, -1, true, &two_pass);
    return two_pass ? -S : S;
}

void selscan_debug_withhold_carry(int unit) { g_dbg_skip_publish = unit; }

selscan_status selscan_check(cudaStream_t stream)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess)
        return SELSCAN_ERR_CUDA;
    unsigned int err = 0;
    if (cudaMemcpyFromSymbol(&err, g_selscan_err, sizeof(err)) != cudaSuccess)
        return SELSCAN_ERR_CUDA;
    if (err) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_selscan_err, &zero, sizeof(zero));
        return SELSCAN_ERR_TIMEOUT;
    }
    return SELSCAN_OK;
}

static selscan_status fwd_impl(const selscan_tensor *u, const selscan_tensor *delta,
                               const selscan_tensor *delta_bias, int delta_softplus,
                               const selscan_tensor *A, const selscan_tensor *B,
                               const selscan_tensor *C, const selscan_tensor *D,
                               const selscan_tensor *z, const selscan_tensor *h0,
                               selscan_tensor *y, selscan_tensor *last_state,
                               cudaStream_t stream)
{
    // ---- validation (no CUDA call before it passes)
    if (!present(u) || !delta || !A || !B || !C || !y)
        return SELSCAN_ERR_NULL;
    if (u->ndim != 3)
        return SELSCAN_ERR_SHAPE;
    const int32_t dt = u->dtype;
    if (dt != SELSCAN_F32 && dt != SELSCAN_BF16)
        return SELSCAN_ERR_DTYPE;
    const int64_t batch = u->shape[0], dim = u->shape[1], L = u->shape[2];
    if (batch < 0 || dim < 0 || L < 0)
        return SELSCAN_ERR_SHAPE;
    if (!present(A))
        return SELSCAN_ERR_NULL;
    if (A->ndim != 2 || A->shape[0] != dim)
        return SELSCAN_ERR_SHAPE;
    const int64_t N = A->shape[1];
    selscan_status st;
    if ((st = check_seq(u, batch, dim, L, dt)) != SELSCAN_OK) return st;
    if ((st = check_seq(delta, batch, dim, L, dt)) != SELSCAN_OK) return st;
    if ((st = check_seq(y, batch, dim, L, dt)) != SELSCAN_OK) return st;
    if (z && z->data && (st = check_seq(z, batch, dim, L, dt)) != SELSCAN_OK) return st;
    {
        const int64_t ashape[2] = {dim, N};
        if ((st = check_param(A, 2, ashape, false)) != SELSCAN_OK) return st;
        const int64_t vshape[1] = {dim};
        if ((st = check_param(delta_bias, 1, vshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(D, 1, vshape, true)) != SELSCAN_OK) return st;
        const int64_t sshape[3] = {batch, dim, N};
        if ((st = check_param(last_state, 3, sshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(h0, 3, sshape, true)) != SELSCAN_OK) return st;
    }
    for (const selscan_tensor *t : {B, C}) {
        if (!present(t))
            return SELSCAN_ERR_NULL;
        if (t->ndim == 4) {
            if (t->shape[1] != 1)
                return SELSCAN_ERR_UNSUPPORTED;  // one group of B/C
            selscan_tensor v = *t;
            v.ndim = 3;
            v.shape[1] = t->shape[2];
            v.shape[2] = t->shape[3];
            v.stride[1] = t->stride[2];
            v.stride[2] = t->stride[3];
            if ((st = check_seq(&v, batch, N, L, dt)) != SELSCAN_OK) return st;
        } else {
            if ((st = check_seq(t, batch, N, L, dt)) != SELSCAN_OK) return st;
        }
    }
    if (N != kDiagN)
        return SELSCAN_ERR_UNSUPPORTED;
    if (batch > 65535 || dim > (int64_t(1) << 30) || L > (int64_t(1) << 31) - 1024)
        return SELSCAN_ERR_UNSUPPORTED;

    // ---- empty problems: nothing to launch
    if (batch == 0 || dim == 0)
        return SELSCAN_OK;
    if (L == 0) {
        // nothing to scan: the final state is the initial one (zero if none)
        if (last_state && last_state->data) {
            const size_t bytes = size_t(batch * dim * N) * 4;
            const cudaError_t e =
                (h0 && h0->data)
                    ? cudaMemcpyAsync(last_state->data, h0->data, bytes, cudaMemcpyDeviceToDevice,
                                      stream)
                    : cudaMemsetAsync(last_state->data, 0, bytes, stream);
            return e == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
        }
        return SELSCAN_OK;
    }

    int dev = 0;
    DeviceInfo *di = nullptr;
    if ((st = device_setup(&dev, &di)) != SELSCAN_OK)
        return st;

    DiagParams prm{};
    prm.batch = int(batch);
    prm.dim = int(dim);
    prm.L = int(L);
    prm.A = static_cast<const float *>(A->data);
    prm.delta_bias = static_cast<const float *>(opt_data(delta_bias));
    prm.Dskip = static_cast<const float *>(opt_data(D));
    prm.h0 = static_cast<const float *>(opt_data(h0));
    prm.last_state = static_cast<float *>(last_state ? last_state->data : nullptr);
    prm.softplus = delta_softplus ? 1 : 0;
    prm.timeout_ns = default_timeout_ns();
    prm.err = di->err;

    const bool gate = z && z->data;
    const int sms = di->sm_count;
    if (dt == SELSCAN_BF16) {
        if (gate)
            return prm.softplus
                       ? launch_diag<1, __nv_bfloat16, 128, 3, true, true>(u, delta, B, C, z, y, prm, sms, stream)
                       : launch_diag<1, __nv_bfloat16, 128, 3, true, false>(u, delta, B, C, z, y, prm, sms, stream);
        return prm.softplus
                   ? launch_diag<1, __nv_bfloat16, 128, 4, false, true>(u, delta, B, C, z, y, prm, sms, stream)
                   : launch_diag<1, __nv_bfloat16, 128, 4, false, false>(u, delta, B, C, z, y, prm, sms, stream);
    }
    return gate ? launch_diag<0, float, 64, 4, true, true>(u, delta, B, C, z, y, prm, sms, stream)
                : launch_diag<0, float, 64, 4, false, true>(u, delta, B, C, z, y, prm, sms, stream);
}

selscan_status selscan_fwd(const selscan_tensor *u, const selscan_tensor *delta,
                           const selscan_tensor *delta_bias, int delta_softplus,
                           const selscan_tensor *A, const selscan_tensor *B,
                           const selscan_tensor *C, const selscan_tensor *D,
                           const selscan_tensor *z, selscan_tensor *y,
                           selscan_tensor *last_state, cudaStream_t stream)
{
    return fwd_impl(u, delta, delta_bias, delta_softplus, A, B, C, D, z, nullptr, y, last_state,
                    stream);
}

selscan_status selscan_fwd_h0(const selscan_tensor *u, const selscan_tensor *delta,
                              const selscan_tensor *delta_bias, int delta_softplus,
                              const selscan_tensor *A, const selscan_tensor *B,
                              const selscan_tensor *C, const selscan_tensor *D,
                              const selscan_tensor *z, const selscan_tensor *h0,
                              selscan_tensor *y, selscan_tensor *last_state, cudaStream_t stream)
{
    return fwd_impl(u, delta, delta_bias, delta_softplus, A, B, C, D, z, h0, y, last_state,
                    stream);
}

static selscan_status scalarA_impl(const selscan_tensor *x, const selscan_tensor *dt,
                                   const selscan_tensor *dt_bias, int dt_softplus,
                                   const selscan_tensor *A, const selscan_tensor *B,
                                   const selscan_tensor *C, const selscan_tensor *D,
                                   const selscan_tensor *z, int64_t headdim,
                                   const selscan_tensor *h0, selscan_tensor *y,
                                   selscan_tensor *last_state, cudaStream_t stream)
{
    if (!present(x) || !dt || !A || !B || !C || !y)
        return SELSCAN_ERR_NULL;
    if (x->ndim != 3 || !present(A) || A->ndim != 1 || headdim <= 0)
        return SELSCAN_ERR_SHAPE;
    if (x->dtype != SELSCAN_BF16)
        return SELSCAN_ERR_DTYPE;
    const int64_t batch = x->shape[0], dim = x->shape[1], L = x->shape[2];
    const int64_t H = A->shape[0];
    if (batch < 0 || L < 0 || H <= 0 || dim != H * headdim)
        return SELSCAN_ERR_SHAPE;
    selscan_status st;
    if ((st = check_seq(x, batch, dim, L, SELSCAN_BF16)) != SELSCAN_OK) return st;
    if ((st = check_seq(y, batch, dim, L, SELSCAN_BF16)) != SELSCAN_OK) return st;
    if (z && z->data && (st = check_seq(z, batch, dim, L, SELSCAN_BF16)) != SELSCAN_OK)
        return st;
    if ((st = check_seq(dt, batch, H, L, SELSCAN_F32)) != SELSCAN_OK) return st;
    for (const selscan_tensor *t : {B, C}) {
        if (!present(t))
            return SELSCAN_ERR_NULL;
        if (t->ndim != 4 || t->shape[0] != batch || t->shape[3] != L)
            return SELSCAN_ERR_SHAPE;
        if (t->dtype != SELSCAN_BF16)
            return SELSCAN_ERR_DTYPE;
    }
    const int64_t G = B->shape[1], N = B->shape[2];
    if (C->shape[1] != G || C->shape[2] != N || G <= 0 || H % G != 0)
        return SELSCAN_ERR_SHAPE;
    for (const selscan_tensor *t : {B, C}) {
        selscan_tensor v = *t;  // view (batch, G*N, L) needs G*N rows evenly strided
        if (t->stride[1] != t->shape[2] * t->stride[2] && G > 1)
            return SELSCAN_ERR_STRIDE;
        v.ndim = 3;
        v.shape[1] = G * N;
        v.shape[2] = L;
        v.stride[1] = t->stride[2];
        v.stride[2] = t->stride[3];
        if ((st = check_seq(&v, batch, G * N, L, SELSCAN_BF16)) != SELSCAN_OK) return st;
    }
    {
        const int64_t hshape[1] = {H};
        if ((st = check_param(A, 1, hshape, false)) != SELSCAN_OK) return st;
        if ((st = check_param(dt_bias, 1, hshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(D, 1, hshape, true)) != SELSCAN_OK) return st;
        const int64_t sshape[4] = {batch, H, headdim, N};
        if ((st = check_param(last_state, 4, sshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(h0, 4, sshape, true)) != SELSCAN_OK) return st;
    }
    if (N != kSsdN || headdim != kSsdP)
        return SELSCAN_ERR_UNSUPPORTED;
    if (batch > 65535 || L > (int64_t(1) << 31) - 1024)
        return SELSCAN_ERR_UNSUPPORTED;
    if (batch == 0)
        return SELSCAN_OK;
    if (L == 0) {
        if (last_state && last_state->data) {
            const size_t bytes = size_t(batch * H * headdim * N) * 4;
            const cudaError_t e =
                (h0 && h0->data)
                    ? cudaMemcpyAsync(last_state->data, h0->data, bytes, cudaMemcpyDeviceToDevice,
                                      stream)
                    : cudaMemsetAsync(last_state->data, 0, bytes, stream);
            return e == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
        }
        return SELSCAN_OK;
    }
    int dev = 0;
    DeviceInfo *di = nullptr;
    if ((st = device_setup(&dev, &di)) != SELSCAN_OK)
        return st;

    // B/C (batch, 1, N, L) -> 3-D maps over (L, N, batch); x over (L, H*P, batch)
    // y (batch, H*P, L) is written back through the same kind of map
    CUtensorMap tm_C, tm_B, tm_X, tm_Y;
    // B/C (batch, G, N, L) viewed as (batch, G*N, L): head h loads rows g*N .. g*N+N-1
    if (!encode_3d(&tm_C, C->data, SELSCAN_BF16, L, G * N, batch, C->stride[2], C->stride[0], 64,
                   kSsdN) ||
        !encode_3d(&tm_B, B->data, SELSCAN_BF16, L, G * N, batch, B->stride[2], B->stride[0], 64,
                   kSsdN) ||
        !encode_3d(&tm_X, x->data, SELSCAN_BF16, L, dim, batch, x->stride[1], x->stride[0], 64,
                   kSsdP) ||
        !encode_3d(&tm_Y, y->data, SELSCAN_BF16, L, dim, batch, y->stride[1], y->stride[0], 64,
                   kSsdP))
        return SELSCAN_ERR_ALIGN;
    SsdParams prm{};
    prm.batch = int(batch);
    prm.H = int(H);
    prm.L = int(L);
    prm.nchunks = int((L + kSsdQ - 1) / kSsdQ);
    prm.heads_per_group = int(H / G);
    prm.dt = static_cast<const float *>(dt->data);
    prm.dt_bs = dt->stride[0];
    prm.dt_hs = dt->stride[1];
    prm.dt_bias = static_cast<const float *>(opt_data(dt_bias));
    prm.softplus = dt_softplus ? 1 : 0;
    prm.A = static_cast<const float *>(A->data);
    prm.Dskip = static_cast<const float *>(opt_data(D));
    const bool gate = z && z->data;
    prm.z = gate ? static_cast<const __nv_bfloat16 *>(z->data) : nullptr;
    prm.z_bs = gate ? z->stride[0] : 0;
    prm.z_cs = gate ? z->stride[1] : 0;
    prm.last_state = static_cast<float *>(last_state ? last_state->data : nullptr);
    prm.h0 = static_cast<const float *>(opt_data(h0));
    prm.timeout_ns = default_timeout_ns();
    prm.err = di->err;

    auto kern = gate ? ssd_scalarA_kernel<true> : ssd_scalarA_kernel<false>;
    static bool attr_set[2][kMaxDevices] = {};
    if (!attr_set[gate][dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SsdLayout::kAlloc) != cudaSuccess)
            return SELSCAN_ERR_CUDA;
        attr_set[gate][dev] = true;
    }
    const int64_t grid = batch * H;
    if (grid > 0x7fffffffll)
        return SELSCAN_ERR_UNSUPPORTED;
    kern<<<unsigned(grid), kSsdWG * 128, SsdLayout::kAlloc, stream>>>(tm_C, tm_B, tm_X, tm_Y,
                                                                       prm);
    return counted_launch() == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
}

selscan_status selscan_fwd_scalarA(const selscan_tensor *x, const selscan_tensor *dt,
                                   const selscan_tensor *dt_bias, int dt_softplus,
                                   const selscan_tensor *A, const selscan_tensor *B,
                                   const selscan_tensor *C, const selscan_tensor *D,
                                   const selscan_tensor *z, int64_t headdim, selscan_tensor *y,
                                   selscan_tensor *last_state, cudaStream_t stream)
{
    return scalarA_impl(x, dt, dt_bias, dt_softplus, A, B, C, D, z, headdim, nullptr, y,
                        last_state, stream);
}

selscan_status selscan_fwd_scalarA_h0(const selscan_tensor *x, const selscan_tensor *dt,
                                      const selscan_tensor *dt_bias, int dt_softplus,
                                      const selscan_tensor *A, const selscan_tensor *B,
                                      const selscan_tensor *C, const selscan_tensor *D,
                                      const selscan_tensor *z, int64_t headdim,
                                      const selscan_tensor *h0, selscan_tensor *y,
                                      selscan_tensor *last_state, cudaStream_t stream)
{
    return scalarA_impl(x, dt, dt_bias, dt_softplus, A, B, C, D, z, headdim, h0, y, last_state,
                        stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// selscan_fwd_noalloc: the same scan with its scratch in a static device
// array instead of stream-ordered allocations (see include/selscan.h).
// ---------------------------------------------------------------------------

// One array per GPU that loads this library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SELSCAN_NOALLOC_SCRATCH_BYTES];

namespace {

uint8_t *g_noalloc_ptr[kMaxDevices] = {};  // device address of the array

// Once per device, with that device current: the array's device address.
// (In host code the symbol name is only a stand-in, not a device address.)
selscan_status noalloc_setup(int dev, uint8_t **out)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
            return SELSCAN_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<uint8_t *>(ptr);
    }
    *out = g_noalloc_ptr[dev];
    return SELSCAN_OK;
}

template <int KIND, typename T, int CH, int STAGES, bool GATE, bool SOFTPLUS>
selscan_status launch_diag_noalloc(const selscan_tensor *u, const selscan_tensor *delta,
                                   const selscan_tensor *B, const selscan_tensor *C,
                                   const selscan_tensor *z, selscan_tensor *y, DiagParams prm,
                                   int sm_count, uint8_t *scratch, cudaStream_t stream)
{
    using V = DiagVariant<KIND, T, CH, STAGES, GATE, SOFTPLUS>;
    constexpr int TC = V::kChunk;
    constexpr int CW = V::kConsWarps;
    const int32_t dt = u->dtype;
    const int64_t batch = prm.batch, dim = prm.dim, L = prm.L;
    auto bc_strides = [](const selscan_tensor *t, int64_t &rs, int64_t &bs) {
        rs = t->ndim == 3 ? t->stride[1] : t->stride[2];
        bs = t->stride[0];
    };
    CUtensorMap tm_u, tm_d, tm_z, tm_B, tm_C, tm_y;
    int64_t brs, bbs, crs, cbs;
    bc_strides(B, brs, bbs);
    bc_strides(C, crs, cbs);
    bool ok = encode_3d(&tm_u, u->data, dt, L, dim, batch, u->stride[1], u->stride[0], TC, CH) &&
              encode_3d(&tm_d, delta->data, dt, L, dim, batch, delta->stride[1],
                        delta->stride[0], TC, CH) &&
              encode_3d(&tm_B, B->data, dt, L, kDiagN, batch, brs, bbs, TC, kDiagN) &&
              encode_3d(&tm_C, C->data, dt, L, kDiagN, batch, crs, cbs, TC, kDiagN) &&
              encode_3d(&tm_y, y->data, dt, L, dim, batch, y->stride[1], y->stride[0], TC, CH);
    if (ok && GATE)
        ok = encode_3d(&tm_z, z->data, dt, L, dim, batch, z->stride[1], z->stride[0], TC, CH);
    else
        tm_z = tm_u;
    if (!ok)
        return SELSCAN_ERR_ALIGN;

    // the work decomposition of selscan_fwd (segments, and the chained or
    // the two-pass form by the same rule)
    const int tpb = int((dim + CH - 1) / CH);
    const int G = int(batch) * tpb;
    const int ctas_max = sm_count;
    const int64_t chunks = (L + TC - 1) / TC;
    bool two_pass_plan = false;
    int64_t S = fwd_segments(G, chunks, ctas_max, g_dbg_diag_mode, KIND == 1, &two_pass_plan);
    if (g_dbg_fwd_segs > 0)
        S = std::min<int64_t>(g_dbg_fwd_segs, std::max<int64_t>(1, chunks));
    const int64_t seg_chunks = (chunks + S - 1) / S;
    S = (chunks + seg_chunks - 1) / seg_chunks;
    const int64_t units = int64_t(G) * S;
    if (units > 0x7fffffffll)
        return SELSCAN_ERR_UNSUPPORTED;
    prm.tiles_per_batch = tpb;
    prm.num_tiles = G;
    prm.seg_len = int(seg_chunks * TC);
    prm.num_segs = int(S);
    prm.total_units = int(units);
    int dev = 0;
    cudaGetDevice(&dev);

    // Few tiles and several segments: the two-pass form, as selscan_fwd
    // chooses it, with its aggregates in the static array (there is no
    // initial state to copy).
    if constexpr (KIND == 1) {
    const bool two_pass = two_pass_plan && S > 1;
    if (two_pass) {
        const int64_t agg_units = int64_t(G) * (S - 1);
        const size_t head = 256;  // two tickets
        const size_t agg_bytes = size_t(agg_units) * CH * kDiagN * 4;
        const size_t sd_bytes = ((size_t(agg_units) * CH * 4 + 255) / 256) * 256;
        if (head + agg_bytes + sd_bytes > size_t(SELSCAN_NOALLOC_SCRATCH_BYTES))
            return SELSCAN_ERR_UNSUPPORTED;  // the static array is too small for this launch
        if (cudaMemsetAsync(scratch, 0, head, stream) != cudaSuccess)
            return SELSCAN_ERR_CUDA;
        prm.flags = nullptr;
        prm.carry = nullptr;
        prm.agg = reinterpret_cast<float *>(scratch + head);
        prm.agg_sd = reinterpret_cast<float *>(scratch + head + agg_bytes);
        prm.dbg_skip_publish = -1;
        DiagParams p1 = prm, p2 = prm;
        p1.ticket = reinterpret_cast<unsigned int *>(scratch);
        p1.total_units = int(agg_units);
        p2.ticket = reinterpret_cast<unsigned int *>(scratch + 64);
        auto k1 = V::template kernel_mode<1>();
        auto k2 = V::template kernel_mode<2>();
        static bool done1[kMaxDevices] = {}, done2[kMaxDevices] = {};
        if (!ensure_smem(k1, V::template smem_mode<1>(), dev, done1) ||
            !ensure_smem(k2, V::template smem_mode<2>(), dev, done2))
            return SELSCAN_ERR_CUDA;
        k1<<<int(std::min<int64_t>(ctas_max, agg_units)), V::kThreads,
             V::template smem_mode<1>(), stream>>>(tm_u, tm_d, tm_z, tm_B, tm_C, tm_y, p1);
        cudaError_t le = counted_launch();
        if (le == cudaSuccess) {
            k2<<<int(std::min<int64_t>(ctas_max, units)), V::kThreads,
                 V::template smem_mode<2>(), stream>>>(tm_u, tm_d, tm_z, tm_B, tm_C, tm_y, p2);
            le = counted_launch();
        }
        return le == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
    }
    }

    // Only units of the first S-1 segments publish a carry and a flag.
    const int64_t linked = int64_t(G) * (S - 1);
    const size_t head = 256;
    const size_t flag_bytes = ((size_t(linked) * CW * 4 + 255) / 256) * 256;
    const size_t carry_bytes = size_t(linked) * CH * kDiagN * 4;
    if (head + flag_bytes + carry_bytes > size_t(SELSCAN_NOALLOC_SCRATCH_BYTES))
        return SELSCAN_ERR_UNSUPPORTED;  // the static array is too small for this launch
    // the previous call's ticket and flags must not leak into this one
    if (cudaMemsetAsync(scratch, 0, head + flag_bytes, stream) != cudaSuccess)
        return SELSCAN_ERR_CUDA;
    prm.ticket = reinterpret_cast<unsigned int *>(scratch);
    prm.flags = reinterpret_cast<unsigned int *>(scratch + head);
    prm.carry = reinterpret_cast<float *>(scratch + head + flag_bytes);
    prm.dbg_skip_publish = -1;

    auto kern = V::kernel();
    static bool attr_set[kMaxDevices] = {};
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 V::kSmem) != cudaSuccess)
            return SELSCAN_ERR_CUDA;
        attr_set[dev] = true;
    }
    const int grid = int(std::min<int64_t>(ctas_max, units));
    kern<<<grid, V::kThreads, V::kSmem, stream>>>(tm_u, tm_d, tm_z, tm_B, tm_C, tm_y, prm);
    return counted_launch() == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
}

}  // namespace

extern "C" selscan_status selscan_fwd_noalloc(
    const selscan_tensor *u, const selscan_tensor *delta, const selscan_tensor *delta_bias,
    int delta_softplus, const selscan_tensor *A, const selscan_tensor *B,
    const selscan_tensor *C, const selscan_tensor *D, const selscan_tensor *z,
    selscan_tensor *y, selscan_tensor *last_state, cudaStream_t stream)
{
    // ---- validation, identical rules to selscan_fwd (no CUDA call before it)
    if (!present(u) || !delta || !A || !B || !C || !y)
        return SELSCAN_ERR_NULL;
    if (u->ndim != 3)
        return SELSCAN_ERR_SHAPE;
    const int32_t dt = u->dtype;
    if (dt != SELSCAN_F32 && dt != SELSCAN_BF16)
        return SELSCAN_ERR_DTYPE;
    const int64_t batch = u->shape[0], dim = u->shape[1], L = u->shape[2];
    if (batch < 0 || dim < 0 || L < 0)
        return SELSCAN_ERR_SHAPE;
    if (!present(A))
        return SELSCAN_ERR_NULL;
    if (A->ndim != 2 || A->shape[0] != dim)
        return SELSCAN_ERR_SHAPE;
    const int64_t N = A->shape[1];
    selscan_status st;
    if ((st = check_seq(u, batch, dim, L, dt)) != SELSCAN_OK) return st;
    if ((st = check_seq(delta, batch, dim, L, dt)) != SELSCAN_OK) return st;
    if ((st = check_seq(y, batch, dim, L, dt)) != SELSCAN_OK) return st;
    if (z && z->data && (st = check_seq(z, batch, dim, L, dt)) != SELSCAN_OK) return st;
    {
        const int64_t ashape[2] = {dim, N};
        if ((st = check_param(A, 2, ashape, false)) != SELSCAN_OK) return st;
        const int64_t vshape[1] = {dim};
        if ((st = check_param(delta_bias, 1, vshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(D, 1, vshape, true)) != SELSCAN_OK) return st;
        const int64_t sshape[3] = {batch, dim, N};
        if ((st = check_param(last_state, 3, sshape, true)) != SELSCAN_OK) return st;
    }
    for (const selscan_tensor *t : {B, C}) {
        if (!present(t))
            return SELSCAN_ERR_NULL;
        if (t->ndim == 4) {
            if (t->shape[1] != 1)
                return SELSCAN_ERR_UNSUPPORTED;
            selscan_tensor v = *t;
            v.ndim = 3;
            v.shape[1] = t->shape[2];
            v.shape[2] = t->shape[3];
            v.stride[1] = t->stride[2];
            v.stride[2] = t->stride[3];
            if ((st = check_seq(&v, batch, N, L, dt)) != SELSCAN_OK) return st;
        } else {
            if ((st = check_seq(t, batch, N, L, dt)) != SELSCAN_OK) return st;
        }
    }
    if (N != kDiagN)
        return SELSCAN_ERR_UNSUPPORTED;
    if (batch > 65535 || dim > (int64_t(1) << 30) || L > (int64_t(1) << 31) - 1024)
        return SELSCAN_ERR_UNSUPPORTED;
    if (batch == 0 || dim == 0)
        return SELSCAN_OK;
    if (L == 0) {
        if (last_state && last_state->data)
            return cudaMemsetAsync(last_state->data, 0, size_t(batch * dim * N) * 4, stream) ==
                           cudaSuccess
                       ? SELSCAN_OK
                       : SELSCAN_ERR_CUDA;
        return SELSCAN_OK;
    }

    int dev = 0;
    DeviceInfo *di = nullptr;
    if ((st = device_setup(&dev, &di)) != SELSCAN_OK)
        return st;
    uint8_t *scratch = nullptr;
    if ((st = noalloc_setup(dev, &scratch)) != SELSCAN_OK)
        return st;

    DiagParams prm{};
    prm.batch = int(batch);
    prm.dim = int(dim);
    prm.L = int(L);
    prm.A = static_cast<const float *>(A->data);
    prm.delta_bias = static_cast<const float *>(opt_data(delta_bias));
    prm.Dskip = static_cast<const float *>(opt_data(D));
    prm.h0 = nullptr;
    prm.last_state = static_cast<float *>(last_state ? last_state->data : nullptr);
    prm.softplus = delta_softplus ? 1 : 0;
    prm.timeout_ns = default_timeout_ns();
    prm.err = di->err;

    const bool gate = z && z->data;
    const int sms = di->sm_count;
    if (dt == SELSCAN_BF16) {
        if (gate)
            return prm.softplus
                       ? launch_diag_noalloc<1, __nv_bfloat16, 128, 3, true, true>(
                             u, delta, B, C, z, y, prm, sms, scratch, stream)
                       : launch_diag_noalloc<1, __nv_bfloat16, 128, 3, true, false>(
                             u, delta, B, C, z, y, prm, sms, scratch, stream);
        return prm.softplus
                   ? launch_diag_noalloc<1, __nv_bfloat16, 128, 4, false, true>(
                         u, delta, B, C, z, y, prm, sms, scratch, stream)
                   : launch_diag_noalloc<1, __nv_bfloat16, 128, 4, false, false>(
                         u, delta, B, C, z, y, prm, sms, scratch, stream);
    }
    return gate ? launch_diag_noalloc<0, float, 64, 4, true, true>(u, delta, B, C, z, y, prm, sms,
                                                                    scratch, stream)
                : launch_diag_noalloc<0, float, 64, 4, false, true>(u, delta, B, C, z, y, prm,
                                                                     sms, scratch, stream);
}

// ------------------------------------------------------------ decode step
namespace {

// A per-token tensor (d0, d1): any non-negative element strides, element-
// aligned data.
selscan_status check_tok(const selscan_tensor *t, int64_t d0, int64_t d1, int32_t dtype)
{
    if (!present(t))
        return SELSCAN_ERR_NULL;
    if (t->ndim != 2 || t->shape[0] != d0 || t->shape[1] != d1)
        return SELSCAN_ERR_SHAPE;
    if (t->dtype != dtype)
        return SELSCAN_ERR_DTYPE;
    if (d0 == 0 || d1 == 0)
        return SELSCAN_OK;
    if (t->stride[0] < 0 || t->stride[1] < 0)
        return SELSCAN_ERR_STRIDE;
    if (reinterpret_cast<uintptr_t>(t->data) % elem_size(dtype))
        return SELSCAN_ERR_ALIGN;
    return SELSCAN_OK;
}

// B or C of one token: (batch, N) or (batch, G, N); returns G through *G.
selscan_status check_tok_bc(const selscan_tensor *t, int64_t batch, int64_t N, int32_t dtype,
                            int64_t *G, int64_t s[3])
{
    if (!present(t))
        return SELSCAN_ERR_NULL;
    if (t->dtype != dtype)
        return SELSCAN_ERR_DTYPE;
    if (t->ndim == 2) {
        if (t->shape[0] != batch || t->shape[1] != N)
            return SELSCAN_ERR_SHAPE;
        *G = 1;
        s[0] = t->stride[0];
        s[1] = 0;
        s[2] = t->stride[1];
    } else if (t->ndim == 3) {
        if (t->shape[0] != batch || t->shape[2] != N || t->shape[1] <= 0)
            return SELSCAN_ERR_SHAPE;
        *G = t->shape[1];
        s[0] = t->stride[0];
        s[1] = t->stride[1];
        s[2] = t->stride[2];
    } else {
        return SELSCAN_ERR_SHAPE;
    }
    if (s[0] < 0 || s[1] < 0 || s[2] < 0)
        return SELSCAN_ERR_STRIDE;
    if (numel(t) > 0 && reinterpret_cast<uintptr_t>(t->data) % elem_size(dtype))
        return SELSCAN_ERR_ALIGN;
    return SELSCAN_OK;
}

template <typename T, bool SCALAR>
cudaError_t launch_step(const StepParams &prm, int64_t batch, int tpc, cudaStream_t stream)
{
    const int64_t inner = SCALAR ? prm.headdim : prm.dim;
    const dim3 grid(unsigned((inner * tpc + 255) / 256), SCALAR ? unsigned(prm.units) : 1u,
                    unsigned(batch));
    switch (tpc) {
    case 2: step_kernel<T, 2, SCALAR><<<grid, 256, 0, stream>>>(prm); break;
    case 4: step_kernel<T, 4, SCALAR><<<grid, 256, 0, stream>>>(prm); break;
    case 8: step_kernel<T, 8, SCALAR><<<grid, 256, 0, stream>>>(prm); break;
    default: step_kernel<T, 16, SCALAR><<<grid, 256, 0, stream>>>(prm); break;
    }
    return counted_launch();
}

// Shared by the diagonal and the scalar (Mamba-2) step.  `scalar` selects
// per-head A / dt / bias / D and a (batch, H, P, N) state.
selscan_status step_impl(bool scalar, selscan_tensor *state, const selscan_tensor *u,
                         const selscan_tensor *delta, const selscan_tensor *delta_bias,
                         int delta_softplus, const selscan_tensor *A, const selscan_tensor *B,
                         const selscan_tensor *C, const selscan_tensor *D,
                         const selscan_tensor *z, int64_t headdim, selscan_tensor *y,
                         cudaStream_t stream)
{
    if (!present(state) || !present(u) || !present(delta) || !present(A) || !B || !C ||
        !present(y))
        return SELSCAN_ERR_NULL;
    const int32_t dt = u->dtype;
    if (dt != SELSCAN_F32 && dt != SELSCAN_BF16)
        return SELSCAN_ERR_DTYPE;
    if (u->ndim != 2)
        return SELSCAN_ERR_SHAPE;
    const int64_t batch = u->shape[0], dim = u->shape[1];
    if (batch < 0 || dim < 0)
        return SELSCAN_ERR_SHAPE;
    int64_t units, N;
    if (scalar) {
        if (A->ndim != 1 || headdim <= 0 || state->ndim != 4)
            return SELSCAN_ERR_SHAPE;
        units = A->shape[0];
        if (units <= 0 || dim != units * headdim)
            return SELSCAN_ERR_SHAPE;
        N = state->shape[3];
    } else {
        if (A->ndim != 2 || A->shape[0] != dim || state->ndim != 3)
            return SELSCAN_ERR_SHAPE;
        units = dim;
        headdim = 1;
        N = A->shape[1];
    }
    selscan_status st;
    if ((st = check_tok(u, batch, dim, dt)) != SELSCAN_OK) return st;
    if ((st = check_tok(y, batch, dim, dt)) != SELSCAN_OK) return st;
    if (z && z->data && (st = check_tok(z, batch, dim, dt)) != SELSCAN_OK) return st;
    if ((st = check_tok(delta, batch, units, scalar ? SELSCAN_F32 : dt)) != SELSCAN_OK)
        return st;
    int64_t G = 1, Gc = 1, sb[3], sc[3];
    if ((st = check_tok_bc(B, batch, N, dt, &G, sb)) != SELSCAN_OK) return st;
    if ((st = check_tok_bc(C, batch, N, dt, &Gc, sc)) != SELSCAN_OK) return st;
    if (Gc != G || units % G != 0)
        return SELSCAN_ERR_SHAPE;
    {
        const int64_t ushape[1] = {units};
        if ((st = check_param(delta_bias, 1, ushape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(D, 1, ushape, true)) != SELSCAN_OK) return st;
        if (scalar) {
            if ((st = check_param(A, 1, ushape, false)) != SELSCAN_OK) return st;
            const int64_t sshape[4] = {batch, units, headdim, N};
            if ((st = check_param(state, 4, sshape, false)) != SELSCAN_OK) return st;
        } else {
            const int64_t ashape[2] = {dim, N};
            if ((st = check_param(A, 2, ashape, false)) != SELSCAN_OK) return st;
            if (!aligned16(A->data))
                return SELSCAN_ERR_ALIGN;
            const int64_t sshape[3] = {batch, dim, N};
            if ((st = check_param(state, 3, sshape, false)) != SELSCAN_OK) return st;
        }
    }
    if (N != 16 && N != 32 && N != 64 && N != 128)
        return SELSCAN_ERR_UNSUPPORTED;
    if (batch == 0 || dim == 0)
        return SELSCAN_OK;
    if (!aligned16(state->data))
        return SELSCAN_ERR_ALIGN;
    const int tpc = int(N / 8);
    if (batch > 65535 || dim * tpc > (int64_t(0x7fffffff) - 255) || units > 65535)
        return SELSCAN_ERR_UNSUPPORTED;

    StepParams prm{};
    prm.dim = int(dim);
    prm.headdim = int(headdim);
    prm.units = int(units);
    prm.per_group = int(units / G);
    {
        // B and C rows readable as aligned 4-element vectors
        const int64_t es = int64_t(elem_size(dt));
        auto vec_ok = [&](const selscan_tensor *t, const int64_t s[3]) {
            return s[2] == 1 && s[0] % 4 == 0 && s[1] % 4 == 0 &&
                   reinterpret_cast<uintptr_t>(t->data) % uintptr_t(4 * es) == 0;
        };
        prm.bc_vec = vec_ok(B, sb) && vec_ok(C, sc) ? 1 : 0;
    }
    prm.u = u->data;
    prm.su0 = u->stride[0];
    prm.su1 = u->stride[1];
    prm.delta = delta->data;
    prm.sd0 = delta->stride[0];
    prm.sd1 = delta->stride[1];
    const bool gate = z && z->data;
    prm.z = gate ? z->data : nullptr;
    prm.sz0 = gate ? z->stride[0] : 0;
    prm.sz1 = gate ? z->stride[1] : 0;
    prm.y = y->data;
    prm.sy0 = y->stride[0];
    prm.sy1 = y->stride[1];
    prm.B = B->data;
    prm.sb0 = sb[0];
    prm.sb1 = sb[1];
    prm.sb2 = sb[2];
    prm.C = C->data;
    prm.sc0 = sc[0];
    prm.sc1 = sc[1];
    prm.sc2 = sc[2];
    prm.A = static_cast<const float *>(A->data);
    prm.delta_bias = static_cast<const float *>(opt_data(delta_bias));
    prm.Dskip = static_cast<const float *>(opt_data(D));
    prm.state = static_cast<float *>(state->data);
    prm.softplus = delta_softplus ? 1 : 0;

    cudaError_t e;
    if (dt == SELSCAN_BF16)
        e = scalar ? launch_step<__nv_bfloat16, true>(prm, batch, tpc, stream)
                   : launch_step<__nv_bfloat16, false>(prm, batch, tpc, stream);
    else
        e = scalar ? launch_step<float, true>(prm, batch, tpc, stream)
                   : launch_step<float, false>(prm, batch, tpc, stream);
    return e == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
}

}  // namespace

extern "C" selscan_status selscan_step(selscan_tensor *state, const selscan_tensor *u,
                                       const selscan_tensor *delta,
                                       const selscan_tensor *delta_bias, int delta_softplus,
                                       const selscan_tensor *A, const selscan_tensor *B,
                                       const selscan_tensor *C, const selscan_tensor *D,
                                       const selscan_tensor *z, selscan_tensor *y,
                                       cudaStream_t stream)
{
    return step_impl(false, state, u, delta, delta_bias, delta_softplus, A, B, C, D, z, 1, y,
                     stream);
}

extern "C" selscan_status selscan_step_scalarA(selscan_tensor *state, const selscan_tensor *x,
                                               const selscan_tensor *dt,
                                               const selscan_tensor *dt_bias, int dt_softplus,
                                               const selscan_tensor *A, const selscan_tensor *B,
                                               const selscan_tensor *C, const selscan_tensor *D,
                                               const selscan_tensor *z, int64_t headdim,
                                               selscan_tensor *y, cudaStream_t stream)
{
    return step_impl(true, state, x, dt, dt_bias, dt_softplus, A, B, C, D, z, headdim, y,
                     stream);
}

// ------------------------------------------------------------ backward
namespace {

}  // namespace

extern "C" selscan_status selscan_bwd(
    const selscan_tensor *u, const selscan_tensor *delta, const selscan_tensor *delta_bias,
    int delta_softplus, const selscan_tensor *A, const selscan_tensor *B,
    const selscan_tensor *C, const selscan_tensor *D, const selscan_tensor *z,
    const selscan_tensor *h0, const selscan_tensor *dy, const selscan_tensor *dlast,
    selscan_tensor *du, selscan_tensor *ddelta, selscan_tensor *dA, selscan_tensor *dB,
    selscan_tensor *dC, selscan_tensor *dD, selscan_tensor *dz, selscan_tensor *ddelta_bias,
    selscan_tensor *dh0, cudaStream_t stream)
{
    if (!present(u) || !present(A))
        return SELSCAN_ERR_NULL;
    if (u->ndim != 3 || A->ndim != 2)
        return SELSCAN_ERR_SHAPE;
    const int32_t dt = u->dtype;
    if (dt != SELSCAN_F32 && dt != SELSCAN_BF16)
        return SELSCAN_ERR_DTYPE;
    const int64_t batch = u->shape[0], dim = u->shape[1], L = u->shape[2];
    const int64_t N = A->shape[1];
    if (batch < 0 || dim < 0 || L < 0 || A->shape[0] != dim)
        return SELSCAN_ERR_SHAPE;
    selscan_status st;
    for (const selscan_tensor *t : {u, delta, dy, static_cast<const selscan_tensor *>(du),
                                    static_cast<const selscan_tensor *>(ddelta)})
        if ((st = check_seq(t, batch, dim, L, dt)) != SELSCAN_OK) return st;
    const bool gate = z && z->data;
    if (gate) {
        if ((st = check_seq(z, batch, dim, L, dt)) != SELSCAN_OK) return st;
        if ((st = check_seq(dz, batch, dim, L, dt)) != SELSCAN_OK) return st;
    }
    // B, C: (batch, N, L) or (batch, 1, N, L); dB, dC: (batch, N, L) fp32 contiguous
    selscan_tensor Bv{}, Cv{};
    for (int k = 0; k < 2; ++k) {
        const selscan_tensor *t = k ? C : B;
        if (!present(t))
            return SELSCAN_ERR_NULL;
        selscan_tensor v = *t;
        if (t->ndim == 4) {
            if (t->shape[1] != 1)
                return SELSCAN_ERR_UNSUPPORTED;
            v.ndim = 3;
            v.shape[1] = t->shape[2];
            v.shape[2] = t->shape[3];
            v.stride[1] = t->stride[2];
            v.stride[2] = t->stride[3];
        }
        if ((st = check_seq(&v, batch, N, L, dt)) != SELSCAN_OK) return st;
        (k ? Cv : Bv) = v;
    }
    {
        const int64_t ashape[2] = {dim, N}, vshape[1] = {dim}, sshape[3] = {batch, dim, N};
        const int64_t bcshape[3] = {batch, N, L};
        if ((st = check_param(A, 2, ashape, false)) != SELSCAN_OK) return st;
        if ((st = check_param(dA, 2, ashape, false)) != SELSCAN_OK) return st;
        if ((st = check_param(delta_bias, 1, vshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(D, 1, vshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(dD, 1, vshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(ddelta_bias, 1, vshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(h0, 3, sshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(dlast, 3, sshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(dh0, 3, sshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(dB, 3, bcshape, false)) != SELSCAN_OK) return st;
        if ((st = check_param(dC, 3, bcshape, false)) != SELSCAN_OK) return st;
    }
    if (N != kBwdN)
        return SELSCAN_ERR_UNSUPPORTED;
    if (batch > 65535 || dim > (int64_t(1) << 30) || L > (int64_t(1) << 30))
        return SELSCAN_ERR_UNSUPPORTED;
    auto zero = [&](selscan_tensor *t) {
        return (!t || !t->data || numel(t) == 0)
                   ? cudaSuccess
                   : cudaMemsetAsync(t->data, 0, size_t(numel(t)) * 4, stream);
    };
    if (batch == 0)  // dA, dD and d bias sum over no batch row: zero, not left as they were
        return zero(dA) == cudaSuccess && zero(dD) == cudaSuccess &&
                       zero(ddelta_bias) == cudaSuccess
                   ? SELSCAN_OK
                   : SELSCAN_ERR_CUDA;
    if (dim == 0)  // dB and dC sum over no channel
        return zero(dB) == cudaSuccess && zero(dC) == cudaSuccess ? SELSCAN_OK
                                                                  : SELSCAN_ERR_CUDA;

    int dev = 0;
    DeviceInfo *di = nullptr;
    if ((st = device_setup(&dev, &di)) != SELSCAN_OK)
        return st;
    // dB and dC are written whole by the final reduction (L > 0)
    if (zero(dA) != cudaSuccess || zero(dD) != cudaSuccess || zero(ddelta_bias) != cudaSuccess)
        return SELSCAN_ERR_CUDA;
    if (L == 0) {
        // nothing to walk back through: the gradient of h0 is that of the final state
        if (dh0 && dh0->data) {
            const size_t bytes = size_t(batch * dim * N) * 4;
            const cudaError_t e =
                (dlast && dlast->data)
                    ? cudaMemcpyAsync(dh0->data, dlast->data, bytes, cudaMemcpyDeviceToDevice,
                                      stream)
                    : cudaMemsetAsync(dh0->data, 0, bytes, stream);
            return e == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
        }
        return SELSCAN_OK;
    }

    BwdParams prm{};
    prm.batch = int(batch);
    prm.dim = int(dim);
    prm.L = int(L);
    prm.nchunks = int((L + kBwdT - 1) / kBwdT);
    prm.u = u->data;
    prm.u_bs = u->stride[0];
    prm.u_ds = u->stride[1];
    prm.delta = delta->data;
    prm.dl_bs = delta->stride[0];
    prm.dl_ds = delta->stride[1];
    prm.z = gate ? z->data : nullptr;
    prm.z_bs = gate ? z->stride[0] : 0;
    prm.z_ds = gate ? z->stride[1] : 0;
    prm.dy = dy->data;
    prm.dy_bs = dy->stride[0];
    prm.dy_ds = dy->stride[1];
    prm.B = Bv.data;
    prm.B_bs = Bv.stride[0];
    prm.B_ns = Bv.stride[1];
    prm.C = Cv.data;
    prm.C_bs = Cv.stride[0];
    prm.C_ns = Cv.stride[1];
    prm.A = static_cast<const float *>(A->data);
    prm.delta_bias = static_cast<const float *>(opt_data(delta_bias));
    prm.Dskip = static_cast<const float *>(opt_data(D));
    prm.h0 = static_cast<const float *>(opt_data(h0));
    prm.dlast = static_cast<const float *>(opt_data(dlast));
    prm.softplus = delta_softplus ? 1 : 0;
    prm.du = du->data;
    prm.du_bs = du->stride[0];
    prm.du_ds = du->stride[1];
    prm.ddelta = ddelta->data;
    prm.dd_bs = ddelta->stride[0];
    prm.dd_ds = ddelta->stride[1];
    prm.dz = gate ? dz->data : nullptr;
    prm.dz_bs = gate ? dz->stride[0] : 0;
    prm.dz_ds = gate ? dz->stride[1] : 0;
    prm.dA = static_cast<float *>(dA->data);
    prm.dB = static_cast<float *>(dB->data);
    prm.dC = static_cast<float *>(dC->data);
    prm.dD = static_cast<float *>(dD ? dD->data : nullptr);
    prm.dbias = static_cast<float *>(ddelta_bias ? ddelta_bias->data : nullptr);
    prm.dh0 = static_cast<float *>(dh0 ? dh0->data : nullptr);

    // Units: (batch row, 32 channels) x time segments, one warp each; the
    // segment count comes from bwd_segments.
    prm.tiles_per_batch = int((dim + 31) / 32);
    prm.tiles = int(batch) * prm.tiles_per_batch;
    {
        int per_sm = 0;
        const cudaError_t oe =
            dt == SELSCAN_BF16
                ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                      &per_sm, selscan_bwd_kernel<__nv_bfloat16>, 32, 0)
                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm,
                                                                selscan_bwd_kernel<float>, 32, 0);
        if (oe != cudaSuccess || per_sm < 1)
            per_sm = 1;
        const int64_t slots = int64_t(per_sm) * di->sm_count;
        int64_t S = g_dbg_bwd_segs > 0
                        ? std::min<int64_t>(g_dbg_bwd_segs, std::max(1, prm.nchunks))
                        : bwd_segments(prm.tiles, prm.nchunks, slots);
        const int64_t seg_chunks = (prm.nchunks + S - 1) / S;
        S = (prm.nchunks + seg_chunks - 1) / seg_chunks;
        if (int64_t(prm.tiles) * S > 0x7fffffffll)
            return SELSCAN_ERR_UNSUPPORTED;
        prm.segs = int(S);
        prm.seg_chunks = int(seg_chunks);
    }
    const int64_t units = int64_t(prm.tiles) * prm.segs;
    // scratch: checkpoints of h every kBwdT tokens [batch][dim][nchunks][16],
    // segment aggregates E, G [units][32][16] and S [units][32] (fp32)
    const size_t ck_bytes = size_t(batch) * dim * prm.nchunks * kBwdN * 4;
    const size_t agg_bytes = prm.segs > 1 ? size_t(units) * 32 * kBwdN * 4 : 0;
    const size_t s_bytes = prm.segs > 1 ? ((size_t(units) * 32 * 4 + 255) / 256) * 256 : 0;
    const int64_t bc_n = batch * kBwdN * L;           // elements of dB (and of dC)
    const size_t part_bytes = size_t(kBwdCopies) * bc_n * 4;
    void *ws = nullptr;
    if (scratch_alloc(&ws, ck_bytes + 2 * agg_bytes + s_bytes + 2 * part_bytes, stream) !=
        cudaSuccess)
        return SELSCAN_ERR_CUDA;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    prm.ckpt = reinterpret_cast<float *>(wsb);
    prm.aggE = reinterpret_cast<float *>(wsb + ck_bytes);
    prm.aggG = reinterpret_cast<float *>(wsb + ck_bytes + agg_bytes);
    prm.aggS = reinterpret_cast<float *>(wsb + ck_bytes + 2 * agg_bytes);
    prm.pB = reinterpret_cast<float *>(wsb + ck_bytes + 2 * agg_bytes + s_bytes);
    prm.pC = prm.pB + size_t(kBwdCopies) * bc_n;
    if (cudaMemsetAsync(prm.pB, 0, 2 * part_bytes, stream) != cudaSuccess) {
        cudaFreeAsync(ws, stream);
        return SELSCAN_ERR_CUDA;
    }
    cudaError_t le = cudaSuccess;
    if (prm.segs > 1) {
        if (dt == SELSCAN_BF16)
            bwd_agg_kernel<__nv_bfloat16><<<unsigned(units), 32, 0, stream>>>(prm);
        else
            bwd_agg_kernel<float><<<unsigned(units), 32, 0, stream>>>(prm);
        le = counted_launch();
    }
    if (le == cudaSuccess) {
        if (dt == SELSCAN_BF16)
            selscan_bwd_kernel<__nv_bfloat16><<<unsigned(units), 32, 0, stream>>>(prm);
        else
            selscan_bwd_kernel<float><<<unsigned(units), 32, 0, stream>>>(prm);
        le = counted_launch();
    }
    if (le == cudaSuccess) {
        const int64_t rows = batch * L;
        const int64_t blocks = std::min<int64_t>((rows + 255) / 256, 8ll * di->sm_count);
        bwd_reduce_bc<<<unsigned(blocks), 256, 0, stream>>>(prm.pB, prm.pC, prm.dB, prm.dC,
                                                            rows, int(L));
        le = counted_launch();
    }
    cudaFreeAsync(ws, stream);
    return le == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
}

extern "C" selscan_status selscan_bwd_scalarA(
    const selscan_tensor *x, const selscan_tensor *dt, const selscan_tensor *dt_bias,
    int dt_softplus, const selscan_tensor *A, const selscan_tensor *B, const selscan_tensor *C,
    const selscan_tensor *D, const selscan_tensor *z, int64_t headdim, const selscan_tensor *h0,
    const selscan_tensor *dy, const selscan_tensor *dlast, selscan_tensor *dx,
    selscan_tensor *ddt, selscan_tensor *dA, selscan_tensor *dB, selscan_tensor *dC,
    selscan_tensor *dD, selscan_tensor *dz, selscan_tensor *ddt_bias, selscan_tensor *dh0,
    cudaStream_t stream)
{
    if (!present(x) || !present(A) || !dt || !B || !C || !dy || !dx || !ddt || !dA || !dB ||
        !dC)
        return SELSCAN_ERR_NULL;
    if (x->ndim != 3 || A->ndim != 1 || headdim <= 0)
        return SELSCAN_ERR_SHAPE;
    if (x->dtype != SELSCAN_BF16)
        return SELSCAN_ERR_DTYPE;
    const int64_t batch = x->shape[0], dim = x->shape[1], L = x->shape[2];
    const int64_t H = A->shape[0];
    if (batch < 0 || L < 0 || H <= 0 || dim != H * headdim)
        return SELSCAN_ERR_SHAPE;
    selscan_status st;
    for (const selscan_tensor *t : {x, dy, static_cast<const selscan_tensor *>(dx)})
        if ((st = check_seq(t, batch, dim, L, SELSCAN_BF16)) != SELSCAN_OK) return st;
    const bool gate = z && z->data;
    if (gate) {
        if ((st = check_seq(z, batch, dim, L, SELSCAN_BF16)) != SELSCAN_OK) return st;
        if ((st = check_seq(dz, batch, dim, L, SELSCAN_BF16)) != SELSCAN_OK) return st;
    }
    if ((st = check_seq(dt, batch, H, L, SELSCAN_F32)) != SELSCAN_OK) return st;
    if ((st = check_seq(ddt, batch, H, L, SELSCAN_F32)) != SELSCAN_OK) return st;
    for (const selscan_tensor *t : {B, C}) {
        if (!present(t))
            return SELSCAN_ERR_NULL;
        if (t->ndim != 4 || t->shape[0] != batch || t->shape[3] != L)
            return SELSCAN_ERR_SHAPE;
        if (t->dtype != SELSCAN_BF16)
            return SELSCAN_ERR_DTYPE;
        if (L > 1 && t->stride[3] != 1)
            return SELSCAN_ERR_STRIDE;
        if (t->stride[0] < 0 || t->stride[1] < 0 || t->stride[2] < 0)
            return SELSCAN_ERR_STRIDE;
        // rows are read with 16-byte loads
        if (L > 0 && (!aligned16(t->data) || ((t->stride[0] * 2) & 15) ||
                      ((t->stride[1] * 2) & 15) || ((t->stride[2] * 2) & 15)))
            return SELSCAN_ERR_ALIGN;
    }
    const int64_t G = B->shape[1], N = B->shape[2];
    if (C->shape[1] != G || C->shape[2] != N || G <= 0 || H % G != 0)
        return SELSCAN_ERR_SHAPE;
    {
        const int64_t hshape[1] = {H};
        const int64_t sshape[4] = {batch, H, headdim, N};
        const int64_t bcshape[4] = {batch, G, N, L};
        if ((st = check_param(A, 1, hshape, false)) != SELSCAN_OK) return st;
        if ((st = check_param(dA, 1, hshape, false)) != SELSCAN_OK) return st;
        if ((st = check_param(dt_bias, 1, hshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(D, 1, hshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(dD, 1, hshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(ddt_bias, 1, hshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(h0, 4, sshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(dlast, 4, sshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(dh0, 4, sshape, true)) != SELSCAN_OK) return st;
        if ((st = check_param(dB, 4, bcshape, false)) != SELSCAN_OK) return st;
        if ((st = check_param(dC, 4, bcshape, false)) != SELSCAN_OK) return st;
    }
    if (N != kSbN || headdim != kSbP)
        return SELSCAN_ERR_UNSUPPORTED;
    if (batch * H > 0x7fffffffll || batch * G > 65535 || L > (int64_t(1) << 30))
        return SELSCAN_ERR_UNSUPPORTED;
    auto zero = [&](selscan_tensor *t) {
        return (!t || !t->data || numel(t) == 0)
                   ? cudaSuccess
                   : cudaMemsetAsync(t->data, 0, size_t(numel(t)) * 4, stream);
    };
    // per-head sums start at zero; dB and dC sum over heads
    if (zero(dA) != cudaSuccess || zero(dD) != cudaSuccess || zero(ddt_bias) != cudaSuccess)
        return SELSCAN_ERR_CUDA;
    if (batch == 0)
        return SELSCAN_OK;
    if (L == 0) {
        if (dh0 && dh0->data) {
            const size_t bytes = size_t(batch * H * headdim * N) * 4;
            const cudaError_t e =
                (dlast && dlast->data)
                    ? cudaMemcpyAsync(dh0->data, dlast->data, bytes, cudaMemcpyDeviceToDevice,
                                      stream)
                    : cudaMemsetAsync(dh0->data, 0, bytes, stream);
            return e == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
        }
        return SELSCAN_OK;
    }
    int dev = 0;
    DeviceInfo *di = nullptr;
    if ((st = device_setup(&dev, &di)) != SELSCAN_OK)
        return st;

    SsdBwdParams prm{};
    prm.batch = int(batch);
    prm.H = int(H);
    prm.L = int(L);
    prm.nchunks = int((L + kSbQ - 1) / kSbQ);
    prm.heads_per_group = int(H / G);
    prm.G = int(G);
    prm.x = static_cast<const __nv_bfloat16 *>(x->data);
    prm.x_bs = x->stride[0];
    prm.x_cs = x->stride[1];
    prm.dy = static_cast<const __nv_bfloat16 *>(dy->data);
    prm.dy_bs = dy->stride[0];
    prm.dy_cs = dy->stride[1];
    prm.z = gate ? static_cast<const __nv_bfloat16 *>(z->data) : nullptr;
    prm.z_bs = gate ? z->stride[0] : 0;
    prm.z_cs = gate ? z->stride[1] : 0;
    prm.dt = static_cast<const float *>(dt->data);
    prm.dt_bs = dt->stride[0];
    prm.dt_hs = dt->stride[1];
    prm.dt_bias = static_cast<const float *>(opt_data(dt_bias));
    prm.softplus = dt_softplus ? 1 : 0;
    prm.A = static_cast<const float *>(A->data);
    prm.Dskip = static_cast<const float *>(opt_data(D));
    prm.B = static_cast<const __nv_bfloat16 *>(B->data);
    prm.B_bs = B->stride[0];
    prm.B_gs = B->stride[1];
    prm.B_ns = B->stride[2];
    prm.C = static_cast<const __nv_bfloat16 *>(C->data);
    prm.C_bs = C->stride[0];
    prm.C_gs = C->stride[1];
    prm.C_ns = C->stride[2];
    prm.h0 = static_cast<const float *>(opt_data(h0));
    prm.dlast = static_cast<const float *>(opt_data(dlast));
    prm.dx = static_cast<__nv_bfloat16 *>(dx->data);
    prm.dx_bs = dx->stride[0];
    prm.dx_cs = dx->stride[1];
    prm.dz = gate ? static_cast<__nv_bfloat16 *>(dz->data) : nullptr;
    prm.dz_bs = gate ? dz->stride[0] : 0;
    prm.dz_cs = gate ? dz->stride[1] : 0;
    prm.ddt = static_cast<float *>(ddt->data);
    prm.ddt_bs = ddt->stride[0];
    prm.ddt_hs = ddt->stride[1];
    prm.dA = static_cast<float *>(dA->data);
    prm.dD = static_cast<float *>(dD ? dD->data : nullptr);
    prm.ddt_bias = static_cast<float *>(ddt_bias ? ddt_bias->data : nullptr);
    prm.dh0 = static_cast<float *>(dh0 ? dh0->data : nullptr);

    // scratch: states at every chunk start [batch*H][nchunks+1][8192] and the
    // partial copies of dB and dC [kSbCopies][batch][G][L][N] (fp32)
    const size_t st_bytes = size_t(batch * H) * (prm.nchunks + 1) * kSbN * kSbP * 4;
    const size_t part = size_t(kSbCopies) * batch * G * L * kSbN;  // floats per tensor
    void *ws = nullptr;
    if (scratch_alloc(&ws, st_bytes + 2 * part * 4, stream) != cudaSuccess)
        return SELSCAN_ERR_CUDA;
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    prm.states = reinterpret_cast<float *>(wsb);
    prm.pB = reinterpret_cast<float *>(wsb + st_bytes);
    prm.pC = prm.pB + part;
    if (cudaMemsetAsync(prm.pB, 0, 2 * part * 4, stream) != cudaSuccess) {
        cudaFreeAsync(ws, stream);
        return SELSCAN_ERR_CUDA;
    }
    auto kern = gate ? ssd_bwd_kernel<true> : ssd_bwd_kernel<false>;
    static bool attr_set[2][kMaxDevices] = {};
    if (!attr_set[gate][dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(sizeof(SbSmem))) != cudaSuccess) {
            cudaFreeAsync(ws, stream);
            return SELSCAN_ERR_CUDA;
        }
        attr_set[gate][dev] = true;
    }
    const unsigned grid = unsigned(batch * H);
    ssd_bwd_states_kernel<<<grid, kSbThreads, 0, stream>>>(prm);
    cudaError_t le = counted_launch();
    if (le == cudaSuccess) {
        kern<<<grid, kSbWalk, sizeof(SbSmem), stream>>>(prm);
        le = counted_launch();
    }
    if (le == cudaSuccess) {
        const dim3 rg(unsigned((L + 31) / 32), unsigned(batch * G));
        ssd_bwd_reduce_bc<<<rg, 256, 0, stream>>>(prm.pB, prm.pC, static_cast<float *>(dB->data),
                                                  static_cast<float *>(dC->data), batch * G,
                                                  int(L));
        le = counted_launch();
    }
    cudaFreeAsync(ws, stream);
    return le == cudaSuccess ? SELSCAN_OK : SELSCAN_ERR_CUDA;
}
