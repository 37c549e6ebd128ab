/*
 * selscan.h -- C ABI of libselscan, the selective scan (S6) on NVIDIA B200
 * (sm_100a): the forward pass over a sequence (diagonal A, and scalar A in
 * the chunked matrix form on the tensor cores), the one-token decode step of
 * both, and the backward pass of the diagonal form.
 *
 * What is computed (diagonal A).  For every batch b, channel d and token t,
 * following "03 -- Modelos de espacio de estados: RWKV, S4, Mamba y el
 * selective scan" (sections "El mecanismo selectivo de Mamba",
 * "Discretizacion", "Parallel scan") and "P20 -- Mamba" (section 5,
 * "Matematica minima"):
 *
 *   delta_t = softplus(delta[b,d,t] + delta_bias[d])   (softplus optional)
 *   h_t[n]  = exp(delta_t * A[d,n]) * h_{t-1}[n] + delta_t * B[b,n,t] * u[b,d,t]
 *   y[b,d,t] = (sum_n C[b,n,t] * h_t[n] + D[d] * u[b,d,t]) * silu(z[b,d,t])
 *
 * with h_{-1} = 0 (or the given initial state), A fixed and diagonal, and
 * B, C, delta depending on the token.  The expanded state (batch, d, L, N)
 * never reaches device memory ("P20 -- Mamba", section 3: the
 * hardware-aware algorithm does not materialise the expanded state in slow
 * memory); only y and the final state are written.
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers of the current CUDA device, owned by
 *     the caller.  The library keeps no pointer after a call returns.
 *   - Calls are asynchronous on `stream`.  Scratch memory the kernels need
 *     (segment carries and flags, segment aggregates, backward checkpoints)
 *     is taken on `stream` from a stream-ordered memory pool that the
 *     library creates per device, and freed with cudaFreeAsync on the same
 *     stream (selscan_fwd_noalloc excepted).  The pool keeps freed memory
 *     for the next call; selscan_release_scratch() hands it back.
 *   - Tensors are described by selscan_tensor: element type, rank, shape and
 *     strides in ELEMENTS.  The last (time) dimension must have stride 1.
 *     Other strides may be anything that keeps rows 16-byte aligned (they
 *     are multiples of 16 bytes) and the base pointer 16-byte aligned; this
 *     is what the bulk tensor copies (TMA) require.  For a contiguous bf16
 *     tensor that means L % 8 == 0; for fp32, L % 4 == 0.  (The decode-step
 *     entry points take per-token tensors with any strides; see there.)
 *   - Validation errors are returned synchronously and nothing is launched.
 *     A failed launch returns SELSCAN_ERR_CUDA.  A device-side wait that ran
 *     out of its iteration limit is recorded on the device and reported by
 *     the next selscan_check().
 *   - There is no CPU fallback: every step runs in this library's kernels.
 */
#ifndef SELSCAN_H
#define SELSCAN_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SELSCAN_VERSION 10000 /* 1.0.0 */

#if defined(__GNUC__)
#define SELSCAN_API __attribute__((visibility("default")))
#else
#define SELSCAN_API
#endif

typedef enum {
    SELSCAN_OK = 0,
    SELSCAN_ERR_NULL = 1,        /* a required pointer is NULL            */
    SELSCAN_ERR_SHAPE = 2,       /* ranks or sizes disagree              */
    SELSCAN_ERR_STRIDE = 3,      /* time stride != 1, or bad layout      */
    SELSCAN_ERR_DTYPE = 4,       /* element type not allowed here        */
    SELSCAN_ERR_ALIGN = 5,       /* pointer / row stride not 16B aligned */
    SELSCAN_ERR_UNSUPPORTED = 6, /* valid but not built (e.g. N != 16)   */
    SELSCAN_ERR_CUDA = 7,        /* a CUDA runtime call failed           */
    SELSCAN_ERR_TIMEOUT = 8      /* a device-side wait gave up           */
} selscan_status;

typedef enum { SELSCAN_F32 = 0, SELSCAN_BF16 = 1 } selscan_dtype;

typedef struct {
    void *data;        /* device pointer (NULL allowed only where noted) */
    int32_t dtype;     /* selscan_dtype                                  */
    int32_t ndim;      /* 1..4                                           */
    int64_t shape[4];  /* sizes, outermost first                         */
    int64_t stride[4]; /* strides in elements                            */
} selscan_tensor;

/*
 * selscan_fwd -- diagonal-A selective scan forward.
 *
 *   u          (batch, D, L)   F32 or BF16; the input x of the pages
 *   delta      (batch, D, L)   same dtype as u; raw step size Delta
 *   delta_bias (D)             F32, contiguous; may be NULL
 *   delta_softplus             nonzero: delta_t = softplus(delta + bias)
 *   A          (D, N)          F32, contiguous; should be < 0 (not checked)
 *   B, C       (batch, N, L) or (batch, 1, N, L)  same dtype as u
 *   D          (D)             F32, contiguous; may be NULL (no skip term)
 *   z          (batch, D, L)   same dtype as u; may be NULL (no gate)
 *   y          (batch, D, L)   same dtype as u; written
 *   last_state (batch, D, N)   F32, contiguous; may be NULL; written
 *
 * N must be 16.  batch, D or L may be 0 (nothing is launched; when L == 0
 * last_state is zero-filled).  Internal arithmetic is fp32; y is rounded to
 * u's dtype (round to nearest even).
 */
SELSCAN_API selscan_status selscan_fwd(const selscan_tensor *u, const selscan_tensor *delta,
                           const selscan_tensor *delta_bias, int delta_softplus,
                           const selscan_tensor *A, const selscan_tensor *B,
                           const selscan_tensor *C, const selscan_tensor *D,
                           const selscan_tensor *z, selscan_tensor *y,
                           selscan_tensor *last_state, cudaStream_t stream);

/*
 * selscan_fwd_h0 -- selscan_fwd continuing from a given state: h_{-1} = h0
 * instead of zero (chunked prefill, or resuming a sequence from a saved
 * state; "Mamba-2 y state-space models", section 4.3: the layer keeps a
 * fixed-size state instead of a KV cache).  h0 (batch, D, N) F32,
 * contiguous, may be NULL (then identical to selscan_fwd).  h0 may be the
 * same buffer as last_state (in-place continuation): every channel's initial
 * state is read before its final state is written.  With L == 0,
 * last_state = h0.
 */
SELSCAN_API selscan_status selscan_fwd_h0(const selscan_tensor *u, const selscan_tensor *delta,
                              const selscan_tensor *delta_bias, int delta_softplus,
                              const selscan_tensor *A, const selscan_tensor *B,
                              const selscan_tensor *C, const selscan_tensor *D,
                              const selscan_tensor *z, const selscan_tensor *h0,
                              selscan_tensor *y, selscan_tensor *last_state,
                              cudaStream_t stream);

/*
 * selscan_fwd_scalarA -- scalar-A (Mamba-2 / SSD) selective scan forward.
 * The transition is one scalar per head times the identity ("Mamba-3: un
 * modelo de espacio de estados centrado en la inferencia", first section),
 * so the scan can be evaluated in the chunked matrix form of structured
 * state-space duality ("Mamba-2 y state-space models", section 4.2) on the
 * tensor cores.  Channel d = h * headdim + p belongs to head h.
 *
 *   x          (batch, H*P, L)  BF16
 *   dt         (batch, H, L)    F32; per-head step size
 *   dt_bias    (H)              F32; may be NULL
 *   dt_softplus                 nonzero: step = softplus(dt + dt_bias)
 *   A          (H)              F32 (< 0)
 *   B, C       (batch, G, N, L) BF16; head h reads group h / (H / G)
 *   D          (H)              F32; may be NULL
 *   z          (batch, H*P, L)  BF16; may be NULL (no gate)
 *   headdim    P
 *   y          (batch, H*P, L)  BF16; written
 *   last_state (batch, H, P, N) F32, contiguous; may be NULL; written
 *
 * Built for N = 128, P = 64 and any number of groups G dividing H; other
 * sizes return SELSCAN_ERR_UNSUPPORTED.
 */
SELSCAN_API selscan_status selscan_fwd_scalarA(const selscan_tensor *x,
                                   const selscan_tensor *dt,
                                   const selscan_tensor *dt_bias,
                                   int dt_softplus, const selscan_tensor *A,
                                   const selscan_tensor *B,
                                   const selscan_tensor *C,
                                   const selscan_tensor *D,
                                   const selscan_tensor *z, int64_t headdim,
                                   selscan_tensor *y,
                                   selscan_tensor *last_state,
                                   cudaStream_t stream);

/*
 * selscan_fwd_scalarA_h0 -- selscan_fwd_scalarA continuing from a given
 * state h0 (batch, H, P, N) F32, contiguous (may be NULL: zero state; may be
 * the same buffer as last_state).
 */
SELSCAN_API selscan_status selscan_fwd_scalarA_h0(const selscan_tensor *x,
                                      const selscan_tensor *dt,
                                      const selscan_tensor *dt_bias, int dt_softplus,
                                      const selscan_tensor *A, const selscan_tensor *B,
                                      const selscan_tensor *C, const selscan_tensor *D,
                                      const selscan_tensor *z, int64_t headdim,
                                      const selscan_tensor *h0, selscan_tensor *y,
                                      selscan_tensor *last_state, cudaStream_t stream);

/*
 * selscan_fwd_noalloc -- selscan_fwd for callers that cannot allocate device
 * memory during a call.  The paper has no counterpart; this entry point
 * exists for deployments such as fixed-footprint inference servers or
 * real-time loops that reserve all memory at start-up and forbid allocation
 * afterwards, and for systems where the stream-ordered allocator (memory
 * pools, which selscan_fwd uses for its scratch) is unavailable.
 *
 * Same arguments, layouts and results as selscan_fwd (bit for bit: the same
 * kernels with the same work decomposition, including the choice between
 * chained carries and the two-pass form for few channel tiles); the caller
 * passes all inputs and outputs.  Instead of the stream-ordered pool, the
 * scratch (tickets, carry flags and segment carries, or the two-pass form's
 * segment aggregates) lives in one file-scope device array of
 * SELSCAN_NOALLOC_SCRATCH_BYTES per GPU, which every GPU that loads the
 * library holds until the process exits.  The call makes no
 * cudaMalloc / cudaFree / allocating call; it clears the part of the array
 * that must start at zero with cudaMemsetAsync on `stream`.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents: calls that overlap on the GPU (different streams, no
 *     ordering between them) race on it.  Serialise them.
 *   - A launch whose scratch would exceed the array returns
 *     SELSCAN_ERR_UNSUPPORTED and launches nothing.  The scratch is 256
 *     bytes plus, per linked unit ((segments - 1) * channel tiles of 128
 *     bf16 or 64 fp32 channels), the carried states (64 bytes per channel)
 *     and either a flag per consumer warp (chained) or a step-size sum per
 *     channel (two-pass form).  The library's scheduling keeps the linked
 *     units below 8 * SM count: at most about 10.3 MiB on a 148-SM B200.
 */
#define SELSCAN_NOALLOC_SCRATCH_BYTES (16u << 20)
SELSCAN_API selscan_status selscan_fwd_noalloc(
    const selscan_tensor *u, const selscan_tensor *delta, const selscan_tensor *delta_bias,
    int delta_softplus, const selscan_tensor *A, const selscan_tensor *B,
    const selscan_tensor *C, const selscan_tensor *D, const selscan_tensor *z,
    selscan_tensor *y, selscan_tensor *last_state, cudaStream_t stream);

/*
 * selscan_step -- one decode step of the diagonal-A scan, state in place.
 * "03 -- Modelos de espacio de estados: RWKV, S4, Mamba y el selective
 * scan", section "Coste de inferencia": per token the layer updates a fixed
 * state and reads it out, with no dependence on the length already seen.
 * For every (b, d):
 *
 *   delta_t = softplus(delta[b,d] + delta_bias[d])   (softplus optional)
 *   state[b,d,n] = exp(delta_t * A[d,n]) * state[b,d,n] + delta_t * B[b,g,n] * u[b,d]
 *   y[b,d] = (sum_n C[b,g,n] * state[b,d,n] + D[d] * u[b,d]) * silu(z[b,d])
 *
 * which is one token of selscan_fwd_h0 with h0 = last_state = state.
 *
 *   state      (batch, D, N)  F32, contiguous, 16-byte aligned; read and
 *                             overwritten with the new state
 *   u, delta   (batch, D)     F32 or BF16 (same); any non-negative strides
 *   delta_bias (D)            F32, contiguous; may be NULL
 *   A          (D, N)         F32, contiguous, 16-byte aligned
 *   B, C       (batch, N) or (batch, G, N)  same dtype as u, any strides;
 *                             channel d reads group d / (D / G)
 *   D          (D)            F32; may be NULL
 *   z          (batch, D)     same dtype as u; may be NULL (no gate)
 *   y          (batch, D)     same dtype as u; written; must not overlap an
 *                             input other than u
 *
 * N must be 16, 32, 64 or 128.  The state must not overlap any other
 * argument.  Arithmetic is fp32 with the library's exp.
 */
SELSCAN_API selscan_status selscan_step(selscan_tensor *state, const selscan_tensor *u,
                            const selscan_tensor *delta, const selscan_tensor *delta_bias,
                            int delta_softplus, const selscan_tensor *A,
                            const selscan_tensor *B, const selscan_tensor *C,
                            const selscan_tensor *D, const selscan_tensor *z,
                            selscan_tensor *y, cudaStream_t stream);

/*
 * selscan_step_scalarA -- one decode step of the scalar-A (Mamba-2) scan,
 * state in place: for channel d = h * headdim + p,
 *
 *   state[b,h,p,n] = exp(dt_t * A[h]) * state[b,h,p,n] + dt_t * B[b,g,n] * x[b,d]
 *   y[b,d] = (sum_n C[b,g,n] * state[b,h,p,n] + D[h] * x[b,d]) * silu(z[b,d])
 *
 * with dt_t = softplus(dt[b,h] + dt_bias[h]) (softplus optional) and
 * g = h / (H / G): one token of selscan_fwd_scalarA_h0.
 *
 *   state      (batch, H, P, N) F32, contiguous, 16-byte aligned; in place
 *   x, z, y    (batch, H*P)     F32 or BF16 (same); any strides; z may be NULL
 *   dt         (batch, H)       F32
 *   dt_bias, D (H)              F32; may be NULL
 *   A          (H)              F32
 *   B, C       (batch, N) or (batch, G, N)  same dtype as x
 *
 * N must be 16, 32, 64 or 128; any headdim.
 */
SELSCAN_API selscan_status selscan_step_scalarA(selscan_tensor *state, const selscan_tensor *x,
                                    const selscan_tensor *dt, const selscan_tensor *dt_bias,
                                    int dt_softplus, const selscan_tensor *A,
                                    const selscan_tensor *B, const selscan_tensor *C,
                                    const selscan_tensor *D, const selscan_tensor *z,
                                    int64_t headdim, selscan_tensor *y, cudaStream_t stream);

/*
 * selscan_bwd -- gradients of selscan_fwd_h0 (diagonal A) for the loss
 *     sum(dy * y) + sum(dlast * last_state)
 * (training differentiates the recurrence of the forward pass; "03 --
 * Modelos de espacio de estados", sections "Discretizacion" and "Parallel
 * scan").  Walking t from the last token down with g = dLoss/dh_t:
 *   dout = dy silu(z), dz = dy out silu'(z) (out = C.h + D u before the gate),
 *   g += dout C_t;  dC_t += dout h_t;  dB_t += g delta u;  dD += dout u
 *   du = dout D + sum_n g delta B_t;  ddelta = sum_n g (A exp(delta A) h_{t-1} + B_t u)
 *   dA += g delta exp(delta A) h_{t-1};  g = exp(delta A) g
 *   d(Delta) = ddelta sigmoid(Delta + bias) with the softplus (ddelta without)
 *   d(bias) = sum d(Delta);  dh0 = g after the first token.
 *
 * Forward inputs exactly as selscan_fwd_h0 (u, delta, delta_bias, softplus,
 * A, B, C, D, z, h0; time stride 1 and 16-byte aligned rows, as there; N =
 * 16, one group of B / C).
 *   dy         (batch, D, L)  same dtype as u: gradient of y
 *   dlast      (batch, D, N)  F32, contiguous; may be NULL (zero)
 * Outputs (all overwritten):
 *   du, ddelta (batch, D, L)  same dtype as u
 *   dz         (batch, D, L)  same dtype as u; required iff z is given
 *   dA         (D, N)         F32, contiguous
 *   dB, dC     (batch, N, L)  F32, contiguous (sums over the channels)
 *   dD, ddelta_bias (D)       F32; may be NULL (not computed)
 *   dh0        (batch, D, N)  F32; may be NULL (not computed)
 * The expanded states are recomputed, never stored: a forward pass keeps h
 * every 8 tokens in stream-ordered scratch (batch * D * ceil(L/8) * 64
 * bytes, plus 2 * 8 * batch * N * L * 4 bytes of dB / dC partial sums and
 * small segment aggregates), then the chunks are walked backwards.  Sums over channels and
 * batch rows use fp32 atomics (dB and dC into 8 partial copies that a
 * last kernel adds), so the last bits of dA, dB, dC, dD and ddelta_bias
 * depend on the order of the additions.
 */
SELSCAN_API selscan_status selscan_bwd(
    const selscan_tensor *u, const selscan_tensor *delta, const selscan_tensor *delta_bias,
    int delta_softplus, const selscan_tensor *A, const selscan_tensor *B,
    const selscan_tensor *C, const selscan_tensor *D, const selscan_tensor *z,
    const selscan_tensor *h0, const selscan_tensor *dy, const selscan_tensor *dlast,
    selscan_tensor *du, selscan_tensor *ddelta, selscan_tensor *dA, selscan_tensor *dB,
    selscan_tensor *dC, selscan_tensor *dD, selscan_tensor *dz, selscan_tensor *ddelta_bias,
    selscan_tensor *dh0, cudaStream_t stream);

/*
 * selscan_bwd_scalarA -- gradients of selscan_fwd_scalarA_h0 (scalar A per
 * head, Mamba-2 / SSD form) for the loss
 *     sum(dy * y) + sum(dlast * last_state).
 * Training differentiates the forward recurrence ("03 -- Modelos de espacio
 * de estados", sections "Discretizacion" and "Parallel scan"; "P20 --
 * Mamba", section 5); with one scalar transition per head ("Mamba-3",
 * first section) the scan of a chunk of tokens is a masked product of
 * matrices ("Mamba-2 y state-space models", section 4.2), and this call
 * differentiates that chunked form from the last chunk to the first.  The
 * result equals the diagonal-A gradients of the same scan with A, the step
 * size, D and dt_bias repeated over each head's channels, summed back per
 * head.
 *
 * Forward inputs exactly as selscan_fwd_scalarA_h0 (x, dt, dt_bias,
 * dt_softplus, A, B, C, D, z, headdim, h0; B / C with time stride 1 and
 * 16-byte aligned rows, as there).
 *   dy         (batch, H*P, L)   BF16, like x: gradient of y
 *   dlast      (batch, H, P, N)  F32, contiguous; may be NULL (zero)
 * Outputs (all overwritten):
 *   dx         (batch, H*P, L)   BF16, like x
 *   dz         (batch, H*P, L)   BF16; required iff z is given
 *   ddt        (batch, H, L)     F32, time stride 1 (gradient of the raw dt)
 *   dA         (H)               F32
 *   dB, dC     (batch, G, N, L)  F32, contiguous (sums over a group's heads)
 *   dD, ddt_bias (H)             F32; may be NULL (not computed)
 *   dh0        (batch, H, P, N)  F32; may be NULL (not computed)
 * Built for N = 128, P = 64 (as the forward); other sizes return
 * SELSCAN_ERR_UNSUPPORTED.  Scratch from the stream-ordered pool: the state
 * at every 32-token chunk start (batch * H * (ceil(L/32) + 1) * 32 KiB) and
 * 8 partial copies of dB and dC (2 * 8 * batch * G * L * N * 4 bytes).
 * Sums over heads and batch rows use fp32 atomics, so the last bits of dA,
 * dB, dC, dD and ddt_bias depend on the order of the additions.
 */
SELSCAN_API selscan_status selscan_bwd_scalarA(
    const selscan_tensor *x, const selscan_tensor *dt, const selscan_tensor *dt_bias,
    int dt_softplus, const selscan_tensor *A, const selscan_tensor *B, const selscan_tensor *C,
    const selscan_tensor *D, const selscan_tensor *z, int64_t headdim, const selscan_tensor *h0,
    const selscan_tensor *dy, const selscan_tensor *dlast, selscan_tensor *dx,
    selscan_tensor *ddt, selscan_tensor *dA, selscan_tensor *dB, selscan_tensor *dC,
    selscan_tensor *dD, selscan_tensor *dz, selscan_tensor *ddt_bias, selscan_tensor *dh0,
    cudaStream_t stream);

/*
 * selscan_check -- synchronise `stream` and report device-side errors that
 * earlier calls recorded (a bounded wait that gave up returns
 * SELSCAN_ERR_TIMEOUT; the record is then cleared).  Returns
 * SELSCAN_ERR_CUDA if the synchronisation itself failed.
 */
SELSCAN_API selscan_status selscan_check(cudaStream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
SELSCAN_API const char *selscan_strerror(selscan_status status);

/* SELSCAN_VERSION of the built library. */
SELSCAN_API int selscan_version(void);

/*
 * Number of kernels this library has launched in the calling process so far
 * (all entry points, all devices).  A selscan_fwd call launches one kernel,
 * or two when it uses the two-pass form (few channel tiles, long
 * sequences); selscan_bwd launches two (three with time segments: the
 * segment aggregates, the gradient walk, the sum of the dB / dC partial
 * copies); selscan_bwd_scalarA launches three (chunk states, the chunk
 * walk, the sum of the dB / dC copies); the other entry points launch one.  Benchmarks read it around
 * a timed region to report how many of the library's kernels ran in it.
 */
SELSCAN_API unsigned long long selscan_launch_count(void);

/*
 * selscan_release_scratch -- return to the driver the scratch memory that
 * the library's pools hold but no call is using (every device the process
 * has called on).  Memory whose cudaFreeAsync has not yet run on its stream
 * is kept; synchronise the streams first to release everything.  Calls
 * after it allocate again as needed.  Returns SELSCAN_ERR_CUDA if a trim
 * failed, else SELSCAN_OK.
 */
SELSCAN_API selscan_status selscan_release_scratch(void);

#ifdef __cplusplus
}
#endif

#endif /* SELSCAN_H */
