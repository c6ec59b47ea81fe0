/*
 * muon.h -- C interface of the B200 (sm_100a) Muon optimizer step.
 *
 * The Muon step (X thread "New training speed record for @karpathy's
 * 124M-parameter NanoGPT setup", tweets 2/8, 5/8 and 6/8) orthogonalises, for
 * every 2-D parameter, the SGD-Nesterov momentum update with a quintic
 * Newton-Schulz iteration run in bfloat16.  Per matrix of stored shape r x c:
 *
 *   buf <- beta*buf + g                       momentum, PyTorch convention
 *                                             ("07. Training neural networks",
 *                                             section "Momentum")
 *   u    = g + beta*buf   (nesterov != 0)     Nesterov look-ahead (tweet 5/8)
 *   u    = buf            (nesterov == 0)
 *   X0   = bf16(u / (||u||_F + 1e-7))         Frobenius normalisation
 *   X0  <- X0^T if r > c                      orient so that rows <= cols
 *   repeat ns_steps times (tweets 5/8, 6/8):
 *     A  = bf16(X X^T)                        fp32 accumulation
 *     B  = bf16(b*A + c*A*A)
 *     X  = bf16(a*X + B*X)
 *   X   <- X^T if r > c
 *   p   <- p + fp32(-(lr*sqrt(max(1, r/c))) * X)   the increment rounded to
 *                                             fp32, then added (a second
 *                                             fp32 rounding)
 *
 * Default coefficients (a, b, c) = (3.4445, -4.7750, 2.0315).
 *
 * Conventions for every entry point:
 *  - Matrices are fp32 (or bf16 where stated), row-major, contiguous
 *    (leading dimension = number of columns), on the current CUDA device.
 *  - "pointer arrays" are HOST arrays whose entries are DEVICE pointers.
 *  - Device pointers must be 16-byte aligned (else MUON_ERR_UNSUPPORTED).
 *  - stream is a cudaStream_t passed as void*; NULL means the legacy default
 *    stream.  Calls are asynchronous: they return after enqueueing; results
 *    are valid in stream order.  At most one call in flight per stream.
 *  - Argument errors are detected on the host before anything is enqueued
 *    and leave every buffer untouched.  n = 0 is a no-op returning MUON_OK.
 *  - Device-side failures (a bounded wait that ran out) never hang: the
 *    kernel records MUON_ERR_TIMEOUT in a per-device status word, which
 *    muon_status() reports.
 *  - NaN/Inf in one matrix's gradient propagate to that matrix only.
 *  - The library owns its scratch memory (bf16 iterates, Gram matrices,
 *    norm partials), cached per device and shape set, allocated with
 *    cudaMalloc on the first call for a shape set and freed by
 *    muon_release().  The caller owns params, grads, bufs and streams.
 *  - Thread safety: the plan cache is guarded by a mutex; distinct streams
 *    may be used from distinct host threads, but two calls sharing one shape
 *    set share scratch memory and must be ordered on the GPU (same stream).
 */
#ifndef MUON_H_
#define MUON_H_

#include <stdint.h>

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = -1,  /* null pointer, bad size, non-finite scalar   */
  MUON_ERR_UNSUPPORTED = -2,  /* misaligned pointer, no sm_100 device, ...   */
  MUON_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed            */
  MUON_ERR_NOMEM = -4,        /* cudaMalloc of scratch memory failed          */
  MUON_ERR_TIMEOUT = -5       /* a device-side bounded wait ran out           */
} muon_status_t;

/* Largest number of matrices one muon_step call groups into a single
 * launch sequence; larger n is processed in consecutive groups. */
#define MUON_MAX_GROUP 512

/*
 * muon_step -- one Muon optimizer step over n 2-D parameters.
 *
 *   params  pointer array [n]: fp32 r_i x c_i, updated in place.
 *   grads   pointer array [n]: fp32 r_i x c_i, read only.
 *   bufs    pointer array [n]: fp32 r_i x c_i momentum buffers, updated in
 *           place (the optimizer's only state).
 *   shapes  host int64 array [2n]: r_0, c_0, r_1, c_1, ...; all > 0 and
 *           r*c < 2^31.
 *   lr      learning rate (finite); beta momentum (finite).
 *   nesterov  non-zero: u = g + beta*buf; zero: u = buf.
 *   ns_steps  Newton-Schulz iterations, 0..100 (0: X = X0).
 *   coeffs  host float[3] (a, b, c), or NULL for the default triple.
 *   stream  cudaStream_t as void*.
 * params, grads and bufs must not alias one another or across matrices.
 * Returns MUON_OK or a negative muon_status_t.
 * The first call for a shape set (and for a set of parameter pointers)
 * allocates and fills the library's scratch and tensor maps, with host
 * copies.  Later calls with the same shapes and parameter pointers enqueue
 * only one memset and the kernels on the stream, so such a call can be
 * captured in a CUDA graph; every replay is one more step on the captured
 * buffers (the binding's capture_step does this).  The tensor maps of the
 * last 8 parameter-pointer sets of a shape set stay cached, so alternating
 * between up to 8 parameter copies of one shape set neither rebuilds them nor
 * synchronises; a 9th set evicts the least recently used one after
 * synchronising the stream (a CUDA graph captured with the evicted set must
 * not be replayed after that).
 */
MUON_API int muon_step(float* const* params, const float* const* grads, float* const* bufs,
              const int64_t* shapes, int n, float lr, float beta, int nesterov,
              int ns_steps, const float* coeffs, void* stream);

/*
 * muon_step_mirrored -- muon_step that also writes every updated parameter
 * matrix to n_mirrors further destinations, from the epilogue of the last
 * Newton-Schulz launch (no separate copy or collective).  For a matrix-
 * sharded step over several GPUs the destinations are the other GPUs'
 * copies of the parameters (peer memory reachable through unified virtual
 * addressing with peer access enabled), so the parameter exchange overlaps
 * the last GEMM tile by tile.  The stores are plain 16-byte global stores,
 * followed in every writing thread by a system-scope fence; readers of a
 * destination must be ordered after the call (for other GPUs: a cross-GPU
 * barrier in stream order).
 *
 *   mirrors    host pointer array [n_mirrors * n]: mirrors[k * n + i] is the
 *              k-th destination of matrix i, fp32 r_i x c_i row-major,
 *              16-byte aligned, aliasing nothing else in the call.
 *   n_mirrors  0..MUON_MAX_MIRRORS (0 is plain muon_step).
 * Other arguments as muon_step.  Needs ns_steps >= 1 and c_i % 4 == 0 for
 * every matrix (the paths that write the update from shared-memory blocks);
 * otherwise MUON_ERR_UNSUPPORTED before anything is enqueued.  The first
 * call with a new set of destination pointers synchronises the stream.
 */
#define MUON_MAX_MIRRORS 7
MUON_API int muon_step_mirrored(float* const* params, const float* const* grads,
                                float* const* bufs, const int64_t* shapes, int n, float lr,
                                float beta, int nesterov, int ns_steps, const float* coeffs,
                                float* const* mirrors, int n_mirrors, void* stream);

/*
 * muon_orthogonalize -- the Newton-Schulz part alone, for one matrix:
 *   out = NS(bf16(x / (||x||_F + 1e-7)))   (orientation handled as above)
 *
 *   x      device fp32 rows x cols (read only).
 *   out    device rows x cols, fp32 (out_is_bf16 == 0) or bf16 bits
 *          (out_is_bf16 != 0); may not alias x.
 * Same coefficient, step and stream rules as muon_step.
 */
MUON_API int muon_orthogonalize(const float* x, void* out, int out_is_bf16, int64_t rows,
                       int64_t cols, int ns_steps, const float* coeffs, void* stream);

/*
 * Stage entry points: each runs one kernel of the step on caller buffers, so
 * that every stage can be checked on its own.  bf16 buffers hold raw bf16
 * bits (uint16_t), row-major with leading dimension ld (elements, ld >= the
 * row length, ld % 8 == 0).
 */

/* muon_momentum_normalize -- the fused first kernel for n matrices:
 *   buf <- beta*buf + g;  u = g + beta*buf (or buf);
 *   x0  = bf16(u / (||u||_F + 1e-7)), written ORIENTED (min(r,c) rows,
 *         max(r,c) columns, leading dimension x0_ld[i]) to x0[i].
 * x0 is a pointer array of device bf16 buffers; x0_ld a host int64 array. */
MUON_API int muon_momentum_normalize(const float* const* grads, float* const* bufs,
                            uint16_t* const* x0, const int64_t* x0_ld,
                            const int64_t* shapes, int n, float beta, int nesterov,
                            void* stream);

/* muon_gram -- a = bf16(x x^T); x: m x n (ld_x), a: m x m (ld_a). */
MUON_API int muon_gram(const uint16_t* x, int64_t ld_x, uint16_t* a, int64_t ld_a,
              int64_t m, int64_t n, void* stream);

/* muon_poly -- b_out = bf16(cb*a + cc*(a a)); a: symmetric m x m. */
MUON_API int muon_poly(const uint16_t* a, int64_t ld_a, uint16_t* b_out, int64_t ld_b,
              int64_t m, float cb, float cc, void* stream);

/* muon_xupdate -- x_out = bf16(ca*x + b x); b: m x m, x, x_out: m x n.
 * x_out may not alias x. */
MUON_API int muon_xupdate(const uint16_t* b, int64_t ld_b, const uint16_t* x, int64_t ld_x,
                 uint16_t* x_out, int64_t ld_out, int64_t m, int64_t n, float ca,
                 void* stream);

/*
 * muon_momentum_normalize_noalloc -- the same computation as
 * muon_momentum_normalize, for callers that cannot allocate device memory
 * when they run the optimizer (a host whose device memory is all handed to
 * its own pool allocator, or a process that must not grow its footprint
 * after start-up).  It allocates nothing: its scratch (work queue, per-matrix
 * counters and flags, norm partials) lives in a fixed array of about 200 KB
 * compiled into the library, which every GPU that loads the library holds
 * until the process exits.  There is no counterpart of this entry point on
 * the pages; it is an interface choice of this library.
 *
 * Arguments as for muon_momentum_normalize, plus:
 *   dev_status  device pointer to one int owned by the caller (or NULL).  A
 *               device-side wait that runs out stores MUON_ERR_TIMEOUT there
 *               (the first error wins; the caller zeroes it).  With NULL such
 *               a failure is not reported.  muon_status() does not see it.
 * Limits: at most MUON_NOALLOC_MAX_MATRICES matrices, and at most
 * MUON_NOALLOC_MAX_ITEMS work items, where a matrix of r x c elements takes
 * 2 * ceil(ceil(r/64) * ceil(c/64) / 4) items (about 134M elements in all);
 * larger calls return MUON_ERR_UNSUPPORTED before doing anything.
 * The first call on a device takes the fixed array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call shares the one array: calls whose
 * executions overlap on the GPU race, so order them on one stream.
 */
#define MUON_NOALLOC_MAX_MATRICES 64
#define MUON_NOALLOC_MAX_ITEMS 16384
MUON_API int muon_momentum_normalize_noalloc(const float* const* grads, float* const* bufs,
                                             uint16_t* const* x0, const int64_t* x0_ld,
                                             const int64_t* shapes, int n, float beta,
                                             int nesterov, int* dev_status, void* stream);

/*
 * muon_adamw_step -- one AdamW step over n fp32 tensors of any shape, for the
 * parameters that the Muon step leaves out (embeddings, LayerNorm gains and
 * biases, linear biases).  "07. Training neural networks", section "Adam,
 * weight decay and AdamW", defines it; per element, with t = step:
 *
 *   p  <- p * (1 - lr*lambda_i)               decoupled weight decay
 *   m  <- beta1*m + (1 - beta1)*g             running average of g
 *   v  <- beta2*v + (1 - beta2)*g*g           running average of g^2
 *   p  <- p - (lr / (1 - beta1^t)) * m / (sqrt(v / (1 - beta2^t)) + eps)
 *
 *   params, grads, exp_avgs (m), exp_avg_sqs (v)
 *           pointer arrays [n] of fp32 device tensors, contiguous; params,
 *           exp_avgs and exp_avg_sqs are updated in place, grads read only.
 *           Before the first step m and v hold zeros.
 *   numels  host int64 array [n]: elements of each tensor (0 skips it;
 *           at most 2^40).
 *   decay   host byte array [n]: non-zero puts tensor i in the decayed group
 *           (lambda_i = weight_decay), zero in the no-decay group
 *           (lambda_i = 0); NULL decays every tensor.
 *   step    t >= 1, the number of this step (bias correction).
 *   lr >= 0, 0 <= beta1, beta2 < 1, eps >= 0, weight_decay >= 0, all finite;
 *           taken as doubles; the per-call constants (lr/(1-beta1^t),
 *           1/sqrt(1-beta2^t), 1-lr*lambda_i) are formed in double on the host
 *           and rounded once to fp32; the per-element arithmetic is fp32.
 *   stream  cudaStream_t as void*.
 * Pointers need only be 4-byte aligned: tensors whose four pointers are all
 * 16-byte aligned take 16-byte vector accesses, the others scalar ones.
 * Tensors must not alias one another.  NaN/Inf stay in the elements they
 * reach.  One kernel launch per 128 tensors; nothing is allocated.
 */
MUON_API int muon_adamw_step(float* const* params, const float* const* grads,
                             float* const* exp_avgs, float* const* exp_avg_sqs,
                             const int64_t* numels, const unsigned char* decay, int n,
                             int64_t step, double lr, double beta1, double beta2, double eps,
                             double weight_decay, void* stream);

/* muon_status -- synchronises the stream, then returns (and clears) the
 * device-side status of the current device: MUON_OK or MUON_ERR_TIMEOUT;
 * MUON_ERR_CUDA if the synchronisation itself failed. */
MUON_API int muon_status(void* stream);

/* muon_error_string -- static description of a status code. */
MUON_API const char* muon_error_string(int code);

/* muon_set_wait_limit_ns -- bound for every device-side wait (default
 * 2e9 ns; read from MUON_SPIN_LIMIT_NS at load time if set).  0 makes every
 * wait that does not succeed at once give up, for fault tests. */
MUON_API void muon_set_wait_limit_ns(uint64_t ns);

/* muon_workspace_bytes -- scratch bytes muon_step would allocate for this
 * shape set (host-only computation; no allocation). */
MUON_API int64_t muon_workspace_bytes(const int64_t* shapes, int n);

/*
 * Per-kernel timing, for measurement.  Between muon_profile_begin() and
 * muon_profile_end() every kernel this library launches is bracketed by a
 * pair of CUDA events recorded on its own stream (cudaEventRecord is
 * asynchronous; the kernels themselves are unchanged).  muon_profile_end()
 * synchronises those events and writes, per kernel kind, the summed device
 * time in milliseconds and the launch count:
 *   0 momentum/norm/cast   1 Gram   2 polynomial   3 X update
 *   4 X update with the fused parameter update   5 update without NS steps
 *   6 AdamW (muon_adamw_step)
 *   7 the chain launch: every Gram, polynomial and X-update phase of a step
 *     but the last update (kinds 1-3 are then used only by the stage entry
 *     points)
 * ms and launches are host arrays of at least nkinds entries.  Returns the
 * number of kinds written, or a negative status.
 */
#define MUON_PROFILE_KINDS 8
MUON_API void muon_profile_begin(void);
MUON_API int muon_profile_end(double* ms, int64_t* launches, int nkinds);

/*
 * muon_guard_check -- a check that no kernel wrote outside the scratch
 * regions it was given (this library's stand-in for a memory checker, which
 * it does not need a GPU tool for).  Every region of a cached plan (bf16
 * iterates, Gram and polynomial matrices, problem and tile tables, work
 * queue, counters, norm partials) is followed by a 256-byte guard band of a
 * fixed pattern, written when the plan is built and never written by any
 * kernel.  This call synchronises the current device and returns the number
 * of guard bytes that no longer hold the pattern, over every plan cached on
 * that device (0: intact), or a negative status.
 */
MUON_API int64_t muon_guard_check(void);

/* muon_release -- synchronises the device and frees every cached plan and
 * scratch buffer of every device this process used. */
MUON_API void muon_release(void);

/* muon_version -- library version string. */
MUON_API const char* muon_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MUON_H_ */
