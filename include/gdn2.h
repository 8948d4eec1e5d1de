/*
 * gdn2.h -- C ABI of the B200 (sm_100a) Gated DeltaNet-2 token mixer.
 *
 * The operation (burn-gdn2 README, docs.rs burn-gdn2 0.1.9, section
 * "Architecture"): for every batch row b and head h, a matrix state
 * S in R^{d_k x d_v} evolves token by token as
 *
 *     S_t = (I - k_t (b_t . k_t)^T) diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T
 *     o_t = S_t^T q_t
 *
 * alpha_t = exp(log_alpha_t) is a per-key-channel decay (KDA-style, as the
 * asapai.co.kr Gated DeltaNet-2 article describes), b_t the per-key-channel
 * erase gate and w_t the per-value-channel write gate (README, text under
 * the equation).  o_t reads the state after the update.  No scaling is
 * applied to q; callers pass q and k already L2-normalised (the README's
 * layer diagram applies an L2-norm before the mixer).
 *
 * Two entry points follow the README's two forward modes ("Chunk WY (train)"
 * and "Fused Recurrent (infer)"):
 *   gdn2_chunk_fwd   -- a whole sequence, chunk-parallel (chunked WY form);
 *   gdn2_decode_step -- one token per sequence against a caller-held state.
 * Their _ex forms also fuse the input prep (L2-norm of q and k, sigmoid
 * gates) and the gated RMS-norm output epilogue around the mixer, and
 * gdn2_chunk_fwd_host runs gdn2_chunk_fwd on host buffers, overlapping the
 * copies with the kernel.
 *
 * Common conventions
 * ------------------
 * Pointers are DEVICE pointers (cudaMalloc'd or torch CUDA tensors) on the
 * current device, unless a function says otherwise.  All tensors are dense,
 * contiguous, row-major:
 *     q, k, log_alpha, b : [B, T, H, d_k]
 *     v, w, o            : [B, T, H, d_v]
 *     S0, S_T, S         : [B, H, d_k, d_v]   always float32
 * Token tensors (q, k, v, log_alpha, b, w, o) share one I/O dtype `io`:
 * GDN2_IO_F32 (float32) or GDN2_IO_BF16 (bfloat16).  log_alpha holds natural
 * logarithms: any value in [-inf, 0] is accepted, -inf (alpha = 0) clearing
 * the state, and every entry point is exact (to rounding) for any decay,
 * however strong.  Positive values (alpha > 1, a growing state) are outside
 * the recurrence's domain.  Every pointer must be 16-byte aligned.
 *
 * The caller owns every buffer; the library allocates no device memory.
 * Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = the
 * legacy default stream) and the call returns without synchronising.
 *
 * Errors are returned as gdn2_status_t; nothing aborts, throws or traps.
 * Argument errors are detected on the host before any launch.  Device-side
 * waits inside the kernels are bounded: a wait that runs out records
 * GDN2_ERR_DEVICE_TIMEOUT in a per-device status word, the kernel releases
 * its tensor memory and returns; gdn2_device_status() reads and clears it.
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN2_IO_F32 = 0,
    GDN2_IO_BF16 = 1
} gdn2_io_t;

typedef enum {
    GDN2_OK = 0,
    GDN2_ERR_INVALID_ARG = 1,     /* null pointer, negative size, bad enum   */
    GDN2_ERR_UNSUPPORTED = 2,     /* valid but outside the built shapes      */
    GDN2_ERR_MISALIGNED = 3,      /* a pointer is not 16-byte aligned        */
    GDN2_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed       */
    GDN2_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait ran out      */
    GDN2_ERR_OUT_OF_BOUNDS = 6    /* debug build: a device-side range check  */
                                  /* failed (the access was skipped)         */
} gdn2_status_t;

/*
 * gdn2_chunk_fwd -- chunk-parallel forward over whole sequences.
 *
 * Computes o_t for t = 0..T-1 and the final state S_T of every (b, h) from
 * the initial state S0 (README "Architecture" equation; "Chunk WY (train)"
 * mode).  The result equals the token-by-token recurrence up to rounding:
 * the chunk form is an exact regrouping, not an approximation.
 *
 *   q, k, log_alpha, b : in,  [B, T, H, d_k], dtype io
 *   v, w               : in,  [B, T, H, d_v], dtype io
 *   S0                 : in,  [B, H, d_k, d_v] float32, or NULL for zeros
 *   o                  : out, [B, T, H, d_v], dtype io
 *   S_T                : out, [B, H, d_k, d_v] float32, or NULL (not written).
 *                        May alias S0 (each block reads its slice of S0
 *                        before it writes that slice of S_T).
 *   chunk              : chunk length: 16, 32 or 64 (README "Configuration",
 *                        chunk_size, default 64).  The result does not
 *                        depend on it beyond rounding.
 *
 * Built shapes: d_k in {64, 128}; d_v a multiple of 64 with d_v <= 512;
 * any T >= 0.  A last chunk shorter than `chunk` is processed as if padded
 * with zero tokens (q = k = v = b = w = 0, log_alpha = 0), which leaves the
 * state and the valid outputs unchanged; nothing is written past T.  T = 0 is
 * allowed: o is empty, token pointers may be NULL, and S_T = S0.
 * Other shapes return GDN2_ERR_UNSUPPORTED.
 *
 * Precision: bf16 I/O with chunk 64 runs the tensor-core kernel (bf16
 * operands, fp32 accumulation, fp32 state carried between chunks); fp32 I/O,
 * and bf16 I/O with chunk 16 or 32, run the CUDA-core kernel with fp32
 * products throughout.  o is rounded to the I/O
 * dtype (round to nearest even); S_T is fp32.
 *
 * Decay range: the chunked form scales its operands by exponentials of the
 * cumulative decay inside a chunk.  The tensor-core kernel takes those
 * relative to the middle of the chunk's range and uses the chunked form while
 * a chunk decays by at most 2^-200 (about e^-139, a mean alpha of 0.11 per
 * token) over its rows 1..63 in every channel; the first chunk that decays
 * more, and the rest of its sequence, run token by token in fp32 (slower per
 * token than the chunked form).  The
 * CUDA-core kernel makes the same choice chunk by chunk at e^-60.  Either way
 * the result is the recurrence's, for any log_alpha in [-inf, 0].
 */
gdn2_status_t gdn2_chunk_fwd(const void *q, const void *k, const void *v,
                             const void *log_alpha, const void *b, const void *w,
                             const float *S0, void *o, float *S_T,
                             int B, int T, int H, int d_k, int d_v, int chunk,
                             gdn2_io_t io, void *stream);

/*
 * gdn2_chunk_fwd_host -- gdn2_chunk_fwd on HOST buffers: the same operation,
 * shapes, dtypes and results (bit for bit: each sequence runs the same
 * kernel), with the copies in and out done by the library.
 *
 *   q, k, log_alpha, b, v, w, S0 : in,  HOST pointers, layouts as above
 *   o, S_T                       : out, HOST pointers (S_T may be NULL)
 *   workspace                    : DEVICE buffer of at least the size that
 *                                  gdn2_chunk_fwd_host_workspace returns,
 *                                  256-byte aligned, owned by the caller and
 *                                  not used by other work until this call's
 *                                  work on `stream` has completed
 *
 * The batch is cut into slices of whole sequences.  Each slice is copied in
 * on a helper stream, computed on `stream` and copied out on a second helper
 * stream, so that the copy-in of the next slice, the kernel of this one and
 * the copy-out of the previous one overlap; the helper streams start after
 * the work already on `stream`, and `stream` waits for the last copy-out
 * before anything enqueued after this call.  The two helper streams and
 * their events are created on the first call on a device and kept for the
 * life of the process; calls on one device enqueue one at a time.  Host buffers should be
 * page-locked (cudaHostAlloc, or torch's pin_memory) for the copies to run
 * asynchronously; pageable buffers give the same results, serialised.  The
 * call returns once the work is enqueued: synchronise `stream` before
 * reading o or S_T.  With T = 0 it waits for `stream` and sets S_T = S0 (or
 * zeros) on the host.  An error returned after the first copy has been
 * enqueued leaves o and S_T partly written; the work already enqueued stays
 * ordered on `stream` (it waits for both helper streams before returning), so
 * synchronising `stream` still waits for every copy of the failed call.
 */
gdn2_status_t gdn2_chunk_fwd_host(const void *q, const void *k, const void *v,
                                  const void *log_alpha, const void *b, const void *w,
                                  const float *S0, void *o, float *S_T,
                                  int B, int T, int H, int d_k, int d_v, int chunk,
                                  gdn2_io_t io, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * gdn2_chunk_fwd_host_workspace -- the device workspace, in bytes, that
 * gdn2_chunk_fwd_host needs for this shape (two slice buffers of whole
 * sequences: their token tensors, o, S0 and S_T).  Returns
 * GDN2_ERR_INVALID_ARG for a null `bytes` or a non-positive size.
 */
gdn2_status_t gdn2_chunk_fwd_host_workspace(int B, int T, int H, int d_k, int d_v,
                                            gdn2_io_t io, size_t *bytes);

/*
 * gdn2_chunk_fwd_host_noalloc -- gdn2_chunk_fwd_host without a workspace
 * argument, for callers that cannot allocate device memory themselves (a
 * plug-in handed host buffers and a CUDA context it does not own; a serving
 * process whose device memory belongs to another allocator after start-up).
 * This entry point is an addition of this library: the pages have no
 * counterpart to it.
 *
 * Arguments, shapes, results and stream behaviour are those of
 * gdn2_chunk_fwd_host (the results are equal bit for bit); the caller still
 * passes every input and output, as HOST pointers.  The staging workspace is
 * a fixed array of GDN2_NOALLOC_WORKSPACE_BYTES (64 MiB) in the library's
 * own device memory.  It is reserved when the library's device code for it
 * is loaded on a GPU (with CUDA's default lazy loading: at the first call of
 * this function on that GPU) and held until the process exits.  The call
 * itself allocates nothing.
 *
 * Shapes whose gdn2_chunk_fwd_host_workspace exceeds that size return
 * GDN2_ERR_UNSUPPORTED before anything is enqueued; use gdn2_chunk_fwd_host
 * with a larger workspace for them.  The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) and caches it: make that
 * first call before any stream capture begins on the device.
 *
 * All calls on a device share the one array, and it keeps the last call's
 * contents (nothing in it needs to start at zero).  Calls on one stream are
 * ordered and safe.  Calls whose work can overlap on the GPU (different
 * streams with no ordering between them) race on the array and corrupt each
 * other's results: order them with events or use one stream.
 */
#define GDN2_NOALLOC_WORKSPACE_BYTES (64u << 20)
gdn2_status_t gdn2_chunk_fwd_host_noalloc(const void *q, const void *k, const void *v,
                                          const void *log_alpha, const void *b, const void *w,
                                          const float *S0, void *o, float *S_T,
                                          int B, int T, int H, int d_k, int d_v, int chunk,
                                          gdn2_io_t io, void *stream);

/*
 * gdn2_chunk_fwd_cuda_core -- the same operation and arguments as
 * gdn2_chunk_fwd, always on the CUDA-core (FFMA, fp32 products) chunk
 * kernel, for either I/O dtype.  It is the fp32-I/O path of gdn2_chunk_fwd
 * and serves as an independent second GPU implementation of the chunk form.
 */
gdn2_status_t gdn2_chunk_fwd_cuda_core(const void *q, const void *k, const void *v,
                                       const void *log_alpha, const void *b, const void *w,
                                       const float *S0, void *o, float *S_T,
                                       int B, int T, int H, int d_k, int d_v, int chunk,
                                       gdn2_io_t io, void *stream);

/*
 * gdn2_decode_step -- one recurrent step for B independent sequences
 * (README "Fused Recurrent (infer)" mode; the README's inference example
 * carries the state between calls in a caller-held variable).
 *
 *   q, k, log_alpha, b : in,  [B, H, d_k], dtype io   (T = 1)
 *   v, w               : in,  [B, H, d_v], dtype io
 *   S                  : in/out, [B, H, d_k, d_v] float32, updated in place
 *                        from S_{t-1} to S_t
 *   o                  : out, [B, H, d_v], dtype io, o_t = S_t^T q_t
 *
 * Built shapes: d_k in {64, 128}; d_v a multiple of 64 with d_v <= 512.
 * The step reads and writes S exactly once.
 */
gdn2_status_t gdn2_decode_step(const void *q, const void *k, const void *v,
                               const void *log_alpha, const void *b, const void *w,
                               float *S, void *o, int B, int H, int d_k, int d_v,
                               gdn2_io_t io, void *stream);

/*
 * Fusion flags of the _ex entry points (burn-gdn2 README, "Architecture":
 * the L2-Norm drawn before the mixer; "Configuration": allow_neg_eigval).
 */
#define GDN2_FUSE_INPUT_PREP 1   /* q, k, b, w are raw projections:
                                    q <- q / sqrt(sum_i q_i^2 + l2_eps) over d_k, k likewise,
                                    b <- sigmoid(b), w <- sigmoid(w) */
#define GDN2_FUSE_NEG_EIGVAL 2   /* with INPUT_PREP: b <- 2 sigmoid(b), in (0, 2) */

/*
 * gdn2_chunk_fwd_ex / gdn2_decode_step_ex -- gdn2_chunk_fwd and
 * gdn2_decode_step generalised in two directions, with the steps the
 * README's "Architecture" diagram draws around the mixer fused into the same
 * pass.
 *
 * Value heads (README "Configuration": num_v_heads):
 *   HV           : number of value heads; 0 means HV = H.  HV must be a
 *                  multiple of H.  Value head hv reads key head
 *                  hv / (HV / H): q, k, log_alpha and b keep H heads, while
 *                  v, w, o, gate and the states carry HV heads:
 *                      v, w, o, gate : [B, T, HV, d_v]
 *                      S0, S_T, S    : [B, HV, d_k, d_v]
 *
 * Packed variable-length sequences (chunk only):
 *   cu_seqlens   : NULL, or a DEVICE int32 array [B + 1] of token offsets,
 *                  cu_seqlens[0] = 0 <= cu_seqlens[1] <= ... <= cu_seqlens[B]
 *                  = T, 4-byte aligned.  The B sequences are then packed one
 *                  after another along T (T = total tokens): every token
 *                  tensor has a leading dimension of 1 ([1, T, H, d_k],
 *                  [1, T, HV, d_v]) and sequence i is tokens
 *                  [cu_seqlens[i], cu_seqlens[i+1]), with its own state
 *                  S0[i] -> S_T[i].  Each sequence is processed exactly as
 *                  a separate call would (its last chunk may be partial;
 *                  an empty sequence has S_T[i] = S0[i]).  The offsets are
 *                  read on the device: a sequence whose offsets are out of
 *                  order or outside [0, T] is skipped (its o rows and S_T
 *                  slice are not written) and GDN2_ERR_INVALID_ARG is
 *                  recorded in the status word that gdn2_device_status()
 *                  returns.
 *
 * Fusion:
 *   flags        : 0 or GDN2_FUSE_INPUT_PREP [| GDN2_FUSE_NEG_EIGVAL].  With
 *                  INPUT_PREP the kernels read raw q, k, b, w and apply the
 *                  maps above while loading them; the recurrence is then the
 *                  one documented for gdn2_chunk_fwd on the prepared values.
 *                  l2_eps (>= 0) is only read with INPUT_PREP.  A zero q or
 *                  k row stays zero for any l2_eps.
 *   gate         : NULL, or the output gate g, laid out as o, dtype io.
 *                  Non-NULL switches the output epilogue ("Gated RMS Norm <-
 *                  SiLU Gate") on: per (token, value head) the stored output
 *                  is
 *                      y_j = o_j / sqrt(mean_j o_j^2 + norm_eps) * norm_weight_j * silu(g_j)
 *                  with silu(x) = x sigmoid(x), instead of o.
 *   norm_weight  : float32 [d_v], one weight vector shared by all heads;
 *                  required with gate (and only with it), 16-byte aligned.
 *   norm_eps     : >= 0 (the README default is 1e-5).
 *
 * The epilogue is applied before o is stored whenever one CTA holds a whole
 * d_v row (tensor-core chunk kernel: d_v = 64 or 128; decode: any d_v, the
 * CTAs of one head forming a thread-block cluster); otherwise (tensor-core
 * chunk kernel with d_v > 128, CUDA-core chunk kernel) o is normalised in
 * place by one more pass in the same stream.  With HV = H (or 0),
 * cu_seqlens = NULL, flags = 0 and gate = NULL these calls are
 * gdn2_chunk_fwd and gdn2_decode_step.  Other arguments, shapes and errors
 * as there; bad flags, a gate without norm_weight (or a weight without a
 * gate), a negative epsilon or HV not a multiple of H return
 * GDN2_ERR_INVALID_ARG.
 */
gdn2_status_t gdn2_chunk_fwd_ex(const void *q, const void *k, const void *v,
                                const void *log_alpha, const void *b, const void *w,
                                const float *S0, void *o, float *S_T,
                                int B, int T, int H, int HV, int d_k, int d_v, int chunk,
                                gdn2_io_t io, const int *cu_seqlens,
                                int flags, float l2_eps,
                                const void *gate, const float *norm_weight, float norm_eps,
                                void *stream);

gdn2_status_t gdn2_decode_step_ex(const void *q, const void *k, const void *v,
                                  const void *log_alpha, const void *b, const void *w,
                                  float *S, void *o, int B, int H, int HV, int d_k, int d_v,
                                  gdn2_io_t io, int flags, float l2_eps,
                                  const void *gate, const float *norm_weight, float norm_eps,
                                  void *stream);

/*
 * gdn2_chunk_fwd_qed / gdn2_decode_step_qed -- the recurrence with a second,
 * query-derived erase direction ("The Query Knows What to Forget",
 * mlsanity 2608.13668, abstract: a direction taken from the query and
 * orthogonal to the key that cancels what the old state holds along the
 * query).  The page gives no formula; the reading implemented is
 *
 *     r_t = q_t - ((q_t . k_t) / (k_t . k_t)) k_t     (q_t when k_t = 0)
 *     u_t = r_t / sqrt(r_t . r_t + qed_eps)          (0 when that is 0)
 *     S_t = (I - k_t (b_t . k_t)^T - u_t (c_t . u_t)^T) diag(alpha_t) S_{t-1}
 *           + k_t (w_t . v_t)^T,          o_t = S_t^T q_t
 *
 *   c       : in, [B, T, H, d_k] (decode: [B, H, d_k]), dtype io, the second
 *             erase gate (c = 0 gives gdn2_chunk_fwd / gdn2_decode_step up
 *             to rounding)
 *   qed_eps : >= 0
 * Other arguments, layouts, shapes and errors as gdn2_chunk_fwd (value heads
 * equal key heads, no packing, no fusion) and gdn2_decode_step.  The chunk
 * form takes 32 tokens per chunk (64 rows of the chunked solve: each token
 * adds its key and its query direction), so its `chunk` is fixed; with bf16
 * I/O it runs on the tensor-core kernel (bf16 operands, fp32 accumulation and
 * state), with fp32 I/O on CUDA cores with fp32 products.  The decode step
 * runs on CUDA cores.  Any log_alpha in [-inf, 0] is exact, as for
 * gdn2_chunk_fwd.
 */
gdn2_status_t gdn2_chunk_fwd_qed(const void *q, const void *k, const void *v,
                                 const void *log_alpha, const void *b, const void *c, const void *w,
                                 const float *S0, void *o, float *S_T,
                                 int B, int T, int H, int d_k, int d_v,
                                 gdn2_io_t io, float qed_eps, void *stream);

gdn2_status_t gdn2_decode_step_qed(const void *q, const void *k, const void *v,
                                   const void *log_alpha, const void *b, const void *c, const void *w,
                                   float *S, void *o, int B, int H, int d_k, int d_v,
                                   gdn2_io_t io, float qed_eps, void *stream);

/*
 * gdn2_device_status -- synchronise `stream`, then read and clear the
 * current device's status word.  Returns GDN2_OK, GDN2_ERR_DEVICE_TIMEOUT if
 * a kernel gave up on a bounded wait since the last call,
 * GDN2_ERR_INVALID_ARG if a kernel skipped a sequence with malformed
 * cu_seqlens offsets, GDN2_ERR_OUT_OF_BOUNDS (debug build only) if a range
 * check failed, or GDN2_ERR_CUDA.
 */
gdn2_status_t gdn2_device_status(void *stream);

/*
 * gdn2_selftest_wait_timeout -- exercise the bounded-wait path without any
 * fault: launches one block that waits on a shared-memory barrier which
 * nothing ever completes, with a limit of `limit_us` microseconds (1..10^6).
 * The kernel records GDN2_ERR_DEVICE_TIMEOUT and returns; the call then
 * returns gdn2_device_status(stream), i.e. GDN2_ERR_DEVICE_TIMEOUT when the
 * mechanism works.
 */
gdn2_status_t gdn2_selftest_wait_timeout(int limit_us, void *stream);

/*
 * Debug build (libgdn2_debug.so: the same sources compiled with
 * -DGDN2_DEBUG_BOUNDS).  Not an operation of the method; a build of the
 * library for finding indexing mistakes.  Every per-thread global load and
 * store of the kernels is checked against the extent of the argument buffer
 * it belongs to; the host entry points publish those extents -- computed from
 * the call's pointers and sizes and the layouts documented above -- in stream
 * order before each launch.  A failed check does not trap or fault: it skips
 * the access (a load yields 0), records GDN2_ERR_OUT_OF_BOUNDS in the status
 * word that gdn2_device_status() returns, and records the site of the first
 * failure.  TMA copies are bounded by their tensor maps.  The extents are one
 * table per device, so the debug build expects one call in flight per device
 * (calls on several streams of one device at once may check against each
 * other's extents).  In the release library the checks are compiled out.
 *
 * gdn2_debug_bounds_site -- synchronise `stream`, then read and clear the
 * site of the first failed check since the last read: *buffer is the
 * argument (0 q, 1 k, 2 v, 3 log_alpha, 4 b, 5 w, 6 c, 7 S0 (decode: S),
 * 8 S_T (decode: S), 9 o, 10 gate, 11 norm_weight, 12 cu_seqlens) and *line
 * the source line of the check; -1 and 0 when none failed.  Returns GDN2_OK,
 * GDN2_ERR_INVALID_ARG for a null output pointer, GDN2_ERR_CUDA, or
 * GDN2_ERR_UNSUPPORTED in the release library.
 *
 * gdn2_selftest_bounds -- exercise the check on addresses alone (nothing is
 * dereferenced): one thread sets a 64-byte extent for buffer 0, checks a
 * range inside it (must pass) and one that runs past its end (must fail).
 * Returns gdn2_device_status(stream): GDN2_ERR_OUT_OF_BOUNDS when the check
 * answered both correctly, GDN2_ERR_INVALID_ARG when it did not; the site then
 * reads buffer 0.  GDN2_ERR_UNSUPPORTED in the release library.
 */
gdn2_status_t gdn2_debug_bounds_site(int *buffer, int *line, void *stream);
gdn2_status_t gdn2_selftest_bounds(void *stream);

/*
 * gdn2_testing_fail_launches -- fault injection on the host, for tests of the
 * error paths (not an operation of the method).  After `pass` more kernel
 * launch sites have run normally, the next `fail` launch sites return
 * GDN2_ERR_CUDA without launching, as a launch that the driver refused would;
 * the calls that reach them return that status.  Nothing faults on the
 * device and the context stays usable.  `fail` = 0 disarms (the default).
 * Process-wide; returns GDN2_ERR_INVALID_ARG for a negative argument.
 */
gdn2_status_t gdn2_testing_fail_launches(int pass, int fail);

/* Human-readable name of a status code (static storage, never NULL). */
const char *gdn2_status_string(gdn2_status_t status);

/* Library version: major * 10000 + minor * 100 + patch. */
int gdn2_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GDN2_H */
