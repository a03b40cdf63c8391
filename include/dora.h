/*
 * dora.h -- C ABI of the DoRA (weight-decomposed low-rank adaptation)
 * linear-layer hot path on NVIDIA B200 (sm_100a).
 *
 * What is computed (sources are named by page title and section):
 *
 *   LoRA update  W = W0 + s B A,  s = alpha / r
 *       ["LoRA & DoRA: The Math, Memory, and Trade-offs", section 1]
 *   DoRA weight  W' = m * (W0 + s B A) / ||W0 + s B A||, one magnitude and one
 *       Euclidean norm per OUTPUT ROW of the [d_out, d_in] weight, the norm
 *       detached from autograd  ["DoRA" (aiwiki), DoRALinear listing;
 *       "Scaling DoRA: High-Rank Adaptation via Factored Norms and Fused
 *       Kernels", Data Availability]
 *   Factored norm  n_i^2 = ||W0_i||^2 + 2 s B_i.(W0 A^T)_i + s^2 B_i G B_i^T,
 *       G = A A^T, never forming the dense product B A
 *       ["Scaling DoRA ...", section 2 "Factored Norm Computation"]
 *   Scale  g = m / max(n, eps)  ["Scaling DoRA ...", section 4, precision]
 *   Compose  y = base + (g - 1) * base + g * s * lora, with (g - 1) formed in
 *       fp32 as (m - n_c) / n_c  ["Scaling DoRA ...", section 3 numerical
 *       stability; Data Availability composition contract]
 *   Backward  d_base = g dy, d_lora = g s dy,
 *       dm = sum_t dy (base + s lora) / n_c  ["Scaling DoRA ...", section 3
 *       backward kernel]
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless a comment says "host".  The caller
 *     owns every buffer, including workspaces; the library never allocates or
 *     frees device memory.
 *   - All matrices are row-major and contiguous: W0 [d_out, d_in],
 *     A [r, d_in], B [d_out, r], activations [T, d_out] (d_out contiguous; the
 *     per-row magnitude of the weight broadcasts along the activations' last
 *     axis).  m, n, g, dm are fp32 [d_out].
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).
 *     Arguments are validated on the host before anything is launched; a
 *     rejected call launches nothing.  A launch failure returns
 *     DORA_ERR_CUDA.  A kernel that gives up on a bounded internal wait
 *     records DORA_ERR_TIMEOUT in a device status word, read (and cleared)
 *     by dora_get_device_status.
 *   - Aliasing: outputs must not overlap inputs, except y == base in
 *     dora_compose_fwd and d_base == dy in dora_compose_bwd (both
 *     element-for-element).
 *   - dtype DORA_BF16: W0, A, B and the activations are bf16; arithmetic is
 *     fp32 (tensor-core bf16 products with fp32 accumulation for the norm).
 *     dtype DORA_F32: everything fp32, CUDA-core fp32 arithmetic.
 *   - Requires an sm_100 device (B200); otherwise DORA_ERR_UNSUPPORTED.
 */
#ifndef DORA_H_
#define DORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *dora_stream_t;

typedef enum {
  DORA_OK = 0,
  DORA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad alias  */
  DORA_ERR_UNSUPPORTED = 2,   /* r > 512, not an sm_100 device, too many problems */
  DORA_ERR_WORKSPACE = 3,     /* workspace missing, too small or misaligned   */
  DORA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed         */
  DORA_ERR_TIMEOUT = 5,       /* a kernel gave up on a bounded wait           */
  DORA_ERR_BOUNDS = 6,        /* DORA_DEBUG build only: a kernel skipped a
                                 store whose computed index was out of range */
  DORA_ERR_INTERNAL = 7       /* dora_norm_plan_check: a schedule invariant
                                 does not hold (a library defect)            */
} dora_status_t;

typedef enum { DORA_F32 = 0, DORA_BF16 = 1 } dora_dtype_t;

/* Largest adapter rank (one fp32 TMEM column per rank index). */
#define DORA_MAX_RANK 512
/* Largest number of modules in one grouped norm call. */
#define DORA_MAX_GROUP 1024

/* ------------------------------------------------------------------------
 * Factored per-output-row norm  ["Scaling DoRA ...", section 2]
 *
 * n_out[i] = sqrt(max(||W0_i||^2 + 2 s B_i.(W0 A^T)_i + s^2 B_i (A A^T) B_i^T, 0))
 * and, when both m and g_out are non-NULL, g_out[i] = m[i] / max(n_out[i], eps)
 * ["Scaling DoRA ...", section 4 precision bullet; appendix B clamp].
 *
 * W0 [d_out, d_in], A [r, d_in], B [d_out, r] in dtype `dt`; 1 <= r <= 512.
 * The dense [d_out, d_in] product is never formed: on the bf16 path, W0 A^T
 * and B (s/2)(A A^T) accumulate in tensor memory and W0 is read from HBM
 * once.  Workspace: dora_factored_norm_workspace_size() bytes, 256-byte
 * aligned, contents undefined on entry and exit.  The result is bitwise
 * reproducible for fixed inputs and sizes.
 * ---------------------------------------------------------------------- */
size_t dora_factored_norm_workspace_size(int64_t d_out, int64_t d_in, int64_t r,
                                         dora_dtype_t dt);
dora_status_t dora_factored_norm(const void *W0, const void *A, const void *B,
                                 dora_dtype_t dt, int64_t d_out, int64_t d_in,
                                 int64_t r, float s, const float *m, float eps,
                                 float *n_out, float *g_out, void *ws,
                                 size_t ws_bytes, dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Grouped factored norm: the same computation for `count` independent
 * modules (e.g. every adapted projection of a layer stack) in one launch
 * per stage.  `problems` is a HOST array of `count` descriptors, read during
 * the call only; the pointers inside are device pointers.  Per problem, m and
 * g_out may be NULL (then g is not written).  All problems share `dt` and
 * `eps`.  1 <= count <= DORA_MAX_GROUP.  bf16 only.
 * ---------------------------------------------------------------------- */
typedef struct {
  const void *W0;   /* [d_out, d_in] */
  const void *A;    /* [r, d_in]     */
  const void *B;    /* [d_out, r]    */
  const float *m;   /* [d_out] or NULL */
  float *n_out;     /* [d_out]         */
  float *g_out;     /* [d_out] or NULL */
  int64_t d_out, d_in, r;
  float s;
} dora_norm_problem_t;

size_t dora_factored_norm_grouped_workspace_size(const dora_norm_problem_t *problems,
                                                 int count, dora_dtype_t dt);
dora_status_t dora_factored_norm_grouped(const dora_norm_problem_t *problems,
                                         int count, dora_dtype_t dt, float eps,
                                         void *ws, size_t ws_bytes,
                                         dora_stream_t stream);

/* ------------------------------------------------------------------------
 * d_in-sharded norm  ["Scaling DoRA ...", section 6: sharded base weights need
 * chunk-wise partial sums followed by an all-reduce; section 2: every term of
 * the squared row norm is a sum over the columns of W0]
 *
 * With W0 and A split by columns into shards k (W0^(k) = W0[:, J_k],
 * A^(k) = A[:, J_k], B whole), the squared row norm is the sum over shards of
 *   sq_i^(k) = ||W0_i^(k)||^2 + 2 s B_i.(W0^(k) A^(k)T)_i + s^2 B_i A^(k) A^(k)T B_i^T.
 * dora_factored_norm_sq computes sq^(k) for one shard (arguments as for
 * dora_factored_norm, with d_in the shard's width; the same workspace size)
 * and writes it to sq_out [d_out] fp32, before any clamp or square root.
 * After the caller sums sq over the shards (one all-reduce of d_out floats),
 * dora_norm_finalize writes n = sqrt(max(sq, 0)) and, when m and g_out are
 * given, g = m / max(n, eps).  n_out may equal sq.
 * ---------------------------------------------------------------------- */
dora_status_t dora_factored_norm_sq(const void *W0, const void *A, const void *B,
                                    dora_dtype_t dt, int64_t d_out, int64_t d_in, int64_t r,
                                    float s, float *sq_out, void *ws, size_t ws_bytes,
                                    dora_stream_t stream);
dora_status_t dora_norm_finalize(const float *sq, const float *m, float eps, int64_t d_out,
                                 float *n_out, float *g_out, dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Fused compose forward  ["Scaling DoRA ...", section 3 and Data Availability]
 *
 * With n_c = max(n, eps), g = m / n_c and (g - 1) = (m - n_c) / n_c in fp32:
 *   y[t, j] = base[t, j] + ((g_j - 1) base[t, j] + (g_j s) lora[t, j])
 * evaluated in fp32 and rounded once to the output dtype (round to nearest
 * even).  base, lora, y: [T, d_out] in dtype `dt`; m, n: fp32 [d_out].
 * One pass: two reads and one write per element.  y may equal base.
 * T == 0 launches nothing (the activation pointers may then be NULL).
 * ---------------------------------------------------------------------- */
dora_status_t dora_compose_fwd(const void *base, const void *lora, const float *m,
                               const float *n, float s, float eps, dora_dtype_t dt,
                               int64_t T, int64_t d_out, void *y,
                               dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Compose forward, delta form  ["Scaling DoRA ...", Data Availability: the
 * module's output is dY = g (s x A^T B^T) + (g - 1) Y_base, which the caller
 * adds to its own Y_base]
 *
 *   dy_out[t, j] = (g_j - 1) base[t, j] + (g_j s) lora[t, j]
 * with g and g - 1 formed as for dora_compose_fwd, evaluated in fp32 and
 * rounded once to `dt`; y of dora_compose_fwd is base + dy_out before that
 * rounding.  base, lora, dy_out: [T, d_out] in dtype `dt`; dy_out may equal
 * base (same element, same thread), no other overlap.  One pass: two reads
 * and one write per element.  T == 0 launches nothing.
 * ---------------------------------------------------------------------- */
dora_status_t dora_compose_fwd_delta(const void *base, const void *lora, const float *m,
                                     const float *n, float s, float eps, dora_dtype_t dt,
                                     int64_t T, int64_t d_out, void *dy_out,
                                     dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Fused compose backward  ["Scaling DoRA ...", section 3 backward kernel]
 *
 *   d_base[t, j] = g_j dy[t, j],  d_lora[t, j] = (g_j s) dy[t, j]
 *   dm[j] = (sum_t dy[t, j] (base[t, j] + s lora[t, j])) / n_c,j
 * The norm is detached (no gradient flows to W0, A or B through n).  dm is
 * accumulated in fp32 as per-chunk column partials summed in a fixed order
 * (no atomics): bitwise reproducible.  d_base may equal dy.  With T == 0
 * the activation pointers may be NULL and dm is set to zero.
 * Workspace: dora_compose_bwd_workspace_size() bytes, 256-byte aligned.
 * ---------------------------------------------------------------------- */
size_t dora_compose_bwd_workspace_size(int64_t T, int64_t d_out, dora_dtype_t dt);
dora_status_t dora_compose_bwd(const void *dy, const void *base, const void *lora,
                               const float *m, const float *n, float s, float eps,
                               dora_dtype_t dt, int64_t T, int64_t d_out,
                               void *d_base, void *d_lora, float *dm, void *ws,
                               size_t ws_bytes, dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Training forward with a second output  ["Scaling DoRA ...", section 4,
 * tier 1: the dual-output kernel computes the output and `inner` together]
 *
 * Writes y exactly as dora_compose_fwd does and, in the same pass,
 *   inner[t, j] = base[t, j] + s lora[t, j]
 * in fp32, rounded once to `dt`.  inner is what the backward needs for dm
 * (dora_compose_bwd_inner), so a training step can keep one activation
 * tensor for the backward instead of base and lora.  y may equal base and
 * inner may equal lora (same element, same thread); no other overlap.
 * One pass: two reads and two writes per element.  T == 0 launches nothing.
 * ---------------------------------------------------------------------- */
dora_status_t dora_compose_fwd_train(const void *base, const void *lora, const float *m,
                                     const float *n, float s, float eps, dora_dtype_t dt,
                                     int64_t T, int64_t d_out, void *y, void *inner,
                                     dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Backward from `inner`  ["Scaling DoRA ...", section 4, tier 1]
 *
 *   d_base = g dy,  d_lora = (g s) dy,  dm[j] = (sum_t dy[t, j] inner[t, j]) / n_c,j
 * with inner = base + s lora from dora_compose_fwd_train.  Same fixed-order
 * dm reduction as dora_compose_bwd.  Four passes per element (dy and inner
 * read, d_base and d_lora written) instead of five.  d_base may equal dy.
 * Workspace: dora_compose_bwd_workspace_size(T, d_out, dt) bytes (the same
 * table as dora_compose_bwd, of which this call uses at most all).
 * ---------------------------------------------------------------------- */
dora_status_t dora_compose_bwd_inner(const void *dy, const void *inner, const float *m,
                                     const float *n, float s, float eps, dora_dtype_t dt,
                                     int64_t T, int64_t d_out, void *d_base, void *d_lora,
                                     float *dm, void *ws, size_t ws_bytes,
                                     dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Backward with the magnitude frozen  ["Scaling DoRA ...", section 4, tier
 * 1 and section 6: with frozen magnitude the inner tensor is skipped]
 *
 *   d_base = g dy,  d_lora = (g s) dy;  no dm, no inner, no workspace.
 * Three passes per element.  d_base may equal dy.  The forward of a
 * frozen-magnitude step is dora_compose_fwd.
 * ---------------------------------------------------------------------- */
dora_status_t dora_compose_bwd_frozen(const void *dy, const float *m, const float *n, float s,
                                      float eps, dora_dtype_t dt, int64_t T, int64_t d_out,
                                      void *d_base, void *d_lora, dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Grouped compose  ["Scaling DoRA ...", section 6: below about 2048 x 6144
 * activations launch latency dominates; one launch covers every module of a
 * layer]
 *
 * One record per module (host array, read during the call only).  Every
 * module is computed exactly as by the single-module call named below; the
 * modules may differ in T, d_out and s, and share dt and eps.
 *   forward  (dora_compose_fwd_grouped): base, lora, m, n, y; inner NULL, or
 *            the second output of dora_compose_fwd_train.  One launch.
 *   backward (dora_compose_bwd_grouped): dy, m, n, d_base, d_lora and
 *            - dm NULL in every record: frozen magnitude
 *              (dora_compose_bwd_frozen), no workspace;
 *            - else inner non-NULL in every record: dora_compose_bwd_inner;
 *            - else base and lora: dora_compose_bwd.
 *            (Records with T == 0 read nothing and may leave inner, base
 *            and lora NULL whatever the variant.)
 *            Mixed records are DORA_ERR_INVALID_ARG.  Two launches (one when
 *            frozen): the stream pass and one fixed-order dm reduction for
 *            all modules.
 * Aliasing inside a record as for the single-module calls; records must not
 * write memory that another record reads or writes.  1 <= count <= 64.
 * Workspace (backward): dora_compose_bwd_grouped_workspace_size() bytes,
 * 256-byte aligned (0 for the frozen form).
 * ---------------------------------------------------------------------- */
#define DORA_MAX_COMPOSE_GROUP 64
typedef struct {
  const void *base;   /* [T, d_out] */
  const void *lora;   /* [T, d_out] */
  void *inner;        /* [T, d_out]: forward output (optional), backward input */
  const float *m;     /* [d_out] */
  const float *n;     /* [d_out] */
  void *y;            /* [T, d_out] forward output */
  const void *dy;     /* [T, d_out] backward input */
  void *d_base;       /* [T, d_out] backward output */
  void *d_lora;       /* [T, d_out] backward output */
  float *dm;          /* [d_out] backward output; NULL = frozen magnitude */
  int64_t T, d_out;
  float s;
} dora_compose_problem_t;

dora_status_t dora_compose_fwd_grouped(const dora_compose_problem_t *problems, int count,
                                       dora_dtype_t dt, float eps, dora_stream_t stream);
size_t dora_compose_bwd_grouped_workspace_size(const dora_compose_problem_t *problems,
                                               int count, dora_dtype_t dt);
dora_status_t dora_compose_bwd_grouped(const dora_compose_problem_t *problems, int count,
                                       dora_dtype_t dt, float eps, void *ws, size_t ws_bytes,
                                       dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Merged inference weight  ["LoRA & DoRA: The Math, Memory, and Trade-offs",
 * section 6: magnitude and direction fold into one dense weight for
 * inference; "Scaling DoRA ...", section 4 precision bullet for g]
 *
 *   W_out[i, j] = g_i (W0[i, j] + s sum_k B[i, k] A[k, j]),  g_i = m_i / max(n_i, eps)
 * with the sum over k formed on the tensor cores in fp32 and the rest in fp32,
 * rounded once to bf16.  n is the row norm of W0 + s B A (from
 * dora_factored_norm); it is not recomputed.  W0, W_out: bf16 [d_out, d_in];
 * A: bf16 [r, d_in]; B: bf16 [d_out, r]; m, n: fp32 [d_out].  W_out may
 * equal W0 (in-place merge); no other overlap.  bf16 only; d_in and r
 * multiples of 8, pointers 16-byte aligned, 1 <= r <= 512
 * (DORA_ERR_UNSUPPORTED otherwise).  Workspace:
 * dora_merge_weight_workspace_size() bytes, 256-byte aligned (holds A^T).
 * Two launches (transpose of A, then the fused GEMM + epilogue).
 * ---------------------------------------------------------------------- */
size_t dora_merge_weight_workspace_size(int64_t d_out, int64_t d_in, int64_t r);
dora_status_t dora_merge_weight(const void *W0, const void *A, const void *B, const float *m,
                                const float *n, float s, float eps, int64_t d_out,
                                int64_t d_in, int64_t r, void *W_out, void *ws,
                                size_t ws_bytes, dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Compose backward without a workspace (no counterpart on the pages: it is
 * an interface convenience, not part of the method).
 *
 * Some callers cannot pass the library a workspace: a plain C host program
 * that links this library without a device allocator of its own, or a
 * latency-critical loop in which cudaMalloc is not allowed because it can
 * synchronise the whole device.  This call computes exactly what
 * dora_compose_bwd computes, with the same arguments minus the workspace:
 * the dm column partials live in a fixed 4 MiB array of device memory that
 * every GPU which loads this library holds until the process exits.  It
 * allocates nothing and calls no allocating routine.
 *   - Shapes whose partial table exceeds 4 MiB (more than 1,048,576 floats,
 *     see dora_compose_bwd_workspace_size) are rejected with
 *     DORA_ERR_UNSUPPORTED before anything is launched; dora_last_error()
 *     then says how much scratch the shape needs.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress),
 *     so the call stays valid after a device reset; a failed lookup returns
 *     DORA_ERR_CUDA and launches nothing.
 *   - All calls share the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race and give wrong results.  Nothing in
 *     the array needs to start at zero: each call writes every slot it
 *     reads before reading it.
 * ---------------------------------------------------------------------- */
dora_status_t dora_compose_bwd_static(const void *dy, const void *base, const void *lora,
                                      const float *m, const float *n, float s, float eps,
                                      dora_dtype_t dt, int64_t T, int64_t d_out, void *d_base,
                                      void *d_lora, float *dm, dora_stream_t stream);

/* ------------------------------------------------------------------------
 * Status and diagnostics
 * ---------------------------------------------------------------------- */
/* Synchronises `stream`, returns the first error any kernel of this library
 * recorded on the current device since the last call (DORA_OK if none), and
 * clears it. */
dora_status_t dora_get_device_status(dora_stream_t stream);
/* Static English description of a status code; never NULL. */
const char *dora_status_string(dora_status_t status);
/* Description of the last CUDA runtime failure seen by a call on the calling
 * host thread (which call, the runtime's message and code), or "" if none.
 * Owned by the library; valid until the next call on that thread. */
const char *dora_last_error(void);
/* Library version, major * 10000 + minor * 100 + patch. */
int dora_version(void);
/* Number of kernels this library has launched in this process. */
uint64_t dora_launch_count(void);
/* Upper bound, in nanoseconds, on any single internal wait of the
 * tensor-core kernels (default 2e9).  0 restores the default.  Host-side
 * setting, applied to launches made after the call; exists so that tests can
 * exercise the give-up path without a real hang. */
void dora_set_wait_timeout_ns(uint64_t ns);
/* Timing hook: the next entry-point call made by the calling host thread
 * records `before` immediately before, and `after` immediately after, the
 * launch of its principal kernel (the fused norm GEMM of the norm calls, the
 * compose kernel of the compose calls) on that call's stream; the hook then
 * clears itself.  Both are cudaEvent_t handles created by the caller (NULL,
 * NULL clears the hook).  Lets a caller time that one kernel with CUDA events
 * on the stream it runs on.  While that stream is being captured into a CUDA
 * graph, the events are recorded as event-record nodes of the graph, so each
 * replay re-records them around the kernel. */
void dora_set_timing_events(void *before, void *after);
/* Diagnostics: when `buf` is non-NULL, later norm calls record 16 uint64
 * words per CTA of the fused norm kernel into it (device memory, 16 * 148
 * words for one B200; a word the kernel does not set keeps its value):
 * [0] entry and [1] exit %globaltimer, cycles the MMA issuer waited [2] for
 * operands and [3] for the accumulator, [4] k-blocks issued, [5] segments,
 * [6] SM id, [7] cycles waited for operands over the first four k-blocks,
 * then %globaltimer when [8] the MMA issuer starts its static W0 units and
 * [9] its first pool item; for the CTA's first Gram job, when its epilogue's
 * first warp [10] holds the accumulator, [14] has its stores of S written
 * and [11] has published them; [12] when the finisher is done with its last
 * segment and [15] when the MMA issuer has issued its last MMA; [13] cycles
 * the first epilogue thread waited for a free hand-over buffer, summed.
 * NULL turns it off.  The buffer must outlive every call made while it is
 * set. */
void dora_set_trace_buffer(void *buf);
/* Host-only self-check of the fused norm's schedule (no device, no launch):
 * plans `count` modules (sizes d_out[i] x d_in[i], rank r[i]; `grouped`
 * non-zero plans them as one grouped call, else count must be 1) for
 * `pairs` CTA pairs (1 .. 512; 74 on a B200) and walks every segment the
 * kernel's roles would take -- each pair's static Gram jobs and W0 range,
 * then every pool item (W0 chunks, G items) -- to check that every W0 and G
 * unit of every tile is covered exactly once, that the Gram jobs partition
 * the wave's jobs, and that the partial slots of every tile are distinct,
 * numbered 0 .. nseg-1, agree on nseg and fit the workspace's slot count.
 * Returns DORA_OK; DORA_ERR_INVALID_ARG / DORA_ERR_UNSUPPORTED for sizes the
 * norm rejects; DORA_ERR_INTERNAL with the first failed invariant in
 * dora_last_error(). */
dora_status_t dora_norm_plan_check(const int64_t *d_out, const int64_t *d_in, const int64_t *r,
                                   int count, int grouped, int pairs);
/* Launches one thread that waits, with the same bounded wait the
 * tensor-core pipelines use, on a barrier that nothing ever signals, giving
 * up after `timeout_ns` (clamped to [1 us, 1 s]).  The give-up is recorded as
 * DORA_ERR_TIMEOUT for dora_get_device_status.  Diagnostic: it lets a test
 * check the give-up path deterministically without a real hang. */
dora_status_t dora_debug_unsignalled_wait(uint64_t timeout_ns, dora_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DORA_H_ */
