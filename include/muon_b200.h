/*
 * muon_b200.h -- C ABI of the B200 (sm_100a) Muon + AdamW optimizer step.
 *
 * The step (sources, by page title and section):
 *   - "Chapter 4: The MuonAdamW Optimizer": The Muon Update Rule (Nesterov
 *     momentum m = beta*m + G, lookahead m~ = beta*m + G); Polar Express:
 *     Newton-Schulz Orthogonalization (X0 = m~/(||m~||_F + 1e-7), tall
 *     matrices iterated as their transpose, A = X X^T, B = b*A + c*A*A,
 *     X = a*X + B*X, five steps, (a,b,c) = (3.4445, -4.7750, 2.0315));
 *     The AdamW Step.
 *   - "Stuck at the optimizer after figuring out backward()" (nanochat
 *     discussion, mira687's reply): cautious weight decay, decay only where
 *     update * param >= 0; per-step coefficient tables.
 *   - "3.9 Optimizers: SGD, Adam, Adafactor, Lion, Muon & Shampoo":
 *     Implementing AdamW from scratch (bias-corrected AdamW with decoupled
 *     decay); Muon: Orthogonalizing the Update (heavy-ball variant).
 *
 * Conventions for every entry point:
 *   Ownership  All tensors and the workspace belong to the caller.  Pointer
 *              arrays and descriptors are host memory, read only during the
 *              call.  The library allocates no device memory.
 *   Layout     Matrices are dense row-major (row pitch = cols elements).
 *              params, momentum, exp_avg, exp_avg_sq are fp32; grads are
 *              fp32 or bf16 as the group says.
 *   In place   params, momentum, exp_avg and exp_avg_sq are updated in place;
 *              grads are read only.
 *   Async      Work is enqueued on `stream` (NULL = the legacy default
 *              stream).  No host synchronisation and no device-to-host copy
 *              happen inside muon_step / muon_orthogonalize / adamw_step.
 *   Errors     Arguments are validated on the host before any launch; a
 *              failed check returns a status and touches no tensor.
 *              muon_last_error() gives a one-line reason.  Launch failures
 *              return MUON_ERR_CUDA.  Device-side bounded waits that run out
 *              record MUON_ERR_TIMEOUT in the workspace status word, read by
 *              muon_query_status().
 *   Threads    Entry points are reentrant; calls on different streams with
 *              different workspaces may run concurrently.
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t.  Declared here so this header needs no CUDA headers. */
typedef struct CUstream_st* muon_stream_t;

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, bad scalar, misaligned pointer */
  MUON_ERR_UNSUPPORTED = 2,  /* valid request this library cannot run (no sm_100 device, ...) */
  MUON_ERR_WORKSPACE = 3,    /* workspace null, misaligned or smaller than muon_workspace_min_size */
  MUON_ERR_CUDA = 4,         /* a CUDA runtime/driver call or kernel launch failed */
  MUON_ERR_TIMEOUT = 5       /* a device-side bounded wait ran out (status word) */
} muon_status;

typedef enum { MUON_F32 = 0, MUON_BF16 = 1 } muon_dtype;

/* muon_step / muon_orthogonalize flags */
enum {
  MUON_NESTEROV = 1u,       /* orthogonalise beta*m + G (else m itself, heavy-ball) */
  MUON_CAUTIOUS_WD = 2u,    /* decay only where update*param >= 0 (else plain decoupled decay) */
  MUON_FP32_DEBUG = 4u,     /* fp32 operands and fp32 FMA GEMMs (slow; tolerance 1e-4 mode) */
  MUON_UNFUSED_UPDATE = 8u, /* apply the update in its own kernel instead of the last B*X epilogue */
  MUON_TC_SINGLE_CTA = 16u, /* run the Newton-Schulz GEMMs on single-CTA 128x256 tiles instead of
                               CTA-pair (cta_group::2) tiles; same results, for comparison */
  MUON_NORMUON = 32u,       /* NorMuon ("Chapter 4: The MuonAdamW Optimizer", NorMuon): divide every
                               row of U (parameter orientation) by (||row||/sqrt(cols) + 1e-8) before
                               the decay and update, so each row's RMS is 1 and the step's is lr */
  MUON_TC_NARROW_TILES = 128u, /* run the Gram and B'X products on 256x256 CTA-pair tiles with two
                               TMEM accumulators (as A*A and the fused update always are) for every
                               shape; same results, for comparison.  By default a product runs on
                               256x512 tiles with one accumulator only where its output width is a
                               multiple of 512 and its K is at least 2048, where they are faster */
  MUON_TC_WIDE_TILES = 256u, /* run the Gram and B'X products on 256x512 CTA-pair tiles for every
                               shape; same results, for comparison (MUON_TC_NARROW_TILES wins if
                               both are given) */
  MUON_ROW_EQUILIBRATE = 64u /* MuonEq row equilibration ("Stuck at the optimizer after figuring out
                               backward()", mira687's reply, names it without a formula): divide every
                               row of m~ (parameter orientation) by (||row|| + 1e-7) before the
                               Frobenius normalisation; the momentum buffer is unchanged.  muon_step
                               only; needs the workspace sizes computed with this flag */
};

/*
 * One shape group: `count` matrices of rows x cols (parameter orientation),
 * the pointers params[first .. first+count-1] (same for grads, momentum).
 * The groups of one call index disjoint ranges (else MUON_ERR_INVALID_ARG).
 * A group with rows > cols is iterated as its transpose ("Polar Express"
 * orientation); no physical transpose is made: the kernels read it
 * MN-major.
 */
typedef struct {
  int32_t rows;
  int32_t cols;
  int32_t count;
  int32_t first;
  int32_t grad_dtype;  /* muon_dtype */
  float lr_scale;      /* per-group learning-rate multiplier (1 => W -= lr*update) */
} muon_group;

/*
 * Workspace bytes to run every matrix of `groups` in a single wave (fastest).
 * muon_workspace_min_size: the least workspace muon_step accepts; with less
 * than muon_workspace_size the matrices are processed in several waves.
 * Returns 0 on invalid groups.  Host only, no CUDA call.
 */
size_t muon_workspace_size(const muon_group* groups, int n_groups, uint32_t flags);
size_t muon_workspace_min_size(const muon_group* groups, int n_groups, uint32_t flags);

/*
 * One Muon step over every matrix of every group.
 *
 *   for each matrix:  m <- beta*m + G;   m~ <- beta*m + G  (MUON_NESTEROV) or m
 *                     (MUON_ROW_EQUILIBRATE: m~_row <- m~_row / (||m~_row|| + 1e-7))
 *                     X0 <- m~ / (||m~||_F + 1e-7)
 *                     ns_steps x { A = X X^T; B = b_k A + c_k A A; X = a_k X + B X }
 *                     (wide orientation: rows > cols iterates on X^T)
 *                     U  <- X (values rounded to bf16, as the pages keep X in bf16)
 *                     (MUON_NORMUON: U_row <- U_row / (||U_row||/sqrt(cols) + 1e-8))
 *                     W  <- W - lr*lr_scale*(U + wd*mask*W),
 *                           mask = (U*W >= 0) with MUON_CAUTIOUS_WD, else 1
 *
 * params[i], momentum[i]: fp32 device, rows x cols, 16-byte aligned.
 * grads[i]: device, rows x cols, dtype per group, 16-byte aligned.
 * coeffs: host, ns_steps rows of (a, b, c); may be NULL only if ns_steps == 0.
 * ns_steps in [0, 16].  beta in [0, 1).  lr, wd finite.
 * workspace: device, 256-byte aligned, >= muon_workspace_min_size bytes; its
 * contents need no initialisation and are scratch between calls.
 * Two calls that share a workspace must be ordered (same stream).
 * Matrices whose element count is a multiple of 8 and whose columns are a
 * multiple of 8 take a faster momentum kernel (bulk copies through shared
 * memory) when every matrix of the call does; the results are the same bits.
 */
muon_status muon_step(float* const* params, const void* const* grads, float* const* momentum,
                      const muon_group* groups, int n_groups,
                      float lr, float beta, float wd, int ns_steps, const float* coeffs,
                      uint32_t flags, void* workspace, size_t workspace_bytes,
                      muon_stream_t stream);

/*
 * muon_step that also writes every updated parameter matrix into
 * n_replicas further copies ("3.9 Optimizers: SGD, Adam, Adafactor, Lion,
 * Muon & Shampoo", Wiring the hybrid recipe: a distributed Muon steps each
 * matrix on one rank, which must then hand the result to every
 * data-parallel rank).  replicas: host array of n_replicas host arrays of
 * device pointers, in the order of `params`: replicas[r][i] is copy r of
 * params[i] (same shape, fp32, 16-byte aligned).  The copies may live in
 * another GPU's memory that this device can address (peer access or a
 * mapped IPC / symmetric-memory allocation): on the default path the last
 * Newton-Schulz product's epilogue stores each updated W tile to W and to
 * every copy with plain stores, so the exchange over NVLink overlaps the
 * GEMM tile by tile; other paths (MUON_UNFUSED_UPDATE, MUON_NORMUON,
 * MUON_FP32_DEBUG, ns_steps == 0) copy W after the update.  No multicast.
 * The copies hold the new values once `stream` passes this call; a reader
 * on another device must order itself after it (an event or a collective).
 * n_replicas in [0, 7]; 0 is muon_step.  Other arguments as muon_step.
 */
muon_status muon_step_replicated(float* const* params, const void* const* grads,
                                 float* const* momentum, const muon_group* groups, int n_groups,
                                 float lr, float beta, float wd, int ns_steps, const float* coeffs,
                                 uint32_t flags, void* workspace, size_t workspace_bytes,
                                 float* const* const* replicas, int n_replicas, muon_stream_t stream);

/*
 * Mean of `count` tensors over n_sources copies, computed by this GPU:
 *   dst[i][e] <- (sources[0][i][e] + ... + sources[n_sources-1][i][e]) * (1/n_sources)
 * summed in fp32 in that order and stored in `dtype` (round to nearest even
 * for bf16).  The data-parallel mean gradient that the owner of a matrix
 * needs before its Muon step ("3.9 Optimizers: SGD, Adam, Adafactor, Lion,
 * Muon & Shampoo", Wiring the hybrid recipe): the sources may be the other
 * ranks' gradient buffers in peer GPU memory (peer access or a mapped IPC /
 * symmetric-memory allocation), read with plain loads over NVLink; no
 * multicast.  dst[i] may be one of sources[r][i] (each element is read
 * before it is written by the same thread).  The sources must not change
 * until `stream` passes this call.
 * dst: host array of `count` device pointers; sources: host array of
 * n_sources host arrays of `count` device pointers; numel: host, elements
 * per tensor.  Every pointer 16-byte aligned.  n_sources in [1, 8].
 */
muon_status muon_reduce_mean(void* const* dst, const void* const* const* sources, int n_sources,
                             const int64_t* numel, int count, int32_t dtype, muon_stream_t stream);

/*
 * muon_step without a caller workspace, for callers that cannot allocate
 * device memory (no counterpart on the optimizer pages: it is a deployment
 * aid).  Programs whose device-memory budget is fixed at start-up by another
 * runtime, or code running inside a framework callback that owns every
 * allocation, cannot hand muon_step a workspace; this entry point takes its
 * scratch from one built-in device array of MUON_NOALLOC_SCRATCH_BYTES instead
 * and allocates nothing.
 *
 * Same arguments and semantics as muon_step, minus the workspace.  Limit: the
 * largest single matrix must fit, i.e. muon_workspace_min_size(groups, flags)
 * <= MUON_NOALLOC_SCRATCH_BYTES (32 MiB: with bf16 operands up to about
 * 2048 x 2048 or 1024 x 7168; with MUON_FP32_DEBUG, whose buffers are twice
 * as large, up to about 1600 x 1600 or 1024 x 3072); larger sets are
 * processed in waves; a matrix that does not fit returns MUON_ERR_WORKSPACE
 * with the sizes in muon_last_error().  Every GPU that loads this library
 * holds the array until the process exits.  Each call looks up the array's
 * device address in the current context; the first call on a device (or
 * after a device reset) also loads the library's device code, so make it
 * before any stream capture.  All calls on a device share the array: calls
 * that overlap on the GPU race and must be ordered by the caller (e.g. one
 * stream).  The status word of the last step is read with
 * muon_query_status() on the address muon_noalloc_scratch() returns.
 */
#define MUON_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
muon_status muon_step_noalloc(float* const* params, const void* const* grads,
                              float* const* momentum, const muon_group* groups, int n_groups,
                              float lr, float beta, float wd, int ns_steps, const float* coeffs,
                              uint32_t flags, muon_stream_t stream);

/*
 * The built-in scratch of muon_step_noalloc on the current device: its device
 * address (*device_ptr) and size (*bytes, MUON_NOALLOC_SCRATCH_BYTES; bytes
 * may be NULL).  Allocates nothing.  Its first 4 bytes are the status word of
 * the last muon_step_noalloc on the device: muon_query_status(*device_ptr,
 * stream) reports MUON_ERR_TIMEOUT if a device-side wait of that step ran
 * out.  The rest of the array is the step's scratch; a caller writes nothing
 * there.  Returns MUON_ERR_INVALID_ARG for a NULL device_ptr and MUON_ERR_CUDA
 * if the address cannot be looked up (no device, or no context).
 */
muon_status muon_noalloc_scratch(void** device_ptr, size_t* bytes);

/*
 * The orthogonaliser alone: outputs[i] <- NS(inputs[i]) as fp32, rows x cols,
 * with the same normalisation, orientation, iteration and bf16 rounding of
 * the result as muon_step.  inputs[i] dtype per group.  Only MUON_FP32_DEBUG,
 * MUON_TC_SINGLE_CTA and MUON_TC_NARROW_TILES are honoured in `flags`.
 */
muon_status muon_orthogonalize(const void* const* inputs, float* const* outputs,
                               const muon_group* groups, int n_groups,
                               int ns_steps, const float* coeffs, uint32_t flags,
                               void* workspace, size_t workspace_bytes, muon_stream_t stream);

/*
 * AdamW group ("3.9 Optimizers", Implementing AdamW from scratch), for t >= 1:
 *   p <- p*(1 - lr*wd);  m <- b1*m + (1-b1)*g;  v <- b2*v + (1-b2)*g^2
 *   p <- p - (lr/(1-b1^t)) * m / (sqrt(v)/sqrt(1-b2^t) + eps)
 * params/exp_avg/exp_avg_sq fp32 device, grads fp32 or bf16 device, each
 * tensor numel[i] >= 0 contiguous elements, 16-byte aligned.
 * Per-group betas and lr carry per-role settings (embeddings, head, gains).
 */
typedef struct {
  float* const* params;
  const void* const* grads;
  float* const* exp_avg;
  float* const* exp_avg_sq;
  const int64_t* numel;
  int32_t count;
  int32_t grad_dtype; /* muon_dtype */
  float lr, beta1, beta2, eps, wd;
} adamw_group;

/* One fused AdamW step over all tensors of all groups (multi-tensor launches).
 * Where every tensor of a launch has a multiple of 8 elements a kernel that
 * streams the tensors through shared memory with bulk copies runs (the same
 * bits); its bounded waits report through adamw_query_status. */
muon_status adamw_step(const adamw_group* groups, int n_groups, int64_t step,
                       muon_stream_t stream);

/*
 * Device-resident schedule state, for steps replayed from a captured CUDA
 * graph: the learning rate and AdamW's step count change between replays
 * without re-recording.  Device memory, 8-byte aligned, owned by the caller;
 * start it at {lr_mult = 1 (or any), step = 0}.
 *   lr_mult  multiplies lr in muon_step_scheduled and every group's lr in
 *            adamw_step_scheduled
 *   step     AdamW's t (>= 1 when adamw_step_scheduled runs)
 */
typedef struct {
  float lr_mult;
  float reserved;
  int64_t step;
} muon_schedule_state;

/*
 * On the device: step <- step + 1, then lr_mult <- the trapezoidal schedule
 * ("Chapter 4: The MuonAdamW Optimizer", Learning Rate Schedule) at the
 * 0-based step (step - 1): linear warmup from 0 over int(total_steps *
 * warmup_frac) steps, 1 on the flat part, linear warmdown to final_frac over
 * int(total_steps * warmdown_frac) steps, final_frac at and after total_steps.
 * One single-thread kernel on `stream`.
 */
muon_status muon_schedule_advance(muon_schedule_state* state, int64_t total_steps,
                                  float warmup_frac, float warmdown_frac, float final_frac,
                                  muon_stream_t stream);

/*
 * On the device: step <- step + 1, then lr_mult <- the warmup + cosine
 * schedule ("Muon vs AdamW, Lion and Sophia: a fair race", the bake-off's
 * learning rate by step) at the 0-based step s = step - 1:
 *   s < warmup_steps              s / warmup_steps (linear climb from 0)
 *   warmup_steps <= s < last      final_frac + (1 - final_frac) * (1 + cos(pi * p)) / 2,
 *                                 p = (s - warmup_steps) / (last - warmup_steps)
 *   s >= last                     final_frac
 * with last = total_steps - 1, so the cosine reaches final_frac (a tenth of
 * the peak on that page) at the last step.  total_steps >= 1,
 * 0 <= warmup_steps <= total_steps, final_frac finite; computed in double.
 * One single-thread kernel on `stream`.
 */
muon_status muon_schedule_advance_cosine(muon_schedule_state* state, int64_t total_steps,
                                         int64_t warmup_steps, float final_frac, muon_stream_t stream);

/* muon_step with the learning rate lr * state->lr_mult read on the device. */
muon_status muon_step_scheduled(float* const* params, const void* const* grads,
                                float* const* momentum, const muon_group* groups, int n_groups,
                                float lr, float beta, float wd, int ns_steps, const float* coeffs,
                                uint32_t flags, void* workspace, size_t workspace_bytes,
                                const muon_schedule_state* state, muon_stream_t stream);

/* adamw_step with each group's lr * state->lr_mult and t = state->step read on the device. */
muon_status adamw_step_scheduled(const adamw_group* groups, int n_groups,
                                 const muon_schedule_state* state, muon_stream_t stream);

/*
 * AdamW's failure channel (it takes no caller workspace).  Synchronises
 * `stream` and returns MUON_ERR_TIMEOUT if, since the previous call, a
 * bounded device wait inside an adamw_step / adamw_step_scheduled kernel on
 * the current device ran out (the kernel then stopped without updating the
 * chunks it had not reached), else MUON_OK; the record is cleared.  The
 * waits are those of the kernel that streams g, p, m and v through shared
 * memory with bulk copies, used when every tensor of a launch has a multiple
 * of 8 elements.
 */
muon_status adamw_query_status(muon_stream_t stream);

/*
 * Synchronises `stream`, reads the workspace status word written by the
 * device during the last muon_step / muon_orthogonalize on it, and returns
 * MUON_OK or the recorded error (MUON_ERR_TIMEOUT).
 */
muon_status muon_query_status(const void* workspace, muon_stream_t stream);

/*
 * Self-test of the device failure channel (no counterpart on the optimizer
 * pages).  Launches one thread that waits, with the same bounded wait the
 * tensor-core kernels use but a limit of `limit_ns` nanoseconds, on an
 * mbarrier that nothing ever arrives on; when the limit runs out it records
 * MUON_ERR_TIMEOUT in the workspace status word (word 0) and returns.  A
 * following muon_query_status(workspace, stream) must report
 * MUON_ERR_TIMEOUT; the CUDA context stays usable.  limit_ns in
 * [1000, 10^9].  The status word is not cleared first.
 */
muon_status muon_selftest_wait_timeout(void* workspace, uint64_t limit_ns, muon_stream_t stream);

const char* muon_status_string(muon_status s);

/* One-line description of the last failure on the calling thread ("" if none). */
const char* muon_last_error(void);

/*
 * Optional per-kernel timing (no counterpart on the optimizer pages; it
 * feeds the benchmark's per-kernel rooflines).  Process-wide state, guarded
 * by a lock.  While enabled, every launch of the library is bracketed by
 * CUDA events on its own stream (the events come from a pool the library
 * owns; enabling adds two event records per launch and nothing else).
 *   muon_profiler_enable   on != 0 enables; returns the previous setting.
 *   muon_profiler_reset    waits for the recorded events, then clears.
 *   muon_profiler_read     waits for the recorded events and writes, for
 *                          kinds 0 .. min(max_kinds, kind count) - 1, the summed
 *                          device milliseconds and launch counts since the
 *                          last reset into the caller's host arrays (either
 *                          may be NULL); returns the kind count.
 *   muon_kernel_kind_count / muon_kernel_kind_name   the kinds' names ("" for
 *                          an index out of range); static strings.
 * Do not enable it while a stream is being captured into a CUDA graph.
 */
int muon_profiler_enable(int on);
void muon_profiler_reset(void);
int muon_profiler_read(double* ms_out, int64_t* launches_out, int max_kinds);
int muon_kernel_kind_count(void);
const char* muon_kernel_kind_name(int kind);

#ifdef __cplusplus
}
#endif

#endif /* MUON_B200_H */
