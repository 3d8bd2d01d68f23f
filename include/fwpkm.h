/*
 * fwpkm.h -- C ABI of the B200 (sm_100a) Fast-weight Product Key Memory step.
 *
 * The library implements the chunked read-then-write memory step of
 * "Fast-weight Product Key Memory" (Zhao & Jones).  Citations name the page
 * and section the operation comes from:
 *   [GS-2]  gist.science "Fast-weight Product Key Memory", section 2
 *           "Methodology" (Core Architecture; Key Technical Choices)
 *   [AF]    agifrontier.github.io "Fast-weight Product Key Memory" tutorial
 *           (memorisation update; product-key addressing; gating)
 *   [PYPI]  pypi.org "fast-weight-product-key-memory" 0.2.2, Usage
 *           (constructor arguments; chaining past/next memories)
 *   [SS-TOC] sciencestack.ai "Fast-weight Product Key Memory", table of
 *           contents (loss aggregation and gradient shaping; marginal
 *           entropy loss)
 *
 * Conventions for every entry point:
 *   - Tensor arguments are plain pointers to memory the CALLER owns.  Unless
 *     stated otherwise they are DEVICE pointers (cudaMalloc / torch CUDA
 *     tensors) on the current CUDA device, C-contiguous, 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it; nothing synchronises
 *     unless stated.
 *   - Every function returns FWPKM_OK (0) or a negative fwpkm_status; the
 *     message of the last failure on the calling thread is available from
 *     fwpkm_last_error().  Argument and shape checks run on the host BEFORE
 *     anything is enqueued: a call that fails them launches nothing and
 *     leaves the state unchanged.
 *   - A state is not thread-safe; calls on one state must be serialised.
 *     Their device work shares the state's scratch, so calls on one state
 *     that use different streams must also be ordered on the device by the
 *     caller (for example with an event); calls on one stream already are.
 */
#ifndef FWPKM_H_
#define FWPKM_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct fwpkm_state fwpkm_state; /* opaque; owns the tables + scratch */

typedef enum {
  FWPKM_OK = 0,
  FWPKM_EINVAL = -1,      /* bad pointer / enum / scalar argument            */
  FWPKM_ESHAPE = -2,      /* sizes violate the constraints listed below      */
  FWPKM_ENOMEM = -3,      /* device or host allocation failed                */
  FWPKM_ECUDA = -4,       /* a CUDA call failed (message has the CUDA error)  */
  FWPKM_EUNSUPPORTED = -5 /* valid request the library does not implement    */
} fwpkm_status;

/* Element types of Q and Vtarget. */
enum { FWPKM_F32 = 0, FWPKM_BF16 = 1 };

/* Upper bounds checked by fwpkm_state_init. */
#define FWPKM_MAX_TOPK 32  /* top-k per head is held one slot per warp lane  */
#define FWPKM_MAX_SUBKEYS 1024 /* n = sqrt(N): a half's n scores live in registers, n/32 per
                                 * lane, selected through one 32-bit mask per lane */

/*
 * fwpkm_state_init -- create a memory of N = n*n slots.  [GS-2, PYPI]
 *   N      number of value slots; must be a perfect square n*n, 4 <= n <= 1024
 *          (N <= 1,048,576).
 *   dq     query width per head; a multiple of 16 (so dq/2, one half, is a
 *          multiple of 8), dq/2 <= 1024.
 *   dv     value width; a multiple of 4, <= 2048.
 *   topk   slots read per head and token; 1 <= topk <= min(n, 32).
 *   chunk  tokens per update chunk, 1 <= chunk <= 2^20; every chunk is read with the tables
 *          left by the previous chunk, then written.  [GS-2 causality]
 *   heads  query heads sharing the one value table (>= 1, <= 16); each head
 *          has its own pair of sub-key tables.
 * The tables start at ZERO; load them with fwpkm_state_set.  eps (the IDW
 * constant) defaults to 1e-3.  On success *out receives the state; the state
 * owns its device memory until fwpkm_state_free.
 */
fwpkm_status fwpkm_state_init(int64_t N, int dq, int dv, int topk, int chunk, int heads,
                              fwpkm_state **out);

/*
 * fwpkm_state_init_batched -- `memories` independent memories in one state,
 * one per sequence: a step over B = memories sequences reads and writes
 * memory b with sequence b only, all of them in the same launches.  (The
 * other reading of a memory per sequence; the package page chains one
 * memory per call, pypi.org fast-weight-product-key-memory, Usage.)  Each
 * memory is a state of fwpkm_state_init's shape; the arguments and limits
 * are those, plus memories >= 1 with memories * (N + 2*heads*n) < 2^31.
 * The tables stack the memories: sub-keys [memories][heads][2][n][dq/2],
 * values [memories][N][dv] (fwpkm_state_get / set copy all of them).  A
 * step's B must equal `memories` (FWPKM_ESHAPE otherwise).  The marginal of
 * the entropy term is each memory's own (its M = chunk * heads
 * token-heads).  Selections read and forced (fwpkm_record_selection /
 * fwpkm_force_selection) are slots of the token's own memory, 0 .. N-1.
 * fwpkm_select_noalloc does not take such a state (FWPKM_EUNSUPPORTED).
 */
fwpkm_status fwpkm_state_init_batched(int64_t N, int dq, int dv, int topk, int chunk, int heads,
                                      int memories, fwpkm_state **out);

/* Release the state and all memory it owns (NULL is a no-op).  Synchronises
 * the device first so no enqueued work still uses the memory. */
void fwpkm_state_free(fwpkm_state *s);

/* IDW constant: score = -log(eps + ||q_half - K_row||^2).  [GS-2]  eps > 0. */
fwpkm_status fwpkm_state_set_eps(fwpkm_state *s, float eps);

/* Options of fwpkm_state_set_options. */
#define FWPKM_HEADS_SUM 1u /* head readouts summed, not averaged                   */
#define FWPKM_AGG_COUNT 2u /* value-row gradient divided by the row's access count */
#define FWPKM_AGG_SUM 4u   /* value-row gradient not divided                       */
#define FWPKM_SCORE_DOT 8u /* sub-key score q_half . K_row instead of the IDW one  */

/*
 * fwpkm_state_set_options -- other readings of points the pages leave open,
 * and the score they name as the alternative, for the steps and selections
 * that follow (0 restores the defaults).
 *   [PYPI multi-head variant]  By default the heads' readouts are averaged,
 *     yhat = (1/H) sum_h sum_r w V[slot]; FWPKM_HEADS_SUM sums them, and the
 *     1/H of the gradients and of C_i goes with it.
 *   [GS-2 averaging of repeated-slot gradients; SS-TOC gradient weighted by
 *     row contribution]  By default a written value row moves by
 *     eta G_i / C_i, C_i = sum of its pairs' w/H; FWPKM_AGG_COUNT divides by
 *     the number of pairs on the row instead, FWPKM_AGG_SUM not at all.
 *     The two exclude each other (FWPKM_EINVAL).
 *   [GS-2 Key Technical Choices]  By default a sub-key row scores
 *     -log(eps + ||q_half - K_row||^2) (IDW); FWPKM_SCORE_DOT scores the
 *     dot product q_half . K_row instead, the alternative the page names.
 *     The selection then takes the largest dot products, and a sub-key row
 *     moves by eta sum(dL/ds q_half) (ds/dK = q_half); eps is unused.
 * The sub-keys always take the raw summed gradient.
 */
fwpkm_status fwpkm_state_set_options(fwpkm_state *s, unsigned options);

/*
 * fwpkm_step -- run the chunk loop over one call.  [GS-2, AF]
 * For every chunk c = 0 .. ceil(T/chunk)-1 in order (the last may be
 * shorter), over all B sequences at once (one shared memory):
 *   read  : for each token t and head h, split q into halves q1 | q2, score
 *           each half against its sub-key table with -log(eps + ||q - K||^2),
 *           take the top-k of each half, merge the k*k Cartesian candidates
 *           (score s1(i) + s2(j), slot i*n + j) to the top-k slots, weight
 *           them by softmax, average the heads' weighted value rows into
 *           yhat_t, and write out_t = gate_t * yhat_t;
 *   write : with L = sum_t gate_t ||yhat_t - Vtarget_t||^2
 *           + lambda_entropy * sum_i pbar_i log pbar_i   (pbar = the chunk's
 *           marginal slot usage), update in place
 *             V_i -= eta * (dL/dV_i) / C_i  (C_i = sum of w/heads on row i)
 *             K   -= eta * dL/dK
 *           on the touched value rows and sub-key rows only; no clipping.
 * Arguments:
 *   B, T      batch and tokens per sequence (>= 1); FWPKM_ESHAPE when
 *             B*T*2*heads >= 2^31 or B*chunk*heads*topk*3 >= 2^31 (32-bit
 *             indices of query halves and pairs), or when a chunk's B*chunk
 *             rows exceed 65535 tiles of 128 rows (the score grid).
 *   Q         device [B][T][heads*dq], element type q_dtype; read by the
 *             selection and, for the sub-key gradients, by the update, so it
 *             must stay unchanged until the step has run.
 *   Vtarget   device [B][T][dv], element type v_dtype (the caller aligns
 *             targets with queries, e.g. the lookahead pairing q_t, v_{t+1}).
 *   gate      device fp32 [B][T]; also the token weight of the MSE loss.
 *   eta       learning rate (>= 0); 0 leaves the tables bit-unchanged.
 *   lambda_entropy  weight of the marginal-entropy addressing term (>= 0).
 *   out       device fp32 [B][T][dv], written for every token.
 * Asynchronous on `stream`; kernel faults surface as FWPKM_ECUDA on a later
 * call or at synchronisation.  Inputs must not alias `out` or the tables.
 */
fwpkm_status fwpkm_step(fwpkm_state *s, int B, int T, const void *Q, int q_dtype,
                        const void *Vtarget, int v_dtype, const float *gate, float eta,
                        float lambda_entropy, float *out, void *stream);

/* Flags of fwpkm_step_ex. */
#define FWPKM_LOOKAHEAD 1 /* write query t towards the target of token t+1 */

/*
 * fwpkm_step_ex -- fwpkm_step with the write's token weights and target
 * pairing chosen by the caller.  [GS-2 lookahead targets; SS-TOC weighting
 * the MSE loss by token importance]
 *   omega     device fp32 [B][T], or NULL: the weight w_t of token t in the
 *             MSE loss, L = sum_t w_t ||yhat_t - target_t||^2 + lambda * ...,
 *             used for dL/dV and dL/dK; NULL makes it the gate, as in
 *             fwpkm_step.  The gate still scales the output, out_t = g_t yhat_t.
 *             A token with weight 0 is read but pulls no row towards its
 *             target (its pairs still count in the rows' C_i = sum of w/H).
 *   flags     0 or FWPKM_LOOKAHEAD.  With FWPKM_LOOKAHEAD the query of token
 *             t is written towards Vtarget[t+1] (of the same sequence), and
 *             the last token of the call, which has no next target, gets
 *             weight 0; the call's tokens are the unit, so chained calls each
 *             lose their last token's write.  Vtarget is then read one row
 *             ahead, the whole [B][T] buffer as in fwpkm_step.
 * Other arguments, checks and asynchrony as fwpkm_step (which is
 * fwpkm_step_ex with omega = NULL and flags = 0).  FWPKM_EINVAL for unknown
 * flags.
 */
fwpkm_status fwpkm_step_ex(fwpkm_state *s, int B, int T, const void *Q, int q_dtype,
                           const void *Vtarget, int v_dtype, const float *gate,
                           const float *omega, int flags, float eta, float lambda_entropy,
                           float *out, void *stream);

/*
 * fwpkm_step_host -- fwpkm_step over HOST buffers (same layouts).  Copies Q,
 * Vtarget and gate to state-owned device staging buffers, runs the step, and
 * copies `out` back, chunk by chunk: a chunk's input rows go in on one copy
 * stream of the state and its output rows come back on another while later
 * chunks compute on `stream`, so the copies overlap the step.  Work already
 * enqueued on `stream` comes first; the call returns once everything it
 * enqueued has finished.  Pinned host memory gives the fastest copies (and
 * the overlap); pageable memory also works.  Calls are not replayed as
 * graphs.
 */
fwpkm_status fwpkm_step_host(fwpkm_state *s, int B, int T, const void *Q_host, int q_dtype,
                             const void *Vtarget_host, int v_dtype, const float *gate_host,
                             float eta, float lambda_entropy, float *out_host, void *stream);

/*
 * fwpkm_step_host_ex -- fwpkm_step_ex over HOST buffers: omega_host (fp32
 * [B][T] or NULL) and flags as in fwpkm_step_ex, everything else as in
 * fwpkm_step_host (which is this call with omega_host = NULL, flags = 0).
 * With FWPKM_LOOKAHEAD a chunk's read waits for the next chunk's input copy,
 * whose first target row it takes.
 */
fwpkm_status fwpkm_step_host_ex(fwpkm_state *s, int B, int T, const void *Q_host, int q_dtype,
                                const void *Vtarget_host, int v_dtype, const float *gate_host,
                                const float *omega_host, int flags, float eta,
                                float lambda_entropy, float *out_host, void *stream);

/*
 * fwpkm_state_get / fwpkm_state_set -- copy the fast weights out / in, for
 * chaining memories across calls and for iterative re-reading.  [PYPI Usage]
 *   subkeys  fp32 [heads][2][n][dq/2]   (half 0 scores the first dq/2 dims)
 *   values   fp32 [N][dv]
 * Either pointer may be NULL to skip that table.  Pointers may be device or
 * host memory (stream-ordered copies).
 */
fwpkm_status fwpkm_state_get(const fwpkm_state *s, float *subkeys, float *values, void *stream);
fwpkm_status fwpkm_state_set(fwpkm_state *s, const float *subkeys, const float *values,
                             void *stream);

/*
 * fwpkm_record_selection -- arm a record of the slots and weights the NEXT
 * fwpkm_step reads (device int32 / fp32, [B][T][heads][topk]; the k slots of
 * a token-head in no particular order),
 * for inspection and parity checks.  Pass NULL, NULL to disarm.  The buffers
 * must hold B*T*heads*topk entries of the next call's B and T.
 */
fwpkm_status fwpkm_record_selection(fwpkm_state *s, int32_t *slots, float *weights);

/*
 * fwpkm_force_selection -- for the NEXT fwpkm_step, make every token-head
 * whose mask byte is non-zero read the given slots instead of its own top-k
 * (their weights are still the softmax of the state's own scores of those
 * slots).  slots: device int32 [B][T][heads][topk], values in [0, N) and
 * distinct per token-head; mask: device uint8 [B][T][heads].  Used to replay
 * a selection, e.g. an external decision at exact or near ties.  NULL, NULL
 * disarms.  Out-of-range slots are clamped into [0, N).
 */
fwpkm_status fwpkm_force_selection(fwpkm_state *s, const int32_t *slots, const uint8_t *mask);

/*
 * fwpkm_set_graphs -- enable (default) or disable the replay of repeated calls
 * as CUDA graphs.  When enabled, a fwpkm_step whose arguments (B, T, tensor
 * pointers, dtypes, eta, lambda, the armed force/record buffers) repeat those
 * of an earlier call -- the usual case of a training or serving loop over
 * fixed buffers -- is captured the second time it is seen and replayed as one
 * graph launch afterwards (at most 8 graphs per state, least recently used
 * dropped).  The results are identical either way.  Graphs are dropped when
 * the scratch grows or eps changes, and never used while profiling is on.
 */
fwpkm_status fwpkm_set_graphs(fwpkm_state *s, int enable);

/*
 * Per-kernel timing.  With profiling on, fwpkm_step records a CUDA event pair
 * around every kernel of the chunk it enqueues and launches without
 * programmatic dependent launch or graphs, so the per-kernel times add up to
 * more than an unprofiled step takes; fwpkm_profile_read synchronises
 * `stream`, adds up the elapsed times per kind, and returns them:
 *   names[i] (static strings), ms[i] (total milliseconds), launches[i]
 *   (kernels launched), for i < *count (<= max_kinds).  Reading resets the
 *   totals.
 */
fwpkm_status fwpkm_set_profiling(fwpkm_state *s, int enable);
fwpkm_status fwpkm_profile_read(fwpkm_state *s, const char **names, double *ms,
                                int64_t *launches, int max_kinds, int *count, void *stream);

/*
 * fwpkm_read_stats -- counters accumulated on the device since the last
 * reset (synchronises `stream`): chunks processed, and the sums over those
 * chunks of distinct value rows written, distinct sub-key rows written and
 * member records grouped (pairs plus sub-key entries; the write traffic of
 * the step is proportional to these).  device_errors receives the sticky
 * device error bits:
 *    1  reserved (no longer set: the read reads its rows directly and waits
 *       for nothing),
 *    2  the apply's partial pool overflowed (the launch sizing rules it out),
 *    4  a bucket-scan CTA gave up waiting for an earlier CTA's total,
 *    8  the score's bounded wait on its TMA ring or its MMAs gave up,
 *   16  reserved (no longer set: the list of large buckets holds them all).
 * A kernel that gives up still lets its own copies in flight land and
 * returns; no kernel traps.  Once a bit is set, the kernels after the bucket
 * scan (read, sort, apply) skip the rest of the call and of later calls,
 * writing nothing, until the bits are reset: the tables keep the values of
 * the last complete chunk.  When any bit is set the call returns
 * FWPKM_ECUDA.  reset != 0 zeroes the counters and the bits after reading.
 * Any output pointer may be NULL.
 */
fwpkm_status fwpkm_read_stats(fwpkm_state *s, int64_t *chunks, int64_t *value_rows,
                              int64_t *key_rows, int64_t *records, uint32_t *device_errors,
                              int reset, void *stream);

/*
 * fwpkm_set_wait_limits -- bounds of the device-side waits of this state's
 * steps (and of fwpkm_select_noalloc on it), for failure detection and its
 * tests.  mbar_polls bounds the first wait on an mbarrier (the score's TMA
 * ring and MMA completion; default 2^26 polls);
 * scan_polls bounds a bucket-scan CTA's wait for the totals of the CTAs
 * before it (default 2^24).  A negative value restores the default; 0 makes
 * the wait give up at once.  A wait that gives up sets its error bit
 * (fwpkm_read_stats), and the kernel still waits, with a fixed bound of its
 * own, for the copies it has in flight before it returns.
 */
fwpkm_status fwpkm_set_wait_limits(fwpkm_state *s, int64_t mbar_polls, int64_t scan_polls);

/*
 * fwpkm_inject_alloc_failures -- make the next `count` device allocations of
 * the library (tables in fwpkm_state_init, scratch growth in fwpkm_step,
 * staging in fwpkm_step_host) fail as an exhausted device would, returning
 * FWPKM_ENOMEM with the state unchanged.  Process-wide; 0 disarms.  For
 * failure-detection tests: it exercises the allocation error paths without
 * exhausting a shared device.
 */
void fwpkm_inject_alloc_failures(int count);

/*
 * fwpkm_select_noalloc -- the product-key selection of the read, for callers
 * that cannot allocate device memory when they call (a serving process that
 * plans every device byte ahead and runs with a fixed budget, or a plugin
 * whose host framework owns the device allocator; cudaMalloc may also
 * synchronise the device).  The paper has no counterpart of this entry point;
 * it is a deployment variant of the selection done inside fwpkm_step.
 *   For every token t of the B sequences and every head h, scores both query
 *   halves against the state's current sub-key tables (with the state's
 *   score: IDW, or the dot product under FWPKM_SCORE_DOT), takes the product-key
 *   top-k and writes the slots and their softmax weights -- the same values
 *   fwpkm_step reads for that token with the same tables.  No readout and no
 *   update: the tables are not modified.
 *   Q        device [B][T][heads*dq], element type q_dtype (FWPKM_F32/BF16).
 *   slots    device int32 [B][T][heads][topk] (output; the k slots of a
 *            token-head in no particular order, the same order fwpkm_step reads).
 *   weights  device fp32  [B][T][heads][topk] (output).
 * Allocates nothing: all scratch is one 16 MiB array in the library's device
 * image (resident on every GPU that loads the library until exit), used in
 * passes of as many time steps as fit.  A time step of B sequences takes
 * B x 2*heads*(dq + n + 1) x 4 bytes (both TF32 parts of each query half,
 * its norm, its n distances); on top comes a fixed part: the hi/lo split of
 * the sub-key tables, their norms, and rounding to whole 128-row score tiles.
 * A call whose single time step does not fit in 16 MiB is rejected with
 * FWPKM_ESHAPE before anything is enqueued; when the fixed part alone (the
 * sub-key tables' split, e.g. heads >= 1 with n = 1024 and dq = 2048) is
 * over 16 MiB, no batch size fits, and the message says so.  The
 * first call on a device looks the arrays' addresses up (cudaGetSymbolAddress,
 * once per device, with that device current); make that first call before any
 * stream capture.  All calls share the arrays: calls that overlap on the GPU
 * (other streams or threads) race and must be ordered by the caller.
 *   device_errors  optional (NULL = not reported): device or host memory
 *            that receives, stream-ordered after the call's kernels, the
 *            call's device error bits (8 = the score's bounded TMA/MMA wait
 *            gave up, see fwpkm_set_wait_limits; 0 = none).  When it is
 *            non-zero the slots and weights of the call are not meaningful
 *            (slots stay in [0, N)).  The bits live in a second static block
 *            of the library image that every call zeroes on its stream first.
 * Asynchronous on `stream`.
 */
fwpkm_status fwpkm_select_noalloc(fwpkm_state *s, int B, int T, const void *Q, int q_dtype,
                                  int32_t *slots, float *weights, uint32_t *device_errors,
                                  void *stream);

/* Message of the last failure on this thread ("" if none). */
const char *fwpkm_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* FWPKM_H_ */
