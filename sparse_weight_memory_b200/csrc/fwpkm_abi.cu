// fwpkm_abi.cu -- host side of the C ABI declared in include/fwpkm.h.
//
// The state owns the fast weights (sub-key tables and value table, fp32) and
// one device scratch arena sized for the largest chunk seen.  fwpkm_step
// validates everything on the host, then enqueues the per-chunk kernel
// sequence on the caller's stream with no host synchronisation: chunk c+1's
// kernels are ordered after chunk c's update by the stream itself
// (gist.science section 2: updates are applied after a chunk; the next chunk
// reads the updated weights).
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <functional>
#include <string>
#include <vector>

#include "../../include/fwpkm.h"
#include "fwpkm_internal.cuh"

using namespace fwpkm;

namespace {

thread_local std::string g_last_error;

fwpkm_status fail(fwpkm_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

fwpkm_status cuda_fail(cudaError_t e, const char *what) {
  return fail(FWPKM_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Device allocations the library is still told to fail (fwpkm_inject_alloc_failures).
std::atomic<int> g_fail_allocs{0};

// cudaMalloc, unless an injected failure is pending: then nothing is
// allocated and the call reports what an exhausted device would.
cudaError_t dev_malloc(void **p, size_t bytes) {
  int n = g_fail_allocs.load();
  while (n > 0) {
    if (g_fail_allocs.compare_exchange_weak(n, n - 1)) {
      *p = nullptr;
      return cudaErrorMemoryAllocation;
    }
  }
  return cudaMalloc(p, bytes);
}

enum Kind { K_PREP, K_SCORE, K_TOPK, K_SCAN, K_READ, K_BSORT, K_APPLY, K_PGRAD, K_COUNT };
const char *kKindNames[K_COUNT] = {"fwpkm_prep", "fwpkm_score", "fwpkm_topk",  "fwpkm_scan",
                                   "fwpkm_read", "fwpkm_bsort", "fwpkm_apply", "fwpkm_pgrad"};
// Kernels one call of a kind enqueues.
const int kKernelsPerCall[K_COUNT] = {1, 1, 1, 1, 1, 1, 1, 1};

struct Timing {
  int kind;
  cudaEvent_t a, b;
};

}  // namespace

// Everything a call's enqueued work depends on besides the state's own
// buffers: a call with the same key enqueues exactly the same kernels with
// the same parameters, so it can replay a captured graph.
struct StepKey {
  int B, T, q_dtype, v_dtype;
  const void *Q, *Vt;
  const float *gate, *omega;
  int lookahead;
  float *out;
  float eta, lam;
  Extras x;
  bool operator==(const StepKey &o) const {
    return B == o.B && T == o.T && q_dtype == o.q_dtype && v_dtype == o.v_dtype && Q == o.Q &&
           Vt == o.Vt && gate == o.gate && omega == o.omega && lookahead == o.lookahead &&
           out == o.out && eta == o.eta && lam == o.lam &&
           x.force_slots == o.x.force_slots && x.force_mask == o.x.force_mask &&
           x.rec_slots == o.x.rec_slots && x.rec_w == o.x.rec_w;
  }
};
struct StepGraph {
  StepKey key;
  cudaGraphExec_t exec;
  uint64_t last_use;
};
constexpr size_t kGraphCache = 8;
constexpr size_t kGraphSeen = 16;

struct fwpkm_state {
  int64_t N = 0;
  int n = 0, dq = 0, dh = 0, dv = 0, k = 0, chunk = 0, H = 0;
  int nmem = 1;  // memories: 1 shared, or one per sequence (fwpkm_state_init_batched)
  float eps = 1e-3f;
  int device = 0;
  int sm_count = 148;
  // bounds of the device-side waits (fwpkm_set_wait_limits)
  long long mbar_polls = kDefaultMbarPolls, scan_polls = kDefaultScanPolls;
  // readings (fwpkm_state_set_options)
  int heads_sum = 0, agg = AGG_WEIGHT, score_dot = 0;
  float *K = nullptr;  // [nmem][H][2][n][dh]
  float *V = nullptr;  // [nmem][N][dv]
  // scratch arena
  void *arena = nullptr;
  size_t arena_bytes = 0;
  int64_t cap_rows = 0;
  Scratch s{};
  TcMaps maps{};  // TMA descriptors of the score operands in the arena
  // optional per-step inputs / outputs, armed for the next step
  Extras x{};
  // host-buffer staging
  void *stage = nullptr;
  size_t stage_bytes = 0;
  // profiling
  bool profiling = false;
  std::vector<Timing> timings;
  std::vector<cudaEvent_t> event_pool;
  double prof_ms[K_COUNT] = {};
  int64_t prof_n[K_COUNT] = {};
  // the TF32 split and chunk norms of the sub-key rows in the arena are out of date
  bool subkey_split_stale = true;
  // host-buffer calls: copy streams (inputs in, outputs out)
  cudaStream_t h2d_stream = nullptr, d2h_stream = nullptr;
  // replay of repeated calls as CUDA graphs
  bool graphs = true;
  cudaStream_t capture_stream = nullptr;
  std::vector<StepGraph> graph_cache;   // at most kGraphCache, least recently used first out
  std::vector<StepKey> graph_seen;      // keys met once, most recent last
  uint64_t graph_tick = 0;
};

namespace {

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Value rows are bucketed by slot >> vshift.  The bucket count follows the
// chunk's pair capacity P: at least 8192 buckets (a few slots each, so rows
// that many pairs share rarely meet in one bucket), more for large chunks
// (about four pairs per bucket without skew), at most 65536 and never more
// than N.  A bucket is then usually small enough for one warp to sort.
int value_shift(int64_t N, int64_t P) {
  int64_t target = 8192;
  while (target < P / 4 && target < 65536) target <<= 1;
  int sh = 0;
  while (sh < 40 && ((N + (1ll << sh) - 1) >> sh) > target) ++sh;
  return sh;
}
int64_t value_buckets(int64_t N, int64_t P) {
  const int sh = value_shift(N, P);
  return (N + (1ll << sh) - 1) >> sh;
}

void clear_graphs(fwpkm_state *st);

// Carve the scratch arena for `rows` token rows per chunk.
fwpkm_status ensure_scratch(fwpkm_state *st, int64_t rows) {
  if (rows <= st->cap_rows) return FWPKM_OK;
  rows = (rows + 127) / 128 * 128;  // query-half stride: whole 128-row score tiles
  const int64_t H = st->H, n = st->n, dh = st->dh, dv = st->dv, k = st->k;
  const int64_t nm = st->nmem, Nt = st->N * nm;  // all memories' value rows
  const int64_t M = rows * H, P = M * k, NB = value_buckets(Nt, P) + 2 * H * nm * n;
  const int64_t Lcap = 3 * P;  // pairs + at most 2 entries per pair
  // Blocks of groups of more than 4 members, 32 members a block: at most
  // L/32 + L/5 of them, under L/4.
  const int64_t pool_cap = Lcap / 4 + 2;
  const int pwidth = kPartHead + (int)(dv > dh ? dv : dh);
  struct Piece {
    void **ptr;
    size_t bytes;
  };
  Scratch s{};
  std::vector<Piece> pieces = {
      {(void **)&s.Qs_hi, sizeof(float) * (size_t)(H * 2 * rows * dh)},
      {(void **)&s.Qs_lo, sizeof(float) * (size_t)(H * 2 * rows * dh)},
      {(void **)&s.qn, sizeof(float) * (size_t)(H * 2 * rows)},
      {(void **)&s.K_hi, sizeof(float) * (size_t)((H * nm * 2 * n + 128) * dh)},
      {(void **)&s.K_lo, sizeof(float) * (size_t)((H * nm * 2 * n + 128) * dh)},
      {(void **)&s.kn, sizeof(float) * (size_t)(H * nm * 2 * n * kKnChunks)},
      {(void **)&s.D, sizeof(float) * (size_t)(H * 2 * rows * n)},
      {(void **)&s.pslot, sizeof(int32_t) * (size_t)P},
      {(void **)&s.pw, sizeof(float) * (size_t)P},
      {(void **)&s.pclaim, sizeof(int32_t) * (size_t)P},
      {(void **)&s.pa, sizeof(float) * (size_t)P},
      {(void **)&s.pb, sizeof(float) * (size_t)P},
      {(void **)&s.esub, sizeof(int32_t) * (size_t)(2 * P)},
      {(void **)&s.emask, sizeof(uint32_t) * (size_t)(2 * P)},
      {(void **)&s.einv, sizeof(float) * (size_t)(2 * P)},
      {(void **)&s.eclaim, sizeof(int32_t) * (size_t)(2 * P)},
      {(void **)&s.ealpha, sizeof(float) * (size_t)(2 * P)},
      {(void **)&s.ecount, sizeof(int32_t) * (size_t)(2 * M)},
      {(void **)&s.bcnt, sizeof(int32_t) * (size_t)NB},
      {(void **)&s.boff, sizeof(int32_t) * (size_t)(NB + 1)},
      {(void **)&s.rec_in, sizeof(Member) * (size_t)Lcap},
      {(void **)&s.rec, sizeof(Member) * (size_t)Lcap},
      {(void **)&s.posmap, sizeof(int32_t) * (size_t)Lcap},
      {(void **)&s.shortlist[0], sizeof(int32_t) * (size_t)Lcap},
      {(void **)&s.shortlist[1], sizeof(int32_t) * (size_t)Lcap},
      {(void **)&s.biglist, sizeof(int32_t) * (size_t)NB},
      {(void **)&s.longlist[0], sizeof(int32_t) * (size_t)Lcap},
      {(void **)&s.longlist[1], sizeof(int32_t) * (size_t)Lcap},
      {(void **)&s.arrive, sizeof(int32_t) * (size_t)pool_cap * kMaxChunks},
      {(void **)&s.sort_tmp, sizeof(uint64_t) * (size_t)(2 * Lcap)},
      {(void **)&s.partial, sizeof(float) * (size_t)pool_cap * pwidth},
      {(void **)&s.scan_sync, sizeof(unsigned long long) * (size_t)(1 + kScanMaxCtas)},
      {(void **)&s.E, sizeof(float) * (size_t)(rows * dv)},
      {(void **)&s.meta, sizeof(Meta)},
  };
  s.Lcap = Lcap;
  s.pwidth = pwidth;
  s.pool_cap = (int)pool_cap;
  size_t total = 0;
  for (auto &p : pieces) total = align_up(total, 256) + align_up(p.bytes, 256);
  cudaError_t e = cudaSuccess;
  if (st->arena) {
    // Work still in flight may use the old arena and update the stats block
    // that is carried over below.
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "scratch growth: synchronise");
  }
  void *arena = nullptr;
  e = dev_malloc(&arena, total);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FWPKM_ENOMEM, "scratch allocation of %zu bytes failed: %s", total,
                cudaGetErrorString(e));
  }
  size_t off = 0;
  for (auto &p : pieces) {
    off = align_up(off, 256);
    *p.ptr = (char *)arena + off;
    off += align_up(p.bytes, 256);
  }
  // Bucket counts start at zero (the kernels leave them at zero); the meta
  // block (stats) carries over.
  e = cudaMemset(s.bcnt, 0, sizeof(int32_t) * (size_t)NB);
  if (e == cudaSuccess) e = cudaMemset(s.arrive, 0, sizeof(int32_t) * (size_t)pool_cap * kMaxChunks);
  if (e == cudaSuccess)
    e = cudaMemset(s.scan_sync, 0, sizeof(unsigned long long) * (size_t)(1 + kScanMaxCtas));
  if (e == cudaSuccess) e = cudaMemset(s.meta, 0, sizeof(Meta));
  if (e == cudaSuccess && st->s.meta)
    e = cudaMemcpy(s.meta, st->s.meta, sizeof(Meta), cudaMemcpyDeviceToDevice);
  // The initialisation ran on the legacy default stream, which a caller's
  // non-blocking stream does not wait for: finish it before any kernel can
  // touch the arena.
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaFree(arena);
    return cuda_fail(e, "scratch initialisation");
  }
  TcMaps maps;
  e = encode_score_maps(&maps, s, (int)H, (int)nm, (int)rows, (int)n, (int)dh);
  if (e != cudaSuccess) {
    cudaFree(arena);
    return cuda_fail(e, "scratch initialisation: tensor maps");
  }
  if (st->arena) cudaFree(st->arena);  // drained above
  clear_graphs(st);  // captured graphs hold the old arena's addresses
  st->maps = maps;
  st->arena = arena;
  st->arena_bytes = total;
  st->s = s;
  st->cap_rows = rows;
  st->subkey_split_stale = true;  // the new arena holds no sub-key split yet
  return FWPKM_OK;
}

cudaEvent_t take_event(fwpkm_state *st) {
  if (!st->event_pool.empty()) {
    cudaEvent_t e = st->event_pool.back();
    st->event_pool.pop_back();
    return e;
  }
  cudaEvent_t e;
  cudaEventCreate(&e);
  return e;
}

// Launch wrapper: optional event pair around the kernel, error check after.
template <typename F>
fwpkm_status run(fwpkm_state *st, int kind, cudaStream_t stream, F &&launch) {
  Timing t{kind, nullptr, nullptr};
  if (st->profiling) {
    t.a = take_event(st);
    t.b = take_event(st);
    cudaEventRecord(t.a, stream);
  }
  cudaError_t e = launch();
  if (e != cudaSuccess) return cuda_fail(e, kKindNames[kind]);
  if (st->profiling) {
    cudaEventRecord(t.b, stream);
    st->timings.push_back(t);
  }
  return FWPKM_OK;
}

bool is_dtype(int t) { return t == FWPKM_F32 || t == FWPKM_BF16; }

// Shapes of chunk c of a call (B sequences of T tokens).
Dims chunk_dims(const fwpkm_state *st, int B, int T, int c, float eta, float lambda_entropy) {
  Dims d{};
  d.n = st->n;
  d.dq = st->dq;
  d.dh = st->dh;
  d.dv = st->dv;
  d.k = st->k;
  d.H = st->H;
  d.N = st->N;
  d.B = B;
  d.T = T;
  d.t0 = c * st->chunk;
  d.Tc = (T - d.t0 < st->chunk) ? T - d.t0 : st->chunk;
  d.rows = B * d.Tc;
  d.qstride = (int)st->cap_rows;
  d.M = d.rows * st->H;
  d.nmem = st->nmem;
  d.Nt = st->N * st->nmem;
  d.rstride = st->nmem > 1 ? (d.Tc + 127) / 128 * 128 : d.Tc;
  d.drows = B * d.rstride;
  d.Mmem = d.M / st->nmem;
  const int64_t cap_pairs = st->cap_rows * st->H * st->k;  // bcnt was sized for this
  d.vshift = value_shift(d.Nt, cap_pairs);
  d.NBv = (int)value_buckets(d.Nt, cap_pairs);
  d.NB = d.NBv + 2 * st->H * st->nmem * st->n;
  d.sm_count = st->sm_count;
  d.pdl = st->profiling ? 0 : 1;  // per-kernel events need plain stream order
  d.eps = st->eps;
  d.eta = eta;
  d.lam = lambda_entropy;
  d.mbar_polls = st->mbar_polls;
  d.scan_polls = st->scan_polls;
  d.heads_sum = st->heads_sum;
  d.agg = st->agg;
  d.score_dot = st->score_dot;
  return d;
}

// The TF32 split and chunk norms of every sub-key row (new tables or a new
// scratch arena); afterwards the update keeps those of the rows it writes.
fwpkm_status split_all_subkeys(fwpkm_state *st, cudaStream_t stream) {
  Dims d = chunk_dims(st, 1, 1, 0, 0.f, 0.f);
  d.pdl = 0;
  return run(st, K_PREP, stream, [&] { return launch_prep_k(d, st->K, st->s, stream); });
}

// Scratch for chunks of `rows_max` rows, and the sub-key split if it is out
// of date (never inside a captured graph: a new arena drops them).
fwpkm_status prepare_step(fwpkm_state *st, int64_t rows_max, cudaStream_t stream) {
  fwpkm_status rc = ensure_scratch(st, rows_max);
  if (rc != FWPKM_OK) return rc;
  if (st->subkey_split_stale) {
    if ((rc = split_all_subkeys(st, stream))) return rc;
    st->subkey_split_stale = false;
  }
  return FWPKM_OK;
}

// Points of the chunk loop where a host-buffer call synchronises its copies:
// need_inputs(c) before the first kernel that reads chunk c's inputs (the
// first chunk's prep, else the previous chunk's sort, which prepares chunk
// c's query halves), read_done(c) once chunk c's outputs are written.
struct ChunkHooks {
  std::function<cudaError_t(int)> need_inputs;
  std::function<cudaError_t(int)> read_done;
};

// The chunk loop of one call: every kernel of every chunk, in order, on
// `stream`.  No host synchronisation.
fwpkm_status enqueue_chunks(fwpkm_state *st, int B, int T, const void *Q, int q_dtype,
                            const void *Vtarget, int v_dtype, const float *gate,
                            const float *omega, int lookahead, float eta,
                            float lambda_entropy, float *out, const Extras &x,
                            cudaStream_t stream, const ChunkHooks *hooks = nullptr) {
  fwpkm_status rc = FWPKM_OK;
  auto hook = [&](const std::function<cudaError_t(int)> &f, int c) -> fwpkm_status {
    if (!hooks || !f) return FWPKM_OK;
    const cudaError_t e = f(c);
    return e == cudaSuccess ? FWPKM_OK : cuda_fail(e, "step_host: copy pipeline");
  };

  const Scratch &s = st->s;
  const int n_chunks = (T + st->chunk - 1) / st->chunk;
  // eta = 0 changes no table, so the write kernels are skipped altogether (a
  // read-only memory, as a static product-key memory is): each chunk is its
  // query halves, the score, the selection and the read.
  const bool readonly = eta == 0.f;
  for (int c = 0; c < n_chunks; ++c) {
    Dims d = chunk_dims(st, B, T, c, eta, lambda_entropy);
    d.lookahead = lookahead;
    d.q_tf32_exact = q_dtype == FWPKM_BF16 ? 1 : 0;
    d.readonly = readonly ? 1 : 0;
    // the halves of a later chunk of the write path come from the previous
    // chunk's sort, two grids or more before this chunk's score
    d.q_early = !readonly && c > 0 ? 1 : 0;
    if (readonly) {
      if ((rc = hook(hooks ? hooks->need_inputs : nullptr, c))) return rc;
      if (lookahead && c + 1 < n_chunks &&
          (rc = hook(hooks ? hooks->need_inputs : nullptr, c + 1)))
        return rc;
      if ((rc = run(st, K_PREP, stream, [&] { return launch_prep_q(d, Q, q_dtype, s, stream); })))
        return rc;
      if ((rc = run(st, K_SCORE, stream, [&] { return launch_score(d, s, st->maps, stream); })))
        return rc;
      if ((rc = run(st, K_TOPK, stream, [&] { return launch_topk(d, s, x, stream); }))) return rc;
      if ((rc = run(st, K_READ, stream, [&] {
             return launch_read(d, st->V, Vtarget, v_dtype, gate, omega, out, s, stream);
           })))
        return rc;
      if ((rc = hook(hooks ? hooks->read_done : nullptr, c))) return rc;
      continue;
    }
    // the next chunk of this call, whose query halves the sort prepares
    Dims dn{};
    if (c + 1 < n_chunks) dn = chunk_dims(st, B, T, c + 1, eta, lambda_entropy);
    float *V = st->V, *K = st->K;
    // the first chunk's query halves; later chunks' come with the previous sort
    if (c == 0 && (rc = hook(hooks ? hooks->need_inputs : nullptr, 0))) return rc;
    if (c == 0 &&
        (rc = run(st, K_PREP, stream, [&] { return launch_prep_q(d, Q, q_dtype, s, stream); })))
      return rc;
    if ((rc = run(st, K_SCORE, stream, [&] { return launch_score(d, s, st->maps, stream); })))
      return rc;
    if ((rc = run(st, K_TOPK, stream, [&] { return launch_topk(d, s, x, stream); }))) return rc;
    if ((rc = run(st, K_SCAN, stream, [&] { return launch_scan(d, s, stream); }))) return rc;
    // with the lookahead pairing the read also takes the first target row of
    // the next chunk, so that chunk's inputs are needed before it
    if (lookahead && dn.rows > 0 && (rc = hook(hooks ? hooks->need_inputs : nullptr, c + 1)))
      return rc;
    if ((rc = run(st, K_READ, stream, [&] {
           return launch_read(d, V, Vtarget, v_dtype, gate, omega, out, s, stream);
         })))
      return rc;
    if ((rc = hook(hooks ? hooks->read_done : nullptr, c))) return rc;
    if (!lookahead && dn.rows > 0 && (rc = hook(hooks ? hooks->need_inputs : nullptr, c + 1)))
      return rc;
    if ((rc = run(st, K_BSORT, stream,
                  [&] { return launch_bsort(d, s, dn, Q, q_dtype, stream); })))
      return rc;
    if (lambda_entropy == 0.f) {
      if ((rc = run(st, K_APPLY, stream, [&] { return launch_apply(d, V, K, Q, q_dtype, s, stream, 0); })))
        return rc;
    } else {
      if ((rc = run(st, K_APPLY, stream, [&] { return launch_apply(d, V, K, Q, q_dtype, s, stream, 1); })))
        return rc;
      if ((rc = run(st, K_PGRAD, stream, [&] { return launch_pgrad(d, s, stream); }))) return rc;
      if ((rc = run(st, K_APPLY, stream, [&] { return launch_apply(d, V, K, Q, q_dtype, s, stream, 2); })))
        return rc;
    }
  }
  return FWPKM_OK;
}

// Captures the chunk loop of `key` into an executable graph on the state's
// own stream (the caller's stream may be the legacy default stream, which
// cannot be captured).  Returns null when capture or instantiation fails.
cudaGraphExec_t capture_chunks(fwpkm_state *st, const StepKey &key) {
  if (!st->capture_stream &&
      cudaStreamCreateWithFlags(&st->capture_stream, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    st->capture_stream = nullptr;
    return nullptr;
  }
  if (cudaStreamBeginCapture(st->capture_stream, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  const fwpkm_status rc =
      enqueue_chunks(st, key.B, key.T, key.Q, key.q_dtype, key.Vt, key.v_dtype, key.gate,
                     key.omega, key.lookahead, key.eta, key.lam, key.out, key.x,
                     st->capture_stream);
  cudaGraph_t graph = nullptr;
  const cudaError_t e = cudaStreamEndCapture(st->capture_stream, &graph);
  cudaGraphExec_t exec = nullptr;
  if (rc == FWPKM_OK && e == cudaSuccess && graph &&
      cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess)
    exec = nullptr;
  if (graph) cudaGraphDestroy(graph);
  cudaGetLastError();  // a failed capture leaves nothing sticky behind
  return exec;
}

void clear_graphs(fwpkm_state *st) {
  for (auto &g : st->graph_cache) cudaGraphExecDestroy(g.exec);
  st->graph_cache.clear();
  st->graph_seen.clear();
}


}  // namespace

namespace fwpkm {
bool state_view(const fwpkm_state *st, StateView *v) {
  if (!st || !v) return false;
  v->N = st->N;
  v->n = st->n;
  v->dq = st->dq;
  v->dh = st->dh;
  v->dv = st->dv;
  v->k = st->k;
  v->chunk = st->chunk;
  v->H = st->H;
  v->device = st->device;
  v->sm_count = st->sm_count;
  v->nmem = st->nmem;
  v->eps = st->eps;
  v->K = st->K;
  v->mbar_polls = st->mbar_polls;
  v->score_dot = st->score_dot;
  return true;
}
void set_last_error(const char *msg) { g_last_error = msg; }
}  // namespace fwpkm

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char *fwpkm_last_error(void) { return g_last_error.c_str(); }

fwpkm_status fwpkm_state_init(int64_t N, int dq, int dv, int topk, int chunk, int heads,
                              fwpkm_state **out) {
  return fwpkm_state_init_batched(N, dq, dv, topk, chunk, heads, 1, out);
}

fwpkm_status fwpkm_state_init_batched(int64_t N, int dq, int dv, int topk, int chunk, int heads,
                                      int memories, fwpkm_state **out) {
  if (!out) return fail(FWPKM_EINVAL, "state_init: out is NULL");
  *out = nullptr;
  int64_t n = (int64_t)std::llround(std::sqrt((double)N));
  while (n * n > N) --n;
  while ((n + 1) * (n + 1) <= N) ++n;
  if (N < 16 || n * n != N || n > FWPKM_MAX_SUBKEYS)
    return fail(FWPKM_ESHAPE, "state_init: N=%lld must be n*n with 4 <= n <= %d", (long long)N,
                FWPKM_MAX_SUBKEYS);
  if (dq < 16 || dq % 16 != 0 || dq / 2 > 1024)
    return fail(FWPKM_ESHAPE, "state_init: dq=%d must be a multiple of 16 (dq/2 a multiple of 8), <= 2048", dq);
  if (dv < 4 || dv % 4 != 0 || dv > 2048)
    return fail(FWPKM_ESHAPE, "state_init: dv=%d must be a multiple of 4 in [4, 2048]", dv);
  if (topk < 1 || topk > FWPKM_MAX_TOPK || topk > n)
    return fail(FWPKM_ESHAPE, "state_init: topk=%d must be in [1, min(n=%lld, %d)]", topk,
                (long long)n, FWPKM_MAX_TOPK);
  if (chunk < 1 || chunk > (1 << 20))
    return fail(FWPKM_ESHAPE, "state_init: chunk=%d must be in [1, 2^20]", chunk);
  if (heads < 1 || heads > 16)
    return fail(FWPKM_ESHAPE, "state_init: heads=%d must be in [1, 16]", heads);
  // member groups are 32-bit: every value row and sub-key row of all memories
  if (memories < 1 || (int64_t)memories * (N + 2 * heads * n) >= ((int64_t)1 << 31))
    return fail(FWPKM_ESHAPE, "state_init: memories=%d must be >= 1 with memories * (N + "
                "2*heads*n) < 2^31", memories);

  fwpkm_state *st = new (std::nothrow) fwpkm_state();
  if (!st) return fail(FWPKM_ENOMEM, "state_init: host allocation failed");
  st->N = N;
  st->n = (int)n;
  st->dq = dq;
  st->dh = dq / 2;
  st->dv = dv;
  st->k = topk;
  st->chunk = chunk;
  st->H = heads;
  st->nmem = memories;
  cudaGetDevice(&st->device);
  cudaDeviceGetAttribute(&st->sm_count, cudaDevAttrMultiProcessorCount, st->device);
  if (st->sm_count < 1) st->sm_count = 1;
  const size_t kbytes = sizeof(float) * (size_t)memories * heads * 2 * n * st->dh;
  const size_t vbytes = sizeof(float) * (size_t)memories * N * dv;
  cudaError_t e = dev_malloc((void **)&st->K, kbytes);
  if (e == cudaSuccess) e = dev_malloc((void **)&st->V, vbytes);
  if (e == cudaSuccess) e = cudaMemset(st->K, 0, kbytes);
  if (e == cudaSuccess) e = cudaMemset(st->V, 0, vbytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    cudaFree(st->K);
    cudaFree(st->V);
    delete st;
    return fail(e == cudaErrorMemoryAllocation ? FWPKM_ENOMEM : FWPKM_ECUDA,
                "state_init: table allocation (%zu + %zu bytes): %s", kbytes, vbytes,
                cudaGetErrorString(e));
  }
  // ensure_scratch ends with a device synchronisation, so the zeroed tables
  // are in place before a caller's stream (non-blocking ones included) copies
  // into them.
  fwpkm_status rc =
      ensure_scratch(st, memories > 1 ? (int64_t)memories * ((chunk + 127) / 128 * 128) : chunk);
  if (rc != FWPKM_OK) {
    cudaFree(st->K);
    cudaFree(st->V);
    delete st;
    return rc;
  }
  *out = st;
  return FWPKM_OK;
}

void fwpkm_state_free(fwpkm_state *st) {
  if (!st) return;
  cudaDeviceSynchronize();
  for (auto &t : st->timings) {
    cudaEventDestroy(t.a);
    cudaEventDestroy(t.b);
  }
  for (auto e : st->event_pool) cudaEventDestroy(e);
  clear_graphs(st);
  if (st->capture_stream) cudaStreamDestroy(st->capture_stream);
  if (st->h2d_stream) cudaStreamDestroy(st->h2d_stream);
  if (st->d2h_stream) cudaStreamDestroy(st->d2h_stream);
  cudaFree(st->arena);
  cudaFree(st->stage);
  cudaFree(st->K);
  cudaFree(st->V);
  delete st;
}

fwpkm_status fwpkm_state_set_eps(fwpkm_state *st, float eps) {
  if (!st) return fail(FWPKM_EINVAL, "set_eps: state is NULL");
  if (!(eps > 0.f) || !std::isfinite(eps)) return fail(FWPKM_EINVAL, "set_eps: eps must be > 0");
  st->eps = eps;
  clear_graphs(st);  // eps is a kernel parameter of the captured launches
  return FWPKM_OK;
}

fwpkm_status fwpkm_set_wait_limits(fwpkm_state *st, int64_t mbar_polls, int64_t scan_polls) {
  if (!st) return fail(FWPKM_EINVAL, "set_wait_limits: state is NULL");
  st->mbar_polls = mbar_polls < 0 ? kDefaultMbarPolls : (long long)mbar_polls;
  st->scan_polls = scan_polls < 0 ? kDefaultScanPolls : (long long)scan_polls;
  clear_graphs(st);  // the limits are kernel parameters of the captured launches
  return FWPKM_OK;
}

void fwpkm_inject_alloc_failures(int count) { g_fail_allocs.store(count > 0 ? count : 0); }

fwpkm_status fwpkm_state_set_options(fwpkm_state *st, unsigned options) {
  if (!st) return fail(FWPKM_EINVAL, "set_options: state is NULL");
  const unsigned known = FWPKM_HEADS_SUM | FWPKM_AGG_COUNT | FWPKM_AGG_SUM | FWPKM_SCORE_DOT;
  if (options & ~known) return fail(FWPKM_EINVAL, "set_options: unknown bits 0x%x", options);
  if ((options & FWPKM_AGG_COUNT) && (options & FWPKM_AGG_SUM))
    return fail(FWPKM_EINVAL, "set_options: FWPKM_AGG_COUNT and FWPKM_AGG_SUM exclude each other");
  st->heads_sum = (options & FWPKM_HEADS_SUM) ? 1 : 0;
  st->score_dot = (options & FWPKM_SCORE_DOT) ? 1 : 0;
  st->agg = (options & FWPKM_AGG_COUNT) ? AGG_COUNT : ((options & FWPKM_AGG_SUM) ? AGG_SUM : AGG_WEIGHT);
  clear_graphs(st);  // the options are kernel parameters of the captured launches
  return FWPKM_OK;
}

fwpkm_status fwpkm_set_graphs(fwpkm_state *st, int enable) {
  if (!st) return fail(FWPKM_EINVAL, "set_graphs: state is NULL");
  st->graphs = enable != 0;
  if (!st->graphs) clear_graphs(st);
  return FWPKM_OK;
}

fwpkm_status fwpkm_step_ex(fwpkm_state *st, int B, int T, const void *Q, int q_dtype,
                           const void *Vtarget, int v_dtype, const float *gate,
                           const float *omega, int flags, float eta, float lambda_entropy,
                           float *out, void *stream_) {
  if (!st) return fail(FWPKM_EINVAL, "step: state is NULL");
  if (!Q || !Vtarget || !gate || !out) return fail(FWPKM_EINVAL, "step: NULL tensor pointer");
  if (!is_dtype(q_dtype) || !is_dtype(v_dtype))
    return fail(FWPKM_EINVAL, "step: dtype must be FWPKM_F32 or FWPKM_BF16");
  if (flags & ~FWPKM_LOOKAHEAD) return fail(FWPKM_EINVAL, "step: unknown flags 0x%x", flags);
  const int lookahead = (flags & FWPKM_LOOKAHEAD) ? 1 : 0;
  if (B < 1 || T < 1) return fail(FWPKM_ESHAPE, "step: B=%d and T=%d must be >= 1", B, T);
  if (!(eta >= 0.f) || !std::isfinite(eta))
    return fail(FWPKM_EINVAL, "step: eta must be finite and >= 0");
  if (!(lambda_entropy >= 0.f) || !std::isfinite(lambda_entropy))
    return fail(FWPKM_EINVAL, "step: lambda_entropy must be finite and >= 0");
  if (st->nmem > 1 && B != st->nmem)
    return fail(FWPKM_ESHAPE, "step: B=%d must equal the state's %d memories (one per sequence)",
                B, st->nmem);
  const int64_t tc_max = T < st->chunk ? T : st->chunk;
  // rows of the query-half layout: one memory per sequence starts each on a whole score tile
  const int64_t rows_max = (int64_t)B * (st->nmem > 1 ? (tc_max + 127) / 128 * 128 : tc_max);
  if (rows_max * st->H * st->k * 3 >= (int64_t)1 << 31 || (int64_t)B * T * st->dv >= (int64_t)1 << 40)
    return fail(FWPKM_ESHAPE, "step: B*chunk*heads*topk too large for 32-bit pair ids");
  if ((int64_t)B * T * 2 * st->H >= (int64_t)1 << 31)
    return fail(FWPKM_ESHAPE, "step: B*T*heads too large for 32-bit query-half indices");
  if ((rows_max + 127) / 128 > 65535)  // row tiles of the score grid (grid y)
    return fail(FWPKM_ESHAPE, "step: B*chunk = %lld rows exceeds 65535 tiles of 128 rows",
                (long long)rows_max);
  if ((((uintptr_t)Q) | ((uintptr_t)Vtarget) | ((uintptr_t)out)) & 15)
    return fail(FWPKM_EINVAL, "step: Q, Vtarget and out must be 16-byte aligned");
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != st->device)
    return fail(FWPKM_EINVAL, "step: current device %d is not the state's device %d", dev,
                st->device);
  cudaStream_t stream = (cudaStream_t)stream_;
  fwpkm_status rc = prepare_step(st, rows_max, stream);
  if (rc != FWPKM_OK) return rc;
  const Extras x = st->x;
  st->x = Extras{};  // armed extras apply to this step only
  if (!st->graphs || st->profiling)
    return enqueue_chunks(st, B, T, Q, q_dtype, Vtarget, v_dtype, gate, omega, lookahead, eta,
                          lambda_entropy, out, x, stream);
  // A call that repeats an earlier call's arguments replays a CUDA graph of
  // its whole chunk sequence (captured the second time the arguments are
  // seen); anything else is launched kernel by kernel.
  const StepKey key{B,   T,         q_dtype, v_dtype, Q,  Vtarget, gate, omega, lookahead,
                    out, eta, lambda_entropy, x};
  for (auto &g : st->graph_cache) {
    if (g.key == key) {
      g.last_use = ++st->graph_tick;
      const cudaError_t e = cudaGraphLaunch(g.exec, stream);
      return e == cudaSuccess ? FWPKM_OK : cuda_fail(e, "step: graph launch");
    }
  }
  bool seen = false;
  for (size_t i = 0; i < st->graph_seen.size(); ++i) {
    if (st->graph_seen[i] == key) {
      seen = true;
      st->graph_seen.erase(st->graph_seen.begin() + (long)i);
      break;
    }
  }
  if (!seen) {
    if (st->graph_seen.size() >= kGraphSeen) st->graph_seen.erase(st->graph_seen.begin());
    st->graph_seen.push_back(key);
    return enqueue_chunks(st, B, T, Q, q_dtype, Vtarget, v_dtype, gate, omega, lookahead, eta,
                          lambda_entropy, out, x, stream);
  }
  cudaGraphExec_t exec = capture_chunks(st, key);
  if (!exec)  // not capturable here: launch directly (reports any real error)
    return enqueue_chunks(st, B, T, Q, q_dtype, Vtarget, v_dtype, gate, omega, lookahead, eta,
                          lambda_entropy, out, x, stream);
  if (st->graph_cache.size() >= kGraphCache) {
    size_t lru = 0;
    for (size_t i = 1; i < st->graph_cache.size(); ++i)
      if (st->graph_cache[i].last_use < st->graph_cache[lru].last_use) lru = i;
    cudaGraphExecDestroy(st->graph_cache[lru].exec);
    st->graph_cache.erase(st->graph_cache.begin() + (long)lru);
  }
  st->graph_cache.push_back(StepGraph{key, exec, ++st->graph_tick});
  const cudaError_t e = cudaGraphLaunch(exec, stream);
  return e == cudaSuccess ? FWPKM_OK : cuda_fail(e, "step: graph launch");
}

fwpkm_status fwpkm_step(fwpkm_state *st, int B, int T, const void *Q, int q_dtype,
                        const void *Vtarget, int v_dtype, const float *gate, float eta,
                        float lambda_entropy, float *out, void *stream) {
  return fwpkm_step_ex(st, B, T, Q, q_dtype, Vtarget, v_dtype, gate, nullptr, 0, eta,
                       lambda_entropy, out, stream);
}

fwpkm_status fwpkm_step_host_ex(fwpkm_state *st, int B, int T, const void *Q_host, int q_dtype,
                                const void *Vt_host, int v_dtype, const float *gate_host,
                                const float *omega_host, int flags, float eta,
                                float lambda_entropy, float *out_host, void *stream_) {
  if (!st) return fail(FWPKM_EINVAL, "step_host: state is NULL");
  if (!Q_host || !Vt_host || !gate_host || !out_host)
    return fail(FWPKM_EINVAL, "step_host: NULL tensor pointer");
  if (!is_dtype(q_dtype) || !is_dtype(v_dtype))
    return fail(FWPKM_EINVAL, "step_host: dtype must be FWPKM_F32 or FWPKM_BF16");
  if (flags & ~FWPKM_LOOKAHEAD) return fail(FWPKM_EINVAL, "step_host: unknown flags 0x%x", flags);
  const int lookahead = (flags & FWPKM_LOOKAHEAD) ? 1 : 0;
  if (B < 1 || T < 1) return fail(FWPKM_ESHAPE, "step_host: B=%d and T=%d must be >= 1", B, T);
  if (!(eta >= 0.f) || !std::isfinite(eta))
    return fail(FWPKM_EINVAL, "step_host: eta must be finite and >= 0");
  if (!(lambda_entropy >= 0.f) || !std::isfinite(lambda_entropy))
    return fail(FWPKM_EINVAL, "step_host: lambda_entropy must be finite and >= 0");
  if (st->nmem > 1 && B != st->nmem)
    return fail(FWPKM_ESHAPE,
                "step_host: B=%d must equal the state's %d memories (one per sequence)", B,
                st->nmem);
  const int64_t tc_max = T < st->chunk ? T : st->chunk;
  const int64_t rows_max = (int64_t)B * (st->nmem > 1 ? (tc_max + 127) / 128 * 128 : tc_max);
  if (rows_max * st->H * st->k * 3 >= (int64_t)1 << 31 || (int64_t)B * T * st->dv >= (int64_t)1 << 40)
    return fail(FWPKM_ESHAPE, "step_host: B*chunk*heads*topk too large for 32-bit pair ids");
  if ((int64_t)B * T * 2 * st->H >= (int64_t)1 << 31)
    return fail(FWPKM_ESHAPE, "step_host: B*T*heads too large for 32-bit query-half indices");
  if ((rows_max + 127) / 128 > 65535)  // row tiles of the score grid (grid y)
    return fail(FWPKM_ESHAPE, "step_host: B*chunk = %lld rows exceeds 65535 tiles of 128 rows",
                (long long)rows_max);
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != st->device)
    return fail(FWPKM_EINVAL, "step_host: current device %d is not the state's device %d", dev,
                st->device);
  // per-token row bytes of each tensor; the staging copy has the caller's layout
  const size_t qrow = (size_t)st->H * st->dq * (q_dtype == FWPKM_BF16 ? 2 : 4);
  const size_t vrow = (size_t)st->dv * (v_dtype == FWPKM_BF16 ? 2 : 4);
  const size_t grow = 4, orow = (size_t)st->dv * 4;
  const size_t tok = (size_t)B * T;
  const size_t oq = 0, ov = align_up(tok * qrow, 256), og = ov + align_up(tok * vrow, 256),
               ow = og + align_up(tok * grow, 256),
               oo = ow + (omega_host ? align_up(tok * grow, 256) : 0),
               total = oo + align_up(tok * orow, 256);
  if (total > st->stage_bytes) {
    cudaDeviceSynchronize();
    cudaFree(st->stage);
    st->stage = nullptr;
    st->stage_bytes = 0;
    cudaError_t e = dev_malloc(&st->stage, total);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(FWPKM_ENOMEM, "step_host: staging allocation of %zu bytes failed", total);
    }
    st->stage_bytes = total;
  }
  for (cudaStream_t *cs : {&st->h2d_stream, &st->d2h_stream}) {
    if (!*cs && cudaStreamCreateWithFlags(cs, cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      *cs = nullptr;
      return fail(FWPKM_ECUDA, "step_host: copy stream creation failed");
    }
  }
  cudaStream_t stream = (cudaStream_t)stream_;
  fwpkm_status rc = prepare_step(st, rows_max, stream);
  if (rc != FWPKM_OK) return rc;

  // Copies pipelined with the chunk loop: chunk c's input rows (strided over
  // the B sequences) go in on one copy stream, its output rows come back on
  // the other as soon as its read has run; the compute stream waits for a
  // chunk's inputs only before the first kernel that reads them.
  char *base = (char *)st->stage;
  const int n_chunks = (T + st->chunk - 1) / st->chunk;
  std::vector<cudaEvent_t> in_ev(n_chunks), out_ev(n_chunks);
  for (auto &e : in_ev) e = take_event(st);
  for (auto &e : out_ev) e = take_event(st);
  cudaEvent_t start = take_event(st);
  cudaError_t e = cudaEventRecord(start, stream);  // after earlier work on the caller's stream
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st->h2d_stream, start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st->d2h_stream, start, 0);
  auto rows_of = [&](int c, int64_t *t0, int64_t *tc) {
    *t0 = (int64_t)c * st->chunk;
    *tc = T - *t0 < st->chunk ? T - *t0 : st->chunk;
  };
  for (int c = 0; c < n_chunks && e == cudaSuccess; ++c) {
    int64_t t0, tc;
    rows_of(c, &t0, &tc);
    e = cudaMemcpy2DAsync(base + oq + t0 * qrow, T * qrow, (const char *)Q_host + t0 * qrow,
                          T * qrow, tc * qrow, B, cudaMemcpyHostToDevice, st->h2d_stream);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(base + ov + t0 * vrow, T * vrow, (const char *)Vt_host + t0 * vrow,
                            T * vrow, tc * vrow, B, cudaMemcpyHostToDevice, st->h2d_stream);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(base + og + t0 * grow, T * grow, (const char *)gate_host + t0 * grow,
                            T * grow, tc * grow, B, cudaMemcpyHostToDevice, st->h2d_stream);
    if (e == cudaSuccess && omega_host)
      e = cudaMemcpy2DAsync(base + ow + t0 * grow, T * grow, (const char *)omega_host + t0 * grow,
                            T * grow, tc * grow, B, cudaMemcpyHostToDevice, st->h2d_stream);
    if (e == cudaSuccess) e = cudaEventRecord(in_ev[c], st->h2d_stream);
  }
  if (e != cudaSuccess) rc = cuda_fail(e, "step_host: host-to-device copy");
  if (rc == FWPKM_OK) {
    const Extras x = st->x;
    st->x = Extras{};  // armed extras apply to this step only
    ChunkHooks hooks;
    hooks.need_inputs = [&](int c) { return cudaStreamWaitEvent(stream, in_ev[c], 0); };
    hooks.read_done = [&](int c) {
      int64_t t0, tc;
      rows_of(c, &t0, &tc);
      cudaError_t r = cudaEventRecord(out_ev[c], stream);
      if (r == cudaSuccess) r = cudaStreamWaitEvent(st->d2h_stream, out_ev[c], 0);
      if (r == cudaSuccess)
        r = cudaMemcpy2DAsync((char *)out_host + t0 * orow, T * orow, base + oo + t0 * orow,
                              T * orow, tc * orow, B, cudaMemcpyDeviceToHost, st->d2h_stream);
      return r;
    };
    rc = enqueue_chunks(st, B, T, base + oq, q_dtype, base + ov, v_dtype,
                        (const float *)(base + og),
                        omega_host ? (const float *)(base + ow) : nullptr, lookahead, eta,
                        lambda_entropy, (float *)(base + oo), x, stream, &hooks);
  }
  // everything this call enqueued is done before it returns (and before its
  // events go back to the pool)
  const cudaError_t s1 = cudaStreamSynchronize(st->d2h_stream);
  const cudaError_t s2 = cudaStreamSynchronize(stream);
  const cudaError_t s3 = cudaStreamSynchronize(st->h2d_stream);
  for (auto ev : in_ev) st->event_pool.push_back(ev);
  for (auto ev : out_ev) st->event_pool.push_back(ev);
  st->event_pool.push_back(start);
  if (rc != FWPKM_OK) return rc;
  if (s1 != cudaSuccess || s2 != cudaSuccess || s3 != cudaSuccess)
    return cuda_fail(s1 != cudaSuccess ? s1 : (s2 != cudaSuccess ? s2 : s3),
                     "step_host: synchronise");
  return FWPKM_OK;
}

fwpkm_status fwpkm_step_host(fwpkm_state *st, int B, int T, const void *Q_host, int q_dtype,
                             const void *Vt_host, int v_dtype, const float *gate_host,
                             float eta, float lambda_entropy, float *out_host, void *stream) {
  return fwpkm_step_host_ex(st, B, T, Q_host, q_dtype, Vt_host, v_dtype, gate_host, nullptr, 0,
                            eta, lambda_entropy, out_host, stream);
}

fwpkm_status fwpkm_state_get(const fwpkm_state *st, float *subkeys, float *values, void *stream) {
  if (!st) return fail(FWPKM_EINVAL, "state_get: state is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (subkeys)
    e = cudaMemcpyAsync(subkeys, st->K,
                        sizeof(float) * (size_t)st->nmem * st->H * 2 * st->n * st->dh,
                        cudaMemcpyDefault, s);
  if (e == cudaSuccess && values)
    e = cudaMemcpyAsync(values, st->V, sizeof(float) * (size_t)st->nmem * st->N * st->dv,
                        cudaMemcpyDefault, s);
  if (e != cudaSuccess) return cuda_fail(e, "state_get");
  return FWPKM_OK;
}

fwpkm_status fwpkm_state_set(fwpkm_state *st, const float *subkeys, const float *values,
                             void *stream) {
  if (!st) return fail(FWPKM_EINVAL, "state_set: state is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (subkeys)
    e = cudaMemcpyAsync(st->K, subkeys,
                        sizeof(float) * (size_t)st->nmem * st->H * 2 * st->n * st->dh,
                        cudaMemcpyDefault, s);
  if (e == cudaSuccess && values)
    e = cudaMemcpyAsync(st->V, values, sizeof(float) * (size_t)st->nmem * st->N * st->dv,
                        cudaMemcpyDefault, s);
  if (e != cudaSuccess) return cuda_fail(e, "state_set");
  if (subkeys && st->arena) {  // new sub-keys: their split, stream-ordered after the copy
    const fwpkm_status rc = split_all_subkeys(st, s);
    if (rc != FWPKM_OK) return rc;
    st->subkey_split_stale = false;
  }
  return FWPKM_OK;
}

fwpkm_status fwpkm_record_selection(fwpkm_state *st, int32_t *slots, float *weights) {
  if (!st) return fail(FWPKM_EINVAL, "record_selection: state is NULL");
  if ((slots == nullptr) != (weights == nullptr))
    return fail(FWPKM_EINVAL, "record_selection: give both buffers or neither");
  st->x.rec_slots = slots;
  st->x.rec_w = weights;
  return FWPKM_OK;
}

fwpkm_status fwpkm_force_selection(fwpkm_state *st, const int32_t *slots, const uint8_t *mask) {
  if (!st) return fail(FWPKM_EINVAL, "force_selection: state is NULL");
  if ((slots == nullptr) != (mask == nullptr))
    return fail(FWPKM_EINVAL, "force_selection: give both buffers or neither");
  st->x.force_slots = slots;
  st->x.force_mask = mask;
  return FWPKM_OK;
}

fwpkm_status fwpkm_set_profiling(fwpkm_state *st, int enable) {
  if (!st) return fail(FWPKM_EINVAL, "set_profiling: state is NULL");
  st->profiling = enable != 0;
  return FWPKM_OK;
}

fwpkm_status fwpkm_profile_read(fwpkm_state *st, const char **names, double *ms,
                                int64_t *launches, int max_kinds, int *count, void *stream) {
  if (!st) return fail(FWPKM_EINVAL, "profile_read: state is NULL");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "profile_read: synchronise");
  for (auto &t : st->timings) {
    float dt = 0.f;
    if (cudaEventElapsedTime(&dt, t.a, t.b) == cudaSuccess) {
      st->prof_ms[t.kind] += dt;
      st->prof_n[t.kind] += kKernelsPerCall[t.kind];
    }
    st->event_pool.push_back(t.a);
    st->event_pool.push_back(t.b);
  }
  st->timings.clear();
  int c = 0;
  for (int i = 0; i < K_COUNT && c < max_kinds; ++i, ++c) {
    if (names) names[c] = kKindNames[i];
    if (ms) ms[c] = st->prof_ms[i];
    if (launches) launches[c] = st->prof_n[i];
    st->prof_ms[i] = 0.0;
    st->prof_n[i] = 0;
  }
  if (count) *count = c;
  return FWPKM_OK;
}

fwpkm_status fwpkm_read_stats(fwpkm_state *st, int64_t *chunks, int64_t *value_rows,
                              int64_t *key_rows, int64_t *records, uint32_t *device_errors,
                              int reset, void *stream) {
  if (!st) return fail(FWPKM_EINVAL, "read_stats: state is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  Meta m{};
  cudaError_t e = cudaMemcpyAsync(&m, st->s.meta, sizeof(Meta), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "read_stats");
  if (chunks) *chunks = (int64_t)m.stat_chunks;
  if (value_rows) *value_rows = (int64_t)m.stat_value_rows;
  if (key_rows) *key_rows = (int64_t)m.stat_key_rows;
  if (records) *records = (int64_t)m.stat_records;
  if (device_errors) *device_errors = m.err;
  if (reset) {
    Meta z{};
    e = cudaMemcpyAsync(st->s.meta, &z, sizeof(Meta), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "read_stats: reset");
  }
  if (m.err)
    return fail(FWPKM_ECUDA,
                "device error bits 0x%x (1 = the read's row-copy wait gave up, 2 = the "
                "apply's partial pool overflowed, 4 = a bucket-scan wait gave up, 8 = the "
                "score's TMA/MMA wait gave up, 16 = reserved; the write kernels of that "
                "chunk and later ones were skipped)",
                m.err);
  return FWPKM_OK;
}

}  // extern "C"
