// fwpkm_noalloc.cu -- product-key selection that allocates no device memory.
//
// fwpkm_select_noalloc runs the selection half of the read (query halves ->
// sub-key distances on the tensor cores -> top-k per half -> k*k merge ->
// softmax) against a
// state's current sub-key tables and writes the chosen slots and weights.  It
// never calls cudaMalloc or cudaFree: its scratch (query halves, norms and the
// distance matrix) lives in one file-scope device array, g_noalloc_scratch,
// that is part of the library image.  That serves callers that cannot
// allocate at call time: a serving process that plans every device byte up
// front and runs with a fixed budget, or a plugin inside a host framework
// whose allocator owns the device; cudaMalloc can also synchronise the whole
// device, which a latency-bound caller cannot afford.
//
// The array is shared by every call in the process: concurrent calls that
// overlap on the GPU (different streams or threads) race on it, so callers
// must order them.  Nothing in it needs to start at zero: each call writes
// every scratch element it later reads.  The array stays resident on every
// GPU that loads the library until the process exits.
//
// The score kernel's waits are bounded; one that gives up sets a bit in a
// second static block, g_noalloc_meta, which every call zeroes on its stream
// before its kernels and copies out to the caller's error word after them.
#include <cstdio>
#include <mutex>

#include "../../include/fwpkm.h"
#include "fwpkm_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB per device

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
// Error bits and counters the kernels write (only `err` is used here).
__device__ __align__(256) fwpkm::Meta g_noalloc_meta;

// The arrays' device addresses, looked up once per device with that device
// current (host code cannot use the symbols themselves as device pointers).
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};
fwpkm::Meta *g_meta_ptr[kMaxDevices] = {};

cudaError_t scratch_on(int dev, void **out, fwpkm::Meta **meta) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr, *m = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(&m, g_noalloc_meta);
    if (e != cudaSuccess) return e;
    g_meta_ptr[dev] = static_cast<fwpkm::Meta *>(m);
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  *meta = g_meta_ptr[dev];
  return cudaSuccess;
}

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

fwpkm_status fail(fwpkm_status st, const char *msg) {
  fwpkm::set_last_error(msg);
  return st;
}

}  // namespace

extern "C" fwpkm_status fwpkm_select_noalloc(fwpkm_state *state, int B, int T, const void *Q,
                                             int q_dtype, int32_t *slots, float *weights,
                                             uint32_t *device_errors, void *stream_) {
  using namespace fwpkm;
  StateView v;
  if (!state_view(state, &v)) return fail(FWPKM_EINVAL, "select_noalloc: state is NULL");
  if (!Q || !slots || !weights) return fail(FWPKM_EINVAL, "select_noalloc: NULL pointer");
  if (q_dtype != FWPKM_F32 && q_dtype != FWPKM_BF16)
    return fail(FWPKM_EINVAL, "select_noalloc: q_dtype must be FWPKM_F32 or FWPKM_BF16");
  if (B < 1 || T < 1) return fail(FWPKM_ESHAPE, "select_noalloc: B and T must be >= 1");
  if (((uintptr_t)Q) & 15) return fail(FWPKM_EINVAL, "select_noalloc: Q must be 16-byte aligned");
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != v.device)
    return fail(FWPKM_EINVAL, "select_noalloc: current device is not the state's device");
  if (v.nmem > 1)
    return fail(FWPKM_EUNSUPPORTED, "select_noalloc: states with one memory per sequence are "
                "not supported");

  // Scratch of one pass of `rows` token rows (fp32, each piece 256-byte
  // aligned; rows rounded up to 128): Qs_hi, Qs_lo [2H][rows][dh], qn
  // [2H][rows], D [2H][rows][n]; fixed: K_hi, K_lo [2H*n + 128][dh], kn
  // [2H][n][kKnChunks].
  const size_t H2 = 2 * (size_t)v.H;
  const size_t fixed = 2 * up256((H2 * v.n + 128) * v.dh * 4) + up256(H2 * v.n * kKnChunks * 4) +
                       4 * 256 + 128 * (2 * H2 * v.dh + H2 + H2 * v.n) * 4;
  const size_t per_row = (2 * H2 * v.dh + H2 + H2 * v.n) * 4;
  if (fixed + per_row > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "select_noalloc: the state's sub-key tables (heads=%d, n=%d, dq=%d) need %zu "
             "bytes of scratch with one token, more than the %zu-byte static scratch; no "
             "batch size fits",
             v.H, v.n, v.dq, fixed + per_row, kNoAllocScratchBytes);
    return fail(FWPKM_ESHAPE, msg);
  }
  if (fixed + per_row * (size_t)B > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "select_noalloc: one time step of B=%d sequences needs %zu bytes of scratch, "
             "more than the %zu-byte static scratch; call it with a smaller B (or a "
             "smaller memory)",
             B, fixed + per_row * (size_t)B, kNoAllocScratchBytes);
    return fail(FWPKM_ESHAPE, msg);
  }
  const int steps_per_pass = (int)((kNoAllocScratchBytes - fixed) / (per_row * (size_t)B));
  const int Tc = steps_per_pass < T ? steps_per_pass : T;
  const int rows_max = (B * Tc + 127) / 128 * 128;  // whole 128-row score tiles

  void *base = nullptr;
  Meta *meta = nullptr;
  const cudaError_t e = scratch_on(dev, &base, &meta);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof msg, "select_noalloc: cudaGetSymbolAddress failed: %s",
             cudaGetErrorString(e));
    return fail(FWPKM_ECUDA, msg);
  }
  char *p = static_cast<char *>(base);
  Scratch s{};
  s.Qs_hi = reinterpret_cast<float *>(p);
  p += up256(H2 * rows_max * v.dh * 4);
  s.Qs_lo = reinterpret_cast<float *>(p);
  p += up256(H2 * rows_max * v.dh * 4);
  s.qn = reinterpret_cast<float *>(p);
  p += up256(H2 * rows_max * 4);
  s.K_hi = reinterpret_cast<float *>(p);
  p += up256((H2 * v.n + 128) * v.dh * 4);
  s.K_lo = reinterpret_cast<float *>(p);
  p += up256((H2 * v.n + 128) * v.dh * 4);
  s.kn = reinterpret_cast<float *>(p);
  p += up256(H2 * v.n * kKnChunks * 4);
  s.D = reinterpret_cast<float *>(p);
  s.meta = meta;
  TcMaps maps;  // host-side descriptors of the operands above (no allocation)
  const cudaError_t me = encode_score_maps(&maps, s, v.H, 1, rows_max, v.n, v.dh);
  if (me != cudaSuccess) return fail(FWPKM_ECUDA, "select_noalloc: tensor map encoding failed");

  Extras x{};
  x.rec_slots = slots;
  x.rec_w = weights;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  // this call's error bits start at zero (a memset allocates nothing)
  cudaError_t ze = cudaMemsetAsync(&meta->err, 0, sizeof(meta->err), stream);
  if (ze != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof msg, "select_noalloc: clearing the error word failed: %s",
             cudaGetErrorString(ze));
    return fail(FWPKM_ECUDA, msg);
  }
  for (int t0 = 0; t0 < T; t0 += Tc) {
    Dims d{};
    d.n = v.n;
    d.dq = v.dq;
    d.dh = v.dh;
    d.dv = v.dv;
    d.k = v.k;
    d.H = v.H;
    d.N = v.N;
    d.B = B;
    d.T = T;
    d.t0 = t0;
    d.Tc = T - t0 < Tc ? T - t0 : Tc;
    d.rows = B * d.Tc;
    d.qstride = rows_max;
    d.M = d.rows * v.H;
    d.nmem = 1;
    d.Nt = v.N;
    d.rstride = d.Tc;
    d.drows = d.rows;
    d.Mmem = d.M;
    d.sm_count = v.sm_count;
    d.pdl = 1;
    d.eps = v.eps;
    d.score_dot = v.score_dot;
    d.mbar_polls = v.mbar_polls;
    d.scan_polls = kDefaultScanPolls;
    d.q_tf32_exact = q_dtype == FWPKM_BF16 ? 1 : 0;
    // the sub-key split once per call, the query halves once per pass
    cudaError_t ke = t0 == 0 ? launch_prep(d, Q, q_dtype, v.K, s, stream)
                             : launch_prep_q(d, Q, q_dtype, s, stream);
    if (ke == cudaSuccess) ke = launch_score(d, s, maps, stream);
    if (ke == cudaSuccess) ke = launch_topk_select(d, s, x, stream);
    if (ke != cudaSuccess) {
      char msg[256];
      snprintf(msg, sizeof msg, "select_noalloc: launch failed: %s", cudaGetErrorString(ke));
      return fail(FWPKM_ECUDA, msg);
    }
  }
  if (device_errors) {
    const cudaError_t ce = cudaMemcpyAsync(device_errors, &meta->err, sizeof(uint32_t),
                                           cudaMemcpyDefault, stream);
    if (ce != cudaSuccess) {
      char msg[256];
      snprintf(msg, sizeof msg, "select_noalloc: copying the error word failed: %s",
               cudaGetErrorString(ce));
      return fail(FWPKM_ECUDA, msg);
    }
  }
  return FWPKM_OK;
}
