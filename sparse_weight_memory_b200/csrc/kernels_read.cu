// kernels_read.cu -- gather, gated readout, residual and dL/dw per pair.
//
// Readout (gist.science "Fast-weight Product Key Memory", section 2: the
// retrieved value; gate g_t; agifrontier tutorial, gating): per token
//   yhat_t = (1/H) sum_h sum_r w_{t,h,r} V[slot_{t,h,r}]
//   out_t  = g_t * yhat_t
// and, for the write that follows (MSE memorisation loss weighted by the
// token's importance, sciencestack table of contents sections 8-12):
//   e_t          = yhat_t - v_t
//   dL/dw_{t,h,r} = (2 w_t / H) e_t . V[slot_{t,h,r}]   (pre-update rows)
// The token weight w_t is the caller's omega_t, or the gate g_t when no
// omega is given.  With the lookahead pairing (gist.science section 2,
// lookahead targets) token t is written towards v_{t+1}: the target row is
// the next token's, and the last token of the call, which has no target, is
// read with weight 0.
// and, when the entropy term is off (so dL/dw is complete here), the softmax
// Jacobian dL/ds_r = w_r (dL/dw_r - sum_r' w_r' dL/dw_r') and, per sub-key
// entry, alpha = (sum of dL/ds over its pairs) / (eps + d).
//
// One CTA per token, one float4 column of the value rows per thread (32, 64
// or 128 threads, as the row is wide).  Each thread sums its column over the
// token's H*k rows straight from global memory, every row load independent
// of the others, so the rows of many tokens are in flight per
// multiprocessor; the dot products then read the rows again, from L1 or L2.
// The token's member records, which go to the bucket scan's offsets, are
// written last: only they wait for the scan, so the rest of the read runs
// while the scan does.
// Only a token whose rows exceed 1 MB is split over a thread-block cluster
// of G CTAs, which exchange their partial sums through distributed shared
// memory and add them in rank order (the same yhat everywhere).  (Staging
// the rows in shared memory by bulk copies, with clusters of about 32 KB of
// rows per CTA, was measured slower: it limits the CTAs resident per
// multiprocessor and adds barriers to each token's chain.)
#include "fwpkm_internal.cuh"

namespace fwpkm {

constexpr size_t kReadCtaRows = 1024 * 1024;  // value-row bytes per CTA before a cluster splits
constexpr int kReadMaxCluster = 8;            // portable cluster size

struct ReadPlan {
  int G;        // CTAs per token (cluster size, a power of two <= 8)
  int per;      // pairs per CTA, ceil(H*k / G)
  int threads;  // 32, 64 or 128: about one float4 column per thread
  size_t smem;  // dynamic shared memory per CTA
};

// Dynamic shared memory layout (floats / ints):
//   ypart, e                dv each (ypart is read by the whole cluster)
//   w, slot, a, dl, claim   H*k each (a is read by the whole cluster)
//   esub, eclaim, emask, einv   2*H*k each (this CTA's entries only)
static size_t read_smem_bytes(const Dims &d) {
  const size_t HK = (size_t)d.H * d.k;
  return 2 * (size_t)d.dv * 4 + HK * 20 + 2 * HK * 16;
}

static ReadPlan read_plan(const Dims &d) {
  const int HK = d.H * d.k;
  const size_t row_bytes = (size_t)d.dv * 4;
  ReadPlan p;
  p.G = 1;
  while (p.G < kReadMaxCluster && p.G < HK &&
         (size_t)((HK + p.G - 1) / p.G) * row_bytes > kReadCtaRows)
    p.G <<= 1;
  p.per = (HK + p.G - 1) / p.G;
  const int dv4 = d.dv / 4;
  p.threads = dv4 <= 32 ? 32 : (dv4 <= 64 ? 64 : 128);
  p.smem = read_smem_bytes(d);
  return p;
}

// --- cluster helpers -------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of every CTA of the cluster; orders shared-memory writes before
// the barrier with the other CTAs' reads after it.  The release waits for
// every earlier write of the CTA, global stores included, so the kernel keeps
// its global stores after the last such barrier.
__device__ __forceinline__ void cluster_barrier() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}
// The same meeting point without ordering: only keeps every CTA's shared
// memory alive until the others are done reading it (their loads have been
// consumed before they arrive).
__device__ __forceinline__ void cluster_barrier_relaxed() {
  asm volatile(
      "barrier.cluster.arrive.relaxed.aligned;\n\t"
      "barrier.cluster.wait.aligned;" ::
          : "memory");
}
// Address of `p` (this CTA's shared memory) in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_smem(const void *p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ float4 ld_peer4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ float ld_peer(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// kVt: float4 columns per thread, ceil(dv / 4 / kThreads) (1, 2 or 4), so
// that the registers holding the target, yhat and e rows are only those the
// row width needs: at dv = 512 the CTAs of a 1024-token chunk then fit the
// multiprocessors in one wave.
template <typename TV, int kThreads, int kVt>
__global__ void __launch_bounds__(kThreads, kThreads == 128 ? 7 : 1) k_read(Dims d, const float *__restrict__ V,
                                                       const TV *__restrict__ Vt,
                                                       const float *__restrict__ gate,
                                                       const float *__restrict__ omega,
                                                       float *__restrict__ out, Scratch s, int G,
                                                       int per) {
  // After the bucket scan (the grid this one follows in the write path) the
  // read waits only before its member records, which go to the scan's bucket
  // offsets.  Everything else it reads was written by the selection and
  // earlier kernels: the selection's grid completed before any scan CTA got
  // past its own wait, and this grid is launched only after every scan CTA
  // has.  At eta = 0 the selection itself comes just before: wait at once.
  if (d.readonly) griddep_wait();
  griddep_launch();
  // An earlier kernel gave up (its bits are stable here, so every CTA of a
  // cluster takes the same branch): nothing of this chunk is read or written.
  if (chunk_aborted(s, ERR_READ_TIMEOUT)) return;
  extern __shared__ __align__(128) unsigned char smem[];
  const int HK = d.H * d.k, dv = d.dv, dv4 = dv >> 2;
  float *ypart = reinterpret_cast<float *>(smem);
  float *e_s = ypart + dv;
  float *w_s = e_s + dv;
  int *slot_s = reinterpret_cast<int *>(w_s + HK);
  float *a_s = reinterpret_cast<float *>(slot_s + HK);
  float *dl_s = a_s + HK;
  int *claim_s = reinterpret_cast<int *>(dl_s + HK);
  int *esub_s = claim_s + HK;
  int *eclaim_s = esub_s + 2 * HK;
  unsigned *emask_s = reinterpret_cast<unsigned *>(eclaim_s + 2 * HK);
  float *einv_s = reinterpret_cast<float *>(emask_s + 2 * HK);

  const int rank = G > 1 ? (int)cluster_rank() : 0;
  const int row = blockIdx.x / G;
  const int j0 = min(HK, rank * per), j1 = min(HK, j0 + per);  // this CTA's pairs
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int b = row / d.Tc, tl = row % d.Tc;
  const int64_t tok = (int64_t)b * d.T + d.t0 + tl;
  const int64_t p0 = (int64_t)row * HK;
  // target row of the token, and whether it has one (lookahead: the next token's)
  const bool last = d.lookahead && d.t0 + tl == d.T - 1;
  const int64_t ttok = d.lookahead && !last ? tok + 1 : tok;

  // Everything that does not depend on the rows is loaded at once: the
  // token's pairs, this CTA's entries (x = rank mod G), the gate and the
  // target row.
  for (int j = tid; j < HK; j += blockDim.x) {
    w_s[j] = s.pw[p0 + j];
    slot_s[j] = s.pslot[p0 + j];
    claim_s[j] = s.pclaim[p0 + j];
  }
  const int64_t e0 = (int64_t)row * 2 * HK;  // entries of this row: e0 + (h*2 + half)*k + idx
  // d.readonly (eta = 0): the read alone -- no records, residual, dL/dw or
  // alphas (the selection wrote no claims or entries either)
  for (int x = rank + G * tid; x < (d.readonly ? 0 : 2 * HK); x += G * blockDim.x) {
    esub_s[x] = s.esub[e0 + x];
    eclaim_s[x] = s.eclaim[e0 + x];
    emask_s[x] = s.emask[e0 + x];
    einv_s[x] = s.einv[e0 + x];
  }
  __syncthreads();
  const float g = gate[tok];
  const float om = last ? 0.f : (omega ? omega[tok] : g);  // the token's MSE weight
  const float invH = d.heads_sum ? 1.f : 1.f / (float)d.H;  // head readouts averaged or summed
  // the token's target row, loaded now so that it is here when e is formed
  float4 vt[kVt];
#pragma unroll
  for (int q = 0; q < kVt; ++q) {
    const int c4 = tid + q * kThreads;
    vt[q] = c4 < dv4 && !d.readonly ? load4(Vt, ttok * dv + 4 * c4)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // pass 1: partial weighted sum of this CTA's rows, one column per thread.
  // Eight rows are loaded before any is added, so that their loads are in
  // flight together; the sum still runs in row order.
  for (int c4 = tid; c4 < dv4; c4 += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float *col = V + 4 * c4;
    int j = j0;
    for (; j + 8 <= j1; j += 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = *reinterpret_cast<const float4 *>(col + (int64_t)slot_s[j + u] * dv);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float w = w_s[j + u];
        acc.x = fmaf(w, v[u].x, acc.x);
        acc.y = fmaf(w, v[u].y, acc.y);
        acc.z = fmaf(w, v[u].z, acc.z);
        acc.w = fmaf(w, v[u].w, acc.w);
      }
    }
    for (; j < j1; ++j) {
      const float w = w_s[j];
      const float4 v = *reinterpret_cast<const float4 *>(col + (int64_t)slot_s[j] * dv);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    *reinterpret_cast<float4 *>(ypart + 4 * c4) = acc;
  }
  if (G > 1) cluster_barrier();
  else __syncthreads();

  // yhat = (partials added in rank order) / H, identical in every CTA; kept
  // in registers (y, e) until the global stores at the end
  float4 y[kVt], e[kVt];
#pragma unroll
  for (int q = 0; q < kVt; ++q) {
    const int c4 = tid + q * kThreads;
    y[q] = e[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c4 >= dv4) continue;
    float4 yy = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < G; ++r) {
      const float4 v = G > 1 ? ld_peer4(peer_smem(ypart + 4 * c4, (uint32_t)r))
                             : *reinterpret_cast<const float4 *>(ypart + 4 * c4);
      yy.x += v.x;
      yy.y += v.y;
      yy.z += v.z;
      yy.w += v.w;
    }
    y[q] = make_float4(yy.x * invH, yy.y * invH, yy.z * invH, yy.w * invH);
    const float4 t = vt[q];
    e[q] = make_float4(y[q].x - t.x, y[q].y - t.y, y[q].z - t.z, y[q].w - t.w);
    *reinterpret_cast<float4 *>(e_s + 4 * c4) = e[q];
  }
  __syncthreads();

  // dL/dw of this CTA's pairs: warp `wid` takes pairs j0 + wid, j0 + wid + warps, ...,
  // two at a time so that both rows' loads are in flight together
  const float coef = 2.f * om * invH;
  constexpr int kWarps = kThreads / 32;
  const int jend = d.readonly ? j0 : j1;
  for (int j = j0 + wid; j < jend; j += 2 * kWarps) {
    const int j2 = j + kWarps;
    const bool two = j2 < jend;
    const float *vr = V + (int64_t)slot_s[j] * dv;
    const float *vr2 = two ? V + (int64_t)slot_s[j2] * dv : vr;
    float acc = 0.f, acc2 = 0.f;
    for (int c4 = lane; c4 < dv4; c4 += 32) {
      const float4 v = *reinterpret_cast<const float4 *>(vr + 4 * c4);
      const float4 v2 = *reinterpret_cast<const float4 *>(vr2 + 4 * c4);
      const float4 e = *reinterpret_cast<const float4 *>(e_s + 4 * c4);
      acc = fmaf(e.x, v.x, acc);
      acc = fmaf(e.y, v.y, acc);
      acc = fmaf(e.z, v.z, acc);
      acc = fmaf(e.w, v.w, acc);
      acc2 = fmaf(e.x, v2.x, acc2);
      acc2 = fmaf(e.y, v2.y, acc2);
      acc2 = fmaf(e.z, v2.z, acc2);
      acc2 = fmaf(e.w, v2.w, acc2);
    }
    acc = warp_sum(acc);
    acc2 = warp_sum(acc2);
    if (lane == 0) {
      a_s[j] = coef * acc;
      if (two) a_s[j2] = coef * acc2;
    }
  }
  // Every CTA is done reading the partials; with the entropy term off the
  // a values are published to the cluster for the alphas.
  if (G > 1) {
    if (d.lam == 0.f) cluster_barrier();
    else cluster_barrier_relaxed();
  }
  __syncthreads();  // this CTA's a values, for its own stores below
  // global stores: out and the residual (rank 0), dL/dw of this CTA's pairs
  if (rank == 0) {
#pragma unroll
    for (int q = 0; q < kVt; ++q) {
      const int c4 = tid + q * kThreads;
      if (c4 >= dv4) continue;
      *reinterpret_cast<float4 *>(out + tok * dv + 4 * c4) =
          make_float4(g * y[q].x, g * y[q].y, g * y[q].z, g * y[q].w);
      if (!d.readonly) *reinterpret_cast<float4 *>(s.E + (int64_t)row * dv + 4 * c4) = e[q];
    }
  }
  for (int j = j0 + tid; j < (d.readonly ? j0 : j1); j += blockDim.x) s.pa[p0 + j] = a_s[j];

  // dL/ds and alpha per entry when the entropy term is off (dL/dw complete)
  if (d.lam == 0.f && !d.readonly) {
    for (int h = wid; h < d.H; h += kThreads / 32) {
      const int j = h * d.k + lane;
      float w = 0.f, a = 0.f;
      if (lane < d.k) {
        w = w_s[j];
        a = G > 1 ? ld_peer(peer_smem(a_s + j, (uint32_t)(j / per))) : a_s[j];
      }
      const float S = warp_sum(w * a);
      if (lane < d.k) dl_s[j] = w * (a - S);
    }
    __syncthreads();
    // alpha of the entries x = rank (mod G) of this row, one thread each
    for (int x = rank + G * tid; x < 2 * HK; x += G * blockDim.x) {
      if (esub_s[x] >= 0) {
        unsigned mask = emask_s[x];
        const float *dl = dl_s + (x / d.k >> 1) * d.k;  // head h = (h*2 + half) >> 1
        float sum = 0.f;
        while (mask) {
          sum += dl[__ffs(mask) - 1];
          mask &= mask - 1;
        }
        einv_s[x] *= sum;  // alpha, which goes into the entry's record below
      }
    }
    // no CTA leaves while another may still read its a values
    if (G > 1) cluster_barrier_relaxed();
  }
  if (d.readonly) return;  // no write follows: no records
  griddep_wait();
  // the scan gave up: its offsets may be wrong, so no record is written (the
  // bits are stable after the wait: every CTA of a cluster takes this branch)
  if (chunk_aborted(s, ERR_READ_TIMEOUT)) return;
  // Member records go to their buckets last, at the scan's offsets: this
  // CTA's pairs -> value bucket slot >> vshift; entries x = rank (mod G) ->
  // sub-key row bucket NBv + (h*2+half)*n + row.  An entry carries its alpha
  // when the entropy term is off; with it on, the apply reads the alpha
  // pgrad computes.
  for (int j = j0 + tid; j < j1; j += blockDim.x) {
    const int64_t p = p0 + j;
    const float w = w_s[j];
    Member m;
    m.g = (uint32_t)slot_s[j];
    m.id = (uint32_t)p;
    m.srow = row;
    m.gstart = 0;
    m.coef = 2.f * om * w * invH;
    m.c0 = d.agg == AGG_COUNT ? 1.f : w * invH;  // the group's sum is the row's divisor
    m.c1 = w;
    m.glen = 0;
    s.rec_in[s.boff[slot_s[j] >> d.vshift] + claim_s[j]] = m;
  }
  const int tab0 = mem_of(d, row) * 2 * d.H;  // the token's memory's first sub-key table
  for (int x = rank + G * tid; x < 2 * HK; x += G * blockDim.x) {
    const int mh = x / d.k;  // entry (h*2 + half)*k + idx of this row
    const int sub = esub_s[x];
    if (sub >= 0) {
      const int64_t e = e0 + x;
      Member m;
      m.g = (uint32_t)d.Nt + (uint32_t)((tab0 + mh) * d.n + sub);
      m.id = (uint32_t)e;
      m.srow = (int)(tok * 2 * d.H + mh);  // this query half in the caller's Q
      m.gstart = 0;
      m.coef = m.c0 = d.lam == 0.f ? einv_s[x] : 0.f;
      m.c1 = 0.f;
      m.glen = 0;
      s.rec_in[s.boff[d.NBv + (tab0 + mh) * d.n + sub] + eclaim_s[x]] = m;
    }
  }
}

template <typename TV, int kThreads, int kVt>
static cudaError_t launch_read_tn(const Dims &d, const float *V, const TV *Vt, const float *gate,
                                  const float *omega, float *out, const Scratch &s,
                                  const ReadPlan &p, cudaStream_t st) {
  auto kernel = k_read<TV, kThreads, kVt>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e != cudaSuccess) return e;
  return launch_kc(d.pdl, p.G, kernel, d.rows * p.G, kThreads, p.smem, st, d, V, Vt, gate,
                   omega, out, s, p.G, p.per);
}

template <typename TV>
static cudaError_t launch_read_t(const Dims &d, const float *V, const TV *Vt, const float *gate,
                                 const float *omega, float *out, const Scratch &s,
                                 cudaStream_t st) {
  const ReadPlan p = read_plan(d);
  if (p.threads == 32) return launch_read_tn<TV, 32, 1>(d, V, Vt, gate, omega, out, s, p, st);
  if (p.threads == 64) return launch_read_tn<TV, 64, 1>(d, V, Vt, gate, omega, out, s, p, st);
  const int dv4 = d.dv / 4;  // at most 4 * 128 (dv <= 2048)
  if (dv4 <= 128) return launch_read_tn<TV, 128, 1>(d, V, Vt, gate, omega, out, s, p, st);
  if (dv4 <= 256) return launch_read_tn<TV, 128, 2>(d, V, Vt, gate, omega, out, s, p, st);
  return launch_read_tn<TV, 128, 4>(d, V, Vt, gate, omega, out, s, p, st);
}

cudaError_t launch_read(const Dims &d, const float *V, const void *Vt, int v_dtype,
                        const float *gate, const float *omega, float *out, const Scratch &s,
                        cudaStream_t st) {
  if (v_dtype == 1)
    return launch_read_t(d, V, (const __nv_bfloat16 *)Vt, gate, omega, out, s, st);
  return launch_read_t(d, V, (const float *)Vt, gate, omega, out, s, st);
}

int read_cluster_size(const Dims &d) { return read_plan(d).G; }

}  // namespace fwpkm
