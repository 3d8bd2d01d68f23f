// kernels_group.cu -- grouping of the chunk's writes and the in-place update.
//
// Update rule (agifrontier tutorial: theta' = theta - eta * grad L_MSE;
// gist.science section 2: keys and values are fast weights, gradients of a
// slot written several times in a chunk are averaged; sciencestack table of
// contents: loss reduced by summation, gradient weighted by row contribution,
// MSE weighted by token importance, no clipping, marginal entropy loss):
//   value row i : V_i -= eta * G_i / C_i,
//                 G_i = sum over its pairs of (2 g_t / H) w e_t,
//                 C_i = sum over its pairs of w / H
//   sub-key row : K -= eta * 2 * (sum_e alpha_e q_e - (sum_e alpha_e) K)
//                 alpha_e = (1/(eps + d)) * sum of dL/ds over the entry's pairs
//   marginal    : pbar_i = (1/M) sum over its pairs of w;
//                 dL_addr/dw = (lam/M) (log pbar_i + 1)
//
// Members: pairs p = m*k + r (value rows) and entries e = (m*2+half)*k + idx
// (sub-key rows), each carried by a 32-byte Member record.  Buckets: value
// bucket slot >> vshift (a range of at most 2^vshift consecutive slots, <= 8192
// buckets), then one bucket per sub-key row, NBv + (h*2+half)*n + row.  The
// selection kernel counted members per bucket and claimed a position; `scan`
// turns counts into bucket offsets; the read kernel writes each record at
// offset + claim (rec_in); `bsort` sorts every bucket by (group, id) into rec,
// so the records are globally ordered by group and, inside a group, by id;
// `apply` sums every group's members in that order and writes the row.  No
// floating-point atomics: the result does not depend on scheduling, whatever
// the skew of slot usage.
#include <math_constants.h>

#include "fwpkm_internal.cuh"

namespace fwpkm {

__device__ __forceinline__ Member load_member(const Member *p) {
  const int4 a = *reinterpret_cast<const int4 *>(p);
  const int4 b = *(reinterpret_cast<const int4 *>(p) + 1);
  Member m;
  m.g = (uint32_t)a.x;
  m.id = (uint32_t)a.y;
  m.srow = a.z;
  m.gstart = a.w;
  m.coef = __int_as_float(b.x);
  m.c0 = __int_as_float(b.y);
  m.c1 = __int_as_float(b.z);
  m.glen = b.w;
  return m;
}
__device__ __forceinline__ void store_member(Member *p, const Member &m) {
  *reinterpret_cast<int4 *>(p) = make_int4((int)m.g, (int)m.id, m.srow, m.gstart);
  *(reinterpret_cast<int4 *>(p) + 1) =
      make_int4(__float_as_int(m.coef), __float_as_int(m.c0), __float_as_int(m.c1), m.glen);
}

// ---------------------------------------------------------------------------
// scan: bucket offsets (single CTA).  Each thread owns a contiguous run of
// buckets; its counts are loaded before the block-wide scan.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 1024;
constexpr int kScanRun = 16;  // counts held in registers per thread and pass

__global__ void __launch_bounds__(kScanThreads) k_bucket_scan(Dims d, Scratch s) {
  __shared__ int red[32];
  const int NB = d.NB;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int per = (NB + kScanThreads - 1) / kScanThreads;  // buckets per thread
  const int b0 = min(threadIdx.x * per, NB), b1 = min(b0 + per, NB);
  int total = 0;
  for (int b = b0; b < b1; b += kScanRun) {
    int v[kScanRun];
#pragma unroll
    for (int i = 0; i < kScanRun; ++i) v[i] = b + i < b1 ? s.bcnt[b + i] : 0;
#pragma unroll
    for (int i = 0; i < kScanRun; ++i) total += v[i];
  }
  // exclusive scan of the per-thread totals
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) red[w] = incl;
  __syncthreads();
  if (w == 0) {
    int x = red[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(FULL, x, o);
      if (lane >= o) x += t;
    }
    red[lane] = x;
  }
  __syncthreads();
  int run = (w > 0 ? red[w - 1] : 0) + incl - total;
  for (int b = b0; b < b1; b += kScanRun) {
    int v[kScanRun];
#pragma unroll
    for (int i = 0; i < kScanRun; ++i) v[i] = b + i < b1 ? s.bcnt[b + i] : 0;
#pragma unroll
    for (int i = 0; i < kScanRun; ++i) {
      if (b + i < b1) {
        s.boff[b + i] = run;
        if (b + i == d.NBv) s.meta->Lv = run;  // value buckets come first
        s.bcnt[b + i] = 0;                       // ready for the next chunk
        run += v[i];
      }
    }
  }
  if (threadIdx.x == kScanThreads - 1) {
    const int L = red[31];
    s.boff[NB] = L;
    s.meta->L = L;
    if (d.NBv == NB) s.meta->Lv = L;
    s.meta->stat_chunks += 1ull;
    s.meta->pool_next = 0;
  }
}

cudaError_t launch_scan(const Dims &d, const Scratch &s, cudaStream_t st) {
  k_bucket_scan<<<1, kScanThreads, 0, st>>>(d, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// bsort: sort each bucket's records (rec_in, claim order) by (group, id) into
// rec, and stamp every record with its group's first position and length.
// Buckets are dealt round-robin to warps.  A bucket of <= 32 members is sorted
// by its warp in registers; larger ones afterwards by the whole CTA in shared
// memory (bitonic over packed keys that carry the record's local index), or,
// beyond kSortCap members, in runs merged through global memory.
// ---------------------------------------------------------------------------
constexpr int kSortThreads = 512;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kSortCap = 4096;  // largest bucket sorted in shared memory (12-bit index)

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int o) {
  const uint32_t lo = __shfl_xor_sync(FULL, (uint32_t)v, o);
  const uint32_t hi = __shfl_xor_sync(FULL, (uint32_t)(v >> 32), o);
  return ((uint64_t)hi << 32) | lo;
}

// In-place ascending bitonic sort of buf[0..n2), n2 a power of two, CTA-wide.
__device__ void block_bitonic(uint64_t *buf, int n2) {
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (n2 >> 1); i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));  // index with the stride bit clear
        const int hi = lo + stride;
        const uint64_t a = buf[lo], b = buf[hi];
        const bool up = (lo & size) == 0;
        if ((a > b) == up) {
          buf[lo] = b;
          buf[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

// Count of elements < key in the sorted run [r, r+len).
__device__ __forceinline__ int lower_rank(const uint64_t *r, int len, uint64_t key) {
  int lo = 0, hi = len;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (r[mid] < key) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// CTA-wide sort of one bucket with more than 32 members.
__device__ void sort_big_bucket(const Scratch &s, int off, int len, bool value, uint32_t gbase,
                                uint64_t *buf, int *nseg) {
  int my_seg = 0;
  if (len <= kSortCap) {
    // key = (g - gbase) << 43 | id << 12 | local index   (g - gbase < 2^21, id < 2^31)
    int n2 = 64;
    while (n2 < len) n2 <<= 1;
    for (int i = threadIdx.x; i < n2; i += blockDim.x) {
      if (i < len) {
        const int4 a = *reinterpret_cast<const int4 *>(s.rec_in + off + i);
        buf[i] = ((uint64_t)((uint32_t)a.x - gbase) << 43) | ((uint64_t)(uint32_t)a.y << 12) |
                 (uint64_t)i;
      } else {
        buf[i] = ~0ull;
      }
    }
    __syncthreads();
    block_bitonic(buf, n2);
    for (int i = threadIdx.x; i < len; i += blockDim.x) {
      const uint64_t kv = buf[i];
      const uint64_t grp = kv >> 43;
      const int first = lower_rank(buf, len, grp << 43);
      const int end = (grp + 1) >= (1ull << 21) ? len : lower_rank(buf, len, (grp + 1) << 43);
      Member m = load_member(s.rec_in + off + (int)(kv & 4095u));
      m.gstart = off + first;
      m.glen = end - first;
      store_member(s.rec + off + i, m);
      my_seg += first == i ? 1 : 0;
    }
  } else {
    // Oversized bucket: keys (g << 32 | id) sorted in runs of kSortCap in
    // shared memory, runs merged pairwise through global memory; each record
    // found again through its position, stored by id in posmap.
    const int pbase = value ? 0 : (int)(s.Lcap / 3);  // pair ids and entry ids apart
    uint64_t *A = s.sort_tmp + off;
    uint64_t *Bb = s.sort_tmp + (size_t)s.Lcap + off;
    for (int i = threadIdx.x; i < len; i += blockDim.x)
      s.posmap[pbase + (int)s.rec_in[off + i].id] = i;
    for (int r0 = 0; r0 < len; r0 += kSortCap) {
      const int rl = min(kSortCap, len - r0);
      int n2 = 64;
      while (n2 < rl) n2 <<= 1;
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        if (i < rl) {
          const int4 a = *reinterpret_cast<const int4 *>(s.rec_in + off + r0 + i);
          buf[i] = ((uint64_t)(uint32_t)a.x << 32) | (uint32_t)a.y;
        } else {
          buf[i] = ~0ull;
        }
      }
      __syncthreads();
      block_bitonic(buf, n2);
      for (int i = threadIdx.x; i < rl; i += blockDim.x) A[r0 + i] = buf[i];
      __syncthreads();
    }
    uint64_t *src = A, *dst = Bb;
    for (int width = kSortCap; width < len; width <<= 1) {
      for (int i = threadIdx.x; i < len; i += blockDim.x) {
        const int a0 = (i / (2 * width)) * 2 * width;
        const int alen = min(width, len - a0);
        const int b0 = a0 + alen;
        const int blen = max(0, min(width, len - b0));
        const uint64_t key = src[i];
        const int pos = i < b0 ? (i - a0) + lower_rank(src + b0, blen, key)
                               : (i - b0) + lower_rank(src + a0, alen, key);
        dst[a0 + pos] = key;
      }
      __syncthreads();
      uint64_t *t = src;
      src = dst;
      dst = t;
    }
    for (int i = threadIdx.x; i < len; i += blockDim.x) {
      const uint64_t kv = src[i];
      const uint64_t grp = kv >> 32;
      const int first = lower_rank(src, len, grp << 32);
      const int end = lower_rank(src, len, (grp + 1) << 32);
      Member m = load_member(s.rec_in + off + s.posmap[pbase + (int)(uint32_t)kv]);
      m.gstart = off + first;
      m.glen = end - first;
      store_member(s.rec + off + i, m);
      my_seg += first == i ? 1 : 0;
    }
  }
  if (my_seg) atomicAdd(nseg, my_seg);
  __syncthreads();
}

__global__ void __launch_bounds__(kSortThreads) k_bucket_sort(Dims d, Scratch s) {
  __shared__ uint64_t buf[kSortCap];
  __shared__ int nseg[2];  // distinct value rows / sub-key rows seen by this CTA
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  if (threadIdx.x < 2) nseg[threadIdx.x] = 0;
  __syncthreads();
  const int stride = gridDim.x * kSortWarps;
  // phase 1: small buckets, one warp each
  for (int b = blockIdx.x * kSortWarps + wib; b < d.NB; b += stride) {
    const int off = s.boff[b], len = s.boff[b + 1] - off;
    if (len == 0 || len > 32) continue;
    Member m{};
    uint64_t key = ~0ull;
    if (lane < len) {
      m = load_member(s.rec_in + off + lane);
      key = ((uint64_t)m.g << 32) | m.id;
    }
    // bitonic sort of (key, source lane) across the warp
    int src = lane;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
      for (int st = size >> 1; st > 0; st >>= 1) {
        const uint64_t ok = shfl_xor64(key, st);
        const int os = __shfl_xor_sync(FULL, src, st);
        const bool up = (lane & size) == 0 || size == 32;
        const bool lower = (lane & st) == 0;
        const bool keep = (lower == up) ? (key <= ok) : (key >= ok);
        if (!keep) {
          key = ok;
          src = os;
        }
      }
    }
    // the record of rank `lane` comes from lane `src`
    Member r;
    r.g = __shfl_sync(FULL, m.g, src);
    r.id = __shfl_sync(FULL, m.id, src);
    r.srow = __shfl_sync(FULL, m.srow, src);
    r.coef = __shfl_sync(FULL, m.coef, src);
    r.c0 = __shfl_sync(FULL, m.c0, src);
    r.c1 = __shfl_sync(FULL, m.c1, src);
    const uint32_t prev_g = __shfl_up_sync(FULL, r.g, 1);
    const bool head = lane < len && (lane == 0 || prev_g != r.g);
    const unsigned heads = __ballot_sync(FULL, head);
    if (lane < len) {
      const unsigned upto = heads & ((2u << lane) - 1u);  // heads at or below this lane
      const int h0 = 31 - __clz(upto);
      const unsigned after = heads & ~((2u << h0) - 1u);  // heads after the group's first
      r.gstart = off + h0;
      r.glen = (after ? __ffs(after) - 1 : len) - h0;
      store_member(s.rec + off + lane, r);
    }
    if (lane == 0) atomicAdd(&nseg[b < d.NBv ? 0 : 1], __popc(heads));
  }
  __syncthreads();
  // phase 2: large buckets of this CTA's warps, by the whole CTA
  for (int base = blockIdx.x * kSortWarps; base < d.NB; base += stride) {
    for (int w = 0; w < kSortWarps && base + w < d.NB; ++w) {
      const int b = base + w;
      const int off = s.boff[b], len = s.boff[b + 1] - off;
      if (len <= 32) continue;
      const bool value = b < d.NBv;
      const uint32_t gbase =
          value ? ((uint32_t)b << d.vshift) : (uint32_t)d.N + (uint32_t)(b - d.NBv);
      sort_big_bucket(s, off, len, value, gbase, buf, &nseg[value ? 0 : 1]);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (nseg[0]) atomicAdd(&s.meta->stat_value_rows, (unsigned long long)nseg[0]);
    if (nseg[1]) atomicAdd(&s.meta->stat_key_rows, (unsigned long long)nseg[1]);
  }
}

cudaError_t launch_bsort(const Dims &d, const Scratch &s, cudaStream_t st) {
  static int per_sm = 0;
  if (!per_sm) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_bucket_sort, kSortThreads, 0);
    if (per_sm < 1) per_sm = 1;
  }
  int blocks = (d.NB + kSortWarps - 1) / kSortWarps;
  if (blocks > d.sm_count * per_sm) blocks = d.sm_count * per_sm;
  k_bucket_sort<<<blocks, kSortThreads, 0, st>>>(d, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// apply: every group is cut into blocks of kBlock members counted from the
// group's first member; the warp that meets a block's first position sums the
// block in order, loading a few source rows at a time (E rows for value rows,
// query halves for sub-key rows) together with the target row.  A group of
// one block is written at once.  A longer group publishes one partial per
// block in a pool; the last block to arrive adds the partials in block order
// and writes the row.  Work per warp is bounded by kBlock members whatever the
// skew, and no sum depends on scheduling.
// ---------------------------------------------------------------------------
constexpr int kApplyWarps = 8;
constexpr int kBlock = 32;

// Columns are processed in blocks of 32 * Q4 float4 (<= 512 floats), so the
// registers a warp holds stay bounded for any row width.
template <int Q4>
__device__ __forceinline__ void load_row(const float *src, int cb, int n4, float4 (&r)[Q4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int q = 0; q < Q4; ++q) {
    const int c4 = cb + lane + 32 * q;
    r[q] = c4 < n4 ? *reinterpret_cast<const float4 *>(src + 4 * c4)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

template <int Q4>
__device__ __forceinline__ void fma_row(float4 (&acc)[Q4], float c, const float4 (&r)[Q4]) {
#pragma unroll
  for (int q = 0; q < Q4; ++q) {
    acc[q].x = fmaf(c, r[q].x, acc[q].x);
    acc[q].y = fmaf(c, r[q].y, acc[q].y);
    acc[q].z = fmaf(c, r[q].z, acc[q].z);
    acc[q].w = fmaf(c, r[q].w, acc[q].w);
  }
}

// Row update (column block at cb) from a group's complete sum.
template <int Q4>
__device__ __forceinline__ void update_row(const Dims &d, bool value, float *dst, int cb,
                                           int n4, const float4 (&row)[Q4],
                                           const float4 (&acc)[Q4], float c0) {
  const int lane = threadIdx.x & 31;
  if (value) {
    if (!(c0 > 0.f)) return;
    const float scale = d.eta / c0;
#pragma unroll
    for (int q = 0; q < Q4; ++q) {
      const int c4 = cb + lane + 32 * q;
      if (c4 < n4) {
        float4 v = row[q];
        v.x -= scale * acc[q].x;
        v.y -= scale * acc[q].y;
        v.z -= scale * acc[q].z;
        v.w -= scale * acc[q].w;
        *reinterpret_cast<float4 *>(dst + 4 * c4) = v;
      }
    }
  } else {
    const float two_eta = 2.f * d.eta;
#pragma unroll
    for (int q = 0; q < Q4; ++q) {
      const int c4 = cb + lane + 32 * q;
      if (c4 < n4) {
        float4 kv = row[q];
        kv.x -= two_eta * (acc[q].x - c0 * kv.x);
        kv.y -= two_eta * (acc[q].y - c0 * kv.y);
        kv.z -= two_eta * (acc[q].z - c0 * kv.z);
        kv.w -= two_eta * (acc[q].w - c0 * kv.w);
        *reinterpret_cast<float4 *>(dst + 4 * c4) = kv;
      }
    }
  }
}

// Entropy term of a value row: dL_addr/dw = (lam/M)(log pbar + 1) for every
// pair of the group, pbar = (sum of the group's weights) / M.
__device__ __forceinline__ void write_entropy_term(const Dims &d, const Scratch &s, float wsum,
                                                   int g0, int len) {
  const float pbar = wsum / (float)d.M;
  const float bterm = (d.lam / (float)d.M) * (logf(pbar) + 1.f);
  for (int x = g0 + (threadIdx.x & 31); x < g0 + len; x += 32) s.pb[s.rec[x].id] = bterm;
}

// Ordered sum over the block's members (member j's metadata in lane j),
// column block cb, a few source rows in flight at a time.
template <int Q4>
__device__ __forceinline__ void sum_block(const Dims &d, const Scratch &s, bool value, int cnt,
                                          int srow_l, float coef_l, int cb, int n4,
                                          float4 (&acc)[Q4]) {
  constexpr int kBatch = Q4 >= 4 ? 2 : 4;
  const float *base = value ? s.E : s.Qs;
  const int width = value ? d.dv : d.dh;
#pragma unroll
  for (int q = 0; q < Q4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < cnt; j += kBatch) {
    float4 r[kBatch][Q4];
    float cf[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int sr = __shfl_sync(FULL, srow_l, (j + u) & 31);
      cf[u] = __shfl_sync(FULL, coef_l, (j + u) & 31);
      if (j + u < cnt) load_row<Q4>(base + (int64_t)sr * width, cb, n4, r[u]);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (j + u < cnt) fma_row<Q4>(acc, cf[u], r[u]);
  }
}

// Last block of a long group: add the block partials in block order and
// write the row (kept out of line so the common path keeps its registers).
template <int Q4>
__device__ __noinline__ void combine_partials(const Dims &d, const Scratch &s, bool value,
                                              float *dst, int n4, int g0, int len,
                                              int nblocks) {
  constexpr int CB = 32 * Q4;
  const int lane = threadIdx.x & 31;
  float4 acc[Q4], row[Q4];
  float C = 0.f, W = 0.f;
  for (int b = 0; b < nblocks; ++b) {
    const float *pp = s.partial + (size_t)__ldcg(&s.slotmap[g0 + b * kBlock]) * s.pwidth;
    C += __ldcg(pp);
    W += __ldcg(pp + 1);
  }
  for (int cb = 0; cb < n4; cb += CB) {
    load_row<Q4>(dst, cb, n4, row);
#pragma unroll
    for (int q = 0; q < Q4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int b = 0; b < nblocks; b += 2) {
      float4 pv[2][Q4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (b + u < nblocks) {
          const float *pp =
              s.partial + (size_t)__ldcg(&s.slotmap[g0 + (b + u) * kBlock]) * s.pwidth;
#pragma unroll
          for (int q = 0; q < Q4; ++q) {
            const int c4 = cb + lane + 32 * q;
            pv[u][q] = c4 < n4 ? __ldcg(reinterpret_cast<const float4 *>(pp + 4 + 4 * c4))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (b + u < nblocks) {
#pragma unroll
          for (int q = 0; q < Q4; ++q) {
            acc[q].x += pv[u][q].x;
            acc[q].y += pv[u][q].y;
            acc[q].z += pv[u][q].z;
            acc[q].w += pv[u][q].w;
          }
        }
      }
    }
    update_row<Q4>(d, value, dst, cb, n4, row, acc, C);
  }
  if (value && d.lam != 0.f) write_entropy_term(d, s, W, g0, len);
}

template <int Q4>
__global__ void __launch_bounds__(kApplyWarps * 32) k_apply(Dims d, float *__restrict__ V,
                                                            float *__restrict__ K, Scratch s,
                                                            int part) {
  constexpr int CB = 32 * Q4;  // float4 columns per block
  const int lane = threadIdx.x & 31;
  const int L = s.meta->L, Lv = s.meta->Lv;
  const int lo = part == 2 ? Lv : 0;  // part 0: all, 1: value rows, 2: sub-key rows
  const int hi = part == 1 ? Lv : L;
  const bool alpha_later = d.lam != 0.f;  // sub-key alphas come from pgrad
  for (int x = lo + blockIdx.x * kApplyWarps + (threadIdx.x >> 5); x < hi;
       x += gridDim.x * kApplyWarps) {
    const int4 head = *reinterpret_cast<const int4 *>(s.rec + x);  // g, id, srow, gstart
    const int g0 = head.w;
    if ((x - g0) % kBlock != 0) continue;  // not the first member of a block
    const int len = s.rec[x].glen;
    const int cnt = min(kBlock, g0 + len - x);
    const uint32_t g = (uint32_t)head.x;
    const bool value = g < (uint32_t)d.N;
    const int n4 = (value ? d.dv : d.dh) >> 2;
    float *dst = value ? V + (int64_t)g * d.dv : K + (int64_t)(g - (uint32_t)d.N) * d.dh;
    // lane j: metadata of member x + j
    int srow_l = 0;
    float coef_l = 0.f, c0_l = 0.f, c1_l = 0.f;
    if (lane < cnt) {
      const Member m = load_member(s.rec + x + lane);
      srow_l = m.srow;
      coef_l = m.coef;
      c0_l = m.c0;
      c1_l = m.c1;
      if (!value && alpha_later) {
        coef_l = s.ealpha[m.id];
        c0_l = coef_l;
      }
    }
    // ordered scalar sums over the block
    float c0 = 0.f, c1 = 0.f;
    for (int j = 0; j < cnt; ++j) {
      c0 += __shfl_sync(FULL, c0_l, j);
      c1 += __shfl_sync(FULL, c1_l, j);
    }
    const bool whole = len <= kBlock;  // the whole group is in this block
    float *p = nullptr;
    if (!whole) {  // long group: this block's partial goes to a pool slot
      int slot = 0;
      if (lane == 0) slot = atomicAdd(&s.meta->pool_next, 1);
      slot = __shfl_sync(FULL, slot, 0);
      if (slot >= s.pool_cap) {  // cannot happen: the pool holds 2*Lcap/kBlock blocks
        if (lane == 0) atomicOr(&s.meta->err, ERR_POOL_OVERFLOW);
        continue;
      }
      p = s.partial + (size_t)slot * s.pwidth;
      if (lane == 0) s.slotmap[x] = slot;
    }
    float4 acc[Q4], row[Q4];
    for (int cb = 0; cb < n4; cb += CB) {
      if (whole) load_row<Q4>(dst, cb, n4, row);  // in flight with the first sources
      sum_block<Q4>(d, s, value, cnt, srow_l, coef_l, cb, n4, acc);
      if (whole) {
        update_row<Q4>(d, value, dst, cb, n4, row, acc, c0);
      } else {
#pragma unroll
        for (int q = 0; q < Q4; ++q) {
          const int c4 = cb + lane + 32 * q;
          if (c4 < n4) *reinterpret_cast<float4 *>(p + 4 + 4 * c4) = acc[q];
        }
      }
    }
    if (whole) {
      if (value && d.lam != 0.f) write_entropy_term(d, s, c1, g0, len);
      continue;
    }
    if (lane == 0) {
      p[0] = c0;
      p[1] = c1;
    }
    __threadfence();
    __syncwarp();
    const int nblocks = (len + kBlock - 1) / kBlock;
    int old = 0;
    if (lane == 0) old = atomicAdd(&s.segcnt[g0], 1);
    old = __shfl_sync(FULL, old, 0);
    if (old != nblocks - 1) continue;
    // last block in: add the partials in block order
    __threadfence();
    combine_partials<Q4>(d, s, value, dst, n4, g0, len, nblocks);
    if (lane == 0) s.segcnt[g0] = 0;  // ready for the next chunk
  }
}

template <int Q4>
static cudaError_t launch_apply_t(const Dims &d, float *V, float *K, const Scratch &s,
                                  cudaStream_t st, int part) {
  static int per_sm = 0;
  if (!per_sm) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_apply<Q4>, kApplyWarps * 32, 0);
    if (per_sm < 1) per_sm = 1;
  }
  int64_t blocks = (s.Lcap + kApplyWarps - 1) / kApplyWarps;
  if (blocks > (int64_t)d.sm_count * per_sm) blocks = (int64_t)d.sm_count * per_sm;
  k_apply<Q4><<<(int)blocks, kApplyWarps * 32, 0, st>>>(d, V, K, s, part);
  return cudaGetLastError();
}

cudaError_t launch_apply(const Dims &d, float *V, float *K, const Scratch &s, cudaStream_t st,
                         int part) {
  const int w4 = ((d.dv > d.dh ? d.dv : d.dh) / 4 + 31) / 32;
  if (w4 <= 1) return launch_apply_t<1>(d, V, K, s, st, part);
  if (w4 <= 2) return launch_apply_t<2>(d, V, K, s, st, part);
  return launch_apply_t<4>(d, V, K, s, st, part);
}

// ---------------------------------------------------------------------------
// pgrad (lam > 0 only): dL/ds_r = w_r (gamma_r - sum_r' w_r' gamma_r'),
// gamma = dL_mse/dw + dL_addr/dw, then alpha of the token-head's entries.
// Warp per token-head, lane r.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_pgrad(Dims d, Scratch s) {
  const int lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (m >= d.M) return;
  const int64_t p = (int64_t)m * d.k + lane;
  float w = 0.f, gam = 0.f;
  if (lane < d.k) {
    w = s.pw[p];
    gam = s.pa[p] + s.pb[p];
  }
  const float S = warp_sum(w * gam);
  const float dl = lane < d.k ? w * (gam - S) : 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int mh = m * 2 + half;
    const int ne = s.ecount[mh];
    for (int idx = 0; idx < ne; ++idx) {
      const int64_t e = (int64_t)mh * d.k + idx;
      const unsigned mask = s.emask[e];
      const float sum = warp_sum((mask >> lane) & 1u ? dl : 0.f);
      if (lane == 0) s.ealpha[e] = s.einv[e] * sum;
    }
  }
}

cudaError_t launch_pgrad(const Dims &d, const Scratch &s, cudaStream_t st) {
  k_pgrad<<<(d.M + 7) / 8, 256, 0, st>>>(d, s);
  return cudaGetLastError();
}

}  // namespace fwpkm
