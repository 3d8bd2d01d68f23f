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

// A bucket of more than this many members is sorted by a whole CTA (the scan
// lists it); smaller ones by one warp.
constexpr int kWarpBucket = 32;

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
// scan: bucket offsets, one pass over up to kScanMaxCtas CTAs.  Each CTA
// holds kScanTile counts in registers (16-byte loads), scans them, publishes
// its total tagged with the chunk's epoch, and adds the totals of the CTAs
// before it (all CTAs of the grid are resident together: at most 64 small
// ones).  Many small CTAs rather than one large one: the kernel is bound by
// the load and store instructions a multiprocessor issues, not by bytes.  The
// waits for those totals are bounded; a timeout sets ERR_SCAN_TIMEOUT.
// Counts are zeroed for the next chunk; CTA 0 resets the work-list counters.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kScanPer = 8;                         // counts per thread
constexpr int kScanTile = kScanThreads * kScanPer;  // counts per CTA
static_assert(kScanTile * kScanMaxCtas >= 65536 + 2 * 16 * 1024, "every bucket count fits");

// A CTA's total is read by the later CTAs for its own value only (nothing
// else this CTA wrote is read through it), and the epoch in its upper half
// tells a stale word from the current one: relaxed stores and loads at GPU
// scope are enough, and the store does not wait for the CTA's earlier ones.
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__global__ void __launch_bounds__(kScanThreads) k_bucket_scan(Dims d, Scratch s) {
  griddep_wait();
  griddep_launch();
  __shared__ int red[32];
  __shared__ int prefix_s;
  const int NB = d.NB, c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const unsigned long long epoch = s.scan_sync[0];  // advanced by this chunk's selection
  const int b0 = c * kScanTile + tid * kScanPer;
  int v[kScanPer];
  if (b0 + kScanPer <= NB) {  // bcnt is 256-byte aligned and b0 a multiple of 8
#pragma unroll
    for (int q = 0; q < kScanPer / 4; ++q) {
      const int4 x = *reinterpret_cast<const int4 *>(s.bcnt + b0 + 4 * q);
      v[4 * q] = x.x;
      v[4 * q + 1] = x.y;
      v[4 * q + 2] = x.z;
      v[4 * q + 3] = x.w;
      *reinterpret_cast<int4 *>(s.bcnt + b0 + 4 * q) = make_int4(0, 0, 0, 0);  // next chunk
    }
  } else {
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
      v[i] = b0 + i < NB ? s.bcnt[b0 + i] : 0;
      if (b0 + i < NB) s.bcnt[b0 + i] = 0;
    }
  }
  int total = 0, nbig = 0;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    total += v[i];
    nbig += v[i] > kWarpBucket ? 1 : 0;
  }
  // The large buckets are listed for the sort, one reservation per warp that
  // has any; the reservation is taken now and its result used only at the
  // end, so that its round trip overlaps the scan.
  int ib = nbig;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(FULL, ib, o);
    if (lane >= o) ib += t;
  }
  int big_base = 0;
  if (lane == 31 && ib) big_base = atomicAdd(&s.meta->nbig, ib);
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) red[w] = incl;
  __syncthreads();
  if (w == 0) {
    int x = lane < kScanWarps ? red[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(FULL, x, o);
      if (lane >= o) x += t;
    }
    red[lane] = x;
  }
  __syncthreads();
  const int cta_total = red[kScanWarps - 1];
  if (tid == 0 && gridDim.x > 1)
    st_relaxed_u64(&s.scan_sync[1 + c], (epoch << 32) | (unsigned)cta_total);
  if (w == 0) {
    // totals of CTAs 0 .. c-1, one per lane and round
    int pre = 0;
    bool ok_all = true;
    for (int j = lane; j < c; j += 32) {
      bool ok = false;
      unsigned long long a = 0;
      for (long long it = 0; it < d.scan_polls; ++it) {
        a = ld_relaxed_u64(&s.scan_sync[1 + j]);
        if ((a >> 32) == (epoch & 0xffffffffull)) {
          ok = true;
          break;
        }
      }
      ok_all = ok_all && ok;
      pre += ok ? (int)(unsigned)a : 0;
    }
    if (!ok_all) atomicOr(&s.meta->err, ERR_SCAN_TIMEOUT);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pre += __shfl_xor_sync(FULL, pre, o);
    if (lane == 0) prefix_s = pre;
  }
  __syncthreads();
  int run = prefix_s + (w > 0 ? red[w - 1] : 0) + incl - total;
  if (b0 + kScanPer <= NB) {
#pragma unroll
    for (int q = 0; q < kScanPer / 4; ++q) {
      int4 o;
      o.x = run;
      run += v[4 * q];
      o.y = run;
      run += v[4 * q + 1];
      o.z = run;
      run += v[4 * q + 2];
      o.w = run;
      run += v[4 * q + 3];
      *reinterpret_cast<int4 *>(s.boff + b0 + 4 * q) = o;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) {
      if (b0 + i < NB) s.boff[b0 + i] = run;
      run += v[i];
    }
  }
  if (__any_sync(FULL, nbig > 0)) {
    int pos = __shfl_sync(FULL, big_base, 31) + ib - nbig;
#pragma unroll
    for (int i = 0; i < kScanPer; ++i)
      if (v[i] > kWarpBucket) s.biglist[pos++] = b0 + i;
  }
  if (tid == 0 && c == gridDim.x - 1) {
    const int L = prefix_s + cta_total;
    s.boff[NB] = L;
    s.meta->L = L;
    s.meta->stat_records += (unsigned long long)L;
  }
  if (tid == 0 && c == 0) {
    s.meta->stat_chunks += 1ull;
#pragma unroll
    for (int kind = 0; kind < 2; ++kind) {
      s.meta->nshort[kind] = 0;
      s.meta->nlong[kind] = 0;
    }
  }
}

cudaError_t launch_scan(const Dims &d, const Scratch &s, cudaStream_t st) {
  const int ctas = (d.NB + kScanTile - 1) / kScanTile;
  if (ctas > kScanMaxCtas) return cudaErrorInvalidValue;
  return launch_k(d.pdl, k_bucket_scan, ctas, kScanThreads, 0, st, d, s);
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

// A record on its way from rec_in to rec.  A sub-key record already carries
// its alpha when the entropy term is off (the read wrote it); with the term
// on, alpha is known only after pgrad and the apply reads it itself.
__device__ __forceinline__ Member fetch_member(const Dims &, const Scratch &, const Member *p) {
  return load_member(p);
}

constexpr int kShortMax = 4;  // groups up to this size are applied by one warp, whole rows
constexpr int kBlock = 32;    // longer groups are applied in blocks of this many members

// Work lists of the apply kernel for a group of kind `kind` (0: value row,
// 1: sub-key row) that starts at position x0: a short group goes to
// shortlist, a longer one to longlist, one entry per block of kBlock members
// (consecutive entries).  Thread-level (one call per group head).
__device__ __forceinline__ void list_group(const Scratch &s, int kind, int x0, int len) {
  if (len <= kShortMax) {
    s.shortlist[kind][atomicAdd(&s.meta->nshort[kind], 1)] = x0;
  } else {
    const int nb = (len + kBlock - 1) / kBlock;
    const int base = atomicAdd(&s.meta->nlong[kind], nb);
    for (int b = 0; b < nb; ++b) s.longlist[kind][base + b] = x0 + b * kBlock;
  }
}

// Rank sort of one bucket with more than 32 members.  Inside a group, every
// member comes from a different token-head m (a token-head's k slots are
// distinct, and its sub-key entries are de-duplicated per row), and member
// ids grow with m (pair p = m*k + r, entry e = (m*2 + half)*k + idx).  So the
// (group, id) order is the (group, m) order, and a member's rank is found
// without sorting: one bitmap of token-heads per group of the bucket, an
// exclusive prefix of the words' popcounts (flat over groups, then words)
// gives every group's start and every member's place.  A few barriers instead
// of a bitonic network's dozens.  Returns false, having written nothing,
// when the bitmaps do not fit or a group repeats a token-head (forced
// selections with duplicate slots); the caller then sorts.
constexpr int kRankWords = kSortCap;  // bitmap words (the prefix takes as many)
constexpr int kRankGroups = 256;      // groups per bucket (slots per value bucket)

struct RankSmem {
  uint32_t *bits;  // [kRankWords]
  uint32_t *pre;   // [kRankWords]
  int *red;        // [32]
  int *flag;
};

__device__ bool rank_big_bucket(const Dims &d, const Scratch &s, int off, int len, bool value,
                                uint32_t gbase, const RankSmem &r, int *nseg) {
  const int G = value ? (1 << d.vshift) : 1;
  const int Mw = (d.M + 31) >> 5;
  const int W = G * Mw;
  if (G > kRankGroups || W > kRankWords) return false;  // the same in every thread
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t kdiv = value ? (uint32_t)d.k : 2u * (uint32_t)d.k;  // id -> token-head
  for (int i = tid; i < W; i += blockDim.x) r.bits[i] = 0u;
  if (tid == 0) *r.flag = 0;
  __syncthreads();
  for (int i = tid; i < len; i += blockDim.x) {
    const int2 gi = *reinterpret_cast<const int2 *>(s.rec_in + off + i);  // g, id
    const int lg = value ? (int)((uint32_t)gi.x - gbase) : 0;
    const uint32_t m = (uint32_t)gi.y / kdiv;
    const uint32_t bit = 1u << (m & 31u);
    if (atomicOr(&r.bits[lg * Mw + (int)(m >> 5)], bit) & bit) *r.flag = 1;
  }
  __syncthreads();
  if (*r.flag) return false;
  // exclusive prefix of the popcounts, kRankWords / kSortThreads words per thread
  constexpr int per = kRankWords / kSortThreads;
  const int w0 = tid * per;
  int v[per], tot = 0;
#pragma unroll
  for (int q = 0; q < per; ++q) {
    v[q] = w0 + q < W ? __popc(r.bits[w0 + q]) : 0;
    tot += v[q];
  }
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) r.red[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int x = lane < kSortWarps ? r.red[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(FULL, x, o);
      if (lane >= o) x += t;
    }
    r.red[lane] = x;
  }
  __syncthreads();
  int run = (warp > 0 ? r.red[warp - 1] : 0) + incl - tot;
#pragma unroll
  for (int q = 0; q < per; ++q) {
    if (w0 + q < W) r.pre[w0 + q] = run;
    run += v[q];
  }
  __syncthreads();
  int my_seg = 0;
  for (int i = tid; i < len; i += blockDim.x) {
    Member mr = fetch_member(d, s, s.rec_in + off + i);
    const int lg = value ? (int)(mr.g - gbase) : 0;
    const uint32_t m = mr.id / kdiv;
    const int wi = lg * Mw + (int)(m >> 5);
    const int pos = (int)r.pre[wi] + __popc(r.bits[wi] & ((1u << (m & 31u)) - 1u));
    const int first = (int)r.pre[lg * Mw];
    // every member set one bit, so the group's size is its words' popcount
    const int end = (lg + 1) * Mw < W ? (int)r.pre[(lg + 1) * Mw] : len;
    mr.gstart = off + first;
    mr.glen = end - first;
    store_member(s.rec + off + pos, mr);
    if (pos == first) {
      my_seg += 1;
      list_group(s, value ? 0 : 1, off + pos, mr.glen);
    }
  }
  if (my_seg) atomicAdd(nseg, my_seg);
  __syncthreads();
  return true;
}

// CTA-wide sort of one bucket with more than 32 members.
__device__ void sort_big_bucket(const Dims &d, const Scratch &s, int off, int len, bool value,
                                uint32_t gbase, uint64_t *buf, const RankSmem &rs, int *nseg) {
  if (rank_big_bucket(d, s, off, len, value, gbase, rs, nseg)) return;
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
      const int end = lower_rank(buf, len, (grp + 1) << 43);
      Member m = fetch_member(d, s, s.rec_in + off + (int)(kv & 4095u));
      m.gstart = off + first;
      m.glen = end - first;
      store_member(s.rec + off + i, m);
      if (first == i) {
        my_seg += 1;
        list_group(s, value ? 0 : 1, off + i, end - first);
      }
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
      Member m = fetch_member(d, s, s.rec_in + off + s.posmap[pbase + (int)(uint32_t)kv]);
      m.gstart = off + first;
      m.glen = end - first;
      store_member(s.rec + off + i, m);
      if (first == i) {
        my_seg += 1;
        list_group(s, value ? 0 : 1, off + i, end - first);
      }
    }
  }
  if (my_seg) atomicAdd(nseg, my_seg);
  __syncthreads();
}

// Work-list entries a sort CTA stages in shared memory per list (short and
// long groups of each kind) before it appends them to the global lists with
// one reservation each; past that many, an entry is appended at once.
constexpr int kListStage = 512;

__device__ __forceinline__ void stage_list(const Scratch &s, int (*lst)[kListStage], int kind,
                                           bool lng, int i, int x) {
  if (i < kListStage) lst[(lng ? 2 : 0) + kind][i] = x;
  else if (lng) s.longlist[kind][atomicAdd(&s.meta->nlong[kind], 1)] = x;
  else s.shortlist[kind][atomicAdd(&s.meta->nshort[kind], 1)] = x;
}

template <typename TQ>
__global__ void __launch_bounds__(kSortThreads)
    k_bucket_sort(Dims d, Scratch s, Dims dn, const TQ *__restrict__ Q, int sort_blocks) {
  __shared__ uint64_t buf[kSortCap];
  __shared__ int nseg[2];  // distinct value rows / sub-key rows seen by this CTA
  __shared__ int rank_red[32], rank_flag;
  __shared__ int lst[4][kListStage];  // staged entries: short[kind], then long[kind]
  __shared__ int lst_n[4], lst_base[4];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  // The next chunk's query halves, one warp per half row, made before the
  // grid dependency wait, while the read finishes: they need only the
  // caller's Q (which the caller's stream orders before this grid), and the
  // halves they overwrite were last read by this chunk's score, which
  // completed before the read was launched.
  {
    const int64_t nq = dn.rows > 0 ? (int64_t)2 * dn.H * dn.rows : 0;
    for (int64_t w = (int64_t)blockIdx.x * kSortWarps + wib; w < nq;
         w += (int64_t)gridDim.x * kSortWarps)
      prep_query_half(dn, Q, s, w);
  }
  griddep_wait();
  griddep_launch();
  // An earlier kernel of the chunk gave up: its offsets or selection may be
  // wrong, so nothing is sorted (the next chunk's halves above are still
  // prepared; they index nothing).
  if (chunk_aborted(s, ERR_SORT_OVERFLOW)) return;
  if (threadIdx.x < 2) nseg[threadIdx.x] = 0;
  if (threadIdx.x < 4) lst_n[threadIdx.x] = 0;
  __syncthreads();
  const int stride = sort_blocks * kSortWarps;
  // phase 1: small buckets, one warp each; large ones are left to phase 2.  Bucket b
  // goes to CTA b % sort_blocks: neighbouring buckets (slots of one popular
  // sub-key row) land in different CTAs.
  // The offsets of a warp's next 32 buckets are loaded together, one per lane.
  int nxt_off = 0, nxt_end = 0;
  for (int b = blockIdx.x + sort_blocks * wib, i = 0; b < d.NB; b += stride, ++i) {
    if ((i & 31) == 0) {
      const int bl = b + lane * stride;
      nxt_off = bl < d.NB ? s.boff[bl] : 0;
      nxt_end = bl < d.NB ? s.boff[bl + 1] : 0;
    }
    const int off = __shfl_sync(FULL, nxt_off, i & 31);
    const int len = __shfl_sync(FULL, nxt_end, i & 31) - off;
    if (len == 0) continue;
    if (len > kWarpBucket) continue;  // listed by the scan; sorted in phase 2
    Member m{};
    uint64_t key = ~0ull;
    if (lane < len) {
      m = fetch_member(d, s, s.rec_in + off + lane);
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
    int glen = 0;
    if (lane < len) {
      const unsigned upto = heads & ((2u << lane) - 1u);  // heads at or below this lane
      const int h0 = 31 - __clz(upto);
      const unsigned after = heads & ~((2u << h0) - 1u);  // heads after the group's first
      r.gstart = off + h0;
      r.glen = glen = (after ? __ffs(after) - 1 : len) - h0;
      store_member(s.rec + off + lane, r);
    }
    // work lists: short groups; longer ones (one block each, <= 32 members)
    const int kind = b < d.NBv ? 0 : 1;
    const bool sh = head && glen <= kShortMax, lg = head && glen > kShortMax;
    const unsigned sb = __ballot_sync(FULL, sh), lb = __ballot_sync(FULL, lg);
    int sbase = 0, lbase = 0;
    if (lane == 0) {
      if (sb) sbase = atomicAdd(&lst_n[kind], __popc(sb));
      if (lb) lbase = atomicAdd(&lst_n[2 + kind], __popc(lb));
    }
    sbase = __shfl_sync(FULL, sbase, 0);
    lbase = __shfl_sync(FULL, lbase, 0);
    if (sh) stage_list(s, lst, kind, false, sbase + __popc(sb & lanemask_lt()), off + lane);
    if (lg) stage_list(s, lst, kind, true, lbase + __popc(lb & lanemask_lt()), off + lane);
    if (lane == 0) atomicAdd(&nseg[b < d.NBv ? 0 : 1], __popc(heads));
  }
  __syncthreads();
  // phase 2: the large buckets, each by a whole CTA, dealt out in the order
  // of the scan's list (one each while there are CTAs enough)
  const int nbig = s.meta->nbig;
  for (int i = blockIdx.x; i < nbig; i += sort_blocks) {
    const int b = s.biglist[i];
    const int off = s.boff[b], len = s.boff[b + 1] - off;
    const bool value = b < d.NBv;
    const uint32_t gbase =
        value ? ((uint32_t)b << d.vshift) : (uint32_t)d.Nt + (uint32_t)(b - d.NBv);
    const RankSmem rs{reinterpret_cast<uint32_t *>(buf), reinterpret_cast<uint32_t *>(buf) + kRankWords,
                      rank_red, &rank_flag};
    sort_big_bucket(d, s, off, len, value, gbase, buf, rs, &nseg[value ? 0 : 1]);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (nseg[0]) atomicAdd(&s.meta->stat_value_rows, (unsigned long long)nseg[0]);
    if (nseg[1]) atomicAdd(&s.meta->stat_key_rows, (unsigned long long)nseg[1]);
  }
  // the staged entries go to the global lists, one reservation per list
  if (threadIdx.x < 4) {
    const int q = threadIdx.x, c = min(lst_n[q], kListStage);
    int *ctr = q < 2 ? &s.meta->nshort[q] : &s.meta->nlong[q - 2];
    lst_base[q] = c ? atomicAdd(ctr, c) : 0;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = min(lst_n[q], kListStage);
    int *dst = q < 2 ? s.shortlist[q] : s.longlist[q - 2];
    for (int i = threadIdx.x; i < c; i += blockDim.x) dst[lst_base[q] + i] = lst[q][i];
  }
}

// The sorting grid: a warp per bucket up to the resident CTAs.  Its warps
// first prepare the next chunk's query halves (dn.rows > 0).
template <typename TQ>
static cudaError_t launch_bsort_t(const Dims &d, const Scratch &s, const Dims &dn, const TQ *Q,
                                  cudaStream_t st) {
  static int per_sm = 0;
  if (!per_sm) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_bucket_sort<TQ>, kSortThreads, 0);
    if (per_sm < 1) per_sm = 1;
  }
  int blocks = (d.NB + kSortWarps - 1) / kSortWarps;
  const int cap = d.sm_count * per_sm;
  if (blocks > cap) blocks = cap;
  return launch_k(d.pdl, k_bucket_sort<TQ>, blocks, kSortThreads, 0, st, d, s, dn, Q, blocks);
}

cudaError_t launch_bsort(const Dims &d, const Scratch &s, const Dims &dn, const void *Q,
                         int q_dtype, cudaStream_t st) {
  if (q_dtype == 1) return launch_bsort_t(d, s, dn, (const __nv_bfloat16 *)Q, st);
  return launch_bsort_t(d, s, dn, (const float *)Q, st);
}

// ---------------------------------------------------------------------------
// apply: the row updates, from the work lists bsort wrote.  One warp per
// work item:
//   - a group of <= kShortMax members: its members are summed over whole rows
//     (two column chunks at a time) and the row is written at once;
//   - a column chunk (128 floats, a float4 per lane) of a block of kBlock
//     members of a longer group: summed into the partial-pool slot of the
//     block's work-list entry, with the block's scalar sums in the slot's
//     header.  The last of a group's blocks to finish a chunk (an integer
//     arrival counter per group and chunk, after a fence) adds the blocks'
//     partials in block order and writes the row chunk.
// Lane j holds member j's record; the members' source rows (E rows for value
// rows, query halves for sub-key rows) are summed in member order, kU rows in
// flight.  Many short dependence chains rather than a few long ones, whatever
// the skew.  Every sum runs in an order fixed by the data, whatever the
// scheduling; nothing is atomic but integer counters.
// ---------------------------------------------------------------------------
constexpr int kApplyThreads = 256;
constexpr int kApplyWarps = kApplyThreads / 32;
constexpr int kChunk4 = 32;  // float4 per column chunk (one per lane)
constexpr int kU = 4;        // source rows in flight per warp

__device__ __forceinline__ float4 load_chunk(const float *row, int c4, int n4) {
  return c4 < n4 ? *reinterpret_cast<const float4 *>(row + 4 * c4)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
}
__device__ __forceinline__ float4 load_chunk(const __nv_bfloat16 *row, int c4, int n4) {
  return c4 < n4 ? load4(row, 4 * (int64_t)c4) : make_float4(0.f, 0.f, 0.f, 0.f);
}

__device__ __forceinline__ void fma4(float4 &a, float c, const float4 &x) {
  a.x = fmaf(c, x.x, a.x);
  a.y = fmaf(c, x.y, a.y);
  a.z = fmaf(c, x.z, a.z);
  a.w = fmaf(c, x.w, a.w);
}
__device__ __forceinline__ void add4(float4 &a, const float4 &x) {
  a.x += x.x;
  a.y += x.y;
  a.z += x.z;
  a.w += x.w;
}

// New value of one float4 of a target row from the group's complete sums.
//   value row : v - (eta / C) * G          (C = sum of w/H; see k_apply for a
//                                           C so small that eta / C overflows)
//   sub-key   : k - 2 eta (G - A k)        (A = sum of alpha; IDW score)
//               k - eta G                  (dot-product score: ds/dK = q)
__device__ __forceinline__ float4 updated(const Dims &d, bool value, const float4 &t,
                                          const float4 &g, float c0) {
  if (value) {
    const float sc = d.agg == AGG_SUM ? d.eta : d.eta / c0;
    return make_float4(t.x - sc * g.x, t.y - sc * g.y, t.z - sc * g.z, t.w - sc * g.w);
  }
  if (d.score_dot)
    return make_float4(t.x - d.eta * g.x, t.y - d.eta * g.y, t.z - d.eta * g.z,
                       t.w - d.eta * g.w);
  const float te = 2.f * d.eta;
  return make_float4(t.x - te * (g.x - c0 * t.x), t.y - te * (g.y - c0 * t.y),
                     t.z - te * (g.z - c0 * t.z), t.w - te * (g.w - c0 * t.w));
}

// Entropy term of a value row: dL_addr/dw = (lam/M)(log pbar + 1) for every
// pair of the group, pbar = (sum of the group's weights) / M, M the
// token-heads of the row's memory.
__device__ __forceinline__ float entropy_term(const Dims &d, float wsum) {
  return (d.lam / (float)d.Mmem) * (logf(wsum / (float)d.Mmem) + 1.f);
}

// Sum of a warp's members (lane j < cnt holds member j's srow and coef) over
// the float4 columns cb + lane + 32*q, q < Q, member order, KU rows in flight;
// member j's source row is base + srow_j * stride (E rows for value rows, the
// caller's query halves for sub-key rows).
template <int Q, int KU, typename TS>
__device__ __forceinline__ void sum_members(const TS *base, int64_t stride, int cnt, int srow,
                                            float coef, int cb, int n4, float4 (&acc)[Q]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int q = 0; q < Q; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = 0; j0 < cnt; j0 += KU) {
    float4 r[KU][Q];
#pragma unroll
    for (int u = 0; u < KU; ++u) {
      const int sr = __shfl_sync(FULL, srow, (j0 + u) & 31);
      const TS *src = base + (int64_t)sr * stride;
#pragma unroll
      for (int q = 0; q < Q; ++q)
        r[u][q] = j0 + u < cnt ? load_chunk(src, cb + lane + 32 * q, n4)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < KU; ++u) {
      const float cj = __shfl_sync(FULL, coef, (j0 + u) & 31);
      if (j0 + u < cnt) {
#pragma unroll
        for (int q = 0; q < Q; ++q) fma4(acc[q], cj, r[u][q]);
      }
    }
  }
}

// A rewritten sub-key row chunk (one float4 per lane, zeros past the row)
// also gets its TF32 split and its chunk norm, exactly as the prep makes them.
__device__ __forceinline__ void resplit_key_chunk(const Dims &d, const Scratch &s, int64_t r,
                                                  int ch, int c4, int n4, const float4 &v) {
  if (c4 < n4) split_store(s.K_hi + r * d.dh, s.K_lo + r * d.dh, 4 * c4, v);
  const float sq = chunk_sqnorm(c4 < n4 ? v : make_float4(0.f, 0.f, 0.f, 0.f));
  if ((threadIdx.x & 31) == 0) s.kn[r * kKnChunks + ch] = sq;
}

template <typename TQ>
__global__ void __launch_bounds__(kApplyThreads, 4) k_apply(Dims d, float *__restrict__ V,
                                                            float *__restrict__ K,
                                                            const TQ *__restrict__ Qin, Scratch s,
                                                            int part) {
  griddep_wait();
  griddep_launch();
  if (chunk_aborted(s, ERR_POOL_OVERFLOW)) return;  // an earlier kernel gave up
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kApplyWarps + (threadIdx.x >> 5);
  const int nw = gridDim.x * kApplyWarps;
  const bool alpha_later = d.lam != 0.f;  // sub-key alphas come from pgrad
  const int cv = (d.dv / 4 + kChunk4 - 1) / kChunk4, ck = (d.dh / 4 + kChunk4 - 1) / kChunk4;
  // Work items, longer groups' blocks first: value blocks and sub-key blocks
  // (one item per column chunk), then value groups and sub-key groups (one
  // item per group, whole rows), each present when `part` takes its kind
  // (0: both, 1: value rows, 2: sub-key rows).
  const int nlv = part != 2 ? s.meta->nlong[0] * cv : 0;
  const int nlk = part != 1 ? s.meta->nlong[1] * ck : 0;
  const int nsv = part != 2 ? s.meta->nshort[0] : 0;
  const int nsk = part != 1 ? s.meta->nshort[1] : 0;
  const int kslot0 = s.meta->nlong[0];  // sub-key partial slots follow the value blocks
  const int total = nlv + nlk + nsv + nsk;
  for (int it = gw; it < total; it += nw) {
    int i = it, kind = 0;
    bool block = true;
    if (i < nlv) {
    } else if ((i -= nlv) < nlk) {
      kind = 1;
    } else if ((i -= nlk) < nsv) {
      block = false;
    } else {
      i -= nsv;
      kind = 1;
      block = false;
    }
    const bool value = kind == 0;
    int chunk = 0;
    if (block) {
      const int nch = value ? cv : ck;
      chunk = i % nch;
      i /= nch;
    }
    const int x = block ? s.longlist[kind][i] : s.shortlist[kind][i];
    Member mj{};
    if ((int64_t)x + lane < s.Lcap) mj = load_member(s.rec + x + lane);  // past the item: unused
    const uint32_t g = __shfl_sync(FULL, mj.g, 0);
    const int g0 = __shfl_sync(FULL, mj.gstart, 0);
    const int len = __shfl_sync(FULL, mj.glen, 0);
    const int cnt = block ? min(kBlock, g0 + len - x) : len;
    float coef = 0.f, c0 = 0.f, c1 = 0.f;
    if (lane < cnt) {
      coef = mj.coef;
      c0 = mj.c0;
      c1 = mj.c1;
      if (!value && alpha_later) coef = c0 = s.ealpha[mj.id];
    }
    // butterfly sums: every lane ends with the same value, in a fixed order
    float C = c0, W = c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      C += __shfl_xor_sync(FULL, C, o);
      W += __shfl_xor_sync(FULL, W, o);
    }
    // A value row whose members' softmax weights are all denormal (scores that
    // far apart, as the dot-product score can give) has a C so small that
    // eta / C overflows: its coefficients and C are scaled by 2^64 first, which
    // is exact and leaves G / C as it is.  (A longer group's block partials are
    // scaled at the group's combine.)
    if (!block && value && d.agg != AGG_SUM && !(C * 0x1p+120f > d.eta)) {
      C *= 0x1p+64f;
      coef *= 0x1p+64f;
    }
    const int n4 = (value ? d.dv : d.dh) >> 2;
    if (block) {
      // one column chunk of a longer group's block, into its partial slot
      const int slot = (value ? 0 : kslot0) + i;
      if (slot >= s.pool_cap) {  // cannot happen: the pool holds Lcap / 4 + 2 blocks
        if (lane == 0) atomicOr(&s.meta->err, ERR_POOL_OVERFLOW);
        continue;
      }
      float *dst = s.partial + (size_t)slot * s.pwidth;
      if (lane == 0) {
        dst[2 * chunk] = C;
        dst[2 * chunk + 1] = W;
      }
      float4 acc[1];
      const int cb = chunk * kChunk4;
      if (value) sum_members<1, kU>(s.E, d.dv, cnt, mj.srow, coef, cb, n4, acc);
      else sum_members<1, kU>(Qin, d.dh, cnt, mj.srow, coef, cb, n4, acc);
      if (cb + lane < n4)
        *reinterpret_cast<float4 *>(dst + kPartHead + 4 * (cb + lane)) = acc[0];
      // The last of the group's blocks to finish this chunk adds the blocks'
      // partials in block order and writes the row chunk.
      const int nb = (len + kBlock - 1) / kBlock;
      const int slot0 = slot - (x - g0) / kBlock;  // the group's first block
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        int *cnt_at = s.arrive + (size_t)slot0 * kMaxChunks + chunk;
        last = atomicAdd(cnt_at, 1) == nb - 1;
        if (last) *cnt_at = 0;  // ready for the next chunk
      }
      if (!__shfl_sync(FULL, last, 0)) continue;
      __threadfence();
      const float *pp = s.partial + (size_t)slot0 * s.pwidth;
      // the blocks' scalar sums: lane b takes blocks b, b + 32, ... (in that
      // order), then a butterfly over the lanes; one round of loads, and an
      // order fixed by the group's length alone
      float Ct = 0.f, Wt = 0.f;
      for (int b = lane; b < nb; b += 32) {
        const float2 cw = __ldcg(reinterpret_cast<const float2 *>(pp + (size_t)b * s.pwidth +
                                                                  2 * chunk));
        Ct += cw.x;
        Wt += cw.y;
      }
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        Ct += __shfl_xor_sync(FULL, Ct, o);
        Wt += __shfl_xor_sync(FULL, Wt, o);
      }
      float *row = value ? V + (int64_t)g * d.dv : K + (int64_t)(g - (uint32_t)d.Nt) * d.dh;
      if (!value || Ct > 0.f) {
        const int c4 = cb + lane;
        const float4 t = load_chunk(row, c4, n4);
        float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int b0 = 0; b0 < nb; b0 += kU) {
          float4 r[kU];
#pragma unroll
          for (int u = 0; u < kU; ++u)
            r[u] = b0 + u < nb && c4 < n4
                       ? __ldcg(reinterpret_cast<const float4 *>(
                             pp + (size_t)(b0 + u) * s.pwidth + kPartHead + 4 * c4))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int u = 0; u < kU; ++u)
            if (b0 + u < nb) add4(tot, r[u]);
        }
        if (value && d.agg != AGG_SUM && !(Ct * 0x1p+120f > d.eta)) {  // as above
          Ct *= 0x1p+64f;
          tot = make_float4(tot.x * 0x1p+64f, tot.y * 0x1p+64f, tot.z * 0x1p+64f,
                            tot.w * 0x1p+64f);
        }
        const float4 nv = updated(d, value, t, tot, Ct);
        if (c4 < n4) *reinterpret_cast<float4 *>(row + 4 * c4) = nv;
        if (!value) resplit_key_chunk(d, s, (int64_t)(g - (uint32_t)d.Nt), chunk, c4, n4, nv);
      }
      if (chunk == 0 && value && d.lam != 0.f) {
        const float bt = entropy_term(d, Wt);
        for (int q = lane; q < len; q += 32) s.pb[s.rec[g0 + q].id] = bt;
      }
      continue;
    }
    // a short group: the whole row, two column chunks at a time
    float *dst = value ? V + (int64_t)g * d.dv : K + (int64_t)(g - (uint32_t)d.Nt) * d.dh;
    if ((!value || C > 0.f) && cnt == 1 && n4 <= 4 * kChunk4) {
      // One member (most groups while slot use is spread): its source row and
      // the target row in one round of loads; the same arithmetic as below.
      const int sr = __shfl_sync(FULL, mj.srow, 0);
      const float cj = __shfl_sync(FULL, coef, 0);
      float4 t[4], x[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        t[q] = load_chunk(dst, lane + q * kChunk4, n4);
        x[q] = value ? load_chunk(s.E + (int64_t)sr * d.dv, lane + q * kChunk4, n4)
                     : load_chunk(Qin + (int64_t)sr * d.dh, lane + q * kChunk4, n4);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c4 = lane + q * kChunk4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        fma4(acc, cj, x[q]);
        const float4 nv = updated(d, value, t[q], acc, C);
        if (c4 < n4) *reinterpret_cast<float4 *>(dst + 4 * c4) = nv;
        if (!value && q * kChunk4 < n4)
          resplit_key_chunk(d, s, (int64_t)(g - (uint32_t)d.Nt), q, c4, n4, nv);
      }
    } else if (!value || C > 0.f) {
      for (int cb = 0; cb < n4; cb += 2 * kChunk4) {
        const float4 t0 = load_chunk(dst, cb + lane, n4);
        const float4 t1 = load_chunk(dst, cb + lane + 32, n4);
        float4 acc[2];
        if (value) sum_members<2, 2>(s.E, d.dv, cnt, mj.srow, coef, cb, n4, acc);
        else sum_members<2, 2>(Qin, d.dh, cnt, mj.srow, coef, cb, n4, acc);
        const float4 nv0 = updated(d, value, t0, acc[0], C);
        const float4 nv1 = updated(d, value, t1, acc[1], C);
        if (cb + lane < n4) *reinterpret_cast<float4 *>(dst + 4 * (cb + lane)) = nv0;
        if (cb + lane + 32 < n4) *reinterpret_cast<float4 *>(dst + 4 * (cb + lane + 32)) = nv1;
        if (!value) {
          const int64_t r = (int64_t)(g - (uint32_t)d.Nt);
          resplit_key_chunk(d, s, r, cb / kChunk4, cb + lane, n4, nv0);
          if (cb + kChunk4 < n4) resplit_key_chunk(d, s, r, cb / kChunk4 + 1, cb + lane + 32, n4, nv1);
        }
      }
    }
    if (value && d.lam != 0.f && lane < len) s.pb[mj.id] = entropy_term(d, W);
  }
}

template <typename TQ>
static cudaError_t launch_apply_t(const Dims &d, float *V, float *K, const TQ *Q,
                                  const Scratch &s, cudaStream_t st, int part) {
  static int per_sm = 0;
  if (!per_sm) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_apply<TQ>, kApplyThreads, 0);
    if (per_sm < 1) per_sm = 1;
  }
  return launch_k(d.pdl, k_apply<TQ>, d.sm_count * per_sm, kApplyThreads, 0, st, d, V, K, Q, s,
                  part);
}

cudaError_t launch_apply(const Dims &d, float *V, float *K, const void *Q, int q_dtype,
                         const Scratch &s, cudaStream_t st, int part) {
  if (q_dtype == 1) return launch_apply_t(d, V, K, (const __nv_bfloat16 *)Q, s, st, part);
  return launch_apply_t(d, V, K, (const float *)Q, s, st, part);
}

// ---------------------------------------------------------------------------
// pgrad (lam > 0 only): dL/ds_r = w_r (gamma_r - sum_r' w_r' gamma_r'),
// gamma = dL_mse/dw + dL_addr/dw, then alpha of the token-head's entries.
// Warp per token-head, lane r.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_pgrad(Dims d, Scratch s) {
  griddep_wait();
  griddep_launch();
  if (chunk_aborted(s, 0u)) return;  // an earlier kernel gave up
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
  return launch_k(d.pdl, k_pgrad, (d.M + 7) / 8, 256, 0, st, d, s);
}

}  // namespace fwpkm
