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
// scan: bucket offsets (single CTA).  The counts are staged in shared memory
// with coalesced 16-byte loads, each thread scans a contiguous run there, and
// the offsets go back with coalesced stores; pieces of kScanPiece buckets.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 1024;
constexpr int kScanPiece = 8192;

__global__ void __launch_bounds__(kScanThreads) k_bucket_scan(Dims d, Scratch s) {
  griddep_wait();
  griddep_launch();
  __shared__ __align__(16) int cnt[kScanPiece];
  __shared__ int red[32];
  __shared__ int carry_s;
  const int NB = d.NB;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  constexpr int per = kScanPiece / kScanThreads;  // 8 buckets per thread and piece
  int carry = 0;
  for (int p0 = 0; p0 < NB; p0 += kScanPiece) {
    const int np = min(kScanPiece, NB - p0);
    // bcnt and boff are 256-byte aligned; p0 is a multiple of 8192
    for (int i = threadIdx.x * 4; i < np; i += kScanThreads * 4) {
      if (i + 4 <= np) {
        *reinterpret_cast<int4 *>(cnt + i) = *reinterpret_cast<const int4 *>(s.bcnt + p0 + i);
        *reinterpret_cast<int4 *>(s.bcnt + p0 + i) = make_int4(0, 0, 0, 0);  // next chunk
      } else {
        for (int j = i; j < np; ++j) {
          cnt[j] = s.bcnt[p0 + j];
          s.bcnt[p0 + j] = 0;
        }
      }
    }
    __syncthreads();
    const int b0 = threadIdx.x * per;
    int v[per];
    int total = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
      v[i] = b0 + i < np ? cnt[b0 + i] : 0;
      total += v[i];
    }
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
    int run = carry + (w > 0 ? red[w - 1] : 0) + incl - total;
#pragma unroll
    for (int i = 0; i < per; ++i) {
      cnt[b0 + i] = run;  // exclusive offsets, in place
      run += v[i];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < np; i += kScanThreads) s.boff[p0 + i] = cnt[i];
    if (threadIdx.x == 0) {
      if (d.NBv >= p0 && d.NBv < p0 + np) s.meta->Lv = cnt[d.NBv - p0];
      carry_s = carry + red[31];
    }
    __syncthreads();
    carry = carry_s;
  }
  if (threadIdx.x == 0) {
    s.boff[NB] = carry;
    s.meta->L = carry;
    if (d.NBv >= NB) s.meta->Lv = carry;
    s.meta->stat_chunks += 1ull;
    s.meta->pool_next = 0;
    s.meta->nshort = 0;
    s.meta->nlong = 0;
  }
}

cudaError_t launch_scan(const Dims &d, const Scratch &s, cudaStream_t st) {
  return launch_k(d.pdl, k_bucket_scan, 1, kScanThreads, 0, st, d, s);
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

// A record on its way from rec_in to rec.  When the entropy term is off the
// read kernel has already computed every entry's alpha (ealpha): it becomes
// the sub-key record's coefficient here.  With the term on, alpha is known
// only after pgrad and the apply reads it itself.
__device__ __forceinline__ Member fetch_member(const Dims &d, const Scratch &s, const Member *p) {
  Member m = load_member(p);
  if (d.lam == 0.f && m.g >= (uint32_t)d.N) m.coef = m.c0 = s.ealpha[m.id];
  return m;
}

constexpr int kShortMax = 32;  // groups up to this size are applied by one warp
constexpr int kBlock = 32;    // longer groups are applied in blocks of this many members

// Work lists of the apply kernel for a group that starts at position x0:
// a short group goes to shortlist, a longer one to longlist, one entry per
// block of kBlock members.  Thread-level (one call per group head).
__device__ __forceinline__ void list_group(const Scratch &s, int x0, int len) {
  if (len <= kShortMax) {
    s.shortlist[atomicAdd(&s.meta->nshort, 1)] = x0;
  } else {
    const int nb = (len + kBlock - 1) / kBlock;
    const int base = atomicAdd(&s.meta->nlong, nb);
    for (int b = 0; b < nb; ++b) s.longlist[base + b] = x0 + b * kBlock;
  }
}

// CTA-wide sort of one bucket with more than 32 members.
__device__ void sort_big_bucket(const Dims &d, const Scratch &s, int off, int len, bool value,
                                uint32_t gbase, uint64_t *buf, int *nseg) {
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
        list_group(s, off + i, end - first);
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
        list_group(s, off + i, end - first);
      }
    }
  }
  if (my_seg) atomicAdd(nseg, my_seg);
  __syncthreads();
}

__global__ void __launch_bounds__(kSortThreads) k_bucket_sort(Dims d, Scratch s) {
  __shared__ uint64_t buf[kSortCap];
  __shared__ int nseg[2];  // distinct value rows / sub-key rows seen by this CTA
  __shared__ int big_n;
  __shared__ int big_b[kSortWarps * 8];  // large buckets met in phase 1
  griddep_wait();
  griddep_launch();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  if (threadIdx.x < 2) nseg[threadIdx.x] = 0;
  if (threadIdx.x == 0) big_n = 0;
  __syncthreads();
  const int stride = gridDim.x * kSortWarps;
  // phase 1: small buckets, one warp each; large ones are listed.  Bucket b
  // goes to CTA b % gridDim.x: neighbouring buckets (slots of one popular
  // sub-key row) land in different CTAs.
  for (int b = blockIdx.x + gridDim.x * wib; b < d.NB; b += stride) {
    const int off = s.boff[b], len = s.boff[b + 1] - off;
    if (len == 0) continue;
    if (len > 32) {
      if (lane == 0) {
        const int slot = atomicAdd(&big_n, 1);
        if (slot < kSortWarps * 8) big_b[slot] = b;
        else atomicOr(&s.meta->err, ERR_POOL_OVERFLOW);  // cannot happen: see launch_bsort
      }
      continue;
    }
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
    // work lists: short groups, and the blocks of longer ones
    const bool sh = head && glen <= kShortMax;
    const unsigned sb = __ballot_sync(FULL, sh);
    int sbase = 0;
    if (lane == 0 && sb) sbase = atomicAdd(&s.meta->nshort, __popc(sb));
    sbase = __shfl_sync(FULL, sbase, 0);
    if (sh) s.shortlist[sbase + __popc(sb & lanemask_lt())] = off + lane;
    const unsigned lb = __ballot_sync(FULL, head && glen > kShortMax);  // <= 32 members: 1 block
    int lbase = 0;
    if (lane == 0 && lb) lbase = atomicAdd(&s.meta->nlong, __popc(lb));
    lbase = __shfl_sync(FULL, lbase, 0);
    if (head && glen > kShortMax) s.longlist[lbase + __popc(lb & lanemask_lt())] = off + lane;
    if (lane == 0) atomicAdd(&nseg[b < d.NBv ? 0 : 1], __popc(heads));
  }
  __syncthreads();
  // phase 2: the large buckets, each by the whole CTA
  const int nbig = min(big_n, kSortWarps * 8);
  for (int i = 0; i < nbig; ++i) {
    const int b = big_b[i];
    const int off = s.boff[b], len = s.boff[b + 1] - off;
    const bool value = b < d.NBv;
    const uint32_t gbase =
        value ? ((uint32_t)b << d.vshift) : (uint32_t)d.N + (uint32_t)(b - d.NBv);
    sort_big_bucket(d, s, off, len, value, gbase, buf, &nseg[value ? 0 : 1]);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (nseg[0]) atomicAdd(&s.meta->stat_value_rows, (unsigned long long)nseg[0]);
    if (nseg[1]) atomicAdd(&s.meta->stat_key_rows, (unsigned long long)nseg[1]);
  }
}

// Every CTA meets at most 8 buckets per warp (so big_b cannot overflow):
// the grid holds at least NB / (8 * kSortWarps) CTAs.
cudaError_t launch_bsort(const Dims &d, const Scratch &s, cudaStream_t st) {
  static int per_sm = 0;
  if (!per_sm) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_bucket_sort, kSortThreads, 0);
    if (per_sm < 1) per_sm = 1;
  }
  int blocks = (d.NB + kSortWarps - 1) / kSortWarps;
  const int min_blocks = (d.NB + 8 * kSortWarps - 1) / (8 * kSortWarps);
  int cap = d.sm_count * per_sm;
  if (cap < min_blocks) cap = min_blocks;
  if (blocks > cap) blocks = cap;
  return launch_k(d.pdl, k_bucket_sort, blocks, kSortThreads, 0, st, d, s);
}

// ---------------------------------------------------------------------------
// apply: the row updates, from the two work lists bsort wrote.
//   phase A, one CTA per block of up to kBlock members of a longer group: the
//     8 warps each take members m = w, w+8, w+16, w+24 and have all their
//     source rows in flight at once (E rows for value rows, query halves for
//     sub-key rows); the warps' sums are added in warp order.  A one-block
//     group is written at once; otherwise the block publishes a partial and
//     the last block of the group adds the partials in block order.
//   phase B, one warp per group of <= kShortMax members: the lanes hold the
//     records, the members' source rows are summed in member order with a
//     few rows in flight, then the row is written.
// Column blocks of 32 * Q4 float4 bound the registers for any row width.
// Every sum runs in an order fixed by the data, whatever the scheduling.
// ---------------------------------------------------------------------------
constexpr int kApplyThreads = 256;
constexpr int kApplyWarps = kApplyThreads / 32;

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
//   value row : v - (eta / C) * G          (C = sum of w/H)
//   sub-key   : k - 2 eta (G - A k)        (A = sum of alpha)
__device__ __forceinline__ float4 updated(const Dims &d, bool value, const float4 &t,
                                          const float4 &g, float c0) {
  if (value) {
    const float sc = d.eta / c0;
    return make_float4(t.x - sc * g.x, t.y - sc * g.y, t.z - sc * g.z, t.w - sc * g.w);
  }
  const float te = 2.f * d.eta;
  return make_float4(t.x - te * (g.x - c0 * t.x), t.y - te * (g.y - c0 * t.y),
                     t.z - te * (g.z - c0 * t.z), t.w - te * (g.w - c0 * t.w));
}

// Entropy term of a value row: dL_addr/dw = (lam/M)(log pbar + 1) for every
// pair of the group, pbar = (sum of the group's weights) / M.
__device__ __forceinline__ float entropy_term(const Dims &d, float wsum) {
  return (d.lam / (float)d.M) * (logf(wsum / (float)d.M) + 1.f);
}

__device__ __forceinline__ const float *source_row(const Dims &d, const Scratch &s, bool value,
                                                   int srow) {
  return value ? s.E + (int64_t)srow * d.dv : s.Qs + (int64_t)srow * d.dh;
}

template <int Q4>
__global__ void __launch_bounds__(kApplyThreads, 3) k_apply(Dims d, float *__restrict__ V,
                                                         float *__restrict__ K, Scratch s,
                                                         int part) {
  constexpr int CB = 32 * Q4;  // float4 columns per column block
  __shared__ float4 red[kApplyWarps][CB];
  __shared__ int m_srow[kBlock];
  __shared__ float m_coef[kBlock], m_c0[kBlock], m_c1[kBlock];
  __shared__ int m_id[kBlock];
  __shared__ int s_slot, s_last;
  griddep_wait();
  griddep_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool alpha_later = d.lam != 0.f;  // sub-key alphas come from pgrad
  auto wanted = [&](uint32_t g) {         // part 0: all, 1: value rows, 2: sub-key rows
    const bool value = g < (uint32_t)d.N;
    return part == 0 || (part == 1) == value;
  };

  // ---------------- phase A: blocks of longer groups ----------------
  const int nlong = s.meta->nlong;
  for (int it = blockIdx.x; it < nlong; it += gridDim.x) {
    const int x = s.longlist[it];
    const int4 head = *reinterpret_cast<const int4 *>(s.rec + x);  // g, id, srow, gstart
    const uint32_t g = (uint32_t)head.x;
    if (!wanted(g)) continue;
    const int g0 = head.w, len = s.rec[x].glen;
    const int cnt = min(kBlock, g0 + len - x);
    const int nblocks = (len + kBlock - 1) / kBlock;
    const bool value = g < (uint32_t)d.N;
    const int n4 = (value ? d.dv : d.dh) >> 2;
    float *dst = value ? V + (int64_t)g * d.dv : K + (int64_t)(g - (uint32_t)d.N) * d.dh;
    if (tid < cnt) {
      const Member m = load_member(s.rec + x + tid);
      m_srow[tid] = m.srow;
      m_id[tid] = (int)m.id;
      float coef = m.coef, c0 = m.c0;
      if (!value && alpha_later) coef = c0 = s.ealpha[m.id];
      m_coef[tid] = coef;
      m_c0[tid] = c0;
      m_c1[tid] = m.c1;
    }
    if (tid == 0 && nblocks > 1) {
      s_slot = atomicAdd(&s.meta->pool_next, 1);
      if (s_slot >= s.pool_cap) atomicOr(&s.meta->err, ERR_POOL_OVERFLOW);
    }
    __syncthreads();
    float C = 0.f, W = 0.f;  // ordered scalar sums of the block (same in every thread)
    for (int j = 0; j < cnt; ++j) {
      C += m_c0[j];
      W += m_c1[j];
    }
    const int slot = nblocks > 1 ? s_slot : 0;
    const bool slot_ok = nblocks == 1 || slot < s.pool_cap;
    float *part_out = s.partial + (size_t)slot * s.pwidth;
    for (int cb = 0; cb < n4; cb += CB) {
      float4 r[4][Q4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = warp + kApplyWarps * u;
        if (j < cnt) load_row<Q4>(source_row(d, s, value, m_srow[j]), cb, n4, r[u]);
      }
      float4 acc[Q4];
#pragma unroll
      for (int q = 0; q < Q4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = warp + kApplyWarps * u;
        if (j < cnt) {
#pragma unroll
          for (int q = 0; q < Q4; ++q) fma4(acc[q], m_coef[j], r[u][q]);
        }
      }
#pragma unroll
      for (int q = 0; q < Q4; ++q) red[warp][lane + 32 * q] = acc[q];
      __syncthreads();
      if (tid < CB && cb + tid < n4) {
        const int c4 = cb + tid;
        float4 tot = red[0][tid];
#pragma unroll
        for (int w = 1; w < kApplyWarps; ++w) add4(tot, red[w][tid]);
        if (nblocks == 1) {
          if (!value || C > 0.f) {
            const float4 t = *reinterpret_cast<const float4 *>(dst + 4 * c4);
            *reinterpret_cast<float4 *>(dst + 4 * c4) = updated(d, value, t, tot, C);
          }
        } else if (slot_ok) {
          *reinterpret_cast<float4 *>(part_out + 4 + 4 * c4) = tot;
          __threadfence();  // visible before the group's arrival count moves
        }
      }
      __syncthreads();
    }
    if (nblocks == 1) {
      if (value && d.lam != 0.f && tid < cnt) s.pb[m_id[tid]] = entropy_term(d, W);
      __syncthreads();
      continue;
    }
    // longer group: publish the partial; the group's last block combines
    if (tid == 0) {
      if (slot_ok) {
        part_out[0] = C;
        part_out[1] = W;
      }
      s.slotmap[x] = slot_ok ? slot : -1;
      __threadfence();
      s_last = atomicAdd(&s.segcnt[g0], 1) == nblocks - 1;
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      float Ct = 0.f, Wt = 0.f;
      bool all_ok = true;
      for (int b = 0; b < nblocks; ++b) {
        const int sl = __ldcg(&s.slotmap[g0 + b * kBlock]);
        if (sl < 0) {
          all_ok = false;
          continue;
        }
        const float *pp = s.partial + (size_t)sl * s.pwidth;
        Ct += __ldcg(pp);
        Wt += __ldcg(pp + 1);
      }
      for (int c4 = tid; c4 < n4 && all_ok; c4 += blockDim.x) {
        float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int b = 0; b < nblocks; ++b) {
          const float *pp =
              s.partial + (size_t)__ldcg(&s.slotmap[g0 + b * kBlock]) * s.pwidth;
          add4(tot, __ldcg(reinterpret_cast<const float4 *>(pp + 4 + 4 * c4)));
        }
        if (!value || Ct > 0.f) {
          const float4 t = *reinterpret_cast<const float4 *>(dst + 4 * c4);
          *reinterpret_cast<float4 *>(dst + 4 * c4) = updated(d, value, t, tot, Ct);
        }
      }
      if (value && d.lam != 0.f && all_ok) {
        const float bt = entropy_term(d, Wt);
        for (int j = tid; j < len; j += blockDim.x) s.pb[s.rec[g0 + j].id] = bt;
      }
      if (tid == 0) s.segcnt[g0] = 0;  // ready for the next chunk
    }
    __syncthreads();
  }

  // ---------------- phase B: groups of <= kShortMax members, a warp each ----------------
  // Lane j holds member j's record; the members' rows are summed in member
  // order, kU rows in flight, for every column block of the target row.
  constexpr int kU = 4;
  const int nshort = s.meta->nshort;
  for (int it = blockIdx.x * kApplyWarps + warp; it < nshort; it += gridDim.x * kApplyWarps) {
    const int x = s.shortlist[it];
    Member mj{};
    if ((int64_t)x + lane < s.Lcap) mj = load_member(s.rec + x + lane);  // past the group: unused
    const uint32_t g = __shfl_sync(FULL, mj.g, 0);
    const int len = __shfl_sync(FULL, mj.glen, 0);
    if (!wanted(g)) continue;
    const bool value = g < (uint32_t)d.N;
    float coef = 0.f, c0 = 0.f, c1 = 0.f;
    if (lane < len) {
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
    const int n4 = (value ? d.dv : d.dh) >> 2;
    float *dst = value ? V + (int64_t)g * d.dv : K + (int64_t)(g - (uint32_t)d.N) * d.dh;
    const bool write = !value || C > 0.f;
    for (int cb = 0; cb < n4 && write; cb += CB) {
      float4 t[Q4], acc[Q4];
      load_row<Q4>(dst, cb, n4, t);
#pragma unroll
      for (int q = 0; q < Q4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j0 = 0; j0 < len; j0 += kU) {
        float4 r[kU][Q4];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int sr = __shfl_sync(FULL, mj.srow, (j0 + u) & 31);
          if (j0 + u < len) load_row<Q4>(source_row(d, s, value, sr), cb, n4, r[u]);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const float cj = __shfl_sync(FULL, coef, (j0 + u) & 31);
          if (j0 + u < len) {
#pragma unroll
            for (int q = 0; q < Q4; ++q) fma4(acc[q], cj, r[u][q]);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < Q4; ++q) {
        const int c4 = cb + lane + 32 * q;
        if (c4 < n4) *reinterpret_cast<float4 *>(dst + 4 * c4) = updated(d, value, t[q], acc[q], C);
      }
    }
    if (value && d.lam != 0.f && lane < len) s.pb[mj.id] = entropy_term(d, W);
  }
}

template <int Q4>
static cudaError_t launch_apply_t(const Dims &d, float *V, float *K, const Scratch &s,
                                  cudaStream_t st, int part) {
  static int per_sm = 0;
  if (!per_sm) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_apply<Q4>, kApplyThreads, 0);
    if (per_sm < 1) per_sm = 1;
  }
  return launch_k(d.pdl, k_apply<Q4>, d.sm_count * per_sm, kApplyThreads, 0, st, d, V, K, s,
                  part);
}

cudaError_t launch_apply(const Dims &d, float *V, float *K, const Scratch &s, cudaStream_t st,
                         int part) {
  // rows up to 128 floats in one column block; wider rows in blocks of 256
  // (2 float4 per lane keeps kU source rows in flight without spilling)
  const int w4 = ((d.dv > d.dh ? d.dv : d.dh) / 4 + 31) / 32;
  if (w4 <= 1) return launch_apply_t<1>(d, V, K, s, st, part);
  return launch_apply_t<2>(d, V, K, s, st, part);
}

// ---------------------------------------------------------------------------
// pgrad (lam > 0 only): dL/ds_r = w_r (gamma_r - sum_r' w_r' gamma_r'),
// gamma = dL_mse/dw + dL_addr/dw, then alpha of the token-head's entries.
// Warp per token-head, lane r.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_pgrad(Dims d, Scratch s) {
  griddep_wait();
  griddep_launch();
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
