// kernels_topk.cu -- product-key selection per token-head.
//
// Product Key Memory addressing (gist.science "Fast-weight Product Key
// Memory", section 2, Core Architecture; agifrontier tutorial, Cartesian
// product addressing): the top-k sub-keys of each query half are found
// separately, then the k*k Cartesian candidates (score s1(i) + s2(j), slot
// i*n + j) are merged to the top-k slots, which equals the top-k over all
// N = n^2 slots.  Weights are the softmax of the selected slot scores.
// Order: score descending, index ascending on ties.
//
// Two warps per token-head, one per half.  Each lane holds n/32 squared
// distances of its half in registers; an MSB-first bisection over the fp32
// bit patterns (distances are >= 0, so the bit order is the value order)
// finds the k smallest, which are compacted one per lane and sorted by
// (score desc, index asc).  The merge then searches only the candidates
// (a, b) of half-1 rank a and half-2 rank b with (a+1)(b+1) <= k, with the
// same bisection over order-preserving keys of the negated scores; an exact
// score tie with a candidate outside that set sends the token-head through
// the full k*k merge, so the result is exactly the top-k under (score desc,
// slot asc).
#include <math_constants.h>

#include "fwpkm_internal.cuh"

namespace fwpkm {

// Number of keys strictly below t across the warp.
template <int NV>
__device__ __forceinline__ int count_lt(const uint32_t (&key)[NV], uint32_t t) {
  int c = 0;
#pragma unroll
  for (int v = 0; v < NV; ++v) c += key[v] < t ? 1 : 0;
  return __reduce_add_sync(FULL, c);
}

// Marks the k smallest keys held across the warp (NV per lane; an unused
// entry holds 0xffffffff and there are at least k used ones).  Equal keys at
// the boundary are taken in increasing `tie` order (tie values are unique).
// Returns this lane's selection as a bit mask over v (so NV <= 32: n <= 1024).
//
// MSB-first bisection over the key bits: t grows one bit at a time while
// fewer than k keys lie below it; it stops early once exactly k do.
template <int NV>
__device__ uint32_t warp_select_smallest(const uint32_t (&key)[NV], const uint32_t (&tie)[NV],
                                         int k) {
  static_assert(NV <= 32, "the selection is one bit per register entry of a 32-bit mask");
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    if (key[v] != 0xffffffffu) {
      kmin = min(kmin, key[v]);
      kmax = max(kmax, key[v]);
    }
  }
  kmin = __reduce_min_sync(FULL, kmin);
  kmax = __reduce_max_sync(FULL, kmax);
  uint32_t kstar = kmin;  // the k-th smallest key unless `exact`
  if (kmin != kmax) {
    const int hb = 31 - __clz(kmin ^ kmax);
    kstar = kmin & ~((2u << hb) - 1u);  // common prefix; every key >= kstar
    for (int bit = hb; bit >= 0; --bit) {
      const uint32_t t = kstar | (1u << bit);
      const int c = count_lt<NV>(key, t);
      if (c == k) {  // exactly k keys below t: done, no tie to break
        uint32_t sel = 0;
#pragma unroll
        for (int v = 0; v < NV; ++v) sel |= (key[v] < t ? 1u : 0u) << v;
        return sel;
      }
      if (c < k) kstar = t;
    }
  }
  uint32_t sel = 0, tied = 0;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    sel |= (key[v] < kstar ? 1u : 0u) << v;
    tied |= (key[v] == kstar ? 1u : 0u) << v;
  }
  // the remaining places go to the tied keys with the smallest tie values
  for (int need = k - __reduce_add_sync(FULL, __popc(sel)); need > 0; --need) {
    uint32_t best = 0xffffffffu;
#pragma unroll
    for (int v = 0; v < NV; ++v)
      if ((tied >> v) & 1u) best = min(best, tie[v]);
    const uint32_t win = __reduce_min_sync(FULL, best);
#pragma unroll
    for (int v = 0; v < NV; ++v)
      if (((tied >> v) & 1u) && tie[v] == win) {
        sel |= 1u << v;
        tied &= ~(1u << v);
      }
  }
  return sel;
}

// Lane r < (number selected) receives the r-th selected entry, in (v, lane)
// order: its value a[v], b[v] and its v.
template <int NV>
__device__ __forceinline__ void compact_selected(uint32_t sel, const uint32_t (&a)[NV],
                                                 const uint32_t (&b)[NV], uint2 *wbuf,
                                                 uint32_t &a_out, uint32_t &b_out,
                                                 int &v_out, int &src_lane) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = lanemask_lt();
  int base = 0;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const bool on = (sel >> v) & 1u;
    const unsigned sb = __ballot_sync(FULL, on);
    if (on) wbuf[base + __popc(sb & lt)] = make_uint2((uint32_t)(v << 5 | lane), 0u);
    base += __popc(sb);
  }
  __syncwarp();
  const uint32_t where = lane < base ? wbuf[lane].x : 0u;
  __syncwarp();
  v_out = (int)(where >> 5);
  src_lane = (int)(where & 31u);
  // fetch the values from the lane that holds them (all lanes take part)
  a_out = 0;
  b_out = 0;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const uint32_t av = __shfl_sync(FULL, a[v], src_lane);
    const uint32_t bv = __shfl_sync(FULL, b[v], src_lane);
    if (v == v_out) {
      a_out = av;
      b_out = bv;
    }
  }
}

// Order-preserving map of a float to an unsigned key (larger float, larger
// key), and its inverse on the bits.
__device__ __forceinline__ uint32_t float_order(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint32_t float_unorder(uint32_t u) {
  return (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
}

// Top-k smallest distances of one half row drow[0..n) (n <= 32*NV), ties by
// index.  Lane r < k returns one winner (distance, index); order unspecified.
// wbuf holds 64 entries.  kSgn: the values may be negative (the negated dot
// products of the dot-product score), so they are keyed by float_order.
//
// With 4 or more entries per lane the search is narrowed first: every lane
// offers its two smallest keys, and the k-th smallest t0 of those 64 is at
// least the k-th smallest of the whole row (they are a subset of it).  So the
// top-k are among the keys <= t0 -- about 1.5k of them for continuous data --
// which are gathered two per lane and selected exactly.  Past 64 such keys
// (heavy ties) the whole row is searched instead.  Either way the result is
// the exact top-k under (key asc, index asc).
template <int NV, bool kSgn>
__device__ __forceinline__ void half_topk(const float *__restrict__ drow, int n, int k,
                                          float &d_out, int &i_out, uint2 *wbuf) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NV], idx[NV];
  // d >= 0: the bit order is the value order; a used entry never takes the
  // unused marker 0xffffffff, whatever the distance's bits.  Rows of a length
  // that is a multiple of 4 are read 16 bytes a lane (entry v of the lane is
  // i = 128 (v / 4) + 4 lane + v % 4); the selection depends only on the set
  // of (key, index) pairs, not on which lane holds which.
  if (NV % 4 == 0 && (n & 3) == 0) {
#pragma unroll
    for (int q = 0; q < NV / 4; ++q) {
      const int i0 = 128 * q + 4 * lane;
      const float4 f = i0 < n ? *reinterpret_cast<const float4 *>(drow + i0)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        key[4 * q + c] = i0 < n ? min(kSgn ? float_order(fv[c]) : __float_as_uint(fv[c]),
                                      0xfffffffeu)
                                : 0xffffffffu;
        idx[4 * q + c] = (uint32_t)(i0 + c);
      }
    }
  } else {
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int i = lane + 32 * v;
      const float dv = i < n ? drow[i] : 0.f;
      key[v] = i < n ? min(kSgn ? float_order(dv) : __float_as_uint(dv), 0xfffffffeu)
                     : 0xffffffffu;
      idx[v] = (uint32_t)i;
    }
  }
  uint32_t kk, ii;
  int v_out, src;
  if (NV >= 4) {
    // the two smallest keys of this lane (n > 96: every lane has two)
    uint32_t m1 = 0xffffffffu, m2 = 0xffffffffu;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const uint32_t x = key[v];
      m2 = min(m2, max(m1, x));
      m1 = min(m1, x);
    }
    const uint32_t pk[2] = {m1, m2};
    const uint32_t pt[2] = {(uint32_t)lane, (uint32_t)lane + 32u};
    const uint32_t psel = warp_select_smallest<2>(pk, pt, k);
    const uint32_t t0 = __reduce_max_sync(
        FULL, max((psel & 1u) ? m1 : 0u, (psel & 2u) ? m2 : 0u));
    // gather the keys <= t0, up to 64, in (lane, v) order
    int cnt = 0;
#pragma unroll
    for (int v = 0; v < NV; ++v) cnt += key[v] <= t0 ? 1 : 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += t;
    }
    const int total = __shfl_sync(FULL, incl, 31);
    if (total <= 64) {
      int pos = incl - cnt;
#pragma unroll
      for (int v = 0; v < NV; ++v)
        if (key[v] <= t0) wbuf[pos++] = make_uint2(key[v], idx[v]);
      __syncwarp();
      uint32_t ck[2], ci[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int c = lane + 32 * q;
        const uint2 e = c < total ? wbuf[c] : make_uint2(0xffffffffu, 0xffffffffu);
        ck[q] = e.x;
        ci[q] = e.y;
      }
      __syncwarp();
      const uint32_t sel = warp_select_smallest<2>(ck, ci, k);
      compact_selected<2>(sel, ck, ci, wbuf, kk, ii, v_out, src);
      d_out = __uint_as_float(kSgn ? float_unorder(kk) : kk);
      i_out = (int)ii;
      return;
    }
  }
  const uint32_t sel = warp_select_smallest<NV>(key, idx, k);
  compact_selected<NV>(sel, key, idx, wbuf, kk, ii, v_out, src);
  d_out = __uint_as_float(kSgn ? float_unorder(kk) : kk);
  i_out = (int)ii;
}

// Bitonic sort of one 64-bit key per lane, ascending across the warp; `src`
// follows each key to the lane it came from.
__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int o) {
  const uint32_t lo = __shfl_xor_sync(FULL, (uint32_t)v, o);
  const uint32_t hi = __shfl_xor_sync(FULL, (uint32_t)(v >> 32), o);
  return ((uint64_t)hi << 32) | lo;
}
__device__ __forceinline__ uint64_t warp_sort_asc(uint64_t key, int &src) {
  const int lane = threadIdx.x & 31;
  src = lane;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int st = size >> 1; st > 0; st >>= 1) {
      const uint64_t ok = shfl_xor64(key, st);
      const int os = __shfl_xor_sync(FULL, src, st);
      const bool up = (lane & size) == 0;
      const bool lower = (lane & st) == 0;
      const bool keep = (lower == up) ? (key <= ok) : (key >= ok);
      if (!keep) {
        key = ok;
        src = os;
      }
    }
  }
  return key;
}

// Candidates of the merge: with both halves' winners sorted by (score desc,
// index asc), rank a of half 1 and rank b of half 2, every candidate (a, b)
// of the top-k has (a+1)(b+1) <= k -- the (a+1)(b+1) - 1 candidates it
// dominates rank ahead of it -- so only that staircase (130 candidates for
// k = 32, instead of k^2 = 1024) is searched.  Per token-head, at most
// kMergeV candidates per lane.
constexpr int kMergeV = 5;
constexpr int kTopkHeads = 4;  // token-heads per CTA, two warps each

// Per-CTA shared memory of the selection.
struct TopkSmem {
  float s[kTopkHeads][2][32];     // winners of each half, sorted: score,
  float dist[kTopkHeads][2][32];  //   distance,
  int idx[kTopkHeads][2][32];     //   sub-key row
  int fin[kTopkHeads][2][32];     // final pairs: sub-key row of each half,
  float find[kTopkHeads][2][32];  //   and its distance
  uint2 wbuf[2 * kTopkHeads][64];
  uint16_t cand[kMergeV * 32];    // staircase candidates, (a << 8) | b
  int ncand;
};

// kSelectOnly: write only the selection record (x.rec_slots / x.rec_w); no
// pair, entry or bucket outputs.
//
// CTA = kTopkHeads token-heads, two warps each: warp 2t + half selects the
// top-k of its half and sorts them; warp 2t merges; then each warp writes
// its half's sub-key entries.  A token-head whose selection is forced reads
// the given slots instead.
template <int NV, int KV, bool kSelectOnly, bool kDot>
__global__ void __launch_bounds__(64 * kTopkHeads) k_topk(Dims d, Scratch s, Extras x) {
  __shared__ TopkSmem sm;
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int t = wib >> 1, half = wib & 1;
  const int m = blockIdx.x * kTopkHeads + t;  // token-head m = row*H + h
  const int k = d.k, n = d.n;
  const float eps = d.eps;
  constexpr bool dot = kDot;  // D = -q.K: the score is -D, ds/dK = q
  // the staircase for this k (warp 0, before the halves are selected)
  if (wib == 0) {
    const int len = lane < k ? min(k, k / (lane + 1)) : 0;
    int incl = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += v;
    }
    for (int b = 0; b < len; ++b) sm.cand[incl - len + b] = (uint16_t)((lane << 8) | b);
    if (lane == 31) sm.ncand = incl;
  }
  griddep_wait();
  griddep_launch();
  // a new chunk epoch for the bucket scan that follows (the step, not the selection-only call)
  // (and an empty list of large buckets, which the scan fills)
  if (!kSelectOnly && blockIdx.x == 0 && threadIdx.x == 0) {
    s.scan_sync[0] += 1ull;
    s.meta->nbig = 0;
  }
  const bool valid = m < d.M;
  const int row = valid ? m / d.H : 0, h = valid ? m % d.H : 0;
  const int lrow = lrow_of(d, row), mb = mem_of(d, row);  // layout row, memory
  const int64_t slot0 = (int64_t)mb * d.N;                // the memory's first value row
  const float *D1 = s.D + ((int64_t)(h * 2 + 0) * d.drows + lrow) * n;
  const float *D2 = s.D + ((int64_t)(h * 2 + 1) * d.drows + lrow) * n;

  // Global token coordinates of this row (for the optional per-token arrays).
  const int b = row / d.Tc, tl = row % d.Tc;
  const int64_t th = ((int64_t)b * d.T + d.t0 + tl) * d.H + h;  // [B][T][H] index
  const bool forced = valid && x.force_mask != nullptr && x.force_mask[th] != 0;

  // ---- each half: top-k, sorted by (score desc, index asc) ----
  if (valid && !forced) {
    float dw;
    int iw;
    half_topk<NV, kDot>(half == 0 ? D1 : D2, n, k, dw, iw, sm.wbuf[wib]);
    const float sw = dot ? -dw : -logf(eps + dw);
    const uint64_t key =
        lane < k ? ((uint64_t)float_order(-sw) << 32) | (uint32_t)iw : ~0ull;
    int src;
    const uint64_t sk = warp_sort_asc(key, src);
    const float s_sorted = __shfl_sync(FULL, sw, src);
    const float d_sorted = __shfl_sync(FULL, dw, src);
    if (lane < k) {
      sm.s[t][half][lane] = s_sorted;
      sm.dist[t][half][lane] = d_sorted;
      sm.idx[t][half][lane] = (int)(uint32_t)sk;
    }
  }
  __syncthreads();

  // ---- merge (warp 2t) ----
  float s_r = -CUDART_INF_F;
  int vclaim = -1;  // this lane's value-bucket claim (merge warps, lane < k)
  int slot_r = 0;
  if (valid && half == 0) {
    int i_r = 0, j_r = 0;
    float d1_r = 0.f, d2_r = 0.f;
    if (forced) {
      if (lane < k) {
        int64_t sl = x.force_slots[th * k + lane];  // a slot of the token's memory
        sl = sl < 0 ? 0 : (sl >= d.N ? d.N - 1 : sl);
        i_r = (int)sl / n;
        j_r = (int)sl % n;
        slot_r = (int)(slot0 + sl);
        d1_r = D1[i_r];
        d2_r = D2[j_r];
        s_r = dot ? -d1_r - d2_r : -logf(eps + d1_r) - logf(eps + d2_r);
      }
    } else {
      const float *S1 = sm.s[t][0], *S2 = sm.s[t][1];
      const int *I1 = sm.idx[t][0], *I2 = sm.idx[t][1];
      const int nc = sm.ncand;
      uint32_t key[kMergeV], slot[kMergeV];
#pragma unroll
      for (int v = 0; v < kMergeV; ++v) {
        const int c = lane + 32 * v;
        key[v] = slot[v] = 0xffffffffu;
        if (c < nc) {
          const int a = sm.cand[c] >> 8, bb = sm.cand[c] & 255;
          key[v] = float_order(-(S1[a] + S2[bb]));
          slot[v] = (uint32_t)(I1[a] * n + I2[bb]);
        }
      }
      const uint32_t sel = warp_select_smallest<kMergeV>(key, slot, k);
      uint32_t wkey, wslot;
      int v_out, src;
      compact_selected<kMergeV>(sel, key, slot, sm.wbuf[wib], wkey, wslot, v_out, src);
      // An exact tie of an outside candidate with the k-th score could change
      // which equal-score slot wins the last places: take the full k x k merge.
      const uint32_t kth = __reduce_max_sync(FULL, lane < k ? wkey : 0u);
      // Only the first outside candidate of each rank a can tie: the ones after
      // it score no higher (S2 descends, and a rounded sum is monotone in each
      // term), and none scores above the k-th, which dominates it.
      const int b0 = lane < k ? k / (lane + 1) : k;
      const bool tie = b0 < k && float_order(-(S1[lane] + S2[b0])) == kth;
      if (__any_sync(FULL, tie)) {
        uint32_t fkey[KV], fslot[KV];
        const float sa = lane < k ? S1[lane] : 0.f;
        const int ia = lane < k ? I1[lane] : 0;
#pragma unroll
        for (int bb = 0; bb < KV; ++bb) {
          const bool ok = lane < k && bb < k;
          fkey[bb] = ok ? float_order(-(sa + S2[bb])) : 0xffffffffu;
          fslot[bb] = ok ? (uint32_t)(ia * n + I2[bb]) : 0xffffffffu;
        }
        const uint32_t fsel = warp_select_smallest<KV>(fkey, fslot, k);
        int b_out, a_out;
        compact_selected<KV>(fsel, fkey, fslot, sm.wbuf[wib], wkey, wslot, b_out, a_out);
        if (lane < k) {
          i_r = I1[a_out];
          j_r = I2[b_out];
          s_r = S1[a_out] + S2[b_out];
          d1_r = sm.dist[t][0][a_out];
          d2_r = sm.dist[t][1][b_out];
          slot_r = (int)wslot;
        }
      } else if (lane < k) {
        const int c = src + 32 * v_out;
        const int a = sm.cand[c] >> 8, bb = sm.cand[c] & 255;
        i_r = I1[a];
        j_r = I2[bb];
        s_r = S1[a] + S2[bb];
        d1_r = sm.dist[t][0][a];
        d2_r = sm.dist[t][1][bb];
        slot_r = (int)wslot;
      }
      slot_r += (int)slot0;  // the selection is within the memory; pairs carry the global row
    }
    if (lane < k) {
      sm.fin[t][0][lane] = i_r;
      sm.fin[t][1][lane] = j_r;
      sm.find[t][0][lane] = d1_r;
      sm.find[t][1][lane] = d2_r;
    }
    // Softmax over the k selected scores.
    const float smax = warp_max(lane < k ? s_r : -CUDART_INF_F);
    const float ex = lane < k ? expf(s_r - smax) : 0.f;
    const float z = warp_sum(ex);
    const float w = ex / z;
    if (kSelectOnly) {
      if (lane < k) {
        x.rec_slots[th * k + lane] = slot_r - (int)slot0;
        x.rec_w[th * k + lane] = w;
      }
    } else {
      const int64_t p = (int64_t)m * k + lane;
      if (lane < k) {
        s.pslot[p] = slot_r;
        s.pw[p] = w;
        // the value bucket's claim; stored at the end, so that its round trip
        // overlaps the entries' claims
        if (!d.readonly) vclaim = atomicAdd(&s.bcnt[slot_r >> d.vshift], 1);
        if (x.rec_slots) {
          x.rec_slots[th * k + lane] = slot_r - (int)slot0;
          x.rec_w[th * k + lane] = w;
        }
      }
    }
  }
  if (kSelectOnly || d.readonly) return;  // no write follows: no entries
  __syncthreads();

  // ---- sub-key entries of this warp's half: one per distinct row among the
  // k pairs ----
  if (!valid) return;
  const int sub = lane < k ? sm.fin[t][half][lane] : 0;
  const float dist = lane < k ? sm.find[t][half][lane] : 0.f;
  const unsigned act = k == 32 ? FULL : ((1u << k) - 1u);
  unsigned peers = 0;
  if (lane < k) peers = __match_any_sync(act, sub);
  const bool leader = lane < k && (__ffs(peers) - 1) == lane;
  const unsigned lb = __ballot_sync(FULL, leader);
  if (leader) {
    const int idx = __popc(lb & lanemask_lt());
    const int64_t e = ((int64_t)m * 2 + half) * k + idx;
    s.esub[e] = sub;
    s.emask[e] = peers;
    s.einv[e] = dot ? 1.f : 1.f / (eps + dist);
    s.eclaim[e] = atomicAdd(&s.bcnt[d.NBv + ((mb * d.H + h) * 2 + half) * n + sub], 1);
  }
  // unused entry slots of this half are marked -1
  if (lane >= __popc(lb) && lane < k) s.esub[((int64_t)m * 2 + half) * k + lane] = -1;
  if (lane == 0) s.ecount[(int64_t)m * 2 + half] = __popc(lb);
  if (vclaim >= 0) s.pclaim[(int64_t)m * k + lane] = vclaim;
}

template <int KV, bool kSelectOnly, bool kDot>
static cudaError_t launch_topk_kv(const Dims &d, const Scratch &s, const Extras &x,
                                  cudaStream_t st) {
  const int blocks = (d.M + kTopkHeads - 1) / kTopkHeads;
  const int nv = (d.n + 31) / 32;
  const int th = 64 * kTopkHeads;
  if (nv <= 1)
    return launch_k(d.pdl, k_topk<1, KV, kSelectOnly, kDot>, blocks, th, 0, st, d, s, x);
  if (nv <= 2)
    return launch_k(d.pdl, k_topk<2, KV, kSelectOnly, kDot>, blocks, th, 0, st, d, s, x);
  if (nv <= 4)
    return launch_k(d.pdl, k_topk<4, KV, kSelectOnly, kDot>, blocks, th, 0, st, d, s, x);
  if (nv <= 8)
    return launch_k(d.pdl, k_topk<8, KV, kSelectOnly, kDot>, blocks, th, 0, st, d, s, x);
  if (nv <= 16)
    return launch_k(d.pdl, k_topk<16, KV, kSelectOnly, kDot>, blocks, th, 0, st, d, s, x);
  if (nv <= 32)
    return launch_k(d.pdl, k_topk<32, KV, kSelectOnly, kDot>, blocks, th, 0, st, d, s, x);
  return cudaErrorInvalidValue;  // n > 1024: rejected when the state is made
}

template <bool kSelectOnly>
static cudaError_t launch_topk_t(const Dims &d, const Scratch &s, const Extras &x,
                                 cudaStream_t st) {
  if (d.score_dot) {
    if (d.k <= 8) return launch_topk_kv<8, kSelectOnly, true>(d, s, x, st);
    if (d.k <= 16) return launch_topk_kv<16, kSelectOnly, true>(d, s, x, st);
    return launch_topk_kv<32, kSelectOnly, true>(d, s, x, st);
  }
  if (d.k <= 8) return launch_topk_kv<8, kSelectOnly, false>(d, s, x, st);
  if (d.k <= 16) return launch_topk_kv<16, kSelectOnly, false>(d, s, x, st);
  return launch_topk_kv<32, kSelectOnly, false>(d, s, x, st);
}

cudaError_t launch_topk(const Dims &d, const Scratch &s, const Extras &x, cudaStream_t st) {
  return launch_topk_t<false>(d, s, x, st);
}

cudaError_t launch_topk_select(const Dims &d, const Scratch &s, const Extras &x,
                               cudaStream_t st) {
  return launch_topk_t<true>(d, s, x, st);
}

}  // namespace fwpkm
