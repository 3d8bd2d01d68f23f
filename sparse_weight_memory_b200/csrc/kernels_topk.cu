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
// One warp per token-head.  Each lane holds n/32 squared distances of a half
// in registers; an MSB-first bisection over the fp32 bit patterns (distances
// are >= 0, so the bit order is the value order) finds the k smallest, which
// are compacted one per lane.  For the merge each lane holds one row of the
// k*k candidate grid and the same bisection, over order-preserving keys of
// the negated scores, picks the k best.
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

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t float_order(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k smallest distances of one half row drow[0..n) (n <= 32*NV), ties by
// index.  Lane r < k returns one winner (distance, index); order unspecified.
template <int NV>
__device__ __forceinline__ void half_topk(const float *__restrict__ drow, int n, int k,
                                          float &d_out, int &i_out, uint2 *wbuf) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NV], idx[NV];
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int i = lane + 32 * v;
    // d >= 0: the bit order is the value order; a used entry never takes the
    // unused marker 0xffffffff, whatever the distance's bits
    key[v] = i < n ? min(__float_as_uint(drow[i]), 0xfffffffeu) : 0xffffffffu;
    idx[v] = (uint32_t)i;
  }
  const uint32_t sel = warp_select_smallest<NV>(key, idx, k);
  uint32_t kk, ii;
  int v_out, src;
  compact_selected<NV>(sel, key, idx, wbuf, kk, ii, v_out, src);
  d_out = __uint_as_float(kk);
  i_out = (int)ii;
}

// kSelectOnly: write only the selection record (x.rec_slots / x.rec_w); no
// pair, entry or bucket outputs.
template <int NV, int KV, bool kSelectOnly>
__global__ void __launch_bounds__(128) k_topk(Dims d, Scratch s, Extras x) {
  __shared__ uint2 wbuf_all[4][32];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int m = blockIdx.x * 4 + wib;  // token-head m = row*H + h
  griddep_wait();
  griddep_launch();
  // a new chunk epoch for the bucket scan that follows (the step, not the selection-only call)
  if (!kSelectOnly && blockIdx.x == 0 && threadIdx.x == 0) s.scan_sync[0] += 1ull;
  if (m >= d.M) return;
  const int row = m / d.H, h = m % d.H;
  const int k = d.k, n = d.n;
  const float eps = d.eps;
  uint2 *wbuf = wbuf_all[wib];
  const float *D1 = s.D + ((int64_t)(h * 2 + 0) * d.rows + row) * n;
  const float *D2 = s.D + ((int64_t)(h * 2 + 1) * d.rows + row) * n;

  // Global token coordinates of this row (for the optional per-token arrays).
  const int b = row / d.Tc, tl = row % d.Tc;
  const int64_t th = ((int64_t)b * d.T + d.t0 + tl) * d.H + h;  // [B][T][H] index

  float s_r = -CUDART_INF_F, d1_r = 0.f, d2_r = 0.f;
  int slot_r = 0, i_r = 0, j_r = 0;
  const bool forced = x.force_mask != nullptr && x.force_mask[th] != 0;
  if (forced) {
    if (lane < k) {
      int64_t sl = x.force_slots[th * k + lane];
      sl = sl < 0 ? 0 : (sl >= d.N ? d.N - 1 : sl);
      slot_r = (int)sl;
      i_r = slot_r / n;
      j_r = slot_r % n;
      d1_r = D1[i_r];
      d2_r = D2[j_r];
      s_r = -logf(eps + d1_r) - logf(eps + d2_r);
    }
  } else {
    float da, db;
    int ia, jb;
    half_topk<NV>(D1, n, k, da, ia, wbuf);
    half_topk<NV>(D2, n, k, db, jb, wbuf);
    const float sa = -logf(eps + da);  // lane a < k: one winner of half 1
    const float sb = -logf(eps + db);  // lane b < k: one winner of half 2
    // Lane a holds row a of the k x k candidate grid: s = sa + sb[b], slot =
    // ia * n + jb[b]; the k best candidates (score desc, slot asc) are the
    // k smallest keys of the negated scores, ties by slot.
    uint32_t key[KV], slot[KV];
#pragma unroll
    for (int b = 0; b < KV; ++b) {
      const float s2 = __shfl_sync(FULL, sb, b);
      const int j2 = __shfl_sync(FULL, jb, b);
      const bool ok = lane < k && b < k;
      key[b] = ok ? float_order(-(sa + s2)) : 0xffffffffu;
      slot[b] = ok ? (uint32_t)(ia * n + j2) : 0xffffffffu;
    }
    const uint32_t sel = warp_select_smallest<KV>(key, slot, k);
    uint32_t wkey, wslot;
    int b_out, a_out;
    compact_selected<KV>(sel, key, slot, wbuf, wkey, wslot, b_out, a_out);
    // winner r (lane r): row a_out of half 1, column b_out of half 2
    const float w_sa = __shfl_sync(FULL, sa, a_out);
    const float w_sb = __shfl_sync(FULL, sb, b_out);
    const float w_d1 = __shfl_sync(FULL, da, a_out);
    const float w_d2 = __shfl_sync(FULL, db, b_out);
    const int w_i = __shfl_sync(FULL, ia, a_out);
    const int w_j = __shfl_sync(FULL, jb, b_out);
    if (lane < k) {
      s_r = w_sa + w_sb;
      slot_r = (int)wslot;
      i_r = w_i;
      j_r = w_j;
      d1_r = w_d1;
      d2_r = w_d2;
    }
  }

  // Softmax over the k selected scores.
  const float smax = warp_max(lane < k ? s_r : -CUDART_INF_F);
  const float ex = lane < k ? expf(s_r - smax) : 0.f;
  const float z = warp_sum(ex);
  const float w = ex / z;

  if (kSelectOnly) {
    if (lane < k) {
      x.rec_slots[th * k + lane] = slot_r;
      x.rec_w[th * k + lane] = w;
    }
    return;
  }
  const int64_t p = (int64_t)m * k + lane;
  if (lane < k) {
    s.pslot[p] = slot_r;
    s.pw[p] = w;
    s.pclaim[p] = atomicAdd(&s.bcnt[slot_r >> d.vshift], 1);  // value bucket
    if (x.rec_slots) {
      x.rec_slots[th * k + lane] = slot_r;
      x.rec_w[th * k + lane] = w;
    }
  }
  // Sub-key entries: one per distinct row of each half among the k pairs.
  const unsigned act = k == 32 ? FULL : ((1u << k) - 1u);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int sub = half == 0 ? i_r : j_r;
    const float dist = half == 0 ? d1_r : d2_r;
    unsigned peers = 0;
    if (lane < k) peers = __match_any_sync(act, sub);
    const bool leader = lane < k && (__ffs(peers) - 1) == lane;
    const unsigned lb = __ballot_sync(FULL, leader);
    if (leader) {
      const int idx = __popc(lb & lanemask_lt());
      const int64_t e = ((int64_t)m * 2 + half) * k + idx;
      s.esub[e] = sub;
      s.emask[e] = peers;
      s.einv[e] = 1.f / (eps + dist);
      s.eclaim[e] = atomicAdd(&s.bcnt[d.NBv + (h * 2 + half) * n + sub], 1);
    }
    // unused entry slots of this half are marked -1
    if (lane >= __popc(lb) && lane < k) s.esub[((int64_t)m * 2 + half) * k + lane] = -1;
    if (lane == 0) s.ecount[(int64_t)m * 2 + half] = __popc(lb);
  }
}

template <int KV, bool kSelectOnly>
static cudaError_t launch_topk_kv(const Dims &d, const Scratch &s, const Extras &x,
                                  cudaStream_t st) {
  const int blocks = (d.M + 3) / 4;
  const int nv = (d.n + 31) / 32;
  if (nv <= 1) return launch_k(d.pdl, k_topk<1, KV, kSelectOnly>, blocks, 128, 0, st, d, s, x);
  if (nv <= 2) return launch_k(d.pdl, k_topk<2, KV, kSelectOnly>, blocks, 128, 0, st, d, s, x);
  if (nv <= 4) return launch_k(d.pdl, k_topk<4, KV, kSelectOnly>, blocks, 128, 0, st, d, s, x);
  if (nv <= 8) return launch_k(d.pdl, k_topk<8, KV, kSelectOnly>, blocks, 128, 0, st, d, s, x);
  if (nv <= 16) return launch_k(d.pdl, k_topk<16, KV, kSelectOnly>, blocks, 128, 0, st, d, s, x);
  if (nv <= 32) return launch_k(d.pdl, k_topk<32, KV, kSelectOnly>, blocks, 128, 0, st, d, s, x);
  return cudaErrorInvalidValue;  // n > 1024: rejected when the state is made
}

template <bool kSelectOnly>
static cudaError_t launch_topk_t(const Dims &d, const Scratch &s, const Extras &x,
                                 cudaStream_t st) {
  if (d.k <= 8) return launch_topk_kv<8, kSelectOnly>(d, s, x, st);
  if (d.k <= 16) return launch_topk_kv<16, kSelectOnly>(d, s, x, st);
  return launch_topk_kv<32, kSelectOnly>(d, s, x, st);
}

cudaError_t launch_topk(const Dims &d, const Scratch &s, const Extras &x, cudaStream_t st) {
  return launch_topk_t<false>(d, s, x, st);
}

cudaError_t launch_topk_select(const Dims &d, const Scratch &s, const Extras &x,
                               cudaStream_t st) {
  return launch_topk_t<true>(d, s, x, st);
}

}  // namespace fwpkm
