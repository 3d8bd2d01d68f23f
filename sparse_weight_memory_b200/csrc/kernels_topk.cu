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
// are >= 0, so the bit order is the value order) finds the k-th smallest
// distance; the k winners are sorted in registers (bitonic across lanes), and
// a frontier merge (one pointer per half-1 rank) extracts the top-k of the
// k*k grid in k rounds of a warp arg-max.
#include <math_constants.h>

#include "fwpkm_internal.cuh"

namespace fwpkm {

// Number of keys (distances) strictly below t across the warp.
template <int NV>
__device__ __forceinline__ int count_lt(const uint32_t (&key)[NV], uint32_t t) {
  int c = 0;
#pragma unroll
  for (int v = 0; v < NV; ++v) c += key[v] < t ? 1 : 0;
  return __reduce_add_sync(FULL, c);
}

// Top-k smallest of the row `drow[0..n)` (n <= 32*NV) under (distance asc,
// index asc).  Lane r < k returns the r-th best (distance, index).
template <int NV>
__device__ void half_topk(const float *__restrict__ drow, int n, int k, float &d_out,
                          int &i_out, uint2 *wbuf) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NV];
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    int idx = lane + 32 * v;
    key[v] = idx < n ? __float_as_uint(drow[idx]) : 0xffffffffu;
  }
  // Range of the real keys (padding lanes hold the largest key and never win).
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    if (lane + 32 * v < n) {
      kmin = min(kmin, key[v]);
      kmax = max(kmax, key[v]);
    }
  }
  kmin = __reduce_min_sync(FULL, kmin);
  kmax = __reduce_max_sync(FULL, kmax);

  // kstar: the k-th smallest key, or `thr` with exactly k keys below it.
  uint32_t kstar = kmin;
  bool exact = false;
  uint32_t thr = 0;
  if (kmin != kmax) {
    const int hb = 31 - __clz(kmin ^ kmax);
    kstar = kmin & ~((2u << hb) - 1u);  // common prefix; every key >= kstar
    for (int bit = hb; bit >= 0; --bit) {
      const uint32_t t = kstar | (1u << bit);
      const int c = count_lt<NV>(key, t);
      if (c == k) {
        exact = true;
        thr = t;
        break;
      }
      if (c < k) kstar = t;
    }
  }
  // Compact the winners into wbuf (warp-private) in index order.
  int need_ties = 0;
  if (!exact) need_ties = k - count_lt<NV>(key, kstar);
  int base = 0, ties_seen = 0;
  const unsigned lt = lanemask_lt();
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    bool sel;
    if (exact) {
      sel = key[v] < thr;
    } else {
      const bool tie = key[v] == kstar;
      const unsigned tb = __ballot_sync(FULL, tie);
      const int rank = ties_seen + __popc(tb & lt);
      ties_seen += __popc(tb);
      sel = key[v] < kstar || (tie && rank < need_ties);
    }
    const unsigned sb = __ballot_sync(FULL, sel);
    if (sel) wbuf[base + __popc(sb & lt)] = make_uint2(key[v], (uint32_t)(lane + 32 * v));
    base += __popc(sb);
  }
  __syncwarp();
  uint32_t kk = 0xffffffffu, ki = 0xffffffffu;
  if (lane < k) {
    uint2 e = wbuf[lane];
    kk = e.x;
    ki = e.y;
  }
  __syncwarp();
  // Bitonic sort of the 32 lanes by (key asc, index asc).
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint32_t ok = __shfl_xor_sync(FULL, kk, stride);
      const uint32_t oi = __shfl_xor_sync(FULL, ki, stride);
      const bool up = (lane & size) == 0 || size == 32;
      const bool lower = (lane & stride) == 0;
      const bool mine_less = kk < ok || (kk == ok && ki < oi);
      const bool keep = (lower == up) ? mine_less : !mine_less;
      if (!keep) {
        kk = ok;
        ki = oi;
      }
    }
  }
  d_out = __uint_as_float(kk);
  i_out = (int)ki;
}

// kSelectOnly: write only the selection record (x.rec_slots / x.rec_w); no
// pair, entry or bucket outputs.
template <int NV, bool kSelectOnly>
__global__ void __launch_bounds__(128) k_topk(Dims d, Scratch s, Extras x) {
  __shared__ uint2 wbuf_all[4][32];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int m = blockIdx.x * 4 + wib;  // token-head m = row*H + h
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
    const float sa = -logf(eps + da);  // lane a: a-th best of half 1
    const float sb = -logf(eps + db);  // lane b: b-th best of half 2
    // Frontier merge: lane a (< k) walks its row (a, 0), (a, 1), ...
    int ptr = 0;
    for (int r = 0; r < k; ++r) {
      const int src = ptr < 32 ? ptr : 31;
      const float s2p = __shfl_sync(FULL, sb, src);
      const int j2p = __shfl_sync(FULL, jb, src);
      float cs = (lane < k && ptr < k) ? sa + s2p : -CUDART_INF_F;
      int cslot = (lane < k && ptr < k) ? ia * n + j2p : 0x7fffffff;
      int clane = lane;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float os = __shfl_xor_sync(FULL, cs, o);
        const int oslot = __shfl_xor_sync(FULL, cslot, o);
        const int olane = __shfl_xor_sync(FULL, clane, o);
        if (os > cs || (os == cs && oslot < cslot)) {
          cs = os;
          cslot = oslot;
          clane = olane;
        }
      }
      const int wptr = __shfl_sync(FULL, ptr, clane);
      const float wd1 = __shfl_sync(FULL, da, clane);
      const int wi = __shfl_sync(FULL, ia, clane);
      const float wd2 = __shfl_sync(FULL, db, wptr);
      const int wj = __shfl_sync(FULL, jb, wptr);
      if (lane == r) {
        s_r = cs;
        slot_r = cslot;
        i_r = wi;
        j_r = wj;
        d1_r = wd1;
        d2_r = wd2;
      }
      if (lane == clane) ++ptr;
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
    if (lane == 0) s.ecount[(int64_t)m * 2 + half] = __popc(lb);
  }
}

template <bool kSelectOnly>
static cudaError_t launch_topk_t(const Dims &d, const Scratch &s, const Extras &x,
                                 cudaStream_t st) {
  const int blocks = (d.M + 3) / 4;
  const int nv = (d.n + 31) / 32;
  if (nv <= 1) k_topk<1, kSelectOnly><<<blocks, 128, 0, st>>>(d, s, x);
  else if (nv <= 2) k_topk<2, kSelectOnly><<<blocks, 128, 0, st>>>(d, s, x);
  else if (nv <= 4) k_topk<4, kSelectOnly><<<blocks, 128, 0, st>>>(d, s, x);
  else if (nv <= 8) k_topk<8, kSelectOnly><<<blocks, 128, 0, st>>>(d, s, x);
  else if (nv <= 16) k_topk<16, kSelectOnly><<<blocks, 128, 0, st>>>(d, s, x);
  else if (nv <= 32) k_topk<32, kSelectOnly><<<blocks, 128, 0, st>>>(d, s, x);
  else if (nv <= 64) k_topk<64, kSelectOnly><<<blocks, 128, 0, st>>>(d, s, x);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_topk(const Dims &d, const Scratch &s, const Extras &x, cudaStream_t st) {
  return launch_topk_t<false>(d, s, x, st);
}

cudaError_t launch_topk_select(const Dims &d, const Scratch &s, const Extras &x,
                               cudaStream_t st) {
  return launch_topk_t<true>(d, s, x, st);
}

}  // namespace fwpkm
