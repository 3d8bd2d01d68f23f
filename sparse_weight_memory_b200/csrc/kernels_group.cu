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
//   sub-key row : K -= eta * sum over its pairs of dL/ds * 2 (q - K)/(eps + d)
//   marginal    : pbar_i = (1/M) sum over its pairs of w;
//                 dL_addr/dw = (lam/M) (log pbar_i + 1)
//
// Groups are value rows [0, N) and sub-key rows N + (h*2+half)*n + i.  The
// selection kernel counted members per group and claimed a position; the scan
// below turns counts into offsets and a list of touched groups; the read
// kernel scatters member ids to offset + claim.  Claim order depends on atomic
// timing, so every group sorts its member ids before summing: the sums run in
// id order and the result is independent of scheduling.
#include <math_constants.h>

#include "fwpkm_internal.cuh"

namespace fwpkm {

// ---------------------------------------------------------------------------
// Scan over the group counts.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 256;
constexpr int kScanPer = kScanTile / kScanThreads;  // 8 consecutive groups per thread

__device__ __forceinline__ int block_sum_int(int v, int *red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  int t = 0;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
  return t;
}

// Exclusive prefix over the block (thread order); returns the block total.
__device__ __forceinline__ int block_excl_scan(int v, int *red, int &total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();
  if (lane == 31) red[w] = incl;
  __syncthreads();
  int before = 0, tot = 0;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
    if (i < w) before += red[i];
    tot += red[i];
  }
  total = tot;
  return before + incl - v;
}

__global__ void __launch_bounds__(kScanThreads) k_scan_tiles(Dims d, Scratch s) {
  __shared__ int red[kScanThreads / 32];
  const int64_t g0 = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanPer;
  int c = 0, nz = 0;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    const int64_t g = g0 + i;
    const int v = g < d.G ? s.count[g] : 0;
    c += v;
    nz += v > 0;
  }
  c = block_sum_int(c, red);
  nz = block_sum_int(nz, red);
  if (threadIdx.x == 0) {
    s.tile_cnt[blockIdx.x] = c;
    s.tile_nz[blockIdx.x] = nz;
  }
}

__global__ void __launch_bounds__(kScanThreads) k_scan_write(Dims d, Scratch s) {
  __shared__ int red[kScanThreads / 32];
  const int tile = blockIdx.x;
  // Offsets of this tile: sums over the previous tiles.
  int bc = 0, bn = 0;
  for (int t = threadIdx.x; t < tile; t += blockDim.x) {
    bc += s.tile_cnt[t];
    bn += s.tile_nz[t];
  }
  bc = block_sum_int(bc, red);
  bn = block_sum_int(bn, red);
  const int64_t g0 = (int64_t)tile * kScanTile + (int64_t)threadIdx.x * kScanPer;
  int cv[kScanPer];
  int c = 0, nz = 0;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    const int64_t g = g0 + i;
    cv[i] = g < d.G ? s.count[g] : 0;
    c += cv[i];
    nz += cv[i] > 0;
  }
  int tot_c, tot_nz;
  int ec = block_excl_scan(c, red, tot_c);
  int en = block_excl_scan(nz, red, tot_nz);
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    const int64_t g = g0 + i;
    if (g >= d.G) break;
    if (g == d.N) {  // first sub-key group: everything before it is a value row
      s.meta->U_v = bn + en;
      atomicAdd(&s.meta->stat_value_rows, (unsigned long long)(bn + en));
    }
    if (cv[i] > 0) {
      const int off = bc + ec;
      const int u = bn + en;
      s.goff[g] = off;
      s.uniq[u] = (int)g;
      s.useg_off[u] = off;
      s.useg_len[u] = cv[i];
      s.count[g] = 0;  // ready for the next chunk
      ec += cv[i];
      en += 1;
    }
  }
  if (tile == (int)gridDim.x - 1 && threadIdx.x == 0) {
    s.meta->U_total = bn + tot_nz;
    atomicAdd(&s.meta->stat_total_rows, (unsigned long long)(bn + tot_nz));
    atomicAdd(&s.meta->stat_chunks, 1ull);
  }
}

cudaError_t launch_scan(const Dims &d, const Scratch &s, cudaStream_t st, int part) {
  const int tiles = (int)((d.G + kScanTile - 1) / kScanTile);
  if (part == 0)
    k_scan_tiles<<<tiles, kScanThreads, 0, st>>>(d, s);
  else
    k_scan_write<<<tiles, kScanThreads, 0, st>>>(d, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Ordered member iteration of one group (warp-cooperative).
//   len <= 32            : ids sorted across the lanes (bitonic)
//   len <= kWarpSortMax  : ids sorted in warp-private shared memory
//   otherwise            : `scan(id)` enumerates every candidate id in order
// `body(id)` is called by the whole warp, in increasing id order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int lane_sort32(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int o = __shfl_xor_sync(FULL, v, stride);
      const bool up = (lane & size) == 0 || size == 32;
      const bool lower = (lane & stride) == 0;
      const bool keep = (lower == up) ? (v <= o) : (v >= o);
      if (!keep) v = o;
    }
  }
  return v;
}

// Sort buf[0..len) ascending in place (warp-private smem, len <= kWarpSortMax).
__device__ void warp_smem_sort(int *buf, int len) {
  const int lane = threadIdx.x & 31;
  int n2 = 64;
  while (n2 < len) n2 <<= 1;
  for (int i = len + lane; i < n2; i += 32) buf[i] = 0x7fffffff;
  __syncwarp();
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < n2; i += 32) {
        const int l = i ^ stride;
        if (l > i) {
          const int a = buf[i], b = buf[l];
          const bool up = (i & size) == 0;
          if ((a > b) == up) {
            buf[i] = b;
            buf[l] = a;
          }
        }
      }
      __syncwarp();
    }
  }
}

template <typename Body, typename Match>
__device__ __forceinline__ void for_members_ordered(const int *ids, int len, int *wbuf,
                                                    int64_t scan_n, Match match, Body body) {
  const int lane = threadIdx.x & 31;
  if (len <= 32) {
    int v = lane < len ? ids[lane] : 0x7fffffff;
    v = lane_sort32(v);
    for (int r = 0; r < len; ++r) body(__shfl_sync(FULL, v, r));
  } else if (len <= kWarpSortMax) {
    for (int i = lane; i < len; i += 32) wbuf[i] = ids[i];
    __syncwarp();
    warp_smem_sort(wbuf, len);
    for (int r = 0; r < len; ++r) body(wbuf[r]);
    __syncwarp();
  } else {
    for (int64_t base = 0; base < scan_n; base += 32) {
      const int64_t id = base + lane;
      unsigned hit = __ballot_sync(FULL, id < scan_n && match((int)id));
      while (hit) {
        const int l = __ffs(hit) - 1;
        hit &= hit - 1;
        body((int)(base + l));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// vapply: per touched value row.
// ---------------------------------------------------------------------------
constexpr int kApplyWarps = 8;

template <int Q4>  // float4 columns per lane: dv <= 128 * Q4
__global__ void __launch_bounds__(kApplyWarps * 32) k_vapply(Dims d, float *__restrict__ V,
                                                             const float *__restrict__ gate,
                                                             Scratch s) {
  __shared__ int wbuf_all[kApplyWarps][kWarpSortMax];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  int *wbuf = wbuf_all[wib];
  const int U_v = s.meta->U_v;
  const int HK = d.H * d.k;
  const int dv4 = d.dv >> 2;
  const float invH = 1.f / (float)d.H;
  const int64_t P = (int64_t)d.M * d.k;
  for (int u = blockIdx.x * kApplyWarps + wib; u < U_v; u += gridDim.x * kApplyWarps) {
    const int slot = s.uniq[u];
    const int off = s.useg_off[u], len = s.useg_len[u];
    float4 G[Q4];
#pragma unroll
    for (int q = 0; q < Q4; ++q) G[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    float C = 0.f, wsum = 0.f;
    auto body = [&](int p) {
      const int row = p / HK;
      const int b = row / d.Tc, tl = row % d.Tc;
      const float g = gate[(int64_t)b * d.T + d.t0 + tl];
      const float w = s.pw[p];
      const float coef = 2.f * g * invH * w;
      const float *e = s.E + (int64_t)row * d.dv;
#pragma unroll
      for (int q = 0; q < Q4; ++q) {
        const int c4 = lane + 32 * q;
        if (c4 < dv4) {
          const float4 ev = *reinterpret_cast<const float4 *>(e + 4 * c4);
          G[q].x = fmaf(coef, ev.x, G[q].x);
          G[q].y = fmaf(coef, ev.y, G[q].y);
          G[q].z = fmaf(coef, ev.z, G[q].z);
          G[q].w = fmaf(coef, ev.w, G[q].w);
        }
      }
      C += w * invH;
      wsum += w;
    };
    auto match = [&](int p) { return s.pslot[p] == slot; };
    for_members_ordered(s.sorted + off, len, wbuf, P, match, body);
    if (C > 0.f) {
      const float scale = d.eta / C;
      float *vr = V + (int64_t)slot * d.dv;
#pragma unroll
      for (int q = 0; q < Q4; ++q) {
        const int c4 = lane + 32 * q;
        if (c4 < dv4) {
          float4 v = *reinterpret_cast<float4 *>(vr + 4 * c4);
          v.x -= scale * G[q].x;
          v.y -= scale * G[q].y;
          v.z -= scale * G[q].z;
          v.w -= scale * G[q].w;
          *reinterpret_cast<float4 *>(vr + 4 * c4) = v;
        }
      }
    }
    if (d.lam != 0.f) {
      const float pbar = wsum / (float)d.M;
      const float bterm = (d.lam / (float)d.M) * (logf(pbar) + 1.f);
      for (int i = lane; i < len; i += 32) s.pb[s.sorted[off + i]] = bterm;
    }
  }
}

cudaError_t launch_vapply(const Dims &d, float *V, const float *gate, const Scratch &s,
                          cudaStream_t st) {
  const int64_t maxU = (int64_t)d.M * d.k;
  int blocks = (int)((maxU + kApplyWarps - 1) / kApplyWarps);
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  const int q4 = (d.dv / 4 + 31) / 32;
  if (q4 <= 1) k_vapply<1><<<blocks, kApplyWarps * 32, 0, st>>>(d, V, gate, s);
  else if (q4 <= 2) k_vapply<2><<<blocks, kApplyWarps * 32, 0, st>>>(d, V, gate, s);
  else if (q4 <= 4) k_vapply<4><<<blocks, kApplyWarps * 32, 0, st>>>(d, V, gate, s);
  else if (q4 <= 8) k_vapply<8><<<blocks, kApplyWarps * 32, 0, st>>>(d, V, gate, s);
  else if (q4 <= 16) k_vapply<16><<<blocks, kApplyWarps * 32, 0, st>>>(d, V, gate, s);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// pgrad: dL/ds_r = w_r (gamma_r - sum_r' w_r' gamma_r'), gamma = dL/dw.
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
    gam = s.pa[p] + (d.lam != 0.f ? s.pb[p] : 0.f);
  }
  const float S = warp_sum(w * gam);
  if (lane < d.k) s.pdl[p] = w * (gam - S);
}

cudaError_t launch_pgrad(const Dims &d, const Scratch &s, cudaStream_t st) {
  k_pgrad<<<(d.M + 7) / 8, 256, 0, st>>>(d, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// kapply: per touched sub-key row (h, half, i):
//   alpha_e = (1/(eps + d)) * sum over the entry's pairs of dL/ds
//   K_i -= eta * 2 * (sum_e alpha_e q_e - (sum_e alpha_e) K_i)
// ---------------------------------------------------------------------------
template <int Q4>  // float4 columns per lane: dh <= 128 * Q4
__global__ void __launch_bounds__(kApplyWarps * 32) k_kapply(Dims d, float *__restrict__ K,
                                                             Scratch s) {
  __shared__ int wbuf_all[kApplyWarps][kWarpSortMax];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  int *wbuf = wbuf_all[wib];
  const int U_v = s.meta->U_v, U_total = s.meta->U_total;
  const int dh4 = d.dh >> 2;
  const int k = d.k, n = d.n;
  const int64_t E = (int64_t)d.M * 2 * k;
  for (int u = U_v + blockIdx.x * kApplyWarps + wib; u < U_total;
       u += gridDim.x * kApplyWarps) {
    const int bucket = (int)(s.uniq[u] - d.N);  // (h*2+half)*n + sub
    const int hh = bucket / n, sub = bucket % n;
    const int off = s.useg_off[u], len = s.useg_len[u];
    float4 G[Q4];
#pragma unroll
    for (int q = 0; q < Q4; ++q) G[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    float A = 0.f;
    auto body = [&](int e) {
      const int m = e / (2 * k);
      const int row = m / d.H;
      const unsigned mask = s.emask[e];
      const float v = (lane < k && ((mask >> lane) & 1u)) ? s.pdl[(int64_t)m * k + lane] : 0.f;
      const float alpha = s.einv[e] * warp_sum(v);
      const float *q = s.Qs + ((int64_t)hh * d.rows + row) * d.dh;
#pragma unroll
      for (int qq = 0; qq < Q4; ++qq) {
        const int c4 = lane + 32 * qq;
        if (c4 < dh4) {
          const float4 qv = *reinterpret_cast<const float4 *>(q + 4 * c4);
          G[qq].x = fmaf(alpha, qv.x, G[qq].x);
          G[qq].y = fmaf(alpha, qv.y, G[qq].y);
          G[qq].z = fmaf(alpha, qv.z, G[qq].z);
          G[qq].w = fmaf(alpha, qv.w, G[qq].w);
        }
      }
      A += alpha;
    };
    auto match = [&](int e) {
      const int mh = e / k, idx = e % k;  // mh = m*2 + half
      const int m = mh >> 1, half = mh & 1;
      return (m % d.H) * 2 + half == hh && idx < s.ecount[mh] && s.esub[e] == sub;
    };
    for_members_ordered(s.sorted + off, len, wbuf, E, match, body);
    float *kr = K + ((int64_t)hh * n + sub) * d.dh;
    const float two_eta = 2.f * d.eta;
#pragma unroll
    for (int qq = 0; qq < Q4; ++qq) {
      const int c4 = lane + 32 * qq;
      if (c4 < dh4) {
        float4 kv = *reinterpret_cast<float4 *>(kr + 4 * c4);
        kv.x -= two_eta * (G[qq].x - A * kv.x);
        kv.y -= two_eta * (G[qq].y - A * kv.y);
        kv.z -= two_eta * (G[qq].z - A * kv.z);
        kv.w -= two_eta * (G[qq].w - A * kv.w);
        *reinterpret_cast<float4 *>(kr + 4 * c4) = kv;
      }
    }
  }
}

cudaError_t launch_kapply(const Dims &d, float *K, const Scratch &s, cudaStream_t st) {
  int blocks = (2 * d.H * d.n + kApplyWarps - 1) / kApplyWarps;
  if (blocks > 148 * 8) blocks = 148 * 8;
  const int q4 = (d.dh / 4 + 31) / 32;
  if (q4 <= 1) k_kapply<1><<<blocks, kApplyWarps * 32, 0, st>>>(d, K, s);
  else if (q4 <= 2) k_kapply<2><<<blocks, kApplyWarps * 32, 0, st>>>(d, K, s);
  else if (q4 <= 4) k_kapply<4><<<blocks, kApplyWarps * 32, 0, st>>>(d, K, s);
  else if (q4 <= 8) k_kapply<8><<<blocks, kApplyWarps * 32, 0, st>>>(d, K, s);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace fwpkm
