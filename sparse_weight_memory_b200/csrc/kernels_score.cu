// kernels_score.cu -- query split and sub-key distances.
//
// IDW scoring (gist.science "Fast-weight Product Key Memory", section 2, Key
// Technical Choices): score = -log(eps + ||q_half - K_row||^2).  The only
// dense contraction of the step is q_half . K_row over every sub-key row;
// this file produces the squared distances
//     D[h][half][row][i] = |q|^2 + |K_i|^2 - 2 q.K_i   (clamped at 0)
// and the selection kernel turns the chosen ones into scores.
#include "fwpkm_internal.cuh"

namespace fwpkm {

// ---------------------------------------------------------------------------
// prep: Qs[h][half][row][:] = query half (fp32), qn = |q_half|^2, and
// kn[h][half][i] = |K_i|^2 for the sub-key tables as they stand.
// Warp per row; rows [0, 2*H*rows) are query halves, the rest sub-key rows.
// ---------------------------------------------------------------------------
template <typename TQ>
__global__ void __launch_bounds__(256) k_prep(Dims d, const TQ *__restrict__ Q,
                                              const float *__restrict__ K, Scratch s) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nq = (int64_t)2 * d.H * d.rows;
  const int64_t nk = (int64_t)2 * d.H * d.n;
  const int dh = d.dh;
  if (warp < nq) {
    const int hh = (int)(warp / d.rows);  // h*2 + half
    const int row = (int)(warp % d.rows);
    const int h = hh >> 1, half = hh & 1;
    const int b = row / d.Tc, tl = row % d.Tc;
    const int64_t src = ((int64_t)b * d.T + d.t0 + tl) * ((int64_t)d.H * d.dq) +
                        (int64_t)h * d.dq + (int64_t)half * dh;
    float *dst = s.Qs + ((int64_t)hh * d.rows + row) * dh;
    float acc = 0.f;
    for (int c = lane * 4; c < dh; c += 128) {
      float4 v = load4(Q, src + c);
      *reinterpret_cast<float4 *>(dst + c) = v;
      acc = fmaf(v.x, v.x, acc);
      acc = fmaf(v.y, v.y, acc);
      acc = fmaf(v.z, v.z, acc);
      acc = fmaf(v.w, v.w, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) s.qn[(int64_t)hh * d.rows + row] = acc;
  } else if (warp < nq + nk) {
    const int64_t r = warp - nq;  // (h*2+half)*n + i
    const float *src = K + r * dh;
    float acc = 0.f;
    for (int c = lane * 4; c < dh; c += 128) {
      float4 v = *reinterpret_cast<const float4 *>(src + c);
      acc = fmaf(v.x, v.x, acc);
      acc = fmaf(v.y, v.y, acc);
      acc = fmaf(v.z, v.z, acc);
      acc = fmaf(v.w, v.w, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) s.kn[r] = acc;
  }
}

cudaError_t launch_prep(const Dims &d, const void *Q, int q_dtype, const float *K,
                        const Scratch &s, cudaStream_t st) {
  const int64_t warps = (int64_t)2 * d.H * d.rows + (int64_t)2 * d.H * d.n;
  const int blocks = (int)((warps + 7) / 8);
  if (q_dtype == 1)
    k_prep<__nv_bfloat16><<<blocks, 256, 0, st>>>(d, (const __nv_bfloat16 *)Q, K, s);
  else
    k_prep<float><<<blocks, 256, 0, st>>>(d, (const float *)Q, K, s);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// score: per (h, half) a [rows x dh] . [dh x n] product.  32x64 tiles, 128
// threads with 4x4 outputs each, k-slices of 8 (dh % 8 == 0); the next slice
// is fetched into registers while the current one is multiplied.
// ---------------------------------------------------------------------------
constexpr int ST_M = 32, ST_N = 64, ST_K = 8;

__global__ void __launch_bounds__(128) k_score_simt(Dims d, const float *__restrict__ K,
                                                    Scratch s) {
  __shared__ float As[2][ST_K][ST_M + 4];
  __shared__ float Bs[2][ST_K][ST_N + 4];
  const int hh = blockIdx.z;
  const int m0 = blockIdx.y * ST_M, n0 = blockIdx.x * ST_N;
  const int rows = d.rows, n = d.n, dh = d.dh;
  const float *A = s.Qs + (int64_t)hh * rows * dh;
  const float *Bm = K + (int64_t)hh * n * dh;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;  // 16 x 8 threads, 4x4 outputs each
  float acc[4][4] = {};
  // loaders: A slice = 32 rows x 2 float4 (threads 0..63), B slice = 64 rows x
  // 2 float4 (all 128 threads)
  const int arow = tid >> 1, aq = tid & 1;
  const int brow = tid >> 1, bq = tid & 1;
  auto fetch = [&](int k0, float4 &va, float4 &vb) {
    va = make_float4(0.f, 0.f, 0.f, 0.f);
    vb = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tid < 64 && m0 + arow < rows)
      va = *reinterpret_cast<const float4 *>(A + (int64_t)(m0 + arow) * dh + k0 + aq * 4);
    if (n0 + brow < n)
      vb = *reinterpret_cast<const float4 *>(Bm + (int64_t)(n0 + brow) * dh + k0 + bq * 4);
  };
  auto stash = [&](int buf, const float4 &va, const float4 &vb) {
    if (tid < 64) {
      As[buf][aq * 4 + 0][arow] = va.x;
      As[buf][aq * 4 + 1][arow] = va.y;
      As[buf][aq * 4 + 2][arow] = va.z;
      As[buf][aq * 4 + 3][arow] = va.w;
    }
    Bs[buf][bq * 4 + 0][brow] = vb.x;
    Bs[buf][bq * 4 + 1][brow] = vb.y;
    Bs[buf][bq * 4 + 2][brow] = vb.z;
    Bs[buf][bq * 4 + 3][brow] = vb.w;
  };
  float4 va, vb;
  fetch(0, va, vb);
  stash(0, va, vb);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < dh; k0 += ST_K) {
    const bool more = k0 + ST_K < dh;
    if (more) fetch(k0 + ST_K, va, vb);  // in flight during the multiply below
#pragma unroll
    for (int kk = 0; kk < ST_K; ++kk) {
      const float4 a = *reinterpret_cast<const float4 *>(&As[buf][kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4 *>(&Bs[buf][kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (more) stash(buf ^ 1, va, vb);
    __syncthreads();
    buf ^= 1;
  }
  const float *qn = s.qn + (int64_t)hh * rows;
  const float *kn = s.kn + (int64_t)hh * n;
  float *D = s.D + (int64_t)hh * rows * n;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + ty * 4 + i;
    if (r >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= n) continue;
      const float v = qn[r] + kn[c] - 2.f * acc[i][j];
      D[(int64_t)r * n + c] = v > 0.f ? v : 0.f;
    }
  }
}

cudaError_t launch_score(const Dims &d, const float *K, const Scratch &s, cudaStream_t st) {
  dim3 grid((d.n + ST_N - 1) / ST_N, (d.rows + ST_M - 1) / ST_M, 2 * d.H);
  k_score_simt<<<grid, 128, 0, st>>>(d, K, s);
  return cudaGetLastError();
}

}  // namespace fwpkm
