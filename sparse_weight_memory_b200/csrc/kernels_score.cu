// kernels_score.cu -- operands of the sub-key distance contraction.
//
// IDW scoring (gist.science "Fast-weight Product Key Memory", section 2, Key
// Technical Choices): score = -log(eps + ||q_half - K_row||^2).  The only
// dense contraction of the step is q_half . K_row over every sub-key row;
// this file prepares its operands (fp32 halves split into a TF32 part and a
// remainder, squared norms); kernels_score_tc.cu runs the contraction on the
// tensor cores.
#include "fwpkm_internal.cuh"

namespace fwpkm {

// ---------------------------------------------------------------------------
// prep: per query half and per sub-key row, the fp32 values, their TF32 part
// (round to nearest) and the remainder, and the squared norm:
//   Qs / Qs_hi / Qs_lo [h][half][row][:], qn    (rows at stride qstride)
//   K_hi / K_lo [h][half][i][:], kn
// Warp per row; rows [0, 2*H*rows) are query halves, the rest sub-key rows.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float tf32_part(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__device__ __forceinline__ void split_store(float *hi, float *lo, int c, const float4 &v) {
  const float4 h = make_float4(tf32_part(v.x), tf32_part(v.y), tf32_part(v.z), tf32_part(v.w));
  *reinterpret_cast<float4 *>(hi + c) = h;
  *reinterpret_cast<float4 *>(lo + c) = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
}

template <typename TQ>
__global__ void __launch_bounds__(256) k_prep(Dims d, const TQ *__restrict__ Q,
                                              const float *__restrict__ K, Scratch s) {
  griddep_wait();
  griddep_launch();
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
    const int64_t o = ((int64_t)hh * d.qstride + row) * dh;
    float acc = 0.f;
    for (int c = lane * 4; c < dh; c += 128) {
      const float4 v = load4(Q, src + c);
      if (s.Qs) *reinterpret_cast<float4 *>(s.Qs + o + c) = v;
      split_store(s.Qs_hi + o, s.Qs_lo + o, c, v);
      acc = fmaf(v.x, v.x, acc);
      acc = fmaf(v.y, v.y, acc);
      acc = fmaf(v.z, v.z, acc);
      acc = fmaf(v.w, v.w, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) s.qn[(int64_t)hh * d.qstride + row] = acc;
  } else if (warp < nq + nk) {
    const int64_t r = warp - nq;  // (h*2+half)*n + i
    const float *src = K + r * dh;
    float acc = 0.f;
    for (int c = lane * 4; c < dh; c += 128) {
      const float4 v = *reinterpret_cast<const float4 *>(src + c);
      split_store(s.K_hi + r * dh, s.K_lo + r * dh, c, v);
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
    return launch_k(d.pdl, k_prep<__nv_bfloat16>, blocks, 256, 0, st, d,
                    (const __nv_bfloat16 *)Q, K, s);
  return launch_k(d.pdl, k_prep<float>, blocks, 256, 0, st, d, (const float *)Q, K, s);
}

}  // namespace fwpkm
