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
// prep: per query half and per sub-key row, the TF32 part (round to nearest)
// and the remainder of every element, and the squared norm:
//   Qs_hi / Qs_lo [h][half][row][:], qn      (rows at stride qstride)
//   K_hi / K_lo [h][half][i][:], kn per 128-float chunk (chunk_sqnorm)
// Warp per row.  k_prep does query halves (rows [0, nq)) and then sub-key
// rows; the step runs the query part alone (launch_prep_q, or inside the
// bucket sort of the previous chunk) and the sub-key part only when the
// tables are new (launch_prep_k): afterwards the update keeps the split of
// the rows it writes.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void prep_subkey_row(const Dims &d, const float *__restrict__ K,
                                                const Scratch &s, int64_t r) {
  const int lane = threadIdx.x & 31;
  const int dh = d.dh, dh4 = dh >> 2;
  const float *src = K + r * dh;
  for (int ch = 0; ch * 32 < dh4; ++ch) {
    const int c4 = ch * 32 + lane;
    const float4 v = c4 < dh4 ? *reinterpret_cast<const float4 *>(src + 4 * c4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    if (c4 < dh4) split_store(s.K_hi + r * dh, s.K_lo + r * dh, 4 * c4, v);
    const float sq = chunk_sqnorm(v);
    if (lane == 0) s.kn[r * kKnChunks + ch] = sq;
  }
}

template <typename TQ>
__global__ void __launch_bounds__(256) k_prep(Dims d, const TQ *__restrict__ Q,
                                              const float *__restrict__ K, Scratch s, int do_q,
                                              int do_k) {
  griddep_wait();
  griddep_launch();
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nq = do_q ? (int64_t)2 * d.H * d.rows : 0;
  const int64_t nk = do_k ? (int64_t)2 * d.H * d.nmem * d.n : 0;
  if (warp < nq) prep_query_half(d, Q, s, warp);
  else if (warp < nq + nk) prep_subkey_row(d, K, s, warp - nq);
}

static cudaError_t launch_prep_parts(const Dims &d, const void *Q, int q_dtype, const float *K,
                                     const Scratch &s, cudaStream_t st, int do_q, int do_k) {
  const int64_t warps =
      (do_q ? (int64_t)2 * d.H * d.rows : 0) + (do_k ? (int64_t)2 * d.H * d.nmem * d.n : 0);
  const int blocks = (int)((warps + 7) / 8);
  if (blocks == 0) return cudaSuccess;
  if (q_dtype == 1)
    return launch_k(d.pdl, k_prep<__nv_bfloat16>, blocks, 256, 0, st, d,
                    (const __nv_bfloat16 *)Q, K, s, do_q, do_k);
  return launch_k(d.pdl, k_prep<float>, blocks, 256, 0, st, d, (const float *)Q, K, s, do_q,
                  do_k);
}

cudaError_t launch_prep(const Dims &d, const void *Q, int q_dtype, const float *K,
                        const Scratch &s, cudaStream_t st) {
  return launch_prep_parts(d, Q, q_dtype, K, s, st, 1, 1);
}
cudaError_t launch_prep_q(const Dims &d, const void *Q, int q_dtype, const Scratch &s,
                          cudaStream_t st) {
  return launch_prep_parts(d, Q, q_dtype, nullptr, s, st, 1, 0);
}
cudaError_t launch_prep_k(const Dims &d, const float *K, const Scratch &s, cudaStream_t st) {
  return launch_prep_parts(d, nullptr, 0, K, s, st, 0, 1);
}

}  // namespace fwpkm
