// kernels_read.cu -- gather, gated readout, residual and dL/dw per pair.
//
// Readout (gist.science "Fast-weight Product Key Memory", section 2: the
// retrieved value; gate g_t; agifrontier tutorial, gating): per token
//   yhat_t = (1/H) sum_h sum_r w_{t,h,r} V[slot_{t,h,r}]
//   out_t  = g_t * yhat_t
// and, for the write that follows (MSE memorisation loss weighted by the
// token's gate, sciencestack table of contents sections 8-12):
//   e_t          = yhat_t - v_t
//   dL/dw_{t,h,r} = (2 g_t / H) e_t . V[slot_{t,h,r}]   (pre-update rows)
// and, when the entropy term is off (so dL/dw is complete here), the softmax
// Jacobian dL/ds_r = w_r (dL/dw_r - sum_r' w_r' dL/dw_r') and, per sub-key
// entry, alpha = (sum of dL/ds over its pairs) / (eps + d).
// One CTA per token row.  The H*k value rows are fetched by 1-D bulk async
// copies (TMA) straight into shared memory, completing on one mbarrier, so
// the whole gather of a token is in flight at once; both passes (weighted
// sum, then the dot products with e_t) read the staged rows.  Rows that do
// not fit in shared memory are read from global memory in both passes.
#include "fwpkm_internal.cuh"

namespace fwpkm {

constexpr int kReadThreads = 128;
constexpr size_t kReadSmemBudget = 200 * 1024;

// Dynamic shared memory layout (bytes):
//   [0, 16)            mbarrier
//   [128, 128+R)       staged rows, R = H*k*dv*4 (staged variant only)
//   then               e (dv floats), w, slot, a, dL/ds (H*k each)
static size_t read_smem_bytes(const Dims &d, bool staged) {
  const size_t HK = (size_t)d.H * d.k;
  return 128 + (staged ? HK * d.dv * 4 : 0) + (size_t)d.dv * 4 + HK * 16;
}

template <typename TV, bool kStaged>
__global__ void __launch_bounds__(kReadThreads) k_read(Dims d, const float *__restrict__ V,
                                                       const TV *__restrict__ Vt,
                                                       const float *__restrict__ gate,
                                                       float *__restrict__ out, Scratch s) {
  griddep_wait();
  griddep_launch();
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
  const int HK = d.H * d.k, dv = d.dv, dv4 = dv >> 2;
  float *rows_s = reinterpret_cast<float *>(smem + 128);
  float *e_s = rows_s + (kStaged ? (size_t)HK * dv : 0);
  float *w_s = e_s + dv;
  int *slot_s = reinterpret_cast<int *>(w_s + HK);
  float *a_s = reinterpret_cast<float *>(slot_s + HK);
  float *dl_s = a_s + HK;

  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int b = row / d.Tc, tl = row % d.Tc;
  const int64_t tok = (int64_t)b * d.T + d.t0 + tl;
  const int64_t p0 = (int64_t)row * HK;

  for (int j = tid; j < HK; j += blockDim.x) {
    w_s[j] = s.pw[p0 + j];
    slot_s[j] = s.pslot[p0 + j];
  }
  if (kStaged) {
    if (tid == 0) mbar_init(bar, 1);
    __syncthreads();
    if (tid == 0) {
      const unsigned row_bytes = (unsigned)dv * 4u;
      mbar_arrive_expect_tx(bar, row_bytes * (unsigned)HK);
      for (int j = 0; j < HK; ++j)
        bulk_g2s(rows_s + (size_t)j * dv, V + (int64_t)slot_s[j] * dv, row_bytes, bar);
    }
    if (!mbar_wait_bounded(bar, 0, s.meta)) {
      mbar_wait_bounded(bar, 0, s.meta);  // let copies in flight land before exit
      return;
    }
  } else {
    __syncthreads();
  }

  const float g = gate[tok];
  const float invH = 1.f / (float)d.H;
  for (int c4 = tid; c4 < dv4; c4 += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < HK; ++j) {
      const float w = w_s[j];
      const float4 v = kStaged ? *reinterpret_cast<const float4 *>(rows_s + (size_t)j * dv + 4 * c4)
                               : *reinterpret_cast<const float4 *>(V + (int64_t)slot_s[j] * dv + 4 * c4);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    const float4 y = make_float4(acc.x * invH, acc.y * invH, acc.z * invH, acc.w * invH);
    *reinterpret_cast<float4 *>(out + tok * dv + 4 * c4) =
        make_float4(g * y.x, g * y.y, g * y.z, g * y.w);
    const float4 t = load4(Vt, tok * dv + 4 * c4);
    const float4 e = make_float4(y.x - t.x, y.y - t.y, y.z - t.z, y.w - t.w);
    *reinterpret_cast<float4 *>(s.E + (int64_t)row * dv + 4 * c4) = e;
    *reinterpret_cast<float4 *>(e_s + 4 * c4) = e;
  }
  __syncthreads();

  // dL/dw per pair: warp `wid` takes pairs j = wid, wid + 4, ...
  const float coef = 2.f * g * invH;
  for (int j = wid; j < HK; j += kReadThreads / 32) {
    const float *vr = kStaged ? rows_s + (size_t)j * dv : V + (int64_t)slot_s[j] * dv;
    float acc = 0.f;
    for (int c4 = lane; c4 < dv4; c4 += 32) {
      const float4 v = *reinterpret_cast<const float4 *>(vr + 4 * c4);
      const float4 e = *reinterpret_cast<const float4 *>(e_s + 4 * c4);
      acc = fmaf(e.x, v.x, acc);
      acc = fmaf(e.y, v.y, acc);
      acc = fmaf(e.z, v.z, acc);
      acc = fmaf(e.w, v.w, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) {
      s.pa[p0 + j] = coef * acc;
      a_s[j] = coef * acc;
    }
  }

  // dL/ds and alpha per entry when the entropy term is off (dL/dw complete)
  __syncthreads();
  const bool alpha_now = d.lam == 0.f;
  if (alpha_now) {
    for (int h = wid; h < d.H; h += kReadThreads / 32) {
      const int j = h * d.k + lane;
      const float w = lane < d.k ? w_s[j] : 0.f;
      const float a = lane < d.k ? a_s[j] : 0.f;
      const float S = warp_sum(w * a);
      if (lane < d.k) dl_s[j] = w * (a - S);
    }
    __syncthreads();
    // alpha of every entry of this row, one thread each
    for (int x = tid; x < 2 * HK; x += blockDim.x) {
      const int mh = x / d.k, idx = x % d.k;  // mh = h*2 + half
      const int64_t mhg = (int64_t)row * 2 * d.H + mh;
      if (idx < s.ecount[mhg]) {
        const int64_t e = mhg * d.k + idx;
        unsigned mask = s.emask[e];
        const float *dl = dl_s + (mh >> 1) * d.k;
        float sum = 0.f;
        while (mask) {
          sum += dl[__ffs(mask) - 1];
          mask &= mask - 1;
        }
        s.ealpha[e] = s.einv[e] * sum;
      }
    }
    __syncthreads();
  }
  // Member records into their buckets: pairs -> value bucket slot >> vshift,
  // entries -> sub-key row bucket NBv + (h*2+half)*n + row.
  for (int j = tid; j < HK; j += blockDim.x) {
    const int64_t p = p0 + j;
    const float w = w_s[j];
    Member m;
    m.g = (uint32_t)slot_s[j];
    m.id = (uint32_t)p;
    m.srow = row;
    m.gstart = 0;
    m.coef = 2.f * g * w * invH;
    m.c0 = w * invH;
    m.c1 = w;
    m.glen = 0;
    s.rec_in[s.boff[slot_s[j] >> d.vshift] + s.pclaim[p]] = m;
  }
  const int ne = 2 * HK;  // entries of this row: (h*2 + half)*k + idx
  for (int x = tid; x < ne; x += blockDim.x) {
    const int mh = x / d.k, idx = x % d.k;  // mh = h*2 + half
    const int64_t mhg = (int64_t)row * 2 * d.H + mh;
    if (idx < s.ecount[mhg]) {
      const int64_t e = mhg * d.k + idx;
      const int sub = s.esub[e];
      const float alpha = alpha_now ? s.ealpha[e] : 0.f;
      Member m;
      m.g = (uint32_t)d.N + (uint32_t)(mh * d.n + sub);
      m.id = (uint32_t)e;
      m.srow = mh * d.qstride + row;
      m.gstart = 0;
      m.coef = alpha;
      m.c0 = alpha;
      m.c1 = 0.f;
      m.glen = 0;
      s.rec_in[s.boff[d.NBv + mh * d.n + sub] + s.eclaim[e]] = m;
    }
  }
}

template <typename TV>
static cudaError_t launch_read_t(const Dims &d, const float *V, const TV *Vt, const float *gate,
                                 float *out, const Scratch &s, cudaStream_t st) {
  const bool staged = read_smem_bytes(d, true) <= kReadSmemBudget;
  const size_t smem = read_smem_bytes(d, staged);
  if (staged) {
    cudaFuncSetAttribute(k_read<TV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    return launch_k(d.pdl, k_read<TV, true>, d.rows, kReadThreads, smem, st, d, V, Vt, gate,
                    out, s);
  } else {
    cudaFuncSetAttribute(k_read<TV, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    return launch_k(d.pdl, k_read<TV, false>, d.rows, kReadThreads, smem, st, d, V, Vt, gate,
                    out, s);
  }
}

cudaError_t launch_read(const Dims &d, const float *V, const void *Vt, int v_dtype,
                        const float *gate, float *out, const Scratch &s, cudaStream_t st) {
  if (v_dtype == 1)
    return launch_read_t(d, V, (const __nv_bfloat16 *)Vt, gate, out, s, st);
  return launch_read_t(d, V, (const float *)Vt, gate, out, s, st);
}

}  // namespace fwpkm
