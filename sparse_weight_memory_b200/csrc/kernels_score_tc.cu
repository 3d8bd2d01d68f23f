// kernels_score_tc.cu -- sub-key distances on the 5th-generation tensor cores.
//
// IDW scoring (gist.science "Fast-weight Product Key Memory", section 2, Key
// Technical Choices) needs ||q_half - K_i||^2 for every sub-key of both halves:
// the step's only dense contraction, q_half . K_i.  Per (head, half) it is a
// [rows x dh] . [dh x n] product; this kernel computes it with tcgen05.mma
// (kind::tf32, fp32 accumulate in tensor memory) on operand tiles brought in
// by TMA, and writes
//     D[h][half][row][i] = |q|^2 + |K_i|^2 - 2 q.K_i      (clamped at 0)
// or, with the dot-product score, D = -q.K_i (the selection takes the
// smallest D either way).
//
// Precision: three TF32 products, hi*hi + hi*lo + lo*hi, where x = hi + lo and
// hi is x rounded to TF32 (the prep writes both parts, and the update rewrites
// them for the sub-key rows it changes).  The dropped
// lo*lo term and the truncation of lo are ~2^-21 relative, so the distances
// match an fp32 evaluation to a few ulps and the selection is decided at
// fp32 accuracy.  A bf16 query is exact in TF32 (its lo part is zero), so
// for bf16 queries the lo*hi product and the query's lo tile are skipped:
// two MMAs per k-step instead of three.
//
// CTA = one 128-row x BN-column output tile of one (head, half); 4 warps.
//   warp 0, one lane: TMA producer over k-blocks of 32 elements (128 bytes,
//                     128-byte swizzle), 2- or 3-deep ring;
//   warp 1:           allocates the accumulator columns in tensor memory;
//                     one lane issues the MMAs and commits each stage back;
//   warps 0-3:        epilogue, one accumulator lane (= output row) per thread.
// Every mbarrier wait is bounded; a wait that gives up sets an error bit.
// The kernel then still waits (up to a fixed drain bound) for the TMA loads
// it issued and for the MMAs in flight, writes zero distances for its tile,
// releases its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "fwpkm_internal.cuh"

namespace fwpkm {

constexpr int kTcRows = 128;      // M of every MMA (cta_group::1)
constexpr int kTcKBlock = 32;     // fp32 elements per 128-byte swizzle row
// Ring depth.  Up to 64 columns: two stages, so that two CTAs share a
// multiprocessor and one's epilogue and ring fill overlap the other's MMAs
// (measured on the 1M-slot shape: 29 -> 20 us per chunk against four stages
// and one CTA); 128 columns: three stages, one CTA.
template <int BN>
constexpr int tc_stages() {
  return BN <= 64 ? 2 : 3;
}
template <int BN>
constexpr int tc_ctas_per_sm() {
  return BN <= 64 ? 2 : 1;
}

// --- tcgen05 helpers (inline PTX, sm_100a) --------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::tf32.
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every MMA issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// 32 consecutive fp32 columns of this thread's accumulator lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 2-D tiled TMA load, into this CTA's shared memory only, of box {32 elements, rows} at {x, y}.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), leading offset field 1, descriptor version 1.
__device__ __forceinline__ uint64_t kmajor_sw128_desc(const void *smem_tile) {
  const uint64_t start = (uint64_t)(smem_u32(smem_tile) >> 4) & 0x3fffull;
  return start | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: D f32, A and B tf32, both K-major, M = 128, N = BN.
template <int BN>
__device__ __forceinline__ uint32_t idesc_tf32() {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(BN >> 3) << 17) |
         ((uint32_t)(kTcRows >> 4) << 24);
}

template <int BN>
struct TcSmem {

  static constexpr int kA = kTcRows * kTcKBlock * 4;  // 16 KiB per operand part
  static constexpr int kB = BN * kTcKBlock * 4;
  static constexpr int kStage = 2 * kA + 2 * kB;      // hi and lo of A and B
  static constexpr int kStages = tc_stages<BN>();
  static constexpr int kBytes =
      kStages * kStage + 1024 /* align */ + 256 /* barriers */ + 4 * BN /* column norms */;
};

template <int BN, bool kALo>
__global__ void __launch_bounds__(128, tc_ctas_per_sm<BN>())
    k_score_tc(const __grid_constant__ CUtensorMap mapAhi, const __grid_constant__ CUtensorMap mapAlo,
               const __grid_constant__ CUtensorMap mapBhi, const __grid_constant__ CUtensorMap mapBlo,
               Dims d, Scratch s) {
  extern __shared__ unsigned char smem_raw[];
  using L = TcSmem<BN>;
  constexpr uint32_t kCols = BN < 32 ? 32 : BN;  // tensor-memory columns (power of 2)
  unsigned char *smem =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr int kTcStages = L::kStages;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kTcStages * L::kStage);
  uint64_t *empty = full + kTcStages;
  uint64_t *done = empty + kTcStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  float *kn_s = reinterpret_cast<float *>(smem + kTcStages * L::kStage + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hh = blockIdx.z;
  const int m0 = blockIdx.y * kTcRows, n0 = blockIdx.x * BN;  // m0: a row of the layout
  // the sub-key table of this tile: (memory, head, half)
  const int tab = (d.nmem > 1 ? m0 / d.rstride : 0) * 2 * d.H + hh;
  const int nkb = (d.dh + kTcKBlock - 1) / kTcKBlock;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapAhi)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapBhi)) : "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The query tiles of the first stages are loaded before the grid dependency
  // wait when they come from an earlier grid than the one just before (which
  // updates the sub-keys): each stage's full byte count is expected now, its
  // sub-key tiles are loaded after the wait.
  int pre = 0;  // k-blocks whose query tiles are in flight before the wait (thread 0)
  if (d.q_early && warp == 0 && lane == 0) {
    pre = nkb < kTcStages ? nkb : kTcStages;
    const int ya = hh * d.qstride + m0;
    for (int kb = 0; kb < pre; ++kb) {
      unsigned char *stage = smem + kb * L::kStage;
      mbar_arrive_expect_tx(&full[kb], kALo ? L::kStage : L::kStage - L::kA);
      tma_load_2d(stage, &mapAhi, kb * kTcKBlock, ya, &full[kb]);
      if (kALo) tma_load_2d(stage + L::kA, &mapAlo, kb * kTcKBlock, ya, &full[kb]);
    }
  }
  griddep_wait();
  griddep_launch();

  // The norms the epilogue adds do not depend on the products, so they are
  // loaded before the main loop: each thread's row norm into a register, the
  // tile's column norms (chunk norms added in chunk order) into shared memory
  // by warps 2 and 3, which have nothing else to do until the epilogue.
  const bool dot = d.score_dot != 0;
  const int my_row = m0 + warp * 32 + lane;
  const float my_qn = !dot && my_row < d.drows ? s.qn[(int64_t)hh * d.qstride + my_row] : 0.f;
  if (warp >= 2 && !dot) {
    const float *kn = s.kn + (int64_t)tab * d.n * kKnChunks;
    const int nkc = (d.dh / 4 + 31) / 32;  // 128-float chunks of a sub-key row
    for (int c = threadIdx.x - 64; c < BN; c += 64) {
      float v = 0.f;
      if (n0 + c < d.n)
        for (int ch = 0; ch < nkc; ++ch) v += kn[(int64_t)(n0 + c) * kKnChunks + ch];
      kn_s[c] = v;
    }
  }

  int issued = 0;  // k-blocks whose loads the producer issued (thread 0)
  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    const int ya = hh * d.qstride + m0;  // row of the query-half tensor
    const int yb = tab * d.n + n0;       // row of the sub-key tensor
    for (int kb = 0; kb < nkb; ++kb, issued = kb) {
      const int st = kb % kTcStages, round = kb / kTcStages;
      unsigned char *stage = smem + st * L::kStage;
      const int x = kb * kTcKBlock;
      if (kb >= pre) {  // (a stage of the first round is free without waiting)
        if (!mbar_wait_bounded(&empty[st], (round & 1) ^ 1, s.meta, d.mbar_polls,
                               ERR_SCORE_TIMEOUT))
          break;
        mbar_arrive_expect_tx(&full[st], kALo ? L::kStage : L::kStage - L::kA);
        tma_load_2d(stage, &mapAhi, x, ya, &full[st]);
        if (kALo) tma_load_2d(stage + L::kA, &mapAlo, x, ya, &full[st]);
      }
      tma_load_2d(stage + 2 * L::kA, &mapBhi, x, yb, &full[st]);
      tma_load_2d(stage + 2 * L::kA + L::kB, &mapBlo, x, yb, &full[st]);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_tf32<BN>();
    bool ok = true;
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int st = kb % kTcStages, round = kb / kTcStages;
      ok = mbar_wait_bounded(&full[st], round & 1, s.meta, d.mbar_polls, ERR_SCORE_TIMEOUT);
      if (!ok) break;
      tc_fence_after();
      const unsigned char *stage = smem + st * L::kStage;
      const unsigned char *ahi = stage, *alo = stage + L::kA;
      const unsigned char *bhi = stage + 2 * L::kA, *blo = stage + 2 * L::kA + L::kB;
#pragma unroll
      for (int k8 = 0; k8 < kTcKBlock / 8; ++k8) {  // 8 tf32 = 32 bytes per MMA
        const int off = k8 * 32;
        const uint32_t acc = (kb > 0 || k8 > 0) ? 1u : 0u;
        mma_tf32(tmem, kmajor_sw128_desc(ahi + off), kmajor_sw128_desc(bhi + off), idesc, acc);
        mma_tf32(tmem, kmajor_sw128_desc(ahi + off), kmajor_sw128_desc(blo + off), idesc, 1u);
        if (kALo)
          mma_tf32(tmem, kmajor_sw128_desc(alo + off), kmajor_sw128_desc(bhi + off), idesc, 1u);
      }
      mma_commit(&empty[st]);  // stage free once these MMAs have read it
    }
    mma_commit(done);  // accumulator complete (or abandoned after an error)
  }
  __syncwarp();
  __syncthreads();  // the column norms are in shared memory

  // ---------------- epilogue: TMEM -> distances ----------------
  // Each warp owns 32 accumulator lanes (rows), one per thread, read 32
  // columns at a time.
  // warp-uniform: tcgen05.ld below is a warp-collective instruction
  const bool ready =
      __all_sync(FULL, mbar_wait_bounded(done, 0, s.meta, d.mbar_polls, ERR_SCORE_TIMEOUT));
  // After a give-up the MMAs already issued must still finish before the
  // tensor memory is released.
  if (!ready) mbar_wait_bounded(done, 0, nullptr, kDrainPolls, 0u);
  tc_fence_after();
  if (!ready) {
    // zero distances: the selection that follows still sees valid values
    float *Dh = s.D + (int64_t)hh * d.drows * d.n;
    for (int r = 0; r < 32; ++r) {
      const int row = m0 + warp * 32 + r;
      for (int c = lane; c < BN; c += 32)
        if (row < d.drows && n0 + c < d.n) Dh[(int64_t)row * d.n + n0 + c] = 0.f;
    }
  }
  if (ready) {
    // Each thread holds its own row's 32 consecutive columns: it forms their
    // distances with its row norm and stores them as 16-byte pieces (rows of
    // a length that is a multiple of 4 are 16-byte aligned), else one by one.
    float *Drow = s.D + ((int64_t)hh * d.drows + my_row) * d.n;
    const bool vec = (d.n & 3) == 0;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
      const int cbase = n0 + c0;
      const int ncols = min(min(32, BN - c0), d.n - cbase);  // columns of the tile and table
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float kn_j = !dot && c0 + j < BN ? kn_s[c0 + j] : 0.f;  // |K_col|^2
        const float dist = my_qn + kn_j - 2.f * v[j];
        v[j] = dot ? -v[j] : (dist > 0.f ? dist : 0.f);
      }
      if (my_row < d.drows) {
        if (vec && ncols == 32) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4 *>(Drow + cbase + 4 * q) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < ncols) Drow[cbase + j] = v[j];
        }
      }
    }
  }
  // Loads the producer issued that no MMA consumed (after a give-up) land
  // before the CTA exits; in a completed run every such wait returns at once.
  if (warp == 0 && lane == 0)
    for (int kb = issued > kTcStages ? issued - kTcStages : 0; kb < issued; ++kb)
      mbar_wait_bounded(&full[kb % kTcStages], (kb / kTcStages) & 1, nullptr, kDrainPolls, 0u);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// --- host side -------------------------------------------------------------
template <int BN>
static cudaError_t launch_tc(const Dims &d, const Scratch &s, const TcMaps &maps, int v,
                             cudaStream_t st) {
  auto kernel = d.q_tf32_exact ? k_score_tc<BN, false> : k_score_tc<BN, true>;
  // set on every launch: the attribute belongs to the current device's context
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       TcSmem<BN>::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((d.n + BN - 1) / BN, (d.drows + kTcRows - 1) / kTcRows, 2 * d.H);
  return launch_k(d.pdl, kernel, grid, 128, TcSmem<BN>::kBytes, st,
                  *reinterpret_cast<const CUtensorMap *>(maps.a_hi),
                  *reinterpret_cast<const CUtensorMap *>(maps.a_lo),
                  *reinterpret_cast<const CUtensorMap *>(maps.b_hi[v]),
                  *reinterpret_cast<const CUtensorMap *>(maps.b_lo[v]), d, s);
}

// Column-tile width: the widest of 128 / 64 / 32 / 16 that still gives at
// least one CTA per multiprocessor (narrower tiles when the chunk is small).
cudaError_t launch_score(const Dims &d, const Scratch &s, const TcMaps &maps, cudaStream_t st) {
  const int64_t base = (int64_t)((d.drows + kTcRows - 1) / kTcRows) * 2 * d.H;
  int bn = 128;
  while (bn > 16 && (bn >= 2 * d.n || base * ((d.n + bn - 1) / bn) < d.sm_count)) bn >>= 1;
  if (bn == 16) return launch_tc<16>(d, s, maps, 0, st);
  if (bn == 32) return launch_tc<32>(d, s, maps, 1, st);
  if (bn == 64) return launch_tc<64>(d, s, maps, 2, st);
  return launch_tc<128>(d, s, maps, 3, st);
}

// fp32 [rows][inner] tensor, box {32 elements, box_rows}, 128-byte swizzle,
// out-of-range elements read as zero.
static cudaError_t encode_2d(void *out, const float *base, uint64_t inner, uint64_t rows,
                             uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * sizeof(float)};
  const cuuint32_t box[2] = {(cuuint32_t)kTcKBlock, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(reinterpret_cast<CUtensorMap *>(out), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                            const_cast<float *>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// qstride must be a multiple of 128 and K_hi / K_lo must hold 128 rows past
// the 2*H*n sub-key rows, so that every box lies inside its tensor.
cudaError_t encode_score_maps(TcMaps *maps, const Scratch &s, int H, int nmem, int qstride,
                              int n, int dh) {
  if (qstride % kTcRows) return cudaErrorInvalidValue;
  const uint64_t qrows = 2ull * H * qstride, krows = 2ull * H * nmem * n + kTcRows;
  cudaError_t e = encode_2d(maps->a_hi, s.Qs_hi, dh, qrows, kTcRows);
  if (e == cudaSuccess) e = encode_2d(maps->a_lo, s.Qs_lo, dh, qrows, kTcRows);
  for (int v = 0; v < 4 && e == cudaSuccess; ++v) {  // column tiles of 16, 32, 64, 128
    e = encode_2d(maps->b_hi[v], s.K_hi, dh, krows, 16u << v);
    if (e == cudaSuccess) e = encode_2d(maps->b_lo[v], s.K_lo, dh, krows, 16u << v);
  }
  return e;
}

}  // namespace fwpkm
