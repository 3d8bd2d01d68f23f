// fwpkm_internal.cuh -- shared declarations of the sm_100a FwPKM kernels.
//
// Per chunk the host enqueues, in order:
//   prep    -> split the chunk's queries into halves (fp32), |q|^2, |K|^2
//   score   -> D[h][half][row][i] = |q_half - K_h,half,i|^2 for every sub-key
//   topk    -> per token-head: top-k per half, k*k merge, softmax; each pair
//              (value row) and each distinct sub-key row it uses (an "entry")
//              counts itself into a bucket and claims a position there
//   scan    -> bucket offsets
//   read    -> gather the selected value rows, out = g * yhat, residual e,
//              dL/dw per pair; scatter member ids into their buckets
//   bsort   -> sort every bucket by (group, member id)
//   apply   -> fixed 32-member tiles of the sorted array: ordered per-group
//              sums, V -= eta G / C and K -= eta dL/dK on touched rows
//   (lam > 0: apply(values) -> pgrad (softmax Jacobian) -> apply(sub-keys))
// No floating-point atomics anywhere: every sum runs in a fixed order (members
// sorted by id inside each group, tiles combined in tile order), so two runs
// are bit-identical, whatever the skew of slot usage.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

struct fwpkm_state;

namespace fwpkm {

constexpr unsigned FULL = 0xffffffffu;
// Device-side error bits (meta->err), one per kernel that can set them, so
// that a kernel checking the word at entry never sees a bit change under it:
// every bit it looks at belongs to a kernel that completed before it started.
enum : unsigned {
  ERR_READ_TIMEOUT = 1u,   // reserved: the read's wait for staged rows (it now waits for nothing)
  ERR_POOL_OVERFLOW = 2u,  // apply: more long-group blocks than the partial pool holds
  ERR_SCAN_TIMEOUT = 4u,   // a scan CTA gave up waiting for an earlier CTA's total
  ERR_SCORE_TIMEOUT = 8u,  // the score's TMA ring or MMA completion wait gave up
  ERR_SORT_OVERFLOW = 16u, // reserved: the large buckets' list holds every bucket
  ERR_ALL = 31u,
};
// Default bound of a wait (polls): a bounded wait that gives up sets its bit,
// and the kernel then still waits, up to kDrainPolls, for its own copies in
// flight before it returns.
constexpr long long kDefaultMbarPolls = 1ll << 26;
constexpr long long kDefaultScanPolls = 1ll << 24;
constexpr long long kDrainPolls = 1ll << 26;

// Written by the kernels, read by later kernels and by the host.
struct Meta {
  int32_t L;              // members of the chunk (pairs + sub-key entries)
  int32_t nbig;           // buckets of more than 32 members, listed by the scan in biglist
  unsigned err;           // ERR_* bits, sticky until the host clears them
  // Work lists of the chunk, per kind (0: value rows, 1: sub-key rows),
  // reset per chunk by the scan:
  int32_t nshort[2];      // groups of <= 4 members in shortlist[kind]
  int32_t nlong[2];       // 32-member blocks of longer groups in longlist[kind]
  int32_t pad2[2];
  unsigned long long stat_chunks;      // chunks processed since reset
  unsigned long long stat_value_rows;  // sum over chunks of distinct value rows written
  unsigned long long stat_key_rows;    // sum over chunks of distinct sub-key rows written
  unsigned long long stat_records;     // sum over chunks of member records (pairs + entries)
};

// Shapes of the chunk being processed.
struct Dims {
  int n, dq, dh, dv, k, H;
  int64_t N;
  int B, T, t0, Tc;   // batch, call length, first token of the chunk, its length
  int rows;           // B * Tc
  int qstride;        // row stride of the query-half arrays (capacity rows)
  int M;              // rows * H token-heads
  int NBv;            // value buckets: slot >> vshift
  int vshift;
  int NB;             // NBv value buckets + 2*H*n sub-key rows
  int sm_count;       // multiprocessors of the device (grid sizing)
  int pdl;            // launch with programmatic dependent launch (see launch_k)
  float eps, eta, lam;
  long long mbar_polls;  // bound of the first wait on an mbarrier (the score's ring and MMAs)
  long long scan_polls;  // bound of a scan CTA's wait for an earlier CTA's total
  int lookahead;         // token t is written towards the target of token t+1
  int q_tf32_exact;      // the queries are bf16, so exact in TF32 (their lo part is zero)
  // Memories: 1 (all sequences share the one memory), or one per sequence
  // (sequence b reads and writes memory b: sub-key tables b*H .. b*H+H-1,
  // value rows b*N .. b*N+N-1).
  int nmem;
  int64_t Nt;            // value rows of all memories, nmem * N
  int rstride;           // rows per sequence in the query-half and distance layouts
  int drows;             // B * rstride: rows of those layouts
  int Mmem;              // token-heads per memory, M / nmem
  int heads_sum;         // head readouts summed instead of averaged
  int readonly;          // eta = 0: the read alone (no claims, entries, records, gradients)
  int agg;               // divisor of a value row's gradient (AGG_*)
  int score_dot;         // sub-key score q . K (D holds -q.K) instead of the IDW one
  int q_early;           // the query halves come from a grid two or more before the score
                         // (the previous chunk's sort): loading them needs no wait
};
// Divisor of a value row's gradient: its row contribution C_i = sum of w/H
// (the sum of its members' c0), its access count (every member's c0 is 1), or
// none.
enum { AGG_WEIGHT = 0, AGG_COUNT = 1, AGG_SUM = 2 };

// Device scratch owned by the state (sized for the largest chunk seen).
constexpr int kScanMaxCtas = 64;  // bucket-scan CTAs: 64 x 2048 buckets
constexpr int kKnChunks = 8;     // 128-float chunks of a sub-key row (dq/2 <= 1024)
constexpr int kMaxChunks = 16;   // 128-float column chunks of the widest row (2048 floats)
constexpr int kPartHead = 2 * kMaxChunks;  // partial slot header: (C, W) per column chunk

struct Scratch {
  float *Qs_hi;     // [H][2][qstride][dh] TF32-rounded query halves
  float *Qs_lo;     // [H][2][qstride][dh] query halves minus their TF32 part
  float *qn;        // [H][2][qstride]     |q_half|^2
  float *K_hi;      // [H][2][n][dh] + 128 padding rows: TF32-rounded sub-keys
  float *K_lo;      // same shape: sub-keys minus their TF32 part
  float *kn;        // [H][2][n][kKnChunks] |K_row|^2 of each 128-float chunk of the row
                    // (chunk_sqnorm); the row's norm is their sum in chunk order
  float *D;         // [H][2][rows][n]    squared distances
  int32_t *pslot;   // [M*k] selected slot of pair p = m*k + r
  float *pw;        // [M*k] softmax weight
  int32_t *pclaim;  // [M*k] position inside the pair's bucket
  float *pa;        // [M*k] dL_mse/dw
  float *pb;        // [M*k] dL_addr/dw (lam > 0)
  int32_t *esub;    // [2*M*k] sub-key row of entry e = (m*2+half)*k + idx; -1 past ecount
  uint32_t *emask;  // [2*M*k] pairs r of token-head m that use that row
  float *einv;      // [2*M*k] 1 / (eps + d_half(row))
  int32_t *eclaim;  // [2*M*k] position inside the entry's bucket
  float *ealpha;    // [2*M*k] sum of dL/ds over the entry's pairs / (eps + d) (pgrad,
                    // with the entropy term on; else the read puts it in the record)
  int32_t *ecount;  // [M*2]   entries per (m, half)
  int32_t *bcnt;    // [NB]    members per bucket (zero between chunks)
  int32_t *boff;    // [NB+1]  bucket offsets into rec_in / rec
  struct Member *rec_in;  // [Lcap] member records in bucket (claim) order
  struct Member *rec;     // [Lcap] the same records sorted by (group, id)
  uint64_t *sort_tmp;  // [2*Lcap] merge buffers for oversized buckets
  int32_t *posmap;  // [Lcap]  position inside its bucket, by member id (oversized buckets)
  int32_t *shortlist[2];  // [Lcap] per kind: first position of every group of <= 4 members
  int32_t *biglist;       // [NB] buckets of more than 32 members (the scan lists them)
  int32_t *longlist[2];   // [Lcap] per kind: first position of every 32-member block of a
                          //        longer group (a group's blocks are consecutive)
  int32_t *arrive;        // [pool_cap][kMaxChunks] blocks of a longer group done with a
                          //        column chunk, at the group's first block (reset to 0)
  // Cross-CTA state of the bucket scan, never reset by the host: [0] the
  // chunk epoch (advanced by the selection), [1 + c] CTA c's total tagged
  // with the epoch it belongs to.
  unsigned long long *scan_sync;  // [1 + kScanMaxCtas]
  float *partial;   // [pool_cap][pwidth] block partial sums: value blocks at their longlist
                    // index, sub-key blocks after all value blocks; a header of
                    // kPartHead floats (the block's scalar sums per column chunk), then the row
                    // (zero between chunks)
  float *E;         // [rows][dv] residual yhat - v
  Meta *meta;
  int64_t Lcap;     // member capacity (3 * M*k)
  int pwidth;       // kPartHead + max(dv, dh) floats
  int pool_cap;     // partial slots: Lcap / 4 + 2
};

// One member of a group (32 bytes).  Value rows: a pair p; sub-key rows: an
// entry e.  Written by the read kernel into the member's bucket, sorted by
// (g, id) and completed (gstart, glen) by the bucket sort.
struct __align__(16) Member {
  uint32_t g;      // group: slot (< N) or N + (h*2+half)*n + row
  uint32_t id;     // pair id p = m*k + r, or entry id e = (m*2+half)*k + idx
  int32_t srow;    // source row: E row (value rows); for sub-key rows the query half
                   // tok*2H + h*2 + half of the caller's Q (element offset srow * dq/2)
  int32_t gstart;  // position of the group's first member
  float coef;      // value rows: 2 g_t w / H; sub-key rows: alpha (lam == 0)
  float c0;        // value rows: w / H;       sub-key rows: alpha
  float c1;        // value rows: w
  int32_t glen;    // members in the group
};

// Optional per-step inputs/outputs.
struct Extras {
  const int32_t *force_slots;  // [B][T][H][k] or null
  const uint8_t *force_mask;   // [B][T][H]
  int32_t *rec_slots;          // [B][T][H][k] or null
  float *rec_w;
};

// ------------------------------------------------------------------------
// Device helpers
// ------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
  return v;
}
__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ float load_elem(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16 *p, int64_t i) {
  return __bfloat162float(p[i]);
}
// Four consecutive elements starting at a multiple of 4.
__device__ __forceinline__ float4 load4(const float *p, int64_t i) {
  return *reinterpret_cast<const float4 *>(p + i);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p, int64_t i) {
  uint2 raw = *reinterpret_cast<const uint2 *>(p + i);
  __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
  __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
  float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}

// --- mbarrier + bulk async copy (TMA, non-tensor form) -------------------
// TF32 part of x (round to nearest); x - tf32_part(x) is the remainder.
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
// Squared norm of a 128-float chunk held as one float4 per lane (lane l:
// floats 4l .. 4l+3; lanes past the row's end hold zeros), summed in a fixed
// order; every lane gets the same value.  The prep and the update both use
// it, so a sub-key row's norm does not depend on which of them wrote it.
__device__ __forceinline__ float chunk_sqnorm(const float4 &v) {
  float a = fmaf(v.w, v.w, fmaf(v.z, v.z, fmaf(v.y, v.y, v.x * v.x)));
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  return a;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: gives up after `limit` polls (each try_wait may itself block
// for a hardware-defined interval), records `bit` in meta->err (when meta is
// not null) and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, unsigned parity, Meta *meta,
                                                  long long limit, unsigned bit) {
  for (long long it = 0; it < limit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  if (meta) atomicOr(&meta->err, bit);
  return false;
}
// Error bits set by kernels that ran before the caller (its `own` bits
// excluded): a kernel after the bucket scan returns at entry, writing
// nothing, when one is set, since the chunk's offsets or selection may then
// be wrong.  The word is sticky, so the rest of the call is skipped too.
__device__ __forceinline__ bool chunk_aborted(const Scratch &s, unsigned own) {
  return (*reinterpret_cast<volatile const unsigned *>(&s.meta->err) & (ERR_ALL & ~own)) != 0u;
}
// Memory of token row `row` (b * Tc + tl) of chunk d, and the row's place in
// the query-half and distance layouts (b * rstride + tl: with one memory per
// sequence every sequence starts a new 128-row score tile, so that a tile
// scores against one memory's sub-keys).
__device__ __forceinline__ int mem_of(const Dims &d, int row) {
  return d.nmem > 1 ? row / d.Tc : 0;
}
__device__ __forceinline__ int lrow_of(const Dims &d, int row) {
  return (row / d.Tc) * d.rstride + row % d.Tc;
}

// One query half (warp w = (h*2 + half)*rows + row of chunk d) into its TF32
// split and squared norm: Qs_hi / Qs_lo [h][half][lrow][:], qn (rows at
// stride qstride).  Warp-level; used by the prep and by the bucket sort's
// CTAs before their grid dependency wait (the next chunk's halves).
template <typename TQ>
__device__ __forceinline__ void prep_query_half(const Dims &d, const TQ *__restrict__ Q,
                                                const Scratch &s, int64_t w) {
  const int lane = threadIdx.x & 31;
  const int dh = d.dh;
  const int hh = (int)(w / d.rows);  // h*2 + half
  const int row = (int)(w % d.rows);
  const int h = hh >> 1, half = hh & 1;
  const int b = row / d.Tc, tl = row % d.Tc;
  const int64_t src = ((int64_t)b * d.T + d.t0 + tl) * ((int64_t)d.H * d.dq) +
                      (int64_t)h * d.dq + (int64_t)half * dh;
  const int64_t o = ((int64_t)hh * d.qstride + lrow_of(d, row)) * dh;
  float acc = 0.f;
  for (int c = lane * 4; c < dh; c += 128) {
    const float4 v = load4(Q, src + c);
    // a bf16 value is its own TF32 part: no remainder to write (the score
    // skips the remainder's product for bf16 queries)
    if (sizeof(TQ) == 2) *reinterpret_cast<float4 *>(s.Qs_hi + o + c) = v;
    else split_store(s.Qs_hi + o, s.Qs_lo + o, c, v);
    acc = fmaf(v.x, v.x, acc);
    acc = fmaf(v.y, v.y, acc);
    acc = fmaf(v.z, v.z, acc);
    acc = fmaf(v.w, v.w, acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) s.qn[(int64_t)hh * d.qstride + lrow_of(d, row)] = acc;
}

// Programmatic dependent launch.  A kernel started by launch_k with d.pdl set
// may become resident while its predecessor on the stream is still running;
// griddep_wait() blocks until that predecessor has completed and its writes
// are visible, so a kernel calls it before it reads anything its predecessor
// writes, and griddep_launch() early, letting its own successor get
// scheduled.  A grid is launched only after every CTA of the one before has
// called griddep_launch().  Every kernel here calls it right after its own
// wait, except the read of the write path, which calls it first (it waits
// only before its member records).  So when a kernel starts, every grid
// before its predecessor has completed, except that the sort, which follows
// the read, may start while the scan still runs.  Three kernels read before
// their wait and rely on exactly that: the read on the selection's output (two
// back), the score on the query halves the previous chunk's sort made (two
// back), and the sort only on the caller's Q and on query-half storage last
// read by the score (four back).  Both are no-ops for a kernel launched
// without the attribute.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch with optional programmatic dependent launch and a thread-block
// cluster of `cluster` CTAs along x (1 = no cluster).
template <typename... KArgs, typename... Args>
cudaError_t launch_kc(bool pdl, int cluster, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                      size_t smem, cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_k(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, Args &&...args) {
  return launch_kc(pdl, 1, kernel, grid, block, smem, st, static_cast<Args &&>(args)...);
}

// ------------------------------------------------------------------------
// Host-side launchers (one per kernel file)
// ------------------------------------------------------------------------
// Query halves and sub-key rows of one chunk (the selection-only entry point).
cudaError_t launch_prep(const Dims &d, const void *Q, int q_dtype, const float *K,
                        const Scratch &s, cudaStream_t st);
// Query halves of one chunk only (the sub-key split is kept by the update).
cudaError_t launch_prep_q(const Dims &d, const void *Q, int q_dtype, const Scratch &s,
                          cudaStream_t st);
// Sub-key rows only (after the tables are set or the scratch is new).
cudaError_t launch_prep_k(const Dims &d, const float *K, const Scratch &s, cudaStream_t st);
// TMA descriptors (CUtensorMap, 128 bytes each) of the score operands.
struct TcMaps {
  alignas(64) unsigned char a_hi[128];
  alignas(64) unsigned char a_lo[128];
  alignas(64) unsigned char b_hi[4][128];  // column tiles of 16, 32, 64, 128
  alignas(64) unsigned char b_lo[4][128];
};
// Encodes the four maps over Qs_hi / Qs_lo ([2H*qstride][dh], qstride a
// multiple of 128) and K_hi / K_lo ([2H*nmem*n + 128][dh]).  Host only;
// returns a CUDA error code.
cudaError_t encode_score_maps(TcMaps *maps, const Scratch &s, int H, int nmem, int qstride,
                              int n, int dh);
cudaError_t launch_score(const Dims &d, const Scratch &s, const TcMaps &maps, cudaStream_t st);
cudaError_t launch_topk(const Dims &d, const Scratch &s, const Extras &x, cudaStream_t st);
// Selection only: fills x.rec_slots / x.rec_w from the distances in s.D.
cudaError_t launch_topk_select(const Dims &d, const Scratch &s, const Extras &x,
                               cudaStream_t st);
cudaError_t launch_scan(const Dims &d, const Scratch &s, cudaStream_t st);
// omega: the tokens' MSE weights [B][T] (null: the gate).
cudaError_t launch_read(const Dims &d, const float *V, const void *Vt, int v_dtype,
                        const float *gate, const float *omega, float *out, const Scratch &s,
                        cudaStream_t st);
// CTAs per token of the read at these shapes (1 unless a token's rows exceed 1 MB).
int read_cluster_size(const Dims &d);
// The bucket sort; with dn.rows > 0 its CTAs first prepare the query halves
// of the next chunk dn (nothing reads this chunk's halves after the score).
cudaError_t launch_bsort(const Dims &d, const Scratch &s, const Dims &dn, const void *Q,
                         int q_dtype, cudaStream_t st);
// part 0: all groups; 1: value rows only; 2: sub-key rows only.  Sub-key
// sources are the caller's query halves Q (q_dtype); updated sub-key rows get
// their TF32 split and chunk norms rewritten.
cudaError_t launch_apply(const Dims &d, float *V, float *K, const void *Q, int q_dtype,
                         const Scratch &s, cudaStream_t st, int part);
cudaError_t launch_pgrad(const Dims &d, const Scratch &s, cudaStream_t st);

// Read-only view of a state's shape and sub-key tables (fwpkm_abi.cu).
struct StateView {
  int64_t N;
  int n, dq, dh, dv, k, chunk, H, device, sm_count, nmem;
  float eps;
  const float *K;
  long long mbar_polls;
  int score_dot;
};
bool state_view(const struct ::fwpkm_state *st, StateView *v);
// Records `msg` as the calling thread's last error (fwpkm_last_error).
void set_last_error(const char *msg);

}  // namespace fwpkm
