// Runtime of the TTT-E2E inner loop: device state, the prefill schedule
// (Algorithm 1 of the technical review, §7) and the decode schedule
// (Algorithm 3), behind the C ABI declared in include/ttt.h.
//
// Schedule of one prefill call over T positions of B sequences:
//   for each segment of S positions (S a multiple of b):
//     frozen phase: embedding, then every frozen block over all B*S rows at
//       once (ordinary parallel sliding-window prefill; the frozen blocks do
//       not depend on the fast weights);
//     adaptive phase: for each chunk of b positions, in order (the chain
//       W_{i-1} -> loss_i -> grad -> W_i is serial):
//       forward of the adaptive blocks with W_{i-1}, LM head + cross-entropy
//       (losses recorded before any update), backward into every adaptive
//       MLP's weights, and the SGD update fused into the weight-gradient GEMM.
// Window caches: per layer and sequence a ring of C = roundup(k + b, 128)
// positions. Rows of the current segment/chunk are read directly; older
// positions from the ring. K/V are appended after use and never recomputed.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "ttt.h"
#include "ttt_devmem.h"
#include "ttt_testing.h"
#include "ttt_attention.cuh"
#include "ttt_attention_mma.cuh"
#include "ttt_attention_tc.cuh"
#include "ttt_common.cuh"
#include "ttt_gemm.cuh"
#include "ttt_ops.cuh"

namespace ttt {

// ============================================================== launch helper
// Launch with programmatic stream serialisation (the kernel must call pdl_wait()
// before touching global memory; see ttt_common.cuh).
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Row-kernel launches (PDL): RMSNorm with row_threads(d) threads per row in
// blocks of 256; RoPE with one thread per 8 pairs.
template <typename T>
static cudaError_t rmsnorm_fwd_launch(const float* x, int64_t ldx, const float* g, float eps, int rows, int d, T* y,
                                      int64_t ldy, float* rstd, cudaStream_t st) {
  const int tpr = row_threads(d), rpb = 256 / tpr;
  const dim3 grid((unsigned)((rows + rpb - 1) / rpb)), blk(256);
  switch (tpr) {
    case 256: return launch_pdl(rmsnorm_fwd_kernel<T, 256>, grid, blk, 0, st, x, ldx, g, eps, rows, d, y, ldy, rstd);
    case 128: return launch_pdl(rmsnorm_fwd_kernel<T, 128>, grid, blk, 0, st, x, ldx, g, eps, rows, d, y, ldy, rstd);
    case 64: return launch_pdl(rmsnorm_fwd_kernel<T, 64>, grid, blk, 0, st, x, ldx, g, eps, rows, d, y, ldy, rstd);
    default: return launch_pdl(rmsnorm_fwd_kernel<T, 32>, grid, blk, 0, st, x, ldx, g, eps, rows, d, y, ldy, rstd);
  }
}

template <typename T>
static cudaError_t rmsnorm_bwd_launch(const float* x, const float* g, const float* rstd, const float* dy,
                                      const float* dres, int rows, int d, float* dx, T* dx_t, cudaStream_t st) {
  const int tpr = row_threads(d), rpb = 256 / tpr;
  const dim3 grid((unsigned)((rows + rpb - 1) / rpb)), blk(256);
  switch (tpr) {
    case 256: return launch_pdl(rmsnorm_bwd_kernel<T, 256>, grid, blk, 0, st, x, g, rstd, dy, dres, rows, d, dx, dx_t);
    case 128: return launch_pdl(rmsnorm_bwd_kernel<T, 128>, grid, blk, 0, st, x, g, rstd, dy, dres, rows, d, dx, dx_t);
    case 64: return launch_pdl(rmsnorm_bwd_kernel<T, 64>, grid, blk, 0, st, x, g, rstd, dy, dres, rows, d, dx, dx_t);
    default: return launch_pdl(rmsnorm_bwd_kernel<T, 32>, grid, blk, 0, st, x, g, rstd, dy, dres, rows, d, dx, dx_t);
  }
}

template <typename T>
static cudaError_t rope_launch(T* qk, int64_t ld, int ncols, int rows, int n, int64_t pos0, int hd,
                               const float2* lo, const float2* hi, int inverse, const int64_t* pos_dev,
                               cudaStream_t st, void* ring_k = nullptr, void* ring_v = nullptr, int C = 0) {
  const int64_t threads = rope_threads(rows, ncols, hd);
  if (threads >= (int64_t)INT32_MAX || ncols % hd) return cudaErrorInvalidValue;
  return launch_pdl(rope_kernel<T>, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, st, qk, ld, ncols, rows,
                    n, pos0, hd, lo, hi, inverse, pos_dev, (T*)ring_k, (T*)ring_v, C);
}

// ============================================================== GEMM dispatch (host)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)ptr;
  }
  return fn;
}

// Operand map: logical [rows][K] (K-major, box {64, box_rows}) or logical [rows][K]
// stored [K][rows] (MN-major, box {64, 64}). 128-byte swizzle, zero fill out of range.
static bool make_operand_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int64_t ld,
                             int64_t batch, int64_t bstride, bool mn_major, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  if (!mn_major) {
    dims[0] = (cuuint64_t)K; dims[1] = (cuuint64_t)rows;
    box[0] = 64; box[1] = (cuuint32_t)box_rows;
  } else {
    dims[0] = (cuuint64_t)rows; dims[1] = (cuuint64_t)K;
    box[0] = 64; box[1] = 64;
  }
  dims[2] = (cuuint64_t)batch;
  box[2] = 1;
  if (bstride == 0) batch = 1;  // shared operand: one slice, always read at batch index 0
  dims[2] = (cuuint64_t)batch;
  strides[0] = (cuuint64_t)ld * 2;
  strides[1] = (cuuint64_t)(batch > 1 ? bstride : (mn_major ? K : rows) * ld) * 2;
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// Single-CTA tcgen05 launch of one product, or of two (p2) in one persistent grid.
template <int BN, bool AM, bool BM>
static cudaError_t launch_tc(const GemmParams& p, cudaStream_t st, int* err, int num_sms, bool* ok,
                             const GemmParams* p2 = nullptr) {
  TcGroup g;
  memset(&g, 0, sizeof(g));
  g.nprob = p2 ? 2 : 1;
  const GemmParams* ps[2] = {&p, p2};
  *ok = true;
  int tiles = 0;
  for (int i = 0; i < g.nprob && *ok; ++i) {
    const GemmParams& q = *ps[i];
    *ok = make_operand_map(&g.tmA[i], q.A, q.M, q.K, q.lda, q.batch, q.sA, AM, TC_BM) &&
          make_operand_map(&g.tmB[i], q.B, q.N, q.K, q.ldb, q.batch, q.sB, BM, BN);
    if (*ok && q.B2) *ok = make_operand_map(&g.tmB2[i], q.B2, q.N, q.K, q.ldb, q.batch, q.sB2, BM, BN);
    else g.tmB2[i] = g.tmB[i];
    g.p[i] = q;
    tiles += ((q.M + TC_BM - 1) / TC_BM) * (q.N / BN) * q.batch;
  }
  if (!*ok) return cudaSuccess;
  using C = TcCfg<BN>;
  const int grid = tiles < num_sms ? tiles : num_sms;
  return launch_pdl(gemm_tc_kernel<BN, AM, BM>, dim3(grid), dim3(TC_THREADS), C::SMEM, st, g, err);
}

// Pairs of CTAs that can be resident at once for one paired-GEMM variant (0 = the
// device cannot place them; then the single-CTA kernel runs). Queried once.
template <int BN, bool AM, bool BM> static int pair_capacity() {
  static int cap = -1;
  if (cap < 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = Tc2Cfg<BN>::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<BN, AM, BM>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cap = n;
  }
  return cap;
}

// Clusters of the K-split kernel that can be resident at once (0: cannot be placed).
template <int BN, bool AM, bool BM> static int tck_capacity() {
  static int cap = -1;
  if (cap < 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = TcCfg<BN>::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_tck_kernel<BN, AM, BM>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cap = n;
  }
  return cap;
}

// K split over a CTA pair, one 128 x BN tile per cluster (gemm_tck_kernel). The caller
// has checked that the k-block count (doubled with B2) is even.
template <int BN, bool AM, bool BM>
static cudaError_t launch_tck(const GemmParams& p, cudaStream_t st, int* err, bool* ok) {
  CUtensorMap ta, tb, tb2;
  *ok = tck_capacity<BN, AM, BM>() > 0 && make_operand_map(&ta, p.A, p.M, p.K, p.lda, p.batch, p.sA, AM, TC_BM) &&
        make_operand_map(&tb, p.B, p.N, p.K, p.ldb, p.batch, p.sB, BM, BN);
  if (*ok && p.B2) *ok = make_operand_map(&tb2, p.B2, p.N, p.K, p.ldb, p.batch, p.sB2, BM, BN);
  else tb2 = tb;
  if (!*ok) return cudaSuccess;
  const int tiles = ((p.M + TC_BM - 1) / TC_BM) * (p.N / BN) * p.batch;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * tiles);
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = TcCfg<BN>::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_tck_kernel<BN, AM, BM>, ta, tb, tb2, p, err);
}

template <int BN, bool AM, bool BM>
static cudaError_t launch_tc2(const GemmParams& p, cudaStream_t st, int* err, bool* ok) {
  CUtensorMap ta, tb, tb2;
  *ok = make_operand_map(&ta, p.A, p.M, p.K, p.lda, p.batch, p.sA, AM, TC_BM) &&
        make_operand_map(&tb, p.B, p.N, p.K, p.ldb, p.batch, p.sB, BM, BN / 2);
  if (*ok && p.B2) *ok = make_operand_map(&tb2, p.B2, p.N, p.K, p.ldb, p.batch, p.sB2, BM, BN / 2);
  else tb2 = tb;
  if (!*ok) return cudaSuccess;
  const int cap = pair_capacity<BN, AM, BM>();
  if (cap <= 0) {
    *ok = false;
    return cudaSuccess;
  }
  const int tiles = ((p.M + 2 * TC_BM - 1) / (2 * TC_BM)) * (p.N / BN) * p.batch;
  const int pairs = tiles < cap ? tiles : cap;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = Tc2Cfg<BN>::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<BN, AM, BM>, ta, tb, tb2, p, err);
}

// ============================================================== tcgen05 attention (host)
bool attn_tc_ok(const AttnParams& p) {
  return (p.hd == 64 || p.hd == 128) && p.q0 % 128 == 0 && (p.q0 == 0 || p.C % 128 == 0) && p.d % 64 == 0 &&
         p.ldq == 3 * p.d && p.ldkv == 3 * p.d && (const char*)p.K == (const char*)p.Q + 2 * p.d &&
         aligned16(p.Q) && (p.q0 == 0 || (aligned16(p.Kc) && aligned16(p.Vc))) && p.n >= 1;
}

// Rows of 'inner' bf16 elements, 'rows' rows, box {64, box_rows}, 128-byte swizzle.
static bool make_rows_map(CUtensorMap* map, const void* base, int64_t inner, int64_t rows, int box_rows = 128) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, 1};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)(inner * rows * 2)};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1}, estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Returns cudaSuccess and sets *ok = false when the maps cannot be built (caller falls back).
cudaError_t attn_fwd_tc_launch(const AttnParams& p, cudaStream_t st, int* err, bool* ok) {
  CUtensorMap tq, tk, tv;
  *ok = make_rows_map(&tq, p.Q, 3 * p.d, (int64_t)p.B * p.n);
  if (*ok && p.q0 > 0) {
    *ok = make_rows_map(&tk, p.Kc, p.d, (int64_t)p.B * p.C) && make_rows_map(&tv, p.Vc, p.d, (int64_t)p.B * p.C);
  } else {
    tk = tq;
    tv = tq;
  }
  if (!*ok) return cudaSuccess;
  dim3 grid((p.n + 127) / 128, p.H, p.B);
  if (p.hd == 128) return launch_pdl(attn_fwd_tc_kernel<128>, grid, dim3(192), AttnTcCfg<128>::SMEM, st, tq, tk, tv, p, err);
  return launch_pdl(attn_fwd_tc_kernel<64>, grid, dim3(192), AttnTcCfg<64>::SMEM, st, tq, tk, tv, p, err);
}

bool attn_dq_tc_ok(const AttnParams& p) {
  return attn_tc_ok(p) && p.lddo == p.d && aligned16(p.dO) && aligned16(p.dQ) && p.lddq % 8 == 0;
}

cudaError_t attn_bwd_dq_tc_launch(const AttnParams& p, cudaStream_t st, int* err, bool* ok) {
  CUtensorMap tq, tkv, tk, tv, tdo;  // Q and dO in 128-row boxes, K and V in 64-row boxes
  *ok = make_rows_map(&tq, p.Q, 3 * p.d, (int64_t)p.B * p.n) &&
        make_rows_map(&tkv, p.Q, 3 * p.d, (int64_t)p.B * p.n, 64) &&
        make_rows_map(&tdo, p.dO, p.d, (int64_t)p.B * p.n);
  if (*ok && p.q0 > 0) {
    *ok = make_rows_map(&tk, p.Kc, p.d, (int64_t)p.B * p.C, 64) &&
          make_rows_map(&tv, p.Vc, p.d, (int64_t)p.B * p.C, 64);
  } else {
    tk = tkv;
    tv = tkv;
  }
  if (!*ok) return cudaSuccess;
  dim3 grid((p.n + 127) / 128, p.H, p.B);
  if (p.hd == 128)
    return launch_pdl(attn_bwd_dq_tc_kernel<128>, grid, dim3(192), AttnDqCfg<128>::SMEM, st, tq, tkv, tk, tv, tdo,
                      p, err);
  return launch_pdl(attn_bwd_dq_tc_kernel<64>, grid, dim3(192), AttnDqCfg<64>::SMEM, st, tq, tkv, tk, tv, tdo, p,
                    err);
}

bool attn_dkv_tc_ok(const AttnParams& p) {
  return attn_dq_tc_ok(p) && aligned16(p.dK) && aligned16(p.dV) && p.window >= 1;
}

cudaError_t attn_bwd_dkv_tc_launch(const AttnParams& p, cudaStream_t st, int* err, bool* ok) {
  CUtensorMap tk, tq, tdo;  // K and V in 128-row boxes, Q and dO in 64-row boxes
  *ok = make_rows_map(&tk, p.Q, 3 * p.d, (int64_t)p.B * p.n) &&
        make_rows_map(&tq, p.Q, 3 * p.d, (int64_t)p.B * p.n, 64) &&
        make_rows_map(&tdo, p.dO, p.d, (int64_t)p.B * p.n, 64);
  if (!*ok) return cudaSuccess;
  dim3 grid((p.n + 127) / 128, p.H, p.B);
  if (p.hd == 128)
    return launch_pdl(attn_bwd_dkv_tc_kernel<128>, grid, dim3(192), AttnDkvCfg<128>::SMEM, st, tk, tq, tdo, p, err);
  return launch_pdl(attn_bwd_dkv_tc_kernel<64>, grid, dim3(192), AttnDkvCfg<64>::SMEM, st, tk, tq, tdo, p, err);
}

// Dynamic shared-memory limits of every large-smem kernel, set once per process
// before any launch (and so never inside a CUDA graph capture).
template <int BN, bool AM, bool BM> static cudaError_t tc_attr() {
  const cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, AM, BM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             TcCfg<BN>::SMEM);
  if (e != cudaSuccess) return e;
  const cudaError_t e2 = cudaFuncSetAttribute(gemm_tck_kernel<BN, AM, BM>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<BN>::SMEM);
  if (e2 != cudaSuccess) return e2;
  return cudaFuncSetAttribute(gemm_tc2_kernel<BN, AM, BM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Tc2Cfg<BN>::SMEM);
}
int prime_kernel_attributes() {
  static int done = 0;
  if (done) return 0;
  cudaError_t e = cudaSuccess;
  const cudaError_t r[] = {tc_attr<128, false, false>(), tc_attr<256, false, false>(), tc_attr<128, false, true>(),
                           tc_attr<256, false, true>(),  tc_attr<128, true, true>(),   tc_attr<256, true, true>(),
                           attn_mma_attributes<64>(),    attn_mma_attributes<128>(),
                           cudaFuncSetAttribute(gemm_rows_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                RW_SMEM_MAX),
                           cudaFuncSetAttribute(gemm_rows_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                RW_SMEM_MAX),
                           cudaFuncSetAttribute(gemm_rows_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                RW_SMEM_MAX),
                           cudaFuncSetAttribute(attn_fwd_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                AttnTcCfg<64>::SMEM),
                           cudaFuncSetAttribute(attn_fwd_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                AttnTcCfg<128>::SMEM),
                           cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                AttnDqCfg<64>::SMEM),
                           cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<128>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, AttnDqCfg<128>::SMEM),
                           cudaFuncSetAttribute(attn_bwd_dkv_tc_kernel<64>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, AttnDkvCfg<64>::SMEM),
                           cudaFuncSetAttribute(attn_bwd_dkv_tc_kernel<128>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, AttnDkvCfg<128>::SMEM)};
  for (cudaError_t x : r)
    if (x != cudaSuccess) e = x;
  if (e != cudaSuccess) return (int)e;
  // resident-pair counts of the paired GEMMs, queried now rather than at a first launch
  pair_capacity<128, false, false>(); pair_capacity<256, false, false>(); pair_capacity<128, false, true>();
  pair_capacity<256, false, true>();  pair_capacity<128, true, true>();   pair_capacity<256, true, true>();
  tck_capacity<256, false, false>();  tck_capacity<256, false, true>();   tck_capacity<256, true, true>();
  done = 1;
  return 0;
}

// Few rows per slice (decode): skinny kernel, all SMs streaming the weight rows.
static bool skinny_ok(const GemmParams& p, int elem_is_bf16) {
  const size_t vec = elem_is_bf16 ? 8 : 4;
  return p.M <= SK_MAXM && p.epi != EPI_CE && !p.a_mn && !p.b_mn && p.K % vec == 0 && p.lda % vec == 0 &&
         p.ldb % vec == 0 && aligned16(p.A) && aligned16(p.B) && (!p.B2 || aligned16(p.B2)) &&
         (p.batch == 1 || (p.sA % vec == 0 && p.sB % vec == 0 && p.sB2 % vec == 0));
}

// Shapes, layouts and alignments the tcgen05 engine takes.
static bool tc_ok(const GemmParams& p, int elem_is_bf16) {
  bool ok = elem_is_bf16 && (p.K % TC_BK == 0) && (p.N % 128 == 0) && aligned16(p.A) && aligned16(p.B) &&
            aligned16(p.D) && (p.lda % 8 == 0) && (p.ldb % 8 == 0) &&
            (p.ldd % (p.d_f32 || p.epi == EPI_RESID || p.epi == EPI_SGD ? 4 : 8) == 0) &&
            (p.batch == 1 || (p.sA % 8 == 0 && p.sB % 8 == 0 && p.sB2 % 8 == 0)) && (!p.a_mn || p.b_mn) &&
            p.M >= 1 && (!p.B2 || aligned16(p.B2));
  if (ok && p.X && !(aligned16(p.X) && p.ldx % (p.epi == EPI_DGELU ? 8 : 4) == 0 && (p.batch == 1 || p.sX % 8 == 0)))
    ok = false;
  if (ok && p.batch > 1 && p.sD % 8 != 0) ok = false;
  if (ok && p.Y && !(aligned16(p.Y) && p.ldy % 8 == 0 && (p.batch == 1 || p.sY % 8 == 0))) ok = false;
  if (ok && p.epi == EPI_CE && !(p.batch == 1 && !p.d_f32 && p.ce_tgt && p.ce_part && p.ce_zt)) ok = false;
  return ok;
}

// Two independent products on one stream: one grouped single-CTA tcgen05 launch where
// both fit it with the same operand layouts and 256-wide tiles (the CTAs then overlap
// one product's epilogues with the other's mainloop), else two launches.
int gemm_launch_pair(const GemmParams& a, const GemmParams& b, int elem_is_bf16, cudaStream_t st, int* err,
                     int num_sms) {
  const bool grp = elem_is_bf16 && a.epi != EPI_CE && b.epi != EPI_CE && a.epi != EPI_QKV_ROPE &&
                   b.epi != EPI_QKV_ROPE && !a.norm_x && !b.norm_x && a.a_mn == b.a_mn && a.b_mn == b.b_mn &&
                   a.N % 256 == 0 && b.N % 256 == 0 && a.M > 0 && b.M > 0 && a.batch > 0 && b.batch > 0 &&
                   gemm_uses_tc(a, 1) && gemm_uses_tc(b, 1);
  if (grp) {
    GemmParams x = a, y = b;  // walk the larger operand of each once (as gemm_launch does)
    x.m_fast = x.N > x.M ? 1 : 0;
    y.m_fast = y.N > y.M ? 1 : 0;
    bool ok = false;
    cudaError_t e;
    if (!a.a_mn && !a.b_mn) e = launch_tc<256, false, false>(x, st, err, num_sms, &ok, &y);
    else if (!a.a_mn && a.b_mn) e = launch_tc<256, false, true>(x, st, err, num_sms, &ok, &y);
    else e = launch_tc<256, true, true>(x, st, err, num_sms, &ok, &y);
    if (e != cudaSuccess) return (int)e;
    if (ok) return 0;
  }
  const int e = gemm_launch(a, elem_is_bf16, st, err, num_sms, GEMM_AUTO);
  if (e != 0) return e;
  return gemm_launch(b, elem_is_bf16, st, err, num_sms, GEMM_AUTO);
}

bool gemm_uses_tc(const GemmParams& p, int elem_is_bf16) {
  if (p.M <= 0 || p.N <= 0 || p.K <= 0 || p.batch <= 0) return false;
  return !skinny_ok(p, elem_is_bf16) && tc_ok(p, elem_is_bf16);
}

// Returns 0 on success, or a cudaError_t value. engine: GEMM_AUTO (tcgen05: CTA pairs
// for large products, the K split over CTA pairs for thin ones, single-CTA tiles
// otherwise; SIMT where tensor cores do not fit), GEMM_SIMT, or GEMM_TC1 (single-CTA
// tiles only).
int gemm_launch(const GemmParams& p, int elem_is_bf16, cudaStream_t st, int* err, int num_sms, int engine) {
  if (p.M <= 0 || p.N <= 0 || p.K <= 0 || p.batch <= 0) return 0;
  if (p.norm_x) {
    const bool rows_path = engine != GEMM_SIMT && skinny_ok(p, elem_is_bf16) && elem_is_bf16 && p.M <= RW_MAXM &&
                           (size_t)p.M * p.K * 2 <= (size_t)RW_SMEM_MAX && p.K % 8 == 0 && p.lda % 8 == 0 &&
                           (p.batch == 1 || p.sA % 8 == 0);
    if (!rows_path) {  // a separate RMSNorm pass into A, then the product
      if (p.batch > 1 && p.sA != (int64_t)p.M * p.lda) return (int)cudaErrorInvalidValue;
      const int rows = p.M * p.batch;
      const cudaError_t e =
          elem_is_bf16 ? rmsnorm_fwd_launch<bf16>(p.norm_x, p.lda, p.norm_g, p.norm_eps, rows, p.K, (bf16*)p.A, p.lda,
                                                  p.norm_rstd, st)
                       : rmsnorm_fwd_launch<float>(p.norm_x, p.lda, p.norm_g, p.norm_eps, rows, p.K, (float*)p.A,
                                                   p.lda, p.norm_rstd, st);
      if (e != cudaSuccess) return (int)e;
      GemmParams q = p;
      q.norm_x = nullptr;
      return gemm_launch(q, elem_is_bf16, st, err, num_sms, engine);
    }
  }
  const bool force_simt = engine == GEMM_SIMT;
  if (p.epi == EPI_CE && (force_simt || !gemm_uses_tc(p, elem_is_bf16))) return (int)cudaErrorInvalidValue;
  if (!force_simt && skinny_ok(p, elem_is_bf16)) {
    GemmParams q = p;
    if (p.epi == EPI_QKV_ROPE) q.epi = EPI_STORE;
    const size_t xbytes = (size_t)p.M * p.K * 2;
    if (elem_is_bf16 && p.M <= RW_MAXM && xbytes <= (size_t)RW_SMEM_MAX) {
      // columns per warp: the most that still gives every SM a CTA (8 warps per CTA)
      const int64_t slices = p.batch;
      const int cw = ((int64_t)(p.N + 31) / 32) * slices >= num_sms ? 4 : ((int64_t)(p.N + 15) / 16) * slices >= num_sms ? 2 : 1;
      cudaError_t e;
      if (cw == 4)
        e = launch_pdl(gemm_rows_kernel<4>, dim3((p.N + 31) / 32, p.batch), dim3(256), xbytes, st, q);
      else if (cw == 2)
        e = launch_pdl(gemm_rows_kernel<2>, dim3((p.N + 15) / 16, p.batch), dim3(256), xbytes, st, q);
      else
        e = launch_pdl(gemm_rows_kernel<1>, dim3((p.N + 7) / 8, p.batch), dim3(256), xbytes, st, q);
      if (e != cudaSuccess) return (int)e;
    } else {
      dim3 grid((p.N + 1) / 2, p.batch);
      if (elem_is_bf16)
        gemm_skinny_kernel<bf16><<<grid, 256, 0, st>>>(q);
      else
        gemm_skinny_kernel<float><<<grid, 256, 0, st>>>(q);
    }
    if (p.epi == EPI_QKV_ROPE) {
      const cudaError_t re =
        elem_is_bf16 ? rope_launch<bf16>((bf16*)p.D, p.ldd, p.rope_cols, p.M, p.rope_n, p.rope_pos0, p.rope_hd,
                                         p.rope_lo, p.rope_hi, 0, p.rope_pos_dev, st, p.rope_ring_k, p.rope_ring_v, p.rope_C)
                     : rope_launch<float>((float*)p.D, p.ldd, p.rope_cols, p.M, p.rope_n, p.rope_pos0, p.rope_hd,
                                          p.rope_lo, p.rope_hi, 0, p.rope_pos_dev, st, p.rope_ring_k, p.rope_ring_v, p.rope_C);
    if (re != cudaSuccess) return (int)re;
    }
    return (int)cudaGetLastError();
  }
  GemmParams pt = p;  // tensor-core launch: the rotation of EPI_QKV_ROPE runs as a separate pass
  if (p.epi == EPI_QKV_ROPE) pt.epi = EPI_STORE;
  const bool use_tc = !force_simt && tc_ok(p, elem_is_bf16);
  if (use_tc) {
    // Tile width. A 128x256 tile does twice the work of a 128x128 one in about 1.32
    // times its time (tensor pipe 68% vs 45% busy on the same frozen-block GEMMs), so
    // 256 wins unless 128-wide tiles need fewer than 1.32x the persistent-grid waves
    // (ceil(tiles / SMs)): the small-M shapes with N = 2048.
    const int m_tiles = (p.M + TC_BM - 1) / TC_BM;
    auto waves = [&](int bn) { return std::ceil((double)m_tiles * (p.N / bn) * p.batch / num_sms); };
    const bool n256 = (p.N % 256 == 0) && waves(128) >= 1.32 * waves(256);
    // walk the larger operand once: column blocks outer when B is the larger matrix
    pt.m_fast = p.N > p.M ? 1 : 0;
    bool ok = false;
    cudaError_t e = cudaSuccess;
    // CTA pairs pay where the tile count is large: the frozen blocks' GEMMs over a whole
    // segment (11% faster at 32768 rows) and the wide LM head (13% faster); on the
    // 1024-row products of an adaptive step they are 2-20% slower than single-CTA tiles
    // (measured per shape on B200), so those keep the single-CTA kernel.
    if (engine != GEMM_TC1 && p.M > TC_BM && (p.M >= 4096 || p.N >= 16384)) {
      // CTA pairs: 256-row tiles, waves counted in resident pairs
      const int cap = pair_capacity<128, false, false>();
      if (cap > 0) {
        const int m2 = (p.M + 2 * TC_BM - 1) / (2 * TC_BM);
        auto waves2 = [&](int bn) { return std::ceil((double)m2 * (p.N / bn) * p.batch / cap); };
        const bool w256 = (p.N % 256 == 0) && waves2(128) >= 1.32 * waves2(256);
        if (!p.a_mn && !p.b_mn)
          e = w256 ? launch_tc2<256, false, false>(pt, st, err, &ok) : launch_tc2<128, false, false>(pt, st, err, &ok);
        else if (!p.a_mn && p.b_mn)
          e = w256 ? launch_tc2<256, false, true>(pt, st, err, &ok) : launch_tc2<128, false, true>(pt, st, err, &ok);
        else
          e = w256 ? launch_tc2<256, true, true>(pt, st, err, &ok) : launch_tc2<128, true, true>(pt, st, err, &ok);
        if (e != cudaSuccess) return (int)e;
      }
    }
    if (ok) {
      if (p.epi == EPI_QKV_ROPE) {
        return (int)rope_launch<bf16>((bf16*)p.D, p.ldd, p.rope_cols, p.M, p.rope_n, p.rope_pos0, p.rope_hd,
                                      p.rope_lo, p.rope_hi, 0, p.rope_pos_dev, st, p.rope_ring_k, p.rope_ring_v, p.rope_C);
      }
      return 0;
    }
    // K split over CTA pairs: thin products whose 128 x 256 tiles fill at most half the
    // SMs (the N = 2048 products of an adaptive step: 64 tiles) run each tile on two SMs
    // with 256-wide tiles instead of 128-wide tiles on one (an M = 128 MMA costs about the
    // same at N = 128 as at N = 256). The exchange of the partial halves costs a few
    // microseconds, so K >= 4096 pays: measured on B200 at 1024 x 2048, K = 8192
    // (W_init + dW) 45.6 -> 35.9 us, K = 6144 35.8 -> 27.6 us, K = 4096 26.2 -> 22.6 us,
    // K = 32000 150 -> 109 us; K = 2048 21.4 -> 22.1 us stays on single CTAs.
    const int t256 = (p.N % 256 == 0) ? m_tiles * (p.N / 256) * p.batch : 0;
    const int kbt = (p.K / TC_BK) * (p.B2 ? 2 : 1);
    if (engine != GEMM_TC1 && p.epi != EPI_CE && t256 > 0 && 2 * t256 <= num_sms && kbt % 2 == 0 && kbt >= 64) {
      if (!p.a_mn && !p.b_mn) e = launch_tck<256, false, false>(pt, st, err, &ok);
      else if (!p.a_mn && p.b_mn) e = launch_tck<256, false, true>(pt, st, err, &ok);
      else e = launch_tck<256, true, true>(pt, st, err, &ok);
      if (e != cudaSuccess) return (int)e;
    }
    if (ok) {
      if (p.epi == EPI_QKV_ROPE) {
        return (int)rope_launch<bf16>((bf16*)p.D, p.ldd, p.rope_cols, p.M, p.rope_n, p.rope_pos0, p.rope_hd,
                                      p.rope_lo, p.rope_hi, 0, p.rope_pos_dev, st, p.rope_ring_k, p.rope_ring_v, p.rope_C);
      }
      return 0;
    }
    if (!p.a_mn && !p.b_mn)
      e = n256 ? launch_tc<256, false, false>(pt, st, err, num_sms, &ok) : launch_tc<128, false, false>(pt, st, err, num_sms, &ok);
    else if (!p.a_mn && p.b_mn)
      e = n256 ? launch_tc<256, false, true>(pt, st, err, num_sms, &ok) : launch_tc<128, false, true>(pt, st, err, num_sms, &ok);
    else
      e = n256 ? launch_tc<256, true, true>(pt, st, err, num_sms, &ok) : launch_tc<128, true, true>(pt, st, err, num_sms, &ok);
    if (e != cudaSuccess) return (int)e;
    if (ok) {
      if (p.epi == EPI_QKV_ROPE) {
        return (int)rope_launch<bf16>((bf16*)p.D, p.ldd, p.rope_cols, p.M, p.rope_n, p.rope_pos0, p.rope_hd,
                                      p.rope_lo, p.rope_hi, 0, p.rope_pos_dev, st, p.rope_ring_k, p.rope_ring_v, p.rope_C);
      }
      return 0;
    }
  }
  if (p.epi == EPI_CE) return (int)cudaErrorInvalidValue;  // the statistics epilogue exists on tcgen05 only
  dim3 grid((p.N + 63) / 64, (p.M + 63) / 64, p.batch);
  GemmParams q = p;
  if (p.epi == EPI_QKV_ROPE) q.epi = EPI_STORE;  // rotation as a separate pass below
  if (elem_is_bf16)
    gemm_simt_kernel<bf16><<<grid, 256, 0, st>>>(q);
  else
    gemm_simt_kernel<float><<<grid, 256, 0, st>>>(q);
  if (p.epi == EPI_QKV_ROPE) {
    const cudaError_t re =
        elem_is_bf16 ? rope_launch<bf16>((bf16*)p.D, p.ldd, p.rope_cols, p.M, p.rope_n, p.rope_pos0, p.rope_hd,
                                         p.rope_lo, p.rope_hi, 0, p.rope_pos_dev, st, p.rope_ring_k, p.rope_ring_v, p.rope_C)
                     : rope_launch<float>((float*)p.D, p.ldd, p.rope_cols, p.M, p.rope_n, p.rope_pos0, p.rope_hd,
                                          p.rope_lo, p.rope_hi, 0, p.rope_pos_dev, st, p.rope_ring_k, p.rope_ring_v, p.rope_C);
    if (re != cudaSuccess) return (int)re;
  }
  return (int)cudaGetLastError();
}

// ============================================================== device memory
// Injected allocation failure: the request with this index (counted from the
// moment it was set) fails; -1 = none. Requests made so far: g_alloc_count.
static std::atomic<int64_t> g_fail_countdown{-1};
static std::atomic<int64_t> g_alloc_count{0};

cudaError_t device_alloc(void** p, size_t bytes) {
  *p = nullptr;
  int64_t c = g_fail_countdown.load();
  while (c >= 0 && !g_fail_countdown.compare_exchange_weak(c, c - 1)) {
  }
  if (c == 0) return cudaErrorMemoryAllocation;
  const cudaError_t e = cudaMalloc(p, bytes);
  if (e == cudaSuccess) g_alloc_count.fetch_add(1);
  return e;
}

void device_free(void* p) {
  if (p) cudaFree(p);
}

struct Arena {
  std::vector<void*> ptrs;
  int64_t bytes = 0;
  bool failed = false;
  void* alloc(size_t n) {
    if (n == 0) n = 16;
    n = (n + 255) & ~(size_t)255;
    void* p = nullptr;
    if (device_alloc(&p, n) != cudaSuccess) {
      cudaGetLastError();
      failed = true;
      return nullptr;
    }
    ptrs.push_back(p);
    bytes += (int64_t)n;
    return p;
  }
  template <typename X> X* get(size_t count) { return (X*)alloc(count * sizeof(X)); }
  void release() {
    for (void* p : ptrs) device_free(p);
    ptrs.clear();
    bytes = 0;
  }
};

// Kernel-class timer: CUDA events recorded on the launching stream around each
// launch of a class, plus the algorithmic FLOPs and bytes of that launch.
enum ProfClass : int { PC_GEMM_FROZEN = 0, PC_GEMM_TTT = 1, PC_ATTN_FWD = 2, PC_ATTN_BWD = 3, PC_COUNT = 4 };
struct Profiler {
  bool on = false;
  std::vector<cudaEvent_t> ev;     // pairs
  std::vector<int> cls;
  std::vector<double> fl, by;
  size_t used = 0;
  double ms[PC_COUNT] = {}, flops[PC_COUNT] = {}, bytes[PC_COUNT] = {};
  int64_t n[PC_COUNT] = {};
  void begin(cudaStream_t st, int c, double f, double b) {
    if (!on) return;
    if (used * 2 + 2 > ev.size()) {
      for (int i = 0; i < 256; ++i) {
        cudaEvent_t e;
        cudaEventCreate(&e);
        ev.push_back(e);
      }
    }
    cls.resize(used + 1); fl.resize(used + 1); by.resize(used + 1);
    cls[used] = c; fl[used] = f; by[used] = b;
    cudaEventRecord(ev[2 * used], st);
  }
  void end(cudaStream_t st) {
    if (!on) return;
    cudaEventRecord(ev[2 * used + 1], st);
    ++used;
  }
  void collect() {  // after the stream has synchronised
    for (size_t i = 0; i < used; ++i) {
      float t = 0.f;
      cudaEventElapsedTime(&t, ev[2 * i], ev[2 * i + 1]);
      ms[cls[i]] += t; flops[cls[i]] += fl[i]; bytes[cls[i]] += by[i]; n[cls[i]] += 1;
    }
    used = 0;
  }
  void clear() {
    for (int c = 0; c < PC_COUNT; ++c) { ms[c] = flops[c] = bytes[c] = 0; n[c] = 0; }
  }
  ~Profiler() { for (auto e : ev) cudaEventDestroy(e); }
};

}  // namespace ttt

// ============================================================== handle
struct ttt_handle {
  virtual ~ttt_handle() {}
  virtual int prefill(const int32_t* tokens, int64_t T, float* out, int32_t kind) = 0;
  virtual int decode(int64_t n, const int32_t* forced, int32_t* out_tok, float* out_loss, int32_t kind) = 0;
  virtual int get_weights(int32_t seq, int32_t blk, float* w1, float* w2, int32_t kind) = 0;
  virtual int reset() = 0;
  virtual int set_device_status(int32_t code) = 0;
  std::string err_msg;
  bool poisoned = false;
  int64_t n_pos = 0;
  int64_t launches = 0;
  int64_t dev_bytes = 0;
  ttt::Profiler prof;
};

namespace ttt {

static int fail(ttt_handle* h, int code, const std::string& msg) {
  if (h) h->err_msg = msg;
  return code;
}

#define TTT_CUDA(call)                                                                           \
  do {                                                                                           \
    cudaError_t _e = (call);                                                                     \
    if (_e != cudaSuccess) {                                                                     \
      poisoned = true;                                                                           \
      return fail(this, TTT_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(_e));       \
    }                                                                                            \
  } while (0)

#define TTT_LAUNCHED()                                                                           \
  do {                                                                                           \
    ++launches;                                                                                  \
    cudaError_t _e = cudaGetLastError();                                                         \
    if (_e != cudaSuccess) {                                                                     \
      poisoned = true;                                                                           \
      return fail(this, TTT_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(_e));         \
    }                                                                                            \
  } while (0)

static inline unsigned nblk(int64_t n, int t) { return (unsigned)((n + t - 1) / t); }

// Per-layer device weights and caches.
template <typename T> struct LayerDev {
  float* g_attn = nullptr;
  T* Wqkv = nullptr;  // [3d][d]
  T* Wo = nullptr;    // [d][d]
  float* g_mlp = nullptr; T* W1 = nullptr; T* W2 = nullptr;           // frozen MLP
  float* g_ttt = nullptr; float* g_static = nullptr;                   // adaptive block
  T* W1s = nullptr; T* W2s = nullptr;
  // Fast weights of the adaptive MLP, per sequence. fp32 path: W itself (W1t32/W2t32,
  // shadows alias them). bf16 path: W = W_init + dW with W_init held once in bf16
  // (shared by all sequences) and the per-sequence update dW as an fp32 master
  // (W1t32/W2t32) plus a bf16 copy for the GEMMs (W1t/W2t): a bf16 copy of
  // W_init + dW would round most of a small update away.
  float* W1t32 = nullptr; float* W2t32 = nullptr;                      // [B][ht][d], [B][d][ht]
  T* W1t = nullptr; T* W2t = nullptr;
  T* W1t_init = nullptr; T* W2t_init = nullptr;                        // [ht][d], [d][ht]
  T* theta_kv = nullptr;  // key-value-binding inner loss: theta_K [d][d] then theta_V [d][d]
  T* ring_k = nullptr; T* ring_v = nullptr;                            // [B][C][d]
};

// Activations of one adaptive block kept for the backward (rows Mc = B*b).
template <typename T> struct BlockAct {
  float* x; float* rstd1; T* qkv; T* o; float* lse; float* a; float* rstd2; T* r2; T* u; T* g;
  float* m; float* rstd3; T* r3; T* us; T* gs;
  T* k;  // key-value-binding variant: the adaptive MLP's input theta_K r2 (else unused)
};

template <typename T> class Engine : public ttt_handle {
 public:
  ttt_config cfg;
  cudaStream_t st = nullptr;
  int num_sms = 148;
  int B, d, V, L, Lt, H, hd, h, ht, hs, kwin, bsz, C, S;
  int first_ttt;
  bool is_bf16;
  bool kvb = false;  // inner loss: layer-wise key-value binding instead of the next-token loss
  Arena arena;
  int* dev_err = nullptr;
  T* E = nullptr;
  float* g_final = nullptr;
  float2* rope_lo = nullptr;
  float2* rope_hi = nullptr;
  static constexpr int kRopeHi = 16384;  // positions < 16384 * 1024
  std::vector<LayerDev<T>> layers;
  // frozen-phase segment buffers (Ms = B*S rows)
  float* xs = nullptr; T* rs = nullptr; T* qkvs = nullptr; T* os = nullptr; T* hids = nullptr;
  // adaptive-phase buffers (Mc = B*b rows)
  std::vector<BlockAct<T>> blk;
  float* tin = nullptr; float* y = nullptr; float* rstdf = nullptr; T* rf = nullptr; T* z = nullptr;
  int32_t* tgt = nullptr;
  float2* ce_part = nullptr; float* ce_zt = nullptr;  // fused LM-head cross-entropy statistics (bf16 path)
  float* G = nullptr; T* GT = nullptr; T* dhid = nullptr; float* dr = nullptr; T* dqkv = nullptr;
  T* dob = nullptr; float* Dsum = nullptr;
  // pending (incomplete) chunk: inputs of the first adaptive block and targets
  float* pend_in = nullptr; int32_t* pend_tgt = nullptr; int pend_cnt = 0;
  int32_t* pend_tok_dev = nullptr;        // [B] pending input id of each sequence
  std::vector<int32_t> pend_tok_host;
  // decode scratch
  int32_t* chosen = nullptr; float* dec_loss = nullptr; float* dec_zmax = nullptr; int32_t* forced_col = nullptr;
  // decode attention over the window in dec_split parts of ~256 keys: partial results
  // [B][H][dec_split][hd + 2] and one ticket per (sequence, head)
  int dec_split = 1; float* dec_part = nullptr; int* dec_ticket = nullptr;
  // per-call growable buffers
  int64_t chunk_pos = 0;                  // absolute position of row 0 of the chunk in the adaptive buffers
  bool decode_mode = false;               // set while a decode token step is being captured
  cudaStream_t cap_st = nullptr;          // private stream the decode step is captured on (the caller's
                                          // stream may be the legacy default stream, which cannot capture)
  int64_t* pos_dev = nullptr;             // device copy of the position of the token being decoded
  int32_t* tok_dev = nullptr; int64_t tok_cap = 0;
  float* loss_dev = nullptr; int64_t loss_cap = 0;
  int32_t* otok_dev = nullptr; int64_t otok_cap = 0;
  float* wexp = nullptr; int64_t wexp_cap = 0;
  Arena call_arena;

  ~Engine() override {
    if (st) cudaStreamSynchronize(st);
    if (cap_st) cudaStreamDestroy(cap_st);
    call_arena.release();
    arena.release();
  }

  int create(const ttt_config* c, const ttt_weights* w);
  int prefill(const int32_t* tokens, int64_t T_, float* out, int32_t kind) override;
  int decode(int64_t n, const int32_t* forced, int32_t* out_tok, float* out_loss, int32_t kind) override;
  int get_weights(int32_t seq, int32_t blk, float* w1, float* w2, int32_t kind) override;
  int reset() override;
  // Test hook: with the stream idle, write `code` into the device status word, as a
  // kernel whose bounded wait ran out would. The next call that checks the word
  // reports it.
  int set_device_status(int32_t code) override {
    TTT_CUDA(cudaStreamSynchronize(st));
    TTT_CUDA(cudaMemcpy(dev_err, &code, sizeof(int), cudaMemcpyHostToDevice));
    return TTT_OK;
  }

 private:
  int gemm_class = PC_GEMM_FROZEN;
  int gemm(GemmParams p) {
    const size_t es = is_bf16 ? 2 : 4;
    prof.begin(st, gemm_class, 2.0 * p.M * p.N * (double)p.K * p.batch,
               (double)p.batch * ((double)p.M * p.K * es + (double)p.N * p.K * es +
                                  (double)p.M * p.N * (p.d_f32 ? 4 : es)));
    const int e = gemm_launch(p, is_bf16 ? 1 : 0, st, dev_err, num_sms, GEMM_AUTO);
    prof.end(st);
    ++launches;
    if (e != 0) {
      poisoned = true;
      return fail(this, TTT_ERR_CUDA, std::string("gemm: ") + cudaGetErrorString((cudaError_t)e));
    }
    return TTT_OK;
  }
  // Two independent products (gemm_launch_pair): one launch where they can share it.
  int gemm2(const GemmParams& a, const GemmParams& b) {
    const size_t es = is_bf16 ? 2 : 4;
    auto bytes = [&](const GemmParams& p) {
      return (double)p.batch * ((double)p.M * p.K * es + (double)p.N * p.K * es + (double)p.M * p.N * (p.d_f32 ? 4 : es));
    };
    prof.begin(st, gemm_class, 2.0 * a.M * a.N * (double)a.K * a.batch + 2.0 * b.M * b.N * (double)b.K * b.batch,
               bytes(a) + bytes(b));
    const int e = gemm_launch_pair(a, b, is_bf16 ? 1 : 0, st, dev_err, num_sms);
    prof.end(st);
    launches += 2;
    if (e != 0) {
      poisoned = true;
      return fail(this, TTT_ERR_CUDA, std::string("gemm: ") + cudaGetErrorString((cudaError_t)e));
    }
    return TTT_OK;
  }
  static GemmParams gp(int M, int N, int K, const void* A, int64_t lda, bool a_mn, const void* Bm, int64_t ldb,
                       bool b_mn, void* D, int64_t ldd, bool d_f32, int epi) {
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.M = M; p.N = N; p.K = K; p.batch = 1;
    p.A = A; p.lda = lda; p.a_mn = a_mn;
    p.B = Bm; p.ldb = ldb; p.b_mn = b_mn;
    p.D = D; p.ldd = ldd; p.d_f32 = d_f32;
    p.alpha = 1.f; p.epi = epi;
    return p;
  }
  // r = RMSNorm(x) (gain g) as the A operand of p: in a decode token step the few-row GEMM
  // normalises while staging its rows (one launch instead of two); elsewhere a separate pass.
  int norm_into(GemmParams& p, const float* x, const float* g, float* rstd, T* r, int rows) {
    if (decode_mode) {
      p.norm_x = x; p.norm_g = g; p.norm_eps = cfg.rms_eps; p.norm_rstd = rstd;
      return TTT_OK;
    }
    ++launches;
    const cudaError_t e = rmsnorm_fwd_launch<T>(x, d, g, cfg.rms_eps, rows, d, r, d, rstd, st);
    if (e == cudaSuccess) return TTT_OK;
    poisoned = true;
    return fail(this, TTT_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  }
  // sum over queries P = q0..q0+n-1 of min(P+1, k): query-key pairs of the window (review eq. (1))
  double attn_pairs(int64_t n, int64_t q0) const {
    double s = 0;
    const int64_t k = kwin;
    // positions below k contribute P+1, the rest k
    const int64_t a = q0, b = q0 + n;  // [a, b)
    const int64_t m = b < k ? b : (a > k ? a : k);  // split point clamp
    if (a < m) s += (double)(m - a) * (a + 1 + m) / 2.0;  // sum_{P=a}^{m-1} (P+1)
    if (m < b) s += (double)(b - (a > m ? a : m)) * k;
    return s;
  }
  // B operand of a product with the fast weights W (per sequence): fp32 path reads W
  // directly; bf16 path accumulates W_init (shared) and dW (per sequence).
  void fast_operand(GemmParams& p, const T* init, const T* delta, int64_t per_seq) const {
    if (is_bf16) {
      p.B = init; p.sB = 0;
      p.B2 = delta; p.sB2 = per_seq;
    } else {
      p.B = delta; p.sB = per_seq;
    }
  }
  int attention_block(const LayerDev<T>& Lw, int layer, float* xin, float* xout, T* r, float* rstd, T* qkv, T* o,
                      float* lse, int n, int64_t q0, bool commit);
  int frozen_mlp(const LayerDev<T>& Lw, float* x, T* r, T* hid, int rows);
  int ttt_forward(int cn, int64_t pos, bool commit);
  int ttt_backward(int cn);
  int kvb_update(int cn);
  int decode_token_launches(int64_t n, int32_t* otok, float* oloss, const int32_t* fdev, int64_t base);
  int ttt_step(const float* in, const int32_t* targets, int cn, int64_t pos, float* loss_out, int64_t loss_ld,
               int64_t loss_off, bool grad, bool commit);
  int sync_and_check();
  int ensure(void** ptr, int64_t* cap, int64_t need, size_t elem);
};

template <typename T> int Engine<T>::ensure(void** ptr, int64_t* cap, int64_t need, size_t elem) {
  if (need <= *cap) return TTT_OK;
  void* p = call_arena.alloc((size_t)need * elem);
  if (!p) return fail(this, TTT_ERR_OOM, "device allocation failed (call buffers)");
  *ptr = p;
  *cap = need;
  dev_bytes = arena.bytes + call_arena.bytes;
  return TTT_OK;
}

template <typename T> int Engine<T>::sync_and_check() {
  TTT_CUDA(cudaStreamSynchronize(st));
  prof.collect();
  int flag = 0;
  TTT_CUDA(cudaMemcpy(&flag, dev_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (flag == DEV_BAD_TOKEN) {
    TTT_CUDA(cudaMemset(dev_err, 0, sizeof(int)));
    poisoned = true;  // the call ran with a clamped id; the state is no longer meaningful
    return fail(this, TTT_ERR_INVALID_ARG, "token id outside [0, vocab)");
  }
  if (flag != 0) {
    poisoned = true;
    return fail(this, TTT_ERR_TIMEOUT, "device wait expired (code " + std::to_string(flag) + ")");
  }
  return TTT_OK;
}

// ------------------------------------------------------------------ create
template <typename T> int Engine<T>::create(const ttt_config* c, const ttt_weights* w) {
  cfg = *c;
  st = (cudaStream_t)cfg.cuda_stream;
  B = cfg.batch; d = cfg.d; V = cfg.vocab; L = cfg.n_layers; Lt = cfg.n_ttt; H = cfg.n_heads;
  hd = d / H; h = cfg.mlp_hidden; ht = cfg.ttt_hidden; hs = cfg.static_hidden; kwin = cfg.window_k;
  bsz = cfg.minibatch_b;
  first_ttt = L - Lt;
  is_bf16 = cfg.dtype == TTT_BF16;
  kvb = cfg.inner_loss == TTT_LOSS_KVB;
  C = ((kwin + bsz + 127) / 128) * 128;
  int seg = cfg.max_segment > 0 ? cfg.max_segment : 32768;
  S = ((seg + bsz - 1) / bsz) * bsz;
  int dev = 0;
  TTT_CUDA(cudaGetDevice(&dev));
  TTT_CUDA((cudaError_t)prime_kernel_attributes());
  TTT_CUDA(cudaStreamCreateWithFlags(&cap_st, cudaStreamNonBlocking));
  TTT_CUDA(cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev));

  const int64_t Ms = (int64_t)B * S, Mc = (int64_t)B * bsz;
  dev_err = arena.get<int>(1);
  E = arena.get<T>((size_t)V * d);
  g_final = arena.get<float>(d);
  rope_lo = arena.get<float2>((size_t)1024 * (hd / 2));
  rope_hi = arena.get<float2>((size_t)kRopeHi * (hd / 2));
  layers.resize(L);
  for (int l = 0; l < L; ++l) {
    LayerDev<T>& Lw = layers[l];
    Lw.g_attn = arena.get<float>(d);
    Lw.Wqkv = arena.get<T>((size_t)3 * d * d);
    Lw.Wo = arena.get<T>((size_t)d * d);
    Lw.ring_k = arena.get<T>((size_t)B * C * d);
    Lw.ring_v = arena.get<T>((size_t)B * C * d);
    if (l < first_ttt) {
      Lw.g_mlp = arena.get<float>(d);
      Lw.W1 = arena.get<T>((size_t)h * d);
      Lw.W2 = arena.get<T>((size_t)d * h);
    } else {
      Lw.g_ttt = arena.get<float>(d);
      Lw.g_static = arena.get<float>(d);
      Lw.W1s = arena.get<T>((size_t)hs * d);
      Lw.W2s = arena.get<T>((size_t)d * hs);
      Lw.W1t32 = arena.get<float>((size_t)B * ht * d);
      Lw.W2t32 = arena.get<float>((size_t)B * d * ht);
      Lw.W1t_init = arena.get<T>((size_t)ht * d);
      Lw.W2t_init = arena.get<T>((size_t)d * ht);
      if (kvb) Lw.theta_kv = arena.get<T>((size_t)2 * d * d);
      if (is_bf16) {
        Lw.W1t = arena.get<T>((size_t)B * ht * d);
        Lw.W2t = arena.get<T>((size_t)B * d * ht);
      } else {
        Lw.W1t = (T*)Lw.W1t32;
        Lw.W2t = (T*)Lw.W2t32;
      }
    }
  }
  const int hmax = h > ht ? (h > hs ? h : hs) : (ht > hs ? ht : hs);
  xs = arena.get<float>((size_t)Ms * d);
  rs = arena.get<T>((size_t)Ms * d);
  qkvs = arena.get<T>((size_t)Ms * 3 * d);
  os = arena.get<T>((size_t)Ms * d);
  hids = arena.get<T>((size_t)Ms * hmax);
  blk.resize(Lt);
  for (int j = 0; j < Lt; ++j) {
    BlockAct<T>& A = blk[j];
    A.x = arena.get<float>((size_t)Mc * d);
    A.rstd1 = arena.get<float>(Mc);
    A.qkv = arena.get<T>((size_t)Mc * 3 * d);
    A.o = arena.get<T>((size_t)Mc * d);
    A.lse = arena.get<float>((size_t)B * H * bsz);
    A.a = arena.get<float>((size_t)Mc * d);
    A.rstd2 = arena.get<float>(Mc);
    A.r2 = arena.get<T>((size_t)Mc * d);
    A.u = arena.get<T>((size_t)Mc * ht);
    A.g = arena.get<T>((size_t)Mc * ht);
    A.m = arena.get<float>((size_t)Mc * d);
    A.rstd3 = arena.get<float>(Mc);
    A.r3 = arena.get<T>((size_t)Mc * d);
    A.us = arena.get<T>((size_t)Mc * hs);
    A.gs = arena.get<T>((size_t)Mc * hs);
    A.k = kvb ? arena.get<T>((size_t)Mc * d) : nullptr;
  }
  // chunk input: the first adaptive block's input buffer, or its own buffer without adaptive blocks
  tin = blk.empty() ? arena.get<float>((size_t)Mc * d) : blk[0].x;
  y = arena.get<float>((size_t)Mc * d);
  rstdf = arena.get<float>(Mc);
  rf = arena.get<T>((size_t)Mc * d);
  z = arena.get<T>((size_t)Mc * V);
  tgt = arena.get<int32_t>(Mc);
  if (is_bf16 && V % 64 == 0) {
    ce_part = arena.get<float2>((size_t)Mc * (V / 64));
    ce_zt = arena.get<float>(Mc);
  }
  G = arena.get<float>((size_t)Mc * d);
  GT = arena.get<T>((size_t)Mc * d);
  dhid = arena.get<T>((size_t)Mc * (ht > hs ? ht : hs));
  dr = arena.get<float>((size_t)Mc * d);
  dqkv = arena.get<T>((size_t)Mc * 3 * d);
  dob = arena.get<T>((size_t)Mc * d);
  Dsum = arena.get<float>((size_t)B * H * bsz);
  pend_in = arena.get<float>((size_t)Mc * d);
  pend_tgt = arena.get<int32_t>(Mc);
  pend_tok_dev = arena.get<int32_t>(B);
  chosen = arena.get<int32_t>(B);
  dec_loss = arena.get<float>(B);
  dec_zmax = arena.get<float>(B);
  forced_col = arena.get<int32_t>(B);
  pos_dev = arena.get<int64_t>(1);
  {
    const int64_t w = kwin < C ? kwin : C;
    dec_split = (int)std::min<int64_t>(16, std::max<int64_t>(1, (w + 255) / 256));
    dec_part = arena.get<float>((size_t)B * H * dec_split * (hd + 2));
    dec_ticket = arena.get<int>((size_t)B * H);
  }
  if (arena.failed) {
    arena.release();
    return fail(this, TTT_ERR_OOM, "device allocation failed");
  }
  dev_bytes = arena.bytes;
  TTT_CUDA(cudaMemsetAsync(dev_err, 0, sizeof(int), st));
  TTT_CUDA(cudaMemsetAsync(dec_ticket, 0, sizeof(int) * (size_t)B * H, st));

  // RoPE tables in double precision: lo[p][i] = angle p*theta_i (p < 1024), hi[q][i] = angle 1024*q*theta_i
  {
    const int half = hd / 2;
    std::vector<float2> lo((size_t)1024 * half), hi((size_t)kRopeHi * half);
    for (int i = 0; i < half; ++i) {
      const double theta = std::pow((double)cfg.rope_base, -2.0 * i / hd);
      for (int p = 0; p < 1024; ++p) {
        const double a = p * theta;
        lo[(size_t)p * half + i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
      for (int q = 0; q < kRopeHi; ++q) {
        const double a = 1024.0 * q * theta;
        hi[(size_t)q * half + i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    }
    TTT_CUDA(cudaMemcpyAsync(rope_lo, lo.data(), lo.size() * sizeof(float2), cudaMemcpyHostToDevice, st));
    TTT_CUDA(cudaMemcpyAsync(rope_hi, hi.data(), hi.size() * sizeof(float2), cudaMemcpyHostToDevice, st));
    TTT_CUDA(cudaStreamSynchronize(st));
  }

  // weights: stage each tensor on the device, then convert into place
  const bool src_bf16 = w->values_dtype == TTT_BF16;
  const size_t src_elem = src_bf16 ? 2 : 4;
  int64_t max_elems = (int64_t)V * d;
  if ((int64_t)h * d > max_elems) max_elems = (int64_t)h * d;
  if ((int64_t)ht * d > max_elems) max_elems = (int64_t)ht * d;
  if ((int64_t)hs * d > max_elems) max_elems = (int64_t)hs * d;
  void* stage = nullptr;
  if (w->ptr_kind == TTT_PTR_HOST) {
    if (device_alloc(&stage, (size_t)max_elems * 4) != cudaSuccess) {
      cudaGetLastError();
      arena.release();
      return fail(this, TTT_ERR_OOM, "device allocation failed (weight staging buffer)");
    }
  }
  int ti = 0;
  auto upload = [&](void* dst, bool dst_f32, int64_t count, bool gain) -> int {
    const void* src = w->tensors[ti++];
    if (!src) return fail(this, TTT_ERR_INVALID_ARG, "null weight tensor " + std::to_string(ti - 1));
    const size_t es = gain ? 4 : src_elem;
    const void* dsrc = src;
    if (w->ptr_kind == TTT_PTR_HOST) {
      TTT_CUDA(cudaMemcpyAsync(stage, src, (size_t)count * es, cudaMemcpyHostToDevice, st));
      dsrc = stage;
    }
    const unsigned g = nblk(count, 256);
    if (gain || !src_bf16) {
      if (dst_f32) convert_kernel<float, float><<<g, 256, 0, st>>>((const float*)dsrc, (float*)dst, count);
      else convert_kernel<float, T><<<g, 256, 0, st>>>((const float*)dsrc, (T*)dst, count);
    } else {
      if (dst_f32) convert_kernel<bf16, float><<<g, 256, 0, st>>>((const bf16*)dsrc, (float*)dst, count);
      else convert_kernel<bf16, T><<<g, 256, 0, st>>>((const bf16*)dsrc, (T*)dst, count);
    }
    TTT_LAUNCHED();
    if (w->ptr_kind == TTT_PTR_HOST) TTT_CUDA(cudaStreamSynchronize(st));  // stage reuse
    return TTT_OK;
  };
  int rc;
#define UP(dst, f32, cnt, gain) if ((rc = upload((dst), (f32), (cnt), (gain))) != TTT_OK) { device_free(stage); return rc; }
  UP(E, false, (int64_t)V * d, false);
  UP(g_final, true, d, true);
  const int64_t dd = (int64_t)d * d;
  for (int l = 0; l < L; ++l) {
    LayerDev<T>& Lw = layers[l];
    UP(Lw.g_attn, true, d, true);
    UP(Lw.Wqkv, false, dd, false);
    UP(Lw.Wqkv + dd, false, dd, false);
    UP(Lw.Wqkv + 2 * dd, false, dd, false);
    UP(Lw.Wo, false, dd, false);
    if (l < first_ttt) {
      UP(Lw.g_mlp, true, d, true);
      UP(Lw.W1, false, (int64_t)h * d, false);
      UP(Lw.W2, false, (int64_t)d * h, false);
    } else {
      UP(Lw.g_ttt, true, d, true);
      UP(Lw.W1t_init, !is_bf16, (int64_t)ht * d, false);
      UP(Lw.W2t_init, !is_bf16, (int64_t)d * ht, false);
      UP(Lw.g_static, true, d, true);
      UP(Lw.W1s, false, (int64_t)hs * d, false);
      UP(Lw.W2s, false, (int64_t)d * hs, false);
      if (kvb) {
        UP(Lw.theta_kv, false, dd, false);
        UP(Lw.theta_kv + dd, false, dd, false);
      }
    }
  }
#undef UP
  device_free(stage);
  return reset();
}

template <typename T> int Engine<T>::reset() {
  if (poisoned) return fail(this, TTT_ERR_POISONED, "handle poisoned by an earlier device error");
  for (int l = first_ttt; l < L; ++l) {
    LayerDev<T>& Lw = layers[l];
    const int64_t n1 = (int64_t)ht * d;
    if (is_bf16) {  // dW = 0
      TTT_CUDA(cudaMemsetAsync(Lw.W1t32, 0, (size_t)B * n1 * 4, st));
      TTT_CUDA(cudaMemsetAsync(Lw.W2t32, 0, (size_t)B * n1 * 4, st));
      TTT_CUDA(cudaMemsetAsync(Lw.W1t, 0, (size_t)B * n1 * sizeof(T), st));
      TTT_CUDA(cudaMemsetAsync(Lw.W2t, 0, (size_t)B * n1 * sizeof(T), st));
    } else {  // W = W_init
      for (int b = 0; b < B; ++b) {
        TTT_CUDA(cudaMemcpyAsync(Lw.W1t32 + b * n1, Lw.W1t_init, n1 * 4, cudaMemcpyDeviceToDevice, st));
        TTT_CUDA(cudaMemcpyAsync(Lw.W2t32 + b * n1, Lw.W2t_init, n1 * 4, cudaMemcpyDeviceToDevice, st));
      }
    }
  }
  for (int l = 0; l < L; ++l) {
    TTT_CUDA(cudaMemsetAsync(layers[l].ring_k, 0, (size_t)B * C * d * sizeof(T), st));
    TTT_CUDA(cudaMemsetAsync(layers[l].ring_v, 0, (size_t)B * C * d * sizeof(T), st));
  }
  n_pos = 0;
  pend_cnt = 0;
  pend_tok_host.assign(B, -1);
  return sync_and_check();
}

// ------------------------------------------------------------------ blocks
// Pre-norm attention sub-block over rows [B][n] at positions q0 + i:
// xout = xin + Wo * Attn(RoPE(Wq r), RoPE(Wk r), Wv r), r = RMSNorm(xin).
template <typename T>
int Engine<T>::attention_block(const LayerDev<T>& Lw, int layer, float* xin, float* xout, T* r, float* rstd, T* qkv,
                               T* o, float* lse, int n, int64_t q0, bool commit) {
  const int rows = B * n;
  int rc;
  // The chunk's keys and values go to the ring in the RoPE pass when that cannot
  // overwrite a slot this attention still reads: rows of a chunk of n <= b positions
  // and the window before them span n + k - 1 < C positions. (A frozen segment is
  // longer than the ring and appends after its attention.) Decode appends its one
  // position there too, then attends over the window entirely from the ring.
  const bool append_in_rope = commit && (decode_mode || n <= bsz);
  // A decode step on the lane-group attention kernel rotates q and k and appends k, v to
  // the ring inside that kernel: the projection then stores q|k|v as they are.
  const bool rope_in_attn = decode_mode && is_bf16 && (hd == 64 || hd == 128);
  {  // q|k|v = r Wqkv^T with RoPE applied to q and k in the GEMM epilogue
    GemmParams pq = gp(rows, 3 * d, d, r, d, false, Lw.Wqkv, d, false, qkv, 3 * d, false,
                       rope_in_attn ? EPI_STORE : EPI_QKV_ROPE);
    pq.rope_lo = rope_lo; pq.rope_hi = rope_hi; pq.rope_hd = hd; pq.rope_cols = 2 * d;
    pq.rope_n = decode_mode ? 1 : n;
    pq.rope_pos0 = decode_mode ? 0 : q0;
    pq.rope_pos_dev = decode_mode ? pos_dev : nullptr;
    if (append_in_rope && !rope_in_attn) { pq.rope_ring_k = Lw.ring_k; pq.rope_ring_v = Lw.ring_v; pq.rope_C = C; }
    if ((rc = norm_into(pq, xin, Lw.g_attn, rstd, r, rows)) != TTT_OK) return rc;
    if ((rc = gemm(pq)) != TTT_OK) return rc;
  }
  if (decode_mode) {
    const float scale = 1.0f / sqrtf((float)hd);
    const dim3 dg(H, B, dec_split);  // the window in dec_split parts, merged by the last CTA of each (head, sequence)
    if (rope_in_attn) {
      if (hd == 64)
        attn_decode_rows_kernel<64><<<dg, 128, 0, st>>>((const bf16*)qkv, 3 * d, (const bf16*)Lw.ring_k,
                                                        (const bf16*)Lw.ring_v, C, d, kwin, pos_dev, scale,
                                                        (bf16*)o, d, dec_part, dec_ticket, rope_lo, rope_hi,
                                                        (bf16*)Lw.ring_k, (bf16*)Lw.ring_v);
      else
        attn_decode_rows_kernel<128><<<dg, 128, 0, st>>>((const bf16*)qkv, 3 * d, (const bf16*)Lw.ring_k,
                                                         (const bf16*)Lw.ring_v, C, d, kwin, pos_dev, scale,
                                                         (bf16*)o, d, dec_part, dec_ticket, rope_lo, rope_hi,
                                                         (bf16*)Lw.ring_k, (bf16*)Lw.ring_v);
      TTT_LAUNCHED();
      GemmParams pd = gp(rows, d, d, o, d, false, Lw.Wo, d, false, xout, d, true, EPI_RESID);
      pd.X = xin; pd.ldx = d;
      return gemm(pd);
    }
    const dim3 dg1(H, B, 1);  // one CTA per (head, sequence) for the register-heavy kernel
    switch (hd) {
      case 16: attn_decode_kernel<T, 16><<<dg1, 256, 0, st>>>(qkv, 3 * d, Lw.ring_k, Lw.ring_v, C, d, kwin, pos_dev, scale, o, d, dec_part, dec_ticket); break;
      case 32: attn_decode_kernel<T, 32><<<dg1, 256, 0, st>>>(qkv, 3 * d, Lw.ring_k, Lw.ring_v, C, d, kwin, pos_dev, scale, o, d, dec_part, dec_ticket); break;
      case 64: attn_decode_kernel<T, 64><<<dg1, 256, 0, st>>>(qkv, 3 * d, Lw.ring_k, Lw.ring_v, C, d, kwin, pos_dev, scale, o, d, dec_part, dec_ticket); break;
      case 128: attn_decode_kernel<T, 128><<<dg1, 256, 0, st>>>(qkv, 3 * d, Lw.ring_k, Lw.ring_v, C, d, kwin, pos_dev, scale, o, d, dec_part, dec_ticket); break;
      default: poisoned = true; return fail(this, TTT_ERR_UNSUPPORTED, "decode: head dim must be 16, 32, 64 or 128");
    }
    TTT_LAUNCHED();
    GemmParams pd = gp(rows, d, d, o, d, false, Lw.Wo, d, false, xout, d, true, EPI_RESID);
    pd.X = xin; pd.ldx = d;
    return gemm(pd);
  }
  AttnParams ap;
  memset(&ap, 0, sizeof(ap));
  ap.B = B; ap.H = H; ap.hd = hd; ap.n = n; ap.d = d; ap.q0 = q0; ap.window = kwin;
  ap.Q = qkv; ap.ldq = 3 * d; ap.K = qkv + d; ap.V = qkv + 2 * d; ap.ldkv = 3 * d;
  ap.Kc = Lw.ring_k; ap.Vc = Lw.ring_v; ap.C = C;
  ap.O = o; ap.ldo = d; ap.lse = lse; ap.scale = 1.0f / sqrtf((float)hd);
  prof.begin(st, PC_ATTN_FWD, 4.0 * hd * H * (double)B * attn_pairs(n, q0), 0.0);
  bool done = false;
  if (is_bf16 && attn_tc_ok(ap)) {
    const cudaError_t e = attn_fwd_tc_launch(ap, st, dev_err, &done);
    if (e != cudaSuccess) {
      poisoned = true;
      return fail(this, TTT_ERR_CUDA, std::string("attention: ") + cudaGetErrorString(e));
    }
  }
  if (!done) {
    if (is_bf16 && attn_mma_ok(ap)) {
      const cudaError_t e = hd == 128 ? attn_fwd_mma_launch<128>(ap, st) : attn_fwd_mma_launch<64>(ap, st);
      (void)e;
    } else {
      attn_fwd_simt_kernel<T><<<nblk((int64_t)rows * H, 4), 128, 0, st>>>(ap);
    }
  }
  prof.end(st);
  TTT_LAUNCHED();
  GemmParams p = gp(rows, d, d, o, d, false, Lw.Wo, d, false, xout, d, true, EPI_RESID);
  p.X = xin; p.ldx = d;
  if ((rc = gemm(p)) != TTT_OK) return rc;
  if (commit && !append_in_rope) {
    const int cnt = n > C ? C : n;
    const int64_t work = sizeof(T) == 2 ? (int64_t)B * cnt * (d / 8) : (int64_t)B * cnt * d;
    kv_append_kernel<T><<<nblk(work, 256), 256, 0, st>>>(qkv, 3 * d, d, 2 * d, n, B, q0, d, Lw.ring_k, Lw.ring_v,
                                                         C);
    TTT_LAUNCHED();
  }
  return TTT_OK;
}

// x += W2 gelu(W1 RMSNorm(x)) (frozen blocks)
template <typename T> int Engine<T>::frozen_mlp(const LayerDev<T>& Lw, float* x, T* r, T* hid, int rows) {
  int rc;
  GemmParams p1 = gp(rows, h, d, r, d, false, Lw.W1, d, false, hid, h, false, EPI_GELU);
  if ((rc = norm_into(p1, x, Lw.g_mlp, nullptr, r, rows)) != TTT_OK) return rc;
  if ((rc = gemm(p1)) != TTT_OK) return rc;
  GemmParams p = gp(rows, d, h, hid, h, false, Lw.W2, h, false, x, d, true, EPI_RESID);
  p.X = x; p.ldx = d;
  return gemm(p);
}

// Forward of the adaptive blocks for cn positions per sequence at pos..pos+cn-1.
// Input in tin, output in y. Activations of each block stay in blk[j].
template <typename T> int Engine<T>::ttt_forward(int cn, int64_t pos, bool commit) {
  const int rows = B * cn;
  int rc;
  if (Lt == 0) {  // no adaptive block: the head reads the frozen stack's output
    TTT_CUDA(cudaMemcpyAsync(y, tin, (size_t)rows * d * 4, cudaMemcpyDeviceToDevice, st));
    return TTT_OK;
  }
  for (int j = 0; j < Lt; ++j) {
    const int l = first_ttt + j;
    const LayerDev<T>& Lw = layers[l];
    BlockAct<T>& A = blk[j];
    if ((rc = attention_block(Lw, l, A.x, A.a, A.r3 /*scratch for r1*/, A.rstd1, A.qkv, A.o, A.lse, cn, pos,
                              commit)) != TTT_OK)
      return rc;
    // TTT-MLP with the fast weights of each sequence (batched over sequences). In the
    // key-value-binding variant it reads the key projection k = theta_K r2, and its
    // output is that binding prediction (the pre-update weights, the key projection).
    if (kvb) {
      GemmParams pk = gp(rows, d, d, A.r2, d, false, Lw.theta_kv, d, false, A.k, d, false, EPI_STORE);
      if ((rc = norm_into(pk, A.a, Lw.g_ttt, A.rstd2, A.r2, rows)) != TTT_OK) return rc;
      if ((rc = gemm(pk)) != TTT_OK) return rc;
    }
    GemmParams p = gp(cn, ht, d, kvb ? A.k : A.r2, d, false, Lw.W1t, d, false, A.g, ht, false, EPI_GELU);
    p.batch = B; p.sA = (int64_t)cn * d; p.sD = (int64_t)cn * ht;
    if (!kvb && (rc = norm_into(p, A.a, Lw.g_ttt, A.rstd2, A.r2, rows)) != TTT_OK) return rc;
    fast_operand(p, Lw.W1t_init, Lw.W1t, (int64_t)ht * d);
    p.Y = A.u; p.ldy = ht; p.sY = (int64_t)cn * ht;
    if ((rc = gemm(p)) != TTT_OK) return rc;
    p = gp(cn, d, ht, A.g, ht, false, Lw.W2t, ht, false, A.m, d, true, EPI_RESID);
    p.batch = B; p.sA = (int64_t)cn * ht; p.sD = (int64_t)cn * d;
    fast_operand(p, Lw.W2t_init, Lw.W2t, (int64_t)d * ht);
    p.X = A.a; p.ldx = d; p.sX = (int64_t)cn * d;
    if ((rc = gemm(p)) != TTT_OK) return rc;
    // static MLP
    p = gp(rows, hs, d, A.r3, d, false, Lw.W1s, d, false, A.gs, hs, false, EPI_GELU);
    p.Y = A.us; p.ldy = hs;
    if ((rc = norm_into(p, A.m, Lw.g_static, A.rstd3, A.r3, rows)) != TTT_OK) return rc;
    if ((rc = gemm(p)) != TTT_OK) return rc;
    float* xnext = (j + 1 < Lt) ? blk[j + 1].x : y;
    p = gp(rows, d, hs, A.gs, hs, false, Lw.W2s, hs, false, xnext, d, true, EPI_RESID);
    p.X = A.m; p.ldx = d;
    if ((rc = gemm(p)) != TTT_OK) return rc;
  }
  return TTT_OK;
}

// Reverse mode from dz (in z) back to every adaptive MLP, with the SGD step
// fused into the weight-gradient GEMMs (W <- W - eta * dW, dW already a mean).
template <typename T> int Engine<T>::ttt_backward(int cn) {
  const int rows = B * cn;
  int rc;
  // LM head: dr = dz E ; G = d loss / d y through the final RMSNorm
  if ((rc = gemm(gp(rows, d, V, z, V, false, E, d, true, dr, d, true, EPI_STORE))) != TTT_OK) return rc;
  rmsnorm_bwd_launch<T>((const float*)y, g_final, rstdf, dr, nullptr, rows, d, G, GT, st);
  TTT_LAUNCHED();
  for (int j = Lt - 1; j >= 0; --j) {
    const int l = first_ttt + j;
    const LayerDev<T>& Lw = layers[l];
    BlockAct<T>& A = blk[j];
    // static MLP (frozen): dm = G + RMSNorm_bwd(W1s^T (gelu'(us) * (W2s^T G)))
    GemmParams p = gp(rows, hs, d, GT, d, false, Lw.W2s, hs, true, dhid, hs, false, EPI_DGELU);
    p.X = A.us; p.ldx = hs;
    if ((rc = gemm(p)) != TTT_OK) return rc;
    if ((rc = gemm(gp(rows, d, hs, dhid, hs, false, Lw.W1s, d, true, dr, d, true, EPI_STORE))) != TTT_OK) return rc;
    rmsnorm_bwd_launch<T>((const float*)A.m, Lw.g_static, A.rstd3, dr, G, rows, d, G, GT, st);
    TTT_LAUNCHED();
    // TTT-MLP data gradients (with W_{i-1}), then the fused weight gradient + SGD
    p = gp(cn, ht, d, GT, d, false, Lw.W2t, ht, true, dhid, ht, false, EPI_DGELU);
    p.batch = B; p.sA = (int64_t)cn * d; p.sD = (int64_t)cn * ht;
    fast_operand(p, Lw.W2t_init, Lw.W2t, (int64_t)d * ht);
    p.X = A.u; p.ldx = ht; p.sX = (int64_t)cn * ht;
    if ((rc = gemm(p)) != TTT_OK) return rc;
    if (j > 0) {
      p = gp(cn, d, ht, dhid, ht, false, Lw.W1t, d, true, dr, d, true, EPI_STORE);
      p.batch = B; p.sA = (int64_t)cn * ht; p.sD = (int64_t)cn * d;
      fast_operand(p, Lw.W1t_init, Lw.W1t, (int64_t)ht * d);
      if ((rc = gemm(p)) != TTT_OK) return rc;
    }
    // dW2t[o][i] = sum_t dm[t][o] g[t][i]  -> W2t32 += -eta * dW2t ; bf16 copy refreshed
    // (bf16 path: W2t32 holds the accumulated update dW, so the copy keeps its precision)
    GemmParams p2w = gp(d, ht, cn, GT, d, true, A.g, ht, true, Lw.W2t32, ht, true, EPI_SGD);
    p2w.batch = B; p2w.sA = (int64_t)cn * d; p2w.sB = (int64_t)cn * ht; p2w.sD = (int64_t)d * ht;
    p2w.alpha = -cfg.eta;
    if (is_bf16) { p2w.Y = Lw.W2t; p2w.ldy = ht; p2w.sY = (int64_t)d * ht; }
    // dW1t[o][i] = sum_t du[t][o] r2[t][i]; independent of dW2t: both in one launch
    GemmParams p1w = gp(ht, d, cn, dhid, ht, true, A.r2, d, true, Lw.W1t32, d, true, EPI_SGD);
    p1w.batch = B; p1w.sA = (int64_t)cn * ht; p1w.sB = (int64_t)cn * d; p1w.sD = (int64_t)ht * d;
    p1w.alpha = -cfg.eta;
    if (is_bf16) { p1w.Y = Lw.W1t; p1w.ldy = d; p1w.sY = (int64_t)ht * d; }
    if ((rc = gemm2(p2w, p1w)) != TTT_OK) return rc;
    if (j == 0) break;  // upstream of the first adaptive MLP does not depend on the fast weights
    rmsnorm_bwd_launch<T>((const float*)A.a, Lw.g_ttt, A.rstd2, dr, G, rows, d, G, GT, st);
    TTT_LAUNCHED();
    // frozen attention: data gradients only; cached K/V are constants
    if ((rc = gemm(gp(rows, d, d, GT, d, false, Lw.Wo, d, true, dob, d, false, EPI_STORE))) != TTT_OK) return rc;
    AttnParams ap;
    memset(&ap, 0, sizeof(ap));
    ap.B = B; ap.H = H; ap.hd = hd; ap.n = cn; ap.d = d; ap.q0 = 0; ap.window = kwin;
    ap.Q = A.qkv; ap.ldq = 3 * d; ap.K = A.qkv + d; ap.V = A.qkv + 2 * d; ap.ldkv = 3 * d;
    ap.Kc = Lw.ring_k; ap.Vc = Lw.ring_v; ap.C = C;
    ap.O = A.o; ap.ldo = d; ap.lse = A.lse; ap.scale = 1.0f / sqrtf((float)hd);
    ap.dO = dob; ap.lddo = d; ap.Dsum = Dsum;
    ap.dQ = dqkv; ap.dK = dqkv + d; ap.dV = dqkv + 2 * d; ap.lddq = 3 * d;
    ap.q0 = chunk_pos;
    // algorithmic (recompute of QK^T not counted): dQ over the window (dO V^T, dS K) and
    // dK, dV over current-chunk keys only (dS^T Q, P^T dO)
    prof.begin(st, PC_ATTN_BWD,
               2.0 * hd * H * (double)B * (2.0 * attn_pairs(cn, chunk_pos) + 2.0 * attn_pairs(cn, 0)), 0.0);
    // dQ and dK/dV: tcgen05 kernels where they apply (the dQ kernel forms D = rowsum(dO * O)
    // itself), else a separate D pass and the mma.sync or SIMT kernels
    bool dq_done = false, dkv_done = false;
    if (is_bf16 && attn_dq_tc_ok(ap)) {
      ap.dsum_in_dq = 1;
      cudaError_t e = attn_bwd_dq_tc_launch(ap, st, dev_err, &dq_done);
      ap.dsum_in_dq = 0;
      if (e == cudaSuccess && dq_done && attn_dkv_tc_ok(ap)) e = attn_bwd_dkv_tc_launch(ap, st, dev_err, &dkv_done);
      if (e != cudaSuccess) {
        poisoned = true;
        return fail(this, TTT_ERR_CUDA, std::string("attention backward: ") + cudaGetErrorString(e));
      }
    }
    if (!dq_done) {
      attn_bwd_prep_kernel<T><<<nblk((int64_t)rows * H, 8), 256, 0, st>>>(ap);
      TTT_LAUNCHED();
    }
    if (!(dq_done && dkv_done)) {
      if (is_bf16 && attn_mma_ok(ap)) {
        const cudaError_t e = hd == 128 ? attn_bwd_mma_launch<128>(ap, st, !dq_done, !dkv_done)
                                        : attn_bwd_mma_launch<64>(ap, st, !dq_done, !dkv_done);
        (void)e;  // checked by the launch accounting below
      } else {
        if (!dq_done) attn_bwd_dq_simt_kernel<T><<<nblk((int64_t)rows * H, 4), 128, 0, st>>>(ap);
        if (!dkv_done) attn_bwd_dkv_simt_kernel<T><<<nblk((int64_t)rows * H, 4), 128, 0, st>>>(ap);
      }
    }
    launches += 1;  // dQ and dK/dV are two launches whichever engine ran them; one more below
    prof.end(st);
    TTT_LAUNCHED();
    rope_launch<T>(dqkv, 3 * d, 2 * d, rows, cn, chunk_pos, hd, rope_lo, rope_hi, 1, nullptr, st);
    TTT_LAUNCHED();
    if ((rc = gemm(gp(rows, d, 3 * d, dqkv, 3 * d, false, Lw.Wqkv, d, true, dr, d, true, EPI_STORE))) != TTT_OK)
      return rc;
    // G <- G + RMSNorm_bwd through the attention norm: gradient w.r.t. this block's input
    rmsnorm_bwd_launch<T>((const float*)A.x, Lw.g_attn, A.rstd1, dr, G, rows, d, G, GT, st);
    TTT_LAUNCHED();
  }
  return TTT_OK;
}

// Key-value-binding variant of the update (technical review §8, eq. (10); summary,
// "Alternative Derivation"): every adaptive block j descends its own chunk loss
// (1/b) sum_t ||g(k_t; W) - v_t||^2, g(k; W) = W2t gelu(W1t k), with k = theta_K r2 and
// v = theta_V r2, r2 the block's normalised rows ahead of its MLP. The forward with
// W_{i-1} already made the prediction: it is the MLP sub-layer's output m - a, with
// u = W1t k and gelu(u) kept in the block's buffers. Layer-wise: no gradient passes
// between blocks, so each block's update reads only its own rows and fast weights.
// de = (2/b)(m - a - v), du = (de W2t) * gelu'(u), dW2t = de^T gelu(u), dW1t = du^T k.
template <typename T> int Engine<T>::kvb_update(int cn) {
  const int rows = B * cn;
  int rc;
  const float two_over_b = 2.0f / (float)bsz;
  for (int j = 0; j < Lt; ++j) {
    const LayerDev<T>& Lw = layers[first_ttt + j];
    BlockAct<T>& A = blk[j];
    // G = -(2/b) v
    GemmParams pv = gp(rows, d, d, A.r2, d, false, Lw.theta_kv + (size_t)d * d, d, false, G, d, true, EPI_STORE);
    pv.alpha = -two_over_b;
    if ((rc = gemm(pv)) != TTT_OK) return rc;
    // G = (2/b)(m - a) + G = de (fp32), GT its element-type copy for the products below
    const cudaError_t e = launch_pdl(kvb_residual_kernel<T>, dim3(nblk((int64_t)rows * d / 4, 256)), dim3(256), 0,
                                     st, (const float*)A.m, (const float*)A.a, G, GT, two_over_b,
                                     (int64_t)rows * d / 4);
    if (e != cudaSuccess) {
      poisoned = true;
      return fail(this, TTT_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
    }
    TTT_LAUNCHED();
    // du = (de W2t) * gelu'(u)
    GemmParams p = gp(cn, ht, d, GT, d, false, Lw.W2t, ht, true, dhid, ht, false, EPI_DGELU);
    p.batch = B; p.sA = (int64_t)cn * d; p.sD = (int64_t)cn * ht;
    fast_operand(p, Lw.W2t_init, Lw.W2t, (int64_t)d * ht);
    p.X = A.u; p.ldx = ht; p.sX = (int64_t)cn * ht;
    if ((rc = gemm(p)) != TTT_OK) return rc;
    // W2t -= eta de^T gelu(u), W1t -= eta du^T k: one launch, SGD fused into the epilogue
    GemmParams p2w = gp(d, ht, cn, GT, d, true, A.g, ht, true, Lw.W2t32, ht, true, EPI_SGD);
    p2w.batch = B; p2w.sA = (int64_t)cn * d; p2w.sB = (int64_t)cn * ht; p2w.sD = (int64_t)d * ht;
    p2w.alpha = -cfg.eta;
    if (is_bf16) { p2w.Y = Lw.W2t; p2w.ldy = ht; p2w.sY = (int64_t)d * ht; }
    GemmParams p1w = gp(ht, d, cn, dhid, ht, true, A.k, d, true, Lw.W1t32, d, true, EPI_SGD);
    p1w.batch = B; p1w.sA = (int64_t)cn * ht; p1w.sB = (int64_t)cn * d; p1w.sD = (int64_t)ht * d;
    p1w.alpha = -cfg.eta;
    if (is_bf16) { p1w.Y = Lw.W1t; p1w.ldy = d; p1w.sY = (int64_t)ht * d; }
    if ((rc = gemm2(p2w, p1w)) != TTT_OK) return rc;
  }
  return TTT_OK;
}

}  // namespace ttt

namespace ttt {

// One adaptive step over cn positions per sequence (rows [B][cn], pos..pos+cn-1):
// forward with W_{i-1}, losses recorded, and (grad) backward + in-place SGD.
template <typename T>
int Engine<T>::ttt_step(const float* in, const int32_t* targets, int cn, int64_t pos, float* loss_out,
                        int64_t loss_ld, int64_t loss_off, bool grad, bool commit) {
  const int rows = B * cn;
  int rc;
  chunk_pos = pos;
  gemm_class = PC_GEMM_TTT;
  grad = grad && Lt > 0;  // without adaptive blocks there is nothing to update
  if (in != tin) {
    TTT_CUDA(cudaMemcpyAsync(tin, in, (size_t)rows * d * 4, cudaMemcpyDeviceToDevice, st));
  }
  if (targets != tgt) {
    TTT_CUDA(cudaMemcpyAsync(tgt, targets, (size_t)rows * 4, cudaMemcpyDeviceToDevice, st));
  }
  if ((rc = ttt_forward(cn, pos, commit)) != TTT_OK) return rc;
  rmsnorm_fwd_launch<T>((const float*)y, d, g_final, cfg.rms_eps, rows, d, rf, d, rstdf, st);
  TTT_LAUNCHED();
  // LM head + cross-entropy, chunked over the vocabulary: the tcgen05 GEMM epilogue
  // keeps an fp32 (max, sum-exp) per row and 64-column chunk and the target's fp32
  // logit; ce_finish merges the chunks, records the loss and writes dz in place of
  // the logits. The gradient is the mean over the b positions of the chunk
  // (summary: mini-batch GD with 1/b).
  GemmParams ph = gp(rows, V, d, rf, d, false, E, d, false, z, V, false, EPI_STORE);
  // the key-value-binding variant needs no dz: its update never reads the head's gradient
  const float gscale = (grad && !kvb) ? 1.0f / bsz : 0.f;
  bool fused = false;
  if (ce_part) {
    GemmParams pc = ph;
    pc.epi = EPI_CE; pc.ce_tgt = tgt; pc.ce_part = ce_part; pc.ce_zt = ce_zt;
    if (gemm_uses_tc(pc, 1)) { ph = pc; fused = true; }
  }
  if ((rc = gemm(ph)) != TTT_OK) return rc;
  if (fused) {
    launch_pdl(ce_finish_kernel<T>, dim3(rows), dim3(256), 0, st, z, V, (const float2*)ce_part,
               (const float*)ce_zt, (const int32_t*)tgt, cn, loss_out, loss_ld, loss_off, gscale, dev_err);
  } else {
    ce_kernel<T><<<rows, 256, 0, st>>>(z, V, tgt, cn, loss_out, loss_ld, loss_off, gscale, dev_err);
  }
  TTT_LAUNCHED();
  if (grad) {
    if ((rc = kvb ? kvb_update(cn) : ttt_backward(cn)) != TTT_OK) return rc;
  }
  return TTT_OK;
}

// ------------------------------------------------------------------ prefill (Algorithm 1)
template <typename T> int Engine<T>::prefill(const int32_t* tokens, int64_t T_, float* out, int32_t kind) {
  if (poisoned) return fail(this, TTT_ERR_POISONED, "handle poisoned by an earlier device error");
  if (!tokens || !out || T_ <= 0) return fail(this, TTT_ERR_INVALID_ARG, "prefill: null buffer or T <= 0");
  if (pend_cnt != 0) return fail(this, TTT_ERR_STREAM, "prefill: a partial chunk is pending; decode completes it");
  if ((n_pos + T_) / 1024 >= kRopeHi) return fail(this, TTT_ERR_INVALID_ARG, "prefill: position limit exceeded");
  launches = 0;
  const int64_t ld = T_ + 1;
  int rc;
  if ((rc = ensure((void**)&tok_dev, &tok_cap, (int64_t)B * ld, 4)) != TTT_OK) return rc;
  if ((rc = ensure((void**)&loss_dev, &loss_cap, (int64_t)B * T_, 4)) != TTT_OK) return rc;
  std::vector<int32_t> first(B), last(B);
  if (kind == TTT_PTR_HOST) {
    for (int b = 0; b < B; ++b) { first[b] = tokens[b * ld]; last[b] = tokens[b * ld + T_]; }
    TTT_CUDA(cudaMemcpyAsync(tok_dev, tokens, (size_t)B * ld * 4, cudaMemcpyHostToDevice, st));
  } else {
    TTT_CUDA(cudaMemcpyAsync(tok_dev, tokens, (size_t)B * ld * 4, cudaMemcpyDeviceToDevice, st));
    for (int b = 0; b < B; ++b) {
      TTT_CUDA(cudaMemcpyAsync(&first[b], tok_dev + b * ld, 4, cudaMemcpyDeviceToHost, st));
      TTT_CUDA(cudaMemcpyAsync(&last[b], tok_dev + b * ld + T_, 4, cudaMemcpyDeviceToHost, st));
    }
    TTT_CUDA(cudaStreamSynchronize(st));
  }
  if (n_pos > 0)
    for (int b = 0; b < B; ++b)
      if (first[b] != pend_tok_host[b]) return fail(this, TTT_ERR_STREAM, "prefill: first id is not the pending token");
  float* lout = kind == TTT_PTR_DEVICE ? out : loss_dev;
  for (int64_t s0 = 0; s0 < T_; s0 += S) {
    const int n = (int)((T_ - s0) < S ? (T_ - s0) : S);
    const int64_t P0 = n_pos + s0;
    const int rows = B * n;
    embed_kernel<T><<<nblk(rows, 4), 128, 0, st>>>(tok_dev, ld, (int)s0, n, rows, E, V, d, xs, dev_err);
    TTT_LAUNCHED();
    gemm_class = PC_GEMM_FROZEN;
    for (int l = 0; l < first_ttt; ++l) {
      if ((rc = attention_block(layers[l], l, xs, xs, rs, nullptr, qkvs, os, nullptr, n, P0, true)) != TTT_OK)
        return rc;
      if ((rc = frozen_mlp(layers[l], xs, rs, hids, rows)) != TTT_OK) return rc;
    }
    for (int c0 = 0; c0 < n; c0 += bsz) {
      const int cn = (n - c0) < bsz ? (n - c0) : bsz;
      gather_chunk_kernel<<<nblk((int64_t)B * cn * (d / 4), 256), 256, 0, st>>>(xs, (int64_t)n * d, c0, cn, B, d, tin,
                                                                                tok_dev, ld, s0 + c0 + 1, tgt);
      TTT_LAUNCHED();
      const bool full = cn == bsz;
      if ((rc = ttt_step(tin, tgt, cn, P0 + c0, lout, T_, s0 + c0, full, true)) != TTT_OK) return rc;
      if (!full) {  // trailing partial chunk: keep its inputs and targets pending
        TTT_CUDA(cudaMemcpy2DAsync(pend_in, (size_t)bsz * d * 4, tin, (size_t)cn * d * 4, (size_t)cn * d * 4, B,
                                   cudaMemcpyDeviceToDevice, st));
        TTT_CUDA(cudaMemcpy2DAsync(pend_tgt, (size_t)bsz * 4, tgt, (size_t)cn * 4, (size_t)cn * 4, B,
                                   cudaMemcpyDeviceToDevice, st));
        pend_cnt = cn;
      }
    }
  }
  gather_tokens_kernel<<<nblk(B, 256), 256, 0, st>>>(tok_dev, ld, T_, 1, B, pend_tok_dev, 1, 0);
  TTT_LAUNCHED();
  if (kind == TTT_PTR_HOST) {
    TTT_CUDA(cudaMemcpyAsync(out, loss_dev, (size_t)B * T_ * 4, cudaMemcpyDeviceToHost, st));
  }
  if ((rc = sync_and_check()) != TTT_OK) return rc;
  n_pos += T_;
  pend_tok_host = last;
  return TTT_OK;
}

// ------------------------------------------------------------------ decode (Algorithm 3)
// One generated token per sequence = one replay of a CUDA graph captured at the
// start of the call: embedding of the pending id, every block for one position
// (window attention read from the rings), LM head, greedy (or forced) choice,
// bookkeeping, position advance. Every b decoded positions the completed chunk is
// re-forwarded with W_{i-1}, differentiated and the fast weights updated.
template <typename T> int Engine<T>::decode_token_launches(int64_t n, int32_t* otok, float* oloss, const int32_t* fdev,
                                                           int64_t base) {
  const int rows = B;
  int rc;
  embed_kernel<T><<<nblk(rows, 4), 128, 0, st>>>(pend_tok_dev, 1, 0, 1, rows, E, V, d, xs, dev_err);
  TTT_LAUNCHED();
  gemm_class = PC_GEMM_FROZEN;
  for (int l = 0; l < first_ttt; ++l) {
    if ((rc = attention_block(layers[l], l, xs, xs, rs, nullptr, qkvs, os, nullptr, 1, 0, true)) != TTT_OK) return rc;
    if ((rc = frozen_mlp(layers[l], xs, rs, hids, rows)) != TTT_OK) return rc;
  }
  // keep the first adaptive block's input of this position for the chunk's update
  pend_store_kernel<<<nblk((int64_t)B * d, 256), 256, 0, st>>>(xs, B, d, pend_in, bsz, pos_dev);
  TTT_LAUNCHED();
  TTT_CUDA(cudaMemcpyAsync(tin, xs, (size_t)B * d * 4, cudaMemcpyDeviceToDevice, st));
  gemm_class = PC_GEMM_TTT;
  if ((rc = ttt_forward(1, 0, true)) != TTT_OK) return rc;
  {
    GemmParams ph = gp(rows, V, d, rf, d, false, E, d, false, z, V, false, EPI_STORE);
    if ((rc = norm_into(ph, y, g_final, rstdf, rf, rows)) != TTT_OK) return rc;
    if ((rc = gemm(ph)) != TTT_OK) return rc;
  }
  const int32_t* fcol = nullptr;
  if (fdev) {
    forced_gather_kernel<<<1, 32 * ((B + 31) / 32), 0, st>>>(fdev, n, B, forced_col, pos_dev, base);
    TTT_LAUNCHED();
    fcol = forced_col;
  }
  argmax_kernel<T><<<rows, 1024, 0, st>>>(z, V, fcol, pend_tok_dev, dec_loss, dec_zmax);
  TTT_LAUNCHED();
  decode_record_kernel<<<1, 32 * ((B + 31) / 32), 0, st>>>(pend_tok_dev, dec_loss, B, n, otok, oloss, pend_tgt, bsz,
                                                           pos_dev, base);
  TTT_LAUNCHED();
  decode_advance_kernel<<<1, 1, 0, st>>>(pos_dev);
  TTT_LAUNCHED();
  return TTT_OK;
}

template <typename T>
int Engine<T>::decode(int64_t n, const int32_t* forced, int32_t* out_tok, float* out_loss, int32_t kind) {
  if (poisoned) return fail(this, TTT_ERR_POISONED, "handle poisoned by an earlier device error");
  if (n <= 0 || !out_tok) return fail(this, TTT_ERR_INVALID_ARG, "decode: n <= 0 or null output");
  if (n_pos == 0) return fail(this, TTT_ERR_STREAM, "decode: nothing prefilled (no pending token)");
  if ((n_pos + n) / 1024 >= kRopeHi) return fail(this, TTT_ERR_INVALID_ARG, "decode: position limit exceeded");
  launches = 0;
  int rc;
  int32_t* otok = out_tok;
  float* oloss = out_loss;
  const int32_t* fdev = nullptr;
  if ((rc = ensure((void**)&otok_dev, &otok_cap, (int64_t)B * n * 2, 4)) != TTT_OK) return rc;
  if ((rc = ensure((void**)&loss_dev, &loss_cap, (int64_t)B * n, 4)) != TTT_OK) return rc;
  if (kind == TTT_PTR_HOST) {
    otok = otok_dev;
    oloss = out_loss ? loss_dev : nullptr;
    if (forced) {
      int32_t* f = otok_dev + (int64_t)B * n;
      TTT_CUDA(cudaMemcpyAsync(f, forced, (size_t)B * n * 4, cudaMemcpyHostToDevice, st));
      fdev = f;
    }
  } else {
    fdev = forced;
  }
  const int64_t base = n_pos;
  TTT_CUDA(cudaMemcpyAsync(pos_dev, &base, sizeof(int64_t), cudaMemcpyHostToDevice, st));
  TTT_CUDA(cudaStreamSynchronize(st));  // the source lives on the host stack
  // capture one token step
  const bool prof_on = prof.on;
  prof.on = false;
  decode_mode = true;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  cudaStream_t user_st = st;
  st = cap_st;  // capture only records: nothing runs on cap_st; the graph runs on the caller's stream
  cudaError_t ce = cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal);
  if (ce != cudaSuccess) {
    st = user_st;
    decode_mode = false;
    prof.on = prof_on;
    poisoned = true;
    return fail(this, TTT_ERR_CUDA, std::string("decode capture: ") + cudaGetErrorString(ce));
  }
  const int64_t before = launches;
  rc = decode_token_launches(n, otok, oloss, fdev, base);
  const int64_t per_token = launches - before;
  ce = cudaStreamEndCapture(st, &graph);
  st = user_st;
  decode_mode = false;
  prof.on = prof_on;
  if (rc != TTT_OK) {
    if (graph) cudaGraphDestroy(graph);
    return rc;
  }
  if (ce == cudaSuccess) ce = cudaGraphInstantiate(&exec, graph, 0);
  if (graph) cudaGraphDestroy(graph);
  if (ce != cudaSuccess) {
    poisoned = true;
    return fail(this, TTT_ERR_CUDA, std::string("decode graph: ") + cudaGetErrorString(ce));
  }
  launches = 0;
  for (int64_t t = 0; t < n; ++t) {
    ce = cudaGraphLaunch(exec, st);
    if (ce != cudaSuccess) break;
    launches += per_token;
    ++pend_cnt;
    ++n_pos;
    if (pend_cnt == bsz) {  // a full chunk of decoded positions: differentiate and update
      if (Lt > 0 && (rc = ttt_step(pend_in, pend_tgt, bsz, n_pos - bsz, nullptr, 0, 0, true, false)) != TTT_OK) {
        cudaGraphExecDestroy(exec);
        return rc;
      }
      pend_cnt = 0;
    }
  }
  if (ce != cudaSuccess) {
    cudaGraphExecDestroy(exec);
    poisoned = true;
    return fail(this, TTT_ERR_CUDA, std::string("decode graph launch: ") + cudaGetErrorString(ce));
  }
  if (kind == TTT_PTR_HOST) {
    TTT_CUDA(cudaMemcpyAsync(out_tok, otok_dev, (size_t)B * n * 4, cudaMemcpyDeviceToHost, st));
    if (out_loss) TTT_CUDA(cudaMemcpyAsync(out_loss, loss_dev, (size_t)B * n * 4, cudaMemcpyDeviceToHost, st));
  }
  TTT_CUDA(cudaMemcpyAsync(pend_tok_host.data(), pend_tok_dev, (size_t)B * 4, cudaMemcpyDeviceToHost, st));
  rc = sync_and_check();
  cudaGraphExecDestroy(exec);
  return rc;
}

template <typename T> int Engine<T>::get_weights(int32_t seq, int32_t j, float* w1, float* w2, int32_t kind) {
  if (poisoned) return fail(this, TTT_ERR_POISONED, "handle poisoned by an earlier device error");
  if (seq < 0 || seq >= B || j < 0 || j >= Lt) return fail(this, TTT_ERR_INVALID_ARG, "get_weights: bad index");
  const LayerDev<T>& Lw = layers[first_ttt + j];
  const int64_t n1 = (int64_t)ht * d;
  const cudaMemcpyKind k = kind == TTT_PTR_HOST ? cudaMemcpyDeviceToHost : cudaMemcpyDeviceToDevice;
  if (!is_bf16) {
    if (w1) TTT_CUDA(cudaMemcpyAsync(w1, Lw.W1t32 + seq * n1, n1 * 4, k, st));
    if (w2) TTT_CUDA(cudaMemcpyAsync(w2, Lw.W2t32 + seq * n1, n1 * 4, k, st));
    return sync_and_check();
  }
  // W = W_init + dW, formed in fp32 on the device
  float* stage = nullptr;
  int64_t cap = 0;
  int rc;
  if ((rc = ensure((void**)&wexp, &wexp_cap, n1, 4)) != TTT_OK) return rc;
  stage = wexp;
  (void)cap;
  for (int m = 0; m < 2; ++m) {
    float* dst = m == 0 ? w1 : w2;
    if (!dst) continue;
    add_init_kernel<T><<<nblk(n1, 256), 256, 0, st>>>(m == 0 ? Lw.W1t_init : Lw.W2t_init,
                                                      (m == 0 ? Lw.W1t32 : Lw.W2t32) + seq * n1, stage, n1);
    TTT_LAUNCHED();
    TTT_CUDA(cudaMemcpyAsync(dst, stage, n1 * 4, k, st));
    TTT_CUDA(cudaStreamSynchronize(st));
  }
  return sync_and_check();
}

static int validate(const ttt_config* c, std::string* why) {
  auto bad = [&](const char* m) { *why = m; return TTT_ERR_INVALID_ARG; };
  if (!c) return bad("null config");
  if (c->vocab <= 0 || c->d <= 0 || c->n_layers <= 0 || c->n_heads <= 0 || c->batch <= 0) return bad("non-positive size");
  if (c->n_ttt < 0 || c->n_ttt > c->n_layers) return bad("n_ttt must be in [0, n_layers]");
  if (c->d % c->n_heads) return bad("d must be a multiple of n_heads");
  const int hd = c->d / c->n_heads;
  if (hd != 16 && hd != 32 && hd != 64 && hd != 128) return bad("head dim must be 16, 32, 64 or 128");
  if (c->minibatch_b <= 0 || c->window_k < c->minibatch_b) return bad("need window_k >= minibatch_b > 0");
  if (c->d % 8 || c->mlp_hidden % 8 || c->ttt_hidden % 8 || c->static_hidden % 8 || c->vocab % 8)
    return bad("widths and vocab must be multiples of 8");
  if (c->mlp_hidden <= 0 || c->ttt_hidden <= 0 || c->static_hidden <= 0) return bad("non-positive hidden width");
  if (c->dtype != TTT_FP32 && c->dtype != TTT_BF16) return bad("dtype must be TTT_FP32 or TTT_BF16");
  if (c->inner_loss != TTT_LOSS_E2E && c->inner_loss != TTT_LOSS_KVB)
    return bad("inner_loss must be TTT_LOSS_E2E or TTT_LOSS_KVB");
  if (!(c->rms_eps > 0.f) || !(c->rope_base > 1.f) || !std::isfinite(c->eta)) return bad("bad eps, rope base or eta");
  return TTT_OK;
}

}  // namespace ttt

// ============================================================== C ABI
using namespace ttt;

extern "C" {

int32_t ttt_num_weight_tensors(const ttt_config* c) {
  if (!c) return -1;
  return 2 + (c->n_layers - c->n_ttt) * 8 + c->n_ttt * (c->inner_loss == TTT_LOSS_KVB ? 13 : 11);
}

int ttt_create(const ttt_config* cfg, const ttt_weights* w, ttt_handle** out) {
  if (!out) return TTT_ERR_INVALID_ARG;
  *out = nullptr;
  std::string why;
  if (validate(cfg, &why) != TTT_OK) return TTT_ERR_INVALID_ARG;
  if (!w || !w->tensors || w->n_tensors != ttt_num_weight_tensors(cfg)) return TTT_ERR_INVALID_ARG;
  ttt_handle* h = nullptr;
  int rc;
  try {
    if (cfg->dtype == TTT_BF16) {
      auto* e = new Engine<bf16>();
      h = e;
      rc = e->create(cfg, w);
    } else {
      auto* e = new Engine<float>();
      h = e;
      rc = e->create(cfg, w);
    }
  } catch (...) {
    delete h;
    return TTT_ERR_OOM;
  }
  if (rc != TTT_OK) {
    delete h;
    return rc;
  }
  *out = h;
  return TTT_OK;
}

int ttt_prefill(ttt_handle* h, const int32_t* tokens, int64_t T, float* out_losses, int32_t ptr_kind) {
  if (!h) return TTT_ERR_INVALID_ARG;
  try { return h->prefill(tokens, T, out_losses, ptr_kind); } catch (...) { return TTT_ERR_OOM; }
}

int ttt_decode(ttt_handle* h, int64_t n, const int32_t* forced, int32_t* out_tokens, float* out_losses,
               int32_t ptr_kind) {
  if (!h) return TTT_ERR_INVALID_ARG;
  try { return h->decode(n, forced, out_tokens, out_losses, ptr_kind); } catch (...) { return TTT_ERR_OOM; }
}

int ttt_get_weights(ttt_handle* h, int32_t seq, int32_t ttt_block, float* w1, float* w2, int32_t ptr_kind) {
  if (!h) return TTT_ERR_INVALID_ARG;
  return h->get_weights(seq, ttt_block, w1, w2, ptr_kind);
}

int ttt_reset(ttt_handle* h) {
  if (!h) return TTT_ERR_INVALID_ARG;
  return h->reset();
}

int64_t ttt_position(const ttt_handle* h) { return h ? h->n_pos : -1; }
int64_t ttt_device_bytes(const ttt_handle* h) { return h ? h->dev_bytes : -1; }
int64_t ttt_last_launch_count(const ttt_handle* h) { return h ? h->launches : -1; }

int ttt_profile(ttt_handle* h, int32_t enable) {
  if (!h) return TTT_ERR_INVALID_ARG;
  h->prof.on = enable != 0;
  h->prof.clear();
  return TTT_OK;
}

int ttt_profile_read(const ttt_handle* h, int32_t n_classes, double* ms, int64_t* launches, double* flops,
                     double* bytes) {
  if (!h || n_classes < 0) return TTT_ERR_INVALID_ARG;
  for (int c = 0; c < n_classes && c < PC_COUNT; ++c) {
    if (ms) ms[c] = h->prof.ms[c];
    if (launches) launches[c] = h->prof.n[c];
    if (flops) flops[c] = h->prof.flops[c];
    if (bytes) bytes[c] = h->prof.bytes[c];
  }
  return PC_COUNT;
}

void ttt_destroy(ttt_handle* h) { delete h; }

void ttt_test_fail_allocation(int64_t n) { g_fail_countdown.store(n < 0 ? -1 : n); }

int64_t ttt_test_allocation_count(void) { return g_alloc_count.load(); }

int ttt_test_set_device_status(ttt_handle* h, int32_t code) {
  if (!h) return TTT_ERR_INVALID_ARG;
  return h->set_device_status(code);
}

const char* ttt_last_error(const ttt_handle* h) { return h ? h->err_msg.c_str() : "null handle"; }

const char* ttt_version(void) { return "ttt-e2e-b200 0.1 (sm_100a)"; }

}  // extern "C"
