// Per-kernel C ABI (include/ttt_kernels.h): one contraction or one attention
// pass at a time, on caller-provided device buffers.
#include <cmath>
#include <cstring>
#include <mutex>

#include "ttt.h"
#include "ttt_attention.cuh"
#include "ttt_attention_mma.cuh"
#include "ttt_common.cuh"
#include "ttt_gemm.cuh"
#include "ttt_kernels.h"
#include "ttt_ce.cuh"
#include "ttt_testing.h"

namespace ttt {

// ---------------------------------------------------------------- library-resident device words
// Status word of the per-kernel entry points: kernels whose bounded wait runs out
// record a code here (see ttt_common.cuh); ttt_k_status reads and clears it. It
// lives in this library's own device image (zero at load), so no entry point
// allocates it.
static __device__ int g_kernel_status;

// Scratch of ttt_k_attention_bwd_noalloc: the per-row sums D = rowsum(dO * O),
// one float per (sequence, head, row). It lives in this library's own device
// image, so every GPU that loads the library holds these 4 MiB until the process
// exits, and no call ever allocates. The host must not pass the symbol itself to
// a kernel (in host code it names a host-side stand-in); it passes the device
// address that cudaGetSymbolAddress returns for the current device.
constexpr int64_t kNoAllocDsumFloats = int64_t(1) << 20;
static __device__ __align__(256) float g_noalloc_dsum[kNoAllocDsumFloats];

// Device addresses of the two words above on the current device, looked up once
// per device (with that device current) under one lock.
struct ResidentPtrs {
  int* status;
  float* dsum;
};
static const ResidentPtrs* resident_ptrs() {
  static std::mutex mu;
  static ResidentPtrs table[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  ResidentPtrs& r = table[dev];
  if (!r.status) {
    void* ps = nullptr;
    void* pd = nullptr;
    if (cudaGetSymbolAddress(&ps, g_kernel_status) != cudaSuccess || !ps ||
        cudaGetSymbolAddress(&pd, g_noalloc_dsum) != cudaSuccess || !pd) {
      cudaGetLastError();
      return nullptr;
    }
    r.dsum = (float*)pd;
    r.status = (int*)ps;
  }
  return &r;
}

static int* status_word() {
  const ResidentPtrs* r = resident_ptrs();
  return r ? r->status : nullptr;
}

static int sm_count() {
  prime_kernel_attributes();
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

template <typename T>
static int attn_fwd(const AttnParams& ap, int engine, cudaStream_t st) {
  if (prime_kernel_attributes() != 0) return TTT_ERR_CUDA;
  const int64_t rows = (int64_t)ap.B * ap.n;
  if (sizeof(T) == 2 && engine == TTT_ENGINE_AUTO && attn_tc_ok(ap)) {
    int* err = status_word();
    if (!err) return TTT_ERR_CUDA;
    bool ok = false;
    const cudaError_t e = attn_fwd_tc_launch(ap, st, err, &ok);
    if (e != cudaSuccess) return TTT_ERR_CUDA;
    if (ok) return TTT_OK;
  }
  if (sizeof(T) == 2 && engine != TTT_ENGINE_SIMT && attn_mma_ok(ap)) {
    const cudaError_t e = ap.hd == 128 ? attn_fwd_mma_launch<128>(ap, st) : attn_fwd_mma_launch<64>(ap, st);
    return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
  }
  attn_fwd_simt_kernel<T><<<(unsigned)((rows * ap.H + 3) / 4), 128, 0, st>>>(ap);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

template <typename T>
static int attn_bwd(const AttnParams& ap, int engine, cudaStream_t st) {
  if (prime_kernel_attributes() != 0) return TTT_ERR_CUDA;
  const int64_t rows = (int64_t)ap.B * ap.n;
  bool dq_done = false, dkv_done = false;
  if (sizeof(T) == 2 && engine == TTT_ENGINE_AUTO && attn_dq_tc_ok(ap)) {
    int* err = status_word();
    if (!err) return TTT_ERR_CUDA;
    AttnParams aq = ap;
    aq.dsum_in_dq = 1;  // the tcgen05 dQ kernel forms D = rowsum(dO * O) and stores it for dK/dV
    cudaError_t e = attn_bwd_dq_tc_launch(aq, st, err, &dq_done);
    if (e == cudaSuccess && dq_done && attn_dkv_tc_ok(ap)) e = attn_bwd_dkv_tc_launch(ap, st, err, &dkv_done);
    if (e != cudaSuccess) return TTT_ERR_CUDA;
  }
  if (!dq_done) attn_bwd_prep_kernel<T><<<(unsigned)((rows * ap.H + 7) / 8), 256, 0, st>>>(ap);
  if (dq_done && dkv_done) return TTT_OK;
  if (sizeof(T) == 2 && engine != TTT_ENGINE_SIMT && attn_mma_ok(ap)) {
    const cudaError_t e = ap.hd == 128 ? attn_bwd_mma_launch<128>(ap, st, !dq_done, !dkv_done)
                                       : attn_bwd_mma_launch<64>(ap, st, !dq_done, !dkv_done);
    return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
  }
  if (!dq_done) attn_bwd_dq_simt_kernel<T><<<(unsigned)((rows * ap.H + 3) / 4), 128, 0, st>>>(ap);
  if (!dkv_done) attn_bwd_dkv_simt_kernel<T><<<(unsigned)((rows * ap.H + 3) / 4), 128, 0, st>>>(ap);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

static AttnParams attn_params(int B, int H, int hd, int n, int64_t q0, int window, const void* qkv, size_t esz,
                              const void* rk, const void* rv, int C, void* out, float* lse) {
  AttnParams ap;
  memset(&ap, 0, sizeof(ap));
  const int d = H * hd;
  ap.B = B; ap.H = H; ap.hd = hd; ap.n = n; ap.d = d; ap.q0 = q0; ap.window = window;
  ap.Q = qkv; ap.ldq = 3 * d;
  ap.K = (const char*)qkv + (size_t)d * esz;
  ap.V = (const char*)qkv + (size_t)2 * d * esz;
  ap.ldkv = 3 * d;
  ap.Kc = rk; ap.Vc = rv; ap.C = C;
  ap.O = out; ap.ldo = d; ap.lse = lse;
  ap.scale = 1.0f / sqrtf((float)hd);
  return ap;
}

}  // namespace ttt

using namespace ttt;

extern "C" {

// Validates one product's arguments and fills its parameter block; false = invalid.
static bool gemm_params_from(const ttt_gemm_desc& g, GemmParams* p) {
  if (g.M < 0 || g.N < 0 || g.K < 0 || g.batch < 1 || !g.A || !g.B || !g.D || g.epi < 0 || g.epi > 4) return false;
  if ((g.epi == EPI_RESID || g.epi == EPI_DGELU) && !g.X) return false;
  if ((g.epi == EPI_RESID || g.epi == EPI_SGD) && !g.d_f32) return false;
  memset(p, 0, sizeof(*p));
  p->M = g.M; p->N = g.N; p->K = g.K; p->batch = g.batch;
  p->A = g.A; p->lda = g.lda; p->sA = g.sA; p->a_mn = g.a_mn;
  p->B = g.B; p->ldb = g.ldb; p->sB = g.sB; p->b_mn = g.b_mn;
  p->B2 = g.B2; p->sB2 = g.sB2;
  p->D = g.D; p->ldd = g.ldd; p->sD = g.sD; p->d_f32 = g.d_f32;
  p->X = g.X; p->ldx = g.ldx; p->sX = g.sX;
  p->Y = g.Y; p->ldy = g.ldy; p->sY = g.sY;
  p->alpha = g.alpha; p->epi = g.epi;
  return true;
}

int ttt_k_gemm(int32_t elem_dtype, int32_t M, int32_t N, int32_t K, int32_t batch, const void* A, int64_t lda,
               int64_t sA, int32_t a_mn, const void* B, int64_t ldb, int64_t sB, int32_t b_mn, const void* B2,
               int64_t sB2, void* D, int64_t ldd,
               int64_t sD, int32_t d_f32, const void* X, int64_t ldx, int64_t sX, void* Y, int64_t ldy, int64_t sY,
               float alpha, int32_t epi, int32_t engine, void* stream) {
  const ttt_gemm_desc g = {M, N, K, batch, A, lda, sA, a_mn, B, ldb, sB, b_mn, B2, sB2, D, ldd, sD, d_f32,
                           X, ldx, sX, Y, ldy, sY, alpha, epi};
  GemmParams p;
  if (!gemm_params_from(g, &p)) return TTT_ERR_INVALID_ARG;
  int* err = status_word();
  if (!err) return TTT_ERR_CUDA;
  const int e = gemm_launch(p, elem_dtype == TTT_BF16 ? 1 : 0, (cudaStream_t)stream, err, sm_count(),
                            engine == TTT_ENGINE_SIMT ? GEMM_SIMT : engine == TTT_ENGINE_TC1 ? GEMM_TC1 : GEMM_AUTO);
  return e == 0 ? TTT_OK : TTT_ERR_CUDA;
}

int ttt_k_gemm_pair(int32_t elem_dtype, const ttt_gemm_desc* first, const ttt_gemm_desc* second, void* stream) {
  if (!first || !second) return TTT_ERR_INVALID_ARG;
  GemmParams a, b;
  if (!gemm_params_from(*first, &a) || !gemm_params_from(*second, &b)) return TTT_ERR_INVALID_ARG;
  int* err = status_word();
  if (!err) return TTT_ERR_CUDA;
  if (prime_kernel_attributes() != 0) return TTT_ERR_CUDA;
  const int e = gemm_launch_pair(a, b, elem_dtype == TTT_BF16 ? 1 : 0, (cudaStream_t)stream, err, sm_count());
  return e == 0 ? TTT_OK : TTT_ERR_CUDA;
}

int ttt_k_lm_head_ce(int32_t M, int32_t V, int32_t d, const void* r, const void* E, const int32_t* targets,
                     void* z, float* loss, float* scratch, float grad_scale, void* stream) {
  if (M < 1 || V < 64 || d < 1 || V % 64 || !r || !E || !targets || !z || !loss || !scratch)
    return TTT_ERR_INVALID_ARG;
  int* err = status_word();
  if (!err) return TTT_ERR_CUDA;
  if (prime_kernel_attributes() != 0) return TTT_ERR_CUDA;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = M; p.N = V; p.K = d; p.batch = 1;
  p.A = r; p.lda = d; p.B = E; p.ldb = d;
  p.D = z; p.ldd = V; p.alpha = 1.f; p.epi = EPI_CE;
  p.ce_tgt = targets;
  p.ce_part = (float2*)scratch;
  p.ce_zt = scratch + (int64_t)2 * M * (V / 64);
  if (!gemm_uses_tc(p, 1)) return TTT_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  if (gemm_launch(p, 1, st, err, sm_count(), GEMM_AUTO) != 0) return TTT_ERR_CUDA;
  ce_finish_kernel<bf16><<<M, 256, 0, st>>>((bf16*)z, V, (const float2*)p.ce_part, p.ce_zt, targets, M, loss, M, 0,
                                           grad_scale, err);
  return cudaGetLastError() == cudaSuccess ? TTT_OK : TTT_ERR_CUDA;
}

int ttt_k_attention_fwd(int32_t elem_dtype, int32_t B, int32_t H, int32_t hd, int32_t n, int64_t q0,
                        int32_t window, const void* qkv, const void* ring_k, const void* ring_v, int32_t C, void* out,
                        float* lse, int32_t engine, void* stream) {
  if (B < 1 || H < 1 || hd < 2 || hd > 128 || n < 1 || window < 1 || !qkv || !out) return TTT_ERR_INVALID_ARG;
  if (q0 > 0 && (!ring_k || !ring_v || C < window)) return TTT_ERR_INVALID_ARG;
  const size_t esz = elem_dtype == TTT_BF16 ? 2 : 4;
  AttnParams ap = attn_params(B, H, hd, n, q0, window, qkv, esz, ring_k, ring_v, C, out, lse);
  if (elem_dtype == TTT_BF16) return attn_fwd<bf16>(ap, engine, (cudaStream_t)stream);
  return attn_fwd<float>(ap, engine, (cudaStream_t)stream);
}

int ttt_k_attention_bwd(int32_t elem_dtype, int32_t B, int32_t H, int32_t hd, int32_t n, int64_t q0,
                        int32_t window, const void* qkv, const void* ring_k, const void* ring_v, int32_t C,
                        const void* out, const float* lse, const void* dout, void* dqkv, float* dsum,
                        int32_t engine, void* stream) {
  if (B < 1 || H < 1 || hd < 2 || hd > 128 || n < 1 || window < 1 || !qkv || !out || !lse || !dout || !dqkv || !dsum)
    return TTT_ERR_INVALID_ARG;
  if (q0 > 0 && (!ring_k || !ring_v || C < window)) return TTT_ERR_INVALID_ARG;
  const size_t esz = elem_dtype == TTT_BF16 ? 2 : 4;
  AttnParams ap = attn_params(B, H, hd, n, q0, window, qkv, esz, ring_k, ring_v, C, const_cast<void*>(out),
                              const_cast<float*>(lse));
  const int d = H * hd;
  ap.dO = dout; ap.lddo = d; ap.Dsum = dsum;
  ap.dQ = dqkv;
  ap.dK = (char*)dqkv + (size_t)d * esz;
  ap.dV = (char*)dqkv + (size_t)2 * d * esz;
  ap.lddq = 3 * d;
  if (elem_dtype == TTT_BF16) return attn_bwd<bf16>(ap, engine, (cudaStream_t)stream);
  return attn_bwd<float>(ap, engine, (cudaStream_t)stream);
}

int ttt_k_attention_bwd_noalloc(int32_t elem_dtype, int32_t B, int32_t H, int32_t hd, int32_t n, int64_t q0,
                                int32_t window, const void* qkv, const void* ring_k, const void* ring_v, int32_t C,
                                const void* out, const float* lse, const void* dout, void* dqkv, int32_t engine,
                                void* stream) {
  if (B < 1 || H < 1 || hd < 2 || hd > 128 || n < 1 || window < 1 || !qkv || !out || !lse || !dout || !dqkv)
    return TTT_ERR_INVALID_ARG;
  if (q0 > 0 && (!ring_k || !ring_v || C < window)) return TTT_ERR_INVALID_ARG;
  if ((int64_t)B * H * n > kNoAllocDsumFloats) return TTT_ERR_INVALID_ARG;  // B*H*n above the fixed scratch
  const ResidentPtrs* res = resident_ptrs();
  if (!res) return TTT_ERR_CUDA;
  float* dsum = res->dsum;
  // Nothing needs clearing: the first kernel of the call writes every D it later reads.
  const size_t esz = elem_dtype == TTT_BF16 ? 2 : 4;
  AttnParams ap = attn_params(B, H, hd, n, q0, window, qkv, esz, ring_k, ring_v, C, const_cast<void*>(out),
                              const_cast<float*>(lse));
  const int d = H * hd;
  ap.dO = dout; ap.lddo = d; ap.Dsum = dsum;
  ap.dQ = dqkv;
  ap.dK = (char*)dqkv + (size_t)d * esz;
  ap.dV = (char*)dqkv + (size_t)2 * d * esz;
  ap.lddq = 3 * d;
  if (elem_dtype == TTT_BF16) return attn_bwd<bf16>(ap, engine, (cudaStream_t)stream);
  return attn_bwd<float>(ap, engine, (cudaStream_t)stream);
}

int ttt_k_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) { cudaGetLastError(); return TTT_ERR_CUDA; }
  int* err = status_word();
  if (!err) return TTT_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpy(&flag, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TTT_ERR_CUDA;
  if (flag) {
    cudaMemset(err, 0, sizeof(int));
    return flag == DEV_BAD_TOKEN ? TTT_ERR_INVALID_ARG : TTT_ERR_TIMEOUT;
  }
  return TTT_OK;
}

int ttt_k_test_set_status(int32_t code) {
  if (cudaDeviceSynchronize() != cudaSuccess) { cudaGetLastError(); return TTT_ERR_CUDA; }
  int* err = status_word();
  if (!err) return TTT_ERR_CUDA;
  if (cudaMemcpy(err, &code, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return TTT_ERR_CUDA;
  return TTT_OK;
}

}  // extern "C"
