/*
 * ttt_kernels.h — per-kernel C ABI of the TTT-E2E library (sm_100a).
 *
 * The same kernels that ttt_prefill/ttt_decode run, exposed one at a time so
 * that each can be checked against the CPU reference and timed against its
 * roofline. All pointers are DEVICE pointers; `stream` is a cudaStream_t (NULL
 * = legacy default stream). Calls are asynchronous: they only enqueue work.
 * ttt_k_status() synchronises the stream and reports launch or device-side
 * errors (bounded waits that expired). Return codes are the TTT_* codes of ttt.h.
 * elem_dtype: TTT_FP32 (float operands) or TTT_BF16 (bf16 operands).
 */
#ifndef TTT_KERNELS_H
#define TTT_KERNELS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogues of ttt_k_gemm (acc = alpha * sum_k A[m][k] B[n][k], fp32):
 *   TTT_EPI_STORE: D = acc (D float if d_f32, else elem type)
 *   TTT_EPI_RESID: D(float) = acc + X(float)             (X may equal D: residual add in place)
 *   TTT_EPI_GELU:  Y = acc (if Y), D = gelu(acc)          (exact erf GELU; elem type)
 *   TTT_EPI_DGELU: D = acc * gelu'(X)                     (X, D elem type)
 *   TTT_EPI_SGD:   D(float) += acc; Y = D (if Y, elem type)  (alpha = -eta: fused SGD step,
 *                  summary of the TTT-E2E paper, mini-batch gradient-descent equation) */
enum { TTT_EPI_STORE = 0, TTT_EPI_RESID = 1, TTT_EPI_GELU = 2, TTT_EPI_DGELU = 3, TTT_EPI_SGD = 4 };

/* Engines: 0 = automatic: GEMMs on tcgen05 tensor cores for bf16 shapes with N % 128 == 0 and
 * K % 64 == 0 (pairs of CTAs on two SMs sharing 256-row tiles for large products; for thin
 * products whose 128 x 256 tiles fill at most half the SMs, pairs of CTAs splitting K of one
 * 128 x 256 tile, summed in a fixed order; one CTA per 128-row tile otherwise); attention forward on tcgen05 for bf16 with head dim 64 or 128,
 * q0 % 128 == 0 and C % 128 == 0; attention on warp-level tensor cores (mma.sync m16n8k16)
 * for bf16 with head dim 64 or 128 and q0 % 64 == 0 (and C % 64 == 0); otherwise, and for
 * fp32, SIMT FFMA kernels. 1 = SIMT only. 2 = attention on the mma.sync kernels. 3 = GEMMs
 * on single-CTA tcgen05 tiles only (tests compare engines). */
enum { TTT_ENGINE_AUTO = 0, TTT_ENGINE_SIMT = 1, TTT_ENGINE_MMA = 2, TTT_ENGINE_TC1 = 3 };

/* Batched GEMM D[z][m][n] = epilogue(alpha * sum_k A[z](m,k) * (B[z](n,k) + B2[z](n,k))).
 * A(m,k) = a_mn ? A[k*lda + m] : A[m*lda + k]   (batch stride sA elements)
 * B(n,k) = b_mn ? B[k*ldb + n] : B[n*ldb + k]   (batch stride sB; 0 = one matrix shared by all z)
 * B2: optional (NULL), same layout and ldb as B, batch stride sB2. The adaptive MLPs use
 *     B = W_init (shared) and B2 = dW (per sequence): the fast weights W_init + dW without
 *     rounding a small dW against W_init into one bf16 value.
 * D, X, Y row-major with leading dims ldd, ldx, ldy and batch strides sD, sX, sY.
 * Forward products use (a_mn, b_mn) = (0, 0), data gradients (0, 1), weight gradients (1, 1). */
int ttt_k_gemm(int32_t elem_dtype, int32_t M, int32_t N, int32_t K, int32_t batch, const void* A, int64_t lda,
               int64_t sA, int32_t a_mn, const void* B, int64_t ldb, int64_t sB, int32_t b_mn, const void* B2,
               int64_t sB2, void* D, int64_t ldd,
               int64_t sD, int32_t d_f32, const void* X, int64_t ldx, int64_t sX, void* Y, int64_t ldy, int64_t sY,
               float alpha, int32_t epi, int32_t engine, void* stream);

/* One product of ttt_k_gemm_pair: the arguments of ttt_k_gemm with the same meaning. */
typedef struct {
  int32_t M, N, K, batch;
  const void* A; int64_t lda, sA; int32_t a_mn;
  const void* B; int64_t ldb, sB; int32_t b_mn;
  const void* B2; int64_t sB2;
  void* D; int64_t ldd, sD; int32_t d_f32;
  const void* X; int64_t ldx, sX;
  void* Y; int64_t ldy, sY;
  float alpha; int32_t epi;
} ttt_gemm_desc;

/* Two independent products (no operand of one is an output of the other; their outputs
 * do not overlap), enqueued on one stream. Where both are bf16 tcgen05 products with the
 * same a_mn/b_mn and N % 256 == 0 they share one persistent single-CTA launch of 128 x 256
 * tiles, the second product's tiles following the first's, so that one product's
 * epilogues overlap the other's mainloop (the two weight-gradient SGD steps of an adaptive
 * MLP block); otherwise each runs as ttt_k_gemm(engine 0) would. Each result equals the
 * single-CTA engine's (engine 3) up to the tile width it picks. The descriptors are read
 * during the call only (the caller keeps ownership); device pointers as in ttt_k_gemm.
 * TTT_ERR_INVALID_ARG for a descriptor ttt_k_gemm would reject, TTT_ERR_CUDA on a launch
 * error. */
int ttt_k_gemm_pair(int32_t elem_dtype, const ttt_gemm_desc* first, const ttt_gemm_desc* second, void* stream);

/* LM head and softmax cross-entropy, chunked over the vocabulary (summary, loss l_t;
 * technical review §3, eq. (3)), bf16 on tcgen05. r [M][d] (final-norm output rows),
 * E [V][d] (tied embedding), targets [M] int32 in [0, V).
 * One GEMM z = r E^T whose epilogue keeps, per row and 64-column vocabulary chunk,
 * the fp32 maximum and sum of exponentials and the target's fp32 logit; then one pass
 * per row merges the chunks into the log-sum-exp, writes loss[m] = lse - z[m][t],
 * and, when grad_scale != 0, overwrites z with dz = (softmax(z) - onehot(t)) * grad_scale.
 * z [M][V] bf16 receives the logits (grad_scale == 0) or dz. scratch: float buffer of
 * 2*M*(V/64) + M elements (device). V % 128 == 0, d % 64 == 0, else
 * TTT_ERR_UNSUPPORTED. An id outside [0, V) gives that row loss 0 and sets the device
 * status, which the next ttt_k_status() reports as TTT_ERR_INVALID_ARG. */
int ttt_k_lm_head_ce(int32_t M, int32_t V, int32_t d, const void* r, const void* E, const int32_t* targets,
                     void* z, float* loss, float* scratch, float grad_scale, void* stream);

/* Causal sliding-window attention forward (technical review §5: window k >= b,
 * causal inside the chunk). Rows [B][n] of qkv ([B*n][3*H*hd]: q | k | v per row,
 * q and k already rotated) are positions q0..q0+n-1; query P attends to keys
 * [max(0, P-window+1), P], taking positions < q0 from the rings ring_k/ring_v
 * ([B][C][H*hd], slot = pos % C) and the others from qkv.
 * out [B*n][H*hd]; lse [B][H][n] (may be NULL). */
int ttt_k_attention_fwd(int32_t elem_dtype, int32_t B, int32_t H, int32_t hd, int32_t n, int64_t q0,
                        int32_t window, const void* qkv, const void* ring_k, const void* ring_v, int32_t C, void* out,
                        float* lse, int32_t engine, void* stream);

/* Backward of ttt_k_attention_fwd for dout [B*n][H*hd]: dq for every row over its
 * whole window, dk and dv only for the current rows (cached keys are constants).
 * dqkv [B*n][3*H*hd] receives dq | dk | dv; dsum [B][H][n] is scratch. */
int ttt_k_attention_bwd(int32_t elem_dtype, int32_t B, int32_t H, int32_t hd, int32_t n, int64_t q0,
                        int32_t window, const void* qkv, const void* ring_k, const void* ring_v, int32_t C,
                        const void* out, const float* lse, const void* dout, void* dqkv, float* dsum,
                        int32_t engine, void* stream);

/* Same as ttt_k_attention_bwd without the dsum argument, for callers that may not
 * allocate device memory: for example a host application that reserved the GPU's
 * memory for its own pool and hands this code only pointers, or a latency-bound
 * thread that must not call cudaMalloc, which can block and synchronise the device.
 * This entry point allocates nothing. Its scratch (one float per sequence, head and
 * row) is a fixed 4 MiB array inside the library that every GPU loading the library
 * keeps until exit. Limit: B*H*n <= 1048576, else TTT_ERR_INVALID_ARG.
 * The first per-kernel call on each device (this entry point or any other of this
 * header) looks up that array's device address (cudaGetSymbolAddress) with the
 * device current; make that first call before any stream capture. All calls share the one array: calls whose work overlaps on
 * the GPU (other streams, other host threads) race on it and must be serialised by
 * the caller. Nothing in it needs clearing: each call writes every element it reads.
 * The pages have no counterpart of this entry point: it is an interface variant. */
int ttt_k_attention_bwd_noalloc(int32_t elem_dtype, int32_t B, int32_t H, int32_t hd, int32_t n, int64_t q0,
                                int32_t window, const void* qkv, const void* ring_k, const void* ring_v, int32_t C,
                                const void* out, const float* lse, const void* dout, void* dqkv, int32_t engine,
                                void* stream);

/* Synchronise `stream` and return TTT_OK, TTT_ERR_CUDA, TTT_ERR_TIMEOUT (a
 * bounded device wait expired) or TTT_ERR_INVALID_ARG (a token id outside the
 * vocabulary reached ttt_k_lm_head_ce). Clears the device status word. The word is
 * one per device, shared by all per-kernel calls on it. */
int ttt_k_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TTT_KERNELS_H */
