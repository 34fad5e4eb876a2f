// Fused LM-head cross-entropy, second half (the first half is the EPI_CE epilogue of
// the tcgen05 GEMM in ttt_gemm.cuh).
#pragma once

#include "ttt_common.cuh"

namespace ttt {

// (m, s) <- merge of two (max, sum exp(x - max)) pairs.
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  const float M = fmaxf(m, m2);
  if (M == -INFINITY) return;
  s = s * expf(m - M) + s2 * expf(m2 - M);
  m = M;
}

// Second half of the fused LM-head cross-entropy: the LM-head GEMM (EPI_CE) left,
// per row, the fp32 (max, sum-exp) of every 64-column vocabulary chunk and the
// target's fp32 logit. One block per row merges the chunks into the log-sum-exp,
// writes the loss lse - z[target], and (grad_scale != 0) overwrites the bf16
// logits with dz = (softmax - onehot) * grad_scale in one read and one write.
template <typename T>
__global__ void __launch_bounds__(256) ce_finish_kernel(T* __restrict__ z, int V, const float2* __restrict__ part,
                                                        const float* __restrict__ zt,
                                                        const int32_t* __restrict__ targets, int n,
                                                        float* loss_out, int64_t loss_ld, int64_t loss_off,
                                                        float grad_scale, int* err) {
  constexpr int VEC = 16 / sizeof(T);
  const int row = blockIdx.x;
  const int nparts = V / 64;
  __shared__ float sm_m[8], sm_s[8];
  __shared__ float bc[1];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  pdl_wait();
  float m = -INFINITY, sum = 0.f;
  for (int i = tid; i < nparts; i += 256) {
    const float2 ms = part[(int64_t)row * nparts + i];
    lse_merge(m, sum, ms.x, ms.y);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, sum, o);
    lse_merge(m, sum, m2, s2);
  }
  if (lane == 0) { sm_m[w] = m; sm_s[w] = sum; }
  __syncthreads();
  if (tid == 0) {
    float M = sm_m[0], S = sm_s[0];
    for (int i = 1; i < 8; ++i) lse_merge(M, S, sm_m[i], sm_s[i]);
    bc[0] = M + logf(S);
  }
  __syncthreads();
  pdl_trigger();
  const float lse = bc[0];
  int t = targets[row];
  const bool bad = t < 0 || t >= V;  // ids are validated here too: the last target of a call is never embedded
  if (bad) {
    if (tid == 0) set_error(err, DEV_BAD_TOKEN);
    t = 0;
  }
  if (tid == 0 && loss_out) {
    const int seq = row / n, i = row % n;
    loss_out[(int64_t)seq * loss_ld + loss_off + i] = bad ? 0.f : lse - zt[row];
  }
  if (grad_scale != 0.f) {
    T* zr = z + (int64_t)row * V;
    for (int c = tid * VEC; c < V; c += 256 * VEC) {
      uint4 u = *reinterpret_cast<const uint4*>(zr + c);
      T* e = reinterpret_cast<T*>(&u);
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        const float pr = __expf(to_f32(e[i]) - lse);
        e[i] = from_f32<T>((pr - (c + i == t ? 1.f : 0.f)) * grad_scale);
      }
      *reinterpret_cast<uint4*>(zr + c) = u;
    }
  }
}

}  // namespace ttt
