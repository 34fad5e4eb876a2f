// Row-wise and elementwise kernels of the TTT-E2E path (HBM-bound work).
//
// Rows of d elements, one warp per row, fp32 statistics. Residual streams are
// fp32; normalised activations (GEMM operands) use the element type T.
#pragma once

#include "ttt_ce.cuh"
#include "ttt_common.cuh"

namespace ttt {

// ---------------------------------------------------------------- embedding (frozen E)
// x[row][:] = E[token][:] for rows of [B][n] positions, token = tok[b*tok_ld + tok_off + i].
template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ tok, int64_t tok_ld, int tok_off, int n, int rows,
                             const T* __restrict__ E, int V, int d, float* __restrict__ x, int* err) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int b = row / n, i = row % n;
  int t = tok[(int64_t)b * tok_ld + tok_off + i];
  if (t < 0 || t >= V) {
    if (lane == 0) set_error(err, DEV_BAD_TOKEN);
    t = 0;
  }
  const T* e = E + (int64_t)t * d;
  float* o = x + (int64_t)row * d;
  for (int c = lane; c < d; c += 32) o[c] = to_f32(e[c]);
}

// ---------------------------------------------------------------- 8-element vectors
// Eight consecutive elements <-> fp32 registers: one 16-byte access for bf16,
// two for fp32. The address must be 16-byte aligned.
__device__ __forceinline__ void ld8(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void ld8(const bf16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x; v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void st8(float* p, const float (&v)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void st8(bf16* p, const float (&v)[8]) {
  uint4 u;
  u.x = pack_bf16x2(v[0], v[1]); u.y = pack_bf16x2(v[2], v[3]);
  u.z = pack_bf16x2(v[4], v[5]); u.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

// Sum over the TPR threads that share a row (TPR a power of two <= 256; the
// block holds 256 / TPR rows). Every thread of the block must call it.
template <int TPR> __device__ __forceinline__ float row_sum(float v, float* red) {
#pragma unroll
  for (int o = (TPR < 32 ? TPR : 32) >> 1; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if constexpr (TPR > 32) {
    constexpr int W = TPR / 32;
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = v;
    __syncthreads();
    const int w0 = w & ~(W - 1);
    v = 0.f;
#pragma unroll
    for (int i = 0; i < W; ++i) v += red[w0 + i];
  }
  return v;
}

// Threads per row of d elements: each thread owns 8-element chunks
// c = (k * TPR + t) * 8, k = 0, 1, ...; the first RC_CACHE chunks stay in
// registers between the two passes of a row kernel.
constexpr int RC_CACHE = 2;
inline int row_threads(int d) {  // two chunks per thread where the row is long enough
  const int ch = d / 16;
  return ch >= 256 ? 256 : ch >= 128 ? 128 : ch >= 64 ? 64 : 32;
}

// ---------------------------------------------------------------- RMSNorm
// y = g * x / sqrt(mean(x^2) + eps); rstd kept for the backward.
// Blocks of 256 threads, TPR threads per row (d % 8 == 0, ldx % 4 == 0, ldy % 8 == 0).
template <typename T, int TPR>
__global__ void __launch_bounds__(256, 4) rmsnorm_fwd_kernel(const float* __restrict__ x, int64_t ldx,
                                                          const float* __restrict__ g, float eps, int rows, int d,
                                                          T* __restrict__ y, int64_t ldy,
                                                          float* __restrict__ rstd_out) {
  __shared__ float red[8];
  pdl_wait();
  pdl_trigger();
  const int t = threadIdx.x % TPR;
  const int row = blockIdx.x * (256 / TPR) + threadIdx.x / TPR;
  const bool live = row < rows;
  const int nch = (d / 8 + TPR - 1) / TPR;
  const float* xr = x + (int64_t)(live ? row : 0) * ldx;
  float cache[RC_CACHE][8];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < RC_CACHE; ++k) {
    const int c = (k * TPR + t) * 8;
    if (k < nch && live && c < d) {
      ld8(xr + c, cache[k]);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss += cache[k][i] * cache[k][i];
    }
  }
  for (int k = RC_CACHE; k < nch; ++k) {
    const int c = (k * TPR + t) * 8;
    if (live && c < d) {
      float v[8];
      ld8(xr + c, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss += v[i] * v[i];
    }
  }
  ss = row_sum<TPR>(ss, red);
  if (!live) return;
  const float rs = rsqrtf(ss / d + eps);
  if (t == 0 && rstd_out) rstd_out[row] = rs;
  T* yr = y + (int64_t)row * ldy;
  for (int k = 0; k < nch; ++k) {
    const int c = (k * TPR + t) * 8;
    if (c >= d) continue;
    float v[8], gg[8];
    if (k < RC_CACHE) {
#pragma unroll
      for (int kk = 0; kk < RC_CACHE; ++kk)
        if (kk == k) {
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = cache[kk][i];
        }
    } else {
      ld8(xr + c, v);
    }
    ld8(g + c, gg);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = v[i] * rs * gg[i];
    st8(yr + c, v);
  }
}

// dx = dres + rstd*(g*dy) - x*rstd^3*sum(g*dy*x)/d ; writes fp32 and (optionally) a T copy.
// dres may alias dx (each element is read before it is written, by the same thread).
template <typename T, int TPR>
__global__ void __launch_bounds__(256, 3) rmsnorm_bwd_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                                          const float* __restrict__ rstd,
                                                          const float* __restrict__ dy, const float* dres, int rows,
                                                          int d, float* dx, T* __restrict__ dx_t) {
  __shared__ float red[8];
  pdl_wait();
  pdl_trigger();
  const int t = threadIdx.x % TPR;
  const int row = blockIdx.x * (256 / TPR) + threadIdx.x / TPR;
  const bool live = row < rows;
  const int nch = (d / 8 + TPR - 1) / TPR;
  const int64_t o = (int64_t)(live ? row : 0) * d;
  float cx[RC_CACHE][8], cgd[RC_CACHE][8];  // x and g * dy of the cached chunks
  float dot = 0.f;
#pragma unroll
  for (int k = 0; k < RC_CACHE; ++k) {
    const int c = (k * TPR + t) * 8;
    if (k < nch && live && c < d) {
      float gg[8];
      ld8(x + o + c, cx[k]);
      ld8(dy + o + c, cgd[k]);
      ld8(g + c, gg);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cgd[k][i] *= gg[i];
        dot += cgd[k][i] * cx[k][i];
      }
    }
  }
  for (int k = RC_CACHE; k < nch; ++k) {
    const int c = (k * TPR + t) * 8;
    if (live && c < d) {
      float xv[8], dv[8], gg[8];
      ld8(x + o + c, xv);
      ld8(dy + o + c, dv);
      ld8(g + c, gg);
#pragma unroll
      for (int i = 0; i < 8; ++i) dot += gg[i] * dv[i] * xv[i];
    }
  }
  dot = row_sum<TPR>(dot, red);
  if (!live) return;
  const float rs = rstd[row];
  const float coef = rs * rs * rs * dot / d;
  for (int k = 0; k < nch; ++k) {
    const int c = (k * TPR + t) * 8;
    if (c >= d) continue;
    float xv[8], gd[8];
    if (k < RC_CACHE) {
#pragma unroll
      for (int kk = 0; kk < RC_CACHE; ++kk)
        if (kk == k) {
#pragma unroll
          for (int i = 0; i < 8; ++i) { xv[i] = cx[kk][i]; gd[i] = cgd[kk][i]; }
        }
    } else {
      float dv[8], gg[8];
      ld8(x + o + c, xv);
      ld8(dy + o + c, dv);
      ld8(g + c, gg);
#pragma unroll
      for (int i = 0; i < 8; ++i) gd[i] = gg[i] * dv[i];
    }
    float r[8];
    if (dres) ld8(dres + o + c, r);
    else {
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] += rs * gd[i] - xv[i] * coef;
    st8(dx + o + c, r);
    if (dx_t) st8(dx_t + o + c, r);
  }
}

// ---------------------------------------------------------------- RoPE
// Rotate pairs (i, i+hd/2) of every head in columns [0, ncols) of rows laid out
// [B][n] at absolute positions pos0 + i. Angles pos * base^(-2i/hd) come from
// two tables built in double precision on the host:
//   cos/sin(p*t) from (p = 1024*hi + lo) by the angle-addition identities.
// inverse != 0 applies the transpose rotation (backward of the forward map).
// The rotation depends on (position, pair index) only, so one thread takes 8
// consecutive pairs of RP_HEADS heads of one row and forms their (cos, sin) once
// (hd % 16 == 0, ncols % hd == 0, ld % 8 == 0).
constexpr int RP_HEADS = 4;
template <typename T>
__global__ void __launch_bounds__(256) rope_kernel(T* __restrict__ qk, int64_t ld, int ncols, int rows, int n,
                                                   int64_t pos0, int hd, const float2* __restrict__ lo_tab,
                                                   const float2* __restrict__ hi_tab, int inverse,
                                                   const int64_t* pos_dev = nullptr, T* __restrict__ ring_k = nullptr,
                                                   T* __restrict__ ring_v = nullptr, int C = 0) {
  pdl_wait();
  pdl_trigger();
  if (pos_dev) pos0 = *pos_dev;  // position held on the device (graph-captured decode step)
  const int half = hd >> 1;
  const int ng = half >> 3;                                  // 8-pair groups per head
  const int nheads = ncols / hd;
  const int per_row = ng * ((nheads + RP_HEADS - 1) / RP_HEADS);
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * per_row) return;
  const int row = idx / per_row;
  const int rem = idx - row * per_row;
  const int hc = rem / ng;
  const int i = (rem - hc * ng) * 8;
  const int64_t pos = pos0 + (row % n);
  const float4* a4 = reinterpret_cast<const float4*>(lo_tab + (pos & 1023) * half + i);  // (cos, sin) of lo * theta
  const float4* b4 = reinterpret_cast<const float4*>(hi_tab + (pos >> 10) * half + i);   // of 1024*hi * theta
  float cs[8], sn[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 a = a4[j], b = b4[j];  // two pairs: (a.x, a.y) and (a.z, a.w)
    cs[2 * j] = a.x * b.x - a.y * b.y;
    sn[2 * j] = a.y * b.x + a.x * b.y;
    cs[2 * j + 1] = a.z * b.z - a.w * b.w;
    sn[2 * j + 1] = a.w * b.z + a.z * b.w;
  }
  if (inverse) {
#pragma unroll
    for (int q = 0; q < 8; ++q) sn[q] = -sn[q];
  }
  T* rowp = qk + (int64_t)row * ld + i;
#pragma unroll
  for (int t = 0; t < RP_HEADS; ++t) {
    const int head = hc * RP_HEADS + t;
    if (head < nheads) {
      T* base = rowp + head * hd;
      float x1[8], x2[8];
      ld8(base, x1);
      ld8(base + half, x2);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float u = x1[q], v = x2[q];
        x1[q] = u * cs[q] - v * sn[q];
        x2[q] = v * cs[q] + u * sn[q];
      }
      st8(base, x1);
      st8(base + half, x2);
      // window ring: a key head's rotated pairs and the same elements of its value head
      // go to the row's slot (position mod C) of sequence row / n
      const int dq = ncols >> 1;  // columns [0, dq) are q, [dq, 2 dq) k, [2 dq, 3 dq) v
      if (ring_k && head * hd >= dq) {
        const int64_t off = ((int64_t)(row / n) * C + pos % C) * dq + (head * hd - dq) + i;
        st8(ring_k + off, x1);
        st8(ring_k + off + half, x2);
        float v1[8], v2[8];
        ld8(base + dq, v1);
        ld8(base + dq + half, v2);
        st8(ring_v + off, v1);
        st8(ring_v + off + half, v2);
      }
    }
  }
}

// Grid of rope_kernel for rows x ncols (head dim hd). With ring_k/ring_v the kernel
// also appends each row's rotated key and its value (columns [ncols/2, 3 ncols/2) of
// the q|k|v row) to the window ring [B][C][ncols/2] at slot (position mod C).
inline int64_t rope_threads(int rows, int ncols, int hd) {
  const int nheads = ncols / hd;
  return (int64_t)rows * (hd >> 4) * ((nheads + RP_HEADS - 1) / RP_HEADS);
}

// ---------------------------------------------------------------- window ring
// Append the K/V of rows [B][n] (positions pos0+i, columns [kcol, kcol+d) and
// [vcol, vcol+d) of src) to the per-sequence rings [B][C][d] at slot pos % C.
// Only the last min(n, C) positions are written.
template <typename T>
__global__ void kv_append_kernel(const T* __restrict__ src, int64_t ld, int kcol, int vcol, int n, int B,
                                 int64_t pos0, int d, T* __restrict__ ring_k, T* __restrict__ ring_v, int C,
                                 const int64_t* pos_dev = nullptr) {
  if (pos_dev) pos0 = *pos_dev;
  const int first = n > C ? n - C : 0;
  const int cnt = n - first;
  const int per_row = d / 8;  // 16-byte chunks (d % 8 == 0 for bf16; float path uses scalar loop)
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (sizeof(T) == 2) {
    if (idx >= (int64_t)B * cnt * per_row) return;
    const int ch = (int)(idx % per_row);
    const int64_t r = idx / per_row;
    const int b = (int)(r / cnt), i = first + (int)(r % cnt);
    const int64_t slot = (pos0 + i) % C;
    const T* s = src + ((int64_t)b * n + i) * ld;
    *(uint4*)(ring_k + ((int64_t)b * C + slot) * d + ch * 8) = *(const uint4*)(s + kcol + ch * 8);
    *(uint4*)(ring_v + ((int64_t)b * C + slot) * d + ch * 8) = *(const uint4*)(s + vcol + ch * 8);
  } else {
    if (idx >= (int64_t)B * cnt * d) return;
    const int c = (int)(idx % d);
    const int64_t r = idx / d;
    const int b = (int)(r / cnt), i = first + (int)(r % cnt);
    const int64_t slot = (pos0 + i) % C;
    const T* s = src + ((int64_t)b * n + i) * ld;
    ring_k[((int64_t)b * C + slot) * d + c] = s[kcol + c];
    ring_v[((int64_t)b * C + slot) * d + c] = s[vcol + c];
  }
}

// ---------------------------------------------------------------- cross entropy
// One CTA per row of logits z [rows][V] (V % (16 / sizeof(T)) == 0).
// loss = logsumexp(z) - z[target], from one pass of 16-byte loads keeping a
// running (max, sum of exp) per thread, merged across the block. If
// grad_scale != 0, z is overwritten in place by dz = (softmax(z) - onehot) *
// grad_scale in a second vectorised pass. Row r belongs to sequence r / n at
// chunk offset r % n; its loss goes to loss_out[(r / n) * loss_ld + loss_off + r % n]
// (skipped when loss_out is null).

template <typename T>
__global__ void __launch_bounds__(256) ce_kernel(T* __restrict__ z, int V, const int32_t* __restrict__ targets,
                                                 int n, float* loss_out, int64_t loss_ld, int64_t loss_off,
                                                 float grad_scale, int* err) {
  constexpr int VEC = 16 / sizeof(T);
  const int row = blockIdx.x;
  T* zr = z + (int64_t)row * V;
  __shared__ float sm_m[8], sm_s[8];
  __shared__ float bc[1];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  float m = -INFINITY, sum = 0.f;
  for (int c = tid * VEC; c < V; c += 256 * VEC) {
    const uint4 u = *reinterpret_cast<const uint4*>(zr + c);
    const T* e = reinterpret_cast<const T*>(&u);
    float x[VEC], mv = -INFINITY;
#pragma unroll
    for (int i = 0; i < VEC; ++i) { x[i] = to_f32(e[i]); mv = fmaxf(mv, x[i]); }
    const float M = fmaxf(m, mv);
    float add = 0.f;
#pragma unroll
    for (int i = 0; i < VEC; ++i) add += expf(x[i] - M);
    sum = (m == -INFINITY ? 0.f : sum * expf(m - M)) + add;
    m = M;
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
  const float lse = bc[0];
  int t = targets[row];
  if (t < 0 || t >= V) {  // ids are validated here too: the last target of a call is never embedded
    if (tid == 0) set_error(err, DEV_BAD_TOKEN);
    t = 0;
  }
  if (tid == 0 && loss_out) {
    const int seq = row / n, i = row % n;
    loss_out[(int64_t)seq * loss_ld + loss_off + i] = lse - to_f32(zr[t]);
  }
  if (grad_scale != 0.f) {
    __syncthreads();  // every thread has read zr[t] before it is overwritten
    for (int c = tid * VEC; c < V; c += 256 * VEC) {
      uint4 u = *reinterpret_cast<const uint4*>(zr + c);
      T* e = reinterpret_cast<T*>(&u);
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        const float p = expf(to_f32(e[i]) - lse);
        e[i] = from_f32<T>((p - (c + i == t ? 1.f : 0.f)) * grad_scale);
      }
      *reinterpret_cast<uint4*>(zr + c) = u;
    }
  }
}

// Greedy choice for decode: argmax (lowest id on ties) unless forced[row] >= 0.
// Writes chosen id, its loss -log p, and the row's max logit. bf16 rows with V % 8 == 0
// take one pass with 16-byte loads: each thread keeps its (max, lowest index of the
// max, sum of exp(z - max)) and the block merges them; otherwise two scalar passes.
__device__ __forceinline__ void amx_merge(float& m, int& i, float& s, float om, int oi, float os) {
  const float mn = fmaxf(m, om);
  s = (m == -INFINITY ? 0.f : s * expf(m - mn)) + (om == -INFINITY ? 0.f : os * expf(om - mn));
  if (om > m || (om == m && oi < i)) i = oi;
  m = mn;
}
template <typename T>
__global__ void __launch_bounds__(1024) argmax_kernel(const T* __restrict__ z, int V,
                                                      const int32_t* __restrict__ forced, int32_t* chosen,
                                                      float* loss, float* zmax_out) {
  const int row = blockIdx.x;
  const T* zr = z + (int64_t)row * V;
  __shared__ float rv[32];
  __shared__ int ri[32];
  __shared__ float rs[32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  if (sizeof(T) == 2 && V % 8 == 0) {
    float m = -INFINITY, s = 0.f;
    int bi = 0x7fffffff;
    for (int c = tid * 8; c < V; c += blockDim.x * 8) {
      const uint4 u = *(const uint4*)(zr + c);
      const T* e = reinterpret_cast<const T*>(&u);
      float x[8], cm = -INFINITY;
      int ci = 0x7fffffff;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        x[k] = to_f32(e[k]);
        if (x[k] > cm) { cm = x[k]; ci = c + k; }  // strict: the lowest index of the chunk's max
      }
      float cs = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) cs += expf(x[k] - cm);
      amx_merge(m, bi, s, cm, ci, cs);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float om = __shfl_xor_sync(0xffffffffu, m, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      const float os = __shfl_xor_sync(0xffffffffu, s, o);
      amx_merge(m, bi, s, om, oi, os);
    }
    if (lane == 0) { rv[w] = m; ri[w] = bi; rs[w] = s; }
    __syncthreads();
    if (tid == 0) {
      float M = rv[0], S = rs[0];
      int I = ri[0];
      for (int i = 1; i < nw; ++i) amx_merge(M, I, S, rv[i], ri[i], rs[i]);
      const int f = forced ? forced[row] : -1;
      const int c = (f >= 0 && f < V) ? f : I;
      chosen[row] = c;
      loss[row] = M + logf(S) - to_f32(zr[c]);
      if (zmax_out) zmax_out[row] = M;
    }
    return;
  }
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int c = tid; c < V; c += blockDim.x) {
    const float v = to_f32(zr[c]);
    if (v > best || (v == best && c < bi)) { best = v; bi = c; }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > best || (ov == best && oi < bi)) { best = ov; bi = oi; }
  }
  if (lane == 0) { rv[w] = best; ri[w] = bi; }
  __syncthreads();
  if (tid == 0) {
    for (int i = 1; i < nw; ++i)
      if (rv[i] > rv[0] || (rv[i] == rv[0] && ri[i] < ri[0])) { rv[0] = rv[i]; ri[0] = ri[i]; }
  }
  __syncthreads();
  const float mx = rv[0];
  float se = 0.f;
  for (int c = tid; c < V; c += blockDim.x) se += expf(to_f32(zr[c]) - mx);
#pragma unroll
  for (int o = 16; o; o >>= 1) se += __shfl_xor_sync(0xffffffffu, se, o);
  if (lane == 0) rs[w] = se;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int i = 0; i < nw; ++i) s += rs[i];
    const int f = forced ? forced[row] : -1;
    const int c = (f >= 0 && f < V) ? f : ri[0];
    chosen[row] = c;
    loss[row] = mx + logf(s) - to_f32(zr[c]);
    if (zmax_out) zmax_out[row] = mx;
  }
}

// ---------------------------------------------------------------- small copies
template <typename S, typename D>
__global__ void convert_kernel(const S* __restrict__ src, D* __restrict__ dst, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = from_f32<D>(to_f32(src[i]));
}

// Residual of the key-value-binding loss of one adaptive block, scaled to its gradient:
// G = s (m - a) + G, where m - a is the MLP's prediction (its sub-layer output) and G
// holds -s v on entry (s = 2/b); GT receives G in the element type. n4 = elements / 4;
// all pointers 16-byte aligned (rows of d % 8 == 0 elements in 256-byte aligned buffers).
template <typename T>
__global__ void __launch_bounds__(256) kvb_residual_kernel(const float* __restrict__ m, const float* __restrict__ a,
                                                           float* __restrict__ G, T* __restrict__ GT, float s,
                                                           int64_t n4) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 mv = reinterpret_cast<const float4*>(m)[i];
  const float4 av = reinterpret_cast<const float4*>(a)[i];
  float4 g = reinterpret_cast<float4*>(G)[i];
  g.x += s * (mv.x - av.x);
  g.y += s * (mv.y - av.y);
  g.z += s * (mv.z - av.z);
  g.w += s * (mv.w - av.w);
  reinterpret_cast<float4*>(G)[i] = g;
  T* o = GT + 4 * i;
  o[0] = from_f32<T>(g.x);
  o[1] = from_f32<T>(g.y);
  o[2] = from_f32<T>(g.z);
  o[3] = from_f32<T>(g.w);
}

// out = init + delta (fast weights W_init + dW exported in fp32)
template <typename T>
__global__ void add_init_kernel(const T* __restrict__ init, const float* __restrict__ delta, float* __restrict__ out,
                                int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = to_f32(init[i]) + delta[i];
}

// ---------------------------------------------------------------- decode step helpers
// The decode step runs as one captured CUDA graph per call; what changes from token
// to token is read from the device: the absolute position *pos (advanced by
// decode_advance_kernel at the end of the step) and the call's first position base.

// pend_in[b][pos % bsz][:] = x[b][:] (input of the first adaptive block of this position)
__global__ void pend_store_kernel(const float* __restrict__ x, int B, int d, float* __restrict__ pend_in, int bsz,
                                  const int64_t* __restrict__ pos) {
  const int64_t slot = *pos % bsz;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)B * d) return;
  const int b = (int)(idx / d), c = (int)(idx % d);
  pend_in[((int64_t)b * bsz + slot) * d + c] = x[idx];
}

// forced_col[b] = forced[b][t] with t = *pos - base (or -1 without forcing)
__global__ void forced_gather_kernel(const int32_t* __restrict__ forced, int64_t n, int B, int32_t* forced_col,
                                     const int64_t* __restrict__ pos, int64_t base) {
  const int b = threadIdx.x;
  if (b < B) forced_col[b] = forced[b * n + (*pos - base)];
}

// out_tok[b][t] = chosen[b]; out_loss[b][t] = loss[b]; pend_tgt[b][pos % bsz] = chosen[b]; t = *pos - base
__global__ void decode_record_kernel(const int32_t* chosen, const float* loss, int B, int64_t n, int32_t* out_tok,
                                     float* out_loss, int32_t* pend_tgt, int bsz, const int64_t* __restrict__ pos,
                                     int64_t base) {
  const int b = threadIdx.x;
  if (b >= B) return;
  const int64_t t = *pos - base;
  out_tok[b * n + t] = chosen[b];
  if (out_loss) out_loss[b * n + t] = loss[b];
  pend_tgt[(int64_t)b * bsz + *pos % bsz] = chosen[b];
}

__global__ void decode_advance_kernel(int64_t* pos) { *pos += 1; }


// targets[b][i] = tok[b*tok_ld + off + i]
__global__ void gather_tokens_kernel(const int32_t* __restrict__ tok, int64_t tok_ld, int64_t off, int n, int B,
                                     int32_t* __restrict__ out, int64_t out_bstride, int64_t out_off) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n * B) return;
  const int b = idx / n, i = idx % n;
  out[b * out_bstride + out_off + i] = tok[(int64_t)b * tok_ld + off + i];
}

// One chunk's inputs, in one launch: rows [b][off, off+n) of the frozen stack's
// output src [B][src rows][d] -> dst [B][n][d] (16-byte copies, d % 4 == 0), and the
// chunk's targets tgt[b][i] = tok[b*tok_ld + tok_off + i].
__global__ void gather_chunk_kernel(const float* __restrict__ src, int64_t src_bstride, int64_t off, int n, int B,
                                    int d, float* __restrict__ dst, const int32_t* __restrict__ tok, int64_t tok_ld,
                                    int64_t tok_off, int32_t* __restrict__ tgt) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t per = (int64_t)n * (d / 4);
  if (idx < (int64_t)n * B) {
    const int b = (int)(idx / n), i = (int)(idx % n);
    tgt[idx] = tok[(int64_t)b * tok_ld + tok_off + i];
  }
  if (idx >= per * B) return;
  const int b = (int)(idx / per);
  const int64_t r = idx % per;
  reinterpret_cast<float4*>(dst + (int64_t)b * n * d)[r] =
      reinterpret_cast<const float4*>(src + b * src_bstride + off * d)[r];
}

}  // namespace ttt
