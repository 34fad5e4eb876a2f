// Causal sliding-window attention of the TTT-E2E path, forward and backward.
//
// Query row i of sequence b sits at absolute position P = q0 + i and attends to
// keys at positions [max(0, P-k+1), P] (window k, causal), as the pages'
// sliding-window attention with k >= b prescribes (b-lab.team summary,
// "Integration with Sliding-Window Attention"; technical review §5).
// Keys come from two places:
//   * positions >= q0: the current rows (same rows as the queries),
//   * positions <  q0: the per-sequence ring cache [B][C][d], slot = pos % C,
//     holding K/V computed when their rows were processed. These cached K/V are
//     constants: the backward produces dK/dV for current rows only.
// Online softmax in fp32; lse = m + log(l) is kept for the backward.
#pragma once

#include "ttt_common.cuh"

namespace ttt {

struct AttnParams {
  int B, H, hd, n, d;
  int64_t q0;
  int window;
  const void* Q; int64_t ldq;          // [B*n][ldq], head h at column h*hd
  const void* K; const void* V; int64_t ldkv;
  const void* Kc; const void* Vc; int C;  // rings [B][C][d]
  void* O; int64_t ldo;
  float* lse;                          // [B][H][n]
  float scale;
  // backward
  const void* dO; int64_t lddo;
  float* Dsum;                         // [B][H][n] = rowsum(dO * O)
  int dsum_in_dq;                      // 1: the tcgen05 dQ kernel forms Dsum itself (no separate pass)
  void* dQ; void* dK; void* dV; int64_t lddq;  // dQ/dK/dV rows [B*n][lddq]
};

template <typename T>
__device__ __forceinline__ const T* key_row(const AttnParams& p, const T* cur, const T* ring, int b, int h,
                                            int64_t pos) {
  if (pos >= p.q0) return cur + ((int64_t)b * p.n + (pos - p.q0)) * p.ldkv + h * p.hd;
  return ring + ((int64_t)b * p.C + pos % p.C) * p.d + h * p.hd;
}

// ---------------------------------------------------------------- SIMT forward
// One warp per (row, head); lanes take 32 consecutive keys at a time.
template <typename T>
__global__ void __launch_bounds__(128) attn_fwd_simt_kernel(AttnParams p) {
  __shared__ float qs[4][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * 4 + warp;
  if (gw >= (int64_t)p.B * p.n * p.H) return;
  const int h = (int)(gw % p.H);
  const int row = (int)(gw / p.H);
  const int b = row / p.n, i = row % p.n;
  const int64_t P = p.q0 + i;
  const int64_t lo = P - p.window + 1 > 0 ? P - p.window + 1 : 0;
  const T* Q = (const T*)p.Q + (int64_t)row * p.ldq + h * p.hd;
  for (int c = lane; c < p.hd; c += 32) qs[warp][c] = to_f32(Q[c]) * p.scale;
  __syncwarp();
  const int nd = (p.hd + 31) / 32;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float m = -INFINITY, l = 0.f;
  for (int64_t j0 = lo; j0 <= P; j0 += 32) {
    const int64_t j = j0 + lane;
    float s = -INFINITY;
    if (j <= P) {
      const T* kr = key_row<T>(p, (const T*)p.K, (const T*)p.Kc, b, h, j);
      float dot = 0.f;
      for (int c = 0; c < p.hd; ++c) dot = fmaf(qs[warp][c], to_f32(kr[c]), dot);
      s = dot;
    }
    float mb = s;
#pragma unroll
    for (int o = 16; o; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const float mnew = fmaxf(m, mb);
    const float pj = (j <= P) ? expf(s - mnew) : 0.f;
    const float corr = expf(m - mnew);
    float ps = pj;
#pragma unroll
    for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    l = l * corr + ps;
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[t] *= corr;
    const int cnt = (int)((P - j0 + 1) < 32 ? (P - j0 + 1) : 32);
    for (int jj = 0; jj < cnt; ++jj) {
      const float pp = __shfl_sync(0xffffffffu, pj, jj);
      const T* vr = key_row<T>(p, (const T*)p.V, (const T*)p.Vc, b, h, j0 + jj);
      for (int t = 0; t < nd; ++t) {
        const int c = lane + 32 * t;
        if (c < p.hd) acc[t] = fmaf(pp, to_f32(vr[c]), acc[t]);
      }
    }
    m = mnew;
  }
  T* O = (T*)p.O + (int64_t)row * p.ldo + h * p.hd;
  const float inv = 1.f / l;
  for (int t = 0; t < nd; ++t) {
    const int c = lane + 32 * t;
    if (c < p.hd) O[c] = from_f32<T>(acc[t] * inv);
  }
  if (lane == 0 && p.lse) p.lse[((int64_t)b * p.H + h) * p.n + i] = m + logf(l);
}

// ---------------------------------------------------------------- backward
// Dsum[b][h][i] = sum_c dO[row][h*hd+c] * O[row][h*hd+c]
template <typename T>
__global__ void attn_bwd_prep_kernel(AttnParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (gw >= (int64_t)p.B * p.n * p.H) return;
  const int h = (int)(gw % p.H);
  const int row = (int)(gw / p.H);
  const T* dO = (const T*)p.dO + (int64_t)row * p.lddo + h * p.hd;
  const T* O = (const T*)p.O + (int64_t)row * p.ldo + h * p.hd;
  float s = 0.f;
  for (int c = lane; c < p.hd; c += 32) s += to_f32(dO[c]) * to_f32(O[c]);
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) p.Dsum[((int64_t)(row / p.n) * p.H + h) * p.n + row % p.n] = s;
}

// dQ for every query over its whole window (cached and current keys).
template <typename T>
__global__ void __launch_bounds__(128) attn_bwd_dq_simt_kernel(AttnParams p) {
  __shared__ float qs[4][128];
  __shared__ float dos[4][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * 4 + warp;
  if (gw >= (int64_t)p.B * p.n * p.H) return;
  const int h = (int)(gw % p.H);
  const int row = (int)(gw / p.H);
  const int b = row / p.n, i = row % p.n;
  const int64_t P = p.q0 + i;
  const int64_t lo = P - p.window + 1 > 0 ? P - p.window + 1 : 0;
  const T* Q = (const T*)p.Q + (int64_t)row * p.ldq + h * p.hd;
  const T* dO = (const T*)p.dO + (int64_t)row * p.lddo + h * p.hd;
  for (int c = lane; c < p.hd; c += 32) { qs[warp][c] = to_f32(Q[c]) * p.scale; dos[warp][c] = to_f32(dO[c]); }
  __syncwarp();
  const int64_t si = ((int64_t)b * p.H + h) * p.n + i;
  const float lse = p.lse[si], D = p.Dsum[si];
  const int nd = (p.hd + 31) / 32;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t j0 = lo; j0 <= P; j0 += 32) {
    const int64_t j = j0 + lane;
    float ds = 0.f;
    if (j <= P) {
      const T* kr = key_row<T>(p, (const T*)p.K, (const T*)p.Kc, b, h, j);
      const T* vr = key_row<T>(p, (const T*)p.V, (const T*)p.Vc, b, h, j);
      float s = 0.f, dp = 0.f;
      for (int c = 0; c < p.hd; ++c) {
        s = fmaf(qs[warp][c], to_f32(kr[c]), s);
        dp = fmaf(dos[warp][c], to_f32(vr[c]), dp);
      }
      const float pr = expf(s - lse);
      ds = pr * (dp - D);
    }
    const int cnt = (int)((P - j0 + 1) < 32 ? (P - j0 + 1) : 32);
    for (int jj = 0; jj < cnt; ++jj) {
      const float g = __shfl_sync(0xffffffffu, ds, jj);
      const T* kr = key_row<T>(p, (const T*)p.K, (const T*)p.Kc, b, h, j0 + jj);
      for (int t = 0; t < nd; ++t) {
        const int c = lane + 32 * t;
        if (c < p.hd) acc[t] = fmaf(g, to_f32(kr[c]), acc[t]);
      }
    }
  }
  T* dQ = (T*)p.dQ + (int64_t)row * p.lddq + h * p.hd;
  for (int t = 0; t < nd; ++t) {
    const int c = lane + 32 * t;
    if (c < p.hd) dQ[c] = from_f32<T>(acc[t] * p.scale);
  }
}

// dK, dV for the current rows only (cached keys are constants).
template <typename T>
__global__ void __launch_bounds__(128) attn_bwd_dkv_simt_kernel(AttnParams p) {
  __shared__ float ks[4][128];
  __shared__ float vs[4][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * 4 + warp;
  if (gw >= (int64_t)p.B * p.n * p.H) return;
  const int h = (int)(gw % p.H);
  const int row = (int)(gw / p.H);
  const int b = row / p.n, jr = row % p.n;
  const T* K = (const T*)p.K + (int64_t)row * p.ldkv + h * p.hd;
  const T* V = (const T*)p.V + (int64_t)row * p.ldkv + h * p.hd;
  for (int c = lane; c < p.hd; c += 32) { ks[warp][c] = to_f32(K[c]) * p.scale; vs[warp][c] = to_f32(V[c]); }
  __syncwarp();
  const int iend = (jr + p.window < p.n) ? jr + p.window : p.n;  // queries i in [jr, iend)
  const int nd = (p.hd + 31) / 32;
  float dk[4] = {0.f, 0.f, 0.f, 0.f}, dv[4] = {0.f, 0.f, 0.f, 0.f};
  for (int i0 = jr; i0 < iend; i0 += 32) {
    const int i = i0 + lane;
    float pr = 0.f, ds = 0.f;
    if (i < iend) {
      const int qrow = b * p.n + i;
      const T* Q = (const T*)p.Q + (int64_t)qrow * p.ldq + h * p.hd;
      const T* dO = (const T*)p.dO + (int64_t)qrow * p.lddo + h * p.hd;
      float s = 0.f, dp = 0.f;
      for (int c = 0; c < p.hd; ++c) {
        s = fmaf(ks[warp][c], to_f32(Q[c]), s);
        dp = fmaf(vs[warp][c], to_f32(dO[c]), dp);
      }
      const int64_t si = ((int64_t)b * p.H + h) * p.n + i;
      pr = expf(s - p.lse[si]);
      ds = pr * (dp - p.Dsum[si]);
    }
    const int cnt = (iend - i0) < 32 ? (iend - i0) : 32;
    for (int ii = 0; ii < cnt; ++ii) {
      const float pp = __shfl_sync(0xffffffffu, pr, ii);
      const float g = __shfl_sync(0xffffffffu, ds, ii);
      const int qrow = b * p.n + i0 + ii;
      const T* Q = (const T*)p.Q + (int64_t)qrow * p.ldq + h * p.hd;
      const T* dO = (const T*)p.dO + (int64_t)qrow * p.lddo + h * p.hd;
      for (int t = 0; t < nd; ++t) {
        const int c = lane + 32 * t;
        if (c < p.hd) {
          dv[t] = fmaf(pp, to_f32(dO[c]), dv[t]);
          dk[t] = fmaf(g, to_f32(Q[c]), dk[t]);
        }
      }
    }
  }
  T* dK = (T*)p.dK + (int64_t)row * p.lddq + h * p.hd;
  T* dV = (T*)p.dV + (int64_t)row * p.lddq + h * p.hd;
  for (int t = 0; t < nd; ++t) {
    const int c = lane + 32 * t;
    if (c < p.hd) { dK[c] = from_f32<T>(dk[t] * p.scale); dV[c] = from_f32<T>(dv[t]); }
  }
}

// ---------------------------------------------------------------- decode (one query)
// One query per sequence at position P = *pos (the token's own K/V already in the
// ring); keys [max(0, P-k+1), P] all read from the ring. One CTA per (head,
// sequence), 8 warps splitting the window: lanes over keys for the scores (each
// key row read with 16-byte loads issued together), lanes over head dims for P·V,
// merged across warps at the end. HBM-bound: each K and V row of the window is
// read once.
template <typename T> __device__ __forceinline__ void load_row_f32(const T* src, float* dst, int n);
template <> __device__ __forceinline__ void load_row_f32<bf16>(const bf16* src, float* dst, int n) {
  for (int v = 0; v < n / 8; ++v) {
    const uint4 u = reinterpret_cast<const uint4*>(src)[v];
    const bf16* e = reinterpret_cast<const bf16*>(&u);
#pragma unroll
    for (int k = 0; k < 8; ++k) dst[v * 8 + k] = __bfloat162float(e[k]);
  }
}
template <> __device__ __forceinline__ void load_row_f32<float>(const float* src, float* dst, int n) {
  for (int v = 0; v < n / 4; ++v) {
    const float4 u = reinterpret_cast<const float4*>(src)[v];
    dst[v * 4] = u.x; dst[v * 4 + 1] = u.y; dst[v * 4 + 2] = u.z; dst[v * 4 + 3] = u.w;
  }
}

template <typename T, int HD>
__global__ void __launch_bounds__(256) attn_decode_kernel(const T* __restrict__ q, int64_t ldq,
                                                          const T* __restrict__ ring_k, const T* __restrict__ ring_v,
                                                          int C, int d, int window, const int64_t* __restrict__ pos,
                                                          float scale, T* __restrict__ out, int64_t ldo,
                                                          float* __restrict__ part, int* __restrict__ ticket) {
  // The window of (head h, sequence b) is split into gridDim.z equal parts, one CTA
  // each. In a CTA each lane owns one key per step: its K row gives the score, its V row
  // is accumulated into the lane's partial output (all row loads independent); the 32
  // partial outputs of a warp are summed once at the end, then the 8 warps'. With more
  // than one part, each CTA stores its (max, sum, unnormalised output) in `part` and the
  // last CTA of the (h, b) to finish (a ticket counter, reset by that CTA) merges the
  // parts in their fixed order, so the result does not depend on which CTA is last.
  constexpr int CH = HD < 32 ? HD : (HD == 128 ? 16 : 32);  // row chunk held in registers
  __shared__ float qs[HD];
  __shared__ float wm[8], wl[8];
  __shared__ float wo[8][HD];
  __shared__ int last;
  const int h = blockIdx.x, b = blockIdx.y, z = blockIdx.z, nz = gridDim.z;
  const int H = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t P = *pos;
  const int64_t lo = P - window + 1 > 0 ? P - window + 1 : 0;
  const int64_t span = (P - lo + nz) / nz;  // keys per part (the last part may be shorter or empty)
  const int64_t zlo = lo + z * span;
  const int64_t zhi = (zlo + span - 1 < P) ? zlo + span - 1 : P;
  for (int c = threadIdx.x; c < HD; c += 256) qs[c] = to_f32(q[(int64_t)b * ldq + h * HD + c]) * scale;
  __syncthreads();
  const T* Kb = ring_k + (int64_t)b * C * d + h * HD;
  const T* Vb = ring_v + (int64_t)b * C * d + h * HD;
  float acc[HD];
#pragma unroll
  for (int c = 0; c < HD; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;  // warp-uniform running max, lane-partial sum
  for (int64_t j0 = zlo + warp * 32; j0 <= zhi; j0 += 256) {
    const int64_t j = j0 + lane;
    const bool valid = j <= zhi;
    const int64_t slot = (valid ? j : zhi) % C;
    float s = 0.f;
#pragma unroll
    for (int c0 = 0; c0 < HD; c0 += CH) {
      float kr[CH];
      load_row_f32<T>(Kb + slot * d + c0, kr, CH);
#pragma unroll
      for (int c = 0; c < CH; ++c) s = fmaf(qs[c0 + c], kr[c], s);
    }
    s = valid ? s : -INFINITY;
    float mb = s;
#pragma unroll
    for (int o = 16; o; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    const float mnew = fmaxf(m, mb);
    const float corr = expf(m - mnew);  // 0 on the first step (m = -inf)
    const float pj = valid ? expf(s - mnew) : 0.f;
    l = l * corr + pj;
#pragma unroll
    for (int c0 = 0; c0 < HD; c0 += CH) {
      float vr[CH];
      load_row_f32<T>(Vb + slot * d + c0, vr, CH);
#pragma unroll
      for (int c = 0; c < CH; ++c) acc[c0 + c] = fmaf(pj, vr[c], acc[c0 + c] * corr);
    }
    m = mnew;
  }
  // warp sums of the lane partials
#pragma unroll
  for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
  for (int c = 0; c < HD; ++c) {
    float v = acc[c];
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    acc[c] = v;
  }
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
#pragma unroll
    for (int c = 0; c < HD; ++c) wo[warp][c] = acc[c];
  }
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < 8; ++w) M = fmaxf(M, wm[w]);
  float Lsum = 0.f;
  for (int w = 0; w < 8; ++w) Lsum += wm[w] == -INFINITY ? 0.f : wl[w] * expf(wm[w] - M);
  if (nz == 1) {
    for (int c = threadIdx.x; c < HD; c += 256) {
      float o = 0.f;
      for (int w = 0; w < 8; ++w)
        if (wm[w] != -INFINITY) o += wo[w][c] * expf(wm[w] - M);
      out[(int64_t)b * ldo + h * HD + c] = from_f32<T>(o / Lsum);
    }
    return;
  }
  // this part -> part[(b, h, z)] = (M, L, O[HD]); the last CTA of (h, b) merges
  float* mine = part + (((int64_t)b * H + h) * nz + z) * (HD + 2);
  for (int c = threadIdx.x; c < HD; c += 256) {
    float o = 0.f;
    for (int w = 0; w < 8; ++w)
      if (wm[w] != -INFINITY) o += wo[w][c] * expf(wm[w] - M);
    mine[2 + c] = o;
  }
  if (threadIdx.x == 0) {
    mine[0] = M;
    mine[1] = Lsum;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(ticket + (int64_t)b * H + h, 1) == nz - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const float* base = part + ((int64_t)b * H + h) * nz * (HD + 2);
  float Mt = -INFINITY;
  for (int zz = 0; zz < nz; ++zz) Mt = fmaxf(Mt, __ldcg(base + zz * (HD + 2)));
  float Lt = 0.f;
  for (int zz = 0; zz < nz; ++zz) {
    const float mz = __ldcg(base + zz * (HD + 2));
    if (mz != -INFINITY) Lt += __ldcg(base + zz * (HD + 2) + 1) * expf(mz - Mt);
  }
  for (int c = threadIdx.x; c < HD; c += 256) {
    float o = 0.f;
    for (int zz = 0; zz < nz; ++zz) {
      const float mz = __ldcg(base + zz * (HD + 2));
      if (mz != -INFINITY) o += __ldcg(base + zz * (HD + 2) + 2 + c) * expf(mz - Mt);
    }
    out[(int64_t)b * ldo + h * HD + c] = from_f32<T>(o / Lt);
  }
  if (threadIdx.x == 0) ticket[(int64_t)b * H + h] = 0;  // ready for the next launch
}

// Decode attention for bf16 at head dims 64 and 128: one CTA of 4 warps per (head h,
// sequence b, part z of the window). The HD/8 lanes of a key group read one key row
// (16 bytes each, so a warp instruction covers whole rows: 4 keys at HD = 64, 2 at
// HD = 128), form the score by a reduction over the group, and keep a running max, sum
// and their 8 output elements; the groups of a warp and then the warps are merged at
// the end. Registers stay few, so the window can be split into many parts; the part
// results are merged by the last CTA of the (h, b) as in attn_decode_kernel. The ring is
// read through plain (coherent) loads: this kernel may write its newest row itself.
template <int HD>
__global__ void __launch_bounds__(128) attn_decode_rows_kernel(const bf16* __restrict__ q, int64_t ldq,
                                                               const bf16* ring_k, const bf16* ring_v, int C, int d,
                                                               int window, const int64_t* __restrict__ pos,
                                                               float scale, bf16* __restrict__ out, int64_t ldo,
                                                               float* __restrict__ part, int* __restrict__ ticket,
                                                               const float2* __restrict__ rope_lo,
                                                               const float2* __restrict__ rope_hi,
                                                               bf16* __restrict__ ring_k_w, bf16* __restrict__ ring_v_w) {
  constexpr int LPK = HD / 8;    // lanes per key row
  constexpr int KPW = 32 / LPK;  // keys per warp step
  constexpr int U = 4;           // steps whose loads are issued together
  __shared__ float wm[4], wl[4];
  __shared__ float wo[4][HD];
  __shared__ int last;
  const int h = blockIdx.x, b = blockIdx.y, z = blockIdx.z, nz = gridDim.z, H = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane / LPK, e = lane % LPK;  // key group within the warp, 16-byte chunk of the row
  const int64_t P = *pos;
  const int64_t lo = P - window + 1 > 0 ? P - window + 1 : 0;
  const int64_t span = (P - lo + nz) / nz;
  const int64_t zlo = lo + z * span;
  const int64_t zhi = (zlo + span - 1 < P) ? zlo + span - 1 : P;
  // With rope_lo set, q and k of this position arrive unrotated: each lane rotates its
  // 8 elements of q (pairs (i, i + HD/2), the partner chunk in lane e ^ LPK/2) at position
  // P from the angle tables, lo[P & 1023] and hi[P >> 10] combined by the angle-addition
  // formulas; the CTA whose part holds key P also writes the rotated k and the v of this
  // position to the ring (slot P mod C) before any of its warps reads the ring.
  const int half_e = e & (LPK / 2 - 1);  // chunk index within its half of the head
  float cs[8], sn[8];
  if (rope_lo) {
    const float2* a2 = rope_lo + (P & 1023) * (HD / 2) + half_e * 8;
    const float2* b2 = rope_hi + (P >> 10) * (HD / 2) + half_e * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 a = a2[i], bb = b2[i];
      cs[i] = a.x * bb.x - a.y * bb.y;
      sn[i] = a.y * bb.x + a.x * bb.y;
    }
  }
  auto rotate = [&](const uint4& own, const uint4& mate, float* outv) {  // this lane's 8 rotated elements
    const bf16* x = reinterpret_cast<const bf16*>(&own);
    const bf16* y = reinterpret_cast<const bf16*>(&mate);
    const bool first_half = e < LPK / 2;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float u = __bfloat162float(x[i]), v = __bfloat162float(y[i]);
      outv[i] = first_half ? u * cs[i] - v * sn[i] : u * cs[i] + v * sn[i];
    }
  };
  float qv[8];
  {
    const uint4 u = *(const uint4*)(q + (int64_t)b * ldq + h * HD + e * 8);
    if (rope_lo) {
      const uint4 mate = *(const uint4*)(q + (int64_t)b * ldq + h * HD + (e ^ (LPK / 2)) * 8);
      rotate(u, mate, qv);
#pragma unroll
      for (int i = 0; i < 8; ++i) qv[i] *= scale;
    } else {
      const bf16* qe = reinterpret_cast<const bf16*>(&u);
#pragma unroll
      for (int i = 0; i < 8; ++i) qv[i] = __bfloat162float(qe[i]) * scale;
    }
  }
  if (rope_lo && ring_k_w && warp == 0 && g == 0 && P >= zlo && P <= zhi) {
    const bf16* kq = q + (int64_t)b * ldq + d + h * HD;  // k follows q in the q|k|v row
    const uint4 ku = *(const uint4*)(kq + e * 8), km = *(const uint4*)(kq + (e ^ (LPK / 2)) * 8);
    float kr[8];
    rotate(ku, km, kr);
    const int64_t off = ((int64_t)b * C + P % C) * d + h * HD + e * 8;
    *(uint4*)(ring_k_w + off) = make_uint4(pack_bf16x2(kr[0], kr[1]), pack_bf16x2(kr[2], kr[3]),
                                           pack_bf16x2(kr[4], kr[5]), pack_bf16x2(kr[6], kr[7]));
    *(uint4*)(ring_v_w + off) = *(const uint4*)(kq + d + e * 8);
  }
  if (rope_lo) __syncthreads();  // the ring row of P is in place for every warp of this CTA
  const bf16* Kb = ring_k + (int64_t)b * C * d + h * HD + e * 8;
  const bf16* Vb = ring_v + (int64_t)b * C * d + h * HD + e * 8;
  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  // the warp's first key per step is uniform across the warp (every lane runs the same
  // iterations and shuffles); group g takes key jw + g
  for (int64_t jw = zlo + warp * KPW; jw <= zhi; jw += (int64_t)4 * KPW * U) {
    uint4 ku[U], vu[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t j = jw + (int64_t)u * 4 * KPW + g;
      const int64_t slot = (j <= zhi ? j : zhi) % C;
      ku[u] = *(const uint4*)(Kb + slot * d);
      vu[u] = *(const uint4*)(Vb + slot * d);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t j = jw + (int64_t)u * 4 * KPW + g;
      const bf16* ke = reinterpret_cast<const bf16*>(&ku[u]);
      float sc = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) sc = fmaf(qv[i], __bfloat162float(ke[i]), sc);
#pragma unroll
      for (int o = 1; o < LPK; o <<= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
      if (j <= zhi) {  // uniform across the key group
        const float mn = fmaxf(m, sc);
        const float corr = expf(m - mn);  // 0 while m = -inf
        const float pj = expf(sc - mn);
        l = l * corr + pj;
        const bf16* ve = reinterpret_cast<const bf16*>(&vu[u]);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(pj, __bfloat162float(ve[i]), acc[i] * corr);
        m = mn;
      }
    }
  }
  // merge the key groups of the warp (lanes with the same chunk e)
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, o);
    const float lo_ = __shfl_xor_sync(0xffffffffu, l, o);
    const float mn = fmaxf(m, mo);
    const float fa = m == -INFINITY ? 0.f : expf(m - mn);
    const float fb = mo == -INFINITY ? 0.f : expf(mo - mn);
    l = l * fa + lo_ * fb;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = acc[i] * fa + __shfl_xor_sync(0xffffffffu, acc[i], o) * fb;
    m = mn;
  }
  if (g == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) wo[warp][e * 8 + i] = acc[i];
    if (e == 0) { wm[warp] = m; wl[warp] = l; }
  }
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w]);
  float Lsum = 0.f;
#pragma unroll
  for (int w = 0; w < 4; ++w) Lsum += wm[w] == -INFINITY ? 0.f : wl[w] * expf(wm[w] - M);
  float* mine = nz > 1 ? part + (((int64_t)b * H + h) * nz + z) * (HD + 2) : nullptr;
  for (int c = threadIdx.x; c < HD; c += 128) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w)
      if (wm[w] != -INFINITY) o += wo[w][c] * expf(wm[w] - M);
    if (nz == 1) out[(int64_t)b * ldo + h * HD + c] = __float2bfloat16_rn(o / Lsum);
    else mine[2 + c] = o;
  }
  if (nz == 1) return;
  if (threadIdx.x == 0) {
    mine[0] = M;
    mine[1] = Lsum;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(ticket + (int64_t)b * H + h, 1) == nz - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const float* base = part + ((int64_t)b * H + h) * nz * (HD + 2);
  float Mt = -INFINITY;
  for (int zz = 0; zz < nz; ++zz) Mt = fmaxf(Mt, __ldcg(base + zz * (HD + 2)));
  float Lt = 0.f;
  for (int zz = 0; zz < nz; ++zz) {
    const float mz = __ldcg(base + zz * (HD + 2));
    if (mz != -INFINITY) Lt += __ldcg(base + zz * (HD + 2) + 1) * expf(mz - Mt);
  }
  for (int c = threadIdx.x; c < HD; c += 128) {
    float o = 0.f;
    for (int zz = 0; zz < nz; ++zz) {
      const float mz = __ldcg(base + zz * (HD + 2));
      if (mz != -INFINITY) o += __ldcg(base + zz * (HD + 2) + 2 + c) * expf(mz - Mt);
    }
    out[(int64_t)b * ldo + h * HD + c] = __float2bfloat16_rn(o / Lt);
  }
  if (threadIdx.x == 0) ticket[(int64_t)b * H + h] = 0;  // ready for the next launch
}

}  // namespace ttt
