// Tensor-core sliding-window attention (bf16 operands, fp32 softmax and
// accumulation) with warp-level mma.sync m16n8k16 tiles: forward, and the
// backward split into a dQ pass over each query's whole window and a dK/dV
// pass over the current rows only (cached K/V are constants).
//
// Tiles: 64 queries x 64 keys per CTA step, 4 warps of 16 query rows (16 key
// rows in the dK/dV pass). K/V/Q/dO tiles are staged by cp.async into
// XOR-swizzled shared memory (16-byte chunk c of row r stored at c ^ (r % 8))
// and read with ldmatrix. Key tiles are 64-aligned in absolute position, so a
// tile lies entirely in the ring (positions < q0) or in the current rows; the
// dispatcher requires q0 % 64 == 0 and C % 64 == 0. Window and causal masks are
// applied only on tiles that cross the diagonal or the window's far edge.
// Softmax runs in the log2 domain (scores pre-multiplied by log2(e)/sqrt(hd)).
#pragma once

#include "ttt_attention.cuh"
#include "ttt_common.cuh"

namespace ttt {

constexpr int AM_BM = 64;   // queries per CTA (forward, dQ) / keys per CTA (dK, dV)
constexpr int AM_BN = 64;   // keys (forward, dQ) / queries (dK, dV) per inner tile
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 bytes read -> 16 zero bytes written
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte chunk c of row r in a swizzled tile with HD/8 chunks per row.
template <int HD> __device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return (uint32_t)(r * (HD * 2) + ((c ^ (r & 7)) << 4));
}

// Stage 64 rows x HD of bf16 into a swizzled tile. Row i comes from src_row(i); rows
// for which valid(i) is false are zero-filled. 128 threads.
template <int HD, typename RowFn, typename ValidFn>
__device__ __forceinline__ void stage_tile(uint32_t sbase, const void* any_valid, RowFn src_row, ValidFn valid) {
  constexpr int CH = HD / 8;
#pragma unroll
  for (int e = threadIdx.x; e < 64 * CH; e += 128) {
    const int r = e / CH, c = e % CH;
    const bool v = valid(r);
    // a zero-byte copy reads nothing; any mapped address serves as its source
    cp_async16(sbase + sw_off<HD>(r, c), v ? (const void*)(src_row(r) + c * 8) : any_valid, v);
  }
}

// Pointer to key/value row of absolute position pos (ring or current rows).
__device__ __forceinline__ const bf16* kv_row(const AttnParams& p, const bf16* cur, const bf16* ring, int b, int h,
                                              int64_t pos) {
  if (pos >= p.q0) return cur + ((int64_t)b * p.n + (pos - p.q0)) * p.ldkv + h * p.hd;
  return ring + ((int64_t)b * p.C + pos % p.C) * p.d + h * p.hd;
}

// ---------------------------------------------------------------- forward
template <int HD>
__global__ void __launch_bounds__(128) attn_fwd_mma_kernel(AttnParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  constexpr int TILE = 64 * HD * 2;
  const uint32_t sQ = smem_u32(sm);
  const uint32_t sK0 = sQ + TILE, sV0 = sQ + 2 * TILE;  // stage s: K at sK0 + 2*s*TILE, V at sV0 + 2*s*TILE
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int i0 = qb * AM_BM;                       // first query row (chunk-relative)
  const int64_t P0 = p.q0 + i0;                    // its absolute position
  const int nq = min(AM_BM, p.n - i0);
  const int64_t Plast = P0 + nq - 1;
  const int64_t jlo = max((int64_t)0, P0 - p.window + 1);
  const int64_t jt0 = (jlo / AM_BN) * AM_BN, jt_end = (Plast / AM_BN) * AM_BN;
  const bf16* Qg = (const bf16*)p.Q;
  const bf16* Kc = (const bf16*)p.K;
  const bf16* Vc = (const bf16*)p.V;
  const bf16* Kr = (const bf16*)p.Kc;
  const bf16* Vr = (const bf16*)p.Vc;

  stage_tile<HD>(sQ, Qg, [&](int r) { return Qg + ((int64_t)b * p.n + i0 + r) * p.ldq + h * HD; },
                 [&](int r) { return r < nq; });
  auto load_kv = [&](int stage, int64_t j0) {
    stage_tile<HD>(sK0 + stage * 2 * TILE, Qg, [&](int r) { return kv_row(p, Kc, Kr, b, h, j0 + r); },
                   [&](int r) { return j0 + r <= Plast; });
    stage_tile<HD>(sV0 + stage * 2 * TILE, Qg, [&](int r) { return kv_row(p, Vc, Vr, b, h, j0 + r); },
                   [&](int r) { return j0 + r <= Plast; });
  };
  load_kv(0, jt0);
  cp_async_commit();

  const float sc = p.scale * kLog2e;
  float o[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int r0 = warp * 16 + g;                // this thread's rows within the CTA: r0, r0 + 8
  const int64_t Pr0 = P0 + r0, Pr1 = Pr0 + 8;

  int stage = 0;
  for (int64_t j0 = jt0; j0 <= jt_end; j0 += AM_BN, stage ^= 1) {
    if (j0 + AM_BN <= jt_end) {
      load_kv(stage ^ 1, j0 + AM_BN);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t sK = sK0 + stage * 2 * TILE, sV = sV0 + stage * 2 * TILE;
    // S = Q K^T for this warp's 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = kk * 2 + (lane >> 4);
        ldsm_x4(sQ + sw_off<HD>(r, c), a0, a1, a2, a3);
      }
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {  // pairs of 8-key tiles
        uint32_t b0, b1, b2, b3;
        const int r = nt * 16 + (lane & 7) + (lane >> 4) * 8;
        const int c = kk * 2 + ((lane >> 3) & 1);
        ldsm_x4(sK + sw_off<HD>(r, c), b0, b1, b2, b3);
        mma16816(s[2 * nt], a0, a1, a2, a3, b0, b1);
        mma16816(s[2 * nt + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // scale, mask, online softmax (log2 domain)
    const bool need_mask = (j0 + AM_BN - 1 > P0) || (j0 < Plast - p.window + 1);
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[nt][e] * sc;
        if (need_mask) {
          const int64_t j = j0 + nt * 8 + 2 * t4 + (e & 1);
          const int64_t P = (e < 2) ? Pr0 : Pr1;
          if (j > P || j < P - p.window + 1) v = -INFINITY;
        }
        s[nt][e] = v;
      }
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
    const float c0 = ex2(m0 - base0), c1 = ex2(m1 - base1);
    m0 = mn0; m1 = mn1;
    float ls0 = 0.f, ls1 = 0.f;
    uint32_t pa[4][4];  // P as A fragments for 4 k-steps of 16 keys
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = ex2(s[nt][0] - base0), p1 = ex2(s[nt][1] - base0);
      const float p2 = ex2(s[nt][2] - base1), p3 = ex2(s[nt][3] - base1);
      ls0 += p0 + p1;
      ls1 += p2 + p3;
      const int ks = nt >> 1, hi = nt & 1;
      pa[ks][hi * 2 + 0] = pack_bf16x2(p0, p1);
      pa[ks][hi * 2 + 1] = pack_bf16x2(p2, p3);
    }
    l0 = l0 * c0 + ls0;
    l1 = l1 * c1 + ls1;
#pragma unroll
    for (int i = 0; i < HD / 8; ++i) { o[i][0] *= c0; o[i][1] *= c0; o[i][2] *= c1; o[i][3] *= c1; }
    // O += P V
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int nt = 0; nt < HD / 16; ++nt) {
        uint32_t b0, b1, b2, b3;
        const int r = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = nt * 2 + (lane >> 4);
        ldsm_x4_t(sV + sw_off<HD>(r, c), b0, b1, b2, b3);
        mma16816(o[2 * nt], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b0, b1);
        mma16816(o[2 * nt + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b2, b3);
      }
    }
    __syncthreads();  // stage reused by the next prefetch
  }
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  bf16* O = (bf16*)p.O;
  const int row0 = i0 + r0, row1 = row0 + 8;
#pragma unroll
  for (int nt = 0; nt < HD / 8; ++nt) {
    const int col = h * HD + nt * 8 + 2 * t4;
    if (r0 < nq) *(uint32_t*)(O + ((int64_t)b * p.n + row0) * p.ldo + col) = pack_bf16x2(o[nt][0] * inv0, o[nt][1] * inv0);
    if (r0 + 8 < nq)
      *(uint32_t*)(O + ((int64_t)b * p.n + row1) * p.ldo + col) = pack_bf16x2(o[nt][2] * inv1, o[nt][3] * inv1);
  }
  if (p.lse && t4 == 0) {
    const float ln2 = 0.6931471805599453f;
    if (r0 < nq) p.lse[((int64_t)b * p.H + h) * p.n + row0] = (m0 + __log2f(l0)) * ln2;
    if (r0 + 8 < nq) p.lse[((int64_t)b * p.H + h) * p.n + row1] = (m1 + __log2f(l1)) * ln2;
  }
}

template <int HD> constexpr int attn_fwd_mma_smem() { return 5 * 64 * HD * 2; }

// 16x64 score block of one warp: s = A_tile(16 rows of sA) x B_tile^T (64 rows of sB), both [64][HD] swizzled.
template <int HD>
__device__ __forceinline__ void warp_scores(uint32_t sA, uint32_t sB, int warp, int lane, float (&s)[8][4]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4(sA + sw_off<HD>(warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, kk * 2 + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sB + sw_off<HD>(nt * 16 + (lane & 7) + (lane >> 4) * 8, kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
      mma16816(s[2 * nt], a0, a1, a2, a3, b0, b1);
      mma16816(s[2 * nt + 1], a0, a1, a2, a3, b2, b3);
    }
  }
}

// acc[16 x HD] += P[16 x 64] (A fragments pa) x Bt, where Bt row k (of 64) is a row of sB: acc += P sB.
template <int HD>
__device__ __forceinline__ void warp_pv(uint32_t sB, int lane, const uint32_t (&pa)[4][4], float (&acc)[HD / 8][4]) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
    for (int nt = 0; nt < HD / 16; ++nt) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sB + sw_off<HD>(ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, nt * 2 + (lane >> 4)), b0, b1, b2, b3);
      mma16816(acc[2 * nt], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b0, b1);
      mma16816(acc[2 * nt + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b2, b3);
    }
  }
}

// pack a 16x64 fp32 accumulator block into bf16 A fragments (4 k-steps of 16)
__device__ __forceinline__ void to_afrag(const float (&x)[8][4], uint32_t (&pa)[4][4]) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int ks = nt >> 1, hi = nt & 1;
    pa[ks][hi * 2 + 0] = pack_bf16x2(x[nt][0], x[nt][1]);
    pa[ks][hi * 2 + 1] = pack_bf16x2(x[nt][2], x[nt][3]);
  }
}

// ---------------------------------------------------------------- backward: dQ
// Per 64 query rows: over every key tile of the window, P = exp(S - lse),
// dP = dO V^T, dS = P (dP - D), dQ += dS K. lse, D from the forward / prep kernel.
template <int HD>
__global__ void __launch_bounds__(128) attn_bwd_dq_mma_kernel(AttnParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  constexpr int TILE = 64 * HD * 2;
  const uint32_t sQ = smem_u32(sm), sdO = sQ + TILE;
  const uint32_t sK0 = sQ + 2 * TILE, sV0 = sQ + 3 * TILE;  // stage s at + 2*s*TILE
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int i0 = qb * AM_BM;
  const int64_t P0 = p.q0 + i0;
  const int nq = min(AM_BM, p.n - i0);
  const int64_t Plast = P0 + nq - 1;
  const int64_t jlo = max((int64_t)0, P0 - p.window + 1);
  const int64_t jt0 = (jlo / AM_BN) * AM_BN, jt_end = (Plast / AM_BN) * AM_BN;
  const bf16* Qg = (const bf16*)p.Q;
  const bf16* dOg = (const bf16*)p.dO;
  stage_tile<HD>(sQ, Qg, [&](int r) { return Qg + ((int64_t)b * p.n + i0 + r) * p.ldq + h * HD; },
                 [&](int r) { return r < nq; });
  stage_tile<HD>(sdO, Qg, [&](int r) { return dOg + ((int64_t)b * p.n + i0 + r) * p.lddo + h * HD; },
                 [&](int r) { return r < nq; });
  auto load_kv = [&](int stage, int64_t j0) {
    stage_tile<HD>(sK0 + stage * 2 * TILE, Qg,
                   [&](int r) { return kv_row(p, (const bf16*)p.K, (const bf16*)p.Kc, b, h, j0 + r); },
                   [&](int r) { return j0 + r <= Plast; });
    stage_tile<HD>(sV0 + stage * 2 * TILE, Qg,
                   [&](int r) { return kv_row(p, (const bf16*)p.V, (const bf16*)p.Vc, b, h, j0 + r); },
                   [&](int r) { return j0 + r <= Plast; });
  };
  load_kv(0, jt0);
  cp_async_commit();
  const float sc = p.scale * kLog2e;
  const int r0 = warp * 16 + g;
  const int64_t Pr0 = P0 + r0, Pr1 = Pr0 + 8;
  const int64_t si = ((int64_t)b * p.H + h) * p.n + i0;
  const float L0 = r0 < nq ? p.lse[si + r0] * kLog2e : INFINITY;
  const float L1 = r0 + 8 < nq ? p.lse[si + r0 + 8] * kLog2e : INFINITY;
  const float D0 = r0 < nq ? p.Dsum[si + r0] : 0.f;
  const float D1 = r0 + 8 < nq ? p.Dsum[si + r0 + 8] : 0.f;
  float dq[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
  int stage = 0;
  for (int64_t j0 = jt0; j0 <= jt_end; j0 += AM_BN, stage ^= 1) {
    if (j0 + AM_BN <= jt_end) {
      load_kv(stage ^ 1, j0 + AM_BN);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t sK = sK0 + stage * 2 * TILE, sV = sV0 + stage * 2 * TILE;
    float s[8][4], dp[8][4];
    warp_scores<HD>(sQ, sK, warp, lane, s);
    warp_scores<HD>(sdO, sV, warp, lane, dp);
    const bool need_mask = (j0 + AM_BN - 1 > P0) || (j0 < Plast - p.window + 1);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool lo_row = e < 2;
        float pr = ex2(s[nt][e] * sc - (lo_row ? L0 : L1));
        if (need_mask) {
          const int64_t j = j0 + nt * 8 + 2 * t4 + (e & 1);
          const int64_t P = lo_row ? Pr0 : Pr1;
          if (j > P || j < P - p.window + 1) pr = 0.f;
        }
        s[nt][e] = pr * (dp[nt][e] - (lo_row ? D0 : D1));  // dS
      }
    }
    uint32_t pa[4][4];
    to_afrag(s, pa);
    warp_pv<HD>(sK, lane, pa, dq);
    __syncthreads();
  }
  bf16* dQ = (bf16*)p.dQ;
#pragma unroll
  for (int nt = 0; nt < HD / 8; ++nt) {
    const int col = h * HD + nt * 8 + 2 * t4;
    if (r0 < nq)
      *(uint32_t*)(dQ + ((int64_t)b * p.n + i0 + r0) * p.lddq + col) = pack_bf16x2(dq[nt][0] * p.scale, dq[nt][1] * p.scale);
    if (r0 + 8 < nq)
      *(uint32_t*)(dQ + ((int64_t)b * p.n + i0 + r0 + 8) * p.lddq + col) =
          pack_bf16x2(dq[nt][2] * p.scale, dq[nt][3] * p.scale);
  }
}

// ---------------------------------------------------------------- backward: dK, dV
// Per 64 current key rows: over the query tiles that see them,
// S^T = K Q^T, P^T = exp(S^T - lse), dP^T = V dO^T, dS^T = P^T (dP^T - D),
// dV += P^T dO, dK += dS^T Q. Keys of earlier chunks get no gradient.
template <int HD>
__global__ void __launch_bounds__(128) attn_bwd_dkv_mma_kernel(AttnParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  constexpr int TILE = 64 * HD * 2;
  const uint32_t sK = smem_u32(sm), sV = sK + TILE;
  const uint32_t sQ0 = sK + 2 * TILE, sdO0 = sK + 3 * TILE;  // stage s at + 2*s*TILE
  float* sLD = (float*)(sm + 6 * TILE);                      // [2 stages][lse2 64 | D 64]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int j0r = kb * AM_BM;                     // first key row (chunk-relative)
  const int nk = min(AM_BM, p.n - j0r);
  const int64_t J0 = p.q0 + j0r;                  // its absolute position
  const int iend = (int)min((int64_t)p.n, (int64_t)j0r + nk - 1 + p.window);  // queries [j0r, iend)
  const bf16* Qg = (const bf16*)p.Q;
  const bf16* dOg = (const bf16*)p.dO;
  stage_tile<HD>(sK, Qg, [&](int r) { return (const bf16*)p.K + ((int64_t)b * p.n + j0r + r) * p.ldkv + h * HD; },
                 [&](int r) { return r < nk; });
  stage_tile<HD>(sV, Qg, [&](int r) { return (const bf16*)p.V + ((int64_t)b * p.n + j0r + r) * p.ldkv + h * HD; },
                 [&](int r) { return r < nk; });
  const int64_t si = ((int64_t)b * p.H + h) * p.n;
  auto load_q = [&](int stage, int i0) {
    stage_tile<HD>(sQ0 + stage * 2 * TILE, Qg, [&](int r) { return Qg + ((int64_t)b * p.n + i0 + r) * p.ldq + h * HD; },
                   [&](int r) { return i0 + r < iend; });
    stage_tile<HD>(sdO0 + stage * 2 * TILE, Qg,
                   [&](int r) { return dOg + ((int64_t)b * p.n + i0 + r) * p.lddo + h * HD; },
                   [&](int r) { return i0 + r < iend; });
    if (threadIdx.x < 64) {
      const int i = i0 + threadIdx.x;
      sLD[stage * 128 + threadIdx.x] = i < iend ? p.lse[si + i] * kLog2e : INFINITY;
      sLD[stage * 128 + 64 + threadIdx.x] = i < iend ? p.Dsum[si + i] : 0.f;
    }
  };
  load_q(0, j0r);
  cp_async_commit();
  const float sc = p.scale * kLog2e;
  const int r0 = warp * 16 + g;                    // this thread's key rows: r0, r0 + 8
  const int64_t Jr0 = J0 + r0, Jr1 = Jr0 + 8;
  float dk[HD / 8][4], dv[HD / 8][4];
#pragma unroll
  for (int i = 0; i < HD / 8; ++i) {
    dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = 0.f;
    dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;
  }
  int stage = 0;
  for (int i0 = j0r; i0 < iend; i0 += AM_BN, stage ^= 1) {
    if (i0 + AM_BN < iend) {
      load_q(stage ^ 1, i0 + AM_BN);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t sQ = sQ0 + stage * 2 * TILE, sdO = sdO0 + stage * 2 * TILE;
    const float* Ls = sLD + stage * 128;
    float st[8][4], dpt[8][4];
    warp_scores<HD>(sK, sQ, warp, lane, st);   // rows: keys, cols: queries
    warp_scores<HD>(sV, sdO, warp, lane, dpt);
    const int64_t Pq0 = p.q0 + i0;
    const bool need_mask = (Pq0 < J0 + AM_BM - 1) || (Pq0 + AM_BN - 1 - p.window + 1 > J0);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qc = nt * 8 + 2 * t4 + (e & 1);
        float pr = ex2(st[nt][e] * sc - Ls[qc]);
        if (need_mask) {
          const int64_t P = Pq0 + qc;
          const int64_t j = (e < 2) ? Jr0 : Jr1;
          if (j > P || j < P - p.window + 1) pr = 0.f;
        }
        st[nt][e] = pr;  // P^T
      }
    }
    uint32_t pa[4][4];
    to_afrag(st, pa);
    warp_pv<HD>(sdO, lane, pa, dv);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[nt][e] *= dpt[nt][e] - Ls[64 + nt * 8 + 2 * t4 + (e & 1)];  // dS^T
    to_afrag(st, pa);
    warp_pv<HD>(sQ, lane, pa, dk);
    __syncthreads();
  }
  bf16* dK = (bf16*)p.dK;
  bf16* dV = (bf16*)p.dV;
#pragma unroll
  for (int nt = 0; nt < HD / 8; ++nt) {
    const int col = h * HD + nt * 8 + 2 * t4;
    if (r0 < nk) {
      const int64_t o = ((int64_t)b * p.n + j0r + r0) * p.lddq + col;
      *(uint32_t*)(dK + o) = pack_bf16x2(dk[nt][0] * p.scale, dk[nt][1] * p.scale);
      *(uint32_t*)(dV + o) = pack_bf16x2(dv[nt][0], dv[nt][1]);
    }
    if (r0 + 8 < nk) {
      const int64_t o = ((int64_t)b * p.n + j0r + r0 + 8) * p.lddq + col;
      *(uint32_t*)(dK + o) = pack_bf16x2(dk[nt][2] * p.scale, dk[nt][3] * p.scale);
      *(uint32_t*)(dV + o) = pack_bf16x2(dv[nt][2], dv[nt][3]);
    }
  }
}

template <int HD> constexpr int attn_bwd_mma_smem() { return 6 * 64 * HD * 2 + 2 * 128 * 4; }

// Launchers: return false when the shape is not served (caller uses the SIMT kernels).
inline bool attn_mma_ok(const AttnParams& p) {
  return (p.hd == 64 || p.hd == 128) && p.q0 % 64 == 0 && (p.q0 == 0 || p.C % 64 == 0) && p.ldq % 8 == 0 &&
         p.ldkv % 8 == 0 && p.d % 8 == 0 && p.n >= 1;
}

template <int HD> inline cudaError_t attn_mma_attributes() {
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_mma_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       attn_fwd_mma_smem<HD>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_dq_mma_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn_bwd_mma_smem<HD>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_dkv_mma_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn_bwd_mma_smem<HD>());
  return e;
}

// (attributes are set by prime_kernel_attributes() before the first launch)
template <int HD> inline cudaError_t attn_fwd_mma_launch(const AttnParams& p, cudaStream_t st) {
  constexpr int smem = attn_fwd_mma_smem<HD>();
  dim3 grid((p.n + AM_BM - 1) / AM_BM, p.H, p.B);
  attn_fwd_mma_kernel<HD><<<grid, 128, smem, st>>>(p);
  return cudaGetLastError();
}

template <int HD>
inline cudaError_t attn_bwd_mma_launch(const AttnParams& p, cudaStream_t st, bool with_dq = true, bool with_dkv = true) {
  constexpr int smem = attn_bwd_mma_smem<HD>();
  dim3 grid((p.n + AM_BM - 1) / AM_BM, p.H, p.B);
  if (with_dq) attn_bwd_dq_mma_kernel<HD><<<grid, 128, smem, st>>>(p);
  if (with_dkv) attn_bwd_dkv_mma_kernel<HD><<<grid, 128, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace ttt
