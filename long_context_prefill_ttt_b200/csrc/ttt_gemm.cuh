// Dense contractions of the TTT-E2E path: D[m][n] = alpha * sum_k A[m][k] * B[n][k]
// with fused epilogues.
//
// Two engines share one parameter block and one epilogue definition:
//  * gemm_tc: tcgen05 tensor cores (bf16 operands, fp32 accumulation in TMEM),
//    operands staged by TMA into 128-byte-swizzled shared memory, a 4-6 stage
//    mbarrier ring, one elected thread issuing MMAs, double-buffered TMEM
//    accumulators so that the epilogue of tile t overlaps the main loop of
//    tile t+1 (persistent CTAs, one per SM).
//  * gemm_simt: plain fp32 FFMA tiles for float operands (the fp32 workload
//    needs fp32-exact products) and for shapes the tensor-core tiles do not fit.
//
// Operand "majors": A is logically [M][K]; stored K-major (A[m*lda+k]) or
// MN-major (A[k*lda+m]). Same for B ([N][K]). Forward products use (K, K),
// data gradients (K, MN), weight gradients (MN, MN).
#pragma once

#include "ttt_common.cuh"

namespace ttt {

enum EpiKind : int {
  EPI_STORE = 0,   // D = acc                              (D f32 or element type)
  EPI_RESID = 1,   // D(f32) = acc + X(f32)                (X may alias D)
  EPI_GELU = 2,    // Y = acc (if Y), D = gelu(acc)        (element type)
  EPI_DGELU = 3,   // D = acc * gelu'(X)                   (element type, X element type)
  EPI_SGD = 4,     // D(f32) += acc, Y = D (if Y)          (alpha = -eta)
  EPI_QKV_ROPE = 5,  // D = acc (element type), then RoPE on columns [0, rope_cols) by a separate pass
  EPI_CE = 6,      // LM head + cross-entropy statistics: D = acc (element type); per row and per
                   // 64-column vocabulary chunk k, ce_part[row][k] = (max, sum exp(acc - max)) in
                   // fp32; ce_zt[row] = acc at column ce_tgt[row] (fp32). tcgen05 engine only.
};

struct GemmParams {
  int M, N, K, batch;
  const void* A; int64_t lda, sA; int a_mn;
  const void* B; int64_t ldb, sB; int b_mn;
  // Optional second B of the same shape and layout, accumulated over the same A:
  // acc = sum_k A(m,k) (B(n,k) + B2(n,k)). Used for fast weights held as
  // W_init (shared, sB = 0) + dW (per sequence), so that a bf16 copy of the
  // small update dW is not rounded away against W_init.
  const void* B2; int64_t sB2;
  void* D; int64_t ldd, sD; int d_f32;
  const void* X; int64_t ldx, sX;
  void* Y; int64_t ldy, sY;
  float alpha;
  int epi;
  // EPI_QKV_ROPE: after the product, rotate pairs (i, i + hd/2) of each head in columns [0, rope_cols) of row m at
  // position rope_pos0 + (m % rope_n) (rope_pos0 read from *rope_pos_dev when given), angles
  // pos * base^(-2i/hd) from the double-precision tables lo[p & 1023][i], hi[p >> 10][i].
  const float2* rope_lo; const float2* rope_hi;
  int64_t rope_pos0; const int64_t* rope_pos_dev;
  int rope_n, rope_hd, rope_cols;
  // Optional: the same pass appends the rotated keys and the values of the rows to the
  // window ring [batch][rope_C][rope_cols/2] at slot (position mod rope_C).
  void* rope_ring_k; void* rope_ring_v; int rope_C;
  // EPI_CE: targets [M] (batch 1), partials [M][N / 64], target logits [M]
  const int32_t* ce_tgt; float2* ce_part; float* ce_zt;
  // Tile order of the tensor-core engine within a batch slice: 0 = row blocks outer
  // (consecutive tiles share A rows), 1 = column blocks outer (consecutive tiles share
  // B rows, so a B larger than L2 streams from DRAM once). Set by the host.
  int m_fast;
  // Optional RMSNorm of the rows of A on the way in: A(m, k) = bf16 of
  // norm_x(m, k) * rstd_m * norm_g[k] with rstd_m = 1 / sqrt(mean_k norm_x(m, k)^2 + norm_eps),
  // norm_x fp32 with A's strides (lda, sA). The few-row engine applies it while staging A
  // (and also writes the normalised rows to A and rstd_m to norm_rstd[z * M + m]); every
  // other path runs a separate RMSNorm pass into A first.
  const float* norm_x; const float* norm_g; float norm_eps; float* norm_rstd;
};

// ============================================================== epilogue (per element)
template <typename T>
__device__ __forceinline__ void epi_apply(const GemmParams& p, int z, int m, int n, float acc) {
  acc *= p.alpha;
  const int64_t od = (int64_t)z * p.sD + (int64_t)m * p.ldd + n;
  switch (p.epi) {
    case EPI_STORE:
      if (p.d_f32) ((float*)p.D)[od] = acc; else ((T*)p.D)[od] = from_f32<T>(acc);
      break;
    case EPI_RESID: {
      const float r = ((const float*)p.X)[(int64_t)z * p.sX + (int64_t)m * p.ldx + n];
      ((float*)p.D)[od] = acc + r;
      break;
    }
    case EPI_GELU:
      if (p.Y) ((T*)p.Y)[(int64_t)z * p.sY + (int64_t)m * p.ldy + n] = from_f32<T>(acc);
      ((T*)p.D)[od] = from_f32<T>(gelu_f(acc));
      break;
    case EPI_DGELU: {
      const float u = to_f32(((const T*)p.X)[(int64_t)z * p.sX + (int64_t)m * p.ldx + n]);
      ((T*)p.D)[od] = from_f32<T>(acc * gelu_prime_f(u));
      break;
    }
    case EPI_SGD: {
      float* w = (float*)p.D + od;
      const float nw = *w + acc;
      *w = nw;
      if (p.Y) ((T*)p.Y)[(int64_t)z * p.sY + (int64_t)m * p.ldy + n] = from_f32<T>(nw);
      break;
    }
  }
}

// ============================================================== SIMT engine
// 64x64 output tile, K step 16, 256 threads with 4x4 outputs each.
template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmParams p) {
  __shared__ float As[16][68];
  __shared__ float Bs[16][68];
  const int z = blockIdx.z;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  const T* A = (const T*)p.A + (int64_t)z * p.sA;
  const T* B = (const T*)p.B + (int64_t)z * p.sB;
  float acc[4][4] = {};
  const int passes = p.B2 ? 2 : 1;
  for (int pass = 0; pass < passes; ++pass) {
  if (pass == 1) B = (const T*)p.B2 + (int64_t)z * p.sB2;
  for (int k0 = 0; k0 < p.K; k0 += 16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = t + i * 256;
      int mm, kk;
      if (p.a_mn) { kk = e >> 6; mm = e & 63; } else { mm = e >> 4; kk = e & 15; }
      const int gm = m0 + mm, gk = k0 + kk;
      float v = 0.f;
      if (gm < p.M && gk < p.K) v = to_f32(p.a_mn ? A[(int64_t)gk * p.lda + gm] : A[(int64_t)gm * p.lda + gk]);
      As[kk][mm] = v;
      int nn;
      if (p.b_mn) { kk = e >> 6; nn = e & 63; } else { nn = e >> 4; kk = e & 15; }
      const int gn = n0 + nn;
      const int gk2 = k0 + kk;
      float w = 0.f;
      if (gn < p.N && gk2 < p.K) w = to_f32(p.b_mn ? B[(int64_t)gk2 * p.ldb + gn] : B[(int64_t)gn * p.ldb + gk2]);
      Bs[kk][nn] = w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < p.M && n < p.N) epi_apply<T>(p, z, m, n, acc[i][j]);
    }
}

// ============================================================== skinny engine (decode)
// At most 16 rows per batch slice (one row per sequence in decode): the work is
// reading the weight matrix once. A CTA owns two output columns; four warps per
// column split K into 16-byte-per-lane slabs, two slabs in flight per warp, so
// every SM keeps many weight loads outstanding. Partial sums meet in shared
// memory and the first lanes of each column apply the shared epilogue, one row
// each. The few activation rows come from L1. K-major operands only.
constexpr int SK_MAXM = 16;
template <typename T>
__global__ void __launch_bounds__(256) gemm_skinny_kernel(GemmParams p) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int SLAB = 32 * VEC;  // elements of K per warp-iteration
  __shared__ float part[8][SK_MAXM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = warp >> 2, kw = warp & 3;  // column within the CTA, K quarter
  const int n = blockIdx.x * 2 + col;
  const int z = blockIdx.y;
  float acc[SK_MAXM];
#pragma unroll
  for (int m = 0; m < SK_MAXM; ++m) acc[m] = 0.f;
  if (n < p.N) {
    const T* A = (const T*)p.A + (int64_t)z * p.sA;
    const T* Bw = (const T*)p.B + (int64_t)z * p.sB + (int64_t)n * p.ldb;
    const T* B2w = p.B2 ? (const T*)p.B2 + (int64_t)z * p.sB2 + (int64_t)n * p.ldb : nullptr;
    auto slab = [&](int k0) {
      float w[VEC];
      {
        const uint4 u = *reinterpret_cast<const uint4*>(Bw + k0);
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int i = 0; i < VEC; ++i) w[i] = to_f32(e[i]);
      }
      if (B2w) {
        const uint4 u = *reinterpret_cast<const uint4*>(B2w + k0);
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int i = 0; i < VEC; ++i) w[i] += to_f32(e[i]);
      }
#pragma unroll
      for (int m = 0; m < SK_MAXM; ++m) {
        if (m < p.M) {
          const uint4 u = *reinterpret_cast<const uint4*>(A + (int64_t)m * p.lda + k0);
          const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
          for (int i = 0; i < VEC; ++i) acc[m] = fmaf(to_f32(e[i]), w[i], acc[m]);
        }
      }
    };
    int k0 = (kw * 32 + lane) * VEC;
    for (; k0 + 4 * SLAB < p.K; k0 += 8 * SLAB) {  // two slabs per iteration (this warp's and +4 warps')
      slab(k0);
      slab(k0 + 4 * SLAB);
    }
    for (; k0 < p.K; k0 += 4 * SLAB) slab(k0);
  }
#pragma unroll
  for (int m = 0; m < SK_MAXM; ++m) {
    if (m < p.M) {
      float v = acc[m];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) part[warp][m] = v;
    }
  }
  __syncthreads();
  if (kw == 0 && lane < p.M && n < p.N) {
    const int m = lane;
    const float v = part[col * 4][m] + part[col * 4 + 1][m] + part[col * 4 + 2][m] + part[col * 4 + 3][m];
    epi_apply<T>(p, z, m, n, v);
  }
}

// ============================================================== few-row engine (decode)
// Up to 8 rows per batch slice (one token per sequence in decode, or one row of a
// sequence against its own fast weights): every weight byte is read once and the
// product is bound by memory latency and bandwidth, not arithmetic. A CTA of 8 warps
// owns 8 * CW output columns; the slice's rows of A are staged once in shared memory,
// each warp streams CW weight rows (and their dW rows) with 16 bytes per lane and all
// of a lane's loads of a row in flight, and each lane's CW x 8 partial sums are reduced
// across the warp by recursive halving, after which lane l holds one (column, row) sum.
// CW is chosen on the host so that narrow products still spread over the SMs.
constexpr int RW_MAXM = 8;
constexpr int RW_SMEM_MAX = 96 * 1024;  // staged A: M * K * 2 bytes
template <int CW>
__global__ void __launch_bounds__(256) gemm_rows_kernel(GemmParams p) {
  constexpr int NV = CW * RW_MAXM;  // partial sums per lane: [column j][row m]
  extern __shared__ uint4 xs4[];    // [M][K / 8] 16-byte chunks of this slice's A
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int z = blockIdx.y;
  const int kc = p.K / 8;
  pdl_wait();  // A (and the epilogue inputs) come from the previous kernel
  if (p.norm_x) {  // warp m normalises row m of the slice (RMSNorm) while staging it
    for (int m = warp; m < p.M; m += 8) {
      const float* xr = p.norm_x + (int64_t)z * p.sA + (int64_t)m * p.lda;
      float ss = 0.f;
      for (int c = lane; c < kc; c += 32) {
        const float4 a = *(const float4*)(xr + c * 8), b = *(const float4*)(xr + c * 8 + 4);
        ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w + b.x * b.x + b.y * b.y + b.z * b.z + b.w * b.w;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float rs = rsqrtf(ss / p.K + p.norm_eps);
      const bool first = blockIdx.x == 0;  // one CTA per slice also writes the normalised rows
      if (first && lane == 0 && p.norm_rstd) p.norm_rstd[(int64_t)z * p.M + m] = rs;
      bf16* Ar = (bf16*)p.A + (int64_t)z * p.sA + (int64_t)m * p.lda;
      for (int c = lane; c < kc; c += 32) {
        const float4 a = *(const float4*)(xr + c * 8), b = *(const float4*)(xr + c * 8 + 4);
        const float4 ga = *(const float4*)(p.norm_g + c * 8), gb = *(const float4*)(p.norm_g + c * 8 + 4);
        const uint4 u = make_uint4(pack_bf16x2(a.x * rs * ga.x, a.y * rs * ga.y), pack_bf16x2(a.z * rs * ga.z, a.w * rs * ga.w),
                                   pack_bf16x2(b.x * rs * gb.x, b.y * rs * gb.y), pack_bf16x2(b.z * rs * gb.z, b.w * rs * gb.w));
        xs4[m * kc + c] = u;
        if (first) *(uint4*)(Ar + c * 8) = u;
      }
    }
  } else {
    const bf16* A = (const bf16*)p.A + (int64_t)z * p.sA;
    for (int i = threadIdx.x; i < p.M * kc; i += 256) {
      const int m = i / kc, c = i - m * kc;
      xs4[i] = *(const uint4*)(A + (int64_t)m * p.lda + c * 8);
    }
  }
  __syncthreads();
  pdl_trigger();
  const int n0 = (blockIdx.x * 8 + warp) * CW;
  const bf16* Bw = (const bf16*)p.B + (int64_t)z * p.sB;
  const bf16* B2w = p.B2 ? (const bf16*)p.B2 + (int64_t)z * p.sB2 : nullptr;
  float v[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = 0.f;
#pragma unroll 4
  for (int c = lane; c < kc; c += 32) {
    uint4 wu[CW], w2[CW];
#pragma unroll
    for (int j = 0; j < CW; ++j) {
      const int n = n0 + j < p.N ? n0 + j : p.N - 1;  // columns past N compute a copy, never stored
      wu[j] = *(const uint4*)(Bw + (int64_t)n * p.ldb + c * 8);
      w2[j] = B2w ? *(const uint4*)(B2w + (int64_t)n * p.ldb + c * 8) : make_uint4(0, 0, 0, 0);
    }
    float w[CW][8];
#pragma unroll
    for (int j = 0; j < CW; ++j) {
      const bf16* e = reinterpret_cast<const bf16*>(&wu[j]);
      const bf16* e2 = reinterpret_cast<const bf16*>(&w2[j]);
#pragma unroll
      for (int i = 0; i < 8; ++i) w[j][i] = __bfloat162float(e[i]) + __bfloat162float(e2[i]);
    }
#pragma unroll
    for (int m = 0; m < RW_MAXM; ++m) {
      if (m < p.M) {
        const uint4 xu = xs4[m * kc + c];
        const bf16* xe = reinterpret_cast<const bf16*>(&xu);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float x = __bfloat162float(xe[i]);
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j * RW_MAXM + m] = fmaf(x, w[j][i], v[j * RW_MAXM + m]);
        }
      }
    }
  }
  // recursive halving over the offsets 16, 8, ...: a lane keeps the half of its values
  // selected by (lane & o) and adds its partner's copy of that half; once one value is
  // left, the remaining offsets sum it over the lanes that share its index
#pragma unroll
  for (int st = 0; st < 5; ++st) {
    const int o = 16 >> st;
    const int cnt = NV >> st;  // values left before this step
    if (cnt > 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < cnt / 2; ++i) {
        const float send = up ? v[i] : v[i + cnt / 2];
        const float keep = up ? v[i + cnt / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  // lane l holds index (l / (32 / NV)) = column j * 8 + row m
  const int idx = lane / (32 / NV);
  const int n = n0 + idx / RW_MAXM, m = idx % RW_MAXM;
  if (lane % (32 / NV) == 0 && m < p.M && n < p.N) epi_apply<bf16>(p, z, m, n, v[0]);
}

// ============================================================== tcgen05 engine
constexpr int TC_BM = 128;
constexpr int TC_BK = 64;
// warp 0: TMA, warp 1: MMA + TMEM owner, warps 2-9: epilogue (two warps per TMEM lane
// quarter, each taking half of the tile's columns)
constexpr int TC_THREADS = 320;
constexpr int TC_EPI_WARPS = 8;
constexpr int EPI_STAGE_BYTES = 32 * 32 * 4;  // epilogue staging per warp: 32 rows x 32 fp32

template <int BN> struct TcCfg {
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/ +
                              TC_EPI_WARPS * EPI_STAGE_BYTES /*epilogue staging*/;
  static constexpr int TMEM_COLS = 2 * BN;
};

// GELU for the bf16 tensor-core epilogues. erf by the rational approximation of
// Abramowitz & Stegun, Handbook of Mathematical Functions, eq. 7.1.28:
// erf(x) = 1 - (1 + a1 x + ... + a6 x^6)^-16 for x >= 0 (|error| <= 3e-7 in exact
// arithmetic, about 2e-6 in fp32 near 0), odd extension for x < 0. Branch-free, one
// reciprocal; its error is far below the bf16 rounding of the outputs. (The fp32 path
// keeps the library erff.)
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));  // rcp(+inf) = +0
  return y;
}
__device__ __forceinline__ float erf_as7128(float x) {
  const float ax = fabsf(x);
  float t = fmaf(ax, 4.30638e-5f, 2.765672e-4f);
  t = fmaf(ax, t, 1.520143e-4f);
  t = fmaf(ax, t, 9.2705272e-3f);
  t = fmaf(ax, t, 4.22820123e-2f);
  t = fmaf(ax, t, 7.05230784e-2f);
  t = fmaf(ax, t, 1.0f);
  t *= t;
  t *= t;
  t *= t;
  t *= t;  // t^16
  return copysignf(1.0f - rcp_approx(t), x);
}
__device__ __forceinline__ float gelu_tc(float u) { return 0.5f * u * (1.0f + erf_as7128(u * 0.70710678118654752f)); }
// d gelu / du = Phi(u) + u phi(u); exp(-u^2/2) as exp2 of (-u^2/2) log2(e)
__device__ __forceinline__ float gelu_prime_tc(float u) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-0.72134752044448170f * u * u));
  return 0.5f * (1.0f + erf_as7128(u * 0.70710678118654752f)) + u * e * 0.39894228040143268f;
}

// ---------------------------------------------------------------- epilogue staging
// Each accumulator row belongs to one thread (TMEM lane = row), so a thread's stores of
// its row are 32 accesses to 32 different 128-byte lines per warp instruction, which the
// load/store unit serves one line at a time (measured: a 128 x 128 fp32 residual
// epilogue took 7.3K clocks). Global traffic of the epilogue therefore goes through a
// per-warp shared-memory buffer of 32 rows x 32 columns: eight lanes cover one row's
// 128 bytes (fp32) or four lanes its 64 bytes (bf16), so that each warp instruction
// moves whole lines, and each thread reads or writes its own row in shared memory. The
// 16-byte word q of row r sits at q ^ (r & 7) (fp32 rows) or q ^ ((r >> 1) & 3) (bf16
// rows), so neither access pattern has bank conflicts.

__device__ __forceinline__ uint32_t stg_f32(int r, int q) { return (uint32_t)(r * 128 + ((q ^ (r & 7)) << 4)); }
__device__ __forceinline__ uint32_t stg_b16(int r, int q) { return (uint32_t)(r * 64 + ((q ^ ((r >> 1) & 3)) << 4)); }

// Global inputs of the epilogue for the warp's 32 rows (from mw) and 32 columns (from
// n): for the staged epilogues, this lane's 16-byte pieces in the coalesced layout of
// the fp32 residual (EPI_RESID) or fp32 master weights (EPI_SGD), rows 4i + lane/8,
// piece lane % 8; for EPI_DGELU, the bf16 pre-activations of the lane's own row (first
// four words). They are fetched one 32-column chunk ahead of their use (the first chunk
// before the accumulator is waited for).
struct EpiIn {
  uint4 w[8];
};
__device__ __forceinline__ void epi_fetch32_mixed(const GemmParams& p, int z, int mw, int n, EpiIn& in) {
  const int lane = threadIdx.x & 31;
  if (p.epi == EPI_RESID || p.epi == EPI_SGD) {
    const float* base = p.epi == EPI_RESID ? (const float*)p.X + (int64_t)z * p.sX : (const float*)p.D + (int64_t)z * p.sD;
    const int64_t ld = p.epi == EPI_RESID ? p.ldx : p.ldd;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = mw + 4 * i + (lane >> 3);
      in.w[i] = row < p.M ? *(const uint4*)(base + (int64_t)row * ld + n + (lane & 7) * 4) : make_uint4(0, 0, 0, 0);
    }
  } else if (p.epi == EPI_DGELU) {  // row-wise: the bf16 pre-activations of this thread's own row
    const int m = mw + lane;
    if (m < p.M) {
      const uint4* x = (const uint4*)((const bf16*)p.X + (int64_t)z * p.sX + (int64_t)m * p.ldx + n);
#pragma unroll
      for (int i = 0; i < 4; ++i) in.w[i] = x[i];
    }
  }
}

// The coalesced pieces of `in` -> shared memory (put), then this thread's row out of
// it (get: f(i, x_i) for its 32 values in column order).
__device__ __forceinline__ void stage_put_f32(uint8_t* stg, const EpiIn& in) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 8; ++i) *(uint4*)(stg + stg_f32(4 * i + (lane >> 3), lane & 7)) = in.w[i];
}
template <typename F>
__device__ __forceinline__ void stage_get_f32(const uint8_t* stg, F f) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 x = *(const float4*)(stg + stg_f32(lane, q));
    f(4 * q, x.x); f(4 * q + 1, x.y); f(4 * q + 2, x.z); f(4 * q + 3, x.w);
  }
  __syncwarp();
}
// This thread's row of 32 values -> shared memory -> coalesced global stores of the
// warp's 32 rows (from mw) at columns [n, n + 32) of dst (leading dimension ld).
__device__ __forceinline__ void stage_out_f32(uint8_t* stg, const float* v, float* dst, int64_t ld, int mw, int M,
                                              int n) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *(float4*)(stg + stg_f32(lane, q)) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 4 * i + (lane >> 3);
    const uint4 w = *(const uint4*)(stg + stg_f32(r, lane & 7));
    if (mw + r < M) *(uint4*)(dst + (int64_t)(mw + r) * ld + n + (lane & 7) * 4) = w;
  }
  __syncwarp();
}
__device__ __forceinline__ void stage_out_b16(uint8_t* stg, const float* v, bf16* dst, int64_t ld, int mw, int M,
                                              int n) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *(uint4*)(stg + stg_b16(lane, q)) =
        make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                   pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 8 * i + (lane >> 2);
    const uint4 w = *(const uint4*)(stg + stg_b16(r, lane & 3));
    if (mw + r < M) *(uint4*)(dst + (int64_t)(mw + r) * ld + n + (lane & 3) * 8) = w;
  }
  __syncwarp();
}

// 32 consecutive accumulator columns [n, n + 32) of this thread's row (m = mw + lane)
// through the epilogue; `in` holds what epi_fetch32 read for the warp's rows (from mw)
// and these columns. All 32 lanes of the warp call it together (rows past M are not
// stored). The fp32 read-modify-write epilogues (residual, SGD) go through the staging
// buffer; the bf16-output epilogues store their rows directly, which measured faster
// for them (GELU 1024x4096x2048: 21 us direct, 24 us staged; SGD weight gradient
// 2048x4096x1024: 37.5 us direct, 31.7 us staged).
// n_next >= 0: once `in` is consumed, it is refilled with the inputs of the chunk at
// columns [n_next, n_next + 32).
__device__ __forceinline__ void epi_row32_mixed(const GemmParams& p, int z, int mw, int n, float* v, EpiIn& in,
                                          uint8_t* stg, int n_next) {
  const int m = mw + (int)(threadIdx.x & 31);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] *= p.alpha;
  if (p.epi == EPI_STORE && p.d_f32) {
    stage_out_f32(stg, v, (float*)p.D + (int64_t)z * p.sD, p.ldd, mw, p.M, n);
  } else if (p.epi == EPI_RESID) {
    stage_put_f32(stg, in);
    if (n_next >= 0) epi_fetch32_mixed(p, z, mw, n_next, in);
    stage_get_f32(stg, [&](int i, float x) { v[i] += x; });
    stage_out_f32(stg, v, (float*)p.D + (int64_t)z * p.sD, p.ldd, mw, p.M, n);
  } else if (p.epi == EPI_SGD) {  // D (fp32 master) += acc, Y = bf16 copy of the new D
    stage_put_f32(stg, in);
    if (n_next >= 0) epi_fetch32_mixed(p, z, mw, n_next, in);
    stage_get_f32(stg, [&](int i, float w) { v[i] += w; });
    stage_out_f32(stg, v, (float*)p.D + (int64_t)z * p.sD, p.ldd, mw, p.M, n);
    if (p.Y) stage_out_b16(stg, v, (bf16*)p.Y + (int64_t)z * p.sY, p.ldy, mw, p.M, n);
  } else if (m < p.M) {
    const int64_t od = (int64_t)z * p.sD + (int64_t)m * p.ldd + n;
    uint4* d = (uint4*)((bf16*)p.D + od);
    if (p.epi == EPI_GELU) {
      if (p.Y) {
        uint4* y = (uint4*)((bf16*)p.Y + (int64_t)z * p.sY + (int64_t)m * p.ldy + n);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          y[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                            pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = gelu_tc(v[i]);
    } else if (p.epi == EPI_DGELU) {  // pre-activations of this row, fetched row-wise by epi_fetch32
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bf16* u = reinterpret_cast<const bf16*>(&in.w[i]);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * i + e] *= gelu_prime_tc(__bfloat162float(u[e]));
      }
    }
    if (p.epi == EPI_DGELU && n_next >= 0) epi_fetch32_mixed(p, z, mw, n_next, in);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      d[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                        pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
  }
}

// Row-wise epilogue (all layouts but the weight-gradient one): the global inputs of the
// epilogue for 32 columns of one row, as raw 16-byte words: the fp32 residual
// (EPI_RESID) or fp32 master weights (EPI_SGD) in all eight, the bf16 pre-activations
// (EPI_DGELU) in the first four. They are fetched one 32-column chunk ahead of their use
// (the first chunk before the accumulator is waited for), so each thread has a whole
// chunk of loads in flight instead of one load per store.
__device__ __forceinline__ void epi_fetch32_row(const GemmParams& p, int z, int m, int n, EpiIn& in) {
  if (m >= p.M) return;
  if (p.epi == EPI_RESID) {
    const uint4* x = (const uint4*)((const float*)p.X + (int64_t)z * p.sX + (int64_t)m * p.ldx + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) in.w[i] = x[i];
  } else if (p.epi == EPI_SGD) {
    const uint4* w = (const uint4*)((const float*)p.D + (int64_t)z * p.sD + (int64_t)m * p.ldd + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) in.w[i] = w[i];
  } else if (p.epi == EPI_DGELU) {
    const uint4* x = (const uint4*)((const bf16*)p.X + (int64_t)z * p.sX + (int64_t)m * p.ldx + n);
#pragma unroll
    for (int i = 0; i < 4; ++i) in.w[i] = x[i];
  }
}

// 32 consecutive accumulator columns of one row through the epilogue, vectorised;
// `in` holds what epi_fetch32 read for the same columns.
template <typename T>
__device__ __forceinline__ void epi_row32_direct(const GemmParams& p, int z, int m, int n, float* v, const EpiIn& in) {
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] *= p.alpha;
  const int64_t od = (int64_t)z * p.sD + (int64_t)m * p.ldd + n;
  if (p.epi == EPI_STORE && p.d_f32) {
    float4* d = (float4*)((float*)p.D + od);
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else if (p.epi == EPI_STORE) {
    uint4* d = (uint4*)((T*)p.D + od);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      d[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                        pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
  } else if (p.epi == EPI_RESID) {
    float4* d = (float4*)((float*)p.D + od);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 r = *reinterpret_cast<const float4*>(&in.w[i]);
      d[i] = make_float4(v[4 * i] + r.x, v[4 * i + 1] + r.y, v[4 * i + 2] + r.z, v[4 * i + 3] + r.w);
    }
  } else if (p.epi == EPI_GELU) {
    if (p.Y) {
      uint4* y = (uint4*)((T*)p.Y + (int64_t)z * p.sY + (int64_t)m * p.ldy + n);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        y[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                          pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = gelu_tc(v[i]);
    uint4* d = (uint4*)((T*)p.D + od);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      d[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                        pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
  } else if (p.epi == EPI_DGELU) {
    uint4* d = (uint4*)((T*)p.D + od);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bf16* u = reinterpret_cast<const bf16*>(&in.w[i]);
      float o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = v[8 * i + j] * gelu_prime_tc(__bfloat162float(u[j]));
      d[i] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                        pack_bf16x2(o[6], o[7]));
    }
  } else {  // EPI_SGD
    float4* w = (float4*)((float*)p.D + od);
    float nw[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 c = *reinterpret_cast<const float4*>(&in.w[i]);
      c.x += v[4 * i]; c.y += v[4 * i + 1]; c.z += v[4 * i + 2]; c.w += v[4 * i + 3];
      w[i] = c;
      nw[4 * i] = c.x; nw[4 * i + 1] = c.y; nw[4 * i + 2] = c.z; nw[4 * i + 3] = c.w;
    }
    if (p.Y) {
      uint4* y = (uint4*)((T*)p.Y + (int64_t)z * p.sY + (int64_t)m * p.ldy + n);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        y[i] = make_uint4(pack_bf16x2(nw[8 * i], nw[8 * i + 1]), pack_bf16x2(nw[8 * i + 2], nw[8 * i + 3]),
                          pack_bf16x2(nw[8 * i + 4], nw[8 * i + 5]), pack_bf16x2(nw[8 * i + 6], nw[8 * i + 7]));
    }
  }
}

// EPI_CE on 32 consecutive columns [n, n+32) of row m: store the logits (element
// type), fold them into the running (max, sum-exp) of the current 64-column
// vocabulary chunk, and keep the target's logit in fp32 when it lies here. The
// caller writes (cm, cs) to ce_part after every second call (a chunk is complete).
__device__ __forceinline__ void epi_ce32(const GemmParams& p, int m, int n, float* v, int tgt, float& cm,
                                         float& cs) {
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] *= p.alpha;
    mx = fmaxf(mx, v[i]);
  }
  uint4* d = (uint4*)((bf16*)p.D + (int64_t)m * p.ldd + n);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    d[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                      pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
  if (tgt >= n && tgt < n + 32) {
    // v[tgt - n] by predicated selects: an indexed read would move v to local memory
    const int k = tgt - n;
    float zt = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      asm("{\n\t.reg .pred q;\n\tsetp.eq.s32 q, %2, %3;\n\tselp.f32 %0, %1, %0, q;\n\t}"
          : "+f"(zt)
          : "f"(v[i]), "r"(k), "r"(i));
    p.ce_zt[m] = zt;
  }
  const float M = fmaxf(cm, mx);
  float add = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) add += __expf(v[i] - M);
  cs = (cm == -INFINITY ? 0.f : cs * __expf(cm - M)) + add;
  cm = M;
}

// Split-K partial tile in shared memory: fp32 [128 rows][BN], the 16-byte word q of a
// row stored at q ^ (row & 7), so that eight consecutive rows writing or reading the
// same columns hit distinct banks.
template <int BN>
__device__ __forceinline__ uint32_t part_addr(uint32_t base, int row, int q) {
  return base + (uint32_t)(row * BN + ((q ^ (row & 7)) << 2)) * 4u;
}

// Epilogue of one accumulator tile for one epilogue warp: the warp fetches the global
// inputs of its first 32 columns, waits for the accumulator (wait_acc() false: the
// wait timed out), then reads its TMEM lane quarter (one output row per thread, row m)
// over its half of the tile's columns [c_first*32, c_first*32 + BN/2), calls release()
// once those columns are read (the accumulator may then be overwritten), and applies
// the epilogue through its staging buffer stg, each chunk's inputs fetched while the
// previous chunk is stored. part: shared address of a split-K partial tile to add to
// the accumulator (0: none, [128 rows][BN] from chunk part_c0 on), row: this thread's
// row in the tile.
template <int BN, typename Wait, typename Release>
__device__ __forceinline__ bool epilogue_tile_staged(const GemmParams& p, uint32_t taddr, int z, int m, int n0, int c_first,
                                              uint8_t* stg, Wait wait_acc, Release release, uint32_t part = 0,
                                              int row = 0, int part_c0 = 0) {
  const int mw = m - (int)(threadIdx.x & 31);  // first row of this warp
  EpiIn nxt;
  epi_fetch32_mixed(p, z, mw, n0 + c_first * 32, nxt);
  if (!wait_acc()) return false;
  tc_fence_after();
  const int tgt = (p.epi == EPI_CE && m < p.M) ? p.ce_tgt[m] : -1;
  float cm = -INFINITY, cs = 0.f;
#pragma unroll 1
  for (int c = c_first; c < c_first + BN / 64; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    if (c == c_first + BN / 64 - 1) {  // this warp's columns are read: its share of the accumulator is free
      tc_fence_before();
      __syncwarp();
      release();
    }
    if (part) {  // acc = acc(first K half) + partial(second K half), in this order
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float4 q;
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(q.x), "=f"(q.y), "=f"(q.z), "=f"(q.w)
                     : "r"(part_addr<BN>(part, row, (c - part_c0) * 8 + i)));
        v[4 * i] += q.x; v[4 * i + 1] += q.y; v[4 * i + 2] += q.z; v[4 * i + 3] += q.w;
      }
    }
    if (p.epi == EPI_CE) {
      if (m < p.M) {
        epi_ce32(p, m, n0 + c * 32, v, tgt, cm, cs);
        if (c & 1) {  // a 64-column vocabulary chunk is complete
          p.ce_part[(int64_t)m * (p.N / 64) + (n0 + c * 32) / 64] = make_float2(cm, cs);
          cm = -INFINITY;
          cs = 0.f;
        }
      }
    } else {
      epi_row32_mixed(p, z, mw, n0 + c * 32, v, nxt, stg, c + 1 < c_first + BN / 64 ? n0 + (c + 1) * 32 : -1);
    }
  }
  return true;
}

// Epilogue of one accumulator tile for one epilogue warp: the warp fetches the global
// inputs of its first 32 columns, waits for the accumulator (wait_acc() false: the
// wait timed out), then reads its TMEM lane quarter (one output row per thread, row m)
// over its half of the tile's columns [c_first*32, c_first*32 + BN/2), calls release()
// once those columns are read (the accumulator may then be overwritten), and applies
// the epilogue, each chunk's inputs fetched while the previous chunk is stored.
// part: shared address of a split-K partial tile ([128 rows][BN] from chunk part_c0 on)
// to add to the accumulator (0: none).
template <int BN, typename Wait, typename Release>
__device__ __forceinline__ bool epilogue_tile_direct(const GemmParams& p, uint32_t taddr, int z, int m, int n0, int c_first,
                                              Wait wait_acc, Release release, uint32_t part = 0, int row = 0,
                                              int part_c0 = 0) {
  EpiIn nxt;
  epi_fetch32_row(p, z, m, n0 + c_first * 32, nxt);
  if (!wait_acc()) return false;
  tc_fence_after();
  const int tgt = (p.epi == EPI_CE && m < p.M) ? p.ce_tgt[m] : -1;
  float cm = -INFINITY, cs = 0.f;
#pragma unroll 1
  for (int c = c_first; c < c_first + BN / 64; ++c) {
    float v[32];
    tmem_ld32(taddr + c * 32, v);
    if (c == c_first + BN / 64 - 1) {  // this warp's columns are read: its share of the accumulator is free
      tc_fence_before();
      __syncwarp();
      release();
    }
    if (part) {  // acc = acc(first K half) + partial(second K half), in this order
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float4 q;
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(q.x), "=f"(q.y), "=f"(q.z), "=f"(q.w)
                     : "r"(part_addr<BN>(part, row, (c - part_c0) * 8 + i)));
        v[4 * i] += q.x; v[4 * i + 1] += q.y; v[4 * i + 2] += q.z; v[4 * i + 3] += q.w;
      }
    }
    const EpiIn cur = nxt;
    if (c + 1 < c_first + BN / 64) epi_fetch32_row(p, z, m, n0 + (c + 1) * 32, nxt);
    if (m < p.M) {
      if (p.epi == EPI_CE) {
        epi_ce32(p, m, n0 + c * 32, v, tgt, cm, cs);
        if (c & 1) {  // a 64-column vocabulary chunk is complete
          p.ce_part[(int64_t)m * (p.N / 64) + (n0 + c * 32) / 64] = make_float2(cm, cs);
          cm = -INFINITY;
          cs = 0.f;
        }
      } else {
        epi_row32_direct<bf16>(p, z, m, n0 + c * 32, v, cur);
      }
    }
  }
  return true;
}

// The epilogue of a tile: staged through shared memory in the weight-gradient layout
// (A and B MN-major: the fused SGD update, whose fp32 read-modify-write of the master
// weights is bound by uncoalesced row accesses: 2048x4096x1024 37.5 -> 30 us staged),
// row-wise everywhere else (the bf16-output and residual epilogues of the other
// layouts measured 2-7 us slower per launch staged, from the registers the staged path
// takes at this kernel's 168-register limit).
template <int BN, bool STAGED, typename Wait, typename Release>
__device__ __forceinline__ bool epilogue_tile(const GemmParams& p, uint32_t taddr, int z, int m, int n0, int c_first,
                                              uint8_t* stg, Wait wait_acc, Release release, uint32_t part = 0,
                                              int row = 0, int part_c0 = 0) {
  if constexpr (STAGED)
    return epilogue_tile_staged<BN>(p, taddr, z, m, n0, c_first, stg, wait_acc, release, part, row, part_c0);
  else
    return epilogue_tile_direct<BN>(p, taddr, z, m, n0, c_first, wait_acc, release, part, row, part_c0);
}

// One or two independent products of the same layout and tile width in one persistent
// launch (the tile list of the second follows that of the first), with their tensor maps.
struct TcGroup {
  CUtensorMap tmA[2], tmB[2], tmB2[2];
  GemmParams p[2];
  int nprob;
};

// Persistent warp-specialised tcgen05 GEMM. Requirements (checked on the host):
// N % BN == 0, K % 64 == 0, 16-byte aligned rows; M may have a tail (TMA fills
// out-of-range rows with zeros and the epilogue skips them). With two products
// (g.nprob = 2) the CTAs walk both tile lists as one, so that the epilogue of one
// product's tiles overlaps the mainloop of the next tiles.
template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(TC_THREADS, 1) gemm_tc_kernel(const __grid_constant__ TcGroup g, int* err) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                    // [STAGES]
  uint64_t* empty = bars + C::STAGES;       // [STAGES]
  uint64_t* acc_full = bars + 2 * C::STAGES;      // [2]
  uint64_t* acc_empty = bars + 2 * C::STAGES + 2; // [2]
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * C::STAGES + 4);

  const int warp = threadIdx.x >> 5;
  // tile counts of each product; tiles [0, nt0) belong to product 0, the rest to product 1
  const int mt0 = (g.p[0].M + TC_BM - 1) / TC_BM, ntl0 = g.p[0].N / BN, tpb0 = mt0 * ntl0;
  const int nt0 = tpb0 * g.p[0].batch;
  const int mt1 = g.nprob > 1 ? (g.p[1].M + TC_BM - 1) / TC_BM : 1, ntl1 = g.nprob > 1 ? g.p[1].N / BN : 1;
  const int tpb1 = mt1 * ntl1;
  const int num_tiles = nt0 + (g.nprob > 1 ? tpb1 * g.p[1].batch : 0);
  // product, batch slice and tile origin of a tile
  auto locate = [&](int tile, int& pi, int& z, int& m0, int& n0) {
    pi = tile >= nt0 ? 1 : 0;
    const int t = tile - (pi ? nt0 : 0);
    const int tpb = pi ? tpb1 : tpb0, mt = pi ? mt1 : mt0, ntl = pi ? ntl1 : ntl0;
    const GemmParams& P = pi ? g.p[1] : g.p[0];
    z = t / tpb;
    const int r = t % tpb;
    m0 = (P.m_fast ? r % mt : r / ntl) * TC_BM;
    n0 = (P.m_fast ? r / mt : r % ntl) * BN;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], TC_EPI_WARPS); }
    fence_mbar_init();
    for (int i = 0; i < g.nprob; ++i) {
      prefetch_tmap(&g.tmA[i]);
      prefetch_tmap(&g.tmB[i]);
      if (g.p[i].B2) prefetch_tmap(&g.tmB2[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();     // operands and epilogue inputs come from the previous kernel
  pdl_trigger();

  if (warp == 0) {
    if (elect_lane0()) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int pi, z, m0, n0;
        locate(tile, pi, z, m0, n0);
        const GemmParams& P = pi ? g.p[1] : g.p[0];
        const CUtensorMap* mA = &g.tmA[pi];
        const int kb_one = P.K / TC_BK;
        const int k_blocks = P.B2 ? 2 * kb_one : kb_one;
        const int zb_scale = P.sB ? 1 : 0;  // shared B (batch stride 0): always batch slice 0
        const int zb2_scale = P.sB2 ? 1 : 0;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t round = it / C::STAGES;
          if (!mbar_wait(&empty[s], (round & 1) ^ 1, err, DEV_TIMEOUT_EMPTY)) { ok = false; break; }
          uint8_t* sa = smem + s * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
          const bool second = kb >= kb_one;
          const int k0 = (second ? kb - kb_one : kb) * TC_BK;
          const CUtensorMap* mb = second ? &g.tmB2[pi] : &g.tmB[pi];
          const int zb = z * (second ? zb2_scale : zb_scale);
          if (A_MN) {
            tma_load_3d(sa, mA, &full[s], m0, k0, z);
            tma_load_3d(sa + 8192, mA, &full[s], m0 + 64, k0, z);
          } else {
            tma_load_3d(sa, mA, &full[s], k0, m0, z);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tma_load_3d(sb + j * 8192, mb, &full[s], n0 + 64 * j, k0, zb);
          } else {
            tma_load_3d(sb, mb, &full[s], k0, n0, zb);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (elect_lane0()) {
      constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, BN, A_MN, B_MN);
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++lt) {
        const GemmParams& P = tile >= nt0 ? g.p[1] : g.p[0];
        const int kb_one = P.K / TC_BK;
        const int k_blocks = P.B2 ? 2 * kb_one : kb_one;
        const int acc = lt & 1;
        const uint32_t use = lt >> 1;
        if (!mbar_wait(&acc_empty[acc], (use & 1) ^ 1, err, DEV_TIMEOUT_ACC)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t round = it / C::STAGES;
          if (!mbar_wait(&full[s], round & 1, err, DEV_TIMEOUT_FULL)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk) {
            const uint64_t ad = A_MN ? smem_desc_sw128(sa + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(sb + kk * 32, 16, 1024);
            tc_mma_f16(d_tmem, ad, bd, idesc, (kb | kk) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
      }
    }
  } else {
    // epilogue warps 2..9: TMEM lane quarter = warp % 4; warps 2-5 take columns
    // [0, BN/2) of the tile, warps 6-9 columns [BN/2, BN)
    const int quarter = warp & 3;
    const int c_first = (warp >= 6 ? 1 : 0) * (BN / 64);
    const int row_in_tile = quarter * 32 + (threadIdx.x & 31);
    uint8_t* stg = smem + C::STAGES * C::STAGE_BYTES + 256 + (warp - 2) * EPI_STAGE_BYTES;
    int lt = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++lt) {
      int pi, z, m0, n0;
      locate(tile, pi, z, m0, n0);
      const int acc = lt & 1;
      const uint32_t use = lt >> 1;
      const uint32_t taddr = tmem_base + acc * BN + ((uint32_t)(quarter * 32) << 16);
      if (!epilogue_tile<BN, A_MN>(
              pi ? g.p[1] : g.p[0], taddr, z, m0 + row_in_tile, n0, c_first, stg,
              [&] { return mbar_wait(&acc_full[acc], use & 1, err, DEV_TIMEOUT_ACC); },
              [&] {
                if (elect_lane0()) mbar_arrive(&acc_empty[acc]);
              }))
        break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ============================================================== tcgen05 engine, K split over a CTA pair
// For the thin products of an adaptive step (1024 rows, N = 2048: 64 tiles of 128 x 256
// for 148 SMs), a cluster of two CTAs computes one 128 x BN tile: CTA r accumulates
// k blocks [r kb/2, (r+1) kb/2) in its own TMEM. Once a CTA's MMAs have completed its
// operand stages are idle; each CTA then writes the half of its partial accumulator
// that the peer finishes into the peer's stages over distributed shared memory, and
// both run the epilogue of their own half of the columns (acc_0 + acc_1 = acc_1 + acc_0
// in fp32: deterministic). The tile count doubles at the operand bytes per FLOP of a
// 128 x BN tile, every MMA is 256 wide, and no global workspace is used. One tile per
// cluster: the grid is exactly two CTAs per tile.
template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(TC_THREADS, 1)
    gemm_tck_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB2, const GemmParams p, int* err) {
  using C = TcCfg<BN>;
  static_assert(TC_BM * BN * 4 <= C::STAGES * C::STAGE_BYTES, "partial tile must fit the operand stages");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                       // [STAGES]
  uint64_t* empty = bars + C::STAGES;          // [STAGES]
  uint64_t* acc_full = bars + 2 * C::STAGES;   // this CTA's MMAs are complete
  uint64_t* part_free = acc_full + 1;          // the peer's stages may be overwritten
  uint64_t* part_full = acc_full + 2;          // the peer's partial is in place (its epilogue threads)
  uint32_t* tmem_slot = (uint32_t*)(acc_full + 3);

  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_ctarank();
  const int m_tiles = (p.M + TC_BM - 1) / TC_BM;
  const int n_tiles = p.N / BN;
  const int tiles_per_batch = m_tiles * n_tiles;
  const int tile = (int)cluster_id_x();
  const int z = tile / tiles_per_batch;
  const int r = tile % tiles_per_batch;
  const int m0 = (p.m_fast ? r % m_tiles : r / n_tiles) * TC_BM;
  const int n0 = (p.m_fast ? r / m_tiles : r % n_tiles) * BN;
  const int kb_one = p.K / TC_BK;
  const int k_half = (p.B2 ? 2 * kb_one : kb_one) / 2;
  const int kb_begin = (int)rank * k_half;
  const int zb_scale = p.sB ? 1 : 0;
  const int zb2_scale = p.sB2 ? 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc_full, 1);
    mbar_init(part_free, 1);
    mbar_init(part_full, TC_EPI_WARPS * 32);
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (p.B2) prefetch_tmap(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // both CTAs' barriers are initialised before either arrives remotely
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (elect_lane0()) {
      for (int i = 0; i < k_half; ++i) {
        const int kb = kb_begin + i;
        const int s = i % C::STAGES;
        const uint32_t round = i / C::STAGES;
        if (!mbar_wait(&empty[s], (round & 1) ^ 1, err, DEV_TIMEOUT_EMPTY)) break;
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        uint8_t* sb = sa + C::A_BYTES;
        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
        const bool second = kb >= kb_one;
        const int k0 = (second ? kb - kb_one : kb) * TC_BK;
        const CUtensorMap* mb = second ? &tmB2 : &tmB;
        const int zb = z * (second ? zb2_scale : zb_scale);
        if (A_MN) {
          tma_load_3d(sa, &tmA, &full[s], m0, k0, z);
          tma_load_3d(sa + 8192, &tmA, &full[s], m0 + 64, k0, z);
        } else {
          tma_load_3d(sa, &tmA, &full[s], k0, m0, z);
        }
        if (B_MN) {
#pragma unroll
          for (int j = 0; j < BN / 64; ++j) tma_load_3d(sb + j * 8192, mb, &full[s], n0 + 64 * j, k0, zb);
        } else {
          tma_load_3d(sb, mb, &full[s], k0, n0, zb);
        }
      }
    }
  } else if (warp == 1) {
    if (elect_lane0()) {
      constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, BN, A_MN, B_MN);
      bool ok = true;
      for (int i = 0; i < k_half; ++i) {
        const int s = i % C::STAGES;
        const uint32_t round = i / C::STAGES;
        if (!mbar_wait(&full[s], round & 1, err, DEV_TIMEOUT_FULL)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
        const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < TC_BK / 16; ++kk) {
          const uint64_t ad = A_MN ? smem_desc_sw128(sa + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(sb + kk * 32, 16, 1024);
          tc_mma_f16(tmem_base, ad, bd, idesc, (i | kk) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      if (ok) tc_commit(acc_full);
    }
  } else {
    // CTA r finishes the columns [r BN/2, (r+1) BN/2) of the tile: it sends its partial
    // accumulator of the other half into the peer's idle operand stages and adds the
    // peer's partial of its own half (a + b = b + a in fp32: the same result on both
    // sides of the pair). Warps 2-5 and 6-9 each take half of every such half.
    constexpr int HALF = BN / 64;  // 32-column chunks per half of the tile
    const int quarter = warp & 3;
    const int grp = warp >= 6 ? 1 : 0;
    const int row = quarter * 32 + (threadIdx.x & 31);
    const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t part = smem_u32(smem);  // the peer's partial of this CTA's half: [128][BN/2] fp32
    uint8_t* stg = smem + C::STAGES * C::STAGE_BYTES + 256 + (warp - 2) * EPI_STAGE_BYTES;
    const int mine0 = (int)rank * HALF, other0 = (1 - (int)rank) * HALF;
    bool ok = mbar_wait(acc_full, 0, err, DEV_TIMEOUT_ACC);
    if (ok) {
      tc_fence_after();
      // this CTA's MMAs are complete, so its stages are free for the peer's partial
      if (warp == 2 && elect_lane0()) mbar_arrive_cluster(mapa_shared(smem_u32(part_free), 1 - rank));
      ok = mbar_wait_cluster(part_free, 0, err, DEV_TIMEOUT_ACC);
    }
    if (ok) {
      const uint32_t peer = mapa_shared(part, 1 - rank);
#pragma unroll 1
      for (int k = 0; k < HALF / 2; ++k) {
        const int c = other0 + grp * (HALF / 2) + k;
        float v[32];
        tmem_ld32(taddr + c * 32, v);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          st_cluster_v4(part_addr<BN / 2>(peer, row, (c - other0) * 8 + i), v[4 * i], v[4 * i + 1], v[4 * i + 2],
                        v[4 * i + 3]);
      }
      mbar_arrive_cluster(mapa_shared(smem_u32(part_full), 1 - rank));
    }
    epilogue_tile<BN / 2, A_MN>(
        p, taddr, z, m0 + row, n0, mine0 + grp * (HALF / 2), stg,
        [&] { return ok && mbar_wait_cluster(part_full, 0, err, DEV_TIMEOUT_ACC); }, [] {}, part, row, mine0);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the peer may still write to or arrive on it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, BN);
  }
}

// ============================================================== tcgen05 engine, CTA pairs
// Pair tile: 256 rows x BN columns, computed by a cluster of two CTAs on two SMs
// with one cta_group::2 MMA stream issued by the even CTA. CTA r of the pair loads
// A rows [m0 + 128 r, +128) and B rows [n0 + r BN/2, +BN/2) into its own shared
// memory; the MMA (M = 256, N = BN) reads both halves and leaves rows [m0 + 128 r,
// +128) of the accumulator, all BN columns, in CTA r's TMEM. Per SM and K step
// that is 128 + BN/2 operand rows for 128 x BN outputs, against 128 + BN for the
// single-CTA tile: 25% (BN = 128) to 33% (BN = 256) less shared-memory and L2
// traffic per FLOP, which the small-M adaptive GEMMs are bound by.
// Barriers: the even CTA's full[s] counts the bytes of both CTAs' loads (their TMA
// completion is signalled there); each MMA commit arrives on empty[s] and acc_full
// of both CTAs; both CTAs' epilogue warps arrive on the even CTA's acc_empty.
template <int BN> struct Tc2Cfg {
  static constexpr int BH = BN / 2;  // B rows loaded per CTA
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BH * TC_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN == 256) ? 6 : 8;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/ +
                              TC_EPI_WARPS * EPI_STAGE_BYTES /*epilogue staging*/;
  static constexpr int TMEM_COLS = 2 * BN;
};

template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(TC_THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB2, const GemmParams p, int* err) {
  using C = Tc2Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                          // [STAGES] (used on the even CTA)
  uint64_t* empty = bars + C::STAGES;             // [STAGES]
  uint64_t* acc_full = bars + 2 * C::STAGES;      // [2]
  uint64_t* acc_empty = bars + 2 * C::STAGES + 2; // [2]   (used on the even CTA)
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * C::STAGES + 4);

  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_ctarank();
  const int pair = (int)cluster_id_x(), npairs = (int)cluster_count_x();
  const int m_tiles = (p.M + 2 * TC_BM - 1) / (2 * TC_BM);
  const int n_tiles = p.N / BN;
  const int tiles_per_batch = m_tiles * n_tiles;
  const int num_tiles = tiles_per_batch * p.batch;
  const int kb_one = p.K / TC_BK;
  const int k_blocks = p.B2 ? 2 * kb_one : kb_one;
  const int zb_scale = p.sB ? 1 : 0;
  const int zb2_scale = p.sB2 ? 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], 2 * TC_EPI_WARPS); }
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (p.B2) prefetch_tmap(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t full0 = mapa_shared(smem_u32(full), 0);
  const uint32_t acc_empty0 = mapa_shared(smem_u32(acc_empty), 0);
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (elect_lane0()) {
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        const int z = tile / tiles_per_batch;
        const int r = tile % tiles_per_batch;
        const int m0 = (p.m_fast ? r % m_tiles : r / n_tiles) * 2 * TC_BM + (int)rank * TC_BM;
        const int n0 = (p.m_fast ? r / m_tiles : r % n_tiles) * BN + (int)rank * C::BH;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t round = it / C::STAGES;
          if (!mbar_wait(&empty[s], (round & 1) ^ 1, err, DEV_TIMEOUT_EMPTY)) { ok = false; break; }
          uint8_t* sa = smem + s * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE_BYTES);
          const uint32_t bar = full0 + 8u * s;
          const bool second = kb >= kb_one;
          const int k0 = (second ? kb - kb_one : kb) * TC_BK;
          const CUtensorMap* mb = second ? &tmB2 : &tmB;
          const int zb = z * (second ? zb2_scale : zb_scale);
          if (A_MN) {
            tma_load_3d_pair(sa, &tmA, bar, m0, k0, z);
            tma_load_3d_pair(sa + 8192, &tmA, bar, m0 + 64, k0, z);
          } else {
            tma_load_3d_pair(sa, &tmA, bar, k0, m0, z);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < C::BH / 64; ++j) tma_load_3d_pair(sb + j * 8192, mb, bar, n0 + 64 * j, k0, zb);
          } else {
            tma_load_3d_pair(sb, mb, bar, k0, n0, zb);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && elect_lane0()) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * TC_BM, BN, A_MN, B_MN);
      int it = 0, lt = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs, ++lt) {
        const int acc = lt & 1;
        const uint32_t use = lt >> 1;
        if (!mbar_wait(&acc_empty[acc], (use & 1) ^ 1, err, DEV_TIMEOUT_ACC)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t round = it / C::STAGES;
          if (!mbar_wait(&full[s], round & 1, err, DEV_TIMEOUT_FULL)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk) {
            const uint64_t ad = A_MN ? smem_desc_sw128(sa + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(sb + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(sb + kk * 32, 16, 1024);
            tc_mma_pair_f16(d_tmem, ad, bd, idesc, (kb | kk) ? 1u : 0u);
          }
          tc_commit_pair(&empty[s], 3);
        }
        if (!ok) break;
        tc_commit_pair(&acc_full[acc], 3);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int c_first = (warp >= 6 ? 1 : 0) * (BN / 64);
    const int row_in_tile = quarter * 32 + (threadIdx.x & 31);
    uint8_t* stg = smem + C::STAGES * C::STAGE_BYTES + 256 + (warp - 2) * EPI_STAGE_BYTES;
    int lt = 0;
    for (int tile = pair; tile < num_tiles; tile += npairs, ++lt) {
      const int z = tile / tiles_per_batch;
      const int r = tile % tiles_per_batch;
      const int m0 = (p.m_fast ? r % m_tiles : r / n_tiles) * 2 * TC_BM + (int)rank * TC_BM;
      const int n0 = (p.m_fast ? r / m_tiles : r % n_tiles) * BN;
      const int acc = lt & 1;
      const uint32_t use = lt >> 1;
      const uint32_t taddr = tmem_base + acc * BN + ((uint32_t)(quarter * 32) << 16);
      if (!epilogue_tile<BN, A_MN>(
              p, taddr, z, m0 + row_in_tile, n0, c_first, stg,
              [&] { return mbar_wait(&acc_full[acc], use & 1, err, DEV_TIMEOUT_ACC); },
              [&] {
                if (elect_lane0()) mbar_arrive_cluster(acc_empty0 + 8u * acc);
              }))
        break;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair's MMAs or arrivals may still touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ============================================================== host side
enum GemmEngine : int { GEMM_AUTO = 0, GEMM_SIMT = 1, GEMM_TC1 = 3 };
int gemm_launch(const GemmParams& p, int elem_is_bf16, cudaStream_t stream, int* err, int num_sms, int engine);
// Two independent products, in one launch where they can share it (same engine, operand
// layouts and tile width); 0 or a cudaError_t.
int gemm_launch_pair(const GemmParams& a, const GemmParams& b, int elem_is_bf16, cudaStream_t stream, int* err,
                     int num_sms);
// Whether gemm_launch would run p on the tcgen05 engine (EPI_CE requires it).
bool gemm_uses_tc(const GemmParams& p, int elem_is_bf16);
// Sets the dynamic shared-memory limits of all large-smem kernels; 0 or a cudaError_t.
int prime_kernel_attributes();
struct AttnParams;
bool attn_tc_ok(const AttnParams& p);
cudaError_t attn_fwd_tc_launch(const AttnParams& p, cudaStream_t st, int* err, bool* ok);
bool attn_dq_tc_ok(const AttnParams& p);
cudaError_t attn_bwd_dq_tc_launch(const AttnParams& p, cudaStream_t st, int* err, bool* ok);
bool attn_dkv_tc_ok(const AttnParams& p);
cudaError_t attn_bwd_dkv_tc_launch(const AttnParams& p, cudaStream_t st, int* err, bool* ok);

}  // namespace ttt
