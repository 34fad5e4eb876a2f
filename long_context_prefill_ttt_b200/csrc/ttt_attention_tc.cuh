// Sliding-window attention forward on tcgen05 tensor cores (bf16 in, fp32 softmax
// and accumulation), for the frozen-phase prefill and the adaptive chunks.
//
// One CTA = 128 queries of one (sequence, head); key tiles of 128 positions,
// 128-aligned in absolute position, each taken whole from the ring (positions
// < q0) or from the current rows (the q|k|v buffer). Warp roles:
//   warp 0     TMA: Q once, then K and V tiles into separate rings (a K stage is
//              freed as soon as its Q K^T is done, a V stage after its P V);
//   warp 1     MMA issue (one thread): S_j = Q K_j^T into one of two TMEM S
//              buffers, then O += P_{j-1} V_{j-1} (P read from TMEM as the A
//              operand, V as an MN-major operand) into the TMEM O accumulator;
//              the completion of P_j V_j frees S buffer j % 2 for S_{j+2};
//   warps 2-5  softmax, one thread per query row (TMEM lane): read S_j, mask on
//              diagonal / window-edge tiles, online softmax in the log2 domain,
//              write P_j (bf16 pairs) over the scores in S_j's TMEM columns. The
//              running maximum is raised only when a row's
//              maximum grows by more than 8 (a factor 256): then the thread's O
//              row is rescaled in TMEM after the previous P·V has completed.
//              Exponents stay below 2^8, so bf16 P and fp32 sums stay exact
//              enough, and O and l always share the same reference maximum.
// The softmax warps first copy their rows of Q from shared memory into TMEM, where the
// S MMAs take them as the A operand (the MMA then reads only the K tile from shared
// memory).
// TMEM: S0 columns [0,128), S1 [128,256), O [256, 256+HD), Q [384, 384+HD/2); 512 allocated.
// Every mbarrier wait is time-bounded and records an error instead of hanging.
#pragma once

#include "ttt_attention.cuh"
#include "ttt_common.cuh"

namespace ttt {

template <int HD> struct AttnTcCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int KST = HD == 64 ? 3 : 2;  // K stages (a third at HD = 128 measured 1% slower)
  static constexpr int VST = HD == 64 ? 3 : 2;  // V stages
  static constexpr int QB = BM * HD * 2;      // Q tile bytes
  static constexpr int KVB = BN * HD * 2;     // K (and V) tile bytes
  static constexpr int OFF_K0 = QB;
  static constexpr int OFF_V0 = OFF_K0 + KST * KVB;
  static constexpr int OFF_BAR = OFF_V0 + VST * KVB;  // P lives in TMEM
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t S_COL = 0, O_COL = 256;
  static constexpr uint32_t Q_COL = 384;  // Q as the A operand of S, copied once into TMEM
};

__device__ __forceinline__ bool warp_any(bool v) { return __any_sync(0xffffffffu, v); }
__device__ __forceinline__ float ex2_tc(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int HD>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_rk,
                       const __grid_constant__ CUtensorMap tm_rv, const AttnParams p, int* err) {
  using Cf = AttnTcCfg<HD>;
  constexpr int KB = HD / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + Cf::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;     // [3]
  uint64_t* k_empty = bars + 4;    // [3]
  uint64_t* v_full = bars + 7;     // [3]
  uint64_t* v_empty = bars + 10;   // [3]
  uint64_t* s_full = bars + 13;    // [2]
  uint64_t* s_free = bars + 15;    // [2]
  uint64_t* p_full = bars + 17;    // [2]
  uint64_t* pv_done = bars + 19;   // [2]
  uint64_t* o_done = bars + 21;
  uint64_t* qt_full = bars + 22;   // Q is in TMEM (4 warps)
  uint32_t* tmem_slot = (uint32_t*)(bars + 23);

  const int warp = threadIdx.x >> 5;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int i0 = qb * Cf::BM;
  const int64_t P0 = p.q0 + i0;
  const int nq = min(Cf::BM, p.n - i0);
  const int64_t Plast = P0 + nq - 1;
  const int64_t jlo = max((int64_t)0, P0 - p.window + 1);
  const int64_t jt0 = (jlo / Cf::BN) * Cf::BN;
  const int ntiles = (int)((Plast / Cf::BN) * Cf::BN - jt0) / Cf::BN + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);  mbar_init(&s_free[s], 1);
      mbar_init(&p_full[s], 4);  mbar_init(&pv_done[s], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(qt_full, 4);
    fence_mbar_init();
    prefetch_tmap(&tm_qkv);
    prefetch_tmap(&tm_rk);
    prefetch_tmap(&tm_rv);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (elect_lane0()) {
      const int qrow = b * p.n + i0;
      mbar_arrive_expect_tx(q_full, Cf::QB);
      for (int kb = 0; kb < KB; ++kb) tma_load_3d(sm + kb * Cf::BM * 128, &tm_qkv, q_full, h * HD + kb * 64, qrow, 0);
      // K runs up to KST tiles ahead of its use; V up to VST tiles. K_j is issued
      // before V_j, and K_{j+1} before V_j when its stage is free, so that the
      // next Q K^T never waits behind a P V.
      int jk = 0, jv = 0;
      bool ok = true;
      auto load = [&](bool isK, int j) -> bool {
        const int st = isK ? j % Cf::KST : j % Cf::VST;
        const int use = isK ? j / Cf::KST : j / Cf::VST;
        uint64_t* emp = isK ? &k_empty[st] : &v_empty[st];
        uint64_t* ful = isK ? &k_full[st] : &v_full[st];
        if (!mbar_wait(emp, (use & 1) ^ 1, err, DEV_TIMEOUT_EMPTY)) return false;
        uint8_t* dst = sm + (isK ? Cf::OFF_K0 : Cf::OFF_V0) + st * Cf::KVB;
        mbar_arrive_expect_tx(ful, Cf::KVB);
        const int64_t j0 = jt0 + (int64_t)j * Cf::BN;
        if (j0 >= p.q0) {
          const int y = b * p.n + (int)(j0 - p.q0);
          const int x0 = (isK ? p.d : 2 * p.d) + h * HD;
          for (int kb = 0; kb < KB; ++kb) tma_load_3d(dst + kb * Cf::BN * 128, &tm_qkv, ful, x0 + kb * 64, y, 0);
        } else {
          const int y = b * p.C + (int)(j0 % p.C);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(dst + kb * Cf::BN * 128, isK ? &tm_rk : &tm_rv, ful, h * HD + kb * 64, y, 0);
        }
        return true;
      };
      while (ok && (jk < ntiles || jv < ntiles)) {
        if (jk < ntiles && jk <= jv + 1) {
          ok = load(true, jk++);
        } else {
          ok = load(false, jv++);
        }
      }
    }
  } else if (warp == 1) {
    if (elect_lane0()) {
      constexpr uint32_t idS = idesc_bf16_f32(128, Cf::BN, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, HD, false, true);
      bool ok = mbar_wait(qt_full, 0, err, DEV_TIMEOUT_FULL);
      tc_fence_after();
      auto issue_pv = [&](int i) -> bool {
        const int s = i & 1;
        const int vs = i % Cf::VST;
        if (!mbar_wait(&v_full[vs], (i / Cf::VST) & 1, err, DEV_TIMEOUT_FULL)) return false;
        if (!mbar_wait(&p_full[s], (i >> 1) & 1, err, DEV_TIMEOUT_FULL)) return false;
        tc_fence_after();
        const uint32_t sV = smem_u32(sm + Cf::OFF_V0 + vs * Cf::KVB);
#pragma unroll
        for (int kk = 0; kk < Cf::BN / 16; ++kk) {  // A = P_i from TMEM (in the columns of S_i)
          const uint64_t bd = smem_desc_sw128(sV + kk * 2048, Cf::BN * 128, 1024);
          tc_mma_f16_ta(tmem + Cf::O_COL, tmem + Cf::S_COL + s * Cf::BN + kk * 8, bd, idO, (i | kk) ? 1u : 0u);
        }
        tc_commit(&pv_done[s]);
        tc_commit(&s_free[s]);  // P_i is consumed: S_{i+2} may overwrite the buffer
        tc_commit(&v_empty[vs]);
        return true;
      };
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j & 1;
        const int ks = j % Cf::KST;
        if (!mbar_wait(&k_full[ks], (j / Cf::KST) & 1, err, DEV_TIMEOUT_FULL)) { ok = false; break; }
        if (!mbar_wait(&s_free[s], ((j >> 1) & 1) ^ 1, err, DEV_TIMEOUT_ACC)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sK = smem_u32(sm + Cf::OFF_K0 + ks * Cf::KVB);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t bd = smem_desc_sw128(sK + (kk >> 2) * (Cf::BN * 128) + (kk & 3) * 32, 16, 1024);
          tc_mma_f16_ta(tmem + Cf::S_COL + s * Cf::BN, tmem + Cf::Q_COL + kk * 8, bd, idS, kk ? 1u : 0u);
        }
        tc_commit(&s_full[s]);
        tc_commit(&k_empty[ks]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(ntiles - 1);
      if (ok) tc_commit(o_done);
    }
  } else {
    // softmax warps: TMEM lane quarter = warp % 4, one query row per thread
    const int quarter = warp & 3;
    const int lane = threadIdx.x & 31;
    const int r = quarter * 32 + lane;
    const int64_t P = P0 + r;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float sc = p.scale * 1.4426950408889634f;
    float m_used = -INFINITY, l = 0.f;
    bool ok = mbar_wait(q_full, 0, err, DEV_TIMEOUT_FULL);
    if (ok) {
      // this row of Q: shared memory (128-byte swizzled) -> TMEM, bf16 pairs in K order
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) {
        float w[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 a = *(const uint4*)(sm + kb * Cf::BM * 128 + r * 128 + ((c ^ (r & 7)) << 4));
          w[4 * c] = __uint_as_float(a.x); w[4 * c + 1] = __uint_as_float(a.y);
          w[4 * c + 2] = __uint_as_float(a.z); w[4 * c + 3] = __uint_as_float(a.w);
        }
        tmem_st32(tmem + lane_base + Cf::Q_COL + kb * 32, w);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qt_full);
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      const int s = j & 1;
      const int64_t j0 = jt0 + (int64_t)j * Cf::BN;
      if (!mbar_wait(&s_full[s], (j >> 1) & 1, err, DEV_TIMEOUT_ACC)) { ok = false; break; }
      tc_fence_after();
      float v[Cf::BN];
      {
        uint32_t* vr = reinterpret_cast<uint32_t*>(v);
#pragma unroll
        for (int c = 0; c < Cf::BN / 32; ++c)
          tmem_ld32_nowait(tmem + lane_base + Cf::S_COL + s * Cf::BN + c * 32, vr + c * 32);
        tmem_ld_wait();
      }
      const bool need_mask = (j0 + Cf::BN - 1 > P0) || (j0 < Plast - p.window + 1);
      if (need_mask) {  // diagonal / window-edge tile: branch-free per-element mask
        const int64_t lo_key = P - p.window + 1;
        const uint32_t span = (uint32_t)(P - lo_key);
#pragma unroll
        for (int c = 0; c < Cf::BN; ++c) {
          const uint32_t off = (uint32_t)(j0 + c - lo_key);
          v[c] = off <= span ? v[c] : -INFINITY;
        }
      }
      // row maximum of the raw scores, eight independent chains
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = v[e];
#pragma unroll
      for (int c = 8; c < Cf::BN; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], v[c]);
      float mt = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      mt *= sc;  // scores are compared in the scaled log2 domain (sc > 0 keeps the order)
      // lazily raised reference maximum
      const bool first = m_used == -INFINITY;
      const bool raise = mt > m_used + 8.f;
      float factor = 1.f;
      if (raise) {
        if (!first) factor = ex2_tc(m_used - mt);
        m_used = mt;
      }
      if (j >= 1 && warp_any(raise && !first)) {
        // O holds P_0..P_{j-1} V: wait for the last of them, then rescale this warp's rows
        if (!mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, err, DEV_TIMEOUT_ACC)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_base + Cf::O_COL + c * 32, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= factor;
          tmem_st32(tmem + lane_base + Cf::O_COL + c * 32, o);
        }
      }
      l *= factor;
      // P_j (bf16 pairs in key order) into the first BN/2 columns of S_j's TMEM buffer,
      // whose scores are all in registers: the P·V MMA takes it as its A operand
      const float nbase = m_used == -INFINITY ? 0.f : -m_used;
      float ls8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kb = 0; kb < Cf::BN / 64; ++kb) {
        float pw[32];  // 64 P values of this row as 32 bf16 pairs
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          float e8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            e8[e] = ex2_tc(fmaf(v[kb * 64 + cc * 8 + e], sc, nbase));  // exp2(s*sc - m): masked -inf -> 0
            ls8[e] += e8[e];
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) pw[cc * 4 + e] = __uint_as_float(pack_bf16x2(e8[2 * e], e8[2 * e + 1]));
        }
        tmem_st32(tmem + lane_base + Cf::S_COL + s * Cf::BN + kb * 32, pw);
      }
      l += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
      tc_fence_before();  // P_j's TMEM stores (waited for) before the MMA warp's P·V
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[s]);
    }
    if (ok && mbar_wait(o_done, 0, err, DEV_TIMEOUT_ACC)) {
      tc_fence_after();
      const float inv = 1.f / l;
      bf16* O = (bf16*)p.O + ((int64_t)b * p.n + i0 + r) * p.ldo + h * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_base + Cf::O_COL + c * 32, o);
        if (r < nq) {
          uint4* dst = (uint4*)(O + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv), pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
        }
      }
      if (r < nq && p.lse) p.lse[((int64_t)b * p.H + h) * p.n + i0 + r] = (m_used + __log2f(l)) * 0.6931471805599453f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- backward dQ on tcgen05
// One CTA = 128 query rows of one (sequence, head), key tiles of 64 positions over
// each row's whole window (ring and current rows). Per tile j: S = Q K^T and
// dP = dO V^T into one of two TMEM buffers (MMA warp); four warps form
// dS = P (dP - D) with P = exp(S*scale - lse) from the forward's log-sum-exp and
// write dS (bf16 pairs) over the scores in the buffer's S columns; the MMA warp
// accumulates dQ += dS K in TMEM (dS as the A operand from TMEM, the K tile read again
// as an MN-major operand), and its completion frees the buffer for tile j+2. With two
// buffers, S_{j+1} and dP_{j+1} run on the tensor cores while the warps form dS_j. dQ is scaled by 1/sqrt(hd) on the way out. The four warps first
// copy their rows of Q and dO from shared memory into TMEM, where the S and dP MMAs
// take them as the A operand.
// TMEM: S0 [0,64), dP0 [64,128), S1 [128,192), dP1 [192,256), dQ [256, 256+HD),
// Q [384, 384+HD/2), dO [448, 448+HD/2).
template <int HD> struct AttnDqCfg {
  static constexpr int BM = 128, BN = 64;
  static constexpr int KST = 3, VST = 3;
  static constexpr int QB = BM * HD * 2;
  static constexpr int KVB = BN * HD * 2;
  static constexpr int OFF_DO = QB;
  static constexpr int OFF_K0 = 2 * QB;
  static constexpr int OFF_V0 = OFF_K0 + KST * KVB;
  static constexpr int OFF_BAR = OFF_V0 + VST * KVB;  // dS lives in TMEM
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t DQ_COL = 256;
  // Q and dO as the A operands of S and dP, copied once into TMEM (bf16 pairs, one row
  // per lane): the MMAs then read only their 64-key B tile from shared memory
  static constexpr uint32_t Q_COL = 384, DO_COL = 448;
  static __device__ __forceinline__ uint32_t s_col(int b) { return b * 128; }
  static __device__ __forceinline__ uint32_t dp_col(int b) { return b * 128 + 64; }
};

template <int HD>
__global__ void __launch_bounds__(192, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                          const __grid_constant__ CUtensorMap tm_rk, const __grid_constant__ CUtensorMap tm_rv,
                          const __grid_constant__ CUtensorMap tm_do, const AttnParams p, int* err) {
  using Cf = AttnDqCfg<HD>;
  constexpr int KB = HD / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + Cf::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;     // [3]
  uint64_t* k_empty = bars + 4;    // [3]
  uint64_t* v_full = bars + 7;     // [3]
  uint64_t* v_empty = bars + 10;   // [3]
  uint64_t* sp_full = bars + 13;   // [2]
  uint64_t* sp_free = bars + 15;   // [2]
  uint64_t* ds_full = bars + 17;   // [2]
  uint64_t* ds_free = bars + 19;   // [2]
  uint64_t* dq_done = bars + 21;
  uint64_t* qt_full = bars + 22;   // Q and dO are in TMEM (4 warps)
  uint32_t* tmem_slot = (uint32_t*)(bars + 23);

  const int warp = threadIdx.x >> 5;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int i0 = qb * Cf::BM;
  const int64_t P0 = p.q0 + i0;
  const int nq = min(Cf::BM, p.n - i0);
  const int64_t Plast = P0 + nq - 1;
  const int64_t jlo = max((int64_t)0, P0 - p.window + 1);
  const int64_t jt0 = (jlo / Cf::BN) * Cf::BN;
  const int ntiles = (int)((Plast / Cf::BN) * Cf::BN - jt0) / Cf::BN + 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sp_full[s], 1); mbar_init(&sp_free[s], 1);
      mbar_init(&ds_full[s], 4); mbar_init(&ds_free[s], 1);
    }
    mbar_init(dq_done, 1);
    mbar_init(qt_full, 4);
    fence_mbar_init();
    prefetch_tmap(&tm_q); prefetch_tmap(&tm_kv); prefetch_tmap(&tm_rk); prefetch_tmap(&tm_rv); prefetch_tmap(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (elect_lane0()) {
      const int qrow = b * p.n + i0;
      mbar_arrive_expect_tx(q_full, 2 * Cf::QB);
      for (int kb = 0; kb < KB; ++kb) {
        tma_load_3d(sm + kb * Cf::BM * 128, &tm_q, q_full, h * HD + kb * 64, qrow, 0);
        tma_load_3d(sm + Cf::OFF_DO + kb * Cf::BM * 128, &tm_do, q_full, h * HD + kb * 64, qrow, 0);
      }
      auto load = [&](bool isK, int j) -> bool {
        const int st = j % 3;
        const int use = j / 3;
        uint64_t* emp = isK ? &k_empty[st] : &v_empty[st];
        uint64_t* ful = isK ? &k_full[st] : &v_full[st];
        if (!mbar_wait(emp, (use & 1) ^ 1, err, DEV_TIMEOUT_EMPTY)) return false;
        uint8_t* dst = sm + (isK ? Cf::OFF_K0 : Cf::OFF_V0) + st * Cf::KVB;
        mbar_arrive_expect_tx(ful, Cf::KVB);
        const int64_t j0 = jt0 + (int64_t)j * Cf::BN;
        if (j0 >= p.q0) {
          const int y = b * p.n + (int)(j0 - p.q0);
          const int x0 = (isK ? p.d : 2 * p.d) + h * HD;
          for (int kb = 0; kb < KB; ++kb) tma_load_3d(dst + kb * Cf::BN * 128, &tm_kv, ful, x0 + kb * 64, y, 0);
        } else {
          const int y = b * p.C + (int)(j0 % p.C);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(dst + kb * Cf::BN * 128, isK ? &tm_rk : &tm_rv, ful, h * HD + kb * 64, y, 0);
        }
        return true;
      };
      for (int j = 0; j < ntiles; ++j)
        if (!load(true, j) || !load(false, j)) break;
    }
  } else if (warp == 1) {
    if (elect_lane0()) {
      constexpr uint32_t idS = idesc_bf16_f32(128, Cf::BN, false, false);
      constexpr uint32_t idQ = idesc_bf16_f32(128, HD, false, true);
      bool ok = mbar_wait(qt_full, 0, err, DEV_TIMEOUT_FULL);
      tc_fence_after();
      auto issue_dq = [&](int i) -> bool {
        const int s = i & 1, ks = i % 3;
        if (!mbar_wait(&ds_full[s], (i >> 1) & 1, err, DEV_TIMEOUT_FULL)) return false;
        tc_fence_after();
        const uint32_t sK = smem_u32(sm + Cf::OFF_K0 + ks * Cf::KVB);
#pragma unroll
        for (int kk = 0; kk < Cf::BN / 16; ++kk) {  // A = dS_i from TMEM (in the columns of S_i)
          const uint64_t bd = smem_desc_sw128(sK + kk * 2048, Cf::BN * 128, 1024);
          tc_mma_f16_ta(tmem + Cf::DQ_COL, tmem + Cf::s_col(s) + kk * 8, bd, idQ, (i | kk) ? 1u : 0u);
        }
        tc_commit(&sp_free[s]);  // dS_i is consumed: S_{i+2} and dP_{i+2} may overwrite the buffer
        tc_commit(&k_empty[ks]);
        return true;
      };
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j & 1, ks = j % 3, vs = j % 3;
        if (!mbar_wait(&k_full[ks], (j / 3) & 1, err, DEV_TIMEOUT_FULL) ||
            !mbar_wait(&v_full[vs], (j / 3) & 1, err, DEV_TIMEOUT_FULL) ||
            !mbar_wait(&sp_free[s], ((j >> 1) & 1) ^ 1, err, DEV_TIMEOUT_ACC)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sK = smem_u32(sm + Cf::OFF_K0 + ks * Cf::KVB);
        const uint32_t sV = smem_u32(sm + Cf::OFF_V0 + vs * Cf::KVB);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t offb = (kk >> 2) * (Cf::BN * 128) + (kk & 3) * 32;
          tc_mma_f16_ta(tmem + Cf::s_col(s), tmem + Cf::Q_COL + kk * 8, smem_desc_sw128(sK + offb, 16, 1024), idS,
                        kk ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t offb = (kk >> 2) * (Cf::BN * 128) + (kk & 3) * 32;
          tc_mma_f16_ta(tmem + Cf::dp_col(s), tmem + Cf::DO_COL + kk * 8, smem_desc_sw128(sV + offb, 16, 1024), idS,
                        kk ? 1u : 0u);
        }
        tc_commit(&sp_full[s]);
        tc_commit(&v_empty[vs]);
        if (j >= 1 && !issue_dq(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_dq(ntiles - 1);
      if (ok) tc_commit(dq_done);
    }
  } else {
    const int quarter = warp & 3;
    const int lane = threadIdx.x & 31;
    const int r = quarter * 32 + lane;
    const int64_t P = P0 + r;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float sc = p.scale * 1.4426950408889634f;
    const int64_t si = ((int64_t)b * p.H + h) * p.n + i0 + r;
    const float nL = r < nq ? -p.lse[si] * 1.4426950408889634f : -INFINITY;  // exp2(s*sc - lse*log2e)
    const int64_t lo_key = P - p.window + 1;
    const uint32_t span = (uint32_t)(P - lo_key);
    float Dr = 0.f;
    bool ok = mbar_wait(q_full, 0, err, DEV_TIMEOUT_FULL);
    if (ok) {
      // this row of Q and of dO: shared memory (128-byte swizzled) -> TMEM, as bf16 pairs in K order
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint8_t* src = sm + (t ? Cf::OFF_DO : 0);
        const uint32_t col = t ? Cf::DO_COL : Cf::Q_COL;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
          float w[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 a = *(const uint4*)(src + kb * Cf::BM * 128 + r * 128 + ((c ^ (r & 7)) << 4));
            w[4 * c] = __uint_as_float(a.x); w[4 * c + 1] = __uint_as_float(a.y);
            w[4 * c + 2] = __uint_as_float(a.z); w[4 * c + 3] = __uint_as_float(a.w);
          }
          tmem_st32(tmem + lane_base + col + kb * 32, w);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qt_full);
    }
    if (p.dsum_in_dq) {
      // D = rowsum(dO * O) of this row and head, from the staged dO tile and O; the
      // dK/dV kernel that follows reads it from Dsum
      if (ok && r < nq) {
        const bf16* Orow = (const bf16*)p.O + ((int64_t)b * p.n + i0 + r) * p.ldo + h * HD;
        float acc = 0.f;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 a = *(const uint4*)(sm + Cf::OFF_DO + kb * Cf::BM * 128 + r * 128 + ((c ^ (r & 7)) << 4));
            const uint4 o = *(const uint4*)(Orow + kb * 64 + c * 8);
            const bf16* ae = reinterpret_cast<const bf16*>(&a);
            const bf16* oe = reinterpret_cast<const bf16*>(&o);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc = fmaf(__bfloat162float(ae[e]), __bfloat162float(oe[e]), acc);
          }
        }
        Dr = acc;
        p.Dsum[si] = Dr;
      }
    } else {
      Dr = r < nq ? p.Dsum[si] : 0.f;
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      const int s = j & 1;
      const int64_t j0 = jt0 + (int64_t)j * Cf::BN;
      const bool need_mask = (j0 + Cf::BN - 1 > P0) || (j0 < Plast - p.window + 1);
      if (!mbar_wait(&sp_full[s], (j >> 1) & 1, err, DEV_TIMEOUT_ACC)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[64], dr[64];
      tmem_ld32_nowait(tmem + lane_base + Cf::s_col(s), sr);
      tmem_ld32_nowait(tmem + lane_base + Cf::s_col(s) + 32, sr + 32);
      tmem_ld32_nowait(tmem + lane_base + Cf::dp_col(s), dr);
      tmem_ld32_nowait(tmem + lane_base + Cf::dp_col(s) + 32, dr + 32);
      tmem_ld_wait();
      // dS_j (bf16 pairs in key order) over the scores in the first BN/2 columns of S_j
      float dsw[Cf::BN / 2];
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        float ds[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = cc * 8 + e;
          float pr = ex2_tc(fmaf(__uint_as_float(sr[c]), sc, nL));
          if (need_mask) {
            const uint32_t off = (uint32_t)(j0 + c - lo_key);
            pr = off <= span ? pr : 0.f;
          }
          ds[e] = pr * (__uint_as_float(dr[c]) - Dr);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) dsw[cc * 4 + e] = __uint_as_float(pack_bf16x2(ds[2 * e], ds[2 * e + 1]));
      }
      tmem_st32(tmem + lane_base + Cf::s_col(s), dsw);
      tc_fence_before();  // dS_j's TMEM stores (waited for) before the MMA warp's dQ product
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full[s]);
    }
    if (ok && mbar_wait(dq_done, 0, err, DEV_TIMEOUT_ACC)) {
      tc_fence_after();
      bf16* dQ = (bf16*)p.dQ + ((int64_t)b * p.n + i0 + r) * p.lddq + h * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_base + Cf::DQ_COL + c * 32, o);
        if (r < nq) {
          uint4* dst = (uint4*)(dQ + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(o[8 * q] * p.scale, o[8 * q + 1] * p.scale),
                                pack_bf16x2(o[8 * q + 2] * p.scale, o[8 * q + 3] * p.scale),
                                pack_bf16x2(o[8 * q + 4] * p.scale, o[8 * q + 5] * p.scale),
                                pack_bf16x2(o[8 * q + 6] * p.scale, o[8 * q + 7] * p.scale));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// ---------------------------------------------------------------- backward dK, dV on tcgen05
// Keys of the current rows only (cached ring keys are constants of the chunk
// step): one CTA = 128 keys of one (sequence, head) at row offsets [k0, k0+128),
// over the query blocks of 64 rows that can see them (query i sees key j when
// 0 <= i - j < window). The roles mirror the dQ kernel with keys as the MMA's M
// dimension. Per query block j: S^T = K Q_j^T and dP^T = V dO_j^T into one of two
// TMEM buffers (MMA warp); four warps (one key row each) form P^T = exp(S^T*scale
// - lse) and dS^T = P^T (dP^T - D) with the per-query lse and D read from shared
// memory, and write both (bf16 pairs) over S^T and dP^T in TMEM; the MMA warp
// accumulates dV += P^T dO_j and dK += dS^T Q_j in TMEM (P^T and dS^T as A operands
// from TMEM, Q_j and dO_j read again as MN-major operands), and its completion frees
// the buffer for block j+2. Query rows past the sequence end get lse = +inf, so their
// P and dS vanish. dK is scaled by 1/sqrt(hd) on the way out.
// TMEM: dV [0,HD), dK [128,128+HD), S^T_b [256+128b, 256+128b+64), dP^T_b next 64.
template <int HD> struct AttnDkvCfg {
  static constexpr int BK = 128, BQ = 64;
  static constexpr int QST = 3;                 // Q / dO stages
  static constexpr int KVB = BK * HD * 2;       // K (and V) tile bytes
  static constexpr int QB = BQ * HD * 2;        // Q (and dO) block bytes
  static constexpr int OFF_V = KVB;
  static constexpr int OFF_Q0 = 2 * KVB;
  static constexpr int OFF_DO0 = OFF_Q0 + QST * QB;
  static constexpr int OFF_LD = OFF_DO0 + QST * QB;  // [2][ -lse*log2e (64) | D (64) ] floats (P^T, dS^T in TMEM)
  static constexpr int OFF_BAR = OFF_LD + 2 * 2 * BQ * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t DV_COL = 0, DK_COL = 128;
  static __device__ __forceinline__ uint32_t s_col(int b) { return 256 + b * 128; }
  static __device__ __forceinline__ uint32_t dp_col(int b) { return 256 + b * 128 + 64; }
};

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <int HD>
__global__ void __launch_bounds__(192, 1)
    attn_bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_do, const AttnParams p, int* err) {
  using Cf = AttnDkvCfg<HD>;
  constexpr int KB = HD / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(sm + Cf::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;     // [3]
  uint64_t* q_empty = bars + 4;    // [3]
  uint64_t* sp_full = bars + 7;    // [2]
  uint64_t* sp_free = bars + 9;    // [2]
  uint64_t* pd_full = bars + 11;   // [2]
  uint64_t* pd_free = bars + 13;   // [2]
  uint64_t* acc_done = bars + 15;
  uint32_t* tmem_slot = (uint32_t*)(bars + 16);
  float* ldbuf = (float*)(sm + Cf::OFF_LD);

  const int warp = threadIdx.x >> 5;
  const int kblk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int k0 = kblk * Cf::BK;                       // first key row (offset within the rows)
  const int nk = min(Cf::BK, p.n - k0);
  const int qlast = (int)min((int64_t)p.n - 1, (int64_t)k0 + Cf::BK - 1 + p.window - 1);
  const int qb0 = k0 / Cf::BQ;
  const int nqb = qlast / Cf::BQ - qb0 + 1;           // >= 1: the key block's own rows see it

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < Cf::QST; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sp_full[s], 1); mbar_init(&sp_free[s], 1);
      mbar_init(&pd_full[s], 4); mbar_init(&pd_free[s], 1);
    }
    mbar_init(acc_done, 1);
    fence_mbar_init();
    prefetch_tmap(&tm_k); prefetch_tmap(&tm_q); prefetch_tmap(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (elect_lane0()) {
      const int krow = b * p.n + k0;
      mbar_arrive_expect_tx(kv_full, 2 * Cf::KVB);
      for (int kb = 0; kb < KB; ++kb) {
        tma_load_3d(sm + kb * Cf::BK * 128, &tm_k, kv_full, p.d + h * HD + kb * 64, krow, 0);
        tma_load_3d(sm + Cf::OFF_V + kb * Cf::BK * 128, &tm_k, kv_full, 2 * p.d + h * HD + kb * 64, krow, 0);
      }
      for (int j = 0; j < nqb; ++j) {
        const int st = j % Cf::QST, use = j / Cf::QST;
        if (!mbar_wait(&q_empty[st], (use & 1) ^ 1, err, DEV_TIMEOUT_EMPTY)) break;
        mbar_arrive_expect_tx(&q_full[st], 2 * Cf::QB);
        const int qrow = b * p.n + (qb0 + j) * Cf::BQ;
        for (int kb = 0; kb < KB; ++kb) {
          tma_load_3d(sm + Cf::OFF_Q0 + st * Cf::QB + kb * Cf::BQ * 128, &tm_q, &q_full[st], h * HD + kb * 64, qrow, 0);
          tma_load_3d(sm + Cf::OFF_DO0 + st * Cf::QB + kb * Cf::BQ * 128, &tm_do, &q_full[st], h * HD + kb * 64, qrow,
                      0);
        }
      }
    }
  } else if (warp == 1) {
    if (elect_lane0()) {
      constexpr uint32_t idS = idesc_bf16_f32(128, Cf::BQ, false, false);
      constexpr uint32_t idA = idesc_bf16_f32(128, HD, false, true);
      const uint32_t sK = smem_u32(sm), sV = smem_u32(sm + Cf::OFF_V);
      bool ok = mbar_wait(kv_full, 0, err, DEV_TIMEOUT_FULL);
      auto issue_acc = [&](int i) -> bool {
        const int s = i & 1, qs = i % Cf::QST;
        if (!mbar_wait(&pd_full[s], (i >> 1) & 1, err, DEV_TIMEOUT_FULL)) return false;
        tc_fence_after();
        const uint32_t sQ = smem_u32(sm + Cf::OFF_Q0 + qs * Cf::QB), sdO = smem_u32(sm + Cf::OFF_DO0 + qs * Cf::QB);
#pragma unroll
        for (int kk = 0; kk < Cf::BQ / 16; ++kk) {  // A = P^T and dS^T from TMEM (over S^T and dP^T)
          tc_mma_f16_ta(tmem + Cf::DV_COL, tmem + Cf::s_col(s) + kk * 8,
                        smem_desc_sw128(sdO + kk * 2048, Cf::BQ * 128, 1024), idA, (i | kk) ? 1u : 0u);
          tc_mma_f16_ta(tmem + Cf::DK_COL, tmem + Cf::dp_col(s) + kk * 8,
                        smem_desc_sw128(sQ + kk * 2048, Cf::BQ * 128, 1024), idA, (i | kk) ? 1u : 0u);
        }
        tc_commit(&sp_free[s]);  // P^T and dS^T are consumed: block i+2 may overwrite the buffer
        tc_commit(&q_empty[qs]);
        return true;
      };
      for (int j = 0; j < nqb && ok; ++j) {
        const int s = j & 1, qs = j % Cf::QST;
        if (!mbar_wait(&q_full[qs], (j / Cf::QST) & 1, err, DEV_TIMEOUT_FULL) ||
            !mbar_wait(&sp_free[s], ((j >> 1) & 1) ^ 1, err, DEV_TIMEOUT_ACC)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sQ = smem_u32(sm + Cf::OFF_Q0 + qs * Cf::QB), sdO = smem_u32(sm + Cf::OFF_DO0 + qs * Cf::QB);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t offa = (kk >> 2) * (Cf::BK * 128) + (kk & 3) * 32;
          const uint32_t offb = (kk >> 2) * (Cf::BQ * 128) + (kk & 3) * 32;
          tc_mma_f16(tmem + Cf::s_col(s), smem_desc_sw128(sK + offa, 16, 1024), smem_desc_sw128(sQ + offb, 16, 1024),
                     idS, kk ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t offa = (kk >> 2) * (Cf::BK * 128) + (kk & 3) * 32;
          const uint32_t offb = (kk >> 2) * (Cf::BQ * 128) + (kk & 3) * 32;
          tc_mma_f16(tmem + Cf::dp_col(s), smem_desc_sw128(sV + offa, 16, 1024),
                     smem_desc_sw128(sdO + offb, 16, 1024), idS, kk ? 1u : 0u);
        }
        tc_commit(&sp_full[s]);
        if (j >= 1 && !issue_acc(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_acc(nqb - 1);
      if (ok) tc_commit(acc_done);
    }
  } else {
    const int quarter = warp & 3;
    const int lane = threadIdx.x & 31;
    const int r = quarter * 32 + lane;              // key row of this thread (TMEM lane)
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float sc = p.scale * 1.4426950408889634f;
    const int64_t sbase = ((int64_t)b * p.H + h) * p.n;
    const int kidx = k0 + r;
    // per-query values of block j: threads r < 64 fetch -lse*log2e of query r, the
    // others D of query r - 64 (rows past the end: +inf lse, zero D)
    auto fetch = [&](int j) -> float {
      const int i = (qb0 + j) * Cf::BQ + (r & 63);
      if (i >= p.n) return r < 64 ? -INFINITY : 0.f;
      return r < 64 ? -p.lse[sbase + i] * 1.4426950408889634f : p.Dsum[sbase + i];
    };
    ldbuf[r] = fetch(0);
    named_bar_sync(1, 128);
    bool ok = true;
    for (int j = 0; j < nqb; ++j) {
      const int s = j & 1;
      const int i0 = (qb0 + j) * Cf::BQ;
      const float nxt = j + 1 < nqb ? fetch(j + 1) : 0.f;
      const bool need_mask = (i0 < k0 + Cf::BK - 1) || (i0 + Cf::BQ - 1 - k0 > p.window - 1);
      // after a timed-out wait the loop still runs to its end (without waiting or
      // computing) so that all four warps meet at every named barrier
      if (ok) ok = mbar_wait(&sp_full[s], (j >> 1) & 1, err, DEV_TIMEOUT_ACC);
      if (ok) {
        tc_fence_after();
        uint32_t sr[64], dr[64];
        tmem_ld32_nowait(tmem + lane_base + Cf::s_col(s), sr);
        tmem_ld32_nowait(tmem + lane_base + Cf::s_col(s) + 32, sr + 32);
        tmem_ld32_nowait(tmem + lane_base + Cf::dp_col(s), dr);
        tmem_ld32_nowait(tmem + lane_base + Cf::dp_col(s) + 32, dr + 32);
        tmem_ld_wait();
        const float* nl = ldbuf + s * 2 * Cf::BQ;
        const float* dd = nl + Cf::BQ;
        float pw[Cf::BQ / 2], dw[Cf::BQ / 2];  // P^T and dS^T of this key row as bf16 pairs
  #pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const float4 nl0 = *(const float4*)(nl + cc * 8), nl1 = *(const float4*)(nl + cc * 8 + 4);
          const float4 d0 = *(const float4*)(dd + cc * 8), d1 = *(const float4*)(dd + cc * 8 + 4);
          const float nlv[8] = {nl0.x, nl0.y, nl0.z, nl0.w, nl1.x, nl1.y, nl1.z, nl1.w};
          const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
          float pv[8], ds[8];
  #pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = cc * 8 + e;
            float pr = ex2_tc(fmaf(__uint_as_float(sr[c]), sc, nlv[e]));
            if (need_mask) {
              const uint32_t off = (uint32_t)(i0 + c - kidx);
              pr = off <= (uint32_t)(p.window - 1) ? pr : 0.f;
            }
            pv[e] = pr;
            ds[e] = pr * (__uint_as_float(dr[c]) - dv[e]);
          }
  #pragma unroll
          for (int e = 0; e < 4; ++e) {
            pw[cc * 4 + e] = __uint_as_float(pack_bf16x2(pv[2 * e], pv[2 * e + 1]));
            dw[cc * 4 + e] = __uint_as_float(pack_bf16x2(ds[2 * e], ds[2 * e + 1]));
          }
        }
        // over the scores in TMEM (both read above): the MMA warp takes them as A operands
        tmem_st32(tmem + lane_base + Cf::s_col(s), pw);
        tmem_st32(tmem + lane_base + Cf::dp_col(s), dw);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pd_full[s]);
      }
      // block j+1's values go to the other half; every thread is past its reads of it
      ldbuf[((j + 1) & 1) * 2 * Cf::BQ + r] = nxt;
      named_bar_sync(1, 128);
    }
    if (ok && mbar_wait(acc_done, 0, err, DEV_TIMEOUT_ACC)) {
      tc_fence_after();
      const int64_t orow = ((int64_t)b * p.n + kidx) * p.lddq + h * HD;
      bf16* dV = (bf16*)p.dV + orow;
      bf16* dK = (bf16*)p.dK + orow;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_base + Cf::DV_COL + c * 32, o);
        if (r < nk) {
          uint4* dst = (uint4*)(dV + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(o[8 * q], o[8 * q + 1]), pack_bf16x2(o[8 * q + 2], o[8 * q + 3]),
                                pack_bf16x2(o[8 * q + 4], o[8 * q + 5]), pack_bf16x2(o[8 * q + 6], o[8 * q + 7]));
        }
        tmem_ld32(tmem + lane_base + Cf::DK_COL + c * 32, o);
        if (r < nk) {
          uint4* dst = (uint4*)(dK + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(o[8 * q] * p.scale, o[8 * q + 1] * p.scale),
                                pack_bf16x2(o[8 * q + 2] * p.scale, o[8 * q + 3] * p.scale),
                                pack_bf16x2(o[8 * q + 4] * p.scale, o[8 * q + 5] * p.scale),
                                pack_bf16x2(o[8 * q + 6] * p.scale, o[8 * q + 7] * p.scale));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace ttt
