// attn_bwd.cuh -- backward of the fused attention: preprocess, main kernel,
// dQ finalize.
//
// The Axis page (zyoralabs.com/axis, feature list) fuses the attention
// backward as well as the forward; the gradient itself is the analytic one of
// softmax attention:
//   P_ij = exp(s_ij - LSE_i),  dP_ij = dO_i . V_j,  Dr_i = dO_i . O_i,
//   dS_ij = P_ij (dP_ij - Dr_i),  dQ_i = scale sum_j dS_ij K_j,
//   dK_j = scale sum_{h in group} sum_i dS_ij Q_i,  dV_j = sum_{h, i} P_ij dO_i.
// Design on sm_100a:
//   * preprocess (HBM-bound): Dr and log2-scaled LSE per row, padded to a
//     multiple of 128 rows (padding rows get Dr = 0, LSE = +inf, so their P is
//     exactly 0); zero the fp32 dQ accumulator;
//   * main kernel: one CTA per (b, kv head, 128-key tile); K_j, V_j stay in
//     shared memory while the CTA walks every query head of the group and every
//     query tile that can see the keys.  Per tile (one thread issues all MMAs):
//       S^T = K Q^T and dP^T = V dO^T into TMEM (thread = key row),
//       P^T = 2^(S^T c - LSE2), dS^T = P^T (dP^T - Dr) by 8 warps from TMEM,
//       P^T back to TMEM (bf16), dS^T to shared memory (bf16, 128B swizzle),
//       dV += P^T dO (A from TMEM), dK += dS^T Q, and dQ of the tile,
//     dQ is read from TMEM by a fourth warpgroup and added into the fp32
//     accumulator with vector atomics; dK, dV stay in TMEM until the end;
//   * dQ finalize (HBM-bound): bf16 copy of the accumulator in [B,S,Hq,D].
// D = 64 uses 128-row query tiles and dQ = dS K (TMEM lane = query row);
// D = 128 uses 64-row query tiles (shared memory) and dQ^T = K^T dS^T (TMEM
// lane = feature), so every MMA has M = 128.
#pragma once

#include "sm100_ptx.cuh"

namespace axis_attn {

struct BwdArgs {
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* lse2;  // [B*Hq][S_pad]  LSE * log2(e); +inf on padding rows
  const float* dr;    // [B*Hq][S_pad]  rowsum(dO * O); 0 on padding rows
  float* dqacc;       // [B*Hq][S][HD]  fp32, pre-scaled by `scale`
  int B, Hq, Hkv, S, S_pad;
  float scale, scale_log2;
};

template <int HD>
struct BwdCfg {
  static constexpr int BM = HD == 64 ? 128 : 64;   // query rows per step
  static constexpr bool QLANE = HD == 64;          // dQ lanes = query rows
  static constexpr int NSLAB = HD / 64;
  static constexpr uint32_t KSLAB = 128 * 128;     // 128 key rows x 128 bytes
  static constexpr uint32_t KTILE = NSLAB * KSLAB;
  static constexpr uint32_t QSLAB = BM * 128;      // BM query rows x 128 bytes
  static constexpr uint32_t QTILE = NSLAB * QSLAB;
  static constexpr uint32_t DS_BYTES = (BM / 64) * 128 * 128;  // dS^T: 128 keys x BM
  static constexpr int ST = 2;
  // shared-memory offsets from the 1024-aligned base
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = KTILE;
  static constexpr uint32_t OFF_Q = 2 * KTILE;
  static constexpr uint32_t OFF_DO = OFF_Q + ST * QTILE;
  static constexpr uint32_t OFF_DS = OFF_DO + ST * QTILE;
  static constexpr uint32_t OFF_LSE = OFF_DS + DS_BYTES;
  static constexpr uint32_t OFF_DR = OFF_LSE + ST * BM * 4;
  static constexpr uint32_t OFF_BAR = OFF_DR + ST * BM * 4;
  static constexpr int NBAR = 8 + 2 * ST;
  static constexpr uint32_t SMEM = OFF_BAR + 8 * NBAR + 16 + 1024;
  // TMEM columns
  static constexpr uint32_t T_S = 0, T_DP = BM, T_DV = 2 * BM, T_DK = 2 * BM + HD,
                            T_DQ = 2 * BM + 2 * HD;
};

enum BwdSite { B_KV = 21, B_QEMPTY, B_QFULL, B_MMADONE, B_DSREADY, B_DQFREE, B_SPFULL, B_DQFULL, B_FIN };

template <int HD, bool CAUSAL>
__global__ void __launch_bounds__(512, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdArgs a) {
  using C = BwdCfg<HD>;
  constexpr int BM = C::BM, ST = C::ST;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V, sDS = base + C::OFF_DS;
  auto sQ = [&](int s) { return base + C::OFF_Q + s * C::QTILE; };
  auto sDO = [&](int s) { return base + C::OFF_DO + s * C::QTILE; };
  const float* lse_s = reinterpret_cast<const float*>(gbase + C::OFF_LSE);
  const float* dr_s = reinterpret_cast<const float*>(gbase + C::OFF_DR);
  const uint32_t bars = base + C::OFF_BAR;
  const uint32_t bar_kv = bars;
  auto bar_qfull = [&](int s) { return bars + 8u * (1 + s); };
  auto bar_qempty = [&](int s) { return bars + 8u * (1 + ST + s); };
  const uint32_t bar_sp = bars + 8u * (1 + 2 * ST);
  const uint32_t bar_ds = bars + 8u * (2 + 2 * ST);
  const uint32_t bar_dqfull = bars + 8u * (3 + 2 * ST);
  const uint32_t bar_dqfree = bars + 8u * (4 + 2 * ST);
  const uint32_t bar_done = bars + 8u * (5 + 2 * ST);
  const uint32_t bar_fin = bars + 8u * (6 + 2 * ST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + 8 * C::NBAR);
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + C::OFF_BAR + 8 * C::NBAR + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: key tiles with the most query tiles first
  const int BKV = a.B * a.Hkv;
  const int j = (int)(blockIdx.x / BKV);
  const int bkv = (int)(blockIdx.x % BKV);
  const int b = bkv / a.Hkv, kvh = bkv % a.Hkv;
  const int G = a.Hq / a.Hkv;
  const int nqt = (a.S + BM - 1) / BM;
  const int i0 = CAUSAL ? (128 * j) / BM : 0;
  const int per_head = nqt - i0;
  const int n_it = G * per_head;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar_qfull(s), 1);
      mbar_init(bar_qempty(s), 1);
    }
    mbar_init(bar_sp, 1);
    mbar_init(bar_ds, 8);
    mbar_init(bar_dqfull, 1);
    mbar_init(bar_dqfree, 4);
    mbar_init(bar_done, 1);
    mbar_init(bar_fin, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 12) {
    // ===================================================== loads
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar_kv, 2 * C::KTILE);
      for (int sl = 0; sl < C::NSLAB; ++sl) {
        tma_load_4d(sK + sl * C::KSLAB, &tm_k, bar_kv, 64 * sl, kvh, 128 * j, b);
        tma_load_4d(sV + sl * C::KSLAB, &tm_v, bar_kv, 64 * sl, kvh, 128 * j, b);
      }
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int s = it % ST;
        if (!mbar_wait_bounded(bar_qempty(s), ((it / ST) & 1) ^ 1, abort, B_QEMPTY)) break;
        const int h = kvh * G + it / per_head;
        const int q0 = (i0 + it % per_head) * BM;
        const size_t row = ((size_t)b * a.Hq + h) * a.S_pad + q0;
        mbar_arrive_expect_tx(bar_qfull(s), 2 * C::QTILE + 2 * BM * 4);
        for (int sl = 0; sl < C::NSLAB; ++sl) {
          tma_load_4d(sQ(s) + sl * C::QSLAB, &tm_q, bar_qfull(s), 64 * sl, h, q0, b);
          tma_load_4d(sDO(s) + sl * C::QSLAB, &tm_do, bar_qfull(s), 64 * sl, h, q0, b);
        }
        bulk_load(base + C::OFF_LSE + s * BM * 4, a.lse2 + row, BM * 4, bar_qfull(s));
        bulk_load(base + C::OFF_DR + s * BM * 4, a.dr + row, BM * 4, bar_qfull(s));
        issued = it + 1;
      }
      volatile int never = 0;
      mbar_wait_bounded(bar_kv, 0, &never, B_KV);
      for (int it = issued - ST > 0 ? issued - ST : 0; it < issued; ++it)
        mbar_wait_bounded(bar_qfull(it % ST), (it / ST) & 1, &never, B_QFULL);
    }
  } else if (warp == 13) {
    // ===================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16(128, BM, 0, 0);   // K|V (K-major) x Q|dO (K-major)
      constexpr uint32_t ID_GV = idesc_bf16(128, HD, 0, 1);  // P^T|dS^T x dO|Q (MN-major)
      constexpr uint32_t ID_Q = C::QLANE ? idesc_bf16(128, HD, 1, 1) : idesc_bf16(128, BM, 1, 1);
      bool ok = mbar_wait_bounded(bar_kv, 0, abort, B_KV);
      for (int it = 0; ok && it < n_it; ++it) {
        const int s = it % ST;
        if (!mbar_wait_bounded(bar_qfull(s), (it / ST) & 1, abort, B_QFULL)) break;
        if (it > 0 && !mbar_wait_bounded(bar_done, (it - 1) & 1, abort, B_MMADONE)) break;
        tc_fence_after();
        // S^T = K Q^T, dP^T = V dO^T  (reduction over the feature dim)
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * C::KSLAB + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * C::QSLAB + (kk & 3) * 32;
          mma_ss(tmem + C::T_S, sw128_desc(sK + ko, 16, 1024), sw128_desc(sQ(s) + qo, 16, 1024), ID_S,
                 kk > 0);
        }
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * C::KSLAB + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * C::QSLAB + (kk & 3) * 32;
          mma_ss(tmem + C::T_DP, sw128_desc(sV + ko, 16, 1024), sw128_desc(sDO(s) + qo, 16, 1024),
                 ID_S, kk > 0);
        }
        mma_commit(bar_sp);
        if (!mbar_wait_bounded(bar_ds, it & 1, abort, B_DSREADY)) break;
        tc_fence_after();
        // dV += P^T dO, dK += dS^T Q  (reduction over the BM query rows)
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t pcol = kk < BM / 32 ? 8 * kk : BM / 2 + 8 * (kk - BM / 32);
          mma_ts(tmem + C::T_DV, tmem + C::T_S + pcol, sw128_desc(sDO(s) + kk * 2048, C::QSLAB, 1024),
                 ID_GV, (it > 0 || kk > 0) ? 1u : 0u);
        }
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t dso = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          mma_ss(tmem + C::T_DK, sw128_desc(sDS + dso, 16, 1024),
                 sw128_desc(sQ(s) + kk * 2048, C::QSLAB, 1024), ID_GV, (it > 0 || kk > 0) ? 1u : 0u);
        }
        // dQ tile (reduction over the 128 keys)
        if (it > 0 && !mbar_wait_bounded(bar_dqfree, (it - 1) & 1, abort, B_DQFREE)) break;
        tc_fence_after();
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ds_mn = sw128_desc(sDS + kk * 2048, 128 * 128, 1024);
          const uint64_t k_mn = sw128_desc(sK + kk * 2048, C::KSLAB, 1024);
          if (C::QLANE)
            mma_ss(tmem + C::T_DQ, ds_mn, k_mn, ID_Q, kk > 0);   // dQ = dS K
          else
            mma_ss(tmem + C::T_DQ, k_mn, ds_mn, ID_Q, kk > 0);   // dQ^T = K^T dS^T
        }
        mma_commit(bar_dqfull);
        mma_commit(bar_qempty(s));
        mma_commit(bar_done);
      }
      mma_commit(bar_fin);
      volatile int never = 0;
      mbar_wait_bounded(bar_fin, 0, &never, B_FIN);
    }
  } else if (warp < 8) {
    // ===================================================== P^T, dS^T (thread = key row)
    const int wq = warp & 3, ch = warp >> 2;
    const int kr = wq * 32 + lane;
    const int key = 128 * j + kr;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int c0 = ch * (BM / 2);
    const float c = a.scale_log2;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % ST;
      // the staged LSE2 / Dr rows of this step (TMA-written) and S^T, dP^T in TMEM
      if (!wait_warp(bar_qfull(s), (it / ST) & 1, abort, B_QFULL) ||
          !wait_warp(bar_sp, it & 1, abort, B_SPFULL)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int q0 = (i0 + it % per_head) * BM;
      const bool need_mask = (CAUSAL && q0 < 128 * j + 127) || (128 * j + 128 > a.S);
      const float* lse_t = lse_s + s * BM;
      const float* dr_t = dr_s + s * BM;
#pragma unroll 1
      for (int cc = 0; cc < BM / 32; ++cc) {
        const int col0 = c0 + 16 * cc;
        uint32_t sv[16], dpv[16];
        tmem_ld16(tmem + lane_off + C::T_S + col0, sv);
        tmem_ld16(tmem + lane_off + C::T_DP + col0, dpv);
        tmem_wait_ld();
        uint32_t pk[8], dk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse_t + col0 + (e & ~3));
          const float4 d4 = *reinterpret_cast<const float4*>(dr_t + col0 + (e & ~3));
          const float la = (e & 3) ? l4.z : l4.x, lb = (e & 3) ? l4.w : l4.y;
          const float da = (e & 3) ? d4.z : d4.x, db = (e & 3) ? d4.w : d4.y;
          float p0 = ex2_approx(fmaf(__uint_as_float(sv[e]), c, -la));
          float p1 = ex2_approx(fmaf(__uint_as_float(sv[e + 1]), c, -lb));
          if (need_mask) {
            const int q = q0 + col0 + e;
            if ((CAUSAL && key > q) || key >= a.S) p0 = 0.f;
            if ((CAUSAL && key > q + 1) || key >= a.S) p1 = 0.f;
          }
          const float ds0 = p0 * (__uint_as_float(dpv[e]) - da);
          const float ds1 = p1 * (__uint_as_float(dpv[e + 1]) - db);
          pk[e / 2] = pack_bf16x2(p0, p1);
          dk[e / 2] = pack_bf16x2(ds0, ds1);
        }
        // P^T (bf16) into TMEM over already-consumed S^T columns of this warp's range
        tmem_st8(tmem + lane_off + C::T_S + c0 + 8 * cc, pk);
        // dS^T (bf16) into the 128B-swizzled [key][query] slabs
        const int slab = col0 >> 6, chunk = (col0 & 63) >> 3;
        const uint32_t rowaddr = sDS + slab * (128 * 128) + (kr >> 3) * 1024 + (kr & 7) * 128;
        const uint32_t a0 = rowaddr + (((chunk) ^ (kr & 7)) << 4);
        const uint32_t a1 = rowaddr + (((chunk + 1) ^ (kr & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a0), "r"(dk[0]), "r"(dk[1]),
                     "r"(dk[2]), "r"(dk[3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a1), "r"(dk[4]), "r"(dk[5]),
                     "r"(dk[6]), "r"(dk[7])
                     : "memory");
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_ds);
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK (x scale)
    if (ok && wait_warp(bar_fin, 0, abort, B_FIN)) {
      tc_fence_after();
      const uint32_t tcol = ch == 0 ? C::T_DV : C::T_DK;
      const float mul = ch == 0 ? 1.f : a.scale;
      __nv_bfloat16* dst_row = (ch == 0 ? a.dv : a.dk) + (((size_t)b * a.S + key) * a.Hkv + kvh) * HD;
#pragma unroll 1
      for (int cc = 0; cc < HD / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + tcol + cc * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
        if (key < a.S) {
          uint4* dst = reinterpret_cast<uint4*>(dst_row + cc * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
    }
  } else if (warp < 12) {
    // ===================================================== dQ tile -> fp32 accumulator
    const int wq = warp & 3;
    const int lr = wq * 32 + lane;   // TMEM lane: query row (D=64) or feature (D=128)
    const uint32_t tq = tmem + ((uint32_t)(wq * 32) << 16) + C::T_DQ;
    for (int it = 0; it < n_it; ++it) {
      if (!wait_warp(bar_dqfull, it & 1, abort, B_DQFULL)) break;
      tc_fence_after();
      uint32_t v0[32], v1[32];
      tmem_ld32(tq, v0);
      tmem_ld32(tq + 32, v1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dqfree);
      const int h = kvh * G + it / per_head;
      const int q0 = (i0 + it % per_head) * BM;
      float* acc = a.dqacc + ((size_t)b * a.Hq + h) * (size_t)a.S * HD;
      const float sc = a.scale;
      if (C::QLANE) {
        const int q = q0 + lr;
        if (q < a.S) {
          float4* dst = reinterpret_cast<float4*>(acc + (size_t)q * HD);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            atomicAdd(dst + i, make_float4(__uint_as_float(v0[4 * i]) * sc, __uint_as_float(v0[4 * i + 1]) * sc,
                                           __uint_as_float(v0[4 * i + 2]) * sc, __uint_as_float(v0[4 * i + 3]) * sc));
#pragma unroll
          for (int i = 0; i < 8; ++i)
            atomicAdd(dst + 8 + i, make_float4(__uint_as_float(v1[4 * i]) * sc, __uint_as_float(v1[4 * i + 1]) * sc,
                                               __uint_as_float(v1[4 * i + 2]) * sc, __uint_as_float(v1[4 * i + 3]) * sc));
        }
      } else {
        // lane = feature d; columns = the BM query rows of the tile
        float* col = acc + lr;
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (q0 + e < a.S) atomicAdd(col + (size_t)(q0 + e) * HD, __uint_as_float(v0[e]) * sc);
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (q0 + 32 + e < a.S) atomicAdd(col + (size_t)(q0 + 32 + e) * HD, __uint_as_float(v1[e]) * sc);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Dr = rowsum(dO * O) (fp32), LSE2 = LSE * log2(e); rows S..S_pad-1 get
// Dr = 0 and LSE2 = +inf.  Also zeroes the dQ accumulator.  One thread per row.
template <int HD>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dout,
                                                            const float* __restrict__ lse, float* lse2,
                                                            float* dr, float4* dqacc, size_t dq_vec4,
                                                            int Hq, int S, int S_pad, int rows) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < rows) {
    const int bh = r / S_pad, i = r % S_pad;
    float d = 0.f, l2 = INFINITY;
    if (i < S) {
      const int b = bh / Hq, h = bh % Hq;
      const size_t off = (((size_t)b * S + i) * Hq + h) * HD;
      const uint4* po = reinterpret_cast<const uint4*>(o + off);
      const uint4* pd = reinterpret_cast<const uint4*>(dout + off);
#pragma unroll
      for (int c = 0; c < HD / 8; ++c) {
        const uint4 x = po[c], y = pd[c];
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[k]));
          const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[k]));
          d = fmaf(xf.x, yf.x, d);
          d = fmaf(xf.y, yf.y, d);
        }
      }
      l2 = lse[(size_t)bh * S + i] * 1.4426950408889634f;
    }
    dr[r] = d;
    lse2[r] = l2;
  }
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < dq_vec4; k += stride)
    dqacc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dq[b,i,h,:] = bf16(dqacc[b,h,i,:]); 8 features per thread.
template <int HD>
__global__ void __launch_bounds__(256) attn_bwd_dq_convert_kernel(const float* __restrict__ dqacc,
                                                                  __nv_bfloat16* __restrict__ dq, int Hq,
                                                                  int S, size_t n8) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < n8; k += stride) {
    const int c8 = (int)(k % (HD / 8));
    const size_t row = k / (HD / 8);   // row in [B, S, Hq] order
    const int h = (int)(row % Hq);
    const size_t bi = row / Hq;        // b * S + i
    const int i = (int)(bi % S);
    const size_t b = bi / S;
    const float4* src = reinterpret_cast<const float4*>(dqacc + (((b * Hq + h) * S + i) * HD) + 8 * c8);
    const float4 x = src[0], y = src[1];
    uint4 out;
    out.x = pack_bf16x2(x.x, x.y);
    out.y = pack_bf16x2(x.z, x.w);
    out.z = pack_bf16x2(y.x, y.y);
    out.w = pack_bf16x2(y.z, y.w);
    reinterpret_cast<uint4*>(dq + row * HD)[c8] = out;
  }
}

}  // namespace axis_attn
