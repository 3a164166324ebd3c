// attn_bwd_dq.cuh -- deterministic dQ pass of the backward: one CTA per
// (b, query head, 128-row query tile) recomputes, for every key tile the rows
// see, S = Q K^T, P = 2^(S c - LSE2) and scale dS = P (scale dP - scale Dr)
// with dP = dO V^T, and accumulates dQ = sum_j (scale dS_j) K_j in tensor
// memory, in the fixed
// order of the key tiles.  No cross-CTA additions: the result is bitwise the
// same from run to run, and the only scratch is the per-row LSE2 and Dr of
// the preprocess (O(B Hq S) floats), so memory stays flat as S grows.
//
// The gradient is the analytic one of softmax attention (the Axis page,
// zyoralabs.com/axis, feature list: fused attention forward and backward):
//   dQ_i = scale * sum_j P_ij (dP_ij - Dr_i) K_j,  dP_ij = dO_i . V_j.
// The main backward kernel, run in its no-dQ mode, supplies dK and dV.
//
// Roles: warps 0-15 compute (thread = query row = TMEM lane; warp w takes rows
// 32 (w % 4) .. + 31 and the key columns 32 (w / 4) .. + 31 of each tile:
// four warps per SM sub-partition hide the latency of the TMEM loads and the
// exponentials); warp 16 loads (TMA: Q and dO once, then the K and V rings);
// warp 17 issues the MMAs and owns TMEM.  TMEM columns: S [0,128),
// dP [128,256), dQ [256, 256 + HD).
#pragma once

#include "attn_rope.cuh"
#include "sm100_ptx.cuh"

namespace axis_attn {

struct DqArgs {
  __nv_bfloat16* dq;   // [B, S, Hq, HD]
  const float* nlse2;  // [B*Hq][S_pad]  -LSE * log2(e); -inf on padding rows
  const float* ndr;    // [B*Hq][S_pad]  -scale rowsum(dO * O); 0 on padding rows
  int B, Hq, Hkv, S, S_pad;
  float scale, scale_log2;
  const double2* rope_cs;  // RoPE: (cos, sin) table [S][HD/2], fp64; dQ leaves through the transposed rotation
};

template <int HD>
struct DqCfg {
  static constexpr int NSLAB = HD / 64;
  static constexpr uint32_t SLAB = 128 * 128;      // 128 rows x 128 bytes
  static constexpr uint32_t TILE = NSLAB * SLAB;   // 128 x HD bf16
  static constexpr uint32_t DS_TILE = 2 * SLAB;    // dS: 128 q rows x 128 keys bf16 (two 64-key slabs)
  static constexpr int KST = HD == 64 ? 3 : 2;     // K ring
  static constexpr int VST = HD == 64 ? 3 : 2;     // V ring
  static constexpr int NDS = HD == 64 ? 2 : 1;     // dS buffers
  static constexpr uint32_t OFF_Q = 0, OFF_DO = TILE, OFF_K = 2 * TILE;
  static constexpr uint32_t OFF_V = OFF_K + KST * TILE;
  static constexpr uint32_t OFF_DS = OFF_V + VST * TILE;
  static constexpr uint32_t OFF_BAR = OFF_DS + NDS * DS_TILE;
  static constexpr int NBAR = 5 + 2 * KST + 2 * VST + 2 * NDS;
  static constexpr uint32_t SMEM = OFF_BAR + 8 * NBAR + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256;
};

constexpr int DQ_THREADS = 576;
constexpr int DQ_WARP_LOAD = 16;
constexpr int DQ_WARP_MMA = 17;

enum DqSite { Q_Q = 61, Q_KEMPTY, Q_VEMPTY, Q_KFULL, Q_VFULL, Q_SFREE, Q_DSFULL, Q_SFULL, Q_DSFREE, Q_FIN };

// scale dS of one thread's 32 key columns of a tile: p = 2^(s c - LSE2),
// ds = p (scale dp - scale Dr), packed to bf16 pairs.  MASK (the diagonal or
// ragged tile): columns from limit on get p = 0; a template parameter, so that
// the other tiles test nothing per pair.
template <bool MASK>
__device__ __forceinline__ void dq_tile_math(const uint32_t (&sv)[32], const uint32_t (&dpv)[32], uint64_t cc2,
                                             uint64_t nl2_2, uint64_t sc2, uint64_t ndr2, int limit,
                                             uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), cc2, nl2_2), x0, x1);
    float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    if constexpr (MASK) {
      if (2 * e >= limit) p0 = 0.f;
      if (2 * e + 1 >= limit) p1 = 0.f;
    }
    const uint64_t ds =
        f2_mul(f2_pack(p0, p1), f2_fma(f2_pack(__uint_as_float(dpv[2 * e]), __uint_as_float(dpv[2 * e + 1])), sc2, ndr2));
    pk[e] = pack_bf16x2(ds);
  }
}

template <int HD, bool CAUSAL>
__global__ void __launch_bounds__(DQ_THREADS, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const DqArgs a) {
  using C = DqCfg<HD>;
  constexpr int KST = C::KST, VST = C::VST, NDS = C::NDS;
  constexpr uint32_t TILE = C::TILE, SLAB = C::SLAB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q, sDO = base + C::OFF_DO, sK = base + C::OFF_K, sV = base + C::OFF_V;
  const uint32_t sDS = base + C::OFF_DS;
  const uint32_t bars = base + C::OFF_BAR;
  const uint32_t bar_q = bars, bar_sfull = bars + 8, bar_sfree = bars + 16, bar_fin = bars + 24;
  auto bar_kfull = [&](int s) { return bars + 8u * (5 + s); };
  auto bar_kempty = [&](int s) { return bars + 8u * (5 + KST + s); };
  auto bar_vfull = [&](int s) { return bars + 8u * (5 + 2 * KST + s); };
  auto bar_vempty = [&](int s) { return bars + 8u * (5 + 2 * KST + VST + s); };
  auto bar_dsfull = [&](int b) { return bars + 8u * (5 + 2 * KST + 2 * VST + b); };
  auto bar_dsfree = [&](int b) { return bars + 8u * (5 + 2 * KST + 2 * VST + NDS + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + 8 * C::NBAR);
  volatile WaitCtl* abort = reinterpret_cast<volatile WaitCtl*>(gbase + C::OFF_BAR + 8 * C::NBAR + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // work item: query tiles with the most key tiles first (causal)
  const int BH = a.B * a.Hq;
  const int nqt = (a.S + 127) / 128, nkv_all = nqt;
  const int qt = nqt - 1 - (int)(blockIdx.x / BH);
  const int bh = (int)(blockIdx.x % BH);
  const int b = bh / a.Hq, h = bh % a.Hq, kvh = h / (a.Hq / a.Hkv);
  const int nkv = CAUSAL ? qt + 1 : nkv_all;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_sfull, 1);
    mbar_init(bar_sfree, 16);
    mbar_init(bar_fin, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_kempty(s), 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int x = 0; x < NDS; ++x) {
      mbar_init(bar_dsfull(x), 16);
      mbar_init(bar_dsfree(x), 1);
    }
    wait_ctl_init(abort);
    fence_barrier_init();
  }
  if (warp == DQ_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == DQ_WARP_LOAD) {
    // ============================================================ loads
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar_q, 2 * TILE);
      for (int sl = 0; sl < C::NSLAB; ++sl) {
        tma_load_4d(sQ + sl * SLAB, &tm_q, bar_q, 64 * sl, h, 128 * qt, b);
        tma_load_4d(sDO + sl * SLAB, &tm_do, bar_q, 64 * sl, h, 128 * qt, b);
      }
      int nk = 0, nv = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % KST;
        if (j >= KST && !mbar_wait_bounded<true>(bar_kempty(s), ((j / KST) & 1) ^ 1, abort, Q_KEMPTY)) break;
        mbar_arrive_expect_tx(bar_kfull(s), TILE);
        for (int sl = 0; sl < C::NSLAB; ++sl)
          tma_load_4d(sK + s * TILE + sl * SLAB, &tm_k, bar_kfull(s), 64 * sl, kvh, 128 * j, b);
        nk = j + 1;
        const int t = j % VST;
        if (j >= VST && !mbar_wait_bounded<true>(bar_vempty(t), ((j / VST) & 1) ^ 1, abort, Q_VEMPTY)) break;
        mbar_arrive_expect_tx(bar_vfull(t), TILE);
        for (int sl = 0; sl < C::NSLAB; ++sl)
          tma_load_4d(sV + t * TILE + sl * SLAB, &tm_v, bar_vfull(t), 64 * sl, kvh, 128 * j, b);
        nv = j + 1;
      }
      // drain: every copy started has landed before the CTA exits
      volatile WaitCtl never = {0, 0, 0};  // drain: bounded by the time limit only
      mbar_wait_bounded<true>(bar_q, 0, &never, Q_Q);
      for (int x = nk - KST > 0 ? nk - KST : 0; x < nk; ++x)
        mbar_wait_bounded<true>(bar_kfull(x % KST), (x / KST) & 1, &never, Q_KFULL);
      for (int x = nv - VST > 0 ? nv - VST : 0; x < nv; ++x)
        mbar_wait_bounded<true>(bar_vfull(x % VST), (x / VST) & 1, &never, Q_VFULL);
    }
  } else if (warp == DQ_WARP_MMA) {
    // ============================================================ MMA issue
    // S(j) = Q K_j^T, dP(j) = dO V_j^T (M = 128 query rows, N = 128 keys),
    // then, once the compute warps have written dS(j) to shared memory,
    // dQ += dS(j) K_j (M = 128 rows, N = HD, K = 128 keys; K_j MN-major).
    // S(j + 1) is issued before dQ(j), as soon as S(j) and dP(j) are read.
    constexpr uint32_t ID_S = idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t ID_DQ = idesc_bf16(128, HD, 0, 1);
    bool ok = wait_warp<true>(bar_q, 0, abort, Q_Q);
    auto issue_dq = [&](int j) -> bool {
      const int x = j % NDS, s = j % KST;
      if (!wait_warp<true>(bar_dsfull(x), (j / NDS) & 1, abort, Q_DSFULL)) return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_w(tmem + C::T_DQ, sw128_desc(sDS + x * C::DS_TILE + (kk >> 2) * SLAB + (kk & 3) * 32, 16, 1024),
                 sw128_desc(sK + s * TILE + kk * 2048, SLAB, 1024), ID_DQ, (j > 0 || kk > 0) ? 1u : 0u);
      mma_commit_w(bar_dsfree(x));
      mma_commit_w(bar_kempty(s));  // K_j: read by S(j) and dQ(j)
      return true;
    };
    for (int j = 0; ok && j < nkv; ++j) {
      const int s = j % KST, t = j % VST;
      if (j > 0 && !(ok = wait_warp<true>(bar_sfree, (j - 1) & 1, abort, Q_SFREE))) break;
      if (!(ok = wait_warp<true>(bar_kfull(s), (j / KST) & 1, abort, Q_KFULL))) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * SLAB + (kk & 3) * 32;
        mma_ss_w(tmem + C::T_S, sw128_desc(sQ + off, 16, 1024), sw128_desc(sK + s * TILE + off, 16, 1024), ID_S,
                 kk > 0);
      }
      if (!(ok = wait_warp<true>(bar_vfull(t), (j / VST) & 1, abort, Q_VFULL))) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * SLAB + (kk & 3) * 32;
        mma_ss_w(tmem + C::T_DP, sw128_desc(sDO + off, 16, 1024), sw128_desc(sV + t * TILE + off, 16, 1024), ID_S,
                 kk > 0);
      }
      mma_commit_w(bar_sfull);
      mma_commit_w(bar_vempty(t));
      if (j > 0 && !(ok = issue_dq(j - 1))) break;
    }
    if (ok && nkv > 0) ok = issue_dq(nkv - 1);
    // all MMAs of the CTA complete before the epilogue reads dQ and TMEM is freed
    mma_commit_w(bar_fin);
    volatile WaitCtl never = {0, 0, 0};  // drain: bounded by the time limit only
    wait_warp<true>(bar_fin, 0, &never, Q_FIN);
  } else {
    // ============================================================ compute: P, dS
    const int wq = warp & 3, qc = warp >> 2;  // lane quarter (rows), column quarter (keys)
    const int r = wq * 32 + lane;
    const int row_g = 128 * qt + r;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const float nl2 = a.nlse2[(size_t)bh * a.S_pad + row_g];  // row_g < S_pad
    const float ndr = a.ndr[(size_t)bh * a.S_pad + row_g];
    const uint64_t cc2 = f2_pack(a.scale_log2, a.scale_log2);
    const uint64_t nl2_2 = f2_pack(nl2, nl2), ndr2 = f2_pack(ndr, ndr);
    const uint64_t sc2 = f2_pack(a.scale, a.scale);  // dS formed scaled: P (scale dP - scale Dr)
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!wait_warp<true>(bar_sfull, j & 1, abort, Q_SFULL)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[32], dpv[32];
      tmem_ld32(tmem + lane_off + C::T_S + 32 * qc, sv);
      tmem_ld32(tmem + lane_off + C::T_DP + 32 * qc, dpv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_sfree);
      // visible keys of this row in this quarter: key = 128 j + 32 qc + e
      const bool masked = CAUSAL ? (j == qt) : (j == nkv - 1 && (a.S & 127) != 0);
      int limit = 32;
      if (masked) {
        limit = a.S - (128 * j + 32 * qc);
        if (CAUSAL && row_g + 1 - (128 * j + 32 * qc) < limit) limit = row_g + 1 - (128 * j + 32 * qc);
      }
      uint32_t pk[16];
      // the mask test once per tile, not per pair (masked is the same for the whole tile)
      if (masked)
        dq_tile_math<true>(sv, dpv, cc2, nl2_2, sc2, ndr2, limit, pk);
      else
        dq_tile_math<false>(sv, dpv, cc2, nl2_2, sc2, ndr2, limit, pk);
      // dS into its buffer (the dQ MMA of j - NDS must be done with it)
      const int x = j % NDS;
      if (j >= NDS && !wait_warp<true>(bar_dsfree(x), ((j / NDS) - 1) & 1, abort, Q_DSFREE)) { ok = false; break; }
      // row r of the 64-key slab qc / 2, chunks 4 (qc & 1) .. + 3 (128B swizzle)
      const uint32_t rowaddr = sDS + x * C::DS_TILE + (qc >> 1) * SLAB + r * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int chunk = 4 * (qc & 1) + c;
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(rowaddr + ((chunk ^ (r & 7)) << 4)),
                     "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                     : "memory");
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dsfull(x));
    }
    // epilogue: dQ (already scaled) -> bf16, this thread's HD / 4 columns of its row
    if (ok && wait_warp<true>(bar_fin, 0, abort, Q_FIN)) {
      tc_fence_after();
      constexpr int NC = HD / 4;  // 16 or 32 columns
      uint32_t v[32];
      if constexpr (NC == 32) {
        tmem_ld32(tmem + lane_off + C::T_DQ + NC * qc, v);
      } else {
        uint32_t v16[16];
        tmem_ld16(tmem + lane_off + C::T_DQ + NC * qc, v16);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = v16[i];
      }
      tmem_wait_ld();
      if (row_g < a.S && a.rope_cs != nullptr) {
        // dQ = R(row)^T dQ': pairs of features NC qc + 2 i
        const double2* t = a.rope_cs + (size_t)row_g * (HD / 2) + NC * qc / 2;
#pragma unroll
        for (int i = 0; i < NC / 2; ++i) {
          float g0 = __uint_as_float(v[2 * i]), g1 = __uint_as_float(v[2 * i + 1]);
          rope_back(g0, g1, t[i]);
          v[2 * i] = __float_as_uint(g0);
          v[2 * i + 1] = __float_as_uint(g1);
        }
      }
      if (row_g < a.S) {
        uint4* dst = reinterpret_cast<uint4*>(a.dq + (((size_t)b * a.S + row_g) * a.Hq + h) * HD + NC * qc);
#pragma unroll
        for (int i = 0; i < NC / 8; ++i)
          dst[i] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                              pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                              pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                              pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == DQ_WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace axis_attn
