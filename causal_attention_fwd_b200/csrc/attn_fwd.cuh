// attn_fwd.cuh -- forward kernel: O = softmax(scale * Q K^T, causal mask) V and
// the per-row log-sum-exp, for one (batch, query head) and 256 query rows per
// CTA.
//
// What it computes is the fused attention forward of the Axis page
// (zyoralabs.com/axis, feature list: fused flash attention; bf16 storage, fp32
// accumulation; probabilities never reach memory): scores and probabilities
// live only in tensor memory.  How, on sm_100a:
//
//   * one CTA owns two 128-row query tiles (Q0, Q1) of one (b, h); they share
//     a ring of K/V tiles (128 keys each) that one TMA thread streams in;
//   * one thread issues every tcgen05.mma: S_t = Q_t K_j^T (both operands
//     K-major in shared memory) into TMEM, then O_t += P_t V_j with P_t read
//     from TMEM (bf16, written in place over S_t) and V_j MN-major in smem;
//   * one warpgroup per query tile runs the online softmax in the log2 domain
//     from TMEM (thread = row): row max, p = 2^(s*c - m), row sum, P back to
//     TMEM.  The running max is only moved when it grows by more than 8 (a
//     factor 256), so the O rescale in TMEM is rare; stale-max values stay
//     below 2^8 and are exact to bf16 relative precision;
//   * causal: kv tiles after a query tile's diagonal are never loaded or
//     multiplied; the element mask runs only on the diagonal (and ragged last)
//     tile;
//   * the two query tiles interleave on the tensor core, so one tile's softmax
//     overlaps the other tile's MMAs.
//
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+HD) O1 [256+HD,256+2HD).
#pragma once

#include "sm100_ptx.cuh"

namespace axis_attn {

struct FwdArgs {
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, S;
  float scale_log2;  // scale * log2(e)
  int n_qblocks;     // ceil(S / 256)
};

template <int HD>
struct FwdCfg {
  static constexpr int NSLAB = HD / 64;                 // 64-column (128-byte) slabs
  static constexpr uint32_t SLAB = 128 * 128;           // 128 rows x 128 bytes
  static constexpr uint32_t TILE = NSLAB * SLAB;        // one 128 x HD bf16 tile
  static constexpr int ST = HD == 64 ? 3 : 2;           // K/V ring depth
  static constexpr int NBAR = 8 + 3 * ST;
  static constexpr uint32_t BAR_OFF = (2 + 2 * ST) * TILE;
  static constexpr uint32_t SMEM = BAR_OFF + 8 * NBAR + 16 + 1024;  // + alignment slack
};

enum FwdSite { F_Q = 1, F_EMPTY, F_KFULL, F_VFULL, F_PFULL, F_OBAR, F_SFULL, F_OWAIT, F_OFIN };

template <int HD, bool CAUSAL>
__global__ void __launch_bounds__(512, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  using C = FwdCfg<HD>;
  constexpr int ST = C::ST;
  constexpr uint32_t TILE = C::TILE, SLAB = C::SLAB;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t sQ = base, sK = base + 2 * TILE, sV = sK + ST * TILE;
  const uint32_t bars = base + C::BAR_OFF;
  const uint32_t bar_q = bars;
  auto bar_kfull = [&](int s) { return bars + 8u * (1 + s); };
  auto bar_vfull = [&](int s) { return bars + 8u * (1 + ST + s); };
  auto bar_empty = [&](int s) { return bars + 8u * (1 + 2 * ST + s); };
  auto bar_sfull = [&](int t) { return bars + 8u * (1 + 3 * ST + t); };
  auto bar_pfull = [&](int t) { return bars + 8u * (3 + 3 * ST + t); };
  auto bar_o = [&](int t) { return bars + 8u * (5 + 3 * ST + t); };
  const uint32_t bar_fin = bars + 8u * (7 + 3 * ST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::BAR_OFF + 8 * C::NBAR);
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + C::BAR_OFF + 8 * C::NBAR + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: heaviest query blocks first (causal), heads of a kv group adjacent
  const int BH = a.B * a.Hq;
  const int m = a.n_qblocks - 1 - (int)(blockIdx.x / BH);
  const int bh = (int)(blockIdx.x % BH);
  const int b = bh / a.Hq, h = bh % a.Hq;
  const int kvh = h / (a.Hq / a.Hkv);
  const int nkv = (a.S + 127) / 128;
  const int qt0 = 2 * m, qt1 = 2 * m + 1;
  const bool has1 = qt1 * 128 < a.S;
  const int n0 = CAUSAL ? qt0 + 1 : nkv;
  const int n1 = has1 ? (CAUSAL ? qt1 + 1 : nkv) : 0;
  const int nmax = n1 > n0 ? n1 : n0;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull(t), 1);
      mbar_init(bar_pfull(t), 4);
      mbar_init(bar_o(t), 1);
    }
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
    // ===================================================== TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bar_q, (has1 ? 2u : 1u) * TILE);
      for (int sl = 0; sl < C::NSLAB; ++sl)
        tma_load_4d(sQ + sl * SLAB, &tm_q, bar_q, 64 * sl, h, 128 * qt0, b);
      if (has1)
        for (int sl = 0; sl < C::NSLAB; ++sl)
          tma_load_4d(sQ + TILE + sl * SLAB, &tm_q, bar_q, 64 * sl, h, 128 * qt1, b);
      int issued = 0;
      for (int j = 0; j < nmax; ++j) {
        const int s = j % ST;
        const uint32_t ph = (j / ST) & 1;
        if (!mbar_wait_bounded(bar_empty(s), ph ^ 1, abort, F_EMPTY)) break;
        mbar_arrive_expect_tx(bar_kfull(s), TILE);
        for (int sl = 0; sl < C::NSLAB; ++sl)
          tma_load_4d(sK + s * TILE + sl * SLAB, &tm_k, bar_kfull(s), 64 * sl, kvh, 128 * j, b);
        mbar_arrive_expect_tx(bar_vfull(s), TILE);
        for (int sl = 0; sl < C::NSLAB; ++sl)
          tma_load_4d(sV + s * TILE + sl * SLAB, &tm_v, bar_vfull(s), 64 * sl, kvh, 128 * j, b);
        issued = j + 1;
      }
      // Drain: every copy this thread started has landed before the CTA exits.
      volatile int never = 0;
      mbar_wait_bounded(bar_q, 0, &never, F_Q);
      for (int j = issued - ST > 0 ? issued - ST : 0; j < issued; ++j) {
        mbar_wait_bounded(bar_kfull(j % ST), (j / ST) & 1, &never, F_KFULL);
        mbar_wait_bounded(bar_vfull(j % ST), (j / ST) & 1, &never, F_VFULL);
      }
    }
  } else if (warp == 13) {
    // ===================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
      constexpr uint32_t ID_PV = idesc_bf16(128, HD, 0, 1);   // P (TMEM) x V (MN-major)
      const int n[2] = {n0, n1};
      auto issue_s = [&](int t, int s) {
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * SLAB + (kk & 3) * 32;
          mma_ss(tmem + t * 128, sw128_desc(sQ + t * TILE + off, 16, 1024),
                 sw128_desc(sK + s * TILE + off, 16, 1024), ID_S, kk > 0);
        }
      };
      bool ok = mbar_wait_bounded(bar_q, 0, abort, F_Q) &&
                mbar_wait_bounded(bar_kfull(0), 0, abort, F_KFULL);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          if (n[t] > 0) {
            issue_s(t, 0);
            mma_commit(bar_sfull(t));
          }
      }
      for (int j = 0; ok && j < nmax; ++j) {
        const int s = j % ST;
        if (!mbar_wait_bounded(bar_vfull(s), (j / ST) & 1, abort, F_VFULL)) break;
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= n[t]) continue;
          if (!mbar_wait_bounded(bar_pfull(t), j & 1, abort, F_PFULL)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tO = tmem + 256 + t * HD, tP = tmem + t * 128;
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tO, tP + kk * 8, sw128_desc(sV + s * TILE + kk * 2048, SLAB, 1024), ID_PV,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar_o(t));
          const bool last_user = (t == 1) || (j >= n[1]);
          if (last_user) mma_commit(bar_empty(s));
          if (j + 1 < n[t]) {
            const int s1 = (j + 1) % ST;
            if (!mbar_wait_bounded(bar_kfull(s1), ((j + 1) / ST) & 1, abort, F_KFULL) ||
                !mbar_wait_bounded(bar_o(t), j & 1, abort, F_OBAR)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(t, s1);
            mma_commit(bar_sfull(t));
          }
        }
      }
      // Drain: all MMAs issued by this thread complete before TMEM is freed.
      mma_commit(bar_fin);
      volatile int never = 0;
      mbar_wait_bounded(bar_fin, 0, &never, F_OFIN);
    }
  } else if (warp < 8) {
    // ===================================================== softmax (tile t)
    const int t = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;                   // row in tile == TMEM lane
    const int n_t = t == 0 ? n0 : n1;
    const int qt = 2 * m + t;
    const int row_g = qt * 128 + r;
    const uint32_t tS = tmem + ((uint32_t)(wq * 32) << 16) + t * 128;
    const uint32_t tO = tmem + ((uint32_t)(wq * 32) << 16) + 256 + t * HD;
    const float c = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
      if (!wait_warp(bar_sfull(t), j & 1, abort, F_SFULL)) { ok = false; break; }
      tc_fence_after();
      const bool masked = CAUSAL ? (j == qt) : (j == nkv - 1 && (a.S & 127) != 0);
      int limit = 128;
      if (masked) {
        limit = a.S - 128 * j;
        if (CAUSAL && r + 1 < limit) limit = r + 1;
      }
      // pass 1: row max of the raw scores
      float mx = -INFINITY;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(tS + cc * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float x = __uint_as_float(v[i]);
          if (masked && cc * 32 + i >= limit) x = -INFINITY;
          mx = fmaxf(mx, x);
        }
      }
      const float m_new = fmaxf(m_used, mx * c);
      const bool resc = m_new > m_used + 8.0f;
      float alpha = 1.f;
      if (resc) {
        alpha = ex2_approx(m_used - m_new);
        m_used = m_new;
      }
      l *= alpha;
      // pass 2: p = 2^(s*c - m), row sum, bf16 P over the first half of S
      float rs = 0.f;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(tS + cc * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int col = cc * 32 + 2 * i;
          float p0 = ex2_approx(fmaf(__uint_as_float(v[2 * i]), c, -m_used));
          float p1 = ex2_approx(fmaf(__uint_as_float(v[2 * i + 1]), c, -m_used));
          if (masked && col >= limit) p0 = 0.f;
          if (masked && col + 1 >= limit) p1 = 0.f;
          rs += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + cc * 16, pk);
      }
      l += rs;
      // rescale O when the max moved (needs the previous P V to have landed)
      if (j > 0 && __any_sync(0xffffffffu, resc)) {
        if (!wait_warp(bar_o(t), (j - 1) & 1, abort, F_OWAIT)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < HD / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tO + cc * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
          tmem_st32(tO + cc * 32, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull(t));
    }
    // epilogue: O / l -> bf16, LSE = (m + log2 l) ln 2
    if (ok && n_t > 0 && wait_warp(bar_o(t), (n_t - 1) & 1, abort, F_OFIN)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = a.o + (((size_t)b * a.S + row_g) * a.Hq + h) * HD;
#pragma unroll 1
      for (int cc = 0; cc < HD / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tO + cc * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv_l, __uint_as_float(v[2 * i + 1]) * inv_l);
        if (row_g < a.S) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (row_g < a.S) a.lse[(size_t)bh * a.S + row_g] = (m_used + log2f(l)) * 0.69314718055994531f;
    }
  }
  // ---- teardown: every role has left its loop; free TMEM
  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace axis_attn
