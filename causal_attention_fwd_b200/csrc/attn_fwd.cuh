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
  // TMEM columns.  D = 64: S0 S1 O0 O1 P0 P1 (P has its own columns, so the
  // next S of a tile can be issued as soon as the softmax has read the last
  // one).  D = 128: S0 S1 O0 O1 fill all 512 columns and P (bf16) is written
  // over the first half of its S, so the next S waits for the P V product.
  static constexpr bool P_SEPARATE = HD == 64;
  static constexpr uint32_t T_S = 0, T_O = 256, T_P = P_SEPARATE ? 256 + 2 * HD : 0;
  static constexpr int NBAR = 10 + 3 * ST;
  static constexpr uint32_t BAR_OFF = (2 + 2 * ST) * TILE;
  static constexpr uint32_t SMEM = BAR_OFF + 8 * NBAR + 16 + 1024;  // + alignment slack
};

enum FwdSite { F_Q = 1, F_EMPTY, F_KFULL, F_VFULL, F_PFULL, F_OBAR, F_SFULL, F_OWAIT, F_OFIN };

// -inf for the columns at or after `limit` (causal diagonal / ragged tail).
__device__ __forceinline__ void mask_row(uint32_t (&v)[32], int col0, int limit) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (col0 + i >= limit) v[i] = __float_as_uint(-INFINITY);
}

__device__ __forceinline__ float row_max32(const uint32_t (&v)[32]) {
  float a = __uint_as_float(v[0]), b = __uint_as_float(v[1]), d = __uint_as_float(v[2]);
#pragma unroll
  for (int i = 3; i < 31; i += 6) {
    a = fmax3(a, __uint_as_float(v[i]), __uint_as_float(v[i + 1]));
    b = fmax3(b, __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
    d = fmax3(d, __uint_as_float(v[i + 4]), __uint_as_float(v[i + 5]));
  }
  return fmax3(a, b, fmax3(d, __uint_as_float(v[30]), __uint_as_float(v[31])));
}

// 32 scores -> 32 probabilities 2^(s*c - m): packed FMA for the argument,
// MUFU ex2 for the exponential, packed add into the running row sum, and the
// bf16 pairs stored to TMEM at column `tP` (16 columns).
__device__ __forceinline__ uint64_t exp_row32(const uint32_t (&v)[32], uint64_t cc2, uint64_t nm2, uint64_t acc,
                                              uint32_t tP) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), cc2, nm2);
    float x0, x1;
    f2_unpack(x, x0, x1);
    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    acc = f2_add(acc, f2_pack(p0, p1));
    pk[i] = pack_bf16x2(p0, p1);
  }
  tmem_st16(tP, pk);
  return acc;
}

// Warp roles: 0-3 softmax of Q tile 0, 4-7 softmax of Q tile 1, 8 TMA
// producer, 9 MMA issuer (and TMEM owner), 10-11 spare.  384 threads leave
// the softmax threads room (up to 168 registers) for a whole 128-column row.
constexpr int FWD_THREADS = 384;
constexpr int FWD_WARP_LOAD = 8;
constexpr int FWD_WARP_MMA = 9;

template <int HD, bool CAUSAL>
__global__ void __launch_bounds__(FWD_THREADS, 1)
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
  auto bar_sfree = [&](int t) { return bars + 8u * (8 + 3 * ST + t); };
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
      mbar_init(bar_sfree(t), 4);
    }
    mbar_init(bar_fin, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == FWD_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == FWD_WARP_LOAD) {
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
  } else if (warp == FWD_WARP_MMA) {
    // ===================================================== MMA issuer
    // Event loop over the two query tiles: issue whichever MMA has its inputs
    // ready (non-blocking tests), so one tile's wait never idles the tensor
    // core while the other tile has work.
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
      constexpr uint32_t ID_PV = idesc_bf16(128, HD, 0, 1);   // P (TMEM) x V (MN-major)
      const int n[2] = {n0, n1};
      auto issue_s = [&](int t, int s) {
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * SLAB + (kk & 3) * 32;
          mma_ss(tmem + C::T_S + t * 128, sw128_desc(sQ + t * TILE + off, 16, 1024),
                 sw128_desc(sK + s * TILE + off, 16, 1024), ID_S, kk > 0);
        }
      };
      bool ok = mbar_wait_bounded(bar_q, 0, abort, F_Q);
      int js[2] = {0, 0}, jp[2] = {0, 0};  // next S / next P V to issue, per tile
      int pv_users[ST];                    // P V products issued per K/V stage
      for (int q = 0; q < ST; ++q) pv_users[q] = 0;
      Watchdog wd;
      while (ok && (jp[0] < n[0] || jp[1] < n[1])) {
        bool moved = false;
        for (int t = 0; t < 2; ++t) {
          // O_t += P_t V_j
          if (jp[t] < js[t]) {
            const int j = jp[t], s = j % ST;
            if (mbar_test(bar_pfull(t), j & 1) && mbar_test(bar_vfull(s), (j / ST) & 1)) {
              tc_fence_after();
              const uint32_t tO = tmem + C::T_O + t * HD;
              const uint32_t tP = tmem + C::T_P + t * (C::P_SEPARATE ? 64 : 128);
              for (int kk = 0; kk < 8; ++kk)
                mma_ts(tO, tP + kk * 8, sw128_desc(sV + s * TILE + kk * 2048, SLAB, 1024), ID_PV,
                       (j > 0 || kk > 0) ? 1u : 0u);
              mma_commit(bar_o(t));
              // the K/V stage is free once every tile that uses kv tile j is done with it
              if (++pv_users[s] == (j < n[0]) + (j < n[1])) {
                pv_users[s] = 0;
                mma_commit(bar_empty(s));
              }
              ++jp[t];
              moved = true;
            }
          }
          // S_t = Q_t K_j^T once S_t's columns are free
          if (js[t] < n[t]) {
            const int j = js[t], s = j % ST;
            bool free_ = true;
            if (j > 0)
              free_ = C::P_SEPARATE ? mbar_test(bar_sfree(t), (j - 1) & 1)
                                    : (jp[t] >= j && mbar_test(bar_o(t), (j - 1) & 1));
            if (free_ && mbar_test(bar_kfull(s), (j / ST) & 1)) {
              tc_fence_after();
              issue_s(t, s);
              mma_commit(bar_sfull(t));
              ++js[t];
              moved = true;
            }
          }
        }
        if (moved) {
          wd.progress();
        } else {
          if (wd.stalled(abort, F_PFULL)) ok = false;
          __nanosleep(32);  // idle pass: leave issue slots to the softmax warps of this SM sub-partition
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
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::T_S + t * 128;
    const uint32_t tO = tmem + lane_off + C::T_O + t * HD;
    const uint32_t tP = tmem + lane_off + C::T_P + t * (C::P_SEPARATE ? 64 : 128);
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
      // the whole 128-column row of S in registers (one TMEM pass)
      uint32_t v0[32], v1[32], v2[32], v3[32];
      tmem_ld32(tS, v0);
      tmem_ld32(tS + 32, v1);
      tmem_ld32(tS + 64, v2);
      tmem_ld32(tS + 96, v3);
      tmem_wait_ld();
      if (C::P_SEPARATE) {
        // S_t is in registers: its columns may take the next S
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sfree(t));
      }
      if (masked) {
        mask_row(v0, 0, limit);
        mask_row(v1, 32, limit);
        mask_row(v2, 64, limit);
        mask_row(v3, 96, limit);
      }
      const float mx = fmax3(fmax3(row_max32(v0), row_max32(v1), row_max32(v2)), row_max32(v3), -INFINITY);
      const float m_new = fmaxf(m_used, mx * c);
      const bool resc = m_new > m_used + 8.0f;
      float alpha = 1.f;
      if (resc) {
        alpha = ex2_approx(m_used - m_new);
        m_used = m_new;
      }
      // the previous P V must have landed before P_t is overwritten and O_t rescaled
      if (j > 0) {
        if (!wait_warp(bar_o(t), (j - 1) & 1, abort, F_OWAIT)) { ok = false; break; }
        tc_fence_after();
      }
      // p = 2^(s*c - m) (masked entries are -inf and give 0), row sum, bf16 P
      const uint64_t cc2 = f2_pack(c, c), nm2 = f2_pack(-m_used, -m_used);
      uint64_t acc = f2_pack(0.f, 0.f);
      acc = exp_row32(v0, cc2, nm2, acc, tP);
      acc = exp_row32(v1, cc2, nm2, acc, tP + 16);
      acc = exp_row32(v2, cc2, nm2, acc, tP + 32);
      acc = exp_row32(v3, cc2, nm2, acc, tP + 48);
      float rs_lo, rs_hi;
      f2_unpack(acc, rs_lo, rs_hi);
      l = l * alpha + (rs_lo + rs_hi);
      // rescale O when the max moved
      if (j > 0 && __any_sync(0xffffffffu, resc)) {
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
  if (warp == FWD_WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace axis_attn
