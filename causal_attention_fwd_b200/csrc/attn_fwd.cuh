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
  // K and V rings (separate: a K stage is free once both S products have read
  // it, long before the P V products free the V stage)
  static constexpr int KST = HD == 64 ? 5 : 3;
  static constexpr int VST = HD == 64 ? 5 : 2;
  // TMEM columns.  D = 64: S0 S1 O0 O1 P0 P1 (P has its own columns, so the
  // next S of a tile can be issued as soon as the softmax has read the last
  // one).  D = 128: S0 S1 O0 O1 fill all 512 columns and P (bf16) is written
  // over the first half of its S, so the next S waits for the P V product.
  static constexpr bool P_SEPARATE = HD == 64;
  static constexpr uint32_t T_S = 0, T_O = 256, T_P = P_SEPARATE ? 256 + 2 * HD : 0;
  static constexpr int NBAR = 12 + 2 * KST + 2 * VST;
  static constexpr uint32_t BAR_OFF = (2 + KST + VST) * TILE;
  static constexpr uint32_t SMEM = BAR_OFF + 8 * NBAR + 16 + 1024;  // + alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
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
// bf16 pairs into `pk`
// (16 registers, to be stored to TMEM).
__device__ __forceinline__ uint64_t exp_row32(const uint32_t (&v)[32], uint64_t cc2, uint64_t nm2, uint64_t acc,
                                              uint32_t (&pk)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), cc2, nm2);
    float x0, x1;
    f2_unpack(x, x0, x1);
    const uint64_t pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
    acc = f2_add(acc, pp);
    pk[i] = pack_bf16x2(pp);
  }
  return acc;
}

// Warp roles: 0-3 softmax of Q tile 0, 4-7 softmax of Q tile 1, 8 TMA
// producer of Q and K, 9 MMA issuer (and TMEM owner), 10 TMA producer of V,
// 11 spare.  384 threads leave
// the softmax threads room (up to 168 registers) for a whole 128-column row.
constexpr int FWD_THREADS = 384;
constexpr int FWD_WARP_LOAD = 8;
constexpr int FWD_WARP_MMA = 9;
constexpr int FWD_WARP_LOADV = 10;

template <int HD, bool CAUSAL>
__global__ void __launch_bounds__(FWD_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  using C = FwdCfg<HD>;
  constexpr int KST = C::KST, VST = C::VST;
  constexpr uint32_t TILE = C::TILE, SLAB = C::SLAB;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t sQ = base, sK = base + 2 * TILE, sV = sK + KST * TILE;
  const uint32_t bars = base + C::BAR_OFF;
  const uint32_t bar_q = bars;
  auto bar_kfull = [&](int s) { return bars + 8u * (1 + s); };
  auto bar_kempty = [&](int s) { return bars + 8u * (1 + KST + s); };
  auto bar_vfull = [&](int s) { return bars + 8u * (1 + 2 * KST + s); };
  auto bar_vempty = [&](int s) { return bars + 8u * (1 + 2 * KST + VST + s); };
  constexpr int B2 = 1 + 2 * KST + 2 * VST;
  auto bar_sfull = [&](int t) { return bars + 8u * (B2 + t); };
  auto bar_pfull = [&](int t) { return bars + 8u * (B2 + 2 + t); };
  auto bar_o = [&](int t) { return bars + 8u * (B2 + 4 + t); };
  const uint32_t bar_fin = bars + 8u * (B2 + 6);
  auto bar_sfree = [&](int t) { return bars + 8u * (B2 + 7 + t); };
  // exponential-phase token: warpgroup t may start its k-th exponential phase
  // once the other warpgroup has finished its own k-th (t = 1) or (k-1)-th
  // (t = 0); the two phases then alternate and each has the MUFU to itself
  auto bar_tok = [&](int t) { return bars + 8u * (B2 + 9 + t); };
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
    for (int s = 0; s < KST; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_kempty(s), 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull(t), 1);
      mbar_init(bar_pfull(t), 4);
      mbar_init(bar_o(t), 1);
      mbar_init(bar_sfree(t), 4);
      mbar_init(bar_tok(t), 4);
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

  if (warp == FWD_WARP_LOAD || warp == FWD_WARP_LOADV) {
    // ===================================================== TMA producers
    // warp 8: Q once, then the K ring (with an L2 prefetch of K and V PF
    // tiles ahead); warp 10: the V ring.  Each lane-0 loop blocks (in
    // hardware) on the stage it needs next; K stages free up long before V
    // stages, so the two rings run independently.
    if (lane == 0) {
      const bool is_k = warp == FWD_WARP_LOAD;
      int issued = 0;
      if (is_k) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        mbar_arrive_expect_tx(bar_q, (has1 ? 2u : 1u) * TILE);
        for (int sl = 0; sl < C::NSLAB; ++sl)
          tma_load_4d(sQ + sl * SLAB, &tm_q, bar_q, 64 * sl, h, 128 * qt0, b);
        if (has1)
          for (int sl = 0; sl < C::NSLAB; ++sl)
            tma_load_4d(sQ + TILE + sl * SLAB, &tm_q, bar_q, 64 * sl, h, 128 * qt1, b);
        constexpr int PF = 4;
        auto prefetch = [&](int j) {
          for (int sl = 0; sl < C::NSLAB; ++sl) {
            tma_prefetch_4d(&tm_k, 64 * sl, kvh, 128 * j, b);
            tma_prefetch_4d(&tm_v, 64 * sl, kvh, 128 * j, b);
          }
        };
        for (int j = 0; j < PF && j < nmax; ++j) prefetch(j);
        for (int j = 0; j < nmax; ++j) {
          const int s = j % KST;
          if (j >= KST && !mbar_wait_bounded(bar_kempty(s), ((j / KST) & 1) ^ 1, abort, F_EMPTY)) break;
          mbar_arrive_expect_tx(bar_kfull(s), TILE);
          for (int sl = 0; sl < C::NSLAB; ++sl)
            tma_load_4d(sK + s * TILE + sl * SLAB, &tm_k, bar_kfull(s), 64 * sl, kvh, 128 * j, b);
          if (j + PF < nmax) prefetch(j + PF);
          issued = j + 1;
        }
      } else {
        tma_prefetch_desc(&tm_v);
        for (int j = 0; j < nmax; ++j) {
          const int s = j % VST;
          if (j >= VST && !mbar_wait_bounded(bar_vempty(s), ((j / VST) & 1) ^ 1, abort, F_EMPTY)) break;
          mbar_arrive_expect_tx(bar_vfull(s), TILE);
          for (int sl = 0; sl < C::NSLAB; ++sl)
            tma_load_4d(sV + s * TILE + sl * SLAB, &tm_v, bar_vfull(s), 64 * sl, kvh, 128 * j, b);
          issued = j + 1;
        }
      }
      // Drain: every copy this thread started has landed before the CTA exits.
      volatile int never = 0;
      if (is_k) {
        mbar_wait_bounded(bar_q, 0, &never, F_Q);
        for (int j = issued - KST > 0 ? issued - KST : 0; j < issued; ++j)
          mbar_wait_bounded(bar_kfull(j % KST), (j / KST) & 1, &never, F_KFULL);
      } else {
        for (int j = issued - VST > 0 ? issued - VST : 0; j < issued; ++j)
          mbar_wait_bounded(bar_vfull(j % VST), (j / VST) & 1, &never, F_VFULL);
      }
    }
  } else if (warp == FWD_WARP_MMA) {
    // ===================================================== MMA issuer
    // A fixed issue order that follows the softmax ping-pong, with blocking
    // (hardware-suspended) waits:
    //   D = 64  (P has its own columns):  S0(j+1) S1(j+1) PV0(j) PV1(j)
    //   D = 128 (P over S):               PV0(j) S0(j+1) PV1(j) S1(j+1)
    // Every wait is on an item that an earlier entry of the order enables, so
    // the order cannot deadlock.  The whole warp runs the loop with
    // warp-uniform waits; lane 0 issues each instruction.
    {
      constexpr uint32_t ID_S = idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
      constexpr uint32_t ID_PV = idesc_bf16(128, HD, 0, 1);   // P (TMEM) x V (MN-major)
      const int n[2] = {n0, n1};
      uint32_t pv_users = 0, s_users = 0;  // products issued per V / K stage (2-bit counters)
      auto do_s = [&](int t, int j) -> bool {  // S_t = Q_t K_j^T
        const int s = j % KST;
        if (j > 0) {
          const bool f = C::P_SEPARATE ? wait_warp(bar_sfree(t), (j - 1) & 1, abort, F_SFULL)
                                       : wait_warp(bar_o(t), (j - 1) & 1, abort, F_OBAR);
          if (!f) return false;
        }
        if (!wait_warp(bar_kfull(s), (j / KST) & 1, abort, F_KFULL)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * SLAB + (kk & 3) * 32;
          mma_ss_w(tmem + C::T_S + t * 128, sw128_desc(sQ + t * TILE + off, 16, 1024),
                   sw128_desc(sK + s * TILE + off, 16, 1024), ID_S, kk > 0);
        }
        mma_commit_w(bar_sfull(t));
        s_users += 1u << (2 * s);
        if (((s_users >> (2 * s)) & 3u) == (uint32_t)((j < n[0]) + (j < n[1]))) {
          s_users &= ~(3u << (2 * s));
          mma_commit_w(bar_kempty(s));
        }
        return true;
      };
      auto do_pv = [&](int t, int j) -> bool {  // O_t += P_t V_j
        const int s = j % VST;
        if (!wait_warp(bar_pfull(t), j & 1, abort, F_PFULL) || !wait_warp(bar_vfull(s), (j / VST) & 1, abort, F_VFULL))
          return false;
        tc_fence_after();
        const uint32_t tO = tmem + C::T_O + t * HD;
        const uint32_t tP = tmem + C::T_P + t * (C::P_SEPARATE ? 64 : 128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts_w(tO, tP + kk * 8, sw128_desc(sV + s * TILE + kk * 2048, SLAB, 1024), ID_PV,
                   (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit_w(bar_o(t));
        pv_users += 1u << (2 * s);
        if (((pv_users >> (2 * s)) & 3u) == (uint32_t)((j < n[0]) + (j < n[1]))) {
          pv_users &= ~(3u << (2 * s));
          mma_commit_w(bar_vempty(s));
        }
        return true;
      };
      bool ok = wait_warp(bar_q, 0, abort, F_Q);
      for (int t = 0; t < 2 && ok; ++t)
        if (n[t] > 0) ok = do_s(t, 0);
      for (int j = 0; ok && j < nmax; ++j) {
        if (C::P_SEPARATE) {
          for (int t = 0; t < 2 && ok; ++t)
            if (j + 1 < n[t]) ok = do_s(t, j + 1);
          for (int t = 0; t < 2 && ok; ++t)
            if (j < n[t]) ok = do_pv(t, j);
        } else {
          for (int t = 0; t < 2 && ok; ++t) {
            if (j < n[t]) ok = do_pv(t, j);
            if (ok && j + 1 < n[t]) ok = do_s(t, j + 1);
          }
        }
      }
      // Drain: all MMAs issued by this warp complete before TMEM is freed.
      mma_commit_w(bar_fin);
      volatile int never = 0;
      wait_warp(bar_fin, 0, &never, F_OFIN);
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
      // take turns with the other warpgroup on the exponentials
      {
        const int other_n = t == 0 ? n1 : n0;
        const int need = t == 0 ? j - 1 : j;   // the other warpgroup's phase to wait for
        if (need >= 0 && need < other_n && !wait_warp(bar_tok(t), need & 1, abort, F_SFULL)) {
          ok = false;
          break;
        }
      }
      // p = 2^(s*c - m) (masked entries are -inf and give 0), row sum, bf16 P
      // pairs in registers: the exponentials overlap the previous P V
      const uint64_t cc2 = f2_pack(c, c), nm2 = f2_pack(-m_used, -m_used);
      uint64_t acc = f2_pack(0.f, 0.f);
      uint32_t pk0[16], pk1[16], pk2[16], pk3[16];
      acc = exp_row32(v0, cc2, nm2, acc, pk0);
      acc = exp_row32(v1, cc2, nm2, acc, pk1);
      acc = exp_row32(v2, cc2, nm2, acc, pk2);
      acc = exp_row32(v3, cc2, nm2, acc, pk3);
      float rs_lo, rs_hi;
      f2_unpack(acc, rs_lo, rs_hi);
      l = l * alpha + (rs_lo + rs_hi);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_tok(1 - t));  // hand the MUFU to the other warpgroup
      // the previous P V must have landed before P_t is overwritten and O_t rescaled
      if (j > 0) {
        if (!wait_warp(bar_o(t), (j - 1) & 1, abort, F_OWAIT)) { ok = false; break; }
        tc_fence_after();
      }
      tmem_st16(tP, pk0);
      tmem_st16(tP + 16, pk1);
      tmem_st16(tP + 32, pk2);
      tmem_st16(tP + 48, pk3);
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
