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
//   * preprocess (HBM-bound): scale Dr and log2-scaled LSE per row, padded to a
//     multiple of 128 rows (padding rows get Dr = 0, LSE = +inf, so their P is
//     exactly 0); zero the fp32 dQ accumulator;
//   * main kernel: one CTA per (b, kv head, 128-key tile); K_j, V_j stay in
//     shared memory while the CTA walks every query head of the group and every
//     query tile that can see the keys.  Per tile (two threads issue the
//     MMAs, one the score products, one the gradient products):
//       S^T = K Q^T and dP^T = V dO^T into TMEM (thread = key row),
//       P^T = 2^(S^T c - LSE2), dS^T = P^T (dP^T - Dr) by the compute warps
//       (16 at D = 64, 8 at D = 128) from TMEM,
//       formed as scale dS^T = P^T (scale dP^T - scale Dr) (the preprocess
//       stores -scale Dr), so dQ and dK leave their products scaled,
//       P^T back to TMEM (bf16), dS^T to shared memory (bf16, 128B swizzle),
//       dV += P^T dO (A from TMEM), dK += dS^T Q, and dQ of the tile,
//     four read-out warps copy each dQ tile from TMEM into a swizzled
//     shared-memory staging tile, which one thread adds into the fp32
//     accumulator with TMA reduce-add copies; dK, dV stay in TMEM until the
//     end.  In the deterministic mode the kernel skips dQ altogether (the
//     separate pass of attn_bwd_dq.cuh recomputes it per query tile);
//   * dQ finalize (HBM-bound): bf16 copy of the accumulator in [B,S,Hq,D].
// D = 64 uses 128-row query tiles and dQ = dS K (TMEM lane = query row);
// D = 128 uses 64-row query tiles (shared memory) and dQ^T = K^T dS^T (TMEM
// lane = feature), so every MMA has M = 128.
#pragma once

#include "attn_rope.cuh"
#include "sm100_ptx.cuh"

namespace axis_attn {

// Compute warps (P^T, dS^T) at head dim 64 / 128: 16 (four per SM
// sub-partition, each thread a key row and a quarter of the 128 query
// columns, in 16-column chunks: more warps hide the TMEM, MUFU and barrier
// latencies of a step; measured 11% faster than 8 at D = 64) or 8 (two per
// sub-partition, half of the columns in 32-column chunks: at D = 128 a step
// has only 64 query columns, and 16 columns a thread measured 5% slower).
// Q / dO ring depth and dS^T buffers at D = 64 (D = 128: 3 and 1).  Two dS^T
// buffers let the compute warps write a step's dS^T while the dK and dQ
// products of the previous step still read theirs; they fit shared memory only
// with a 2-deep ring.  Measured (llm1b main kernel, same box): 3 / 1 251.5 us,
// 2 / 1 264.2 us, 2 / 2 270.0 us: the ring depth matters more than that wait.
#ifndef AXIS_ATTN_BWD_ST64
#define AXIS_ATTN_BWD_ST64 3
#endif
#ifndef AXIS_ATTN_BWD_NDS64
#define AXIS_ATTN_BWD_NDS64 1
#endif
#ifndef AXIS_ATTN_BWD_CW64
#define AXIS_ATTN_BWD_CW64 16
#endif
#ifndef AXIS_ATTN_BWD_CW128
#define AXIS_ATTN_BWD_CW128 8
#endif
// Unroll factor of the per-step loop over a compute thread's TMEM chunks.
#ifndef AXIS_ATTN_BWD_CC_UNROLL
#define AXIS_ATTN_BWD_CC_UNROLL 4
#endif

struct BwdArgs {
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* nlse2;  // [B*Hq][S_pad]  -LSE * log2(e); -inf on padding rows
  const float* ndr;    // [B*Hq][S_pad]  -rowsum(dO * O); 0 on padding rows
  float* dqacc;        // [B*Hq][S][HD] fp32, pre-scaled by `scale` (unused when no_dq)
  int B, Hq, Hkv, S, S_pad;
  float scale, scale_log2;
  int no_dq;           // 1: dK, dV only (deterministic mode: attn_bwd_dq_kernel computes dQ)
  const double2* rope_cs;  // RoPE: (cos, sin) table [S][HD/2], fp64; dK leaves through the transposed rotation
  // Head split (small grids): hsplit CTAs share a (b, kv head, key tile), each
  // taking G / hsplit of the group's query heads, and write fp32 partial dK
  // (x scale), dV to dk_part, dv_part [hsplit][B][S][Hkv][HD] for
  // attn_bwd_dkv_sum_kernel to add up; hsplit = 1: dK, dV straight to dk, dv.
  int hsplit;
  float* dk_part;
  float* dv_part;
};

template <int HD>
struct BwdCfg {
  static constexpr int BM = HD == 64 ? 128 : 64;   // query rows per step
  static constexpr bool QLANE = HD == 64;          // dQ lanes = query rows (else features)
  static constexpr int NSLAB = HD / 64;
  static constexpr uint32_t KSLAB = 128 * 128;     // 128 key rows x 128 bytes
  static constexpr uint32_t KTILE = NSLAB * KSLAB;
  static constexpr uint32_t QSLAB = BM * 128;      // BM query rows x 128 bytes
  static constexpr uint32_t QTILE = NSLAB * QSLAB;
  static constexpr uint32_t PS_BYTES = (BM / 64) * 128 * 128;  // dS^T: 128 keys x BM bf16
  static constexpr int ST = HD == 64 ? AXIS_ATTN_BWD_ST64 : 3;    // Q / dO / LSE / Dr ring depth
  static constexpr int NDS = HD == 64 ? AXIS_ATTN_BWD_NDS64 : 1;  // dS^T buffers
  // warps: 0 .. CW-1 compute; CW loads; CW+1 score MMAs (and TMEM owner);
  // CW+2 TMA reduce-adds; CW+3 gradient MMAs; CW+4 .. CW+7 dQ read-out
  static constexpr int CW = HD == 64 ? AXIS_ATTN_BWD_CW64 : AXIS_ATTN_BWD_CW128;
  static_assert(CW == 8 || CW == 16, "8 or 16 compute warps");
  static constexpr int THREADS = (CW + 8) * 32;
  static constexpr int W_LOAD = CW, W_MMA = CW + 1, W_RED = CW + 2, W_GRAD = CW + 3, W_DQ0 = CW + 4;
  static constexpr int COLS = BM / (CW / 4);                     // query columns per compute thread
  static constexpr int SUBW = CW == 16 ? 16 : 32;                // columns per TMEM load
  static constexpr int NSUB = COLS / SUBW;                       // loads per step
  // dQ tile staged for the TMA reduce-add: fp32, four 128B-swizzled boxes of
  // 32 columns x 64 rows (D = 64: rows = queries, columns = features; D = 128:
  // the tile is 64 queries x 128 features, one box per 32 features)
  static constexpr uint32_t DQ_BOX = 64 * 128;
  static constexpr uint32_t STAGE_BYTES = 4 * DQ_BOX;
  // shared-memory offsets from the 1024-aligned base
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = KTILE;
  static constexpr uint32_t OFF_Q = 2 * KTILE;
  static constexpr uint32_t OFF_DO = OFF_Q + ST * QTILE;
  static constexpr uint32_t OFF_DST = OFF_DO + ST * QTILE;
  static constexpr uint32_t OFF_STG = OFF_DST + NDS * PS_BYTES;
  static constexpr uint32_t OFF_LSE = OFF_STG + STAGE_BYTES;
  static constexpr uint32_t OFF_DR = OFF_LSE + ST * BM * 4;
  static constexpr uint32_t OFF_BAR = OFF_DR + ST * BM * 4;
  static constexpr int NBAR = 13 + 2 * ST;
  static constexpr uint32_t SMEM = OFF_BAR + 8 * NBAR + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
  // TMEM columns: S^T, dP^T, dV, dK, dQ tile, P^T (bf16 pairs)
  static constexpr uint32_t T_S = 0, T_DP = BM, T_DV = 2 * BM, T_DK = 2 * BM + HD, T_DQ = 2 * BM + 2 * HD,
                            T_P = T_DQ + 64;
  static_assert(T_P + BM / 2 <= 512, "TMEM budget");
};

// Which of the 16 column pairs of a 32-column block take the FP32-pipe
// polynomial for 2^x instead of the MUFU (bit i: pair i).
#ifndef AXIS_ATTN_BWD_POLY_MASK
#define AXIS_ATTN_BWD_POLY_MASK 0x0000
#endif

// P^T and dS^T of one chunk of a compute thread's key row (SUBW query columns
// from q_first): p = 2^(s c - LSE2) and scale dS = p (scale dp - scale Dr),
// each packed to bf16 pairs.  lse, dr: the staged -LSE2 and -scale Dr of those
// columns.  MASK (the diagonal or ragged step): p = 0 where the key lies above
// the query (causal) or past S; a template parameter, so that the other steps
// test nothing per pair.
template <int SUBW, bool MASK, bool CAUSAL>
__device__ __forceinline__ void bwd_chunk_math(const uint32_t (&sv)[SUBW], const uint32_t (&dpv)[SUBW],
                                               const float* lse, const float* dr, uint64_t cc2, uint64_t sc2,
                                               int key, int q_first, int S, uint32_t (&pk)[SUBW / 2],
                                               uint32_t (&dk)[SUBW / 2]) {
#pragma unroll
  for (int e = 0; e < SUBW; e += 4) {
    const float4 l4 = *reinterpret_cast<const float4*>(lse + e);
    const float4 d4 = *reinterpret_cast<const float4*>(dr + e);
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int ee = e + 2 * h2;
      const uint64_t nl = h2 ? f2_pack(l4.z, l4.w) : f2_pack(l4.x, l4.y);
      const uint64_t nd = h2 ? f2_pack(d4.z, d4.w) : f2_pack(d4.x, d4.y);
      const uint64_t x = f2_fma(f2_pack(__uint_as_float(sv[ee]), __uint_as_float(sv[ee + 1])), cc2, nl);
      float p0, p1;
      if ((AXIS_ATTN_BWD_POLY_MASK >> (ee / 2)) & 1) {
        f2_unpack(f2_exp2_poly(x), p0, p1);
      } else {
        float x0, x1;
        f2_unpack(x, x0, x1);
        p0 = ex2_approx(x0);
        p1 = ex2_approx(x1);
      }
      if constexpr (MASK) {
        const int q = q_first + ee;
        if ((CAUSAL && key > q) || key >= S) p0 = 0.f;
        if ((CAUSAL && key > q + 1) || key >= S) p1 = 0.f;
      }
      const uint64_t pp = f2_pack(p0, p1);
      const uint64_t dd =
          f2_mul(pp, f2_fma(f2_pack(__uint_as_float(dpv[ee]), __uint_as_float(dpv[ee + 1])), sc2, nd));
      pk[ee / 2] = pack_bf16x2(pp);
      dk[ee / 2] = pack_bf16x2(dd);
    }
  }
}

// Warps 0 .. CW-1: P^T / dS^T (thread = key row); CW loads; CW+1 issues the
// score MMAs and owns TMEM; CW+2 issues the TMA reduce-adds of the dQ tiles
// into the fp32 accumulator; CW+3 issues the gradient MMAs; CW+4 .. CW+7 copy
// each dQ tile from TMEM into the swizzled staging tile (one TMEM lane quarter
// each), off the compute warps' critical path (BwdCfg).
constexpr int BWD_CC_UNROLL = AXIS_ATTN_BWD_CC_UNROLL;

enum BwdSite { B_KV = 21, B_QEMPTY, B_QFULL, B_SPFREE, B_PDSFULL, B_DQFREE, B_SPFULL, B_DQFULL, B_FIN, B_PDSFREE,
               B_STGFULL, B_STGFREE };

// Swizzled store of 8 bf16 pairs (16 query columns) of one key row into a
// [key][query] 128B-swizzled buffer of 64-column slabs.
__device__ __forceinline__ void store_row16(uint32_t buf, int kr, int col0, const uint32_t* v) {
  const int slab = col0 >> 6, chunk = (col0 & 63) >> 3;
  const uint32_t rowaddr = buf + slab * (128 * 128) + (kr >> 3) * 1024 + (kr & 7) * 128;
  const uint32_t a0 = rowaddr + ((chunk ^ (kr & 7)) << 4);
  const uint32_t a1 = rowaddr + (((chunk + 1) ^ (kr & 7)) << 4);
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a0), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
               : "memory");
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a1), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// Launch order of the (key tile j, (b, kv head) unit) work items.  The
// (b, kv) units are taken in groups of UG; within a group the key tiles with
// the most query tiles come first (causal), every unit of the group at each
// key tile.  CTAs resident at the same time then share the Q and dO tiles and
// the dQ accumulator rows of only about UG units, which stay in L2; UG = 0
// puts all units in one group (key-tile-major order over the whole grid).
// Measured: UG = 8 is 1% (llm1b) to 3% (llm8b_gqa) faster than UG = 0, UG = 4
// 16% slower at llm1b (a group of 4 units at 16 key tiles is less than one
// wave of CTAs, so the light key tiles of one group wait behind the next).
#ifndef AXIS_ATTN_BWD_UNIT_GROUP
#define AXIS_ATTN_BWD_UNIT_GROUP 8
#endif
__device__ __forceinline__ void bwd_item(int BKV, int nkv, int x, int& j, int& bkv) {
  const int UG = AXIS_ATTN_BWD_UNIT_GROUP > 0 && AXIS_ATTN_BWD_UNIT_GROUP < BKV ? AXIS_ATTN_BWD_UNIT_GROUP : BKV;
  const int full = BKV / UG * UG;  // units in whole groups
  if (x < full * nkv) {
    const int g = x / (UG * nkv), r = x % (UG * nkv);
    j = r / UG;
    bkv = g * UG + r % UG;
  } else {  // the last, partial group
    const int rem = BKV - full, r = x - full * nkv;
    j = r / rem;
    bkv = full + r % rem;
  }
}

template <int HD, bool CAUSAL>
__global__ void __launch_bounds__(BwdCfg<HD>::THREADS, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdArgs a) {
  using C = BwdCfg<HD>;
  constexpr int BM = C::BM, ST = C::ST, COLS = C::COLS, SUBW = C::SUBW, NSUB = C::NSUB;
  constexpr int BWD_CW = C::CW, BWD_WARP_LOAD = C::W_LOAD, BWD_WARP_MMA = C::W_MMA, BWD_WARP_RED = C::W_RED,
                BWD_WARP_GRAD = C::W_GRAD, BWD_WARP_DQ0 = C::W_DQ0;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V;
  const uint32_t sDST = base + C::OFF_DST, sSTG = base + C::OFF_STG;
  auto sQ = [&](int s) { return base + C::OFF_Q + s * C::QTILE; };
  auto sDO = [&](int s) { return base + C::OFF_DO + s * C::QTILE; };
  const float* lse_s = reinterpret_cast<const float*>(gbase + C::OFF_LSE);
  const float* dr_s = reinterpret_cast<const float*>(gbase + C::OFF_DR);
  const uint32_t bars = base + C::OFF_BAR;
  const uint32_t bar_kv = bars;
  auto bar_qfull = [&](int s) { return bars + 8u * (1 + s); };
  auto bar_qempty = [&](int s) { return bars + 8u * (1 + ST + s); };
  const uint32_t bar_spfull = bars + 8u * (1 + 2 * ST);   // S^T, dP^T of a step are in TMEM
  const uint32_t bar_spfree = bars + 8u * (2 + 2 * ST);   // ... and have been read (the compute warps)
  const uint32_t bar_pdsfull = bars + 8u * (3 + 2 * ST);  // P^T (TMEM), dS^T (smem) written (the compute warps)
  const uint32_t bar_ptfree = bars + 8u * (4 + 2 * ST);   // dV of a step is done with P^T
  const uint32_t bar_dqfull = bars + 8u * (5 + 2 * ST);   // dQ tile of a step is in TMEM
  const uint32_t bar_dqfree = bars + 8u * (6 + 2 * ST);   // ... and has been read (4 read-out warps)
  const uint32_t bar_fin = bars + 8u * (7 + 2 * ST);
  // dK, dQ of a step are done with dS^T buffer x
  auto bar_dstfree = [&](int x) { return bars + 8u * (x == 0 ? 8 + 2 * ST : 11 + 2 * ST); };
  auto sDSB = [&](int it) { return sDST + (uint32_t)(it % C::NDS) * C::PS_BYTES; };  // dS^T buffer of step it
  const uint32_t bar_stgfull = bars + 8u * (9 + 2 * ST);  // dQ tile staged (4 read-out warps)
  const uint32_t bar_stgfree = bars + 8u * (10 + 2 * ST); // staged tile read by the TMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::OFF_BAR + 8 * C::NBAR);
  volatile WaitCtl* abort = reinterpret_cast<volatile WaitCtl*>(gbase + C::OFF_BAR + 8 * C::NBAR + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: key tile j of unit (b, kv head); with a head split, the
  // hsplit CTAs of a unit and key tile are adjacent in the launch order (they
  // share K_j, V_j in L2) and take consecutive blocks of the group's heads
  const int BKV = a.B * a.Hkv;
  const int hs = (int)blockIdx.x % a.hsplit;
  int j, bkv;
  bwd_item(BKV, (a.S + 127) / 128, (int)blockIdx.x / a.hsplit, j, bkv);
  const int b = bkv / a.Hkv, kvh = bkv % a.Hkv;
  const int G = a.Hq / a.Hkv / a.hsplit;  // query heads of this CTA
  const int h0 = kvh * (G * a.hsplit) + hs * G;
  const int nqt = (a.S + BM - 1) / BM;
  const int i0 = CAUSAL ? (128 * j) / BM : 0;
  const int per_head = nqt - i0;
  const int n_it = G * per_head;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar_qfull(s), 1);
      mbar_init(bar_qempty(s), 2);  // one commit from each MMA issuer
    }
    mbar_init(bar_spfull, 1);
    mbar_init(bar_spfree, BWD_CW);
    mbar_init(bar_pdsfull, BWD_CW);
    mbar_init(bar_ptfree, 1);
    mbar_init(bar_dqfull, 1);
    mbar_init(bar_dqfree, 4);
    mbar_init(bar_fin, 2);
    for (int x = 0; x < C::NDS; ++x) mbar_init(bar_dstfree(x), 1);
    mbar_init(bar_stgfull, 4);
    mbar_init(bar_stgfree, 1);
    wait_ctl_init(abort);
    fence_barrier_init();
  }
  if (warp == BWD_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == BWD_WARP_LOAD) {
    if (lane == 0) {
      // ===================================================== loads
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar_kv, 2 * C::KTILE);
      for (int sl = 0; sl < C::NSLAB; ++sl) {
        tma_load_4d(sK + sl * C::KSLAB, &tm_k, bar_kv, 64 * sl, kvh, 128 * j, b);
        tma_load_4d(sV + sl * C::KSLAB, &tm_v, bar_kv, 64 * sl, kvh, 128 * j, b);
      }
      // L2 prefetch of the Q / dO tiles PF steps ahead of the loads
      constexpr int PF = 4;
      auto prefetch = [&](int it) {
        const int h = h0 + it / per_head;
        const int q0 = (i0 + it % per_head) * BM;
        for (int sl = 0; sl < C::NSLAB; ++sl) {
          tma_prefetch_4d(&tm_q, 64 * sl, h, q0, b);
          tma_prefetch_4d(&tm_do, 64 * sl, h, q0, b);
        }
      };
      for (int it = 0; it < PF && it < n_it; ++it) prefetch(it);
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int s = it % ST;
        if (it + PF < n_it) prefetch(it + PF);
        if (!mbar_wait_bounded(bar_qempty(s), ((it / ST) & 1) ^ 1, abort, B_QEMPTY)) break;
        const int h = h0 + it / per_head;
        const int q0 = (i0 + it % per_head) * BM;
        const size_t row = ((size_t)b * a.Hq + h) * a.S_pad + q0;
        mbar_arrive_expect_tx(bar_qfull(s), 2 * C::QTILE + 2 * BM * 4);
        for (int sl = 0; sl < C::NSLAB; ++sl) {
          tma_load_4d(sQ(s) + sl * C::QSLAB, &tm_q, bar_qfull(s), 64 * sl, h, q0, b);
          tma_load_4d(sDO(s) + sl * C::QSLAB, &tm_do, bar_qfull(s), 64 * sl, h, q0, b);
        }
        bulk_load(base + C::OFF_LSE + s * BM * 4, a.nlse2 + row, BM * 4, bar_qfull(s));
        bulk_load(base + C::OFF_DR + s * BM * 4, a.ndr + row, BM * 4, bar_qfull(s));
        issued = it + 1;
      }
      volatile WaitCtl never = {0, 0, 0};  // drain: bounded by the time limit only
      mbar_wait_bounded(bar_kv, 0, &never, B_KV);
      for (int it = issued - ST > 0 ? issued - ST : 0; it < issued; ++it)
        mbar_wait_bounded(bar_qfull(it % ST), (it / ST) & 1, &never, B_QFULL);
    }
  } else if (warp == BWD_WARP_MMA || warp == BWD_WARP_GRAD) {
    // ===================================================== MMA issuers
    // Two warps issue the MMAs, each running as far ahead as its own barriers
    // allow: warp 9 the score products S^T = K Q^T, dP^T = V dO^T of every
    // step (into TMEM once the compute warps have read the previous ones),
    // warp 11 the gradient products of every step (dV, dK, dQ).  Q and dO of
    // a step are released once both have read them (qempty counts two
    // commits).  Each whole warp runs its loop (warp-uniform waits and
    // descriptors); lane 0 issues each MMA and commit.
    constexpr uint32_t ID_S = idesc_bf16(128, BM, 0, 0);   // K|V (K-major) x Q|dO (K-major)
    constexpr uint32_t ID_GV = idesc_bf16(128, HD, 0, 1);  // P^T (TMEM) | dS^T (smem, K-major) x dO|Q (MN-major)
    constexpr uint32_t ID_Q = C::QLANE ? idesc_bf16(128, HD, 1, 1) : idesc_bf16(128, BM, 1, 1);
    bool ok = wait_warp<true>(bar_kv, 0, abort, B_KV);
    if (warp == BWD_WARP_MMA) {
      for (int it = 0; ok && it < n_it; ++it) {
        const int s = it % ST;
        if (!wait_warp<true>(bar_qfull(s), (it / ST) & 1, abort, B_QFULL) ||
            (it > 0 && !wait_warp<true>(bar_spfree, (it - 1) & 1, abort, B_SPFREE)))
          break;
        tc_fence_after();
        // S^T = K Q^T and dP^T = V dO^T (reduction over the features)
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * C::KSLAB + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * C::QSLAB + (kk & 3) * 32;
          mma_ss_w(tmem + C::T_S, sw128_desc(sK + ko, 16, 1024), sw128_desc(sQ(s) + qo, 16, 1024), ID_S, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * C::KSLAB + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * C::QSLAB + (kk & 3) * 32;
          mma_ss_w(tmem + C::T_DP, sw128_desc(sV + ko, 16, 1024), sw128_desc(sDO(s) + qo, 16, 1024), ID_S,
                   kk > 0);
        }
        mma_commit_w(bar_spfull);
        mma_commit_w(bar_qempty(s));  // this warp is done with Q, dO of the step
      }
    } else {
      for (int it = 0; ok && it < n_it; ++it) {
        const int s = it % ST;
        if (!wait_warp<true>(bar_pdsfull, it & 1, abort, B_PDSFULL)) break;
        tc_fence_after();
        // dV += P^T dO (A = P^T from TMEM; reduction over the BM query rows)
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ts_w(tmem + C::T_DV, tmem + C::T_P + 8 * kk, sw128_desc(sDO(s) + kk * 2048, C::QSLAB, 1024), ID_GV,
                   (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit_w(bar_ptfree);
        // dK += dS^T Q
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t po = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          mma_ss_w(tmem + C::T_DK, sw128_desc(sDSB(it) + po, 16, 1024), sw128_desc(sQ(s) + kk * 2048, C::QSLAB, 1024),
                   ID_GV, (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_w(bar_qempty(s));  // this warp is done with Q, dO of the step
        if (a.no_dq) {  // dQ comes from the separate deterministic pass
          mma_commit_w(bar_dstfree(it % C::NDS));
          continue;
        }
        // dQ tile (reduction over the 128 keys) once the previous one has been read
        if (it >= 1 && !wait_warp<true>(bar_dqfree, (it - 1) & 1, abort, B_DQFREE)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ds_mn = sw128_desc(sDSB(it) + kk * 2048, 128 * 128, 1024);
          const uint64_t k_mn = sw128_desc(sK + kk * 2048, C::KSLAB, 1024);
          if (C::QLANE)
            mma_ss_w(tmem + C::T_DQ, ds_mn, k_mn, ID_Q, kk > 0);   // dQ = dS K
          else
            mma_ss_w(tmem + C::T_DQ, k_mn, ds_mn, ID_Q, kk > 0);   // dQ^T = K^T dS^T
        }
        mma_commit_w(bar_dqfull);
        mma_commit_w(bar_dstfree(it % C::NDS));
      }
    }
    // Drain: all MMAs issued by this warp complete before TMEM is freed.
    mma_commit_w(bar_fin);
    volatile WaitCtl never = {0, 0, 0};  // drain: bounded by the time limit only
    wait_warp<true>(bar_fin, 0, &never, B_FIN);
  } else if (warp == BWD_WARP_RED) {
    if (lane == 0 && !a.no_dq) {
      // ===================================================== dQ tiles -> fp32 accumulator (TMA reduce-add)
      tma_prefetch_desc(&tm_dq);
      for (int t = 0; t < n_it; ++t) {
        if (!mbar_wait_bounded(bar_stgfull, t & 1, abort, B_STGFULL)) break;
        const int h = h0 + t / per_head;
        const int q0 = (i0 + t % per_head) * BM;
        const int bh = b * a.Hq + h;
        for (int bx = 0; bx < 4; ++bx) {
          // D = 64: box (feature block bx & 1, row block bx >> 1); D = 128: feature block bx
          const int c0 = C::QLANE ? 32 * (bx & 1) : 32 * bx;
          const int r0 = C::QLANE ? q0 + 64 * (bx >> 1) : q0;
          if (r0 >= a.S) continue;
          tma_reduce_add_3d(&tm_dq, sSTG + bx * C::DQ_BOX, c0, r0, bh);
        }
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(bar_stgfree);
      }
      bulk_wait0();
    }
  } else if (warp >= BWD_WARP_DQ0) {
    // ===================================================== dQ tiles: TMEM -> staging tile
    // D = 64: TMEM lane = query row, 64 feature columns; D = 128: lane =
    // feature, 64 query-row columns.  Both halves of the tile go to the
    // staging tile as four 128B-swizzled fp32 boxes of 64 rows x 32 columns.
    if (!a.no_dq) {
      const int wq = warp & 3;
      const int kr = wq * 32 + lane;
      const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
      for (int t = 0; t < n_it; ++t) {
        if (!wait_warp(bar_dqfull, t & 1, abort, B_DQFULL)) break;
        if (t > 0 && !wait_warp(bar_stgfree, (t - 1) & 1, abort, B_STGFREE)) break;
        tc_fence_after();
        // one 32-column half at a time (32 registers); TMEM is released after the second load
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + C::T_DQ + 32 * ch, v);
          tmem_wait_ld();
          if (ch == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_dqfree);
          }
          if (C::QLANE) {
            // lane = query row kr, columns = features [32 ch, 32 ch + 32): one 128-byte box row
            // (dQ is already scaled: dS was formed scaled)
            const uint32_t row = sSTG + ((kr >> 6) * 2 + ch) * C::DQ_BOX + (kr & 63) * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(row + ((c ^ (kr & 7)) << 4)),
                           "r"(v[4 * c]), "r"(v[4 * c + 1]), "r"(v[4 * c + 2]), "r"(v[4 * c + 3])
                           : "memory");
          } else {
            // lane = feature kr (box kr / 32, column kr % 32), columns = query rows 32 ch + e
            const uint32_t boxb = sSTG + wq * C::DQ_BOX + ((lane & 3) << 2);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int q = 32 * ch + e;
              asm volatile("st.shared.b32 [%0], %1;" ::"r"(boxb + q * 128 + (((lane >> 2) ^ (q & 7)) << 4)),
                           "r"(v[e])
                           : "memory");
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_stgfull);
      }
    }
  } else if (warp < BWD_CW) {
    // ===================================================== P^T, dS^T (thread = key row)
    const int wq = warp & 3, ch = warp >> 2;  // lane quarter, column group
    const int kr = wq * 32 + lane;
    const int key = 128 * j + kr;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int c0 = ch * COLS;
    const uint64_t cc2 = f2_pack(a.scale_log2, a.scale_log2);
    const uint64_t sc2 = f2_pack(a.scale, a.scale);  // dS is formed scaled: P (scale dP - scale Dr)
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % ST;
      // the staged -LSE2 / -Dr rows of this step (TMA-written) and S^T, dP^T in TMEM
      if (!wait_warp(bar_qfull(s), (it / ST) & 1, abort, B_QFULL) ||
          !wait_warp(bar_spfull, it & 1, abort, B_SPFULL)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int q0 = (i0 + it % per_head) * BM;
      const bool need_mask = (CAUSAL && q0 < 128 * j + 127) || (128 * j + 128 > a.S);
      const float* lse_t = lse_s + s * BM + c0;
      const float* dr_t = dr_s + s * BM + c0;
#pragma unroll BWD_CC_UNROLL
      for (int cc = 0; cc < NSUB; ++cc) {
        uint32_t sv[SUBW], dpv[SUBW];
        if constexpr (SUBW == 32) {
          tmem_ld32(tmem + lane_off + C::T_S + c0 + SUBW * cc, sv);
          tmem_ld32(tmem + lane_off + C::T_DP + c0 + SUBW * cc, dpv);
        } else {
          tmem_ld16(tmem + lane_off + C::T_S + c0 + SUBW * cc, sv);
          tmem_ld16(tmem + lane_off + C::T_DP + c0 + SUBW * cc, dpv);
        }
        tmem_wait_ld();
        if (cc == NSUB - 1) {
          // all of this thread's S^T, dP^T are in registers: TMEM may take the next step's
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_spfree);
        }
        uint32_t pk[SUBW / 2], dk[SUBW / 2];
        // the mask test once per chunk, not per pair (need_mask is the same for the whole step)
        if (need_mask)
          bwd_chunk_math<SUBW, true, CAUSAL>(sv, dpv, lse_t + SUBW * cc, dr_t + SUBW * cc, cc2, sc2, key,
                                             q0 + c0 + SUBW * cc, a.S, pk, dk);
        else
          bwd_chunk_math<SUBW, false, CAUSAL>(sv, dpv, lse_t + SUBW * cc, dr_t + SUBW * cc, cc2, sc2, key,
                                              q0 + c0 + SUBW * cc, a.S, pk, dk);
        // the previous step's dV must be done with P^T before it is overwritten
        if (cc == 0 && it > 0 && !wait_warp(bar_ptfree, (it - 1) & 1, abort, B_PDSFREE)) {
          ok = false;
          break;
        }
        if constexpr (SUBW == 32)
          tmem_st16(tmem + lane_off + C::T_P + (c0 >> 1) + (SUBW / 2) * cc, pk);
        else
          tmem_st8(tmem + lane_off + C::T_P + (c0 >> 1) + (SUBW / 2) * cc, pk);
        // ... and the previous step's dK, dQ with dS^T
        // (with two buffers: the step before the previous one's)
        if (cc == 0 && it >= C::NDS &&
            !wait_warp(bar_dstfree(it % C::NDS), ((it - C::NDS) / C::NDS) & 1, abort, B_PDSFREE)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int x = 0; x < SUBW / 16; ++x) store_row16(sDSB(it), kr, c0 + SUBW * cc + 16 * x, &dk[8 * x]);
      }
      if (!ok) break;
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !(AXIS_ATTN_TEST_DROP_ARRIVE == 2 && it == 0)) mbar_arrive(bar_pdsfull);
    }
    // epilogue: the first half of the column groups writes dV, the second dK
    // (already scaled: dS was formed scaled); with 16 warps each group takes
    // half of the features
    constexpr int NG = BWD_CW / 4, GPT = NG / 2;  // column groups, groups per tensor
    if (ok && wait_warp(bar_fin, 0, abort, B_FIN)) {
      tc_fence_after();
      const bool is_dv = ch < GPT;
      const int f0 = (ch % GPT) * (HD / GPT);  // first feature of this group
      const uint32_t tcol = (is_dv ? C::T_DV : C::T_DK) + f0;
      const size_t row_off = (((size_t)b * a.S + key) * a.Hkv + kvh) * HD + f0;
      __nv_bfloat16* dst_row = (is_dv ? a.dv : a.dk) + row_off;
      float* part_row = a.hsplit > 1 ? (is_dv ? a.dv_part : a.dk_part) + (size_t)hs * a.B * a.S * a.Hkv * HD + row_off
                                     : nullptr;
#pragma unroll 1
      for (int cc = 0; cc < HD / GPT / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + tcol + cc * 32, v);
        tmem_wait_ld();
        if (part_row != nullptr) {  // head split: this CTA's fp32 share, summed (and rotated) later
          if (key < a.S) {
            float4* dst = reinterpret_cast<float4*>(part_row + cc * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                   __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
          continue;
        }
        uint32_t pk2[16];
        if (a.rope_cs != nullptr && !is_dv && key < a.S) {
          // dK = R(key)^T dK': pairs of features f0 + 32 cc + 2 i
          const double2* t = a.rope_cs + (size_t)key * (HD / 2) + (f0 + 32 * cc) / 2;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float g0 = __uint_as_float(v[2 * i]), g1 = __uint_as_float(v[2 * i + 1]);
            rope_back(g0, g1, t[i]);
            pk2[i] = pack_bf16x2(g0, g1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk2[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        }
        if (key < a.S) {
          uint4* dst = reinterpret_cast<uint4*>(dst_row + cc * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk2[4 * i], pk2[4 * i + 1], pk2[4 * i + 2], pk2[4 * i + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == BWD_WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// -scale Dr = -scale rowsum(dO * O) (fp32) and -LSE2 = -LSE * log2(e) per
// (b, h, i) (the backward forms dS scaled: P (scale dP - scale Dr)); rows
// S..S_pad-1 of each (b, h) get 0 and -inf (so their P is exactly 0).  Also
// zeroes the dQ accumulator (its own half of the blocks).  HBM-bound: D/8
// threads per row with one 16-byte load each of O and dO (every row a whole
// 128- or 256-byte line) and a shuffle reduction inside the row's thread group.  Rows are visited in [B, Hq, S]
// order, the order of the two fp32 outputs, so that consecutive rows of a warp
// write consecutive floats (in [B, S, Hq] order each 4-byte result would sit in
// a 32-byte sector of its own).
template <int HD>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dout,
                                                            const float* __restrict__ lse, float* nlse2,
                                                            float* ndr, float4* dqacc, size_t dq_vec4,
                                                            int Hq, int S, int S_pad, int rows, float scale) {
  constexpr int TPR = HD / 8;  // threads per row
  // With an accumulator to zero, the second half of the blocks does only that,
  // while the first half reads O and dO: the writes and the reads run at the
  // same time on different SMs (llm1b 29.8 -> 28.8 us against every thread
  // doing both in turn).
  const unsigned nb = dq_vec4 > 0 ? gridDim.x / 2 : gridDim.x;
  const bool zero_role = blockIdx.x >= nb;
  const size_t gtid = (size_t)(zero_role ? blockIdx.x - nb : blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t nthreads = (size_t)nb * blockDim.x;
  if (zero_role) {
    for (size_t k = gtid; k < dq_vec4; k += nthreads) dqacc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const size_t real_rows = (size_t)rows / S_pad * S;  // B * Hq * S, in [B, Hq, S] order
  const size_t total = real_rows * TPR;
  const size_t warp0 = gtid - (threadIdx.x & 31);  // warp-uniform loop: every lane joins the shuffles
  for (size_t tw = warp0; tw < total; tw += nthreads) {
    const size_t t = tw + (threadIdx.x & 31);
    const bool act = t < total;
    const size_t r = t / TPR;  // (b * Hq + h) * S + i
    const int part = (int)(t % TPR);
    const int i = (int)(r % S);
    const size_t bh = r / S;
    const size_t src = ((bh / Hq) * S + i) * Hq + bh % Hq;  // row of O, dO in [B, S, Hq]
    float d = 0.f;
    if (act) {
      const uint4 x = reinterpret_cast<const uint4*>(o + src * HD)[part];
      const uint4 y = reinterpret_cast<const uint4*>(dout + src * HD)[part];
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[k]));
        const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[k]));
        d = fmaf(xf.x, yf.x, d);
        d = fmaf(xf.y, yf.y, d);
      }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off, TPR);
    if (act && part == 0) {
      ndr[bh * S_pad + i] = -d * scale;
      nlse2[bh * S_pad + i] = -lse[bh * S + i] * 1.4426950408889634f;
    }
  }
  // padding rows of every (b, h)
  const int pad = S_pad - S;
  const size_t npad = (size_t)rows / S_pad * pad;
  for (size_t t = gtid; t < npad; t += nthreads) {
    const size_t bh = t / pad;
    const int i = S + (int)(t % pad);
    ndr[bh * S_pad + i] = 0.f;
    nlse2[bh * S_pad + i] = -INFINITY;
  }
}

// Iterations of a grid-stride loop whose loads a thread issues together
// before using any (one pair of 16-byte loads at a time per thread left the
// finalize at 0.75 of HBM bandwidth).
constexpr int BWD_STREAM_U = 4;

// dq[b,i,h,:] = bf16(dqacc[b,h,i,:]); 8 features per thread.  With a RoPE
// table the row leaves through the transposed rotation of position i.  The
// fp32 accumulator (twice the bytes of the output) is read in its own
// [B, Hq, S, D] order, 32 contiguous bytes per thread; the bf16 rows go to
// their [B, S, Hq, D] places as whole 128- or 256-byte lines.
template <int HD>
__global__ void __launch_bounds__(256, 4) attn_bwd_dq_convert_kernel(const float* __restrict__ dqacc,
                                                                     __nv_bfloat16* __restrict__ dq, int Hq,
                                                                     int S, size_t n8,
                                                                     const double2* __restrict__ rope_cs) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const float4* src = reinterpret_cast<const float4*>(dqacc);
  for (size_t k0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k0 < n8; k0 += BWD_STREAM_U * stride) {
    float4 x[BWD_STREAM_U], y[BWD_STREAM_U];
#pragma unroll
    for (int u = 0; u < BWD_STREAM_U; ++u) {
      const size_t k = k0 + u * stride;
      if (k < n8) {
        x[u] = src[2 * k];
        y[u] = src[2 * k + 1];
      }
    }
#pragma unroll
    for (int u = 0; u < BWD_STREAM_U; ++u) {
      const size_t k = k0 + u * stride;
      if (k >= n8) continue;
      const int c8 = (int)(k % (HD / 8));
      const size_t r = k / (HD / 8);  // (b * Hq + h) * S + i
      const int i = (int)(r % S);
      const size_t bh = r / S;
      const size_t row = (bh / Hq * S + i) * Hq + bh % Hq;  // (b * S + i) * Hq + h
      if (rope_cs != nullptr) {  // pairs 4 c8 .. 4 c8 + 3 at position i, transposed rotation
        const double2* t = rope_cs + (size_t)i * (HD / 2) + 4 * c8;
        rope_back(x[u].x, x[u].y, t[0]);
        rope_back(x[u].z, x[u].w, t[1]);
        rope_back(y[u].x, y[u].y, t[2]);
        rope_back(y[u].z, y[u].w, t[3]);
      }
      uint4 out;
      out.x = pack_bf16x2(x[u].x, x[u].y);
      out.y = pack_bf16x2(x[u].z, x[u].w);
      out.z = pack_bf16x2(y[u].x, y[u].y);
      out.w = pack_bf16x2(y[u].z, y[u].w);
      reinterpret_cast<uint4*>(dq + row * HD)[c8] = out;
    }
  }
}

// Head split: dk[b,j,kv,:] = bf16(sum over the hsplit partial rows), likewise
// dv; the partials are added in a fixed order (bitwise reproducible).  With a
// RoPE table dK leaves through the transposed rotation of position j.  8
// features per thread.
template <int HD>
__global__ void __launch_bounds__(256) attn_bwd_dkv_sum_kernel(const float* __restrict__ dk_part,
                                                               const float* __restrict__ dv_part,
                                                               __nv_bfloat16* __restrict__ dk,
                                                               __nv_bfloat16* __restrict__ dv, int hsplit,
                                                               int S, int Hkv, size_t n8,
                                                               const double2* __restrict__ rope_cs) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t part = n8 * 8;  // floats of one partial tensor
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < 2 * n8; k += stride) {
    const bool is_k = k < n8;
    const size_t e = is_k ? k : k - n8;  // 8-feature chunk in [B, S, Hkv, HD / 8]
    const float* src = (is_k ? dk_part : dv_part) + 8 * e;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
    for (int g = 0; g < hsplit; ++g) {
      const float4 a0 = reinterpret_cast<const float4*>(src + g * part)[0];
      const float4 a1 = reinterpret_cast<const float4*>(src + g * part)[1];
      x.x += a0.x; x.y += a0.y; x.z += a0.z; x.w += a0.w;
      y.x += a1.x; y.y += a1.y; y.z += a1.z; y.w += a1.w;
    }
    const int c8 = (int)(e % (HD / 8));
    if (is_k && rope_cs != nullptr) {
      const int pos = (int)((e / (HD / 8) / Hkv) % S);
      const double2* t = rope_cs + (size_t)pos * (HD / 2) + 4 * c8;
      rope_back(x.x, x.y, t[0]);
      rope_back(x.z, x.w, t[1]);
      rope_back(y.x, y.y, t[2]);
      rope_back(y.z, y.w, t[3]);
    }
    uint4 out;
    out.x = pack_bf16x2(x.x, x.y);
    out.y = pack_bf16x2(x.z, x.w);
    out.z = pack_bf16x2(y.x, y.y);
    out.w = pack_bf16x2(y.z, y.w);
    reinterpret_cast<uint4*>(is_k ? dk : dv)[e] = out;
  }
}

}  // namespace axis_attn
