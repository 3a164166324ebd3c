// attn_fwd.cuh -- forward kernel: O = softmax(scale * Q K^T, causal mask) V and
// the per-row log-sum-exp.  Persistent: one CTA per SM walks a list of work
// items, each 256 query rows of one (batch, query head) (128 rows when items
// of 256 would leave SMs idle).
//
// What it computes is the fused attention forward of the Axis page
// (zyoralabs.com/axis, feature list: fused flash attention; bf16 storage, fp32
// accumulation; probabilities never reach memory): scores and probabilities
// live only in tensor memory.  How, on sm_100a:
//
//   * a work item is two 128-row query tiles (Q0, Q1) of one (b, h); they
//     share a ring of K tiles and a ring of V tiles (128 keys each) that two
//     TMA threads stream in.  When two-tile items would be fewer than the
//     SMs, an item is one tile (Q1 absent, as for a ragged last block): twice
//     the items and half the longest chain of kv tiles.  Items are dealt heaviest first (causal) in a
//     snake order over the CTAs, which balances the causal triangle;
//   * two threads issue the tcgen05.mma work, one S_t = Q_t K_j^T (both
//     operands K-major in shared memory) into TMEM, the other O_t += P_t V_j
//     with P_t read from TMEM (bf16) and V_j MN-major in smem; each runs ahead
//     as far as its own barriers allow, so neither waits behind the other's
//     queue;
//   * two warpgroups per query tile run the online softmax in the log2 domain
//     from TMEM (thread = half a row: warps w and w + 4 share TMEM lanes and
//     take columns 0-63 and 64-127): row max (the halves swap partial maxima
//     through shared memory), p = 2^(s*c - m), row sum, P back to TMEM.  Two
//     warps per SM sub-partition keep the MUFU busy through the exponentials,
//     which one warp alone cannot (its in-order issue leaves the MUFU idle
//     while it issues the FMA-pipe work).  The running max is only moved when
//     it grows by more than 8 (a factor 256), so the O rescale in TMEM is rare;
//     stale-max values stay below 2^8 and are exact to bf16 relative precision;
//   * the two query tiles run their softmax phases independently, so one
//     tile's exponentials overlap the other tile's TMEM traffic, row max and
//     MMAs (forcing them to alternate with a token barrier, reading the other
//     half's scores from TMEM instead of exchanging partial maxima, one
//     thread per whole row, and starting the exponentials before the
//     exchange completes all measured slower);
//   * causal: kv tiles after a query tile's diagonal are never loaded or
//     multiplied; the element mask runs only on the diagonal (and ragged last)
//     tile;
//   * across items: the next item's Q is loaded as soon as the last S product
//     of the current one has read Q, and its first P V product waits only for
//     the epilogue to have read O out of TMEM.
//
// TMEM columns: D = 64: S0 [0,128) S1 [128,256) O0 [256,320) O1 [320,384)
// P0 [384,448) P1 [448,512); D = 128: S [0,128) (shared by the two tiles, which
// take turns) P0 [128,192) P1 [192,256) O0 [256,384) O1 [384,512).
#pragma once

#include "sm100_ptx.cuh"

namespace axis_attn {

struct FwdArgs {
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, S;
  float scale_log2;  // scale * log2(e)
  int tpi;           // 128-row query tiles per item: 2, or 1 when two-tile items cannot fill the SMs
  int n_qblocks;     // ceil(S / (128 * tpi))
  int n_items;       // n_qblocks * B * Hq
};

// The it-th item of this CTA: snake order over the grid (even passes left to
// right, odd passes right to left), so that with items sorted heaviest first
// every CTA gets a near-equal share of the causal triangle.
__device__ __forceinline__ int fwd_item(int it) {
  const int G = (int)gridDim.x;
  const int c = (it & 1) ? G - 1 - (int)blockIdx.x : (int)blockIdx.x;
  return it * G + c;
}

struct FwdItem {
  int b, h, bh, kvh, qt0;  // batch, head, b * Hq + h, kv head, first 128-row query tile
  int n0, n1, nmax;        // kv tiles of query tile 0 / 1 (0: no tile 1), max
  bool has1;
};

__device__ __forceinline__ FwdItem fwd_decode(const FwdArgs& a, int w, bool causal) {
  FwdItem it;
  const int BH = a.B * a.Hq;
  const int m = a.n_qblocks - 1 - w / BH;  // heaviest (last) query blocks first
  it.bh = w % BH;
  it.b = it.bh / a.Hq;
  it.h = it.bh % a.Hq;
  it.kvh = it.h / (a.Hq / a.Hkv);
  const int nkv = (a.S + 127) / 128;
  const int qt0 = a.tpi * m, qt1 = qt0 + 1;
  it.qt0 = qt0;
  it.has1 = a.tpi == 2 && qt1 * 128 < a.S;
  it.n0 = causal ? qt0 + 1 : nkv;
  it.n1 = it.has1 ? (causal ? qt1 + 1 : nkv) : 0;
  it.nmax = it.n1 > it.n0 ? it.n1 : it.n0;
  return it;
}

template <int HD>
struct FwdCfg {
  static constexpr int NSLAB = HD / 64;                 // 64-column (128-byte) slabs
  static constexpr uint32_t SLAB = 128 * 128;           // 128 rows x 128 bytes
  static constexpr uint32_t TILE = NSLAB * SLAB;        // one 128 x HD bf16 tile
  // K and V rings (separate: a K stage is free once both S products have read
  // it, long before the P V products free the V stage)
  static constexpr int KST = HD == 64 ? 5 : 2;
  static constexpr int VST = HD == 64 ? 5 : 2;
  // TMEM columns (512).  D = 64: S0 S1 O0 O1 P0 P1.  D = 128: one S shared by
  // the two tiles, P0 P1, O0 O1 (the tiles take turns, so S alternates between
  // them; the S of one tile is issued as soon as the other tile has read its
  // own out).  P always has its own columns: the next S never waits for a
  // P V product.
  static constexpr bool SHARED_S = HD == 128;
  static constexpr uint32_t T_P = SHARED_S ? 128 : 384, T_O = 256;
  static __host__ __device__ constexpr uint32_t t_s(int t) { return SHARED_S ? 0u : 128u * t; }
  static constexpr int NBAR = 21 + 2 * KST + 2 * VST;
  static constexpr uint32_t XCH_OFF = (2 + KST + VST) * TILE;  // row-max / row-sum exchange
  static constexpr uint32_t XCH_BYTES = 2 * 2 * 2 * 128 * 4;   // [parity][tile][half][row] fp32
  static constexpr uint32_t BAR_OFF = XCH_OFF + XCH_BYTES;
  static constexpr uint32_t SMEM = BAR_OFF + 8 * NBAR + 16 + 1024;  // + alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
};

enum FwdSite { F_Q = 1, F_EMPTY, F_KFULL, F_VFULL, F_PFULL, F_OBAR, F_SFULL, F_OWAIT, F_OFIN, F_XCH, F_QEMPTY,
               F_OFREE };

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

// Which of the 16 column pairs of a 32-column block take the FP32-pipe
// polynomial for 2^x instead of the MUFU (bit i: pair i).  The MUFU does 16
// exponentials per clock per SM, which at head dim 64 is below the rate of
// the two MMAs; moving a share of them to the FP32 pipe balances the two.
#ifndef AXIS_ATTN_FWD_POLY_MASK
#define AXIS_ATTN_FWD_POLY_MASK 0x0000
#endif
// Scores v[2 I0 .. 2 (I0 + N)) -> probabilities 2^(s*c - m): packed FMA for
// the argument, MUFU ex2 (or the polynomial, for the pairs the mask selects)
// for the exponential, packed add into the running row sum, and the bf16
// pairs into pk[I0 .. I0 + N) (to be stored to TMEM).
template <int I0, int N>
__device__ __forceinline__ uint64_t exp_pairs(const uint32_t (&v)[32], uint64_t cc2, uint64_t nm2, uint64_t acc,
                                              uint32_t (&pk)[16]) {
#pragma unroll
  for (int i = I0; i < I0 + N; ++i) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), cc2, nm2);
    uint64_t pp;
    if ((AXIS_ATTN_FWD_POLY_MASK >> i) & 1) {
      pp = f2_exp2_poly(x);
    } else {
      float x0, x1;
      f2_unpack(x, x0, x1);
      pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
    }
    acc = f2_add(acc, pp);
    pk[i] = pack_bf16x2(pp);
  }
  return acc;
}

// Within each group of N lanes, transpose the N 16-byte chunks every lane
// holds (chunk k = c[4k .. 4k+3]): afterwards lane g*N + i holds, as its
// chunk k, chunk i of what lane g*N + k held.  A butterfly over the lane bits
// (shfl_xor with distance N/2, ..., 1), 2 N log2(N) shuffles per lane.
template <int N>
__device__ __forceinline__ void xpose_chunks(uint32_t (&c)[4 * N], int lane) {
#pragma unroll
  for (int b = N / 2; b >= 1; b >>= 1) {
    const bool hi = (lane & b) != 0;
#pragma unroll
    for (int k0 = 0; k0 < N; ++k0) {
      if (k0 & b) continue;
      const int k1 = k0 | b;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t send = hi ? c[4 * k0 + w] : c[4 * k1 + w];
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, b);
        if (hi)
          c[4 * k0 + w] = recv;
        else
          c[4 * k1 + w] = recv;
      }
    }
  }
}

// Warp roles: 0-7 softmax of Q tile 0 (0-3 columns 0-63, 4-7 columns 64-127),
// 8-15 softmax of Q tile 1, 16 TMA producer of Q and K, 17 S issuer (and TMEM
// owner), 18 TMA producer of V, 19 P V issuer.  Five warps per SM
// sub-partition leave 96 registers a thread: half a row of scores (64) plus
// its packed probabilities.
constexpr int FWD_SOFTMAX_WARPS = 16;
constexpr int FWD_SMW_PER_TILE = FWD_SOFTMAX_WARPS / 2;  // softmax warps of one query tile
constexpr int FWD_THREADS = (FWD_SOFTMAX_WARPS + 4) * 32;
constexpr int FWD_WARP_LOAD = FWD_SOFTMAX_WARPS;
constexpr int FWD_WARP_MMA = FWD_SOFTMAX_WARPS + 1;
constexpr int FWD_WARP_LOADV = FWD_SOFTMAX_WARPS + 2;
constexpr int FWD_WARP_PV = FWD_SOFTMAX_WARPS + 3;

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
  const uint32_t bar_q = bars, bar_qempty = bars + 8u;
  auto bar_kfull = [&](int s) { return bars + 8u * (2 + s); };
  auto bar_kempty = [&](int s) { return bars + 8u * (2 + KST + s); };
  auto bar_vfull = [&](int s) { return bars + 8u * (2 + 2 * KST + s); };
  auto bar_vempty = [&](int s) { return bars + 8u * (2 + 2 * KST + VST + s); };
  constexpr int B2 = 2 + 2 * KST + 2 * VST;
  auto bar_sfull = [&](int t) { return bars + 8u * (B2 + t); };
  auto bar_pfull = [&](int t) { return bars + 8u * (B2 + 2 + t); };
  auto bar_o = [&](int t) { return bars + 8u * (B2 + 4 + t); };
  const uint32_t bar_fin = bars + 8u * (B2 + 6);
  auto bar_sfree = [&](int t) { return bars + 8u * (B2 + 7 + t); };
  // partial-max / row-sum exchange between the two halves of a row block
  // (tile t, lane quarter wq): one phase per kv tile and one per epilogue
  auto bar_xch = [&](int t, int wq) { return bars + 8u * (B2 + 9 + 4 * t + wq); };
  // O_t has been read out by the epilogue: the next item may overwrite it
  auto bar_ofree = [&](int t) { return bars + 8u * (B2 + 17 + t); };
  float* xch = reinterpret_cast<float*>(gbase + C::XCH_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + C::BAR_OFF + 8 * C::NBAR);
  volatile WaitCtl* abort = reinterpret_cast<volatile WaitCtl*>(gbase + C::BAR_OFF + 8 * C::NBAR + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkv = (a.S + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_qempty, 1);
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
      mbar_init(bar_pfull(t), FWD_SMW_PER_TILE);
      mbar_init(bar_o(t), 1);
      mbar_init(bar_sfree(t), FWD_SMW_PER_TILE);
      mbar_init(bar_ofree(t), FWD_SMW_PER_TILE);
      for (int wq = 0; wq < 4; ++wq) mbar_init(bar_xch(t, wq), 2);
    }
    mbar_init(bar_fin, 2);  // one commit from each MMA issuer
    wait_ctl_init(abort);
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
    // warp 16: per item Q (once the previous item's S products are done with
    // it), then the K ring (with an L2 prefetch of K and V PF tiles ahead);
    // warp 18: the V ring.  Ring positions count kv tiles over all items.
    // Each lane-0 loop blocks (in hardware) on the stage it needs next.
    if (lane == 0) {
      const bool is_k = warp == FWD_WARP_LOAD;
      int g = 0, nq = 0;  // kv tiles / Q pairs issued
      bool ok = true;
      if (is_k) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      } else {
        tma_prefetch_desc(&tm_v);
      }
      for (int it = 0; ok; ++it) {
        const int w = fwd_item(it);
        if (w >= a.n_items) break;
        const FwdItem I = fwd_decode(a, w, CAUSAL);
        if (is_k) {
          if (it > 0 && !mbar_wait_bounded<true>(bar_qempty, (it - 1) & 1, abort, F_QEMPTY)) break;
          mbar_arrive_expect_tx(bar_q, (I.has1 ? 2u : 1u) * TILE);
          for (int sl = 0; sl < C::NSLAB; ++sl)
            tma_load_4d(sQ + sl * SLAB, &tm_q, bar_q, 64 * sl, I.h, 128 * I.qt0, I.b);
          if (I.has1)
            for (int sl = 0; sl < C::NSLAB; ++sl)
              tma_load_4d(sQ + TILE + sl * SLAB, &tm_q, bar_q, 64 * sl, I.h, 128 * I.qt0 + 128, I.b);
          ++nq;
          constexpr int PF = 4;
          auto prefetch = [&](int j) {
            for (int sl = 0; sl < C::NSLAB; ++sl) {
              tma_prefetch_4d(&tm_k, 64 * sl, I.kvh, 128 * j, I.b);
              tma_prefetch_4d(&tm_v, 64 * sl, I.kvh, 128 * j, I.b);
            }
          };
          for (int j = 0; j < PF && j < I.nmax; ++j) prefetch(j);
          for (int j = 0; j < I.nmax; ++j, ++g) {
            const int s = g % KST;
            if (g >= KST && !mbar_wait_bounded<true>(bar_kempty(s), ((g / KST) & 1) ^ 1, abort, F_EMPTY)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar_kfull(s), TILE);
            for (int sl = 0; sl < C::NSLAB; ++sl)
              tma_load_4d(sK + s * TILE + sl * SLAB, &tm_k, bar_kfull(s), 64 * sl, I.kvh, 128 * j, I.b);
            if (j + PF < I.nmax) prefetch(j + PF);
          }
        } else {
          for (int j = 0; j < I.nmax; ++j, ++g) {
            const int s = g % VST;
            if (g >= VST && !mbar_wait_bounded<true>(bar_vempty(s), ((g / VST) & 1) ^ 1, abort, F_EMPTY)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar_vfull(s), TILE);
            for (int sl = 0; sl < C::NSLAB; ++sl)
              tma_load_4d(sV + s * TILE + sl * SLAB, &tm_v, bar_vfull(s), 64 * sl, I.kvh, 128 * j, I.b);
          }
        }
      }
      // Drain: every copy this thread started has landed before the CTA exits
      // (each stage's most recent phase; nothing newer can have started).
      volatile WaitCtl never = {0, 0, 0};  // drain: bounded by the time limit only
      const int NS = is_k ? KST : VST;
      if (is_k && nq > 0) mbar_wait_bounded<true>(bar_q, (nq - 1) & 1, &never, F_Q);
      for (int x = g - NS > 0 ? g - NS : 0; x < g; ++x)
        mbar_wait_bounded<true>(is_k ? bar_kfull(x % KST) : bar_vfull(x % VST), (x / NS) & 1, &never,
                          is_k ? F_KFULL : F_VFULL);
    }
  } else if (warp == FWD_WARP_MMA) {
    // ===================================================== S issuer
    // S_t(j) = Q_t K_j^T in the order S0(0) S1(0) S0(1) S1(1) ... over all
    // items.  An S may overwrite its columns once the softmax has read the
    // previous S held there (sfree): S_t(j-1) at D = 64, the previous S of
    // either tile at D = 128 (one shared S).  After an item's last S, Q may
    // take the next item (qempty).  The whole warp runs the loop with warp-uniform
    // waits; lane 0 issues each instruction.  js[t]: S products of tile t so
    // far (over all items), g: kv tiles of earlier items.
    constexpr uint32_t ID_S = idesc_bf16(128, 128, 0, 0);   // Q (K-major) x K (K-major)
    uint32_t s_users = 0;  // products issued per K stage (2-bit counters)
    int js[2] = {0, 0};
    int g = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int w = fwd_item(it);
      if (w >= a.n_items) break;
      const FwdItem I = fwd_decode(a, w, CAUSAL);
      const int n[2] = {I.n0, I.n1};
      int s_left = I.n0 + I.n1;
      ok = wait_warp<true>(bar_q, it & 1, abort, F_Q);
      for (int j = 0; ok && j < I.nmax; ++j) {
        const int s = (g + j) % KST;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || j >= n[t]) continue;
          // S_t may overwrite its columns once their last S has been read
          const int prev = C::SHARED_S ? js[0] + js[1] - 1 : js[t] - 1;
          if (prev >= 0 && !(ok = wait_warp<true>(bar_sfree(C::SHARED_S ? 0 : t), prev & 1, abort, F_SFULL)))
            break;
          if (!(ok = wait_warp<true>(bar_kfull(s), ((g + j) / KST) & 1, abort, F_KFULL))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * SLAB + (kk & 3) * 32;
            mma_ss_w(tmem + C::t_s(t), sw128_desc(sQ + t * TILE + off, 16, 1024),
                     sw128_desc(sK + s * TILE + off, 16, 1024), ID_S, kk > 0);
          }
          mma_commit_w(bar_sfull(t));
          ++js[t];
          s_users += 1u << (2 * s);
          if (((s_users >> (2 * s)) & 3u) == (uint32_t)((j < n[0]) + (j < n[1]))) {
            s_users &= ~(3u << (2 * s));
            mma_commit_w(bar_kempty(s));
          }
          if (--s_left == 0) mma_commit_w(bar_qempty);  // Q may take the next item
        }
      }
      g += I.nmax;
    }
    // Drain: all MMAs issued by this warp complete before TMEM is freed.
    mma_commit_w(bar_fin);
    volatile WaitCtl never = {0, 0, 0};  // drain: bounded by the time limit only
    wait_warp<true>(bar_fin, 0, &never, F_OFIN);
  } else if (warp == FWD_WARP_PV) {
    // ===================================================== P V issuer
    // O_t += P_t(j) V_j in the order PV0(0) PV1(0) PV0(1) PV1(1) ... (the
    // order in which the softmax tiles finish their exponentials).  An item's
    // first P V overwrites O_t and waits until the epilogue of the previous
    // item has read O_t out (ofree).  jp[t]: P V products of tile t so far,
    // nit[t]: earlier items with a tile t, g: kv tiles of earlier items.
    constexpr uint32_t ID_PV = idesc_bf16(128, HD, 0, 1);   // P (TMEM) x V (MN-major)
    uint32_t pv_users = 0;  // products issued per V stage (2-bit counters)
    int jp[2] = {0, 0}, nit[2] = {0, 0};
    int g = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int w = fwd_item(it);
      if (w >= a.n_items) break;
      const FwdItem I = fwd_decode(a, w, CAUSAL);
      const int n[2] = {I.n0, I.n1};
      for (int j = 0; ok && j < I.nmax; ++j) {
        const int s = (g + j) % VST;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || j >= n[t]) continue;
          if (j == 0 && nit[t] > 0 && !(ok = wait_warp<true>(bar_ofree(t), (nit[t] - 1) & 1, abort, F_OFREE)))
            break;
          if (!(ok = wait_warp<true>(bar_pfull(t), jp[t] & 1, abort, F_PFULL))) break;
          if (!(ok = wait_warp<true>(bar_vfull(s), ((g + j) / VST) & 1, abort, F_VFULL))) break;
          tc_fence_after();
          const uint32_t tO = tmem + C::T_O + t * HD;
          const uint32_t tP = tmem + C::T_P + t * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_w(tO, tP + kk * 8, sw128_desc(sV + s * TILE + kk * 2048, SLAB, 1024), ID_PV,
                     (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit_w(bar_o(t));
          ++jp[t];
          pv_users += 1u << (2 * s);
          if (((pv_users >> (2 * s)) & 3u) == (uint32_t)((j < n[0]) + (j < n[1]))) {
            pv_users &= ~(3u << (2 * s));
            mma_commit_w(bar_vempty(s));
          }
        }
      }
      for (int t = 0; t < 2; ++t) nit[t] += n[t] > 0;
      g += I.nmax;
    }
    mma_commit_w(bar_fin);
    volatile WaitCtl never = {0, 0, 0};  // drain: bounded by the time limit only
    wait_warp<true>(bar_fin, 0, &never, F_OFIN);
  } else if (warp < FWD_SOFTMAX_WARPS) {
    // ===================================================== softmax (tile t, half hf)
    const int t = warp >> 3, hf = (warp >> 2) & 1, wq = warp & 3;
    const int r = wq * 32 + lane;                   // row in tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::t_s(t) + hf * 64;
    const uint32_t tO = tmem + lane_off + C::T_O + t * HD + hf * (HD / 2);
    const uint32_t tP = tmem + lane_off + C::T_P + t * 64 + hf * 32;
    const uint32_t bx = bar_xch(t, wq);
    // exchange slot of this thread's row: [parity][tile][half][row]
    auto xslot = [&](int par, int half) { return xch + ((par * 2 + t) * 2 + half) * 128 + r; };
    const float c = a.scale_log2;
    const uint64_t cc2 = f2_pack(c, c);
    // phases over all items: J kv tiles of this tile, X exchanges
    int J = 0, X = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int w = fwd_item(it);
      if (w >= a.n_items) break;
      const FwdItem I = fwd_decode(a, w, CAUSAL);
      const int n_t = t == 0 ? I.n0 : I.n1;
      const int qt = I.qt0 + t;
      const int row_g = qt * 128 + r;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < n_t; ++j, ++J, ++X) {
        if (!wait_warp<true>(bar_sfull(t), J & 1, abort, F_SFULL)) { ok = false; break; }
        tc_fence_after();
        const bool masked = CAUSAL ? (j == qt) : (j == nkv - 1 && (a.S & 127) != 0);
        int limit = 128;
        if (masked) {
          limit = a.S - 128 * j;
          if (CAUSAL && r + 1 < limit) limit = r + 1;
        }
        limit -= hf * 64;  // in this half's columns
        // this half of the 128-column row of S in registers (one TMEM pass)
        uint32_t v0[32], v1[32];
        tmem_ld32(tS, v0);
        tmem_ld32(tS + 32, v1);
        tmem_wait_ld();
        // S is in registers: its columns may take the next S
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sfree(C::SHARED_S ? 0 : t));
        if (masked) {
          mask_row(v0, 0, limit);
          mask_row(v1, 32, limit);
        }
        // row max: this half's, then the other half's (through shared memory)
        float mx = fmaxf(row_max32(v0), row_max32(v1));
        *xslot(X & 1, hf) = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(bx);
        if (!wait_warp<true>(bx, X & 1, abort, F_XCH)) { ok = false; break; }
        mx = fmaxf(mx, *xslot(X & 1, hf ^ 1));
        const float m_new = fmaxf(m_used, mx * c);
        const bool resc = m_new > m_used + 8.0f;
        float alpha = 1.f;
        if (resc) {
          alpha = ex2_approx(m_used - m_new);
          m_used = m_new;
        }
        // p = 2^(s*c - m) (masked entries are -inf and give 0), row sum, bf16
        // P pairs in registers
        const uint64_t nm2 = f2_pack(-m_used, -m_used);
        uint64_t acc = f2_pack(0.f, 0.f);
        uint32_t pk0[16], pk1[16];
        acc = exp_pairs<0, 16>(v0, cc2, nm2, acc, pk0);
        acc = exp_pairs<0, 16>(v1, cc2, nm2, acc, pk1);
        float rs_lo, rs_hi;
        f2_unpack(acc, rs_lo, rs_hi);
        l = l * alpha + (rs_lo + rs_hi);
        // the previous P V must have landed before P_t is overwritten and O_t rescaled
        if (J > 0) {
          if (!wait_warp<true>(bar_o(t), (J - 1) & 1, abort, F_OWAIT)) { ok = false; break; }
          tc_fence_after();
        }
        tmem_st16(tP, pk0);
        tmem_st16(tP + 16, pk1);
        // rescale this half's O columns when the max moved
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int cc = 0; cc < HD / 64; ++cc) {
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
        if (lane == 0 && !(AXIS_ATTN_TEST_DROP_ARRIVE == 1 && J == 0 && t == 0)) mbar_arrive(bar_pfull(t));
      }
      if (!ok || n_t == 0) continue;
      // epilogue: the halves' row sums are added, O / l -> bf16 (each half
      // its HD/2 columns), LSE = (m + log2 l) ln 2
      *xslot(X & 1, hf) = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(bx);
      if (!wait_warp<true>(bx, X & 1, abort, F_XCH)) { ok = false; break; }
      l += *xslot(X & 1, hf ^ 1);
      ++X;
      if (!wait_warp<true>(bar_o(t), (J - 1) & 1, abort, F_OFIN)) { ok = false; break; }
      tc_fence_after();
      const float inv_l = __fdividef(1.f, l);  // l >= 1: the row max contributes 2^(>= 0)
      // O / l as bf16: this thread's half row is NCK 16-byte chunks
      constexpr int NCK = HD / 16;
      uint32_t pk[4 * NCK];
#pragma unroll
      for (int cc = 0; cc < HD / 64; ++cc) {
        uint32_t v[32];
        tmem_ld32(tO + cc * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[16 * cc + i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv_l, __uint_as_float(v[2 * i + 1]) * inv_l);
      }
      // O_t is out of TMEM: the next item's first P V may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_ofree(t));
      // Coalesced stores: after the chunk transpose, store k of the warp
      // writes 32 / NCK whole half rows (NCK consecutive lanes per row)
      // instead of 32 scattered 16-byte pieces.
      xpose_chunks<NCK>(pk, lane);
      const int ck = lane % NCK, rbase = qt * 128 + wq * 32 + (lane / NCK) * NCK;
#pragma unroll
      for (int k = 0; k < NCK; ++k) {
        const int row = rbase + k;
        if (row < a.S) {
          uint4* dst =
              reinterpret_cast<uint4*>(a.o + (((size_t)I.b * a.S + row) * a.Hq + I.h) * HD + hf * (HD / 2)) + ck;
          *dst = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
      }
      if (hf == 0 && row_g < a.S) a.lse[(size_t)I.bh * a.S + row_g] = (m_used + __log2f(l)) * 0.69314718055994531f;
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
