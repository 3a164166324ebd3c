// attn_decode.cuh -- decode step: one (or a few) new query rows per sequence
// against its paged KV cache, and the combine of split partial results.
//
// What it computes is the step the axiomlm inference engine repeats per
// generated token (axiomlm page, Key Features: "State-cached Key-Value (KV)
// decode engine"; Quick Start section 4: the paged KV-cache engine), with GQA
// heads (Key Features, Grouped-Query Attention): for sequence b and query
// head h (kv head h / G) the new token attends to every cached key of its
// sequence, itself included:
//   o[b,h,:] = sum_j softmax_j(scale q[b,h,:] . K_j) V_j,   lse = ln sum_j exp(...)
//
// Design on sm_100a.  The step reads every cached key and value once and does
// about 4 G flops per byte, far below the tensor cores' ridge, so it is
// HBM-bound: the kernel is built to keep the memory system busy.
//   * persistent: as many CTAs as fit on the SMs walk the work items (b, kv
//     head, split of the sequence); a producer warp prepares 32 pieces at a
//     time (one lane per piece reads its block-table entries and forms its
//     copies' coordinates) and streams 32-key pieces of the cache pages
//     through TMA (a 3-D tensor map over the cache, 128B swizzle) into a ring
//     of shared-memory stages, K and V of a piece on one mbarrier, running
//     ahead across item boundaries;
//   * the compute warps (4 at D = 64, 1 at D = 128) take the pieces in turn
//     and keep their own running max, sum and O for the G <= 8 query heads
//     of the item.  The products
//     run on the warp-level tensor-core MMA (m16n8k16, bf16 in, fp32 out),
//     the heads as rows of a 16-row tile: S = Q K^T with K's fragments
//     loaded straight from the swizzled rows (ldmatrix), the online softmax in
//     the accumulator layout (a row's 32 keys in the 4 lanes of a quad), P
//     kept in registers as the A operand of O += P V, V through the
//     transposing load.  Per 8 KB piece that is about a tenth of the
//     instructions of the same arithmetic on the CUDA cores;
//   * at the end of an item the warps' states are merged in shared
//     memory; a split writes its unnormalised (m, l, O) to the workspace,
//     which a second kernel merges (split-K over long sequences keeps every
//     SM busy at small batch); with one split the CTA writes O and LSE itself.
// Several new tokens per sequence (q_len > 1: a prompt chunk appended to the
// cache, or proposed tokens checked together) are the last q_len positions;
// a work item then takes a tile of 8 or 16 (token, head) rows of a kv head,
// every row masked at its own position, and the tiles of a kv head, adjacent
// in the item order, stream the same pieces (the later reads hit L2).
// Page indices and sequence lengths are device data: a page index outside
// [0, num_pages) or a length outside [q_len, max_pages * page_size] is never used
// for an access; it sets bit 1 of the device status word (reported by
// axis_attn_get_status as AXIS_ATTN_ERR_INDEX) and the piece is skipped.
#pragma once

#include "sm100_ptx.cuh"

namespace axis_attn {

struct DecArgs {
  const __nv_bfloat16* q;  // [B, q_len, Hq, D]
  const int* block_table;  // [B, max_pages]
  const int* seq_lens;     // [B]
  __nv_bfloat16* o;        // [B, q_len, Hq, D]
  float* lse;              // [B, Hq, q_len]
  float* part;             // [B * q_len * Hq][n_splits][D + 2]: m, l, O (n_splits > 1)
  int B, Hq, Hkv, G, page_size, max_pages, num_pages;
  int q_len;               // new tokens per sequence: the last q_len positions
  int n_rt;                // row tiles per (b, kv head): 1 with at most 8 (token, head) rows, else
                           // ceil(G * q_len / 16) tiles of 16
  int hnd;                 // cache layout: 0 [pages, page_size, Hkv, D]; 1 [pages, Hkv, page_size, D]
  int keys_per_split;      // a multiple of 32
  int n_splits;
  float scale_log2;        // scale * log2(e)
};

// Compute warps per CTA and ring stages (warp 0 is the producer).  Each CTA's
// producer and compute warps form one dependent chain per piece, and an SM's
// bytes in flight are its CTAs x stages x piece bytes.  Two configurations per
// head dim, chosen per call by the host:
//   * wide (many small CTAs per SM) when the items fill them: measured at page
//     size 16 to 64 (HBM fraction), D = 64 4 warps x 4 stages (4 CTAs / SM, by
//     registers) 0.79-0.91 against 0.70-0.72 with 8 stages (3 CTAs / SM);
//     D = 128 1 warp x 2 stages (5 CTAs / SM) 0.94-0.98 against 0.90-0.96 with
//     4 x 4;
//   * deep (fewer CTAs, more stages each) when a small batch leaves most of
//     the wide configuration's CTAs without an item.
#ifndef AXIS_ATTN_DEC_CW64
#define AXIS_ATTN_DEC_CW64 4
#endif
#ifndef AXIS_ATTN_DEC_NST64
#define AXIS_ATTN_DEC_NST64 4
#endif
#ifndef AXIS_ATTN_DEC_CW128
#define AXIS_ATTN_DEC_CW128 1
#endif
#ifndef AXIS_ATTN_DEC_NST128
#define AXIS_ATTN_DEC_NST128 2
#endif
#ifndef AXIS_ATTN_DEC_DEEP_CW64
#define AXIS_ATTN_DEC_DEEP_CW64 4
#endif
#ifndef AXIS_ATTN_DEC_DEEP_NST64
#define AXIS_ATTN_DEC_DEEP_NST64 8
#endif
#ifndef AXIS_ATTN_DEC_DEEP_CW128
#define AXIS_ATTN_DEC_DEEP_CW128 4
#endif
#ifndef AXIS_ATTN_DEC_DEEP_NST128
#define AXIS_ATTN_DEC_DEEP_NST128 4
#endif

// MODE: 0 one new token per sequence (q_len = 1 at compile time); 1 several,
// at most 8 (token, head) rows per kv head (8-row tiles); 2 several, more rows
// (16-row tiles: both halves of the MMA's 16 rows carry rows).
template <int HD, bool DEEP, int MODE = 0>
struct DecCfg {
  static constexpr int RT = MODE == 2 ? 16 : 8;  // (token, head) rows per work item
  static constexpr int NSLAB = HD / 64;
  static constexpr uint32_t SLAB = 32 * 128;            // 32 rows x 128 bytes
  static constexpr uint32_t PIECE = NSLAB * SLAB;       // 32 keys x HD bf16
  static constexpr int CW = DEEP ? (HD == 64 ? AXIS_ATTN_DEC_DEEP_CW64 : AXIS_ATTN_DEC_DEEP_CW128)
                                 : (HD == 64 ? AXIS_ATTN_DEC_CW64 : AXIS_ATTN_DEC_CW128);  // compute warps
  static constexpr int THREADS = 32 * (1 + CW);
  static constexpr int NST = DEEP ? (HD == 64 ? AXIS_ATTN_DEC_DEEP_NST64 : AXIS_ATTN_DEC_DEEP_NST128)
                                  : (HD == 64 ? AXIS_ATTN_DEC_NST64 : AXIS_ATTN_DEC_NST128);  // ring stages
  // A compute warp waits on the phase of a stage only after the stage's
  // previous phase has completed (a parity wait cannot tell phase k from
  // phase k - 2): the previous piece in a stage must be the same warp's,
  // which holds when the ring depth is a multiple of the warp count.
  static_assert(NST % CW == 0, "ring depth must be a multiple of the compute warps");
  // Resident CTAs per SM the registers must allow (0: no bound).  The wide
  // D = 64 configuration (160 threads) fits 4 per SM only at <= 102 registers
  // a thread; left alone ptxas takes 125-128 and 3 fit (page size 16: 58.6 us
  // against 52.8 us with the bound, at a few dozen bytes of spills; 4 new
  // tokens per sequence in 16-row tiles: 63.2 against 56.3 us).
  static constexpr int MIN_CTAS = (HD == 64 && !DEEP) ? 4 : 0;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = NST * PIECE;
  static constexpr uint32_t OFF_C = 2 * NST * PIECE;              // fp32 [CW][RT][HD + 2]
  static constexpr uint32_t OFF_FLAG = OFF_C + CW * RT * (HD + 2) * 4;  // int [NST]: piece usable
  static constexpr uint32_t OFF_TBL = OFF_FLAG + NST * 4;                  // int [32][4]: pages of 32 pieces
  static constexpr uint32_t OFF_BAR = (OFF_TBL + 32 * 4 * 4 + 7) & ~7u;
  static constexpr uint32_t SMEM = OFF_BAR + 8 * 2 * NST + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};

enum DecSite { D_EMPTY = 41, D_FULL };

// One work item: (b, kv head, split of the sequence, row tile), its key
// range and pieces.  The row tiles of a (b, kv head, split) are adjacent in
// the item order, so the CTAs that read the same pieces run at the same time
// (the second reader finds them in L2).  len: the sequence's length (its
// q_len new tokens included).
struct DecItem {
  int b, kv, split, rt, k0, k1, n_pieces, len;
};
// The item's indices (no memory access).  q_len, n_rt: the launch's
// (compile-time 1, 1 in the one-token instantiation).
__device__ __forceinline__ DecItem dec_index(const DecArgs& a, int w, int n_rt) {
  DecItem it;
  it.rt = w % n_rt;
  w /= n_rt;
  it.split = w % a.n_splits;
  const int bkv = w / a.n_splits;
  it.b = bkv / a.Hkv;
  it.kv = bkv % a.Hkv;
  it.k0 = it.split * a.keys_per_split;
  return it;
}
// ... and its length (one load), key range and pieces.
__device__ __forceinline__ void dec_length(const DecArgs& a, DecItem& it, bool report, int q_len) {
  int len = a.seq_lens[it.b];
  const int cap = a.max_pages * a.page_size;
  if (len < q_len || len > cap) {  // clamped (cap >= q_len); reported once (by the producer)
    if (report) atomicOr(&g_status, 2u);
    len = len < q_len ? q_len : cap;
  }
  it.len = len;
  it.k1 = min(len, it.k0 + a.keys_per_split);
  it.n_pieces = it.k1 > it.k0 ? (it.k1 - it.k0 + 31) / 32 : 0;
}
__device__ __forceinline__ DecItem dec_item(const DecArgs& a, int w, bool report, int q_len, int n_rt) {
  DecItem it = dec_index(a, w, n_rt);
  dec_length(a, it, report, q_len);
  return it;
}

// Persistent: each CTA walks the items w = blockIdx.x, blockIdx.x + gridDim.x,
// ...; the ring positions count pieces over all of its items, so the producer
// streams the next item's pieces while the compute warps finish this one.
// Compute warp (g mod CW) takes the CTA's g-th piece.
template <int HD, bool DEEP, int MODE>
__global__ void __launch_bounds__(DecCfg<HD, DEEP, MODE>::THREADS, DecCfg<HD, DEEP, MODE>::MIN_CTAS)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const DecArgs a) {
  using C = DecCfg<HD, DEEP, MODE>;
  constexpr int NST = C::NST, CW = C::CW;
  constexpr bool MULTI = MODE > 0;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V;
  float* c_s = reinterpret_cast<float*>(gbase + C::OFF_C);
  volatile int* flag = reinterpret_cast<volatile int*>(gbase + C::OFF_FLAG);
  const uint32_t bars = base + C::OFF_BAR;
  auto bar_full = [&](int s) { return bars + 8u * s; };
  auto bar_empty = [&](int s) { return bars + 8u * (NST + s); };
  volatile WaitCtl* ctl = reinterpret_cast<volatile WaitCtl*>(gbase + C::OFF_BAR + 16 * NST + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The split merge (launched as this grid's programmatic dependent) may be
  // scheduled now: its CTAs wait for this grid's completion and memory
  // (griddepcontrol.wait) before reading a partial result, so only its launch
  // latency overlaps this kernel.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // several new tokens per sequence, or one (MODE 0: q_len = 1 and one row
  // tile at compile time, the code of the one-token step)
  const int q_len = MULTI ? a.q_len : 1, n_rt = MULTI ? a.n_rt : 1;
  const int n_items = a.B * a.Hkv * a.n_splits * n_rt;
  const int G = a.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    wait_ctl_init(ctl);
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ============================================================ producer
    // Per block of 32 pieces, lane j prepares piece j at once with the other
    // lanes: it reads the block-table entries of its piece's pages (32
    // independent loads instead of one dependent global read in front of
    // every copy), checks them and forms its boxes' coordinates.  The lanes
    // then take their turns at the ring: lane j waits for its stage, sets its
    // flag and issues its copies.  The single issuing thread's work per piece
    // is thereby the wait and the copies alone (a thread doing all of it
    // issued one 8 KB piece per ~0.5 us: below HBM speed with 3 CTAs per SM).
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    const int rows = a.page_size < 32 ? a.page_size : 32;  // rows per TMA box
    const int nbox = 32 / rows;                              // boxes per 32-key piece
    const int ps_shift = 31 - __clz(a.page_size);            // page_size is a power of two
    const int ps_mask = a.page_size - 1;
    int g = 0;  // pieces issued (over all items); the same in every lane
    bool ok = true;
    const int cap = a.max_pages * a.page_size;
    for (int w = (int)blockIdx.x; ok && w < n_items; w += (int)gridDim.x) {
      DecItem I = dec_index(a, w, n_rt);
      const int* row_tbl = a.block_table + (size_t)I.b * a.max_pages;
      // the block-table entries of the item's first 32 pieces, loaded together
      // with its length (they do not depend on it; which of them are used does)
      int page0[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int key = I.k0 + 32 * lane + x * rows;
        page0[x] = x < nbox && key < cap ? row_tbl[key >> ps_shift] : 0;
      }
      dec_length(a, I, lane == 0, q_len);
      for (int t0 = 0; ok && t0 < I.n_pieces; t0 += 32) {
        const int kt = I.k0 + 32 * (t0 + lane);  // this lane's piece
        // boxes x < nload of this lane's piece: cache coordinates (c1[x], c2[x]) of box row 0
        int c1[4], c2[4], nload = 0, usable = 1;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int key = kt + x * rows;
          c1[x] = c2[x] = 0;
          if (t0 + lane < I.n_pieces && x < nbox && key < I.k1) {
            const int page = t0 == 0 ? page0[x] : row_tbl[key >> ps_shift];
            if (page < 0 || page >= a.num_pages) usable = 0;
            c1[x] = a.hnd ? (key & ps_mask) : I.kv;
            c2[x] = a.hnd ? page * a.Hkv + I.kv : page * a.page_size + (key & ps_mask);
            ++nload;
          }
        }
        const int n = min(32, I.n_pieces - t0);
        for (int j = 0; j < n; ++j, ++g) {
          if (lane == j) {
            const int s = g % NST;
            if (g >= NST && !mbar_wait_bounded<true>(bar_empty(s), ((g / NST) & 1) ^ 1, ctl, D_EMPTY)) {
              ok = false;
            } else {
              flag[s] = usable;
              if (!usable) {
                atomicOr(&g_status, 2u);
                mbar_arrive(bar_full(s));
              } else {
                mbar_arrive_expect_tx(bar_full(s), (uint32_t)(nload * rows * HD * 2 * 2));
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                  if (x >= nload) break;
#pragma unroll
                  for (int sl = 0; sl < C::NSLAB; ++sl) {
                    const uint32_t off = s * C::PIECE + sl * C::SLAB + x * rows * 128;
                    tma_load_3d(sK + off, &tm_k, bar_full(s), 64 * sl, c1[x], c2[x]);
                    tma_load_3d(sV + off, &tm_v, bar_full(s), 64 * sl, c1[x], c2[x]);
                  }
                }
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, j);
          if (!ok) break;
        }
      }
    }
    // drain: every copy started has landed before the CTA exits
    if (lane == 0) {
      volatile WaitCtl never = {0, 0, 0};
      for (int x = g - NST > 0 ? g - NST : 0; x < g; ++x)
        mbar_wait_bounded<true>(bar_full(x % NST), (x / NST) & 1, &never, D_FULL);
    }
  } else {
    // ============================================================ compute warps
    // Per 32-key piece: S (16 x 32) = Q K^T and O (16 x D) += P V on the
    // warp-level MMA, the item's RT (token, head) rows as rows of a 16-row
    // tile: row r = RT rt + i of the unit is new token r / G and head r % G
    // (rows past G q_len unused).  RT = 8 (MODE 0, 1): rows 0..7 of the MMA
    // tile, rows 8..15 zero; RT = 16 (MODE 2): all 16 rows.  Lane l
    // holds, in the accumulator layout, rows g0 = l / 4 (half 0) and g0 + 8
    // (half 1) and the columns 2 (l % 4) + {0, 1} of every 8-column tile.
    constexpr int NR = MODE == 2 ? 2 : 1;  // row halves this lane works on
    constexpr int RT = C::RT;          // rows per tile: 8 NR
    const int cw = warp - 1;
    const float c = a.scale_log2;
    constexpr int KS = HD / 16;  // k-steps of the score product (features)
    constexpr int ND = HD / 8;   // 8-feature column tiles of O
    constexpr int FPL = HD / 32;  // features per lane in the merge
    const int g0 = lane >> 2, q2 = 2 * (lane & 3);
    int gbase_item = 0;  // pieces of this CTA's earlier items
    bool ok = true;
    // Every compute warp walks every item, also after a wait has given up
    // (its later waits then return at once: the CTA's abort flag is set), so
    // that all of them reach each of the named barriers below.
    for (int w = (int)blockIdx.x; w < n_items; w += (int)gridDim.x) {
      const DecItem I = dec_item(a, w, false, q_len, n_rt);
      bool row_ok[NR];
      int row_end[NR];
      // Q as A fragments: (row, columns 16 ks + q2 + {0,1}) and (+8) of each half
      uint32_t qf[NR][KS][2];
#pragma unroll
      for (int hb = 0; hb < NR; ++hb) {
        const int row = RT * I.rt + g0 + 8 * hb;
        row_ok[hb] = row < G * q_len;
        const int tok = row / G, gh = row % G;  // new token, head in the group
        // this row's keys end after its own position len - q_len + tok (the
        // later new tokens are masked): keys of piece t below row_end - 32 t - k0
        row_end[hb] = I.len - q_len + tok + 1;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          qf[hb][ks][0] = qf[hb][ks][1] = 0u;
          if (row_ok[hb]) {
            const __nv_bfloat16* qrow =
                a.q + (((size_t)I.b * q_len + tok) * a.Hq + I.kv * G + gh) * HD + 16 * ks + q2;
            qf[hb][ks][0] = *reinterpret_cast<const uint32_t*>(qrow);
            qf[hb][ks][1] = *reinterpret_cast<const uint32_t*>(qrow + 8);
          }
        }
      }
      float o_acc[ND][4];
#pragma unroll
      for (int nd = 0; nd < ND; ++nd) o_acc[nd][0] = o_acc[nd][1] = o_acc[nd][2] = o_acc[nd][3] = 0.f;
      // per half: running max (log2 units), this lane's share of the row sum
      float m_run[NR], l_part[NR];
#pragma unroll
      for (int hb = 0; hb < NR; ++hb) m_run[hb] = -INFINITY, l_part[hb] = 0.f;
      // this warp's pieces of the item: the CTA's piece gbase_item + t goes to warp (gbase_item + t) % CW
      for (int t = (cw - gbase_item % CW + CW) % CW; ok && t < I.n_pieces; t += CW) {
        const int gp = gbase_item + t;
        const int s = gp % NST;
        if (!wait_warp<true>(bar_full(s), (gp / NST) & 1, ctl, D_FULL)) { ok = false; break; }
        const int n_valid = min(32, I.k1 - (I.k0 + 32 * t));
        if (flag[s]) {
          const uint32_t kb = sK + s * C::PIECE, vb = sV + s * C::PIECE;
          // rows past the sequence's end hold whatever the page pool holds there:
          // zero their V (a 0 weight times a NaN would still be NaN in the MMA)
          if (n_valid < 32) {
            for (int x = lane; x < (32 - n_valid) * (HD / 8); x += 32) {
              const int key = n_valid + x / (HD / 8), ch = x % (HD / 8);
              const uint32_t addr = vb + (ch >> 3) * C::SLAB + key * 128 + (((ch & 7) ^ (key & 7)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(addr), "r"(0u) : "memory");
            }
            __syncwarp();
          }
          // ---- S = Q K^T: 4 tiles of 8 keys; B fragments straight from the swizzled K rows
          float sc[4][4];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
            sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < KS / 2; ++k2) {
              // matrix lane / 8: features 32 k2 + 8 (lane / 8) .. + 7 of key 8 nt + lane % 8
              const int key = 8 * nt + (lane & 7), f0 = 32 * k2 + 8 * (lane >> 3);
              uint32_t bk[4];
              ldsm_x4(kb + (f0 >> 6) * C::SLAB + key * 128 + ((((f0 & 63) >> 3) ^ (key & 7)) << 4), bk);
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_16816(sc[nt], qf[0][2 * k2 + kk][0], NR > 1 ? qf[NR - 1][2 * k2 + kk][0] : 0u,
                          qf[0][2 * k2 + kk][1], NR > 1 ? qf[NR - 1][2 * k2 + kk][1] : 0u, bk[2 * kk],
                          bk[2 * kk + 1]);
            }
          }
          // ---- online softmax of each row (the 4 lanes of a quad hold its 32 keys);
          // a row sees this piece's keys below lim (its own position included).
          // p = 2^(s c - m), bf16 P as the A fragments of P V (k-step k2: key
          // tiles 2 k2 and 2 k2 + 1).  A row that has seen no key of its own yet
          // (m = -inf: this piece and the warp's earlier ones all lie past its
          // position) gets p = 0, not 2^(-inf + inf).
          uint32_t pf[NR][4];
#pragma unroll
          for (int hb = 0; hb < NR; ++hb) {
            const int lim = min(n_valid, row_end[hb] - (I.k0 + 32 * t));
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                if (8 * nt + q2 + e >= lim) sc[nt][2 * hb + e] = -INFINITY;
                mx = fmaxf(mx, sc[nt][2 * hb + e]);
              }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m_run[hb], mx * c);
            if (m_new > m_run[hb] + 8.0f) {  // the running max moves only by more than 8 (a factor 256)
              const float alpha = ex2_approx(m_run[hb] - m_new);  // 0 on the first piece
              m_run[hb] = m_new;
              l_part[hb] *= alpha;
#pragma unroll
              for (int nd = 0; nd < ND; ++nd) {
                o_acc[nd][2 * hb] *= alpha;
                o_acc[nd][2 * hb + 1] *= alpha;
              }
            }
            const float nm = m_run[hb] == -INFINITY ? 0.f : -m_run[hb];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
              const float p0 = ex2_approx(fmaf(sc[nt][2 * hb], c, nm));
              const float p1 = ex2_approx(fmaf(sc[nt][2 * hb + 1], c, nm));
              l_part[hb] += p0 + p1;
              pf[hb][nt] = pack_bf16x2(p0, p1);
            }
          }
          // ---- O += P V: B fragments of V (rows = keys) through the transposing load
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2)
#pragma unroll
            for (int n2 = 0; n2 < ND / 2; ++n2) {
              // matrix lane / 8: keys 16 k2 + 8 ((lane / 8) & 1) .., features 16 n2 + 8 (lane / 16)
              const int key = 16 * k2 + 8 * ((lane >> 3) & 1) + (lane & 7), f0 = 16 * n2 + 8 * (lane >> 4);
              uint32_t bv[4];
              ldsm_x4_t(vb + (f0 >> 6) * C::SLAB + key * 128 + ((((f0 & 63) >> 3) ^ (key & 7)) << 4), bv);
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_16816(o_acc[2 * n2 + kk], pf[0][2 * k2], NR > 1 ? pf[NR - 1][2 * k2] : 0u, pf[0][2 * k2 + 1],
                          NR > 1 ? pf[NR - 1][2 * k2 + 1] : 0u, bv[2 * kk], bv[2 * kk + 1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(s));
      }
      gbase_item += I.n_pieces;
      // ---- this warp's (m, l, O) of each row, then the merge of the CW warps
#pragma unroll
      for (int hb = 0; hb < NR; ++hb) {
        float l = l_part[hb];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (row_ok[hb]) {
          float* cs = c_s + (cw * RT + g0 + 8 * hb) * (HD + 2);
#pragma unroll
          for (int nd = 0; nd < ND; ++nd) {
            cs[2 + 8 * nd + q2] = o_acc[nd][2 * hb];
            cs[3 + 8 * nd + q2] = o_acc[nd][2 * hb + 1];
          }
          if ((lane & 3) == 0) {
            cs[0] = m_run[hb];
            cs[1] = l;
          }
        }
      }
      named_bar_sync(1, 32 * CW);
      for (int g = cw; g < RT && RT * I.rt + g < G * q_len; g += CW) {
        float mm = -INFINITY;
#pragma unroll
        for (int x = 0; x < CW; ++x) mm = fmaxf(mm, c_s[(x * RT + g) * (HD + 2)]);
        float lt = 0.f, ov[FPL];
#pragma unroll
        for (int f = 0; f < FPL; ++f) ov[f] = 0.f;
#pragma unroll
        for (int x = 0; x < CW; ++x) {
          const float* cs = c_s + (x * RT + g) * (HD + 2);
          const float e = cs[1] > 0.f ? ex2_approx(cs[0] - mm) : 0.f;  // warps without keys weigh 0
          lt += cs[1] * e;
#pragma unroll
          for (int f = 0; f < FPL; ++f) ov[f] += cs[2 + lane * FPL + f] * e;
        }
        // output row (b, new token, head) of o [B, q_len, Hq, D]; lse is [B, Hq, q_len]
        const int r = RT * I.rt + g, h = I.kv * G + r % G, tk = r / G;
        const size_t orow = ((size_t)I.b * q_len + tk) * a.Hq + h;
        if (a.n_splits == 1) {
          const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll
          for (int f = 0; f < FPL; ++f) a.o[orow * HD + lane * FPL + f] = __float2bfloat16_rn(ov[f] * inv);
          if (lane == 0)
            a.lse[((size_t)I.b * a.Hq + h) * q_len + tk] = (mm + __log2f(lt)) * 0.69314718055994531f;
        } else {
          float* dst = a.part + (orow * a.n_splits + I.split) * (HD + 2);
#pragma unroll
          for (int f = 0; f < FPL; ++f) dst[2 + lane * FPL + f] = ov[f];
          if (lane == 0) {
            dst[0] = mm;
            dst[1] = lt;
          }
        }
      }
      // the merge has read every warp's share before the next item's are written
      named_bar_sync(1, 32 * CW);
    }
  }
}

// Merge the splits of every (b, new token, h): one 256-thread CTA per row.  The maximum
// over the splits comes from all threads at once (one split each); then warp w
// takes splits w, w + 8, ... (lanes over features, DEC_COMBINE_U splits'
// loads in flight at a time) and the 8 warps' sums meet in shared memory.
// The few round trips to L2 this leaves per row matter: with one warp walking
// tens of splits the merge took as long as the decode kernel itself.
constexpr int DEC_COMBINE_U = 4;
template <int HD>
__global__ void __launch_bounds__(256) attn_decode_combine_kernel(const float* __restrict__ part,
                                                                  __nv_bfloat16* __restrict__ o,
                                                                  float* __restrict__ lse, int rows, int n_splits,
                                                                  int Hq, int q_len) {
  constexpr int FPL = HD / 32, NW = 8;
  __shared__ float s_red[NW];
  __shared__ float s_o[NW][HD];
  const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31;
  // launched as the decode kernel's programmatic dependent: wait until that
  // grid has completed and its partial results are visible (a no-op when
  // launched in the ordinary way)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int bh = (int)blockIdx.x; bh < rows; bh += (int)gridDim.x) {
    const float* p = part + (size_t)bh * n_splits * (HD + 2);
    // the maximum over the splits that saw keys (l > 0; a split past the end of the sequence has none)
    float mm = -INFINITY;
    for (int s = (int)threadIdx.x; s < n_splits; s += 32 * NW) {
      const float2 ml = *reinterpret_cast<const float2*>(p + (size_t)s * (HD + 2));
      if (ml.y > 0.f) mm = fmaxf(mm, ml.x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, off));
    if (lane == 0) s_red[warp] = mm;
    __syncthreads();
    mm = s_red[0];
#pragma unroll
    for (int w = 1; w < NW; ++w) mm = fmaxf(mm, s_red[w]);
    // this warp's splits, weighted by 2^(m_s - mm)
    float l = 0.f, ov[FPL];
#pragma unroll
    for (int f = 0; f < FPL; ++f) ov[f] = 0.f;
    for (int s0 = warp; s0 < n_splits; s0 += NW * DEC_COMBINE_U) {
      float2 ml[DEC_COMBINE_U];
      float v[DEC_COMBINE_U][FPL];
#pragma unroll
      for (int u = 0; u < DEC_COMBINE_U; ++u) {
        const int sp = s0 + NW * u;
        ml[u] = make_float2(0.f, 0.f);
        if (sp < n_splits) {
          const float* ps = p + (size_t)sp * (HD + 2);
          ml[u] = *reinterpret_cast<const float2*>(ps);
#pragma unroll
          for (int f = 0; f < FPL; ++f) v[u][f] = ps[2 + lane * FPL + f];
        }
      }
#pragma unroll
      for (int u = 0; u < DEC_COMBINE_U; ++u) {
        if (!(ml[u].y > 0.f)) continue;
        const float e = ex2_approx(ml[u].x - mm);
        l += ml[u].y * e;
#pragma unroll
        for (int f = 0; f < FPL; ++f) ov[f] += v[u][f] * e;
      }
    }
    __syncthreads();  // every warp has read s_red
#pragma unroll
    for (int f = 0; f < FPL; ++f) s_o[warp][lane * FPL + f] = ov[f];
    if (lane == 0) s_red[warp] = l;
    __syncthreads();
    if (warp == 0) {
      float lt = 0.f, ot[FPL];
#pragma unroll
      for (int f = 0; f < FPL; ++f) ot[f] = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        lt += s_red[w];
#pragma unroll
        for (int f = 0; f < FPL; ++f) ot[f] += s_o[w][lane * FPL + f];
      }
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll
      for (int f = 0; f < FPL; ++f) o[(size_t)bh * HD + lane * FPL + f] = __float2bfloat16_rn(ot[f] * inv);
      // row bh = (b q_len + token) Hq + h of o; lse is [B, Hq, q_len]
      if (lane == 0)
        lse[((size_t)(bh / (q_len * Hq)) * Hq + bh % Hq) * q_len + (bh / Hq) % q_len] =
            (mm + __log2f(lt)) * 0.69314718055994531f;
    }
    __syncthreads();  // warp 0 has read s_red and s_o before the next row writes them
  }
}

}  // namespace axis_attn
