// attn_decode.cuh -- decode step: one new query row per sequence against its
// paged KV cache, and the combine of split partial results.
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
// HBM-bound: the kernel is built to keep the memory system busy, not the MMA
// units.
//   * one CTA per (b, kv head, split of the sequence); a producer warp reads
//     the block table 32 pieces ahead into shared memory and one of its
//     threads streams 32-key pieces of the cache pages through TMA (a 3-D
//     tensor map over the cache, 128B swizzle) into a ring of shared-memory
//     stages, K and V of a piece on one mbarrier;
//   * four compute warps take the pieces in turn (piece t -> warp t % 4) and
//     keep their own running max, sum and O for the G query heads: scores with
//     lane = key (q broadcast from shared memory, packed fp32 FMA), per-head
//     max by warp shuffles, p = 2^(s - m) on the MUFU, then O += p V with
//     lane = feature slice;
//   * at the end the four warps' states are merged in shared memory; a split
//     writes its unnormalised (m, l, O) to the workspace, which a second kernel
//     merges (split-K over long sequences keeps every SM busy at small batch);
//     with one split the CTA writes O and LSE itself.
// Page indices and sequence lengths are device data: a page index outside
// [0, num_pages) or a length outside [1, max_pages * page_size] is never used
// for an access; it sets bit 1 of the device status word (reported by
// axis_attn_get_status as AXIS_ATTN_ERR_INDEX) and the piece is skipped.
#pragma once

#include "sm100_ptx.cuh"

namespace axis_attn {

struct DecArgs {
  const __nv_bfloat16* q;  // [B, Hq, D]
  const int* block_table;  // [B, max_pages]
  const int* seq_lens;     // [B]
  __nv_bfloat16* o;        // [B, Hq, D]
  float* lse;              // [B, Hq]
  float* part;             // [B * Hq][n_splits][D + 2]: m, l, O (n_splits > 1)
  int B, Hq, Hkv, G, page_size, max_pages, num_pages;
  int keys_per_split;      // a multiple of 32
  int n_splits;
  float scale_log2;        // scale * log2(e)
};

constexpr int DEC_THREADS = 160;  // warp 0: producer; warps 1-4: compute
constexpr int DEC_CW = 4;         // compute warps

template <int HD>
struct DecCfg {
  static constexpr int NSLAB = HD / 64;
  static constexpr uint32_t SLAB = 32 * 128;            // 32 rows x 128 bytes
  static constexpr uint32_t PIECE = NSLAB * SLAB;       // 32 keys x HD bf16
  static constexpr int NST = HD == 64 ? 8 : 4;          // ring stages (2 or 1 per compute warp)
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = NST * PIECE;
  static constexpr uint32_t OFF_Q = 2 * NST * PIECE;              // fp32 [8][HD], pre-scaled
  static constexpr uint32_t OFF_P = OFF_Q + 8 * HD * 4;           // fp32 [DEC_CW][32][8]
  static constexpr uint32_t OFF_C = OFF_P + DEC_CW * 32 * 8 * 4;  // fp32 [DEC_CW][8][HD + 2]
  static constexpr uint32_t OFF_FLAG = OFF_C + DEC_CW * 8 * (HD + 2) * 4;  // int [NST]: piece usable
  static constexpr uint32_t OFF_TBL = OFF_FLAG + NST * 4;                  // int [32][4]: pages of 32 pieces
  static constexpr uint32_t OFF_BAR = (OFF_TBL + 32 * 4 * 4 + 7) & ~7u;
  static constexpr uint32_t SMEM = OFF_BAR + 8 * 2 * NST + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};

enum DecSite { D_EMPTY = 41, D_FULL };

// Sequence length of b, clamped to the valid range (an out-of-range value is
// reported through the status word).
__device__ __forceinline__ int dec_len(const DecArgs& a, int b) {
  int len = a.seq_lens[b];
  const int cap = a.max_pages * a.page_size;
  if (len < 1 || len > cap) {
    atomicOr(&g_status, 2u);
    len = len < 1 ? 1 : cap;
  }
  return len;
}

// GM: the head group (1, 2, 3 or 4 exactly; 5..8 rounded up to 8, the kernel
// then handling the first G): every head costs the same score and P V work,
// so a padded head is pure overhead.
template <int HD, int GM>
__global__ void __launch_bounds__(DEC_THREADS)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const DecArgs a) {
  using C = DecCfg<HD>;
  constexpr int NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V;
  float* q_s = reinterpret_cast<float*>(gbase + C::OFF_Q);
  float* p_s = reinterpret_cast<float*>(gbase + C::OFF_P);
  float* c_s = reinterpret_cast<float*>(gbase + C::OFF_C);
  volatile int* flag = reinterpret_cast<volatile int*>(gbase + C::OFF_FLAG);
  const uint32_t bars = base + C::OFF_BAR;
  auto bar_full = [&](int s) { return bars + 8u * s; };
  auto bar_empty = [&](int s) { return bars + 8u * (NST + s); };
  volatile WaitCtl* ctl = reinterpret_cast<volatile WaitCtl*>(gbase + C::OFF_BAR + 16 * NST + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = (int)(blockIdx.x % a.n_splits);
  const int bkv = (int)(blockIdx.x / a.n_splits);
  const int b = bkv / a.Hkv, kv = bkv % a.Hkv;
  const int G = a.G;
  const int len = dec_len(a, b);
  const int k0 = split * a.keys_per_split;
  const int k1 = min(len, k0 + a.keys_per_split);
  const int n_pieces = k1 > k0 ? (k1 - k0 + 31) / 32 : 0;

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
    // The whole warp reads the block-table entries of 32 pieces at a time
    // into shared memory (32 independent loads instead of one dependent
    // global read per page in front of every copy); lane 0 then checks them
    // and issues the copies.
    if (n_pieces > 0) {
      int* tbl = reinterpret_cast<int*>(gbase + C::OFF_TBL);
      if (lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      const int rows = a.page_size < 32 ? a.page_size : 32;  // rows per TMA box
      const int nbox = 32 / rows;                              // boxes per 32-key piece
      int issued = 0;
      bool ok = true;
      for (int t0 = 0; ok && t0 < n_pieces; t0 += 32) {
        for (int e = lane; e < 32 * nbox; e += 32) {  // e = (t - t0) * nbox + x
          const int t = t0 + e / nbox, key = k0 + 32 * t + (e % nbox) * rows;
          tbl[e] = t < n_pieces && key < k1 ? a.block_table[(size_t)b * a.max_pages + key / a.page_size] : 0;
        }
        __syncwarp();
        if (lane == 0) {
          const int t1 = min(n_pieces, t0 + 32);
          for (int t = t0; t < t1; ++t) {
            const int s = t % NST;
            if (t >= NST && !mbar_wait_bounded<true>(bar_empty(s), ((t / NST) & 1) ^ 1, ctl, D_EMPTY)) {
              ok = false;
              break;
            }
            const int kt = k0 + 32 * t;
            // pages of this piece (at most 4: page_size >= 8), checked before any copy
            int usable = 1, nload = 0, pages[4] = {0, 0, 0, 0};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const int key = kt + x * rows;
              if (x < nbox && key < k1) {
                pages[x] = tbl[(t - t0) * nbox + x];
                if (pages[x] < 0 || pages[x] >= a.num_pages) usable = 0;
                ++nload;
              }
            }
            flag[s] = usable;
            if (!usable) {
              atomicOr(&g_status, 2u);
              mbar_arrive(bar_full(s));
            } else {
              mbar_arrive_expect_tx(bar_full(s), (uint32_t)(nload * rows * HD * 2 * 2));
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                if (x >= nload) break;
                const int key = kt + x * rows;
                const int row = pages[x] * a.page_size + key % a.page_size;
#pragma unroll
                for (int sl = 0; sl < C::NSLAB; ++sl) {
                  const uint32_t off = s * C::PIECE + sl * C::SLAB + x * rows * 128;
                  tma_load_3d(sK + off, &tm_k, bar_full(s), 64 * sl, kv, row);
                  tma_load_3d(sV + off, &tm_v, bar_full(s), 64 * sl, kv, row);
                }
              }
            }
            issued = t + 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();  // lane 0 is done with this block of table entries
      }
      // drain: every copy started has landed before the CTA exits
      if (lane == 0) {
        volatile WaitCtl never = {0, 0, 0};
        for (int t = issued - NST > 0 ? issued - NST : 0; t < issued; ++t)
          mbar_wait_bounded<true>(bar_full(t % NST), (t / NST) & 1, &never, D_FULL);
      }
    }
  } else {
    // ============================================================ compute warps
    const int cw = warp - 1;
    // q of the group's G heads -> shared memory, fp32, pre-scaled to log2 units
    for (int x = threadIdx.x - 32; x < GM * HD; x += DEC_CW * 32) {
      const int g = x / HD;
      q_s[x] = g < G ? __bfloat162float(a.q[((size_t)b * a.Hq + kv * G + g) * HD + x % HD]) * a.scale_log2 : 0.f;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");

    constexpr int FPL = HD / 32;  // features per lane in O += p V
    float m[GM], lsum[GM];
    uint64_t acc_o[GM][FPL / 2];  // O of each head, packed feature pairs (fp32 x2)
#pragma unroll
    for (int g = 0; g < GM; ++g) {
      m[g] = -INFINITY;
      lsum[g] = 0.f;
#pragma unroll
      for (int f = 0; f < FPL / 2; ++f) acc_o[g][f] = f2_pack(0.f, 0.f);
    }
    float* pw = p_s + cw * 32 * 8;
    bool ok = true;
    for (int t = cw; ok && t < n_pieces; t += DEC_CW) {
      const int s = t % NST;
      if (!wait_warp<true>(bar_full(s), (t / NST) & 1, ctl, D_FULL)) { ok = false; break; }
      const int n_valid = min(32, k1 - (k0 + 32 * t));
      if (flag[s]) {
        // ---- scores: lane = key row of the piece
        const int r = lane;
        uint64_t sc2[GM];
#pragma unroll
        for (int g = 0; g < GM; ++g) sc2[g] = f2_pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < HD / 8; ++c) {
          const uint32_t addr = sK + s * C::PIECE + (c >> 3) * C::SLAB + r * 128 + (((c & 7) ^ (r & 7)) << 4);
          uint32_t kx, ky, kz, kw;
          asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(kx), "=r"(ky), "=r"(kz), "=r"(kw) : "r"(addr));
          const uint64_t k01 = f2_pack(__uint_as_float(kx << 16), __uint_as_float(kx & 0xffff0000u));
          const uint64_t k23 = f2_pack(__uint_as_float(ky << 16), __uint_as_float(ky & 0xffff0000u));
          const uint64_t k45 = f2_pack(__uint_as_float(kz << 16), __uint_as_float(kz & 0xffff0000u));
          const uint64_t k67 = f2_pack(__uint_as_float(kw << 16), __uint_as_float(kw & 0xffff0000u));
#pragma unroll
          for (int g = 0; g < GM; ++g) {
            const float4 qa = *reinterpret_cast<const float4*>(q_s + g * HD + 8 * c);
            const float4 qb = *reinterpret_cast<const float4*>(q_s + g * HD + 8 * c + 4);
            sc2[g] = f2_fma(f2_pack(qa.x, qa.y), k01, sc2[g]);
            sc2[g] = f2_fma(f2_pack(qa.z, qa.w), k23, sc2[g]);
            sc2[g] = f2_fma(f2_pack(qb.x, qb.y), k45, sc2[g]);
            sc2[g] = f2_fma(f2_pack(qb.z, qb.w), k67, sc2[g]);
          }
        }
        // ---- online softmax per head (log2 domain)
#pragma unroll
        for (int g = 0; g < GM; ++g) {
          float lo, hi;
          f2_unpack(sc2[g], lo, hi);
          const float sv = r < n_valid ? lo + hi : -INFINITY;
          float mx = sv;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          const float m_new = fmaxf(m[g], mx);
          const float alpha = ex2_approx(m[g] - m_new);  // 0 on the first piece (m = -inf)
          const float p = ex2_approx(sv - m_new);        // masked keys: 0
          m[g] = m_new;
          lsum[g] = lsum[g] * alpha + p;
#pragma unroll
          for (int f = 0; f < FPL / 2; ++f) acc_o[g][f] = f2_mul(acc_o[g][f], f2_pack(alpha, alpha));
          pw[r * 8 + g] = p;
        }
        __syncwarp();
        // ---- O += p V: lane = FPL consecutive features of every key row (unrolled
        // so that several rows' shared-memory loads are in flight at once; rows
        // past the sequence's end are never read: they hold whatever the page
        // pool holds there)
#pragma unroll 4
        for (int rr = 0; rr < n_valid; ++rr) {
          const uint32_t byte = lane * FPL * 2;  // this lane's bytes in the row
          const uint32_t vaddr = sV + s * C::PIECE + (byte >> 7) * C::SLAB + rr * 128 +
                                 ((((byte & 127) >> 4) ^ (rr & 7)) << 4) + (byte & 15);
          float vf[FPL];
          if constexpr (FPL == 4) {
            uint32_t vx, vy;
            asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(vx), "=r"(vy) : "r"(vaddr));
            vf[0] = __uint_as_float(vx << 16);
            vf[1] = __uint_as_float(vx & 0xffff0000u);
            vf[2] = __uint_as_float(vy << 16);
            vf[3] = __uint_as_float(vy & 0xffff0000u);
          } else {
            uint32_t vx;
            asm volatile("ld.shared.b32 %0, [%1];" : "=r"(vx) : "r"(vaddr));
            vf[0] = __uint_as_float(vx << 16);
            vf[1] = __uint_as_float(vx & 0xffff0000u);
          }
          // the row's p of every head in one or two 16-byte loads
          float pr[8];
          *reinterpret_cast<float4*>(pr) = *reinterpret_cast<const float4*>(pw + rr * 8);
          if constexpr (GM > 4) *reinterpret_cast<float4*>(pr + 4) = *reinterpret_cast<const float4*>(pw + rr * 8 + 4);
#pragma unroll
          for (int g = 0; g < GM; ++g) {
            const uint64_t p2 = f2_pack(pr[g], pr[g]);
#pragma unroll
            for (int f = 0; f < FPL / 2; ++f) acc_o[g][f] = f2_fma(p2, f2_pack(vf[2 * f], vf[2 * f + 1]), acc_o[g][f]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(s));
    }
    // ---- merge the four warps' states, then write the split's result
#pragma unroll
    for (int g = 0; g < GM; ++g) {
      float l = lsum[g];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      float* cs = c_s + (cw * 8 + g) * (HD + 2);
#pragma unroll
      for (int f = 0; f < FPL / 2; ++f) f2_unpack(acc_o[g][f], cs[2 + lane * FPL + 2 * f], cs[3 + lane * FPL + 2 * f]);
      if (lane == 0) {
        cs[0] = m[g];
        cs[1] = l;
      }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    for (int g = cw; g < G; g += DEC_CW) {
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < DEC_CW; ++w) mm = fmaxf(mm, c_s[(w * 8 + g) * (HD + 2)]);
      float l = 0.f, ov[FPL];
#pragma unroll
      for (int f = 0; f < FPL; ++f) ov[f] = 0.f;
#pragma unroll
      for (int w = 0; w < DEC_CW; ++w) {
        const float* cs = c_s + (w * 8 + g) * (HD + 2);
        const float e = cs[1] > 0.f ? ex2_approx(cs[0] - mm) : 0.f;  // warps without keys weigh 0
        l += cs[1] * e;
#pragma unroll
        for (int f = 0; f < FPL; ++f) ov[f] += cs[2 + lane * FPL + f] * e;
      }
      const int bh = b * a.Hq + kv * G + g;
      if (a.n_splits == 1) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int f = 0; f < FPL; ++f) a.o[(size_t)bh * HD + lane * FPL + f] = __float2bfloat16_rn(ov[f] * inv);
        if (lane == 0) a.lse[bh] = (mm + __log2f(l)) * 0.69314718055994531f;
      } else {
        float* dst = a.part + ((size_t)bh * a.n_splits + split) * (HD + 2);
#pragma unroll
        for (int f = 0; f < FPL; ++f) dst[2 + lane * FPL + f] = ov[f];
        if (lane == 0) {
          dst[0] = mm;
          dst[1] = l;
        }
      }
    }
  }
}

// Merge the splits of every (b, h): one warp per row, lanes over features.
template <int HD>
__global__ void __launch_bounds__(256) attn_decode_combine_kernel(const float* __restrict__ part,
                                                                  __nv_bfloat16* __restrict__ o,
                                                                  float* __restrict__ lse, int rows, int n_splits) {
  constexpr int FPL = HD / 32;
  const int lane = threadIdx.x & 31;
  for (int bh = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5); bh < rows;
       bh += (int)((gridDim.x * blockDim.x) >> 5)) {
    const float* p = part + (size_t)bh * n_splits * (HD + 2);
    float mm = -INFINITY;
    for (int s = 0; s < n_splits; ++s)
      if (p[s * (HD + 2) + 1] > 0.f) mm = fmaxf(mm, p[s * (HD + 2)]);
    float l = 0.f, ov[FPL];
#pragma unroll
    for (int f = 0; f < FPL; ++f) ov[f] = 0.f;
    for (int s = 0; s < n_splits; ++s) {
      const float* ps = p + s * (HD + 2);
      if (!(ps[1] > 0.f)) continue;  // a split past the end of the sequence
      const float e = ex2_approx(ps[0] - mm);
      l += ps[1] * e;
#pragma unroll
      for (int f = 0; f < FPL; ++f) ov[f] += ps[2 + lane * FPL + f] * e;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int f = 0; f < FPL; ++f) o[(size_t)bh * HD + lane * FPL + f] = __float2bfloat16_rn(ov[f] * inv);
    if (lane == 0) lse[bh] = (mm + __log2f(l)) * 0.69314718055994531f;
  }
}

}  // namespace axis_attn
