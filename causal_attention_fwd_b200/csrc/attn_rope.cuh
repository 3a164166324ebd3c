// attn_rope.cuh -- rotary position embedding (RoPE) for the attention inputs:
// the cos/sin table, the HBM-bound rotation of a [B, S, H, D] tensor (forward
// and transposed), and the transposed rotation of one gradient pair that the
// backward's epilogues apply to dQ and dK.
//
// The axiomlm page (PyPI) lists RoPE among its Key Features and its Quick
// Start (section 8) calls precompute_rope_frequencies(dim, end) and then
// apply_rope(q, k, freqs_cis) before attention; it gives no formula.  The
// reading taken (the complex-pair form that the name freqs_cis points to): in
// the row at sequence position s, the pair (x[2p], x[2p+1]) is turned by the
// angle s * theta_p, theta_p = base^(-2p / D):
//   x'[2p]   = x[2p] cos - x[2p+1] sin,   x'[2p+1] = x[2p] sin + x[2p+1] cos,
// and gradients go back through the transposed rotation (angle -s theta_p).
//
// Precision: the rotated Q and K are attention inputs stored in bf16, so the
// table (fp64 cos, sin) and the input rotations run in fp64 and round once to
// bf16 (round to nearest even, directly from fp64): the stored result is the
// correctly rounded rotation.  The gradient rotations (dQ, dK, fp32 values
// from the accumulators) use the same table in fp32.
#pragma once

#include "sm100_ptx.cuh"

namespace axis_attn {

// cs[s * D/2 + p] = (cos, sin)(s * base^(-2p/D)), fp64.
__global__ void __launch_bounds__(256) rope_table_kernel(double2* __restrict__ cs, long long n, int half_d,
                                                         double log2_base) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const long long s = i / half_d;
    const int p = (int)(i % half_d);
    const double theta = exp2(-2.0 * p / (2.0 * half_d) * log2_base);
    double sn, c;
    sincos((double)s * theta, &sn, &c);
    cs[i] = make_double2(c, sn);
  }
}

// Rotate the 4 pairs of one 16-byte word (8 bf16) by table entries t[0..3]
// (fp64), each result rounded once from fp64 to bf16 (round to nearest even:
// CUDA's __double2bfloat16), so the stored value is the correctly rounded
// rotation.
__device__ __forceinline__ uint4 rope_rotate8_f64(uint4 x, const double2* __restrict__ t) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double2 cs = t[i];
    const double x0 = (double)__uint_as_float(w[i] << 16), x1 = (double)__uint_as_float(w[i] & 0xffff0000u);
    const uint32_t y0 = __bfloat16_as_ushort(__double2bfloat16(fma(x0, cs.x, -x1 * cs.y)));
    const uint32_t y1 = __bfloat16_as_ushort(__double2bfloat16(fma(x0, cs.y, x1 * cs.x)));
    o[i] = y0 | (y1 << 16);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// The transposed rotation of one pair of fp32 gradient values.
__device__ __forceinline__ void rope_back(float& g0, float& g1, double2 cs) {
  const float c = (float)cs.x, s = (float)cs.y;
  const float a = fmaf(g0, c, g1 * s), b = fmaf(-g0, s, g1 * c);
  g0 = a;
  g1 = b;
}

// The 16-byte words of [B, S, H, D] bf16 are walked position by position
// (b, s): a position's H * D / 8 words are contiguous and share one row of the
// table, so the position index costs one modulo per position, not three
// 64-bit divisions per word.  A block takes ppb positions at a time (several
// when a position has fewer words than the block has threads).
struct RopeWalk {
  int wpp, ppb;  // words per position, positions per block step
  __device__ RopeWalk(int H, int D) : wpp(H * D / 8), ppb(wpp < (int)blockDim.x ? (int)blockDim.x / wpp : 1) {}
};

// Positions per thread and loop trip whose loads are in flight together (the
// kernel is bound by memory latency: one 16-byte load at a time per thread
// reached 2.4 TB/s).
constexpr int ROPE_U = 4;

// y = R x for x, y [B, S, H, D] bf16 (in place allowed: a thread reads all of
// its words of a trip before it writes any, and no two threads share a word);
// HBM-bound (the table stays in L2 / L1).
__global__ void __launch_bounds__(256) rope_apply_kernel(const uint4* x, uint4* y, const double2* __restrict__ cs,
                                                         long long npos, int S, int H, int D) {
  const RopeWalk rw(H, D);
  const int wpr = D / 8;  // words per head row (8 or 16)
  const int sub = (int)threadIdx.x / rw.wpp, w0 = (int)threadIdx.x % rw.wpp;
  if (sub >= rw.ppb) return;
  const long long pstep = (long long)gridDim.x * rw.ppb;
  for (int w = w0; w < rw.wpp; w += rw.ppb == 1 ? (int)blockDim.x : rw.wpp) {
    const int tw = 4 * (w & (wpr - 1));
    for (long long p0 = (long long)blockIdx.x * rw.ppb + sub; p0 < npos; p0 += ROPE_U * pstep) {
      uint4 xv[ROPE_U];
#pragma unroll
      for (int u = 0; u < ROPE_U; ++u) {
        const long long p = p0 + u * pstep;
        if (p < npos) xv[u] = x[(size_t)p * rw.wpp + w];
      }
#pragma unroll
      for (int u = 0; u < ROPE_U; ++u) {
        const long long p = p0 + u * pstep;
        if (p < npos) y[(size_t)p * rw.wpp + w] = rope_rotate8_f64(xv[u], cs + (size_t)(p % S) * (D / 2) + tw);
      }
    }
  }
}

// y = R^T x (the gradient direction), fp32 math, for the standalone call.
__global__ void __launch_bounds__(256) rope_apply_back_kernel(const uint4* x, uint4* y,
                                                              const double2* __restrict__ cs, long long npos, int S,
                                                              int H, int D) {
  const RopeWalk rw(H, D);
  const int wpr = D / 8;
  const int sub = (int)threadIdx.x / rw.wpp, w0 = (int)threadIdx.x % rw.wpp;
  if (sub >= rw.ppb) return;
  const long long pstep = (long long)gridDim.x * rw.ppb;
  for (int w = w0; w < rw.wpp; w += rw.ppb == 1 ? (int)blockDim.x : rw.wpp) {
    const int tw = 4 * (w & (wpr - 1));
    for (long long p0 = (long long)blockIdx.x * rw.ppb + sub; p0 < npos; p0 += ROPE_U * pstep) {
      uint4 xv[ROPE_U];
#pragma unroll
      for (int u = 0; u < ROPE_U; ++u) {
        const long long p = p0 + u * pstep;
        if (p < npos) xv[u] = x[(size_t)p * rw.wpp + w];
      }
#pragma unroll
      for (int u = 0; u < ROPE_U; ++u) {
        const long long p = p0 + u * pstep;
        if (p >= npos) continue;
        const double2* t = cs + (size_t)(p % S) * (D / 2) + tw;
        const uint32_t v[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float g0 = __uint_as_float(v[k] << 16), g1 = __uint_as_float(v[k] & 0xffff0000u);
          rope_back(g0, g1, t[k]);
          o[k] = pack_bf16x2(g0, g1);
        }
        y[(size_t)p * rw.wpp + w] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

}  // namespace axis_attn
