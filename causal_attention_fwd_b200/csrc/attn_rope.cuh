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

// fp64 -> bf16 bits, round to nearest even from the fp64 value itself (one
// rounding: 45 mantissa bits dropped).  Values below the smallest normal bf16
// flush to signed zero; the attention inputs never come near either end of
// the range.
__device__ __forceinline__ uint32_t f64_to_bf16_rn(double x) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(x);
  const uint32_t sign = (uint32_t)(u >> 63) << 15;
  int e = (int)((u >> 52) & 0x7ff) - 1023 + 127;
  if (e <= 0) return sign;
  unsigned long long keep = (u >> 45) & 0x7f;
  const unsigned long long rest = u & ((1ull << 45) - 1), half = 1ull << 44;
  if (rest > half || (rest == half && (keep & 1))) {
    if (++keep == 0x80) {
      keep = 0;
      ++e;
    }
  }
  if (e >= 255) return sign | 0x7f80u;
  return sign | ((uint32_t)e << 7) | (uint32_t)keep;
}

// Rotate the 4 pairs of one 16-byte word (8 bf16) by table entries t[0..3]
// (fp64), result correctly rounded to bf16.
__device__ __forceinline__ uint4 rope_rotate8_f64(uint4 x, const double2* __restrict__ t) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double2 cs = t[i];
    const double x0 = (double)__uint_as_float(w[i] << 16), x1 = (double)__uint_as_float(w[i] & 0xffff0000u);
    const uint32_t y0 = f64_to_bf16_rn(fma(x0, cs.x, -x1 * cs.y));
    const uint32_t y1 = f64_to_bf16_rn(fma(x0, cs.y, x1 * cs.x));
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

// y = R x for x, y [B, S, H, D] bf16 (in place allowed), one thread per
// 16-byte word (4 pairs), grid-stride; HBM-bound (the table stays in L2).
__global__ void __launch_bounds__(256) rope_apply_kernel(const uint4* x, uint4* y, const double2* __restrict__ cs,
                                                         long long n16, int S, int H, int D) {
  const int w_per_row = D / 8;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) {
    const long long row = i / w_per_row;  // (b * S + s) * H + h
    const int wd = (int)(i % w_per_row);
    const int s = (int)((row / H) % S);
    y[i] = rope_rotate8_f64(x[i], cs + (size_t)s * (D / 2) + 4 * wd);
  }
}

// y = R^T x (the gradient direction), fp32 math, for the standalone call.
__global__ void __launch_bounds__(256) rope_apply_back_kernel(const uint4* x, uint4* y,
                                                              const double2* __restrict__ cs, long long n16, int S,
                                                              int H, int D) {
  const int w_per_row = D / 8;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) {
    const long long row = i / w_per_row;
    const int wd = (int)(i % w_per_row);
    const int s = (int)((row / H) % S);
    const double2* t = cs + (size_t)s * (D / 2) + 4 * wd;
    const uint4 xv = x[i];
    const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float g0 = __uint_as_float(w[k] << 16), g1 = __uint_as_float(w[k] & 0xffff0000u);
      rope_back(g0, g1, t[k]);
      o[k] = pack_bf16x2(g0, g1);
    }
    y[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace axis_attn
