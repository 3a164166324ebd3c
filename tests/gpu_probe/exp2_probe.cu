// Test-only probe: evaluates, on the GPU, the polynomial 2^x that the
// attention kernels use for part of their exponentials (f2_exp2_poly in
// sm100_ptx.cuh) and the MUFU ex2.approx.ftz it replaces, on the same inputs,
// so a test can compare both with the exact 2^x.  Built by the test into a
// temporary directory; not part of the library.
#include <cuda_runtime.h>

#include "../../causal_attention_fwd_b200/csrc/sm100_ptx.cuh"

using namespace axis_attn;

__global__ void exp2_probe_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                  float* __restrict__ y_mufu, int n_pairs) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_pairs; i += gridDim.x * blockDim.x) {
    const float a = x[2 * i], b = x[2 * i + 1];
    float p0, p1;
    f2_unpack(f2_exp2_poly(f2_pack(a, b)), p0, p1);
    y_poly[2 * i] = p0;
    y_poly[2 * i + 1] = p1;
    y_mufu[2 * i] = ex2_approx(a);
    y_mufu[2 * i + 1] = ex2_approx(b);
  }
}

// x, y_poly, y_mufu: device pointers to 2 * n_pairs floats.  Returns a cudaError_t.
extern "C" int exp2_probe(const float* x, float* y_poly, float* y_mufu, int n_pairs, void* stream) {
  if (n_pairs <= 0) return 0;
  const int blocks = (n_pairs + 255) / 256 < 1184 ? (n_pairs + 255) / 256 : 1184;
  exp2_probe_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly, y_mufu, n_pairs);
  return (int)cudaGetLastError();
}
