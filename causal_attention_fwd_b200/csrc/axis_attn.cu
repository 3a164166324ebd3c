// axis_attn.cu -- host side of the C ABI declared in include/axis_attn.h:
// argument validation, TMA tensor maps, workspace layout and kernel launches.
// All device work is in attn_fwd.cuh and attn_bwd.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/axis_attn.h"
#include "attn_bwd.cuh"
#include "attn_bwd_dq.cuh"
#include "attn_decode.cuh"
#include "attn_fwd.cuh"
#include "attn_rope.cuh"

namespace axis_attn {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Device check, cached per device: compute capability 10.0 only.
int check_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return AXIS_ATTN_ERR_CUDA;
  static int cached[64];  // 0 unknown, 1 ok, 2 unsupported
  if (dev < 0 || dev >= 64) return AXIS_ATTN_ERR_UNSUPPORTED;
  if (cached[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return AXIS_ATTN_ERR_CUDA;
    cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  *dev_out = dev;
  return cached[dev] == 1 ? AXIS_ATTN_OK : AXIS_ATTN_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int Hq, int Hkv, int S, int D, float scale) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || Hq % Hkv != 0) return AXIS_ATTN_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return AXIS_ATTN_ERR_SHAPE;
  if (D != 64 && D != 128) return AXIS_ATTN_ERR_UNSUPPORTED;
  const long long elems = (long long)B * S * (Hq > Hkv ? Hq : Hkv) * D;
  if (elems >= (1LL << 31)) return AXIS_ATTN_ERR_SHAPE;
  return AXIS_ATTN_OK;
}

// 4-D map over a [B, S, H, D] bf16 tensor: dims (D, H, S, B), box (64, 1, rows, 1),
// 128-byte swizzle, out-of-range rows read as zero.
bool make_map(CUtensorMap* map, const void* ptr, int B, int S, int H, int D, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)S * H * D * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the fp32 dQ accumulator [B*Hq][S][D]: dims (D, S, B*Hq), box
// (32, 64, 1), 128-byte swizzle; used by TMA reduce-adds (rows past S skipped).
bool make_dq_map(CUtensorMap* map, const float* ptr, int BH, int S, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)S * D * 4};
  const cuuint32_t box[3] = {32, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

// Head split of the backward main kernel: with fewer than BWD_SPLIT_CTAS
// (b, kv head, key tile) CTAs and more than one query head per kv head, the
// group's heads are dealt over hsplit CTAs (the smallest divisor of G that
// reaches that many CTAs, else G), which write fp32 partial dK, dV.
#ifndef AXIS_ATTN_BWD_SPLIT_CTAS
#define AXIS_ATTN_BWD_SPLIT_CTAS 148
#endif
constexpr long long BWD_SPLIT_CTAS = AXIS_ATTN_BWD_SPLIT_CTAS;
int bwd_hsplit(int B, int Hq, int Hkv, int S) {
  const int G = Hq / Hkv;
  const long long ctas = (long long)((S + 127) / 128) * B * Hkv;
  if (G <= 1 || ctas >= BWD_SPLIT_CTAS) return 1;
  for (int d = 2; d < G; ++d)
    if (G % d == 0 && ctas * d >= BWD_SPLIT_CTAS) return d;
  return G;
}

struct WsLayout {
  size_t lse2, dr, dqacc, dkpart, dvpart, total;
  int S_pad, hsplit;
};

// det: no dQ accumulator (the deterministic dQ pass keeps dQ in TMEM).  With a
// head split, two fp32 partial sections [hsplit][B][S][Hkv][D] follow.
WsLayout ws_layout(int B, int Hq, int Hkv, int S, int D, bool det = false) {
  WsLayout w;
  w.S_pad = (S + 127) / 128 * 128;
  w.hsplit = bwd_hsplit(B, Hq, Hkv, S);
  const size_t rows = (size_t)B * Hq * w.S_pad;
  w.lse2 = 0;
  w.dr = round256(rows * 4);
  w.dqacc = w.dr + round256(rows * 4);
  w.dkpart = w.dqacc + (det ? 0 : round256((size_t)B * Hq * S * D * 4));
  const size_t part = w.hsplit > 1 ? round256((size_t)w.hsplit * B * S * Hkv * D * 4) : 0;
  w.dvpart = w.dkpart + part;
  w.total = w.dvpart + part;
  return w;
}

// Number of SMs of device `dev` (cached; the persistent kernels launch one CTA per SM).
int sm_count(int dev) {
  static int count[64];
  if (count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    count[dev] = n;
  }
  return count[dev];
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
// `done` is a static of the calling template instantiation, so each kernel has
// its own flags.
template <typename K>
int set_smem(K kernel, uint32_t bytes, int dev, bool (&done)[64]) {
  if (!done[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
      return AXIS_ATTN_ERR_CUDA;
    done[dev] = true;
  }
  return AXIS_ATTN_OK;
}

template <int HD, bool CAUSAL>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FwdArgs& a,
               cudaStream_t st, int dev) {
  auto kern = attn_fwd_kernel<HD, CAUSAL>;
  static bool done[64];
  if (int rc = set_smem(kern, FwdCfg<HD>::SMEM, dev, done)) return rc;
  // persistent: one CTA per SM (the kernel walks its share of the items)
  const unsigned grid = (unsigned)(a.n_items < sm_count(dev) ? a.n_items : sm_count(dev));
  kern<<<grid, FWD_THREADS, FwdCfg<HD>::SMEM, st>>>(mq, mk, mv, a);
  return cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

// 0: always two query tiles per forward item.
#ifndef AXIS_ATTN_FWD_SINGLE_TILE_ITEMS
#define AXIS_ATTN_FWD_SINGLE_TILE_ITEMS 1
#endif

// The forward kernel over (q, k, v).
int run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int S, int D,
            float scale, int causal, cudaStream_t st, int dev) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, B, S, Hq, D, 128) || !make_map(&mk, k, B, S, Hkv, D, 128) ||
      !make_map(&mv, v, B, S, Hkv, D, 128))
    return AXIS_ATTN_ERR_CUDA;
  FwdArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.S = S;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  // two query tiles per item, unless that leaves SMs without an item: then
  // one (twice the items, half the longest chain of kv tiles)
  a.tpi = AXIS_ATTN_FWD_SINGLE_TILE_ITEMS && (long long)((S + 255) / 256) * B * Hq < sm_count(dev) ? 1 : 2;
  a.n_qblocks = (S + 128 * a.tpi - 1) / (128 * a.tpi);
  a.n_items = a.n_qblocks * B * Hq;
  if (D == 64)
    return causal ? launch_fwd<64, true>(mq, mk, mv, a, st, dev) : launch_fwd<64, false>(mq, mk, mv, a, st, dev);
  return causal ? launch_fwd<128, true>(mq, mk, mv, a, st, dev) : launch_fwd<128, false>(mq, mk, mv, a, st, dev);
}

// y = R x (inverse: R^T x) for x, y [B, S, H, D] bf16 with the table cs [S][D/2].
int run_rope(const void* x, void* y, const double* cs, int B, int S, int H, int D, int inverse, cudaStream_t st) {
  const long long npos = (long long)B * S;
  const int wpp = H * D / 8;
  const long long ppb = wpp < 256 ? 256 / wpp : 1;  // positions per block step (RopeWalk)
  const long long blocks = (npos + ppb - 1) / ppb;
  const unsigned grid = (unsigned)(blocks < 148 * 8 ? blocks : 148 * 8);
  const auto* t = reinterpret_cast<const double2*>(cs);
  if (inverse)
    rope_apply_back_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(x), static_cast<uint4*>(y), t, npos, S,
                                                 H, D);
  else
    rope_apply_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(x), static_cast<uint4*>(y), t, npos, S, H, D);
  return cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

template <int HD, bool CAUSAL>
int launch_bwd_dq(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                  const DqArgs& a, cudaStream_t st, int dev) {
  auto kern = attn_bwd_dq_kernel<HD, CAUSAL>;
  static bool done[64];
  if (int rc = set_smem(kern, DqCfg<HD>::SMEM, dev, done)) return rc;
  const unsigned grid = (unsigned)((a.S + 127) / 128) * a.B * a.Hq;
  kern<<<grid, DQ_THREADS, DqCfg<HD>::SMEM, st>>>(mq, mk, mv, mdo, a);
  return cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

template <int HD, bool CAUSAL>
int launch_bwd_main(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                    const CUtensorMap& mdq, const BwdArgs& a, cudaStream_t st, int dev) {
  auto kern = attn_bwd_kernel<HD, CAUSAL>;
  static bool done[64];
  if (int rc = set_smem(kern, BwdCfg<HD>::SMEM, dev, done)) return rc;
  const unsigned grid = (unsigned)((a.S + 127) / 128) * a.B * a.Hkv * a.hsplit;
  kern<<<grid, BwdCfg<HD>::THREADS, BwdCfg<HD>::SMEM, st>>>(mq, mk, mv, mdo, mdq, a);
  return cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

}  // namespace
}  // namespace axis_attn

using namespace axis_attn;

extern "C" int axis_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                             int Hkv, int S, int D, float scale, int causal, void* stream) {
  if (!q || !k || !v || !o || !lse) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return AXIS_ATTN_ERR_ALIGN;
  if (int rc = check_shape(B, Hq, Hkv, S, D, scale)) return rc;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  return run_fwd(q, k, v, o, lse, B, Hq, Hkv, S, D, scale, causal, static_cast<cudaStream_t>(stream), dev);
}

extern "C" size_t axis_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int S, int D) {
  if (check_shape(B, Hq, Hkv, S, D, 1.f) != AXIS_ATTN_OK) return 0;
  return ws_layout(B, Hq, Hkv, S, D).total;
}

extern "C" int axis_attn_bwd_head_split(int B, int Hq, int Hkv, int S, int D) {
  if (check_shape(B, Hq, Hkv, S, D, 1.f) != AXIS_ATTN_OK) return 0;
  return bwd_hsplit(B, Hq, Hkv, S);
}

namespace {

int check_ws(void* workspace, size_t workspace_bytes, const WsLayout& w) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < w.total)
    return AXIS_ATTN_ERR_WORKSPACE;
  return AXIS_ATTN_OK;
}

struct WsPtrs {
  float *lse2, *dr, *dqacc, *dkpart, *dvpart;
};

WsPtrs ws_ptrs(void* workspace, const WsLayout& w) {
  char* ws = static_cast<char*>(workspace);
  return {reinterpret_cast<float*>(ws + w.lse2), reinterpret_cast<float*>(ws + w.dr),
          reinterpret_cast<float*>(ws + w.dqacc), reinterpret_cast<float*>(ws + w.dkpart),
          reinterpret_cast<float*>(ws + w.dvpart)};
}

}  // namespace

namespace {

// Stage 1: -scale*Dr and -LSE*log2(e) rows (padding rows 0 / -inf); zero the
// dQ accumulator unless the deterministic mode's slices are used.
int run_prepare(const void* o, const void* dO, const float* lse, int B, int Hq, int S, int D, float scale,
                const WsLayout& w, const WsPtrs& p, bool zero_dq, cudaStream_t st) {
  const int rows = B * Hq * w.S_pad;
  const size_t dq_vec4 = zero_dq ? (size_t)B * Hq * S * D / 4 : 0;
  // grid-stride kernel: a few waves of 256-thread blocks over the 148 SMs, twice
  // as many when half of them zero the accumulator
  const size_t work = (size_t)B * Hq * S * (D / 8);
  unsigned grid = (unsigned)((work + 255) / 256 < 148 * 16 ? (work + 255) / 256 : 148 * 16);
  if (dq_vec4 > 0) grid *= 2;
  const auto* ob = static_cast<const __nv_bfloat16*>(o);
  const auto* db = static_cast<const __nv_bfloat16*>(dO);
  if (D == 64)
    attn_bwd_prep_kernel<64><<<grid, 256, 0, st>>>(ob, db, lse, p.lse2, p.dr, reinterpret_cast<float4*>(p.dqacc),
                                                   dq_vec4, Hq, S, w.S_pad, rows, scale);
  else
    attn_bwd_prep_kernel<128><<<grid, 256, 0, st>>>(ob, db, lse, p.lse2, p.dr, reinterpret_cast<float4*>(p.dqacc),
                                                    dq_vec4, Hq, S, w.S_pad, rows, scale);
  return cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

// Stage 2: the main kernel; det: dK, dV only (no dQ accumulator).
int run_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, int B, int Hq,
             int Hkv, int S, int D, float scale, int causal, const WsLayout& w, const WsPtrs& p, bool det,
             cudaStream_t st, int dev, const double* rope_cs = nullptr) {
  const int BM = D == 64 ? BwdCfg<64>::BM : BwdCfg<128>::BM;
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, q, B, S, Hq, D, BM) || !make_map(&mdo, dO, B, S, Hq, D, BM) ||
      !make_map(&mk, k, B, S, Hkv, D, 128) || !make_map(&mv, v, B, S, Hkv, D, 128))
    return AXIS_ATTN_ERR_CUDA;
  CUtensorMap mdq = {};  // not read by the kernel in the deterministic mode
  if (!det && !make_dq_map(&mdq, p.dqacc, B * Hq, S, D)) return AXIS_ATTN_ERR_CUDA;
  BwdArgs a;
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.nlse2 = p.lse2;
  a.ndr = p.dr;
  a.dqacc = p.dqacc;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.S = S;
  a.S_pad = w.S_pad;
  a.scale = scale;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  a.no_dq = det ? 1 : 0;
  a.rope_cs = reinterpret_cast<const double2*>(rope_cs);
  a.hsplit = w.hsplit;
  a.dk_part = p.dkpart;
  a.dv_part = p.dvpart;
  int rc;
  if (D == 64)
    rc = causal ? launch_bwd_main<64, true>(mq, mk, mv, mdo, mdq, a, st, dev)
                : launch_bwd_main<64, false>(mq, mk, mv, mdo, mdq, a, st, dev);
  else
    rc = causal ? launch_bwd_main<128, true>(mq, mk, mv, mdo, mdq, a, st, dev)
                : launch_bwd_main<128, false>(mq, mk, mv, mdo, mdq, a, st, dev);
  if (rc || w.hsplit == 1) return rc;
  // head split: add up the partial dK, dV (fixed order) into bf16 dk, dv
  const size_t n8 = (size_t)B * S * Hkv * D / 8;
  const unsigned grid = (unsigned)((2 * n8 + 255) / 256 < 148 * 8 ? (2 * n8 + 255) / 256 : 148 * 8);
  auto* dkb = static_cast<__nv_bfloat16*>(dk);
  auto* dvb = static_cast<__nv_bfloat16*>(dv);
  const double2* cs = reinterpret_cast<const double2*>(rope_cs);
  if (D == 64)
    attn_bwd_dkv_sum_kernel<64><<<grid, 256, 0, st>>>(p.dkpart, p.dvpart, dkb, dvb, w.hsplit, S, Hkv, n8, cs);
  else
    attn_bwd_dkv_sum_kernel<128><<<grid, 256, 0, st>>>(p.dkpart, p.dvpart, dkb, dvb, w.hsplit, S, Hkv, n8, cs);
  return cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

// Stage 3: dQ to bf16 [B,S,Hq,D].
int run_finalize(void* dq, int B, int Hq, int S, int D, const WsPtrs& p, cudaStream_t st,
                 const double* rope_cs = nullptr) {
  const size_t n8 = (size_t)B * S * Hq * D / 8;
  const unsigned grid = (unsigned)((n8 + 255) / 256 < 148 * 16 ? (n8 + 255) / 256 : 148 * 16);
  auto* out = static_cast<__nv_bfloat16*>(dq);
  const double2* cs = reinterpret_cast<const double2*>(rope_cs);
  if (D == 64) {
    attn_bwd_dq_convert_kernel<64><<<grid, 256, 0, st>>>(p.dqacc, out, Hq, S, n8, cs);
  } else {
    attn_bwd_dq_convert_kernel<128><<<grid, 256, 0, st>>>(p.dqacc, out, Hq, S, n8, cs);
  }
  return cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

}  // namespace

extern "C" int axis_attn_bwd_prepare(const void* o, const void* dO, const float* lse, int B, int Hq, int Hkv,
                                     int S, int D, float scale, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!o || !dO || !lse) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(o) || !aligned16(dO) || !aligned16(lse)) return AXIS_ATTN_ERR_ALIGN;
  if (int rc = check_shape(B, Hq, Hkv, S, D, scale)) return rc;
  const WsLayout w = ws_layout(B, Hq, Hkv, S, D);
  if (int rc = check_ws(workspace, workspace_bytes, w)) return rc;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  return run_prepare(o, dO, lse, B, Hq, S, D, scale, w, ws_ptrs(workspace, w), true,
                     static_cast<cudaStream_t>(stream));
}

extern "C" int axis_attn_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                                  int B, int Hq, int Hkv, int S, int D, float scale, int causal, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !dO || !dk || !dv) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) || !aligned16(dv))
    return AXIS_ATTN_ERR_ALIGN;
  if (int rc = check_shape(B, Hq, Hkv, S, D, scale)) return rc;
  const WsLayout w = ws_layout(B, Hq, Hkv, S, D);
  if (int rc = check_ws(workspace, workspace_bytes, w)) return rc;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  return run_main(q, k, v, dO, dk, dv, B, Hq, Hkv, S, D, scale, causal, w, ws_ptrs(workspace, w), false,
                  static_cast<cudaStream_t>(stream), dev);
}

extern "C" int axis_attn_bwd_finalize(void* dq, int B, int Hq, int Hkv, int S, int D, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!dq) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(dq)) return AXIS_ATTN_ERR_ALIGN;
  if (int rc = check_shape(B, Hq, Hkv, S, D, 1.f)) return rc;
  const WsLayout w = ws_layout(B, Hq, Hkv, S, D);
  if (int rc = check_ws(workspace, workspace_bytes, w)) return rc;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  return run_finalize(dq, B, Hq, S, D, ws_ptrs(workspace, w), static_cast<cudaStream_t>(stream));
}

namespace {

// Deterministic mode, stage 3: dQ recomputed per 128-row query tile.
int run_dq_pass(const void* q, const void* k, const void* v, const void* dO, void* dq, int B, int Hq, int Hkv,
                int S, int D, float scale, int causal, const WsLayout& w, const WsPtrs& p, cudaStream_t st,
                int dev, const double* rope_cs = nullptr) {
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, q, B, S, Hq, D, 128) || !make_map(&mdo, dO, B, S, Hq, D, 128) ||
      !make_map(&mk, k, B, S, Hkv, D, 128) || !make_map(&mv, v, B, S, Hkv, D, 128))
    return AXIS_ATTN_ERR_CUDA;
  DqArgs a;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.nlse2 = p.lse2;
  a.ndr = p.dr;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.S = S;
  a.S_pad = w.S_pad;
  a.scale = scale;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  a.rope_cs = reinterpret_cast<const double2*>(rope_cs);
  if (D == 64)
    return causal ? launch_bwd_dq<64, true>(mq, mk, mv, mdo, a, st, dev)
                  : launch_bwd_dq<64, false>(mq, mk, mv, mdo, a, st, dev);
  return causal ? launch_bwd_dq<128, true>(mq, mk, mv, mdo, a, st, dev)
                : launch_bwd_dq<128, false>(mq, mk, mv, mdo, a, st, dev);
}

// The backward; with a RoPE table, q and k hold the rotated inputs and dQ, dK
// leave through the transposed rotation.
int run_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse, void* dq,
            void* dk, void* dv, int B, int Hq, int Hkv, int S, int D, float scale, int causal, void* workspace,
            size_t workspace_bytes, void* stream, bool det, const double* rope_cs = nullptr) {
  // Validate everything first so that no stage runs when a later one would fail.
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (rope_cs && !aligned16(rope_cs)))
    return AXIS_ATTN_ERR_ALIGN;
  if (int rc = check_shape(B, Hq, Hkv, S, D, scale)) return rc;
  const WsLayout w = ws_layout(B, Hq, Hkv, S, D, det);
  if (int rc = check_ws(workspace, workspace_bytes, w)) return rc;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  const WsPtrs p = ws_ptrs(workspace, w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (int rc = run_prepare(o, dO, lse, B, Hq, S, D, scale, w, p, !det, st)) return rc;
  if (int rc = run_main(q, k, v, dO, dk, dv, B, Hq, Hkv, S, D, scale, causal, w, p, det, st, dev, rope_cs))
    return rc;
  if (det) return run_dq_pass(q, k, v, dO, dq, B, Hq, Hkv, S, D, scale, causal, w, p, st, dev, rope_cs);
  return run_finalize(dq, B, Hq, S, D, p, st, rope_cs);
}

}  // namespace

extern "C" int axis_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                             const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S, int D,
                             float scale, int causal, void* workspace, size_t workspace_bytes, void* stream) {
  return run_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal, workspace, workspace_bytes,
                 stream, false);
}

extern "C" size_t axis_attn_bwd_det_workspace_bytes(int B, int Hq, int Hkv, int S, int D) {
  if (check_shape(B, Hq, Hkv, S, D, 1.f) != AXIS_ATTN_OK) return 0;
  return ws_layout(B, Hq, Hkv, S, D, true).total;
}

extern "C" int axis_attn_bwd_det(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                 const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S,
                                 int D, float scale, int causal, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  return run_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal, workspace, workspace_bytes,
                 stream, true);
}

// ----------------------------------------------------------------------------
// Rotary position embedding (RoPE) of Q and K, fused with the attention.

extern "C" int axis_attn_rope_table(double* cs, int S, int D, double base, void* stream) {
  if (!cs) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(cs)) return AXIS_ATTN_ERR_ALIGN;
  if (S < 1 || D < 8 || D % 8 != 0 || !(std::isfinite(base) && base > 1.0)) return AXIS_ATTN_ERR_SHAPE;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  const long long n = (long long)S * (D / 2);
  const unsigned grid = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  rope_table_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(reinterpret_cast<double2*>(cs), n, D / 2,
                                                                         std::log2(base));
  return cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

extern "C" int axis_attn_rope(const void* x, void* y, const double* cs, int B, int S, int H, int D, int inverse,
                              void* stream) {
  if (!x || !y || !cs) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(x) || !aligned16(y) || !aligned16(cs)) return AXIS_ATTN_ERR_ALIGN;
  if (B < 1 || S < 1 || H < 1 || D < 8 || D % 8 != 0 || (long long)B * S * H * D >= (1LL << 40))
    return AXIS_ATTN_ERR_SHAPE;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  return run_rope(x, y, cs, B, S, H, D, inverse, static_cast<cudaStream_t>(stream));
}

extern "C" int axis_attn_fwd_rope(const void* q, const void* k, const void* v, const double* cs, void* o, float* lse,
                                  void* q_rot, void* k_rot, int B, int Hq, int Hkv, int S, int D, float scale,
                                  int causal, void* stream) {
  if (!q || !k || !v || !cs || !o || !lse || !q_rot || !k_rot) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(cs) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(q_rot) || !aligned16(k_rot))
    return AXIS_ATTN_ERR_ALIGN;
  if (int rc = check_shape(B, Hq, Hkv, S, D, scale)) return rc;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (int rc = run_rope(q, q_rot, cs, B, S, Hq, D, 0, st)) return rc;
  if (int rc = run_rope(k, k_rot, cs, B, S, Hkv, D, 0, st)) return rc;
  return run_fwd(q_rot, k_rot, v, o, lse, B, Hq, Hkv, S, D, scale, causal, st, dev);
}

extern "C" int axis_attn_bwd_rope(const void* q_rot, const void* k_rot, const void* v, const double* cs,
                                  const void* o, const void* dO, const float* lse, void* dq, void* dk, void* dv,
                                  int B, int Hq, int Hkv, int S, int D, float scale, int causal, int deterministic,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!cs) return AXIS_ATTN_ERR_NULL;
  return run_bwd(q_rot, k_rot, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal, workspace,
                 workspace_bytes, stream, deterministic != 0, cs);
}

// ----------------------------------------------------------------------------
// axis_attn_bwd_noalloc: the backward with library-owned scratch, for callers
// that may not call cudaMalloc (allocator callbacks, pre-reserved memory pools,
// paths that must not block on the allocator) and have no workspace to pass.
// The scratch is a fixed device array; the library never allocates or frees.

// The array's name in host code is only a handle for the runtime; the device
// address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[AXIS_ATTN_NOALLOC_SCRATCH_BYTES];

namespace axis_attn {
namespace {

void* g_noalloc_addr[64];
std::mutex g_noalloc_mutex;

int noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return AXIS_ATTN_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return AXIS_ATTN_OK;
}

}  // namespace
}  // namespace axis_attn

extern "C" int axis_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                     const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S,
                                     int D, float scale, int causal, void* stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return AXIS_ATTN_ERR_ALIGN;
  if (int rc = check_shape(B, Hq, Hkv, S, D, scale)) return rc;
  if (ws_layout(B, Hq, Hkv, S, D).total > (size_t)AXIS_ATTN_NOALLOC_SCRATCH_BYTES) return AXIS_ATTN_ERR_WORKSPACE;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  void* scratch = nullptr;
  if (int rc = noalloc_scratch(dev, &scratch)) return rc;
  return axis_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal, scratch,
                       (size_t)AXIS_ATTN_NOALLOC_SCRATCH_BYTES, stream);
}

// ----------------------------------------------------------------------------
// Decode step against a paged KV cache.

namespace axis_attn {
namespace {

bool pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

// q_len: new tokens per sequence (1 .. 64; a sequence must have room for them).
int check_decode_shape(int B, int Hq, int Hkv, int D, int page_size, int max_pages, int num_pages, float scale,
                       int q_len = 1) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || max_pages < 1 || num_pages < 1 || q_len < 1)
    return AXIS_ATTN_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return AXIS_ATTN_ERR_SHAPE;
  if (D != 64 && D != 128) return AXIS_ATTN_ERR_UNSUPPORTED;
  if (Hq / Hkv > 8 || !pow2_in(page_size, 8, 256) || q_len > 64) return AXIS_ATTN_ERR_UNSUPPORTED;
  if ((long long)max_pages * page_size >= (1LL << 30) || (long long)num_pages * page_size >= (1LL << 31) ||
      (long long)B * max_pages >= (1LL << 31) || (long long)B * q_len * Hq * D >= (1LL << 31) ||
      (long long)max_pages * page_size < q_len)
    return AXIS_ATTN_ERR_SHAPE;
  return AXIS_ATTN_OK;
}

// Splits of each sequence: at least 296 items (two per SM) when the batch is
// small, at least 256 keys (8 pieces) per split.  Measured against filling
// every CTA that fits at once (740 items): that rule was slower at batch 1-4
// (more partial results and per-item start-up for the same bytes) and faster
// only around batch 8 at D = 128.  A pure function of the shape, so that the
// workspace query needs no device.
struct DecSplit {
  int n_splits, keys_per_split;
};
#ifndef AXIS_ATTN_DEC_SPLIT_ITEMS
#define AXIS_ATTN_DEC_SPLIT_ITEMS 296
#endif
// The kernel's mode: 0 one new token; 1 several, at most 8 (token, head) rows
// per kv head (one 8-row tile); 2 more rows (tiles of 16).  A (b, kv head)
// unit is n_rt tiles.
int decode_mode(int Hq, int Hkv, int q_len) { return q_len == 1 ? 0 : Hq / Hkv * q_len <= 8 ? 1 : 2; }
int decode_row_tiles(int Hq, int Hkv, int q_len) {
  return decode_mode(Hq, Hkv, q_len) == 2 ? (Hq / Hkv * q_len + 15) / 16 : 1;
}
DecSplit decode_split(int B, int Hkv, int page_size, int max_pages, int n_rt = 1) {
  const long long keys = (long long)max_pages * page_size;
  const long long units = (long long)B * Hkv * n_rt;
  long long n = (AXIS_ATTN_DEC_SPLIT_ITEMS + units - 1) / units;
  const long long n_max = (keys + 255) / 256;
  if (n > n_max) n = n_max;
  if (n < 1) n = 1;
  long long kps = ((keys + n - 1) / n + 31) / 32 * 32;
  n = (keys + kps - 1) / kps;
  return {(int)n, (int)kps};
}

// partial (m, l, O) of every (b, new token, head) row and split
size_t decode_ws_bytes(int B, int Hq, int D, const DecSplit& sp, int q_len = 1) {
  return sp.n_splits > 1 ? (size_t)B * q_len * Hq * sp.n_splits * (D + 2) * 4 : 0;
}

// 3-D map over a paged cache [num_pages * page_size rows][Hkv][D] (bf16):
// dims (D, Hkv, rows), box (64, 1, min(page_size, 32)), 128-byte swizzle.
bool make_cache_map(CUtensorMap* map, const void* ptr, int rows, int Hkv, int D, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same pool in the head-major layout [num_pages, Hkv, page_size, D]: a
// 3-D map (D, page_size, num_pages * Hkv), box (64, box_rows, 1); a box lands
// in shared memory exactly as the other layout's does (box_rows rows of 128 B).
bool make_cache_map_hnd(CUtensorMap* map, const void* ptr, int num_pages, int page_size, int Hkv, int D,
                        int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)page_size, (cuuint64_t)num_pages * Hkv};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)page_size * D * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Persistent decode: as many CTAs as fit on the SMs at once (or one per item).
template <int HD, bool DEEP, int MODE>
int launch_decode_cfg(const CUtensorMap& mk, const CUtensorMap& mv, const DecArgs& a, cudaStream_t st, int dev,
                      long long items) {
  using C = DecCfg<HD, DEEP, MODE>;
  auto kern = attn_decode_kernel<HD, DEEP, MODE>;
  static bool done[64];
  static int per_sm[64];
  if (int rc = set_smem(kern, C::SMEM, dev, done)) return rc;
  if (per_sm[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, C::THREADS, C::SMEM) != cudaSuccess || n < 1) n = 1;
    per_sm[dev] = n;
  }
  const long long cap = (long long)per_sm[dev] * sm_count(dev);
  const unsigned grid = (unsigned)(items < cap ? items : cap);
  kern<<<grid, C::THREADS, C::SMEM, st>>>(mk, mv, a);
  return cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

// Resident CTAs per SM of a configuration, from its shared memory and threads
// (228 KB per SM, 1 KB reserved per CTA; 2048 threads).
template <int HD, bool DEEP, int MODE>
constexpr int dec_per_sm() {
  using C = DecCfg<HD, DEEP, MODE>;
  constexpr int by_smem = 233472 / (int)(C::SMEM + 1024), by_threads = 2048 / C::THREADS;
  return by_smem < by_threads ? by_smem : by_threads;
}

// The deep configuration when all items fit its CTAs in one wave (a small
// batch: the wide configuration's extra CTAs would have no item), else the
// wide one.  Measured (HBM fraction): 296-304 items, deep 0.43-0.56 against
// wide 0.39-0.51; 512 items, wide 0.80 against deep 0.59.
template <int HD>
int launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, const DecArgs& a, cudaStream_t st, int dev) {
  const long long items = (long long)a.B * a.Hkv * a.n_splits * a.n_rt;
  const int mode = decode_mode(a.Hq, a.Hkv, a.q_len);
  const int deep_per_sm = mode == 2 ? dec_per_sm<HD, true, 2>() : dec_per_sm<HD, true, 0>();
  const bool deep = items <= (long long)deep_per_sm * sm_count(dev);
  if (mode == 2)
    return deep ? launch_decode_cfg<HD, true, 2>(mk, mv, a, st, dev, items)
                : launch_decode_cfg<HD, false, 2>(mk, mv, a, st, dev, items);
  if (mode == 1)
    return deep ? launch_decode_cfg<HD, true, 1>(mk, mv, a, st, dev, items)
                : launch_decode_cfg<HD, false, 1>(mk, mv, a, st, dev, items);
  return deep ? launch_decode_cfg<HD, true, 0>(mk, mv, a, st, dev, items)
              : launch_decode_cfg<HD, false, 0>(mk, mv, a, st, dev, items);
}

}  // namespace
}  // namespace axis_attn

extern "C" size_t axis_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int D, int page_size, int max_pages) {
  if (check_decode_shape(B, Hq, Hkv, D, page_size, max_pages, 1, 1.f) != AXIS_ATTN_OK) return 0;
  return decode_ws_bytes(B, Hq, D, decode_split(B, Hkv, page_size, max_pages));
}

extern "C" size_t axis_attn_decode_q_workspace_bytes(int B, int q_len, int Hq, int Hkv, int D, int page_size,
                                                     int max_pages) {
  if (check_decode_shape(B, Hq, Hkv, D, page_size, max_pages, 1, 1.f, q_len) != AXIS_ATTN_OK) return 0;
  const int n_rt = decode_row_tiles(Hq, Hkv, q_len);
  return decode_ws_bytes(B, Hq, D, decode_split(B, Hkv, page_size, max_pages, n_rt), q_len);
}

namespace axis_attn {
namespace {
int run_decode(const void* q, const void* k_cache, const void* v_cache, const int* block_table, const int* seq_lens,
               void* o, float* lse, int B, int Hq, int Hkv, int D, int page_size, int max_pages, int num_pages,
               float scale, void* workspace, size_t workspace_bytes, void* stream, bool hnd, int q_len) {
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !o || !lse) return AXIS_ATTN_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return AXIS_ATTN_ERR_ALIGN;
  if (int rc = check_decode_shape(B, Hq, Hkv, D, page_size, max_pages, num_pages, scale, q_len)) return rc;
  const int n_rt = decode_row_tiles(Hq, Hkv, q_len);
  const DecSplit sp = decode_split(B, Hkv, page_size, max_pages, n_rt);
  const size_t need = decode_ws_bytes(B, Hq, D, sp, q_len);
  if (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need))
    return AXIS_ATTN_ERR_WORKSPACE;
  int dev = 0;
  if (int rc = check_device(&dev)) return rc;
  CUtensorMap mk, mv;
  const int box_rows = page_size < 32 ? page_size : 32;
  const bool maps_ok =
      hnd ? make_cache_map_hnd(&mk, k_cache, num_pages, page_size, Hkv, D, box_rows) &&
                make_cache_map_hnd(&mv, v_cache, num_pages, page_size, Hkv, D, box_rows)
          : make_cache_map(&mk, k_cache, num_pages * page_size, Hkv, D, box_rows) &&
                make_cache_map(&mv, v_cache, num_pages * page_size, Hkv, D, box_rows);
  if (!maps_ok) return AXIS_ATTN_ERR_CUDA;
  DecArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.part = static_cast<float*>(workspace);
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.page_size = page_size;
  a.max_pages = max_pages;
  a.num_pages = num_pages;
  a.hnd = hnd ? 1 : 0;
  a.q_len = q_len;
  a.n_rt = n_rt;
  a.keys_per_split = sp.keys_per_split;
  a.n_splits = sp.n_splits;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc = D == 64 ? launch_decode<64>(mk, mv, a, st, dev) : launch_decode<128>(mk, mv, a, st, dev);
  if (rc || sp.n_splits == 1) return rc;
  const int rows = B * q_len * Hq;
  const unsigned grid = (unsigned)(rows < 148 * 8 ? rows : 148 * 8);  // one CTA per (b, new token, h) row
  // programmatic dependent launch: the merge grid is scheduled while the decode
  // grid runs and waits in its first instruction for that grid's results
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  float* part = a.part;
  __nv_bfloat16* out = a.o;
  const int ns = sp.n_splits;
  const cudaError_t e = D == 64 ? cudaLaunchKernelEx(&cfg, attn_decode_combine_kernel<64>, (const float*)part, out,
                                                     lse, rows, ns, Hq, q_len)
                                : cudaLaunchKernelEx(&cfg, attn_decode_combine_kernel<128>, (const float*)part, out,
                                                     lse, rows, ns, Hq, q_len);
  return e == cudaSuccess && cudaPeekAtLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}
}  // namespace
}  // namespace axis_attn

extern "C" int axis_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                                const int* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int D,
                                int page_size, int max_pages, int num_pages, float scale, void* workspace,
                                size_t workspace_bytes, void* stream) {
  return axis_attn::run_decode(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size,
                               max_pages, num_pages, scale, workspace, workspace_bytes, stream, false, 1);
}

extern "C" int axis_attn_decode_hnd(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                                    const int* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int D,
                                    int page_size, int max_pages, int num_pages, float scale, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  return axis_attn::run_decode(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size,
                               max_pages, num_pages, scale, workspace, workspace_bytes, stream, true, 1);
}

extern "C" int axis_attn_decode_q(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                                  const int* seq_lens, void* o, float* lse, int B, int q_len, int Hq, int Hkv, int D,
                                  int page_size, int max_pages, int num_pages, float scale, int head_major,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  return axis_attn::run_decode(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size,
                               max_pages, num_pages, scale, workspace, workspace_bytes, stream, head_major != 0,
                               q_len);
}

static unsigned int g_last_status_word;

extern "C" unsigned int axis_attn_last_status_word(void) { return g_last_status_word; }

extern "C" int axis_attn_get_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return AXIS_ATTN_ERR_CUDA;
  unsigned int st = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&st, g_status, sizeof(st)) != cudaSuccess) return AXIS_ATTN_ERR_CUDA;
  g_last_status_word = st;
  if (st != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return AXIS_ATTN_ERR_CUDA;
  if (st & 1u) return AXIS_ATTN_ERR_TIMEOUT;
  if (st & 2u) return AXIS_ATTN_ERR_INDEX;
  return cudaGetLastError() == cudaSuccess ? AXIS_ATTN_OK : AXIS_ATTN_ERR_CUDA;
}

extern "C" const char* axis_attn_strerror(int code) {
  switch (code) {
    case AXIS_ATTN_OK: return "ok";
    case AXIS_ATTN_ERR_NULL: return "a required pointer is NULL";
    case AXIS_ATTN_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case AXIS_ATTN_ERR_SHAPE: return "invalid size, head ratio or scale";
    case AXIS_ATTN_ERR_UNSUPPORTED: return "unsupported head dim (need 64 or 128) or device (need sm_100)";
    case AXIS_ATTN_ERR_WORKSPACE: return "workspace NULL, not 256-byte aligned, or too small";
    case AXIS_ATTN_ERR_CUDA: return "CUDA runtime or driver error";
    case AXIS_ATTN_ERR_TIMEOUT: return "a device-side wait timed out";
    case AXIS_ATTN_ERR_INDEX: return "a device-side index (page table entry or sequence length) was out of range";
    default: return "unknown status";
  }
}
