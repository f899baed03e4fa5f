// sala.cu -- libsala: C ABI entry points, host-side argument checks and launches.
//
// All kernels are compiled into this one translation unit so that they share
// the device error word.  Host code here does marshalling only: argument
// validation, tensor-map encoding for TMA, grid sizing and launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "lightning_cc.cuh"
#include "lightning_decode.cuh"
#include "lightning_tc.cuh"
#include "lightning_out.cuh"
#include "proj_gemm.cuh"
#include "sparse_attn.cuh"
#include "sparse_decode.cuh"
#include "sparse_select.cuh"
#include "sparse_select_tc.cuh"
#include "sparse_select_hsm_tc.cuh"

using namespace sala;

namespace {

#define SALA_CHECK_LAUNCH()                                \
  do {                                                     \
    if (cudaPeekAtLastError() != cudaSuccess) {            \
      (void)cudaGetLastError();                            \
      return SALA_ERR_CUDA;                                \
    }                                                      \
  } while (0)

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Strides (elements) of a [B,T,H,D] tensor: non-negative, rows 16-byte aligned.
inline bool strides_ok(const sala_strides& s, size_t esize) {
  if (s.b < 0 || s.t < 0 || s.h < 0) return false;
  return ((s.b * esize) % 16 == 0) && ((s.t * esize) % 16 == 0) && ((s.h * esize) % 16 == 0);
}

inline size_t esize_of(sala_dtype dt) { return dt == SALA_BF16 ? 2 : 4; }

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D 16-bit (bf16, or fp16 when `f16`) tensor map over a [B, T, H, D] activation
// with a (64, box_h, rows, 1) box and 128-byte swizzle (64 elements = 128 bytes
// per box row).
bool make_tmap_bhtd(CUtensorMap* map, const void* base, int B, int T, int H, int D,
                    const sala_strides& s, int box_rows, int box_h = 1, bool f16 = false) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)s.h * 2, (cuuint64_t)s.t * 2, (cuuint64_t)s.b * 2};
  // Degenerate extents get a harmless stride (never stepped over).
  if (H == 1 && strides[0] == 0) strides[0] = 16;
  if (B == 1 && strides[2] == 0) strides[2] = 16;
  cuuint32_t box[4] = {64, (cuuint32_t)box_h, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Per-segment statistics of v that the state pass writes, after the segment states.
void set_tc_stats(TcParams& p, void* stats_base) {
  uint8_t* base = static_cast<uint8_t*>(stats_base);
  p.vmax = reinterpret_cast<float*>(base);
  p.vssq = reinterpret_cast<float*>(base + lightning_tc_vmax_bytes(p.B, p.H, p.G));
}

// Heads whose v is outlier-heavy are recomputed in fp32 after a tensor-core prefill (or
// state-only pass, o == nullptr); all other heads' CTAs return at once.
bool launch_lightning_fixup(const void* q, const void* k, const void* v, const void* g, void* o,
                            float* state, const float* qw, const float* kw, sala_strides sq,
                            sala_strides sk, sala_strides sv, sala_strides sg, sala_strides so,
                            const TcParams& p, cudaStream_t st) {
  auto kern = lightning_cc_fixup_kernel<128>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)CCSmem<128>::bytes) != cudaSuccess)
    return false;
  kern<<<p.B * p.H, kCCThreads, CCSmem<128>::bytes, st>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
      (const __nv_bfloat16*)g, (__nv_bfloat16*)o, state, qw, kw, p.H, p.T, sq, sk, sv, sg, so,
      p.pos0, p.log2_base, p.eps, p.ws, p.G, p.vmax, p.vssq);
  return cudaPeekAtLastError() == cudaSuccess;
}

// dst = (accumulate ? dst : 0) + sum over i < count of src[i * stride + e], e < n.
__global__ void __launch_bounds__(256)
state_prefix_sum_kernel(const float* __restrict__ src, size_t n, int count, size_t stride,
                        float* __restrict__ dst, int accumulate) {
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    float acc = accumulate ? dst[e] : 0.0f;
    for (int i = 0; i < count; ++i) acc += src[(size_t)i * stride + e];
    dst[e] = acc;
  }
}

template <typename KernelT>
bool set_smem(KernelT* k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) ==
         cudaSuccess;
}

}  // namespace

namespace sala {

// Per-head softmax-normalised scores on tcgen05 for group size G (a power of two up to
// 32): one persistent CTA per SM over the rows [geo.r0, geo.r1) of a score pass.
template <int D, int G>
static bool launch_hsm_tc(cudaStream_t st, const __nv_bfloat16* q, sala_strides sq,
                          const CUtensorMap& th, const CUtensorMap& tm, const CUtensorMap& tl,
                          float* scores, HtGeom geo, int rows_pass) {
  auto kern = select_hsm_tc_kernel<D, G>;
  if (!set_smem(kern, HtSmem<D>::bytes)) return false;
  geo.R = kHtLanes / G;
  geo.nitems = (geo.r1 - geo.r0 + geo.R - 1) / geo.R * geo.hb;
  const int grid = std::max(1, std::min(geo.nitems, num_sms()));
  geo.nrounds = (geo.nitems + grid - 1) / grid;
  kern<<<grid, kHtThreads, HtSmem<D>::bytes, st>>>(q, sq, th, tm, tl, scores, geo, rows_pass);
  return true;
}
template <int D>
static bool launch_hsm_tc_g(int G, cudaStream_t st, const __nv_bfloat16* q, sala_strides sq,
                            const CUtensorMap& th, const CUtensorMap& tm, const CUtensorMap& tl,
                            float* scores, const HtGeom& geo, int rows_pass) {
  switch (G) {
    case 1: return launch_hsm_tc<D, 1>(st, q, sq, th, tm, tl, scores, geo, rows_pass);
    case 2: return launch_hsm_tc<D, 2>(st, q, sq, th, tm, tl, scores, geo, rows_pass);
    case 4: return launch_hsm_tc<D, 4>(st, q, sq, th, tm, tl, scores, geo, rows_pass);
    case 8: return launch_hsm_tc<D, 8>(st, q, sq, th, tm, tl, scores, geo, rows_pass);
    case 16: return launch_hsm_tc<D, 16>(st, q, sq, th, tm, tl, scores, geo, rows_pass);
    case 32: return launch_hsm_tc<D, 32>(st, q, sq, th, tm, tl, scores, geo, rows_pass);
    default: return false;
  }
}

}  // namespace sala

extern "C" {

const char* sala_status_string(sala_status s) {
  switch (s) {
    case SALA_OK: return "SALA_OK";
    case SALA_ERR_INVALID_ARG: return "SALA_ERR_INVALID_ARG";
    case SALA_ERR_UNSUPPORTED: return "SALA_ERR_UNSUPPORTED";
    case SALA_ERR_CUDA: return "SALA_ERR_CUDA";
    case SALA_ERR_TIMEOUT: return "SALA_ERR_TIMEOUT";
    case SALA_ERR_WORKSPACE: return "SALA_ERR_WORKSPACE";
    case SALA_ERR_RANGE: return "SALA_ERR_RANGE";
    case SALA_ERR_BOUNDS: return "SALA_ERR_BOUNDS";
  }
  return "SALA_ERR_UNKNOWN";
}

const char* sala_version(void) {
#ifdef SALA_DEBUG
  return "sala-b200 0.1 (sm_100a, SALA_DEBUG index checks)";
#else
  return "sala-b200 0.1 (sm_100a)";
#endif
}

// ------------------------------------------------------------------ Lightning prefill
size_t sala_lightning_prefill_workspace(int B, int T, int H, int D, int chunk, sala_dtype dt) {
  if (dt == SALA_BF16 && D == 128) return lightning_tc_workspace(B, T, H, chunk, num_sms());
  return 0;
}

sala_status sala_lightning_prefill(const void* q, const void* k, const void* v, const void* g,
                                   void* o, float* state, const float* q_norm_w,
                                   const float* k_norm_w, int B, int T, int H, int D,
                                   sala_strides sq, sala_strides sk, sala_strides sv,
                                   sala_strides sg, sala_strides so, int chunk, int64_t pos0,
                                   float rope_base, float eps, int init_zero, void* workspace,
                                   size_t workspace_bytes, sala_dtype dt, void* stream) {
  if (!state || (T > 0 && (!q || !k || !v || !o))) return SALA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || T < 0 || pos0 < 0 || !(rope_base > 1.0f) || !(eps >= 0.0f))
    return SALA_ERR_INVALID_ARG;
  if (dt != SALA_BF16 && dt != SALA_F32) return SALA_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return SALA_ERR_UNSUPPORTED;
  if (chunk != 64 && chunk != 128) return SALA_ERR_UNSUPPORTED;
  const size_t es = esize_of(dt);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state) ||
      (g && !aligned16(g)))
    return SALA_ERR_INVALID_ARG;
  if (!strides_ok(sq, es) || !strides_ok(sk, es) || !strides_ok(sv, es) || !strides_ok(so, es) ||
      (g && !strides_ok(sg, es)))
    return SALA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const double log2_base = std::log2((double)rope_base);
  if (T == 0) {
    if (init_zero && cudaMemsetAsync(state, 0, sizeof(float) * (size_t)B * H * D * D, st) !=
                         cudaSuccess)
      return SALA_ERR_CUDA;
    return SALA_OK;
  }
  if (dt == SALA_BF16 && D == 128 && chunk == kTcC) {
    const int nsm = num_sms();
    const size_t need = lightning_tc_workspace(B, T, H, chunk, nsm);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SALA_ERR_WORKSPACE;
    CUtensorMap tq, tk, tv;
    if (!make_tmap_bhtd(&tq, q, B, T, H, D, sq, kTcC) || !make_tmap_bhtd(&tk, k, B, T, H, D, sk, kTcC) ||
        !make_tmap_bhtd(&tv, v, B, T, H, D, sv, kTcC))
      return SALA_ERR_CUDA;
    TcParams p;
    p.g = (const __nv_bfloat16*)g;
    p.o = (__nv_bfloat16*)o;
    p.qw = q_norm_w;
    p.kw = k_norm_w;
    p.ws = (float*)workspace;
    p.sg = sg;
    p.so = so;
    p.B = B; p.T = T; p.H = H;
    p.G = lightning_tc_segments(B, H, T, nsm);
    set_tc_stats(p, (uint8_t*)workspace + lightning_tc_states_bytes(B, H, p.G));
    p.NC = (T + kTcC - 1) / kTcC;
    p.pos0 = pos0;
    p.log2_base = log2_base;
    p.eps = eps;
    const unsigned grid = (unsigned)(B * H * p.G);
    auto ka = lightning_state_kernel<false>;
    auto kc = lightning_out_kernel<false>;
    if (!set_smem(ka, TcSmem<true>::bytes) || !set_smem(kc, TcSmem<false>::bytes)) return SALA_ERR_CUDA;
    ka<<<grid, kStThreads, TcSmem<true>::bytes, st>>>(tk, tv, p);
    SALA_CHECK_LAUNCH();
    lightning_scan_kernel<<<dim3(B * H, 16), 256, 0, st>>>(p.ws, state, p.G, init_zero);
    SALA_CHECK_LAUNCH();
    kc<<<grid, kTcThreads, TcSmem<false>::bytes, st>>>(tq, tk, tv, p);
    SALA_CHECK_LAUNCH();
    if (!launch_lightning_fixup(q, k, v, g, o, state, q_norm_w, k_norm_w, sq, sk, sv, sg, so, p,
                                st))
      return SALA_ERR_CUDA;
    return SALA_OK;
  }
  const int grid = B * H;
  if (dt == SALA_F32) {
    if (D == 64) {
      auto kern = lightning_prefill_cc_kernel<float, 64>;
      if (!set_smem(kern, CCSmem<64>::bytes)) return SALA_ERR_CUDA;
      kern<<<grid, kCCThreads, CCSmem<64>::bytes, st>>>(
          (const float*)q, (const float*)k, (const float*)v, (const float*)g, (float*)o, state,
          q_norm_w, k_norm_w, H, T, sq, sk, sv, sg, so, pos0, log2_base, eps, init_zero);
    } else {
      auto kern = lightning_prefill_cc_kernel<float, 128>;
      if (!set_smem(kern, CCSmem<128>::bytes)) return SALA_ERR_CUDA;
      kern<<<grid, kCCThreads, CCSmem<128>::bytes, st>>>(
          (const float*)q, (const float*)k, (const float*)v, (const float*)g, (float*)o, state,
          q_norm_w, k_norm_w, H, T, sq, sk, sv, sg, so, pos0, log2_base, eps, init_zero);
    }
  } else if (D == 64) {
    auto kern = lightning_prefill_cc_kernel<__nv_bfloat16, 64>;
    if (!set_smem(kern, CCSmem<64>::bytes)) return SALA_ERR_CUDA;
    kern<<<grid, kCCThreads, CCSmem<64>::bytes, st>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
        (const __nv_bfloat16*)g, (__nv_bfloat16*)o, state, q_norm_w, k_norm_w, H, T, sq, sk, sv,
        sg, so, pos0, log2_base, eps, init_zero);
  } else {
    auto kern = lightning_prefill_cc_kernel<__nv_bfloat16, 128>;
    if (!set_smem(kern, CCSmem<128>::bytes)) return SALA_ERR_CUDA;
    kern<<<grid, kCCThreads, CCSmem<128>::bytes, st>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
        (const __nv_bfloat16*)g, (__nv_bfloat16*)o, state, q_norm_w, k_norm_w, H, T, sq, sk, sv,
        sg, so, pos0, log2_base, eps, init_zero);
  }
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

// Lightning prefill on prepared operands (the outputs of sala_lightning_projection):
// fp16 q and k already normalised and rotated, bf16 v, fp16 gate multiplier.
sala_status sala_lightning_prefill_prepared(const void* qh, const void* kh, const void* v,
                                            const void* gate, void* o, float* state, int B,
                                            int T, int H, int D, sala_strides sq,
                                            sala_strides sk, sala_strides sv, sala_strides sg,
                                            sala_strides so, int chunk, int init_zero,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream) {
  if (!state || (T > 0 && (!qh || !kh || !v || !o))) return SALA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || T < 0) return SALA_ERR_INVALID_ARG;
  if (D != 128 || chunk != kTcC) return SALA_ERR_UNSUPPORTED;
  if (!aligned16(qh) || !aligned16(kh) || !aligned16(v) || !aligned16(o) || !aligned16(state) ||
      (gate && !aligned16(gate)))
    return SALA_ERR_INVALID_ARG;
  if (!strides_ok(sq, 2) || !strides_ok(sk, 2) || !strides_ok(sv, 2) || !strides_ok(so, 2) ||
      (gate && !strides_ok(sg, 2)))
    return SALA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (T == 0) {
    if (init_zero && cudaMemsetAsync(state, 0, sizeof(float) * (size_t)B * H * D * D, st) !=
                         cudaSuccess)
      return SALA_ERR_CUDA;
    return SALA_OK;
  }
  const int nsm = num_sms();
  const size_t need = lightning_tc_workspace(B, T, H, chunk, nsm);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SALA_ERR_WORKSPACE;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bhtd(&tq, qh, B, T, H, D, sq, kTcC, 1, true) ||
      !make_tmap_bhtd(&tk, kh, B, T, H, D, sk, kTcC, 1, true) ||
      !make_tmap_bhtd(&tv, v, B, T, H, D, sv, kTcC))
    return SALA_ERR_CUDA;
  TcParams p{};
  p.g = (const __nv_bfloat16*)gate;
  p.o = (__nv_bfloat16*)o;
  p.ws = (float*)workspace;
  p.sg = sg;
  p.so = so;
  p.B = B; p.T = T; p.H = H;
  p.G = lightning_tc_segments(B, H, T, nsm);
  set_tc_stats(p, (uint8_t*)workspace + lightning_tc_states_bytes(B, H, p.G));
  p.NC = (T + kTcC - 1) / kTcC;
  p.pos0 = 0;
  p.log2_base = std::log2(10000.0);  // unused: the operands are already rotated
  p.eps = 0.f;
  const unsigned grid = (unsigned)(B * H * p.G);
  auto ka = lightning_state_kernel<true>;
  auto kc = lightning_out_kernel<true>;
  if (!set_smem(ka, TcSmem<true>::bytes) || !set_smem(kc, TcSmem<false>::bytes)) return SALA_ERR_CUDA;
  ka<<<grid, kStThreads, TcSmem<true>::bytes, st>>>(tk, tv, p);
  SALA_CHECK_LAUNCH();
  lightning_scan_kernel<<<dim3(B * H, 16), 256, 0, st>>>(p.ws, state, p.G, init_zero);
  SALA_CHECK_LAUNCH();
  kc<<<grid, kTcThreads, TcSmem<false>::bytes, st>>>(tq, tk, tv, p);
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

// ------------------------------------------------------------------ Lightning decode
sala_status sala_lightning_decode(const void* q, const void* k, const void* v, const void* g,
                                  void* o, float* state, const float* q_norm_w,
                                  const float* k_norm_w, const int32_t* pos, int B, int H, int D,
                                  sala_strides sq, sala_strides sk, sala_strides sv,
                                  sala_strides sg, sala_strides so, float rope_base, float eps,
                                  sala_dtype dt, void* stream) {
  if (!q || !k || !v || !o || !state || !pos) return SALA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || !(rope_base > 1.0f) || !(eps >= 0.0f)) return SALA_ERR_INVALID_ARG;
  if (dt != SALA_BF16 && dt != SALA_F32) return SALA_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return SALA_ERR_UNSUPPORTED;
  const size_t es = esize_of(dt);
  if (!aligned16(state) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (g && !aligned16(g)))
    return SALA_ERR_INVALID_ARG;
  sala_strides z[5] = {sq, sk, sv, sg, so};
  for (int i = 0; i < 5; ++i) {
    if (i == 3 && !g) continue;
    z[i].t = 0;
    if (!strides_ok(z[i], es)) return SALA_ERR_INVALID_ARG;
  }
  cudaStream_t st = as_stream(stream);
  const double l2b = std::log2((double)rope_base);
  const int grid = B * H;
#define SALA_DEC(TT, DD)                                                                    \
  lightning_decode_kernel<TT, DD><<<grid, kDecThreads, 0, st>>>(                            \
      (const TT*)q, (const TT*)k, (const TT*)v, (const TT*)g, (TT*)o, state, q_norm_w,      \
      k_norm_w, pos, H, sq, sk, sv, sg, so, l2b, eps)
  if (dt == SALA_BF16) {
    if (D == 128) SALA_DEC(__nv_bfloat16, 128); else SALA_DEC(__nv_bfloat16, 64);
  } else {
    if (D == 128) SALA_DEC(float, 128); else SALA_DEC(float, 64);
  }
#undef SALA_DEC
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

// ------------------------------------------------------------------ Lightning input projection
namespace {
// 2-D bf16 tensor map over `rows` rows of `cols` elements (row stride in elements) with a
// (64, box_rows) box and 128-byte swizzle.
bool make_tmap_2d(CUtensorMap* map, const void* base, int64_t rows, int cols, int64_t row_stride,
                  int box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_stride * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

sala_status sala_lightning_projection(const void* x, const void* w, const float* q_norm_w,
                                      const float* k_norm_w, void* qh, void* kh, void* v,
                                      void* gate, int B, int T, int hidden, int H, int D,
                                      int64_t x_row_stride, sala_strides sq, sala_strides sk,
                                      sala_strides sv, sala_strides sg, int64_t pos0,
                                      float rope_base, float eps, sala_dtype dt, void* stream) {
  if (B <= 0 || T < 0 || H <= 0 || hidden <= 0 || pos0 < 0 || !(rope_base > 1.0f) ||
      !(eps >= 0.0f))
    return SALA_ERR_INVALID_ARG;
  if (T > 0 && (!x || !w || !qh || !kh || !v || !gate)) return SALA_ERR_INVALID_ARG;
  if (dt != SALA_BF16) return SALA_ERR_UNSUPPORTED;
  if ((D != 64 && D != 128) || hidden % kPjBK != 0 || (H * D) % kPjBN != 0)
    return SALA_ERR_UNSUPPORTED;
  if (x_row_stride < hidden || (x_row_stride * 2) % 16 != 0) return SALA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(qh) || !aligned16(kh) || !aligned16(v) ||
      !aligned16(gate))
    return SALA_ERR_INVALID_ARG;
  if (!strides_ok(sq, 2) || !strides_ok(sk, 2) || !strides_ok(sv, 2) || !strides_ok(sg, 2))
    return SALA_ERR_INVALID_ARG;
  if (T == 0) return SALA_OK;
  const int64_t M = (int64_t)B * T;
  const int64_t N = 4 * (int64_t)H * D;
  if (M > (int64_t)INT32_MAX || N > (int64_t)INT32_MAX) return SALA_ERR_UNSUPPORTED;
  CUtensorMap tx, tw;
  if (!make_tmap_2d(&tx, x, M, hidden, x_row_stride, kPjBM) ||
      !make_tmap_2d(&tw, w, N, hidden, hidden, kPjBN))
    return SALA_ERR_CUDA;
  ProjParams p;
  p.qh = (__half*)qh;
  p.kh = (__half*)kh;
  p.v = (__nv_bfloat16*)v;
  p.gate = (__half*)gate;
  p.sq = sq; p.sk = sk; p.sv = sv; p.sg = sg;
  p.qw = q_norm_w;
  p.kw = k_norm_w;
  p.M = M;
  p.T = T; p.H = H; p.hidden = hidden;
  p.m_tiles = (int)((M + kPjBM - 1) / kPjBM);
  p.n_tiles = (int)(N / kPjBN);
  p.pos0 = pos0;
  p.log2_base = std::log2((double)rope_base);
  p.eps = eps;
  const int64_t ntiles = (int64_t)p.m_tiles * p.n_tiles;
  if (ntiles > (int64_t)INT32_MAX) return SALA_ERR_UNSUPPORTED;
  const unsigned grid = (unsigned)std::min<int64_t>(ntiles, num_sms());
  cudaStream_t st = as_stream(stream);
  if (D == 128) {
    auto kern = lightning_proj_kernel<128>;
    if (!set_smem(kern, kPjSmem)) return SALA_ERR_CUDA;
    kern<<<grid, kPjThreads, kPjSmem, st>>>(tx, tw, p);
  } else {
    auto kern = lightning_proj_kernel<64>;
    if (!set_smem(kern, kPjSmem)) return SALA_ERR_CUDA;
    kern<<<grid, kPjThreads, kPjSmem, st>>>(tx, tw, p);
  }
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

// ------------------------------------------------------------------ sequence-split Lightning
// A segment's state contribution (no outputs): the state pass and scan of the tensor-core
// path, or the CUDA-core kernel with its output half skipped.
sala_status sala_lightning_state(const void* k, const void* v, float* state, const float* k_norm_w,
                                 int B, int T, int H, int D, sala_strides sk, sala_strides sv,
                                 int chunk, int64_t pos0, float rope_base, float eps,
                                 int init_zero, void* workspace, size_t workspace_bytes,
                                 sala_dtype dt, void* stream) {
  if (!state || (T > 0 && (!k || !v))) return SALA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || T < 0 || pos0 < 0 || !(rope_base > 1.0f) || !(eps >= 0.0f))
    return SALA_ERR_INVALID_ARG;
  if (dt != SALA_BF16 && dt != SALA_F32) return SALA_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return SALA_ERR_UNSUPPORTED;
  if (chunk != 64 && chunk != 128) return SALA_ERR_UNSUPPORTED;
  const size_t es = esize_of(dt);
  if (!aligned16(k) || !aligned16(v) || !aligned16(state)) return SALA_ERR_INVALID_ARG;
  if (!strides_ok(sk, es) || !strides_ok(sv, es)) return SALA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const double log2_base = std::log2((double)rope_base);
  if (T == 0) {
    if (init_zero && cudaMemsetAsync(state, 0, sizeof(float) * (size_t)B * H * D * D, st) !=
                         cudaSuccess)
      return SALA_ERR_CUDA;
    return SALA_OK;
  }
  if (dt == SALA_BF16 && D == 128 && chunk == kTcC) {
    const int nsm = num_sms();
    const size_t need = lightning_tc_workspace(B, T, H, chunk, nsm);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return SALA_ERR_WORKSPACE;
    CUtensorMap tk, tv;
    if (!make_tmap_bhtd(&tk, k, B, T, H, D, sk, kTcC) || !make_tmap_bhtd(&tv, v, B, T, H, D, sv, kTcC))
      return SALA_ERR_CUDA;
    TcParams p{};
    p.kw = k_norm_w;
    p.ws = (float*)workspace;
    p.B = B; p.T = T; p.H = H;
    p.G = lightning_tc_segments(B, H, T, nsm);
    set_tc_stats(p, (uint8_t*)workspace + lightning_tc_states_bytes(B, H, p.G));
    p.NC = (T + kTcC - 1) / kTcC;
    p.pos0 = pos0;
    p.log2_base = log2_base;
    p.eps = eps;
    auto ka = lightning_state_kernel<false>;
    if (!set_smem(ka, TcSmem<true>::bytes)) return SALA_ERR_CUDA;
    ka<<<(unsigned)(B * H * p.G), kStThreads, TcSmem<true>::bytes, st>>>(tk, tv, p);
    SALA_CHECK_LAUNCH();
    lightning_scan_kernel<<<dim3(B * H, 16), 256, 0, st>>>(p.ws, state, p.G, init_zero);
    SALA_CHECK_LAUNCH();
    {
      const sala_strides none{0, 0, 0};
      if (!launch_lightning_fixup(k, k, v, nullptr, nullptr, state, nullptr, k_norm_w, sk, sk, sv,
                                  none, none, p, st))
        return SALA_ERR_CUDA;
    }
    return SALA_OK;
  }
  // CUDA-core kernel with o == nullptr: q is read but unused, so k stands in for it
  const sala_strides none{0, 0, 0};
  const int grid = B * H;
  if (dt == SALA_F32) {
    if (D == 64) {
      auto kern = lightning_prefill_cc_kernel<float, 64>;
      if (!set_smem(kern, CCSmem<64>::bytes)) return SALA_ERR_CUDA;
      kern<<<grid, kCCThreads, CCSmem<64>::bytes, st>>>(
          (const float*)k, (const float*)k, (const float*)v, nullptr, nullptr, state, nullptr,
          k_norm_w, H, T, sk, sk, sv, none, none, pos0, log2_base, eps, init_zero);
    } else {
      auto kern = lightning_prefill_cc_kernel<float, 128>;
      if (!set_smem(kern, CCSmem<128>::bytes)) return SALA_ERR_CUDA;
      kern<<<grid, kCCThreads, CCSmem<128>::bytes, st>>>(
          (const float*)k, (const float*)k, (const float*)v, nullptr, nullptr, state, nullptr,
          k_norm_w, H, T, sk, sk, sv, none, none, pos0, log2_base, eps, init_zero);
    }
  } else if (D == 64) {
    auto kern = lightning_prefill_cc_kernel<__nv_bfloat16, 64>;
    if (!set_smem(kern, CCSmem<64>::bytes)) return SALA_ERR_CUDA;
    kern<<<grid, kCCThreads, CCSmem<64>::bytes, st>>>(
        (const __nv_bfloat16*)k, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, nullptr,
        nullptr, state, nullptr, k_norm_w, H, T, sk, sk, sv, none, none, pos0, log2_base, eps,
        init_zero);
  } else {
    auto kern = lightning_prefill_cc_kernel<__nv_bfloat16, 128>;
    if (!set_smem(kern, CCSmem<128>::bytes)) return SALA_ERR_CUDA;
    kern<<<grid, kCCThreads, CCSmem<128>::bytes, st>>>(
        (const __nv_bfloat16*)k, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, nullptr,
        nullptr, state, nullptr, k_norm_w, H, T, sk, sk, sv, none, none, pos0, log2_base, eps,
        init_zero);
  }
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

sala_status sala_state_prefix_sum(const float* src, size_t n, int count, size_t stride,
                                  float* dst, int accumulate, void* stream) {
  if (!dst || (count > 0 && !src) || count < 0 || (count > 1 && stride < n))
    return SALA_ERR_INVALID_ARG;
  if (n == 0 || (count == 0 && accumulate)) return SALA_OK;  // nothing to add
  const int64_t want = 4 * (int64_t)num_sms();
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, ((int64_t)n + 255) / 256));
  state_prefix_sum_kernel<<<grid, 256, 0, as_stream(stream)>>>(src, n, count, stride, dst,
                                                               accumulate);
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

// ------------------------------------------------------------------ sparse selection
// The fused path (select_tc_kernel) scores and selects in one persistent kernel: topk <=
// kSelFusedMaxK and block indices that fit 16 bits.  Otherwise scores go through a
// bounded scratch.
static bool sel_fused(int T, int topk) { return topk <= kSelFusedMaxK && T / kSelBlk <= 65535; }

size_t sala_sparse_select_rows_workspace(int B, int Tq, int Tk, int Hq, int Hkv, int D,
                                         int block, int topk, int score) {
  (void)Hq;
  if (B <= 0 || Tq <= 0 || Tk <= 0 || Hkv <= 0 || block != kSelBlk || (D != 64 && D != 128) ||
      topk < 1 || (score != 0 && score != 1))
    return 0;
  const SelLayout L = sel_layout(B, Tq, Tk, Hkv, D);
  return score == 0 && sel_fused(Tk, topk) ? L.total_fused : L.total;
}

size_t sala_sparse_select_workspace(int B, int T, int Hq, int Hkv, int D, int block, int topk) {
  return sala_sparse_select_rows_workspace(B, T, T, Hq, Hkv, D, block, topk, 0);
}

size_t sala_sparse_select_head_softmax_workspace(int B, int T, int Hq, int Hkv, int D,
                                                 int block) {
  (void)Hq;
  if (B <= 0 || T <= 0 || Hkv <= 0 || D <= 0 || block != kSelBlk) return 0;
  return sel_layout(B, T, T, Hkv, D).total;
}

// mode 0: group-summed scores (fused tensor-core path for topk <= 64, else the score
// scratch); mode 1: per-head softmax-normalised scores (score scratch).  The T query rows
// are positions qpos0 .. qpos0 + T - 1 of a sequence whose keys cover 0 .. Tk - 1.
static sala_status sparse_select_impl(const void* q, const void* k, int B, int T, int qpos0,
                                      int Tk, int Hq, int Hkv, int D, sala_strides sq,
                                      sala_strides sk, int block, int topk, int n_init,
                                      int n_local, int32_t* idx, void* ws, size_t ws_bytes,
                                      sala_dtype dt, void* stream, int mode) {
  if (T > 0 && (!q || !k || !idx)) return SALA_ERR_INVALID_ARG;
  if (B <= 0 || T < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return SALA_ERR_INVALID_ARG;
  if (qpos0 < 0 || Tk < 0 || (int64_t)qpos0 + T > (int64_t)Tk) return SALA_ERR_INVALID_ARG;
  if (topk < 1 || n_init < 0 || n_local < 1) return SALA_ERR_INVALID_ARG;
  if (dt != SALA_BF16) return SALA_ERR_UNSUPPORTED;
  if (block != kSelBlk || (D != 64 && D != 128) || topk > 256 || Hq / Hkv > 32)
    return SALA_ERR_UNSUPPORTED;
  if (mode == 1 && ((Hq / Hkv) & (Hq / Hkv - 1)) != 0) return SALA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !strides_ok(sq, 2) || !strides_ok(sk, 2))
    return SALA_ERR_INVALID_ARG;
  if (T == 0) return SALA_OK;
  const SelLayout L = sel_layout(B, T, Tk, Hkv, D);
  const bool fused = mode == 0 && sel_fused(Tk, topk);
  if (!ws || ws_bytes < (fused ? L.total_fused : L.total)) return SALA_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* kbar = reinterpret_cast<float*>(wsb + L.kbar_off);
  __nv_bfloat16* khi = reinterpret_cast<__nv_bfloat16*>(wsb + L.khi_off);
  __nv_bfloat16* klo = reinterpret_cast<__nv_bfloat16*>(wsb + L.klo_off);
  // the third part of the means: per-head softmax scores only (workspace `total`)
  __nv_bfloat16* klo2 = mode == 1 ? reinterpret_cast<__nv_bfloat16*>(wsb + L.klo2_off) : nullptr;
  float* scores = reinterpret_cast<float*>(wsb + L.score_off);
  const int G = Hq / Hkv;
  const float inv_sqrt_d = 1.0f / std::sqrt((float)D);
  // per-head softmax: the bf16 parts carry the means times log2(e) / sqrt(D), so the
  // MMAs give the scores in the log2 domain of the exponentials
  const float part_scale = mode == 1 ? inv_sqrt_d * 1.4426950408889634f : 1.0f;
  if (L.nb > 0) {
    dim3 gm(L.nb, Hkv, B);
    if (D == 128)
      block_means_kernel<128><<<gm, 128, 0, st>>>((const __nv_bfloat16*)k, kbar, khi, klo, klo2,
                                                   part_scale, L.nb, Hkv, sk);
    else
      block_means_kernel<64><<<gm, 64, 0, st>>>((const __nv_bfloat16*)k, kbar, khi, klo, klo2,
                                                 part_scale, L.nb, Hkv, sk);
    SALA_CHECK_LAUNCH();
  }
  CUtensorMap hh, hm, hl;  // per-head softmax path: the means' three bf16 parts
  if (mode == 1 && L.nb > 0) {
    const sala_strides skb{(int64_t)L.nb * Hkv * D, (int64_t)Hkv * D, (int64_t)D};
    if (!make_tmap_bhtd(&hh, khi, B, L.nb, Hkv, D, skb, kHtN) ||
        !make_tmap_bhtd(&hm, klo, B, L.nb, Hkv, D, skb, kHtN) ||
        !make_tmap_bhtd(&hl, klo2, B, L.nb, Hkv, D, skb, kHtN))
      return SALA_ERR_CUDA;
  }
  if (fused) {
    // block means (bf16 hi / lo) as a [B, nb, Hkv, D] tensor, 32-candidate boxes
    const int nbm = L.nb > 0 ? L.nb : 1;
    const sala_strides skb{(int64_t)nbm * Hkv * D, (int64_t)Hkv * D, (int64_t)D};
    CUtensorMap th, tl;
    if (!make_tmap_bhtd(&th, khi, B, nbm, Hkv, D, skb, kStcN) ||
        !make_tmap_bhtd(&tl, klo, B, nbm, Hkv, D, skb, kStcN))
      return SALA_ERR_CUDA;
    const int nitems = (T + kStcRows - 1) / kStcRows * Hkv * B;
    const int grid = std::min(nitems, num_sms());
    if (D == 128) {
      auto kern = select_tc_kernel<128>;
      if (!set_smem(kern, StcSmem<128>::bytes)) return SALA_ERR_CUDA;
      kern<<<grid, kStcThreads, StcSmem<128>::bytes, st>>>(th, tl, (const __nv_bfloat16*)q, idx,
                                                          T, qpos0, L.nb, Hkv, B, G, sq, topk,
                                                          n_init, n_local);
    } else {
      auto kern = select_tc_kernel<64>;
      if (!set_smem(kern, StcSmem<64>::bytes)) return SALA_ERR_CUDA;
      kern<<<grid, kStcThreads, StcSmem<64>::bytes, st>>>(th, tl, (const __nv_bfloat16*)q, idx,
                                                         T, qpos0, L.nb, Hkv, B, G, sq, topk,
                                                         n_init, n_local);
    }
    SALA_CHECK_LAUNCH();
    return SALA_OK;
  }
  for (int r0 = 0; r0 < T; r0 += L.rows_pass) {
    const int r1 = std::min(T, r0 + L.rows_pass);
    if (L.nb > 0 && mode == 1) {
      HtGeom geo{};
      geo.r0 = r0;
      geo.r1 = r1;
      geo.Tq = T;
      geo.qpos0 = qpos0;
      geo.nb = L.nb;
      geo.Hkv = Hkv;
      geo.hb = Hkv * B;
      geo.n_init = n_init;
      geo.n_local = n_local;
      const __nv_bfloat16* qb = (const __nv_bfloat16*)q;
      const bool ok = D == 128 ? launch_hsm_tc_g<128>(G, st, qb, sq, hh, hm, hl, scores, geo,
                                                      L.rows_pass)
                               : launch_hsm_tc_g<64>(G, st, qb, sq, hh, hm, hl, scores, geo,
                                                     L.rows_pass);
      if (!ok) return SALA_ERR_CUDA;
      SALA_CHECK_LAUNCH();
    } else if (L.nb > 0) {
      dim3 gs((r1 - r0 + kScTile - 1) / kScTile, Hkv, B);
      if (D == 128) {
        auto kern = block_scores_kernel<128>;
        if (!set_smem(kern, score_smem_bytes<128>())) return SALA_ERR_CUDA;
        kern<<<gs, 256, score_smem_bytes<128>(), st>>>((const __nv_bfloat16*)q, kbar, scores,
                                                        L.nb, Hkv, G, sq, qpos0, r0, r1,
                                                        L.rows_pass, n_init, n_local, inv_sqrt_d);
      } else {
        auto kern = block_scores_kernel<64>;
        if (!set_smem(kern, score_smem_bytes<64>())) return SALA_ERR_CUDA;
        kern<<<gs, 256, score_smem_bytes<64>(), st>>>((const __nv_bfloat16*)q, kbar, scores,
                                                       L.nb, Hkv, G, sq, qpos0, r0, r1,
                                                       L.rows_pass, n_init, n_local, inv_sqrt_d);
      }
      SALA_CHECK_LAUNCH();
    }
    const int64_t nwarps = (int64_t)B * Hkv * (r1 - r0);
    const int64_t nblk = (nwarps + kTopkWarps - 1) / kTopkWarps;
    topk_select_kernel<<<(unsigned)nblk, kTopkWarps * 32, 0, st>>>(
        scores, idx, B, T, qpos0, Hkv, L.nb > 0 ? L.nb : 1, r0, r1, L.rows_pass, topk, n_init,
        n_local);
    SALA_CHECK_LAUNCH();
  }
  return SALA_OK;
}

sala_status sala_sparse_select(const void* q, const void* k, int B, int T, int Hq, int Hkv,
                               int D, sala_strides sq, sala_strides sk, int block, int topk,
                               int n_init, int n_local, int32_t* idx, void* ws, size_t ws_bytes,
                               sala_dtype dt, void* stream) {
  return sparse_select_impl(q, k, B, T, 0, T, Hq, Hkv, D, sq, sk, block, topk, n_init, n_local,
                            idx, ws, ws_bytes, dt, stream, 0);
}

sala_status sala_sparse_select_head_softmax(const void* q, const void* k, int B, int T, int Hq,
                                            int Hkv, int D, sala_strides sq, sala_strides sk,
                                            int block, int topk, int n_init, int n_local,
                                            int32_t* idx, void* ws, size_t ws_bytes,
                                            sala_dtype dt, void* stream) {
  return sparse_select_impl(q, k, B, T, 0, T, Hq, Hkv, D, sq, sk, block, topk, n_init, n_local,
                            idx, ws, ws_bytes, dt, stream, 1);
}

sala_status sala_sparse_select_rows(const void* q, const void* k, int B, int Tq, int qpos0,
                                    int Tk, int Hq, int Hkv, int D, sala_strides sq,
                                    sala_strides sk, int block, int topk, int n_init,
                                    int n_local, int score, int32_t* idx, void* ws,
                                    size_t ws_bytes, sala_dtype dt, void* stream) {
  if (score != 0 && score != 1) return SALA_ERR_INVALID_ARG;
  return sparse_select_impl(q, k, B, Tq, qpos0, Tk, Hq, Hkv, D, sq, sk, block, topk, n_init,
                            n_local, idx, ws, ws_bytes, dt, stream, score);
}

// ------------------------------------------------------------------ sparse attention
// Workspace: the fp16 copy of v [B, T, Hkv, D], the per-chunk largest |v| and sum-of-
// squares partials [B * Hkv][kVChunks] each, the exponents and the outlier flags
// [B * Hkv] each, every part 256-byte aligned.
namespace {
struct SaLayout {
  size_t part_off, part_ss_off, vexp_off, vflag_off, total;
};
SaLayout sa_layout(int B, int T, int Hkv, int D) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  SaLayout L{};
  L.part_off = up((size_t)B * T * Hkv * D * 2);
  L.part_ss_off = L.part_off + up((size_t)B * Hkv * kVChunks * sizeof(float));
  L.vexp_off = L.part_ss_off + up((size_t)B * Hkv * kVChunks * sizeof(float));
  L.vflag_off = L.vexp_off + up((size_t)B * Hkv * sizeof(int));
  L.total = L.vflag_off + up((size_t)B * Hkv * sizeof(int));
  return L;
}
}  // namespace

size_t sala_sparse_attn_workspace(int B, int T, int Hkv, int D) {
  if (B <= 0 || T <= 0 || Hkv <= 0 || D <= 0) return 0;
  return sa_layout(B, T, Hkv, D).total;
}

// The T query rows (q, g, o, idx) are positions qpos0 .. qpos0 + T - 1; k and v hold
// positions 0 .. Tk - 1.
static sala_status sparse_attn_impl(const void* q, const void* k, const void* v, const void* g,
                                    const int32_t* idx, int n_sel, void* o, int B, int T,
                                    int qpos0, int Tk, int Hq, int Hkv, int D, sala_strides sq,
                                    sala_strides sk, sala_strides sv, sala_strides sg,
                                    sala_strides so, int block, float scale, void* ws,
                                    size_t ws_bytes, sala_dtype dt, void* stream) {
  if (T > 0 && (!q || !k || !v || !o || !idx)) return SALA_ERR_INVALID_ARG;
  if (B <= 0 || T < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || n_sel <= 0 || !(scale >= 0.0f))
    return SALA_ERR_INVALID_ARG;
  if (qpos0 < 0 || Tk < 0 || (int64_t)qpos0 + T > (int64_t)Tk) return SALA_ERR_INVALID_ARG;
  if (dt != SALA_BF16) return SALA_ERR_UNSUPPORTED;
  if (block != kSaBlk || (D != 64 && D != 128) || Hq / Hkv > 16) return SALA_ERR_UNSUPPORTED;
  if (Hkv > 65535 || B > 65535) return SALA_ERR_UNSUPPORTED;  // grid y / z of the v pre-pass
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (g && !aligned16(g)))
    return SALA_ERR_INVALID_ARG;
  if (!strides_ok(sq, 2) || !strides_ok(sk, 2) || !strides_ok(sv, 2) || !strides_ok(so, 2) ||
      (g && !strides_ok(sg, 2)))
    return SALA_ERR_INVALID_ARG;
  if (T == 0) return SALA_OK;
  if (!ws || !aligned16(ws) || ws_bytes < sala_sparse_attn_workspace(B, Tk, Hkv, D))
    return SALA_ERR_WORKSPACE;
  // the fp16 copy of v: contiguous [B, Tk, Hkv, D]
  const sala_strides sv16 = {(int64_t)Tk * Hkv * D, (int64_t)Hkv * D, (int64_t)D};
  CUtensorMap tk, tv;
  if (!make_tmap_bhtd(&tk, k, B, Tk, Hkv, D, sk, kSaBlk) ||
      !make_tmap_bhtd(&tv, ws, B, Tk, Hkv, D, sv16, kSaBlk, 1, true))
    return SALA_ERR_CUDA;
  SaParams p;
  p.q = (const __nv_bfloat16*)q;
  p.g = (const __nv_bfloat16*)g;
  p.o = (__nv_bfloat16*)o;
  p.idx = idx;
  const SaLayout L = sa_layout(B, Tk, Hkv, D);
  float* vpart = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.part_off);
  float* vpart_ss = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.part_ss_off);
  int* vexp = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.vexp_off);
  int* vflag = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + L.vflag_off);
  p.vexp = vexp;
  p.vflag = vflag;
  p.sq = sq; p.sg = sg; p.so = so;
  p.n_sel = n_sel; p.B = B; p.T = T; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
  const float sc = scale > 0.0f ? scale : 1.0f / std::sqrt((float)D);
  p.scale_log2 = sc * 1.4426950408889634f;
  p.rows = (int64_t)B * Hkv * T;
  p.qpos0 = qpos0;
  p.nkb = (Tk + kSaBlk - 1) / kSaBlk;
  cudaStream_t st = as_stream(stream);
  const int64_t want = num_sms();
  const unsigned grid = (unsigned)std::min<int64_t>(want, p.rows);
  {
    // fp16 copy of v for the P.V MMAs, scaled by 2^-e per (sequence, KV head) so that
    // every bf16 value keeps its significant bits; a non-finite v raises SALA_ERR_RANGE
    const dim3 gv(kVChunks, Hkv, B);
    v_absmax_kernel<<<gv, 256, 0, st>>>((const __nv_bfloat16*)v, sv, Tk, Hkv, D, vpart,
                                        vpart_ss);
    SALA_CHECK_LAUNCH();
    to_f16_copy_kernel<<<gv, 256, 0, st>>>((const __nv_bfloat16*)v, sv, Tk, Hkv, D, vpart,
                                           vpart_ss, vexp, vflag, (__half*)ws);
    SALA_CHECK_LAUNCH();
  }
  // the common variant, then the one for outlier-heavy heads (which returns at once
  // when there are none)
  if (D == 128) {
    constexpr int NS = 3;
    auto k0 = sparse_attn_kernel<128, NS, false>;
    auto k1 = sparse_attn_kernel<128, NS, true>;
    if (!set_smem(k0, SaSmem<128, NS>::bytes) || !set_smem(k1, SaSmem<128, NS>::bytes))
      return SALA_ERR_CUDA;
    k0<<<grid, kSaThreads, SaSmem<128, NS>::bytes, st>>>(tk, tv, p);
    SALA_CHECK_LAUNCH();
    k1<<<grid, kSaThreads, SaSmem<128, NS>::bytes, st>>>(tk, tv, p);
  } else {
    constexpr int NS = 6;
    auto k0 = sparse_attn_kernel<64, NS, false>;
    auto k1 = sparse_attn_kernel<64, NS, true>;
    if (!set_smem(k0, SaSmem<64, NS>::bytes) || !set_smem(k1, SaSmem<64, NS>::bytes))
      return SALA_ERR_CUDA;
    k0<<<grid, kSaThreads, SaSmem<64, NS>::bytes, st>>>(tk, tv, p);
    SALA_CHECK_LAUNCH();
    k1<<<grid, kSaThreads, SaSmem<64, NS>::bytes, st>>>(tk, tv, p);
  }
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

sala_status sala_sparse_attn(const void* q, const void* k, const void* v, const void* g,
                             const int32_t* idx, int n_sel, void* o, int B, int T, int Hq,
                             int Hkv, int D, sala_strides sq, sala_strides sk, sala_strides sv,
                             sala_strides sg, sala_strides so, int block, float scale,
                             void* ws, size_t ws_bytes, sala_dtype dt, void* stream) {
  return sparse_attn_impl(q, k, v, g, idx, n_sel, o, B, T, 0, T, Hq, Hkv, D, sq, sk, sv, sg, so,
                          block, scale, ws, ws_bytes, dt, stream);
}

sala_status sala_sparse_attn_rows(const void* q, const void* k, const void* v, const void* g,
                                  const int32_t* idx, int n_sel, void* o, int B, int Tq,
                                  int qpos0, int Tk, int Hq, int Hkv, int D, sala_strides sq,
                                  sala_strides sk, sala_strides sv, sala_strides sg,
                                  sala_strides so, int block, float scale, void* ws,
                                  size_t ws_bytes, sala_dtype dt, void* stream) {
  return sparse_attn_impl(q, k, v, g, idx, n_sel, o, B, Tq, qpos0, Tk, Hq, Hkv, D, sq, sk, sv,
                          sg, so, block, scale, ws, ws_bytes, dt, stream);
}

// ------------------------------------------------------------------ sparse-layer decode
namespace {
// Resident CTAs per SM of sd_attn_kernel<D> after its shared-memory opt-in, per device
// (the opt-in is a per-device function attribute); 0 on failure.
int sd_attn_occupancy(int D) {
  constexpr int kDev = 64;
  static std::mutex mu;
  static int cache[2][kDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDev) return 0;
  const int w = D == 128 ? 1 : 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[w][dev] == 0) {
    int occ = 0;
    bool ok;
    if (D == 128)
      ok = set_smem(sd_attn_kernel<128>, SdAttnSmem<128>::bytes) &&
           cudaOccupancyMaxActiveBlocksPerMultiprocessor(
               &occ, sd_attn_kernel<128>, kSdAttnWarps * 32, SdAttnSmem<128>::bytes) == cudaSuccess;
    else
      ok = set_smem(sd_attn_kernel<64>, SdAttnSmem<64>::bytes) &&
           cudaOccupancyMaxActiveBlocksPerMultiprocessor(
               &occ, sd_attn_kernel<64>, kSdAttnWarps * 32, SdAttnSmem<64>::bytes) == cudaSuccess;
    if (!ok || occ < 1) return 0;
    cache[w][dev] = occ;
  }
  return cache[w][dev];
}

struct SdLayout {
  size_t scores_off, idx_off, part_off, total;
};
SdLayout sd_layout(int B, int Tmax, int Hkv, int D, int n_sel) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t nbcap = (size_t)(Tmax / kSdBlk);
  SdLayout L{};
  L.scores_off = 0;
  L.idx_off = up((size_t)B * Hkv * nbcap * 4);
  L.part_off = L.idx_off + up((size_t)B * Hkv * n_sel * 4);
  L.total = L.part_off + up((size_t)B * Hkv * kSdMaxSplit * 16 * (D + 2) * 4);
  return L;
}
}  // namespace

size_t sala_sparse_decode_workspace(int B, int Tmax, int Hq, int Hkv, int D, int n_sel) {
  (void)Hq;
  if (B <= 0 || Tmax < kSdBlk || Tmax % kSdBlk != 0 || Hkv <= 0 || n_sel <= 0 ||
      (D != 64 && D != 128))
    return 0;
  return sd_layout(B, Tmax, Hkv, D, n_sel).total;
}

sala_status sala_sparse_decode(const void* q, const void* k_cache, const void* v_cache,
                               const void* g, float* kbar, const int32_t* pos, void* o,
                               int32_t* idx_out, int B, int Tmax, int Hq, int Hkv, int D,
                               sala_strides sq, sala_strides sk, sala_strides sv, sala_strides sg,
                               sala_strides so, int block, int topk, int n_init, int n_local,
                               float scale, void* ws, size_t ws_bytes, sala_dtype dt,
                               void* stream) {
  if (!q || !k_cache || !v_cache || !kbar || !pos || !o) return SALA_ERR_INVALID_ARG;
  if (B <= 0 || Tmax < kSdBlk || Tmax % kSdBlk != 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 ||
      topk < 1 || n_init < 0 || n_local < 1 || !(scale >= 0.0f))
    return SALA_ERR_INVALID_ARG;
  if (dt != SALA_BF16) return SALA_ERR_UNSUPPORTED;
  if (block != kSdBlk || (D != 64 && D != 128) || Hq / Hkv > 16) return SALA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      !aligned16(kbar) || (g && !aligned16(g)) ||
      (idx_out && (reinterpret_cast<uintptr_t>(idx_out) & 3u)))
    return SALA_ERR_INVALID_ARG;
  if (!strides_ok(sq, 2) || !strides_ok(sk, 2) || !strides_ok(sv, 2) || !strides_ok(so, 2) ||
      (g && !strides_ok(sg, 2)))
    return SALA_ERR_INVALID_ARG;
  const int n_sel = n_init + topk + n_local;
  const SdLayout L = sd_layout(B, Tmax, Hkv, D, n_sel);
  if (!ws || !aligned16(ws) || ws_bytes < L.total) return SALA_ERR_WORKSPACE;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  SdParams p;
  p.q = (const __nv_bfloat16*)q;
  p.g = (const __nv_bfloat16*)g;
  p.o = (__nv_bfloat16*)o;
  p.k = (const __nv_bfloat16*)k_cache;
  p.v = (const __nv_bfloat16*)v_cache;
  p.kbar = kbar;
  p.pos = pos;
  p.idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(wsb + L.idx_off);
  p.scores = reinterpret_cast<float*>(wsb + L.scores_off);
  p.part = reinterpret_cast<float*>(wsb + L.part_off);
  p.sq = sq; p.sg = sg; p.so = so; p.sk = sk; p.sv = sv;
  p.B = B; p.Tmax = Tmax; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv; p.D = D;
  p.nbcap = Tmax / kSdBlk;
  p.n_init = n_init; p.topk = topk; p.n_local = n_local; p.n_sel = n_sel;
  const int rows = B * Hkv, nsm = num_sms();
  // attention splits: fill the resident CTA slots once (cp.async tiles take 64 KB per CTA
  // at D = 128); score chunks: the score grid covers the SMs twice.  The shared-memory
  // opt-in and the occupancy are looked up once per device and kernel.
  int occ = sd_attn_occupancy(D);
  if (occ < 1) return SALA_ERR_CUDA;
  const int slots = std::max(1, occ) * nsm;
  p.nsplit = std::max(1, std::min({(slots + rows / 2) / rows, kSdMaxSplit, n_sel}));
  {
    const int64_t want = ((int64_t)p.nbcap * rows + 2 * nsm - 1) / (2 * nsm);
    p.chunk = (int)std::max<int64_t>(64, std::min<int64_t>(kSdScoreChunk, (want + 31) / 32 * 32));
  }
  const float sc = scale > 0.0f ? scale : 1.0f / std::sqrt((float)D);
  p.scale_log2 = sc * 1.4426950408889634f;
  cudaStream_t st = as_stream(stream);
  const dim3 gs((p.nbcap + p.chunk - 1) / p.chunk, Hkv, B);
  const dim3 ga(p.nsplit, Hkv, B);
  if (D == 128) {
    sd_score_kernel<128><<<gs, 256, 0, st>>>(p);
  } else {
    sd_score_kernel<64><<<gs, 256, 0, st>>>(p);
  }
  SALA_CHECK_LAUNCH();
  sd_topk_kernel<<<dim3(Hkv, B), kSdTopkThreads, 0, st>>>(p);
  SALA_CHECK_LAUNCH();
  if (D == 128) {
    sd_attn_kernel<128><<<ga, kSdAttnWarps * 32, SdAttnSmem<128>::bytes, st>>>(p);
    SALA_CHECK_LAUNCH();
    sd_combine_kernel<128><<<dim3(Hq, B), 128, 0, st>>>(p);
  } else {
    sd_attn_kernel<64><<<ga, kSdAttnWarps * 32, SdAttnSmem<64>::bytes, st>>>(p);
    SALA_CHECK_LAUNCH();
    sd_combine_kernel<64><<<dim3(Hq, B), 64, 0, st>>>(p);
  }
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

sala_status sala_sparse_block_means(const void* k, int B, int T, int Hkv, int D, sala_strides sk,
                                    float* kbar, int kbar_blocks, sala_dtype dt, void* stream) {
  if (T > 0 && (!k || !kbar)) return SALA_ERR_INVALID_ARG;
  if (B <= 0 || T < 0 || Hkv <= 0 || kbar_blocks < T / kSdBlk) return SALA_ERR_INVALID_ARG;
  if (dt != SALA_BF16) return SALA_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return SALA_ERR_UNSUPPORTED;
  if (T / kSdBlk == 0) return SALA_OK;
  if (!aligned16(k) || !aligned16(kbar) || !strides_ok(sk, 2)) return SALA_ERR_INVALID_ARG;
  const dim3 grid(T / kSdBlk, Hkv, B);
  cudaStream_t st = as_stream(stream);
  if (D == 128)
    sd_block_means_kernel<128><<<grid, 128, 0, st>>>((const __nv_bfloat16*)k, sk, kbar_blocks,
                                                      Hkv, kbar);
  else
    sd_block_means_kernel<64><<<grid, 64, 0, st>>>((const __nv_bfloat16*)k, sk, kbar_blocks, Hkv,
                                                    kbar);
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

// ------------------------------------------------------------------ no-allocation prefill
}  // extern "C"

namespace {

// Fixed scratch for sala_lightning_prefill_noalloc: room for 256 fp32 128x128
// segment states (16 MiB) followed by their 256 largest-|v| words (one 256-byte
// line is enough; 64 KiB are reserved).  Host code may not use the symbol itself as a
// device address; the per-device address comes from cudaGetSymbolAddress below.
constexpr size_t kNoAllocStateBytes = size_t(16) << 20;
constexpr size_t kNoAllocScratchBytes = kNoAllocStateBytes + (size_t(64) << 10);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[256] = {};

// Device address of the scratch array for the current device (looked up once).
void* noalloc_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    g_noalloc_addr[dev] = ptr;
  }
  return g_noalloc_addr[dev];
}

}  // namespace

extern "C" {

sala_status sala_lightning_prefill_noalloc(const void* q, const void* k, const void* v,
                                           const void* g, void* o, float* state,
                                           const float* q_norm_w, const float* k_norm_w, int B,
                                           int T, int H, int D, sala_strides sq,
                                           sala_strides sk, sala_strides sv, sala_strides sg,
                                           sala_strides so, int chunk, int64_t pos0,
                                           float rope_base, float eps, int init_zero,
                                           sala_dtype dt, void* stream) {
  const bool tc_path = dt == SALA_BF16 && D == 128 && chunk == kTcC;
  if (!tc_path || T <= 0)  // these paths use no scratch at all
    return sala_lightning_prefill(q, k, v, g, o, state, q_norm_w, k_norm_w, B, T, H, D, sq, sk,
                                  sv, sg, so, chunk, pos0, rope_base, eps, init_zero, nullptr, 0,
                                  dt, stream);
  if (!state || !q || !k || !v || !o) return SALA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || pos0 < 0 || !(rope_base > 1.0f) || !(eps >= 0.0f))
    return SALA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state) ||
      (g && !aligned16(g)))
    return SALA_ERR_INVALID_ARG;
  if (!strides_ok(sq, 2) || !strides_ok(sk, 2) || !strides_ok(sv, 2) || !strides_ok(so, 2) ||
      (g && !strides_ok(sg, 2)))
    return SALA_ERR_INVALID_ARG;
  constexpr int64_t kStateBytes = 128 * 128 * sizeof(float);
  const int64_t capacity = (int64_t)(kNoAllocStateBytes / kStateBytes);  // segment states
  if ((int64_t)B * H > capacity) return SALA_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_address();
  if (!scratch) return SALA_ERR_CUDA;
  cudaStream_t st = as_stream(stream);
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bhtd(&tq, q, B, T, H, D, sq, kTcC) || !make_tmap_bhtd(&tk, k, B, T, H, D, sk, kTcC) ||
      !make_tmap_bhtd(&tv, v, B, T, H, D, sv, kTcC))
    return SALA_ERR_CUDA;
  TcParams p;
  p.g = (const __nv_bfloat16*)g;
  p.o = (__nv_bfloat16*)o;
  p.qw = q_norm_w;
  p.kw = k_norm_w;
  p.ws = (float*)scratch;
  p.sg = sg;
  p.so = so;
  p.B = B; p.T = T; p.H = H;
  p.NC = (T + kTcC - 1) / kTcC;
  int G = lightning_tc_segments(B, H, T, num_sms());
  const int g_cap = (int)(capacity / ((int64_t)B * H));
  if (G > g_cap) G = g_cap;
  p.G = G;
  set_tc_stats(p, (uint8_t*)scratch + kNoAllocStateBytes);
  p.pos0 = pos0;
  p.log2_base = std::log2((double)rope_base);
  p.eps = eps;
  const unsigned grid = (unsigned)(B * H * p.G);
  auto ka = lightning_state_kernel<false>;
  auto kc = lightning_out_kernel<false>;
  if (!set_smem(ka, TcSmem<true>::bytes) || !set_smem(kc, TcSmem<false>::bytes)) return SALA_ERR_CUDA;
  ka<<<grid, kStThreads, TcSmem<true>::bytes, st>>>(tk, tv, p);
  SALA_CHECK_LAUNCH();
  lightning_scan_kernel<<<dim3(B * H, 16), 256, 0, st>>>(p.ws, state, p.G, init_zero);
  SALA_CHECK_LAUNCH();
  kc<<<grid, kTcThreads, TcSmem<false>::bytes, st>>>(tq, tk, tv, p);
  SALA_CHECK_LAUNCH();
  if (!launch_lightning_fixup(q, k, v, g, o, state, q_norm_w, k_norm_w, sq, sk, sv, sg, so, p,
                              st))
    return SALA_ERR_CUDA;
  return SALA_OK;
}

// ------------------------------------------------------------------ failure-path self-test
}  // extern "C"

namespace {
// One thread waits, with the kernels' own bounded wait, on an mbarrier whose phase
// never completes (nothing arrives), then returns having raised SALA_ERR_TIMEOUT.
__global__ void selftest_wait_timeout_kernel(long long budget) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    (void)mbar_wait(&bar, 0, budget);
  }
}
}  // namespace

extern "C" {

sala_status sala_selftest_wait_timeout(long long cycles, void* stream) {
  if (cycles < 1 || cycles > kSpinCycleBudget) return SALA_ERR_INVALID_ARG;
  selftest_wait_timeout_kernel<<<1, 32, 0, as_stream(stream)>>>(cycles);
  SALA_CHECK_LAUNCH();
  return SALA_OK;
}

// ------------------------------------------------------------------ device error word
int sala_debug_bounds_line(void) {
#ifdef SALA_DEBUG
  if (cudaDeviceSynchronize() != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  int line = 0;
  if (cudaMemcpyFromSymbol(&line, g_bounds_line, sizeof(int)) != cudaSuccess) return 0;
  if (line != 0) {
    const int zero = 0;
    (void)cudaMemcpyToSymbol(g_bounds_line, &zero, sizeof(int));
  }
  return line;
#else
  return -1;
#endif
}

sala_status sala_get_device_error(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) {
    (void)cudaGetLastError();
    return SALA_ERR_CUDA;
  }
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_device_error, sizeof(int)) != cudaSuccess) return SALA_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess)
      return SALA_ERR_CUDA;
  }
  return (sala_status)h;
}

}  // extern "C"
