// lightning_tc.cuh -- Lightning prefill for bf16, head_dim 128 (provisional:
// runs the fp32 CUDA-core chunked kernel).
#pragma once

#include "lightning_cc.cuh"

namespace sala {

inline size_t lightning_tc_workspace(int B, int T, int H, int chunk, int nsm) {
  (void)B; (void)T; (void)H; (void)chunk; (void)nsm;
  return 0;
}

inline sala_status lightning_tc_launch(const void* q, const void* k, const void* v, const void* g,
                                       void* o, float* state, const float* qw, const float* kw,
                                       int B, int T, int H, sala_strides sq, sala_strides sk,
                                       sala_strides sv, sala_strides sg, sala_strides so,
                                       int chunk, int64_t pos0, double log2_base, float eps,
                                       int init_zero, void* ws, int nsm, cudaStream_t st) {
  (void)chunk; (void)ws; (void)nsm;
  auto kern = lightning_prefill_cc_kernel<__nv_bfloat16, 128>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)CCSmem<128>::bytes) != cudaSuccess)
    return SALA_ERR_CUDA;
  kern<<<B * H, kCCThreads, CCSmem<128>::bytes, st>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
      (const __nv_bfloat16*)g, (__nv_bfloat16*)o, state, qw, kw, H, T, sq, sk, sv, sg, so, pos0,
      log2_base, eps, init_zero);
  if (cudaPeekAtLastError() != cudaSuccess) { (void)cudaGetLastError(); return SALA_ERR_CUDA; }
  return SALA_OK;
}

}  // namespace sala
