// lightning_decode.cuh -- one Lightning decode step per (batch, head).
//
// S <- S + kh v^T ; o = qh^T S ; y = sigmoid(g) * o, with qh/kh the RMS-normalised,
// rotate-half-rotated q and k at position pos[b] (MiniCPM-SALA summary page,
// "Prerequisites / Linear Attention": constant per-token compute and memory).
// The step is a single streaming pass over the D x D fp32 state: every CTA
// reads its (b, h) state once with 16-byte loads, writes it back once, and
// reduces the readout across warps in shared memory.  Bound: HBM bandwidth.
#pragma once

#include "common.cuh"

namespace sala {

constexpr int kDecThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads)
lightning_decode_kernel(const T* __restrict__ q, const T* __restrict__ k,
                        const T* __restrict__ v, const T* __restrict__ g, T* __restrict__ o,
                        float* __restrict__ state, const float* __restrict__ qw,
                        const float* __restrict__ kw, const int32_t* __restrict__ pos, int H,
                        sala_strides sq, sala_strides sk, sala_strides sv, sala_strides sg,
                        sala_strides so, double log2_base, float eps) {
  constexpr int kW = kDecThreads / 32;   // warps
  constexpr int kVec = D / 32;           // columns per lane (4 or 2)
  __shared__ float qh[D], kh[D], vs[D];
  __shared__ float part[kW][D];
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t p = pos[b];

  if (warp < 2) {
    // warp 0 normalises/rotates q, warp 1 k
    const T* src = warp == 0 ? q + b * sq.b + h * sq.h : k + b * sk.b + h * sk.h;
    const float* w = warp == 0 ? qw : kw;
    float x[kVec];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      x[u] = ld(src + lane + 32 * u);
      ss += x[u] * x[u];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float r = rsqrtf(ss / D + eps);
#pragma unroll
    for (int u = 0; u < kVec; ++u) x[u] *= r * (w ? w[lane + 32 * u] : 1.0f);
#pragma unroll
    for (int u = 0; u < kVec / 2; ++u) {
      float c, s;
      rope_cos_sin(p, lane + 32 * u, D, log2_base, &c, &s);
      const float x0 = x[u], x1 = x[u + kVec / 2];
      x[u] = x0 * c - x1 * s;
      x[u + kVec / 2] = x1 * c + x0 * s;
    }
    float* dst = warp == 0 ? qh : kh;
#pragma unroll
    for (int u = 0; u < kVec; ++u) dst[lane + 32 * u] = x[u];
  } else if (warp == 2) {
#pragma unroll
    for (int u = 0; u < kVec; ++u) vs[lane + 32 * u] = ld(v + b * sv.b + h * sv.h + lane + 32 * u);
  }
  __syncthreads();

  // Each lane owns kVec consecutive columns; warp w owns rows w, w+8, ...
  float* S = state + (size_t)bh * D * D;
  const int j0 = lane * kVec;
  float vj[kVec], acc[kVec];
#pragma unroll
  for (int u = 0; u < kVec; ++u) { vj[u] = vs[j0 + u]; acc[u] = 0.f; }
#pragma unroll 4
  for (int i = warp; i < D; i += kW) {
    float* row = S + (size_t)i * D + j0;
    float sv_[kVec];
    if constexpr (kVec == 4) {
      const float4 x = *reinterpret_cast<const float4*>(row);
      sv_[0] = x.x; sv_[1] = x.y; sv_[2] = x.z; sv_[3] = x.w;
    } else {
      const float2 x = *reinterpret_cast<const float2*>(row);
      sv_[0] = x.x; sv_[1] = x.y;
    }
    const float ki = kh[i], qi = qh[i];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      sv_[u] = fmaf(ki, vj[u], sv_[u]);
      acc[u] = fmaf(qi, sv_[u], acc[u]);
    }
    if constexpr (kVec == 4) {
      *reinterpret_cast<float4*>(row) = make_float4(sv_[0], sv_[1], sv_[2], sv_[3]);
    } else {
      *reinterpret_cast<float2*>(row) = make_float2(sv_[0], sv_[1]);
    }
  }
#pragma unroll
  for (int u = 0; u < kVec; ++u) part[warp][j0 + u] = acc[u];
  __syncthreads();
  for (int j = tid; j < D; j += kDecThreads) {
    float y = 0.f;
#pragma unroll
    for (int w = 0; w < kW; ++w) y += part[w][j];
    if (g) y *= sigmoidf_(ld(g + b * sg.b + h * sg.h + j));
    st(o + b * so.b + h * so.h + j, y);
  }
}

}  // namespace sala
