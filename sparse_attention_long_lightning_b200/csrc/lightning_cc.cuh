// lightning_cc.cuh -- Lightning attention prefill on CUDA cores, fp32 arithmetic.
//
// Chunked evaluation of the Lightning recurrence S_t = S_{t-1} + k_t v_t^T,
// o_t = q_t^T S_t (MiniCPM-SALA summary page, "Prerequisites / Linear
// Attention"), with per-head RMSNorm + rotate-half RoPE on q and k and the
// sigmoid output gate (tech-report mirror, section 02 (3) and (4)).
// Per chunk of kCT tokens:
//   A   = (Qh Kh^T) masked to s <= t (diagonal included)
//   O   = A V + Qh S_prev ;  y = sigmoid(g) * O
//   S  += Kh^T V
// One CTA per (b, h) walks the chunks in order; the state lives in shared
// memory in fp32.  This path serves fp32 inputs (where fp32 products are
// required end to end) and head_dim 64; bf16 with head_dim 128 runs on the
// tensor-core kernel.
#pragma once

#include "common.cuh"

namespace sala {

constexpr int kCT = 64;           // chunk tile (tokens)
constexpr int kCCThreads = 256;

template <int D>
struct CCSmem {
  static constexpr int kLd = D + 1;  // padded row stride of the token tiles
  static constexpr size_t S = size_t(D) * D;
  static constexpr size_t Q = size_t(kCT) * kLd;
  static constexpr size_t A = size_t(kCT) * (kCT + 1);
  static constexpr size_t bytes = (S + 3 * Q + A) * sizeof(float);
};

// One head (b, h) = bh through all T_len tokens, starting from S0 ([D][D], or zero when
// null) and leaving the final state in Sg.
template <typename T, int D>
__device__ __forceinline__ void lightning_cc_head(
    int bh, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ g, T* __restrict__ o, const float* S0, float* Sg,
    const float* __restrict__ qw, const float* __restrict__ kw, int H, int T_len,
    sala_strides sq, sala_strides sk, sala_strides sv, sala_strides sg, sala_strides so,
    int64_t pos0, double log2_base, float eps) {
  constexpr int kLd = CCSmem<D>::kLd;
  extern __shared__ float smem[];
  float* S = smem;                        // [D][D]
  float* Qs = S + CCSmem<D>::S;           // [kCT][kLd]
  float* Ks = Qs + CCSmem<D>::Q;
  float* Vs = Ks + CCSmem<D>::Q;
  float* As = Vs + CCSmem<D>::Q;          // [kCT][kCT+1]

  const int b = bh / H, h = bh % H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int e = tid; e < D * D; e += kCCThreads) S[e] = S0 ? S0[e] : 0.0f;

  const T* qb = q + b * sq.b + h * sq.h;
  const T* kb = k + b * sk.b + h * sk.h;
  const T* vb = v + b * sv.b + h * sv.h;
  const T* gb = g ? g + b * sg.b + h * sg.h : nullptr;
  const bool write_o = o != nullptr;
  T* ob = write_o ? o + b * so.b + h * so.h : nullptr;
  constexpr int kPer = D / 32;  // elements per lane in a row

  for (int t0 = 0; t0 < T_len; t0 += kCT) {
    const int n = min(kCT, T_len - t0);
    __syncthreads();  // previous chunk fully consumed
    // ---- load, normalise and rotate q and k; load v (one warp per row) ----
    for (int r = warp; r < kCT; r += kCCThreads / 32) {
      float xq[kPer], xk[kPer], xv[kPer];
      const bool valid = r < n;
      const int64_t t = t0 + r;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int d = lane + 32 * u;
        xq[u] = valid ? ld(qb + t * sq.t + d) : 0.0f;
        xk[u] = valid ? ld(kb + t * sk.t + d) : 0.0f;
        xv[u] = valid ? ld(vb + t * sv.t + d) : 0.0f;
      }
      float ssq = 0.0f, ssk = 0.0f;
#pragma unroll
      for (int u = 0; u < kPer; ++u) { ssq += xq[u] * xq[u]; ssk += xk[u] * xk[u]; }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
        ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
      }
      const float rq = rsqrtf(ssq / D + eps), rk = rsqrtf(ssk / D + eps);
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int d = lane + 32 * u;
        xq[u] *= rq * (qw ? qw[d] : 1.0f);
        xk[u] *= rk * (kw ? kw[d] : 1.0f);
      }
      // rotate-half: element u pairs with u + kPer/2 (d and d + D/2 in this lane)
#pragma unroll
      for (int u = 0; u < kPer / 2; ++u) {
        const int i = lane + 32 * u;  // pair index < D/2
        float c, s;
        rope_cos_sin(pos0 + t, i, D, log2_base, &c, &s);
        const float q0 = xq[u], q1 = xq[u + kPer / 2];
        const float k0 = xk[u], k1 = xk[u + kPer / 2];
        xq[u] = q0 * c - q1 * s;  xq[u + kPer / 2] = q1 * c + q0 * s;
        xk[u] = k0 * c - k1 * s;  xk[u + kPer / 2] = k1 * c + k0 * s;
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int d = lane + 32 * u;
        Qs[r * kLd + d] = valid ? xq[u] : 0.0f;
        Ks[r * kLd + d] = valid ? xk[u] : 0.0f;
        Vs[r * kLd + d] = xv[u];
      }
    }
    __syncthreads();
    if (write_o) {  // o == nullptr: the state update alone
      // ---- A = Qh Kh^T, lower-triangular inclusive ----
      {
        const int r = tid >> 2;
#pragma unroll 4
        for (int m = 0; m < kCT / 4; ++m) {
          const int s = (tid & 3) + 4 * m;
          float a = 0.0f;
          if (s <= r) {
#pragma unroll 8
            for (int i = 0; i < D; ++i) a = fmaf(Qs[r * kLd + i], Ks[s * kLd + i], a);
          }
          As[r * (kCT + 1) + s] = a;
        }
      }
      __syncthreads();
      // ---- O = A V + Qh S, gate, store ----
      {
        const int rr = tid >> 5, jj = tid & 31;
        constexpr int kNJ = D / 32;
        float acc[8][kNJ];
#pragma unroll
        for (int m = 0; m < 8; ++m)
#pragma unroll
          for (int nj = 0; nj < kNJ; ++nj) acc[m][nj] = 0.0f;
        for (int s = 0; s < kCT; ++s) {
          float vv[kNJ];
#pragma unroll
          for (int nj = 0; nj < kNJ; ++nj) vv[nj] = Vs[s * kLd + jj + 32 * nj];
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float a = As[(rr + 8 * m) * (kCT + 1) + s];
#pragma unroll
            for (int nj = 0; nj < kNJ; ++nj) acc[m][nj] = fmaf(a, vv[nj], acc[m][nj]);
          }
        }
        for (int i = 0; i < D; ++i) {
          float sv_[kNJ];
#pragma unroll
          for (int nj = 0; nj < kNJ; ++nj) sv_[nj] = S[i * D + jj + 32 * nj];
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float qi = Qs[(rr + 8 * m) * kLd + i];
#pragma unroll
            for (int nj = 0; nj < kNJ; ++nj) acc[m][nj] = fmaf(qi, sv_[nj], acc[m][nj]);
          }
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int r = rr + 8 * m;
          if (r < n) {
            const int64_t t = t0 + r;
#pragma unroll
            for (int nj = 0; nj < kNJ; ++nj) {
              const int j = jj + 32 * nj;
              float y = acc[m][nj];
              if (gb) y *= sigmoidf_(ld(gb + t * sg.t + j));
              st(ob + t * so.t + j, y);
            }
          }
        }
      }
    }
    __syncthreads();  // everyone has read S for this chunk
    // ---- S += Kh^T V ----
    {
      const int ii = tid >> 5, jj = tid & 31;
      constexpr int kNJ = D / 32;
      for (int mb = 0; mb < D / 8; mb += 4) {
        float acc[4][kNJ];
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
          for (int nj = 0; nj < kNJ; ++nj) acc[m][nj] = 0.0f;
        for (int s = 0; s < kCT; ++s) {
          float vv[kNJ];
#pragma unroll
          for (int nj = 0; nj < kNJ; ++nj) vv[nj] = Vs[s * kLd + jj + 32 * nj];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const float kk = Ks[s * kLd + ii + 8 * (mb + m)];
#pragma unroll
            for (int nj = 0; nj < kNJ; ++nj) acc[m][nj] = fmaf(kk, vv[nj], acc[m][nj]);
          }
        }
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
          for (int nj = 0; nj < kNJ; ++nj) S[(ii + 8 * (mb + m)) * D + jj + 32 * nj] += acc[m][nj];
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < D * D; e += kCCThreads) Sg[e] = S[e];
}

template <typename T, int D>
__global__ void __launch_bounds__(kCCThreads)
lightning_prefill_cc_kernel(const T* __restrict__ q, const T* __restrict__ k,
                            const T* __restrict__ v, const T* __restrict__ g,
                            T* __restrict__ o, float* __restrict__ state,
                            const float* __restrict__ qw, const float* __restrict__ kw,
                            int H, int T_len, sala_strides sq, sala_strides sk, sala_strides sv,
                            sala_strides sg, sala_strides so, int64_t pos0, double log2_base,
                            float eps, int init_zero) {
  float* Sg = state + (size_t)blockIdx.x * D * D;
  lightning_cc_head<T, D>(blockIdx.x, q, k, v, g, o, init_zero ? nullptr : Sg, Sg, qw, kw, H,
                          T_len, sq, sk, sv, sg, so, pos0, log2_base, eps);
}

// Largest |v| of a head far above its rms: the tensor-core path's fp16 operands (11
// significant bits) would leave errors of ~2^-11 of the products with that value, which
// for a head dominated by a few large values exceeds the 1e-2 bound relative to the
// output's rms.  Such heads are recomputed in fp32.
constexpr float kCCOutlierRatio = 16.0f;

// Recomputes, on CUDA cores in fp32, every head (grid B*H) of a tensor-core prefill
// whose v is outlier-heavy (largest |v| > kCCOutlierRatio x rms(v), from the per-segment
// statistics the state pass wrote: vmax, vssq [B*H][G]); other heads return at once.
// The start state comes from ws (segment 0's start state, [B*H][G][D][D]) since the
// scan has already overwritten `state` with the final state.
template <int D>
__global__ void __launch_bounds__(kCCThreads)
lightning_cc_fixup_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                          const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ g,
                          __nv_bfloat16* __restrict__ o, float* __restrict__ state,
                          const float* __restrict__ qw, const float* __restrict__ kw, int H,
                          int T_len, sala_strides sq, sala_strides sk, sala_strides sv,
                          sala_strides sg, sala_strides so, int64_t pos0, double log2_base,
                          float eps, const float* __restrict__ ws, int G,
                          const float* __restrict__ vmax, const float* __restrict__ vssq) {
  const int bh = blockIdx.x;
  __shared__ int s_flag;
  if (threadIdx.x == 0) {
    float m = 0.f;
    double ss = 0.0;
    for (int s = 0; s < G; ++s) {
      m = fmaxf(m, vmax[(size_t)bh * G + s]);
      ss += (double)vssq[(size_t)bh * G + s];
    }
    const double rms = sqrt(ss / ((double)T_len * D));
    s_flag = (m < INFINITY) && (double)m > (double)kCCOutlierRatio * rms;
  }
  __syncthreads();
  if (!s_flag) return;
  lightning_cc_head<__nv_bfloat16, D>(bh, q, k, v, g, o, ws + (size_t)bh * G * D * D,
                                      state + (size_t)bh * D * D, qw, kw, H, T_len, sq, sk, sv,
                                      sg, so, pos0, log2_base, eps);
}

}  // namespace sala
