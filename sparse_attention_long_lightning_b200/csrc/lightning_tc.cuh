// lightning_tc.cuh -- Lightning attention prefill on 5th-gen tensor cores (tcgen05 + TMEM),
// bf16 activations, head_dim 128, chunk 128.
//
// Method: the Lightning state recurrence S_t = S_{t-1} + k_t v_t^T read out as
// o_t = q_t^T S_t (MiniCPM-SALA summary page, "Prerequisites / Linear Attention"),
// with per-head QK RMSNorm, rotate-half RoPE and a sigmoid output gate
// (tech-report mirror, section 02 (3) and (4)), evaluated chunk by chunk:
//   P_c = (Qh_c Kh_c^T) masked to s <= t,  O_c = P_c V_c + Qh_c S_{c-1},
//   S_c = S_{c-1} + Kh_c^T V_c,            y_c = sigmoid(g_c) * O_c.
//
// Sequence parallelism.  One head has only T/128 sequential chunks, so each
// head's chunks are split into G contiguous segments and the work runs in three
// launches:
//   (A) state pass   -- per segment, dS = sum_c Kh_c^T V_c  (reads k, v only)
//   (B) scan         -- per head, exclusive prefix of the segment sums (+ S0);
//                       also writes the final state
//   (C) output pass  -- per segment, start from its prefix state and emit y.
//
// Per chunk inside a CTA (128 threads, one per token row of the chunk):
//   * TMA brings the raw bf16 q/k/v tiles (128 tokens x 128 dims, 128-byte
//     swizzle, two 64-column slabs each) into a double-buffered stage.
//   * Each thread normalises/rotates its q and k row and converts q, k, v to
//     fp16 IN PLACE (same swizzled layout), so the tile is directly a tcgen05
//     operand.  fp16 (10-bit mantissa) keeps the rounding of the normalised,
//     rotated operands well inside the 1e-2 tolerance, where bf16 would not.
//   * One thread issues the MMAs (fp32 accumulation in tensor memory):
//       TMEM[P] = Qh Kh^T             (A, B K-major)
//       TMEM[O] = Qh S_op             (B = fp16 copy of S, MN-major)
//       TMEM[S] += Kh^T V             (A, B MN-major views of the same tiles)
//     then, after the threads turned P into a causally masked fp16 copy in
//     TMEM, TMEM[O] += P V with A read straight from tensor memory.
//   * The fp16 copy of S is rescaled by a power of two per chunk (2^-e) so it
//     stays inside the fp16 range at any length; P uses the same factor and
//     the epilogue multiplies O by 2^e (exact).
#pragma once

#include "lightning_cc.cuh"
#include "ptx.cuh"

namespace sala {

constexpr int kTcC = 128;                 // chunk (tokens)
constexpr int kTcThreads = 512;             // 16 warps: 4 per SM sub-partition
constexpr int kTcSlab = 128 * 128;        // one 128-row x 64-col 16-bit slab: 16 KB
constexpr int kTcTile = 2 * kTcSlab;      // 128 x 128 16-bit tile: 32 KB

template <bool kStateOnly>
struct TcSmem {
  static constexpr int kStages = kStateOnly ? 3 : 2;
  static constexpr int kStageBytes = (kStateOnly ? 2 : 3) * kTcTile;
  static constexpr int kSop = kStateOnly ? 0 : kTcTile;
  static constexpr int kMisc = 2048;
  static constexpr size_t bytes = 1024 /*alignment slack*/ + size_t(kStages) * kStageBytes + kSop + kMisc;
  static constexpr uint32_t kTmemCols = kStateOnly ? 128 : 512;
};

struct TcParams {
  const __nv_bfloat16* g;
  __nv_bfloat16* o;
  const float* qw;
  const float* kw;
  float* ws;  // [B*H][G][128][128] fp32: segment sums, turned into segment start states
  sala_strides sg, so;
  int B, T, H, G, NC;
  int64_t pos0;
  double log2_base;
  float eps;
};

// Block-wide max of |values| -> power-of-two exponent e >= 0 with max * 2^-e < 2^15.
__device__ __forceinline__ int tc_block_scale_exp(float m, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < kTcThreads / 32; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  int x = 0;
  frexpf(m, &x);
  return x > 15 ? x - 15 : 0;
}

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ uint4 f32x8_to_f16(const float* f) {
  return make_uint4(pack_f16x2(f[0], f[1]), pack_f16x2(f[2], f[3]), pack_f16x2(f[4], f[5]),
                    pack_f16x2(f[6], f[7]));
}
__device__ __forceinline__ uint32_t f16x8_nonfinite(const uint4& u) {
  return f16x2_nonfinite(u.x) | f16x2_nonfinite(u.y) | f16x2_nonfinite(u.z) |
         f16x2_nonfinite(u.w);
}

// Normalise + rotate a quarter of raw bf16 row r of the k (and q) tile and convert
// it, and a quarter of the v row, to fp16 in place.  Four consecutive lanes share
// a row: quarter qd owns rotation pairs i in [16 qd, 16 qd + 16) (chunks 2qd, 2qd+1
// of both 64-column slabs) and v chunks 4qd..4qd+3.  Tiles are two 64-column slabs
// of 128 rows x 128 bytes with the 128-byte swizzle.  An fp16 overflow here shows up
// downstream as a non-finite output or state, which the epilogue reports.
template <bool kWithQ>
__device__ __forceinline__ void tc_prep_quarter(uint8_t* sQ, uint8_t* sK, uint8_t* sV, int r,
                                                    int qd, const TcParams& p,
                                                    const float2* ang_base) {
  float ssq = 0.f, ssk = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = 2 * qd + (u & 1);
    const uint32_t a = (u >> 1) * kTcSlab + swz128(r, j);
    float f[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK + a), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) ssk = fmaf(f[e], f[e], ssk);
    if (kWithQ) {
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(sQ + a), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) ssq = fmaf(f[e], f[e], ssq);
    }
  }
  ssk += __shfl_xor_sync(0xffffffffu, ssk, 1);
  ssk += __shfl_xor_sync(0xffffffffu, ssk, 2);
  ssq += __shfl_xor_sync(0xffffffffu, ssq, 1);
  ssq += __shfl_xor_sync(0xffffffffu, ssq, 2);
  const float rk = rsqrtf(ssk * (1.0f / 128.0f) + p.eps);
  const float rq = rsqrtf(ssq * (1.0f / 128.0f) + p.eps);
  const float two_pi = 6.28318530717958647692f, inv_two_pi = 0.15915494309189533577f;
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {
    const int j = 2 * qd + jj;
    const uint32_t alo = swz128(r, j), ahi = kTcSlab + swz128(r, j);
    float klo[8], khi[8], qlo[8], qhi[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK + alo), klo);
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK + ahi), khi);
    if (kWithQ) {
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(sQ + alo), qlo);
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(sQ + ahi), qhi);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = 8 * j + e;  // rotation pair (i, i + 64)
      // angle = (chunk base angle, reduced in fp64) + r * inv_freq_i, re-reduced in fp32
      const float2 bf = ang_base[i];
      float ang = fmaf((float)r, bf.y, bf.x);
      ang = fmaf(-rintf(ang * inv_two_pi), two_pi, ang);
      float sn, cs;
      __sincosf(ang, &sn, &cs);
      const float wk0 = p.kw ? __ldg(p.kw + i) : 1.f, wk1 = p.kw ? __ldg(p.kw + i + 64) : 1.f;
      const float k0 = klo[e] * rk * wk0, k1 = khi[e] * rk * wk1;
      klo[e] = k0 * cs - k1 * sn;
      khi[e] = k1 * cs + k0 * sn;
      if (kWithQ) {
        const float wq0 = p.qw ? __ldg(p.qw + i) : 1.f, wq1 = p.qw ? __ldg(p.qw + i + 64) : 1.f;
        const float q0 = qlo[e] * rq * wq0, q1 = qhi[e] * rq * wq1;
        qlo[e] = q0 * cs - q1 * sn;
        qhi[e] = q1 * cs + q0 * sn;
      }
    }
    *reinterpret_cast<uint4*>(sK + alo) = f32x8_to_f16(klo);
    *reinterpret_cast<uint4*>(sK + ahi) = f32x8_to_f16(khi);
    if (kWithQ) {
      *reinterpret_cast<uint4*>(sQ + alo) = f32x8_to_f16(qlo);
      *reinterpret_cast<uint4*>(sQ + ahi) = f32x8_to_f16(qhi);
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int cj = 4 * qd + u;
    const uint32_t a = (cj >> 3) * kTcSlab + swz128(r, cj & 7);
    uint4 x = *reinterpret_cast<const uint4*>(sV + a);
    x.x = bf16x2_to_f16x2(x.x); x.y = bf16x2_to_f16x2(x.y);
    x.z = bf16x2_to_f16x2(x.z); x.w = bf16x2_to_f16x2(x.w);
    *reinterpret_cast<uint4*>(sV + a) = x;
  }
}

// K-major operand (rows = M or N, 128-byte rows along K), k-step kk of 16 elements.
__device__ __forceinline__ uint64_t tc_desc_k(const uint8_t* base, int kk) {
  return umma_desc_sw128(smem_u32(base) + (kk >> 2) * kTcSlab + (kk & 3) * 32, 16, 1024);
}
// MN-major operand (rows = K, 128-byte rows along MN, two 64-wide MN slabs), k-step kk.
__device__ __forceinline__ uint64_t tc_desc_mn(const uint8_t* base, int kk) {
  return umma_desc_sw128(smem_u32(base) + kk * 2048, kTcSlab, 1024);
}

// Gated bf16 epilogue of one chunk: thread (trow, cg) reads 32 fp32 columns of O from
// TMEM, scales by 2^e, multiplies by sigmoid(g) (prefetched) and stores 64 bytes.
__device__ __forceinline__ void tc_epilogue(uint32_t t_o, const uint4 (&gv)[4], bool gated,
                                            float os, __nv_bfloat16* orow, bool live,
                                            uint32_t& bad) {
  uint32_t r[32];
  tc_ld32(t_o, r);
  tc_wait_ld();
  if (!live) return;
  float chk = 0.f;
#pragma unroll
  for (int c8 = 0; c8 < 4; ++c8) {
    float y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = __uint_as_float(r[8 * c8 + e]) * os;
    if (gated) {
      float gf[8];
      bf16x8_to_f32(gv[c8], gf);
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] *= sigmoidf_(gf[e]);
    }
    // inf or NaN anywhere makes the running sum non-finite
#pragma unroll
    for (int e = 0; e < 8; ++e) chk += y[e];
    uint4 w;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]), h1 = __floats2bfloat162_rn(y[2], y[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(y[4], y[5]), h3 = __floats2bfloat162_rn(y[6], y[7]);
    w.x = *reinterpret_cast<uint32_t*>(&h0); w.y = *reinterpret_cast<uint32_t*>(&h1);
    w.z = *reinterpret_cast<uint32_t*>(&h2); w.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(orow + 8 * c8) = w;
  }
  bad |= !(fabsf(chk) <= 3.0e38f);
}

// Software pipeline per CTA (one segment of one head), chunk u:
//   A  wait TMA(u); prep(u) in place                      [tensor core: PV(u-1)]
//   B  wait PV(u-1); TMA(u+1) into the freed stage; issue score/inter/state MMAs of u
//   C  epilogue(u-1) from the other O buffer             [tensor core: MMAs of u]
//   D  wait MMAs of u; P -> masked fp16 (in place, TMEM); S -> fp16 operand for u+1
//   E  issue PV(u)
// TMEM columns: P fp32 [0,128) with its fp16 copy in [0,64), O[2] [128,384), S [384,512).
template <bool kStateOnly>
__global__ void __launch_bounds__(kTcThreads, 1)
lightning_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const TcParams p) {
  using L = TcSmem<kStateOnly>;
  constexpr uint32_t kIdScore = umma_idesc_f16(128, 128, false, false);
  constexpr uint32_t kIdInter = umma_idesc_f16(128, 128, false, true);
  constexpr uint32_t kIdState = umma_idesc_f16(128, 128, true, true);
  constexpr uint32_t kIdPV = umma_idesc_f16(128, 128, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* sop = smem + L::kStages * L::kStageBytes;
  uint8_t* misc = sop + L::kSop;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);      // [kStages]
  uint64_t* mma1_bar = full + 3;                           // score/inter/state done
  uint64_t* mma2_bar = full + 4;                           // PV done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + 5);
  float* red = reinterpret_cast<float*>(misc + 64);        // [16]
  double* inv_freq = reinterpret_cast<double*>(misc + 128);  // [64]
  float2* ang_tab = reinterpret_cast<float2*>(misc + 640);   // [2][64]: (base angle, inv_freq)
  uint32_t* smax = reinterpret_cast<uint32_t*>(misc + 1792);  // [2] bits of the |S| maximum

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int prow = 8 * warp + (lane >> 2), pqd = lane & 3;  // prep: 4 lanes per row
  const int lq = warp & 3, cg = warp >> 2;                  // TMEM: lanes 32lq.., cols 32cg..
  const int trow = 32 * lq + lane;
  // Heads vary fastest across the grid: CTAs running at the same time cover all heads
  // of the same token range, so whole [H, D] token rows are fetched together (DRAM
  // row locality) instead of one 256-byte head slice per 8 KB row.
  const int bh = blockIdx.x % (p.B * p.H);
  const int seg = blockIdx.x / (p.B * p.H);
  const int b = bh / p.H, h = bh % p.H;
  const int c_begin = (int)((int64_t)seg * p.NC / p.G);
  const int c_end = (int)((int64_t)(seg + 1) * p.NC / p.G);
  const int nchunks = c_end - c_begin;

  if (tid == 0) {
    smax[0] = 0u;
    smax[1] = 0u;
    for (int i = 0; i < L::kStages; ++i) mbar_init(&full[i], 1);
    mbar_init(mma1_bar, 1);
    mbar_init(mma2_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(tmem_slot, L::kTmemCols);
  if (tid < 64) inv_freq[tid] = exp2(-(2.0 * tid / 128.0) * p.log2_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_p = tmem, t_o0 = tmem + 128, t_s = kStateOnly ? tmem : tmem + 384;
  const uint32_t lane_off = (uint32_t)(32 * lq) << 16;

  // base angle of each rotation pair at the first token of chunk u (fp64 reduction)
  auto fill_angles = [&](int u) {
    if (tid < 64) {
      const double a = (double)(p.pos0 + (int64_t)(c_begin + u) * kTcC) * inv_freq[tid];
      const double two_pi = 6.283185307179586476925286766559;
      const double red_a = a - rint(a * (1.0 / two_pi)) * two_pi;
      ang_tab[(u & 1) * 64 + tid] = make_float2((float)red_a, (float)inv_freq[tid]);
    }
  };
  auto issue = [&](int u) {
    const int si = u % L::kStages;
    uint8_t* st = stages + si * L::kStageBytes;
    const int t0 = (c_begin + u) * kTcC;
    mbar_arrive_expect_tx(&full[si], L::kStageBytes);
    uint8_t* dk = st + (kStateOnly ? 0 : kTcTile);
    uint8_t* dv = dk + kTcTile;
    if (!kStateOnly) {
      tma_load_4d(st, &tmq, &full[si], 0, h, t0, b);
      tma_load_4d(st + kTcSlab, &tmq, &full[si], 64, h, t0, b);
    }
    tma_load_4d(dk, &tmk, &full[si], 0, h, t0, b);
    tma_load_4d(dk + kTcSlab, &tmk, &full[si], 64, h, t0, b);
    tma_load_4d(dv, &tmv, &full[si], 0, h, t0, b);
    tma_load_4d(dv + kTcSlab, &tmv, &full[si], 64, h, t0, b);
  };
  int issued = 0;
  if (tid == 0) {
    if (!kStateOnly) prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    for (; issued < L::kStages && issued < nchunks; ++issued) issue(issued);
  }
  __syncthreads();  // inv_freq visible
  fill_angles(0);

  float* wseg = p.ws + ((size_t)bh * p.G + seg) * (128 * 128);
  int e_cur = 0, e_prev = 0;
  uint32_t bad = 0;
  if (!kStateOnly) {
    // segment start state -> TMEM[S] (fp32) and its fp16 operand copy
    const float* src = wseg + (size_t)trow * 128 + 32 * cg;
    uint32_t r[32];
    float mx = 0.f;
#pragma unroll
    for (int v4 = 0; v4 < 8; ++v4) {
      const float4 x = *reinterpret_cast<const float4*>(src + 4 * v4);
      r[4 * v4 + 0] = __float_as_uint(x.x); r[4 * v4 + 1] = __float_as_uint(x.y);
      r[4 * v4 + 2] = __float_as_uint(x.z); r[4 * v4 + 3] = __float_as_uint(x.w);
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
    }
    tc_st32(t_s + lane_off + 32 * cg, r);
    tc_wait_st();
    e_cur = tc_block_scale_exp(mx, red);
    const float sc = pow2i(-e_cur);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * c4 + e]) * sc;
      const int cj = 4 * cg + c4;
      *reinterpret_cast<uint4*>(sop + (cj >> 3) * kTcSlab + swz128(trow, cj & 7)) = f32x8_to_f16(f);
    }
    fence_proxy_async_smem();
  }
  __syncthreads();  // angle table for chunk 0 visible

  uint32_t ph1 = 0, ph2 = 0;  // completed-phase counters of mma1_bar / mma2_bar
  bool ok = true;
  uint4 gv[4] = {};           // gate of this thread's row/columns for the pending epilogue
  const bool gated = p.g != nullptr;
  for (int u = 0; u < nchunks; ++u) {
    const int s = u % L::kStages;
    uint8_t* st = stages + s * L::kStageBytes;
    uint8_t* sQ = st;
    uint8_t* sK = st + (kStateOnly ? 0 : kTcTile);
    uint8_t* sV = sK + kTcTile;
    // ---- A: prep(u) while the tensor core runs PV(u-1)
    ok = ok && mbar_wait(&full[s], (u / L::kStages) & 1);
    if (ok) tc_prep_quarter<!kStateOnly>(sQ, sK, sV, prow, pqd, p, ang_tab + (u & 1) * 64);
    fence_proxy_async_smem();
    // angles of chunk u+1 (other parity; prep(u-1), the last reader, is behind a barrier)
    if (u + 1 < nchunks) fill_angles(u + 1);
    // ---- B: wait for the previous chunk's last MMAs, refill its stage, issue this chunk's
    if (u > 0) {
      ok = ok && mbar_wait(kStateOnly ? mma1_bar : mma2_bar,
                           (kStateOnly ? ph1 : ph2) & 1);
      if (kStateOnly) ++ph1; else ++ph2;
    }
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    tc_fence_after();
    if (tid == 0) {
      smax[(u + 1) & 1] = 0u;  // last read before this barrier; next written after the next one
      if (u > 0 && issued < nchunks) issue(issued++);  // stage of chunk u-1 is free
      const uint32_t t_o = t_o0 + 128 * (u & 1);
      if (!kStateOnly) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_ss(t_o, tc_desc_k(sQ, kk), tc_desc_mn(sop, kk), kIdInter, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        tc_mma_ss(t_s, tc_desc_mn(sK, kk), tc_desc_mn(sV, kk), kIdState,
                  (kStateOnly && u == 0 && kk == 0) ? 0u : 1u);
      if (!kStateOnly) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_ss(t_p, tc_desc_k(sQ, kk), tc_desc_k(sK, kk), kIdScore, kk > 0);
      }
      tc_commit(mma1_bar);
    }
    if (kStateOnly) continue;
    // ---- C: epilogue(u-1) while the tensor core runs this chunk's MMAs
    if (u > 0) {
      const int64_t t = (int64_t)(c_begin + u - 1) * kTcC + trow;
      __nv_bfloat16* orow = p.o + b * p.so.b + t * p.so.t + (int64_t)h * p.so.h + 32 * cg;
      tc_epilogue(t_o0 + 128 * ((u - 1) & 1) + lane_off + 32 * cg, gv, gated, pow2i(e_prev),
                  orow, t < p.T, bad);
    }
    {
      // prefetch this chunk's gate for its epilogue (next iteration)
      const int64_t t = (int64_t)(c_begin + u) * kTcC + trow;
      if (gated && t < p.T) {
        const uint4* gp = reinterpret_cast<const uint4*>(p.g + b * p.sg.b + t * p.sg.t +
                                                         (int64_t)h * p.sg.h + 32 * cg);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) gv[c8] = __ldg(gp + c8);
      }
    }
    // ---- D: P -> masked fp16 copy (in place), S -> fp16 operand for the next chunk
    ok = mbar_wait(mma1_bar, ph1 & 1);
    ++ph1;
    tc_fence_after();
    {
      uint32_t r[32];
      tc_ld32(t_p + lane_off + 32 * cg, r);
      tc_wait_ld();
      tc_fence_before();
      ok = __syncthreads_and(ok);  // every P column read before any fp16 copy lands on it
      if (!ok) break;
      tc_fence_after();
      const float ps = pow2i(-e_cur);
      uint32_t pk[16];
      if (lq > cg) {          // rows 32lq.. all lie below columns 32cg..32cg+31: no mask
#pragma unroll
        for (int m = 0; m < 16; ++m)
          pk[m] = pack_f16x2(__uint_as_float(r[2 * m]) * ps, __uint_as_float(r[2 * m + 1]) * ps);
      } else if (lq < cg) {   // strictly above the diagonal: all masked
#pragma unroll
        for (int m = 0; m < 16; ++m) pk[m] = 0u;
      } else {                // diagonal block: keep s <= t
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int col = 2 * m;
          const float a = col <= lane ? __uint_as_float(r[2 * m]) * ps : 0.f;
          const float c = col + 1 <= lane ? __uint_as_float(r[2 * m + 1]) * ps : 0.f;
          pk[m] = pack_f16x2(a, c);
        }
      }
      tc_st16(t_p + lane_off + 16 * cg, pk);
      tc_wait_st();
    }
    e_prev = e_cur;
    if (u + 1 < nchunks) {
      // |S| maximum of the block through one shared atomic per warp; it is read after
      // the next barrier, so the scale needs no barrier of its own
      uint32_t r[32];
      tc_ld32(t_s + lane_off + 32 * cg, r);
      tc_wait_ld();
      float mx = 0.f;
#pragma unroll
      for (int m = 0; m < 32; ++m) mx = fmaxf(mx, fabsf(__uint_as_float(r[m])));
      bad |= !(mx <= 3.0e38f);  // inf or NaN in the state
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (lane == 0) atomicMax(&smax[u & 1], __float_as_uint(mx));
    }
    // ---- E: PV(u)
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t t_o = t_o0 + 128 * (u & 1);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) tc_mma_ts(t_o, t_p + 8 * kk, tc_desc_mn(sV, kk), kIdPV, 1u);
      tc_commit(mma2_bar);
    }
    // ---- S -> fp16 operand for chunk u+1 (its last reader, the inter MMA of chunk u,
    // completed before D; the state MMA of chunk u+1 is issued only after the next barrier)
    if (u + 1 < nchunks) {
      tc_fence_after();
      uint32_t r[32];
      tc_ld32(t_s + lane_off + 32 * cg, r);
      tc_wait_ld();
      int x = 0;
      frexpf(__uint_as_float(smax[u & 1]), &x);
      const int e_next = x > 15 ? x - 15 : 0;
      const float sc = pow2i(-e_next);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * c4 + e]) * sc;
        const int cj = 4 * cg + c4;
        *reinterpret_cast<uint4*>(sop + (cj >> 3) * kTcSlab + swz128(trow, cj & 7)) =
            f32x8_to_f16(f);
      }
      fence_proxy_async_smem();
      e_cur = e_next;
    }
  }

  // drain: the last chunk's MMAs, then its epilogue / the segment sum
  if (ok && nchunks > 0) {
    ok = mbar_wait(kStateOnly ? mma1_bar : mma2_bar, (kStateOnly ? ph1 : ph2) & 1);
    tc_fence_after();
    if (ok) {
      if (kStateOnly) {
        float* dst = wseg + (size_t)trow * 128 + 32 * cg;
        uint32_t r[32];
        tc_ld32(t_s + lane_off + 32 * cg, r);
        tc_wait_ld();
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4)
          *reinterpret_cast<float4*>(dst + 4 * v4) =
              make_float4(__uint_as_float(r[4 * v4]), __uint_as_float(r[4 * v4 + 1]),
                          __uint_as_float(r[4 * v4 + 2]), __uint_as_float(r[4 * v4 + 3]));
      } else {
        const int u = nchunks;
        const int64_t t = (int64_t)(c_begin + u - 1) * kTcC + trow;
        __nv_bfloat16* orow = p.o + b * p.so.b + t * p.so.t + (int64_t)h * p.so.h + 32 * cg;
        tc_epilogue(t_o0 + 128 * ((u - 1) & 1) + lane_off + 32 * cg, gv, gated, pow2i(e_prev),
                    orow, t < p.T, bad);
      }
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_device_error(SALA_ERR_RANGE);
  if (!ok && tid == 0) {
    // wind down: let the last issued copies land before the CTA's shared memory goes away
    for (int u = issued > L::kStages ? issued - L::kStages : 0; u < issued; ++u)
      mbar_wait(&full[u % L::kStages], (u / L::kStages) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tc_dealloc(tmem, L::kTmemCols);
  }
}

// Exclusive prefix over the segment sums of each (b, h), in place; the final
// state (initial + all segments) goes to `state`.  grid (B*H, 16), 256 threads:
// each thread owns one float4 of the 128x128 state and walks the G segments.
__global__ void __launch_bounds__(256)
lightning_scan_kernel(float* __restrict__ ws, float* __restrict__ state, int G, int init_zero) {
  const int bh = blockIdx.x;
  const int e = (blockIdx.y * 256 + threadIdx.x) * 4;
  float* base = ws + (size_t)bh * G * (128 * 128) + e;
  float* sg = state + (size_t)bh * (128 * 128) + e;
  float4 run = init_zero ? make_float4(0.f, 0.f, 0.f, 0.f) : *reinterpret_cast<const float4*>(sg);
  float4 nxt = G > 0 ? *reinterpret_cast<const float4*>(base) : run;
  for (int s = 0; s < G; ++s) {
    float4* cell = reinterpret_cast<float4*>(base + (size_t)s * (128 * 128));
    const float4 d = nxt;
    if (s + 1 < G) nxt = *reinterpret_cast<const float4*>(base + (size_t)(s + 1) * (128 * 128));
    *cell = run;
    run.x += d.x; run.y += d.y; run.z += d.z; run.w += d.w;
  }
  *reinterpret_cast<float4*>(sg) = run;
}

inline int lightning_tc_segments(int B, int H, int T, int nsm) {
  const int NC = (T + kTcC - 1) / kTcC;
  int G = (8 * nsm) / (B * H);
  if (G < 1) G = 1;
  if (G > NC) G = NC;
  return G;
}

inline size_t lightning_tc_workspace(int B, int T, int H, int chunk, int nsm) {
  if (chunk != kTcC || T <= 0) return 0;
  return (size_t)B * H * lightning_tc_segments(B, H, T, nsm) * 128 * 128 * sizeof(float);
}

}  // namespace sala
