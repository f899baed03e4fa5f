// proj_gemm.cuh -- input projection of a Lightning layer on tcgen05 tensor cores, with
// the layer's operand preparation fused into the GEMM epilogue.
//
// Method (tech-report mirror, section 02 (3): QK-normalisation and an output gate in
// the linear layers; section 02 (4): RoPE in the linear layers): the hidden states x
// [B*T, hidden] are projected by one weight W [4 H D, hidden] (q heads, then k, v, g),
//   [q | k | v | g] = x W^T,
// and the epilogue writes what the Lightning recurrence consumes:
//   qh = RoPE(RMSNorm(q) * qw), kh = RoPE(RMSNorm(k) * kw) at position pos0 + t (fp16),
//   v as projected (bf16), gate = sigmoid(g) (fp16, the output gate's multiplier: in
//   (0, 1), where fp16's 11 significant bits lose nothing to its range).
//
// Design (sm_100a).  A persistent CTA per SM walks 128 x 256 output tiles (128 tokens,
// 256 output features = 256 / D whole heads, so every head's RMSNorm and rotation pairs
// live in one thread's accumulator row).  Warp 0 streams 64-wide K slices of x and W
// with TMA (128-byte swizzle) into a 4-stage ring; warp 1 issues the tcgen05 MMAs
// (M = 128, N = 256, K = 16, bf16 in, fp32 in TMEM) into one of two TMEM accumulators,
// so the epilogue of tile i overlaps the main loop of tile i + 1; warps 2-5 read the
// accumulator row of their token (tcgen05.ld), finish the head in registers and store
// it.  Tiles are visited in groups of 16 row tiles x all column tiles, so the CTAs that
// run at the same time share x and W tiles through L2.  Every wait is bounded; on
// expiry the kernel raises SALA_ERR_TIMEOUT, drains its copies and MMAs and returns.
#pragma once

#include "ptx.cuh"

namespace sala {

constexpr int kPjBM = 128;              // tokens per tile
constexpr int kPjBN = 256;              // output features per tile
constexpr int kPjBK = 64;               // K per stage (128 bytes of bf16)
constexpr int kPjStages = 4;
constexpr int kPjThreads = 6 * 32;      // TMA warp, MMA warp, 4 epilogue warps
constexpr int kPjGroupM = 16;           // row tiles per raster group
constexpr int kPjATile = kPjBM * kPjBK * 2;   // 16 KB
constexpr int kPjBTile = kPjBN * kPjBK * 2;   // 32 KB
constexpr int kPjStage = kPjATile + kPjBTile;
constexpr size_t kPjSmem = 1024 + size_t(kPjStages) * kPjStage + 1024;

struct ProjParams {
  __half* qh;            // [B, T, H, D] outputs (element strides below)
  __half* kh;
  __nv_bfloat16* v;
  __half* gate;
  sala_strides sq, sk, sv, sg;
  const float* qw;       // [D] or null
  const float* kw;
  int64_t M;             // B * T rows
  int T, H, hidden;
  int m_tiles, n_tiles;
  int64_t pos0;
  double log2_base;
  float eps;
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Tile i of the grouped raster -> (row tile, column tile).
__device__ __forceinline__ void pj_tile(int i, int m_tiles, int n_tiles, int& m, int& n) {
  const int group = i / (kPjGroupM * n_tiles);
  const int first = group * kPjGroupM;
  const int gm = min(kPjGroupM, m_tiles - first);
  const int local = i - group * kPjGroupM * n_tiles;
  m = first + local % gm;
  n = local / gm;
}

// 32 fp32 values -> 16 packed fp16 / bf16 words stored as 64 bytes.
__device__ __forceinline__ void pj_store_f16(__half* dst, const float* y) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(dst + 8 * c) =
        make_uint4(pack_f16x2(y[8 * c], y[8 * c + 1]), pack_f16x2(y[8 * c + 2], y[8 * c + 3]),
                   pack_f16x2(y[8 * c + 4], y[8 * c + 5]), pack_f16x2(y[8 * c + 6], y[8 * c + 7]));
}
__device__ __forceinline__ void pj_store_bf16(__nv_bfloat16* dst, const float* y) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(dst + 8 * c) =
        make_uint4(pack_bf16x2(y[8 * c], y[8 * c + 1]), pack_bf16x2(y[8 * c + 2], y[8 * c + 3]),
                   pack_bf16x2(y[8 * c + 4], y[8 * c + 5]),
                   pack_bf16x2(y[8 * c + 6], y[8 * c + 7]));
}

// Epilogue of one head (D accumulator columns at TMEM address `tacc`) of the row at
// token t.  sec: 0 = q, 1 = k (normalise, weight, rotate, fp16), 2 = v (bf16), 3 = gate
// (sigmoid, fp16).  Every lane of the warp runs the (warp-collective) TMEM loads; only
// lanes whose row exists (`valid`) store.
template <int D>
__device__ __forceinline__ void pj_head(uint32_t tacc, int sec, int64_t t, void* dst,
                                        const float* w, float eps, const double* inv_freq,
                                        bool valid) {
  float y[32];
  uint32_t r[32];
  if (sec >= 2) {
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      tc_ld32(tacc + 32 * c, r);
      tc_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float x = __uint_as_float(r[e]);
        y[e] = sec == 3 ? sigmoidf_(x) : x;
      }
      if (valid) {
        if (sec == 3)
          pj_store_f16(reinterpret_cast<__half*>(dst) + 32 * c, y);
        else
          pj_store_bf16(reinterpret_cast<__nv_bfloat16*>(dst) + 32 * c, y);
      }
    }
    return;
  }
  // RMS over the head
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    tc_ld32(tacc + 32 * c, r);
    tc_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(r[e]), __uint_as_float(r[e]), ss);
  }
  const float rs = rsqrtf(ss * (1.0f / D) + eps);
  const double two_pi = 6.283185307179586476925286766559;
  // rotation pairs (i, i + D/2), 32 at a time
#pragma unroll 1
  for (int c = 0; c < D / 64; ++c) {
    uint32_t r1[32];
    tc_ld32(tacc + 32 * c, r);
    tc_ld32(tacc + D / 2 + 32 * c, r1);
    tc_wait_ld();
    float lo[32], hi[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int i = 32 * c + e;
      float x0 = __uint_as_float(r[e]) * rs, x1 = __uint_as_float(r1[e]) * rs;
      if (w) {
        x0 *= __ldg(w + i);
        x1 *= __ldg(w + i + D / 2);
      }
      // angle t * inv_freq_i reduced to [-pi, pi] in fp64, then fp32 sine / cosine
      const double a = (double)t * inv_freq[i];
      float sn, cs;
      sincosf((float)(a - rint(a * (1.0 / two_pi)) * two_pi), &sn, &cs);
      lo[e] = fmaf(x0, cs, -x1 * sn);
      hi[e] = fmaf(x1, cs, x0 * sn);
    }
    if (valid) {
      __half* o = reinterpret_cast<__half*>(dst);
      pj_store_f16(o + 32 * c, lo);
      pj_store_f16(o + D / 2 + 32 * c, hi);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kPjThreads, 1)
lightning_proj_kernel(const __grid_constant__ CUtensorMap tmx,
                      const __grid_constant__ CUtensorMap tmw, const ProjParams p) {
  constexpr uint32_t kIdesc = umma_idesc_bf16(kPjBM, kPjBN, false, false);
  constexpr int kHeadsPerTile = kPjBN / D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* misc = smem + size_t(kPjStages) * kPjStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);          // [kPjStages]
  uint64_t* empty = full + kPjStages;                          // [kPjStages]
  uint64_t* acc_full = empty + kPjStages;                      // [2]
  uint64_t* acc_empty = acc_full + 2;                          // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  double* inv_freq = reinterpret_cast<double*>(misc + 256);     // [D / 2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.m_tiles * p.n_tiles;
  const int kblocks = p.hidden / kPjBK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPjStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < D / 2) inv_freq[threadIdx.x] = exp2(-(2.0 * threadIdx.x / D) * p.log2_base);
  if (warp == 1) tc_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmx);
      prefetch_tmap(&tmw);
      uint32_t it = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < ntiles && ok; i += gridDim.x) {
        int m, n;
        pj_tile(i, p.m_tiles, p.n_tiles, m, n);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kPjStages;
          if (*abort_flag || !mbar_wait(&empty[s], ((it / kPjStages) & 1) ^ 1)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + size_t(s) * kPjStage;
          mbar_arrive_expect_tx(&full[s], kPjStage);
          tma_load_2d(st, &tmx, &full[s], kb * kPjBK, m * kPjBM);
          tma_load_2d(st + kPjATile, &tmw, &full[s], kb * kPjBK, n * kPjBN);
        }
      }
      if (!ok) *abort_flag = 1;
      // every copy issued lands before shared memory is released
      const uint32_t n_out = it < (uint32_t)kPjStages ? it : (uint32_t)kPjStages;
      for (uint32_t u = it - n_out; u < it; ++u) mbar_wait(&full[u % kPjStages], (u / kPjStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < ntiles && ok; i += gridDim.x, ++tc) {
        const int a = tc & 1;
        if (*abort_flag || !mbar_wait(&acc_empty[a], ((tc >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + a * kPjBN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kPjStages;
          if (!mbar_wait(&full[s], (it / kPjStages) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + size_t(s) * kPjStage), sb = sa + kPjATile;
#pragma unroll
          for (int kk = 0; kk < kPjBK / 16; ++kk)
            tc_mma_ss(d, umma_desc_sw128(sa + kk * 32, 16, 1024),
                      umma_desc_sw128(sb + kk * 32, 16, 1024), kIdesc, (kb | kk) != 0);
          tc_commit(&empty[s]);  // the stage is free once these MMAs have read it
        }
        if (!ok) break;
        tc_commit(&acc_full[a]);
      }
      if (!ok) *abort_flag = 1;
      // every MMA issued completes before TMEM is released
      tc_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q4 = warp & 3;                      // TMEM lane quadrant of this warp
    const int row = 32 * q4 + lane;
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const int nsec = p.H * D / kPjBN;             // column tiles per section (q, k, v, g)
    uint32_t tc = 0;
    for (int i = blockIdx.x; i < ntiles; i += gridDim.x, ++tc) {
      const int a = tc & 1;
      if (*abort_flag || !mbar_wait(&acc_full[a], (tc >> 1) & 1)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      int m, n;
      pj_tile(i, p.m_tiles, p.n_tiles, m, n);
      const int sec = n / nsec;
      const int64_t gm = (int64_t)m * kPjBM + row;
      const bool valid = gm < p.M;  // rows past M (a ragged last tile) only load
      {
        const int b = valid ? (int)(gm / p.T) : 0;
        const int64_t t = valid ? gm % p.T : 0;
#pragma unroll 1
        for (int hh = 0; hh < kHeadsPerTile; ++hh) {
          const int h = (n % nsec) * kHeadsPerTile + hh;
          void* dst;
          const float* w = nullptr;
          if (sec == 0) {
            dst = p.qh + b * p.sq.b + t * p.sq.t + (int64_t)h * p.sq.h;
            w = p.qw;
          } else if (sec == 1) {
            dst = p.kh + b * p.sk.b + t * p.sk.t + (int64_t)h * p.sk.h;
            w = p.kw;
          } else if (sec == 2) {
            dst = p.v + b * p.sv.b + t * p.sv.t + (int64_t)h * p.sv.h;
          } else {
            dst = p.gate + b * p.sg.b + t * p.sg.t + (int64_t)h * p.sg.h;
          }
          pj_head<D>(tmem + a * kPjBN + hh * D + lane_off, sec, p.pos0 + t, dst, w, p.eps,
                     inv_freq, valid);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tc_dealloc(tmem, 512);
  }
}

}  // namespace sala
