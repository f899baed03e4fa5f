// lightning_tc.cuh -- Lightning attention prefill on 5th-gen tensor cores (tcgen05 + TMEM),
// bf16 activations, head_dim 128, chunk 128: shared pieces, the state pass and the scan.
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
//   (A) state pass   -- per segment, dS = sum_c Kh_c^T V_c  (reads k, v only; here)
//   (B) scan         -- per head, exclusive prefix of the segment sums (+ S0);
//                       also writes the final state (here)
//   (C) output pass  -- per segment, start from its prefix state and emit y
//                       (lightning_out.cuh).
//
// Operands.  TMA brings the raw bf16 tiles (128 tokens x 128 dims, 128-byte swizzle,
// two 64-column slabs each) into shared memory; threads normalise/rotate q and k and
// convert q, k, v to fp16 IN PLACE (same swizzled layout), so a tile is directly a
// tcgen05 operand.  fp16 (10-bit mantissa) keeps the rounding of the normalised,
// rotated operands well inside the 1e-2 tolerance, where bf16 would not.  A single
// thread issues each kernel's MMAs (in the state pass, the producer warp's), fp32
// accumulation in tensor memory.
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
  // barriers, TMEM slot, inv_freq and scratch (< 704 bytes used).  The per-chunk angle
  // tables are static __shared__ arrays of the kernels (4 KiB state pass, 1 KiB output
  // pass) and count against the same 232448-byte per-block limit.
  static constexpr int kMisc = 1024;
  static constexpr size_t bytes = 1024 /*alignment slack*/ + size_t(kStages) * kStageBytes + kSop + kMisc;
  static_assert(bytes + (kStateOnly ? 4096 : 1024) <= 232448, "shared memory per block");
  static constexpr uint32_t kTmemCols = kStateOnly ? 128 : 512;
};

struct TcParams {
  const __nv_bfloat16* g;
  __nv_bfloat16* o;
  const float* qw;
  const float* kw;
  float* ws;  // [B*H][G][128][128] fp32: segment sums, turned into segment start states
  float* vmax;  // [B*H][G]: max |v| over each segment (written by the state pass)
  float* vssq;  // [B*H][G]: sum of v^2 over each segment (written by the state pass)
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

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void f16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = h.x;
    f[2 * i + 1] = h.y;
  }
}
__device__ __forceinline__ uint4 f32x8_to_f16(const float* f) {
  return make_uint4(pack_f16x2(f[0], f[1]), pack_f16x2(f[2], f[3]), pack_f16x2(f[4], f[5]),
                    pack_f16x2(f[6], f[7]));
}

// cos and sin of r * inv_freq_i for the 16 rotation pairs that a state-pass prep thread
// owns (its row r never changes; pair i = 16 qd + 8 jj + e).  The angle of pair i at
// token r of a chunk is (chunk base angle B_i) + r * inv_freq_i, so with the chunk's
// (cos B_i, sin B_i) from shared memory its cos and sin follow by angle addition -- four
// multiply-adds, no special-function unit work in the per-chunk loop.
struct TcRowRot {
  float c[16], s[16];
};

__device__ __forceinline__ void tc_row_rot_init(TcRowRot& rr, int r, int qd, const double* inv_freq) {
  const double two_pi = 6.283185307179586476925286766559;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const double a = (double)r * inv_freq[16 * qd + k];
    const float red = (float)(a - rint(a * (1.0 / two_pi)) * two_pi);
    sincosf(red, &rr.s[k], &rr.c[k]);
  }
}

// A quarter of raw bf16 row r of the v tile to fp16 in place, times vscale (a power of
// two); its largest |v| goes into vmax and its sum of squares into vss.
__device__ __forceinline__ void tc_prep_v_quarter(uint8_t* sV, int r, int qd, float vscale,
                                                  float& vmax, float& vss) {
  auto ld = [](const uint8_t* base, uint32_t off) {
    return *reinterpret_cast<const uint4*>(base + off);
  };
  auto st = [](uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
  };
  // v: quarter qd converts chunks 4 (qd & 1) .. +3 of slab qd >> 1, the slab-1 quarters
  // two chunks out of step, so the 8 lanes of a quarter-warp hit 8 different bank groups
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = 4 * (qd & 1) + ((u + 2 * (qd >> 1)) & 3);
    const uint32_t a = (qd >> 1) * kTcSlab + swz128(r, c);
    uint4 x = ld(sV, a);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
      vmax = fmaxf(vmax, fmaxf(fabsf(lo), fabsf(hi)));
      vss = fmaf(lo, lo, fmaf(hi, hi, vss));
    }
    if (vscale == 1.0f) {
      x.x = bf16x2_to_f16x2(x.x); x.y = bf16x2_to_f16x2(x.y);
      x.z = bf16x2_to_f16x2(x.z); x.w = bf16x2_to_f16x2(x.w);
    } else {
      x.x = bf16x2_to_f16x2_scaled(x.x, vscale); x.y = bf16x2_to_f16x2_scaled(x.y, vscale);
      x.z = bf16x2_to_f16x2_scaled(x.z, vscale); x.w = bf16x2_to_f16x2_scaled(x.w, vscale);
    }
    st(sV, a, x);
  }
}

// Normalise + rotate a quarter of raw bf16 row r of the k tile and convert it, and a
// quarter of the v row (times vscale, a power of two; its largest |v| goes into vmax),
// to fp16 in place.  Four consecutive lanes share a row: quarter
// qd owns rotation pairs i in [16 qd, 16 qd + 16) (chunks 2qd, 2qd+1 of both 64-column
// slabs) and four v chunks.  Tiles are two 64-column slabs of 128 rows x 128
// bytes with the 128-byte swizzle.  `cs_tab` (a static shared array, read with ordinary
// loads the compiler can schedule) holds the chunk's (cos B_i, sin B_i, cos B_i+1,
// sin B_i+1) for even i at item (i mod 16) / 2 * 4 + i / 16, so the four quarters of a
// row read adjacent 16-byte words.
__device__ __forceinline__ int tc_ang_item(int i) { return ((i & 15) >> 1) * 4 + (i >> 4); }

__device__ __forceinline__ void tc_prep_kv_quarter(uint8_t* sK, uint8_t* sV, int r, int qd,
                                                   const TcParams& p, const float4* cs_tab,
                                                   const TcRowRot& rr, float vscale,
                                                   float& vmax, float& vss) {
  // ordinary 16-byte accesses: sK and sV point into the kernel's __shared__ array, so these
  // are shared-memory instructions the compiler is free to schedule
  auto ld = [](const uint8_t* base, uint32_t off) {
    return *reinterpret_cast<const uint4*>(base + off);
  };
  auto st = [](uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
  };
  float ss[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = 2 * qd + (u & 1);
    float f[8];
    bf16x8_to_f32(ld(sK, (u >> 1) * kTcSlab + swz128(r, j)), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) ss[u] = fmaf(f[e], f[e], ss[u]);
  }
  float ssk = (ss[0] + ss[1]) + (ss[2] + ss[3]);
  ssk += __shfl_xor_sync(0xffffffffu, ssk, 1);
  ssk += __shfl_xor_sync(0xffffffffu, ssk, 2);
  const float rk = rsqrtf(ssk * (1.0f / 128.0f) + p.eps);
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {
    const int j = 2 * qd + jj;
    const uint32_t alo = swz128(r, j), ahi = kTcSlab + swz128(r, j);
    float klo[8], khi[8];
    bf16x8_to_f32(ld(sK, alo), klo);
    bf16x8_to_f32(ld(sK, ahi), khi);
    float4 cb;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i = 8 * j + e;  // rotation pair (i, i + 64)
      const int k = 8 * jj + e;
      // (cos B, sin B) of pairs i, i + 1: one shared 16-byte load per two pairs
      if ((e & 1) == 0) cb = cs_tab[tc_ang_item(i)];
      const float cB = (e & 1) ? cb.z : cb.x;
      const float sB = (e & 1) ? cb.w : cb.y;
      // cos, sin of B + r inv_freq_i, times the row's RMS scale
      const float cs = fmaf(cB, rr.c[k], -sB * rr.s[k]) * rk;
      const float sn = fmaf(sB, rr.c[k], cB * rr.s[k]) * rk;
      float k0 = klo[e], k1 = khi[e];
      if (p.kw) {
        k0 *= __ldg(p.kw + i);
        k1 *= __ldg(p.kw + i + 64);
      }
      klo[e] = fmaf(k0, cs, -k1 * sn);
      khi[e] = fmaf(k1, cs, k0 * sn);
    }
    st(sK, alo, f32x8_to_f16(klo));
    st(sK, ahi, f32x8_to_f16(khi));
  }
  tc_prep_v_quarter(sV, r, qd, vscale, vmax, vss);
}

// K-major operand (rows = M or N, 128-byte rows along K), k-step kk of 16 elements.
__device__ __forceinline__ uint64_t tc_desc_k(const uint8_t* base, int kk) {
  return umma_desc_sw128(smem_u32(base) + (kk >> 2) * kTcSlab + (kk & 3) * 32, 16, 1024);
}
// MN-major operand (rows = K, 128-byte rows along MN, two 64-wide MN slabs), k-step kk.
__device__ __forceinline__ uint64_t tc_desc_mn(const uint8_t* base, int kk) {
  return umma_desc_sw128(smem_u32(base) + kk * 2048, kTcSlab, 1024);
}

// State pass: per segment, dS = sum over its chunks of Kh_c^T V_c (TMEM accumulator),
// written to the workspace as fp32.
//   warps 0-15 (512 threads), per chunk u: wait TMA(u); prep k and v of chunk u in place
//     (4 lanes per row); each warp then arrives on prepped[u % S];
//   warp 16 runs the pipeline: once the MMA of u - 1 is done, that stage is refilled with
//     chunk u - 1 + S; once all 16 warps have prepped chunk u it issues the state MMA of u
//     (committing to mma_done[u % S]).  Before each copy it writes the chunk's table of
//     (cos, sin) of the RoPE base angles into an 8-slot ring; the copy's mbarrier orders
//     those writes before the prep warps' reads.  No CTA-wide barrier in the loop.
// TMEM: S in columns [0,128).
constexpr int kStThreads = kTcThreads + 32;
constexpr int kStAngRing = 8;  // > the largest lag (4 chunks) between producer and prep warps

// kPrepared: k arrives already normalised and rotated as fp16 (the projection epilogue's
// output), so the prep warps only convert v.
template <bool kPrepared>
__global__ void __launch_bounds__(kStThreads, 1)
lightning_state_kernel(const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const TcParams p) {
  using L = TcSmem<true>;
  constexpr int S = L::kStages;
  constexpr uint32_t kIdState = umma_idesc_f16(128, 128, true, true);
  constexpr int kPrepWarps = kTcThreads / 32;

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, derived from the __shared__ array so it stays a shared pointer
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  uint8_t* misc = stages + S * L::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);      // [S]: the stage's chunk landed
  uint64_t* mma_done = full + S;                           // [S]: its state MMA completed
  uint64_t* prepped = full + 2 * S;                        // [S]: all prep warps done with it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 96);
  double* inv_freq = reinterpret_cast<double*>(misc + 128);  // [64]
  // [kStAngRing][32] items of two pairs' (cos, sin) of the chunk's base angles
  __shared__ float4 ang_ring[kStAngRing * 32];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp == kPrepWarps;
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
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&mma_done[i], 1);
      mbar_init(&prepped[i], kPrepWarps);
    }
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(tmem_slot, L::kTmemCols);
  if (tid < 64) inv_freq[tid] = exp2(-(2.0 * tid / 128.0) * p.log2_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t t_s = *tmem_slot;
  const uint32_t lane_off = (uint32_t)(32 * lq) << 16;
  bool ok = true;
  // The first attempt converts v to fp16 as is and records the segment's largest |v|.
  // If that lies outside what fp16 holds exactly (v_operand_exp != 0), the segment runs
  // once more with v scaled by 2^-ev and the sum is scaled back by 2^ev when written:
  // the workspace always holds unscaled fp32 sums.  Stage and phase bookkeeping runs on
  // chunk counts that continue across the attempts.
  float vmax = 0.f, vss = 0.f, vss_seg = 0.f;
  float vscale = 1.0f;
  int ev = 0;
  __shared__ uint32_t s_vmax;
  __shared__ float s_vss;
  TcRowRot rr;
  if constexpr (!kPrepared) {
    if (!producer) tc_row_rot_init(rr, prow, pqd, inv_freq);
  }

  for (int attempt = 0; attempt < 2; ++attempt) {
    const int base = attempt * nchunks;  // global chunk count before this attempt
    if (producer) {
      // (cos, sin) of each rotation pair's angle at the first token of chunk n (fp64
      // reduction), written by the 32 lanes, then chunk n's copy (lane 0)
      auto fill_and_issue = [&](int n) {
        const int gi = base + n;
        if constexpr (!kPrepared) {
          const double two_pi = 6.283185307179586476925286766559;
          const double t0 = (double)(p.pos0 + (int64_t)(c_begin + n) * kTcC);
          float cs[2], sn[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {  // pairs 2 lane, 2 lane + 1
            const double a = t0 * inv_freq[2 * lane + k];
            const float red = (float)(a - rint(a * (1.0 / two_pi)) * two_pi);
            sincosf(red, &sn[k], &cs[k]);
          }
          ang_ring[(gi % kStAngRing) * 32 + tc_ang_item(2 * lane)] =
              make_float4(cs[0], sn[0], cs[1], sn[1]);
        }
        __syncwarp();
        if (lane == 0) {
          const int si = gi % S;
          uint8_t* dk = stages + si * L::kStageBytes;
          uint8_t* dv = dk + kTcTile;
          const int tok = (c_begin + n) * kTcC;
          mbar_arrive_expect_tx(&full[si], L::kStageBytes);  // release: orders the table writes
          tma_load_4d(dk, &tmk, &full[si], 0, h, tok, b);
          tma_load_4d(dk + kTcSlab, &tmk, &full[si], 64, h, tok, b);
          tma_load_4d(dv, &tmv, &full[si], 0, h, tok, b);
          tma_load_4d(dv + kTcSlab, &tmv, &full[si], 64, h, tok, b);
        }
        __syncwarp();
      };
      if (lane == 0 && attempt == 0) {
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
      }
      int issued = 0;
      for (; issued < S && issued < nchunks; ++issued) fill_and_issue(issued);
      int mmas = 0;  // state MMAs issued in this attempt (chunks 0 .. mmas-1)
      for (int u = 0; u < nchunks; ++u) {
        const int gu = base + u;
        const int s = gu % S;
        // refill the stage of chunk u - 1 as soon as its MMA has read it (early in prep(u))
        if (u >= 1 && issued < nchunks) {
          if (lane == 0) ok = mbar_wait(&mma_done[(gu - 1) % S], ((gu - 1) / S) & 1);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          fill_and_issue(issued++);
        }
        if (lane == 0) {
          ok = mbar_wait(&prepped[s], (gu / S) & 1);
          if (ok) {
            tc_fence_after();
            uint8_t* sK = stages + s * L::kStageBytes;
            uint8_t* sV = sK + kTcTile;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc_mma_ss(t_s, tc_desc_mn(sK, kk), tc_desc_mn(sV, kk), kIdState,
                        (u == 0 && kk == 0) ? 0u : 1u);
            tc_commit(&mma_done[s]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        mmas = u + 1;
      }
      if (lane == 0) {
        // the last MMA issued completes before TMEM is read, re-initialised or released
        if (mmas > 0 &&
            !mbar_wait(&mma_done[(base + mmas - 1) % S], ((base + mmas - 1) / S) & 1))
          ok = false;
        // every copy issued lands before the CTA's shared memory goes away (on the normal
        // path the prep warps have consumed them all already)
        for (int n = issued > S ? issued - S : 0; n < issued; ++n)
          mbar_wait(&full[(base + n) % S], ((base + n) / S) & 1);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    } else {
      for (int u = 0; u < nchunks; ++u) {
        const int gu = base + u;
        const int s = gu % S;
        uint8_t* sK = stages + s * L::kStageBytes;
        uint8_t* sV = sK + kTcTile;
        ok = mbar_wait(&full[s], (gu / S) & 1);
        if (ok) {
          if constexpr (kPrepared)
            tc_prep_v_quarter(sV, prow, pqd, vscale, vmax, vss);
          else
            tc_prep_kv_quarter(sK, sV, prow, pqd, p, ang_ring + (gu % kStAngRing) * 32, rr,
                               vscale, vmax, vss);
        }
        fence_proxy_async_smem();
        // a warp whose wait failed stops arriving; the producer's wait then runs out too
        if (!__all_sync(0xffffffffu, ok)) break;
        if (lane == 0) mbar_arrive(&prepped[s]);
      }
    }
    if (tid == 0) {
      s_vmax = 0u;
      s_vss = 0.f;
    }
    ok = __syncthreads_and(ok);
    if (attempt == 1 || !ok) break;
    // the segment's largest |v| (non-negative floats order as their bit patterns) and sum
    // of squares
    if (!producer) {
      const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(vmax));
      float ss = vss;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (lane == 0) {
        atomicMax(&s_vmax, m);
        atomicAdd(&s_vss, ss);
      }
    }
    __syncthreads();
    vmax = __uint_as_float(s_vmax);
    vss_seg = s_vss;
    ev = v_operand_exp(vmax);
    if (ev == 0) break;
    vscale = pow2i(-ev);
  }
  if (tid == 0 && ok) {
    p.vmax[(size_t)bh * p.G + seg] = vmax;
    p.vssq[(size_t)bh * p.G + seg] = vss_seg;
  }
  tc_fence_after();
  if (!producer && ok && nchunks > 0) {
    float* dst = p.ws + ((size_t)bh * p.G + seg) * (128 * 128) + (size_t)trow * 128 + 32 * cg;
    uint32_t r[32];
    tc_ld32(t_s + lane_off + 32 * cg, r);
    tc_wait_ld();
    const float us = pow2i(ev);  // undo the v scale of a second attempt (1 otherwise)
#pragma unroll
    for (int v4 = 0; v4 < 8; ++v4)
      *reinterpret_cast<float4*>(dst + 4 * v4) =
          make_float4(__uint_as_float(r[4 * v4]) * us, __uint_as_float(r[4 * v4 + 1]) * us,
                      __uint_as_float(r[4 * v4 + 2]) * us, __uint_as_float(r[4 * v4 + 3]) * us);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tc_dealloc(t_s, L::kTmemCols);
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

// Segments per head: about five one-CTA-per-SM waves over all heads.  Each CTA pays a
// fixed cost (setup, pipeline fill, the segment state's write), so fewer, longer segments
// are faster (B1 H32 T131072: 2.16 ms per layer with 5 waves, 2.23 with 8, 2.38 with 16).
inline int lightning_tc_segments(int B, int H, int T, int nsm) {
  const int NC = (T + kTcC - 1) / kTcC;
  int G = (5 * nsm) / (B * H);
  if (G < 1) G = 1;
  if (G > NC) G = NC;
  return G;
}

// Workspace: [B*H][G] segment states (fp32 128x128), then [B*H][G] floats of the
// segments' largest |v| and [B*H][G] floats of their sums of v^2 (256-byte aligned).
inline size_t lightning_tc_states_bytes(int B, int H, int G) {
  return (size_t)B * H * G * 128 * 128 * sizeof(float);
}
inline size_t lightning_tc_vmax_bytes(int B, int H, int G) {
  return ((size_t)B * H * G * sizeof(float) + 255) / 256 * 256;
}
// the segments' sums of v^2 follow their maxima
inline size_t lightning_tc_stats_bytes(int B, int H, int G) {
  return 2 * lightning_tc_vmax_bytes(B, H, G);
}
inline size_t lightning_tc_workspace(int B, int T, int H, int chunk, int nsm) {
  if (chunk != kTcC || T <= 0) return 0;
  const int G = lightning_tc_segments(B, H, T, nsm);
  return lightning_tc_states_bytes(B, H, G) + lightning_tc_stats_bytes(B, H, G);
}

}  // namespace sala
