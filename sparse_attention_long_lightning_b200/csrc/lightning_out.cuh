// lightning_out.cuh -- output pass of the bf16 / head_dim 128 Lightning prefill with
// warp-specialised phases (tcgen05 + TMEM).
//
// Pass (C) of the scheme in lightning_tc.cuh (MiniCPM-SALA summary page, "Prerequisites
// / Linear Attention"; tech-report mirror, section 02 (3) and (4)): for every chunk c
// of a segment, starting from the segment's prefix state,
//   O_c = mask(Qh_c Kh_c^T) V_c + Qh_c S_{c-1},  S_c = S_{c-1} + Kh_c^T V_c,
//   y_c = sigmoid(g_c) * O_c,
// with per-head RMSNorm + rotate-half RoPE on q and k.  The CUDA-core work of a chunk
// (operand preparation, P and S conversions, the gated output) is split between two
// warp groups so that the preparation of chunk u+1 overlaps the rest of chunk u; with
// every warp running every phase in turn between block barriers, nothing overlaps.
// The 16 warps split:
//   PREP (warps 0-7): wait for the TMA tiles of chunk u, normalise/rotate q and k and
//        convert q, k, v to fp16 in place (two threads per token row), signal the
//        issuer, then move on to chunk u+1 while the rest of chunk u is still running;
//   CONV (warps 8-15, two per TMEM lane quadrant, 64 columns each): thread 256 issues
//        the MMAs and the TMA copies; the group turns P into its masked fp16 copy, S
//        into the scaled fp16 operand of the next chunk, and O into gated bf16 output.
// Per chunk u the CONV group: issues Qh S_op / Kh^T V / Qh Kh^T (once PREP is done),
// writes the output of chunk u-1 when its P V has landed (and refills that chunk's
// stage with chunk u+1), converts P(u) and S(u), issues P V of chunk u.
// Two stages of q/k/v tiles and the fp16 S operand fill shared memory.  q/k and v of
// a stage are refilled separately: q/k as soon as the score/inter/state MMAs of their
// chunk are done, v once its P V is.  Every wait is bounded, and each group leaves
// together at its next named barrier after a failure.
#pragma once

#include "lightning_tc.cuh"

namespace sala {

constexpr int kLoPrepThreads = 256;   // warps 0-7
constexpr int kLoConvThreads = 256;   // warps 8-15
constexpr int kLoIssuer = kLoPrepThreads;  // first CONV thread issues MMAs and copies

// Item of the per-chunk angle table that holds rotation pairs i and i + 1 (i even): the
// two halves of a row read adjacent 16-byte words.
__device__ __forceinline__ int lo_ang_item(int i) { return ((i & 31) >> 1) * 2 + (i >> 5); }

// Normalise + rotate half of raw bf16 row r of the q and k tiles and convert it to fp16
// in place.  Two consecutive lanes share a row: half hf owns rotation pairs i in
// [32 hf, 32 hf + 32) (chunks 4hf..4hf+3 of both 64-column slabs).  Tiles are two
// 64-column slabs of 128 rows x 128 bytes with the 128-byte swizzle.  `ang` holds
// (base angle, inv_freq) of pairs i, i + 1 at item lo_ang_item(i).  The tiles and the
// table are in the kernel's __shared__ arrays: ordinary accesses, which the compiler
// is free to schedule.
__device__ __forceinline__ void lo_prep_qk_half(uint8_t* sQ, uint8_t* sK, int r, int hf,
                                                const TcParams& p, const float4* ang) {
  auto ld = [](const uint8_t* base, uint32_t off) {
    return *reinterpret_cast<const uint4*>(base + off);
  };
  auto st = [](uint8_t* base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4*>(base + off) = v;
  };
  float ssq[2] = {0.f, 0.f}, ssk[2] = {0.f, 0.f};
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int j = 4 * hf + (u & 3);
    const uint32_t a = (u >> 2) * kTcSlab + swz128(r, j);
    float f[8];
    bf16x8_to_f32(ld(sK, a), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) ssk[u & 1] = fmaf(f[e], f[e], ssk[u & 1]);
    bf16x8_to_f32(ld(sQ, a), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) ssq[u & 1] = fmaf(f[e], f[e], ssq[u & 1]);
  }
  float sk = ssk[0] + ssk[1], sq = ssq[0] + ssq[1];
  sk += __shfl_xor_sync(0xffffffffu, sk, 1);
  sq += __shfl_xor_sync(0xffffffffu, sq, 1);
  const float rk = rsqrtf(sk * (1.0f / 128.0f) + p.eps);
  const float rq = rsqrtf(sq * (1.0f / 128.0f) + p.eps);
  const float two_pi = 6.28318530717958647692f, inv_two_pi = 0.15915494309189533577f;
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int j = 4 * hf + jj;
    const uint32_t alo = swz128(r, j), ahi = kTcSlab + swz128(r, j);
    // cos, sin of the 8 pairs' angles first (shared by q and k), then k, then q: fewer
    // values live at once
    float cs[8], sn[8];
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      const float4 bb = ang[lo_ang_item(8 * j + 2 * e2)];
#pragma unroll
      for (int o = 0; o < 2; ++o) {
        // angle = (chunk base angle, reduced in fp64) + r * inv_freq_i, re-reduced in fp32
        float a = o ? fmaf((float)r, bb.w, bb.z) : fmaf((float)r, bb.y, bb.x);
        // nearest multiple of 2 pi by adding and removing 1.5 * 2^23 (exact rounding to
        // nearest for |a / 2 pi| < 2^22; plain adds instead of a rounding instruction)
        const float turns = (a * inv_two_pi + 12582912.0f) - 12582912.0f;
        a = fmaf(-turns, two_pi, a);
        __sincosf(a, &sn[2 * e2 + o], &cs[2 * e2 + o]);
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {  // t = 0: k, t = 1: q
      uint8_t* base = t ? sQ : sK;
      const float rs = t ? rq : rk;
      const float* w = t ? p.qw : p.kw;
      float xlo[8], xhi[8];
      bf16x8_to_f32(ld(base, alo), xlo);
      bf16x8_to_f32(ld(base, ahi), xhi);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = 8 * j + e;  // rotation pair (i, i + 64)
        // the row's RMS scale rides on cos/sin; the optional weights on the elements
        const float c = cs[e] * rs, sg = sn[e] * rs;
        float x0 = xlo[e], x1 = xhi[e];
        if (w) {
          x0 *= __ldg(w + i);
          x1 *= __ldg(w + i + 64);
        }
        xlo[e] = fmaf(x0, c, -x1 * sg);
        xhi[e] = fmaf(x1, c, x0 * sg);
      }
      st(base, alo, f32x8_to_f16(xlo));
      st(base, ahi, f32x8_to_f16(xhi));
    }
  }
}

// Half of the v row (slab hf) to fp16 in place; half 1 runs four chunks out of step so
// the two lanes of a row hit different bank groups.
// v is scaled by vscale (a power of two chosen from the segment's largest |v|; 1 for
// values that fp16 holds as they are).
__device__ __forceinline__ void lo_prep_v_half(uint8_t* sV, int r, int hf, float vscale) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    uint4* a = reinterpret_cast<uint4*>(sV + hf * kTcSlab + swz128(r, (u + 4 * hf) & 7));
    uint4 x = *a;
    if (vscale == 1.0f) {
      x.x = bf16x2_to_f16x2(x.x); x.y = bf16x2_to_f16x2(x.y);
      x.z = bf16x2_to_f16x2(x.z); x.w = bf16x2_to_f16x2(x.w);
    } else {
      x.x = bf16x2_to_f16x2_scaled(x.x, vscale); x.y = bf16x2_to_f16x2_scaled(x.y, vscale);
      x.z = bf16x2_to_f16x2_scaled(x.z, vscale); x.w = bf16x2_to_f16x2_scaled(x.w, vscale);
    }
    *a = x;
  }
}

// Gated bf16 epilogue of 32 columns: y = O * os * sigmoid(g) (os = 2^e undoes the operand
// scales), stored as 64 bytes.  kGateMult: the gate tensor already holds the multiplier,
// as fp16.
template <bool kGateMult>
__device__ __forceinline__ void lo_store32(const uint32_t (&r)[32], const uint4* gv, bool gated,
                                           float os, __nv_bfloat16* orow, uint32_t& bad) {
  float chk = 0.f;
#pragma unroll
  for (int c8 = 0; c8 < 4; ++c8) {
    float y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = __uint_as_float(r[8 * c8 + e]) * os;
    if (gated) {
      float gf[8];
      if (kGateMult)
        f16x8_to_f32(gv[c8], gf);
      else
        bf16x8_to_f32(gv[c8], gf);
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] *= kGateMult ? gf[e] : sigmoidf_(gf[e]);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) chk += y[e];
    uint4 w;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]), h1 = __floats2bfloat162_rn(y[2], y[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(y[4], y[5]), h3 = __floats2bfloat162_rn(y[6], y[7]);
    w.x = *reinterpret_cast<uint32_t*>(&h0); w.y = *reinterpret_cast<uint32_t*>(&h1);
    w.z = *reinterpret_cast<uint32_t*>(&h2); w.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(orow + 8 * c8) = w;
  }
  bad |= !(fabsf(chk) <= 3.0e38f);  // inf or NaN in the output
}

// TMEM columns: P fp32 [0,128) with its fp16 copy in [0,32) and [64,96), O[2] [128,384),
// S [384,512).
// kPrepared: q and k arrive already normalised and rotated as fp16 and the gate tensor
// holds sigmoid(g) as fp16 (the projection epilogue's outputs), so the PREP warps only
// convert v; they then also write each chunk's gated output (reading O from TMEM with the
// CONV warps' lane mapping), which takes that phase off the CONV warps: O buffer x is
// handed back through o_free[x], and the chunk's S-operand exponent arrives in e_ring[x].
template <bool kPrepared>
__global__ void __launch_bounds__(kTcThreads, 1)
lightning_out_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const TcParams p) {
  using L = TcSmem<false>;
  static_assert(L::kStages == 2, "two q/k/v stages");
  constexpr uint32_t kIdScore = umma_idesc_f16(128, 128, false, false);
  constexpr uint32_t kIdInter = umma_idesc_f16(128, 128, false, true);
  constexpr uint32_t kIdState = umma_idesc_f16(128, 128, true, true);
  constexpr uint32_t kIdPV = umma_idesc_f16(128, 128, false, true);

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, derived from the __shared__ array so it stays a shared pointer
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  uint8_t* sop = smem + 2 * L::kStageBytes;
  uint8_t* misc = sop + L::kSop;
  uint64_t* full_qk = reinterpret_cast<uint64_t*>(misc);        // [2] q/k tiles landed
  uint64_t* full_v = full_qk + 2;                              // [2] v tile landed
  uint64_t* prep_done = full_qk + 4;                           // [2] PREP warps done (count 8)
  uint64_t* mma1_bar = full_qk + 6;                            // score/inter/state done
  uint64_t* mma2_bar = full_qk + 7;                            // P V done
  uint64_t* drain_bar = full_qk + 8;                           // every MMA done (exit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 88);
  uint32_t* smax = reinterpret_cast<uint32_t*>(misc + 96);      // [2] bits of the |S| maximum
  volatile int* prep_abort = reinterpret_cast<volatile int*>(misc + 104);
  volatile int* conv_abort = reinterpret_cast<volatile int*>(misc + 108);
  float* red = reinterpret_cast<float*>(misc + 112);           // [16]
  double* inv_freq = reinterpret_cast<double*>(misc + 192);    // [64]
  // prepared operands only: the PREP warps write each chunk's output, so O buffer x is
  // handed back (o_free[x], count 8), P V of the chunk in O buffer x has its own barrier
  // (mma2b[x]), and the S-operand exponent of the chunk reaches them through e_ring[x]
  // (e_ready[x])
  uint64_t* o_free = reinterpret_cast<uint64_t*>(misc + 704);  // [2]
  uint64_t* mma2b = o_free + 2;                                // [2]
  uint64_t* e_ready = o_free + 4;                              // [2]
  int* e_ring = reinterpret_cast<int*>(misc + 752);            // [2]
  // [2][32]: (base angle, inv_freq) of rotation pairs i, i + 1 at item lo_ang_item(i)
  __shared__ float4 ang_tab[2 * 32];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_prep = tid < kLoPrepThreads;
  const int bh = blockIdx.x % (p.B * p.H);
  const int seg = blockIdx.x / (p.B * p.H);
  const int b = bh / p.H, h = bh % p.H;
  const int c_begin = (int)((int64_t)seg * p.NC / p.G);
  const int c_end = (int)((int64_t)(seg + 1) * p.NC / p.G);
  const int nchunks = c_end - c_begin;
  // v of this segment enters the MMAs as fp16 times 2^-ev (ev = 0 unless the segment's
  // largest |v|, recorded by the state pass, lies outside what fp16 holds); the TMEM
  // state and outputs carry the same factor, undone in the epilogue
  const int ev = v_operand_exp(__ldg(p.vmax + (size_t)bh * p.G + seg));
  const float vscale = pow2i(-ev), oscale = pow2i(ev);
  // CONV thread: TMEM lane row trow, columns 64*ch .. 64*ch+63
  const int lq = warp & 3, ch = (warp - 8) >> 2;
  const int trow = 32 * lq + lane;
  const uint32_t lane_off = (uint32_t)(32 * lq) << 16;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full_qk[i], 1);
      mbar_init(&full_v[i], 1);
      mbar_init(&prep_done[i], kLoPrepThreads / 32);
    }
    mbar_init(mma1_bar, 1);
    mbar_init(mma2_bar, 1);
    mbar_init(drain_bar, 1);
    if constexpr (kPrepared) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(&o_free[i], kLoPrepThreads / 32);
        mbar_init(&mma2b[i], 1);
        mbar_init(&e_ready[i], 1);
      }
    }
    smax[0] = smax[1] = 0u;
    *prep_abort = 0;
    *conv_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(tmem_slot, 512);
  if (tid < 64) inv_freq[tid] = exp2(-(2.0 * tid / 128.0) * p.log2_base);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_p = tmem, t_o0 = tmem + 128, t_s = tmem + 384;

  // base angle of each rotation pair at the first token of chunk u (fp64 reduction)
  auto fill_angles = [&](int u) {
    if (tid < 32) {  // pairs 2 tid, 2 tid + 1
      const double t0 = (double)(p.pos0 + (int64_t)(c_begin + u) * kTcC);
      const double two_pi = 6.283185307179586476925286766559;
      const double a0 = t0 * inv_freq[2 * tid], a1 = t0 * inv_freq[2 * tid + 1];
      const double r0 = a0 - rint(a0 * (1.0 / two_pi)) * two_pi;
      const double r1 = a1 - rint(a1 * (1.0 / two_pi)) * two_pi;
      ang_tab[(u & 1) * 32 + lo_ang_item(2 * tid)] =
          make_float4((float)r0, (float)inv_freq[2 * tid], (float)r1, (float)inv_freq[2 * tid + 1]);
    }
  };
  // q/k of chunk u (free once the score/inter/state MMAs of chunk u-2 are done) and v of
  // chunk u (free once P V of chunk u-2 is done) travel separately
  auto issue_qk = [&](int u) {
    const int si = u & 1;
    uint8_t* st = stages + si * L::kStageBytes;
    const int t0 = (c_begin + u) * kTcC;
    mbar_arrive_expect_tx(&full_qk[si], 2 * kTcTile);
    tma_load_4d(st, &tmq, &full_qk[si], 0, h, t0, b);
    tma_load_4d(st + kTcSlab, &tmq, &full_qk[si], 64, h, t0, b);
    tma_load_4d(st + kTcTile, &tmk, &full_qk[si], 0, h, t0, b);
    tma_load_4d(st + kTcTile + kTcSlab, &tmk, &full_qk[si], 64, h, t0, b);
  };
  auto issue_v = [&](int u) {
    const int si = u & 1;
    uint8_t* st = stages + si * L::kStageBytes;
    const int t0 = (c_begin + u) * kTcC;
    mbar_arrive_expect_tx(&full_v[si], kTcTile);
    tma_load_4d(st + 2 * kTcTile, &tmv, &full_v[si], 0, h, t0, b);
    tma_load_4d(st + 2 * kTcTile + kTcSlab, &tmv, &full_v[si], 64, h, t0, b);
  };
  int qk_issued = 0, v_issued = 0;
  if (tid == kLoIssuer) {
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    for (; qk_issued < 2 && qk_issued < nchunks; ++qk_issued) issue_qk(qk_issued);
    for (; v_issued < 2 && v_issued < nchunks; ++v_issued) issue_v(v_issued);
  }
  __syncthreads();  // inv_freq visible
  fill_angles(0);

  // segment start state -> TMEM[S] (fp32) and its fp16 operand copy (CONV threads)
  float* wseg = p.ws + ((size_t)bh * p.G + seg) * (128 * 128);
  int e_cur = 0;  // exponent of the fp16 S operand used by the current chunk
  {
    float mx = 0.f;
    uint32_t r0[32], r1[32];
    if (!is_prep) {
      const float* src = wseg + (size_t)trow * 128 + 64 * ch;
#pragma unroll
      for (int v4 = 0; v4 < 8; ++v4) {
        float4 x = *reinterpret_cast<const float4*>(src + 4 * v4);
        float4 y = *reinterpret_cast<const float4*>(src + 32 + 4 * v4);
        x.x *= vscale; x.y *= vscale; x.z *= vscale; x.w *= vscale;
        y.x *= vscale; y.y *= vscale; y.z *= vscale; y.w *= vscale;
        r0[4 * v4 + 0] = __float_as_uint(x.x); r0[4 * v4 + 1] = __float_as_uint(x.y);
        r0[4 * v4 + 2] = __float_as_uint(x.z); r0[4 * v4 + 3] = __float_as_uint(x.w);
        r1[4 * v4 + 0] = __float_as_uint(y.x); r1[4 * v4 + 1] = __float_as_uint(y.y);
        r1[4 * v4 + 2] = __float_as_uint(y.z); r1[4 * v4 + 3] = __float_as_uint(y.w);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(y.x), fabsf(y.y)), fmaxf(fabsf(y.z), fabsf(y.w))));
      }
      tc_st32(t_s + lane_off + 64 * ch, r0);
      tc_st32(t_s + lane_off + 64 * ch + 32, r1);
      tc_wait_st();
    }
    e_cur = tc_block_scale_exp(mx, red);
    if (!is_prep) {
      const float sc = pow2i(-e_cur);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float((hh ? r1 : r0)[8 * c4 + e]) * sc;
          const int cj = 8 * ch + 4 * hh + c4;
          *reinterpret_cast<uint4*>(sop + (cj >> 3) * kTcSlab + swz128(trow, cj & 7)) =
              f32x8_to_f16(f);
        }
      }
      fence_proxy_async_smem();
    }
  }
  tc_fence_before();
  __syncthreads();  // angle table of chunk 0, start state and its operand copy visible
  tc_fence_after();

  uint32_t bad = 0;
  if (is_prep) {
    // ------------------------------------------------------------------ PREP
    const int prow = tid >> 1, phf = tid & 1;
    bool fail = false;
    // prepared operands: PREP only converts v, so it also writes the gated output of each
    // chunk (TMEM lane row prow_o, columns 64 * pch ..), which the CONV warps otherwise do
    const int prow_o = 32 * (warp & 3) + lane, pch = warp >> 2;
    const uint32_t plane_off = (uint32_t)(32 * (warp & 3)) << 16;
    auto output_chunk = [&](int uu) -> bool {
      const int ob = uu & 1;
      const int64_t t = (int64_t)(c_begin + uu) * kTcC + prow_o;
      uint4 gq[8] = {};
      if (p.g != nullptr && t < p.T) {
        const uint4* gp = reinterpret_cast<const uint4*>(p.g + b * p.sg.b + t * p.sg.t +
                                                         (int64_t)h * p.sg.h + 64 * pch);
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) gq[c8] = __ldg(gp + c8);
      }
      if (!mbar_wait(&mma2b[ob], (uu >> 1) & 1) || !mbar_wait(&e_ready[ob], (uu >> 1) & 1))
        return false;
      tc_fence_after();
      const float os = pow2i(e_ring[ob]) * oscale;
      __nv_bfloat16* orow = p.o + b * p.so.b + t * p.so.t + (int64_t)h * p.so.h + 64 * pch;
      const uint32_t t_o = t_o0 + 128 * ob + plane_off + 64 * pch;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        tc_ld32(t_o + 32 * hh, r);
        tc_wait_ld();
        if (t < p.T) lo_store32<kPrepared>(r, gq + 4 * hh, p.g != nullptr, os, orow + 32 * hh, bad);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[ob]);  // O buffer ob may take chunk uu + 2
      return true;
    };
    for (int u = 0; u < nchunks; ++u) {
      const int s = u & 1;
      uint8_t* st = stages + s * L::kStageBytes;
      fail |= !mbar_wait(&full_qk[s], (u >> 1) & 1);
      if constexpr (!kPrepared) {
        if (!fail) lo_prep_qk_half(st, st + kTcTile, prow, phf, p, ang_tab + s * 32);
      }
      fail |= !mbar_wait(&full_v[s], (u >> 1) & 1);
      if (!fail) lo_prep_v_half(st + 2 * kTcTile, prow, phf, vscale);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&prep_done[s]);
      if (u + 1 < nchunks) fill_angles(u + 1);  // the other table; its last reader was prep(u-1)
      if constexpr (kPrepared) {
        if (u > 0 && !fail) fail = !output_chunk(u - 1);
      }
      if (fail) *prep_abort = 1;
      if (named_bar_or(2, kLoPrepThreads, fail) && *prep_abort) break;
    }
    if constexpr (kPrepared) {
      if (nchunks > 0 && !*prep_abort && !output_chunk(nchunks - 1)) *prep_abort = 1;
    }
  } else {
    // ------------------------------------------------------------------ CONV
    const bool iss = tid == kLoIssuer;
    const bool gated = p.g != nullptr;
    bool fail = false;
    int e_prev = 0;   // exponent of the chunk whose output is pending
    uint4 gv[8] = {}; // gate of this thread's row / 64 columns for the pending output
    for (int u = 0; u < nchunks; ++u) {
      const int s = u & 1;
      uint8_t* st = stages + s * L::kStageBytes;
      uint8_t* sQ = st;
      uint8_t* sK = st + kTcTile;
      uint8_t* sV = st + 2 * kTcTile;
      // ---- issue Qh S_op, Kh^T V, Qh Kh^T of chunk u once its operands are prepared
      if (iss) {
        smax[(u + 1) & 1] = 0u;  // last read before the previous barrier; next written below
        // operands prepared; P V of chunk u-1 (which reads the TMEM columns the score MMA
        // overwrites) has completed
        bool ok = mbar_wait(&prep_done[s], (u >> 1) & 1) &&
                  (u == 0 || mbar_wait(mma2_bar, (u - 1) & 1));
        if constexpr (kPrepared) {
          // O buffer s held chunk u - 2, whose output the PREP warps write; then the
          // exponent of this chunk's S operand for that output
          ok = ok && (u < 2 || mbar_wait(&o_free[s], ((u - 2) >> 1) & 1));
          if (ok) {
            e_ring[s] = e_cur;
            mbar_arrive(&e_ready[s]);
          }
        }
        fail |= !ok;
        if (ok) {
          tc_fence_after();
          const uint32_t t_o = t_o0 + 128 * s;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_ss(t_o, tc_desc_k(sQ, kk), tc_desc_mn(sop, kk), kIdInter, kk > 0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_ss(t_s, tc_desc_mn(sK, kk), tc_desc_mn(sV, kk), kIdState, 1u);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_ss(t_p, tc_desc_k(sQ, kk), tc_desc_k(sK, kk), kIdScore, kk > 0);
          tc_commit(mma1_bar);
        }
      }
      // ---- output of chunk u-1 once its P V has landed; refill its stage with chunk u+1
      if (u > 0 && kPrepared) {
        fail |= !mbar_wait(mma2_bar, (u - 1) & 1);
        tc_fence_after();
        if (iss && !fail && v_issued < nchunks) issue_v(v_issued++);  // v of chunk u-1 is free
      }
      if (u > 0 && !kPrepared) {
        fail |= !mbar_wait(mma2_bar, (u - 1) & 1);
        tc_fence_after();
        if (iss && !fail && v_issued < nchunks) issue_v(v_issued++);  // v of chunk u-1 is free
        const int64_t t = (int64_t)(c_begin + u - 1) * kTcC + trow;
        __nv_bfloat16* orow = p.o + b * p.so.b + t * p.so.t + (int64_t)h * p.so.h + 64 * ch;
        const uint32_t t_o = t_o0 + 128 * ((u - 1) & 1) + lane_off + 64 * ch;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t r[32];
          tc_ld32(t_o + 32 * hh, r);
          tc_wait_ld();
          if (t < p.T) lo_store32<kPrepared>(r, gv + 4 * hh, gated, pow2i(e_prev) * oscale, orow + 32 * hh,
                              bad);
        }
      }
      if (!kPrepared) {
        // gate of chunk u for its output (next iteration)
        const int64_t t = (int64_t)(c_begin + u) * kTcC + trow;
        if (gated && t < p.T) {
          const uint4* gp = reinterpret_cast<const uint4*>(p.g + b * p.sg.b + t * p.sg.t +
                                                           (int64_t)h * p.sg.h + 64 * ch);
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) gv[c8] = __ldg(gp + c8);
        }
      }
      // ---- P(u) -> causally masked fp16 copy, |S(u)| maximum.  A thread's fp16 copy of
      // its keys 64ch.. lands on TMEM columns 64ch + (0..31), which only this thread
      // reads as fp32 (half 0 before its copy is written, half 1 not overlapped), so no
      // other warp has to be waited for.
      fail |= !mbar_wait(mma1_bar, u & 1);
      tc_fence_after();
      if (iss && !fail && qk_issued < nchunks) issue_qk(qk_issued++);  // q/k of chunk u are free
      const float ps = pow2i(-e_cur);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        tc_ld32(t_p + lane_off + 64 * ch + 32 * hh, r);
        tc_wait_ld();
        const int cb = 64 * ch + 32 * hh;  // first column (key) of these 32
        uint32_t pk[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int col = cb + 2 * m;
          const float a = col <= trow ? __uint_as_float(r[2 * m]) * ps : 0.f;
          const float c = col + 1 <= trow ? __uint_as_float(r[2 * m + 1]) * ps : 0.f;
          pk[m] = pack_f16x2(a, c);
        }
        tc_st16(t_p + lane_off + 64 * ch + 16 * hh, pk);
      }
      tc_wait_st();
      float mx = 0.f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[32];
        tc_ld32(t_s + lane_off + 64 * ch + 32 * hh, r);
        tc_wait_ld();
#pragma unroll
        for (int m = 0; m < 32; ++m) mx = fmaxf(mx, fabsf(__uint_as_float(r[m])));
      }
      bad |= !(mx <= 3.0e38f);  // inf or NaN in the state
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (lane == 0) atomicMax(&smax[s], __float_as_uint(mx));
      tc_fence_before();
      if (fail) *conv_abort = 1;
      // the fp16 P copy is complete and the S maximum final
      if (named_bar_or(1, kLoConvThreads, fail) && *conv_abort) break;
      // ---- P V of chunk u
      if (iss) {
        tc_fence_after();
        const uint32_t t_o = t_o0 + 128 * s;
        // fp16 P: keys 0..63 in TMEM columns 0..31, keys 64..127 in columns 64..95
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_ts(t_o, t_p + 8 * kk + (kk >= 4 ? 32 : 0), tc_desc_mn(sV, kk), kIdPV, 1u);
        tc_commit(mma2_bar);
        if constexpr (kPrepared) tc_commit(&mma2b[s]);  // the PREP warps' output of chunk u
      }
      e_prev = e_cur;
      // ---- S(u) -> fp16 operand of chunk u+1 (its last reader, Qh S_op of chunk u, is done)
      if (u + 1 < nchunks) {
        tc_fence_after();
        int x = 0;
        frexpf(__uint_as_float(smax[s]), &x);
        const int e_next = x > 15 ? x - 15 : 0;
        const float sc = pow2i(-e_next);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t r[32];
          tc_ld32(t_s + lane_off + 64 * ch + 32 * hh, r);
          tc_wait_ld();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * c4 + e]) * sc;
            const int cj = 8 * ch + 4 * hh + c4;
            *reinterpret_cast<uint4*>(sop + (cj >> 3) * kTcSlab + swz128(trow, cj & 7)) =
                f32x8_to_f16(f);
          }
        }
        fence_proxy_async_smem();
        e_cur = e_next;
      }
      tc_fence_before();
      named_bar_sync(1, kLoConvThreads);  // S operand written, output reads of O done
    }
    // ---- output of the last chunk (the PREP warps write it for prepared operands)
    if (!kPrepared && nchunks > 0 && !*conv_abort) {
      const int u = nchunks;
      const bool ok = mbar_wait(mma2_bar, (u - 1) & 1);
      tc_fence_after();
      if (ok) {
        const int64_t t = (int64_t)(c_begin + u - 1) * kTcC + trow;
        __nv_bfloat16* orow = p.o + b * p.so.b + t * p.so.t + (int64_t)h * p.so.h + 64 * ch;
        const uint32_t t_o = t_o0 + 128 * ((u - 1) & 1) + lane_off + 64 * ch;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t r[32];
          tc_ld32(t_o + 32 * hh, r);
          tc_wait_ld();
          if (t < p.T) lo_store32<kPrepared>(r, gv + 4 * hh, gated, pow2i(e_prev) * oscale, orow + 32 * hh,
                              bad);
        }
      }
    }
    if (iss) {
      // wind down: every MMA complete, every copy landed, before resources are released
      tc_commit(drain_bar);
      mbar_wait(drain_bar, 0);
      for (int u = qk_issued > 2 ? qk_issued - 2 : 0; u < qk_issued; ++u)
        mbar_wait(&full_qk[u & 1], (u >> 1) & 1);
      for (int u = v_issued > 2 ? v_issued - 2 : 0; u < v_issued; ++u)
        mbar_wait(&full_v[u & 1], (u >> 1) & 1);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_device_error(SALA_ERR_RANGE);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tc_dealloc(tmem, 512);
  }
}

}  // namespace sala
