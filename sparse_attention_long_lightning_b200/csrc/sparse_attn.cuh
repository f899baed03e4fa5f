// sparse_attn.cuh -- block-sparse softmax attention over selected KV blocks (NoPE).
//
// InfLLM-v2 style sparse layer (MiniCPM-SALA tech-report mirror, section 02 (2)
// and (4)): every query row t of KV head hk attends to the union of the blocks
// listed in idx[b][hk][t][:] (keys s <= t only), softmax scaled by `scale`, and
// the GQA group of hk (query heads hk*G .. hk*G+G-1) shares that selection.
//
// Design (sm_100a).  The per-row selections are random-access gathers, so the
// kernel is bound by moving 64-key K/V blocks from L2 into shared memory and
// through it, not by arithmetic: each gathered block serves only the group's
// G <= 16 query rows (16 flop per byte of K/V).  A persistent CTA runs two
// independent row pipelines ("groups").  One producer warp drives both: lane g
// walks group g's rows and, for every selected block, issues TMA tile loads of
// K and V (128-byte swizzle, no multicast) into the group's NS-deep ring,
// recording the block id beside the stage.  Each group has four consumer
// warps that split every 64-key block 16 keys apiece: the group's 16 query
// heads form the M = 16 operand of m16n8k16 tensor-core MMAs (Q K^T in bf16
// with four independent accumulator chains, P V in fp16 on an fp16 copy of V
// that a pre-pass writes once and checks for values outside the fp16 range;
// fp32 accumulation), the online softmax runs per warp in registers with a
// lazily raised reference maximum (rescaling only when a
// score exceeds it by more than 2^8), and the four partial (max, sum, O)
// triples are merged through shared memory at the end of the row.  All waits
// are bounded; a wait that runs out raises SALA_ERR_TIMEOUT in the device
// error word and the kernel winds down instead of hanging.
#pragma once

#include "ptx.cuh"

namespace sala {

constexpr int kSaBlk = 64;          // keys per KV block
constexpr int kSaConsumers = 4;     // consumer warps per group (16 keys each)
constexpr int kSaGroups = 2;        // independent row pipelines per CTA
constexpr int kSaThreads = (kSaGroups * kSaConsumers + 1) * 32;
constexpr float kSaLazy = 8.0f;     // log2 headroom before the reference max is raised

template <int D, int NS>
struct SaSmem {
  static constexpr int kHalf = kSaBlk * 64 * 2;                 // one 64-col box: 8 KB
  static constexpr int kTile = kSaBlk * D * 2;                  // K or V block
  static constexpr int kStage = 2 * kTile;                      // K then V
  // The row's last stage doubles as the merge buffer for the four warps' partial O.
  static_assert(kSaConsumers * 16 * D * 4 <= kStage, "merge buffer must fit in a stage");
  static constexpr int kML = kSaConsumers * 16 * 2 * 4;         // partial m, l
  static constexpr int kGroup = NS * kStage;                    // multiple of 1024
  static constexpr int kBars = ((2 * NS + 2) * 8 + NS * 4 + 16 + 15) / 16 * 16;  // barriers, ids, flag
  static constexpr size_t bytes = 1024 + size_t(kSaGroups) * (kGroup + kML + kBars);
};

struct SaParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* g;
  __nv_bfloat16* o;
  const int32_t* idx;
  sala_strides sq, sg, so;
  int n_sel, B, T, Hq, Hkv, G;
  float scale_log2;  // softmax scale * log2(e)
  int64_t rows;      // B * Hkv * T
};

// A selected block j takes part in row t iff j >= 0 and its first key is <= t.
__device__ __forceinline__ bool sa_block_live(int j, int64_t t) {
  return j >= 0 && (int64_t)j * kSaBlk <= t;
}

template <int D, int NS>
__global__ void __launch_bounds__(kSaThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const SaParams p) {
  using L = SaSmem<D, NS>;
  constexpr int kKSteps = D / 16;   // QK^T k-steps
  constexpr int kNT = D / 8;        // PV n-tiles
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t T = p.T;
  uint8_t* bar_base = smem + size_t(kSaGroups) * L::kGroup;  // per group: [bars][ML]
  constexpr int kGB = L::kBars + L::kML;

  if (threadIdx.x < kSaGroups) {
    uint8_t* gb = bar_base + threadIdx.x * kGB;
    uint64_t* full = reinterpret_cast<uint64_t*>(gb);
    uint64_t* empty = full + NS;
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kSaConsumers);
    }
    mbar_init(empty + NS, kSaConsumers);      // merge: last stage fully read
    mbar_init(empty + NS + 1, kSaConsumers);  // merge: partials written
    *reinterpret_cast<volatile int*>(gb + (2 * NS + 2) * 8 + NS * 4) = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kSaGroups * kSaConsumers) {
    // ------------------------------------------------------------ producer
    if (lane < kSaGroups) {
      const int grp = lane;
      uint8_t* stages = smem + size_t(grp) * L::kGroup;
      uint8_t* gb = bar_base + grp * kGB;
      uint64_t* full = reinterpret_cast<uint64_t*>(gb);
      uint64_t* empty = full + NS;
      int32_t* stage_j = reinterpret_cast<int32_t*>(gb + (2 * NS + 2) * 8);
      volatile int* abort_flag = reinterpret_cast<volatile int*>(stage_j + NS);
      if (grp == 0) {
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_v);
      }
      uint32_t it = 0;
      bool ok = true;
      for (int64_t r = blockIdx.x + (int64_t)grp * gridDim.x; r < p.rows && ok;
           r += (int64_t)kSaGroups * gridDim.x) {
        const int64_t t = r % T;
        const int hk = (int)((r / T) % p.Hkv);
        const int b = (int)(r / (T * p.Hkv));
        const int32_t* ir = p.idx + r * p.n_sel;
        for (int e = 0; e < p.n_sel; ++e) {
          const int j = __ldg(ir + e);
          if (!sa_block_live(j, t)) continue;
          const int s = it % NS;
          if (*abort_flag || !mbar_wait(&empty[s], ((it / NS) & 1) ^ 1)) { ok = false; break; }
          uint8_t* st = stages + size_t(s) * L::kStage;
          stage_j[s] = j;
          mbar_arrive_expect_tx(&full[s], L::kStage);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf) {
            tma_load_4d(st + hf * L::kHalf, &tmap_k, &full[s], hf * 64, hk, j * kSaBlk, b);
            tma_load_4d(st + L::kTile + hf * L::kHalf, &tmap_v, &full[s], hf * 64, hk,
                        j * kSaBlk, b);
          }
          ++it;
        }
      }
      if (!ok) *abort_flag = 1;
      // Wait (bounded) until every copy this thread issued has landed.
      const uint32_t n_out = it < (uint32_t)NS ? it : (uint32_t)NS;
      for (uint32_t u = it - n_out; u < it; ++u) mbar_wait(&full[u % NS], (u / NS) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int grp = warp / kSaConsumers, wq = warp % kSaConsumers;
  uint8_t* stages = smem + size_t(grp) * L::kGroup;
  uint8_t* gb = bar_base + grp * kGB;
  uint64_t* full = reinterpret_cast<uint64_t*>(gb);
  uint64_t* empty = full + NS;
  uint64_t* mrg_read = empty + NS;       // all warps finished reading the last stage
  uint64_t* mrg_written = mrg_read + 1;  // all warps wrote their partials
  const int32_t* stage_j = reinterpret_cast<const int32_t*>(gb + (2 * NS + 2) * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + (2 * NS + 2) * 8 + NS * 4);
  float* mergeML = reinterpret_cast<float*>(gb + L::kBars);

  const int gq = lane >> 2, tq = lane & 3;  // mma group id / thread in group
  uint32_t it = 0, nmrg = 0;
  float* myML = mergeML + wq * 32;
  const int ct = wq * 32 + lane;            // 0..127 within the group
  for (int64_t r = blockIdx.x + (int64_t)grp * gridDim.x; r < p.rows;
       r += (int64_t)kSaGroups * gridDim.x) {
    const int64_t t = r % T;
    const int hk = (int)((r / T) % p.Hkv);
    const int b = (int)(r / (T * p.Hkv));

    // number of live blocks of this row (the producer streams exactly these)
    int nblk = 0;
    {
      const int32_t* ir = p.idx + r * p.n_sel;
      for (int e0 = 0; e0 < p.n_sel; e0 += 32) {
        const int e = e0 + lane;
        const bool live = e < p.n_sel && sa_block_live(__ldg(ir + e), t);
        nblk += __popc(__ballot_sync(0xffffffffu, live));
      }
    }
    // Q fragments: rows = the group's query heads (padded to 16 with zeros).
    uint32_t qa[kKSteps][4];
    {
      const __nv_bfloat16* qr = p.q + b * p.sq.b + t * p.sq.t + (int64_t)(hk * p.G) * p.sq.h;
#pragma unroll
      for (int kk = 0; kk < kKSteps; ++kk) {
#pragma unroll
        for (int rg = 0; rg < 4; ++rg) {
          const int row = gq + (rg & 1) * 8;
          const int col = kk * 16 + tq * 2 + (rg >> 1) * 8;
          qa[kk][rg] = row < p.G
                           ? *reinterpret_cast<const uint32_t*>(qr + (int64_t)row * p.sq.h + col)
                           : 0u;
        }
      }
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows gq, gq+8 (log2 domain)
    float oacc[kNT][4];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
    bool ok = !*abort_flag;
    int s_last = 0;

    for (int e = 0; e < nblk && ok; ++e) {
      const int s = it % NS;
      if (!mbar_wait(&full[s], (it / NS) & 1)) { ok = false; break; }
      const int j = stage_j[s];
      const uint32_t kb = smem_u32(stages + size_t(s) * L::kStage);
      const uint32_t vb = kb + L::kTile;

      // ---- S = Q K^T for keys 16*wq .. 16*wq+15 of the block
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        float sd[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const int mat = lane >> 3, rin = lane & 7;
        const uint32_t krow = wq * 16 + (mat >> 1) * 8 + rin;
#pragma unroll
        for (int kk = 0; kk < kKSteps; ++kk) {
          const uint32_t chunk = 2 * kk + (mat & 1);
          const uint32_t addr = kb + (chunk >> 3) * L::kHalf + swz128(krow, chunk & 7);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
          if (kk & 1) {
            mma_bf16_16816(sd[0], qa[kk], b0, b1);
            mma_bf16_16816(sd[1], qa[kk], b2, b3);
          } else {
            mma_bf16_16816(sc[0], qa[kk], b0, b1);
            mma_bf16_16816(sc[1], qa[kk], b2, b3);
          }
        }
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) sc[a][c] += sd[a][c];
      }
      // ---- this warp's V fragments go to registers, then the stage is released at once
      // (except the row's last block, whose stage is reused for the merge)
      uint32_t vv[kNT / 2][4];
      {
        const int mat = lane >> 3, rin = lane & 7;
        const uint32_t vrow = wq * 16 + (mat & 1) * 8 + rin;
#pragma unroll
        for (int pp = 0; pp < kNT / 2; ++pp) {
          const uint32_t chunk = 2 * pp + (mat >> 1);
          const uint32_t addr = vb + (chunk >> 3) * L::kHalf + swz128(vrow, chunk & 7);
          ldsm_x4_t(addr, vv[pp][0], vv[pp][1], vv[pp][2], vv[pp][3]);
        }
      }
      __syncwarp();
      if (e + 1 < nblk) {
        if (lane == 0) mbar_arrive(&empty[s]);
      } else {
        s_last = s;
      }
      // ---- scale; causal mask only where the block reaches past t
      const bool straddle = (int64_t)j * kSaBlk + kSaBlk - 1 > t;
      const int64_t key0 = (int64_t)j * kSaBlk + wq * 16 + tq * 2;
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float x = sc[nt][c] * p.scale_log2;
          if (straddle && key0 + nt * 8 + (c & 1) > t) x = -INFINITY;
          sc[nt][c] = x;
        }
        mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
      }
      // ---- lazy reference max: raise it (and rescale) only when exceeded by > 2^8
      if (__any_sync(0xffffffffu, mx0 > m0 + kSaLazy || mx1 > m1 + kSaLazy)) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float al0 = (n0 == -INFINITY) ? 1.f : exp2f(m0 - n0);
        const float al1 = (n1 == -INFINITY) ? 1.f : exp2f(m1 - n1);
        m0 = n0;
        m1 = n1;
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          oacc[nt][0] *= al0; oacc[nt][1] *= al0;
          oacc[nt][2] *= al1; oacc[nt][3] *= al1;
        }
      }
      const float mu0 = m0 == -INFINITY ? 0.f : m0, mu1 = m1 == -INFINITY ? 0.f : m1;
      // P in fp16 (10-bit mantissa), V is the fp16 copy
      uint32_t pa[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float p0 = exp2f(sc[nt][0] - mu0), p1 = exp2f(sc[nt][1] - mu0);
        const float p2 = exp2f(sc[nt][2] - mu1), p3 = exp2f(sc[nt][3] - mu1);
        l0 += p0 + p1;
        l1 += p2 + p3;
        pa[nt * 2 + 0] = pack_f16x2(p0, p1);
        pa[nt * 2 + 1] = pack_f16x2(p2, p3);
      }
      // ---- O += P V
#pragma unroll
      for (int pp = 0; pp < kNT / 2; ++pp) {
        mma_f16_16816(oacc[2 * pp], pa, vv[pp][0], vv[pp][1]);
        mma_f16_16816(oacc[2 * pp + 1], pa, vv[pp][2], vv[pp][3]);
      }
      ++it;
    }
    if (!ok) { *abort_flag = 1; return; }

    // ---- merge the four warps' partial softmax states through the last stage
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    constexpr int kCols = D / 8;
    const int row = ct >> 3;  // query head within the group (output phase)
    const int c0 = (ct & 7) * kCols;
    const int h = hk * p.G + row;
    if (nblk == 0) {
      // no key at all: the output is zero
      if (row < p.G) {
        __nv_bfloat16* orow = p.o + b * p.so.b + t * p.so.t + (int64_t)h * p.so.h;
#pragma unroll
        for (int c = 0; c < kCols; c += 2)
          *reinterpret_cast<__nv_bfloat162*>(orow + c0 + c) = __floats2bfloat162_rn(0.f, 0.f);
      }
      continue;
    }
    float* mO = reinterpret_cast<float*>(stages + size_t(s_last) * L::kStage);
    if (lane == 0) mbar_arrive(mrg_read);
    if (!mbar_wait(mrg_read, nmrg & 1)) { *abort_flag = 1; return; }
    {
      float* myO = mO + wq * 16 * D;
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
        const int col = nt * 8 + tq * 2;
        *reinterpret_cast<float2*>(myO + gq * D + (col ^ ((gq & 7) << 3))) =
            make_float2(oacc[nt][0], oacc[nt][1]);
        *reinterpret_cast<float2*>(myO + (gq + 8) * D + (col ^ (((gq + 8) & 7) << 3))) =
            make_float2(oacc[nt][2], oacc[nt][3]);
      }
    }
    if (tq == 0) {
      myML[gq] = m0; myML[gq + 8] = m1;
      myML[16 + gq] = l0; myML[16 + gq + 8] = l1;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(mrg_written);
    if (!mbar_wait(mrg_written, nmrg & 1)) { *abort_flag = 1; return; }
    ++nmrg;
    if (row < p.G) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kSaConsumers; ++w) M = fmaxf(M, mergeML[w * 32 + row]);
      float wgt[kSaConsumers], Lsum = 0.f;
#pragma unroll
      for (int w = 0; w < kSaConsumers; ++w) {
        const float mw = mergeML[w * 32 + row];
        wgt[w] = (M == -INFINITY) ? 0.f : exp2f(mw - M);
        Lsum += wgt[w] * mergeML[w * 32 + 16 + row];
      }
      const float inv = Lsum > 0.f ? 1.0f / Lsum : 0.f;
      const __nv_bfloat16* gr = p.g ? p.g + b * p.sg.b + t * p.sg.t + (int64_t)h * p.sg.h : nullptr;
      __nv_bfloat16* orow = p.o + b * p.so.b + t * p.so.t + (int64_t)h * p.so.h;
#pragma unroll
      for (int c = 0; c < kCols; c += 2) {
        const int cc = (c0 + c) ^ ((row & 7) << 3);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int w = 0; w < kSaConsumers; ++w) {
          const float2 ow = *reinterpret_cast<const float2*>(mO + (w * 16 + row) * D + cc);
          a0 = fmaf(wgt[w], ow.x, a0);
          a1 = fmaf(wgt[w], ow.y, a1);
        }
        a0 *= inv;
        a1 *= inv;
        if (gr) {
          const __nv_bfloat162 gg = *reinterpret_cast<const __nv_bfloat162*>(gr + c0 + c);
          a0 *= sigmoidf_(__bfloat162float(gg.x));
          a1 *= sigmoidf_(__bfloat162float(gg.y));
        }
        *reinterpret_cast<__nv_bfloat162*>(orow + c0 + c) = __floats2bfloat162_rn(a0, a1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s_last]);
  }
}

// Writes the fp16 copy of a bf16 [B, T, H, D] tensor (contiguous [B, T, H, D]
// output) that the P.V MMAs read.  bf16 -> fp16 is exact for normal values
// below 65504 (8 significant bits fit in 11); values that would not survive
// (|x| >= 65536 in bf16, inf or NaN) raise SALA_ERR_RANGE.  Tiny values become
// fp16 subnormals (absolute error below 2^-25).
__global__ void __launch_bounds__(256)
to_f16_copy_kernel(const __nv_bfloat16* __restrict__ x, sala_strides s, int B, int T, int H,
                   int D, __half* __restrict__ y) {
  const int64_t rows = (int64_t)B * T * H;
  const int per_row = D / 8;
  uint32_t bad = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * per_row;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / per_row;
    const int c = (int)(i % per_row);
    const int h = (int)(row % H);
    const int64_t t = (row / H) % T;
    const int b = (int)(row / ((int64_t)H * T));
    const uint4 u = *reinterpret_cast<const uint4*>(x + b * s.b + t * s.t + h * s.h + 8 * c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t hv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      bad |= ((w[k] & 0x7fffu) >= 0x4780u) | (((w[k] >> 16) & 0x7fffu) >= 0x4780u);
      hv[k] = bf16x2_to_f16x2(w[k]);
    }
    *reinterpret_cast<uint4*>(y + i * 8) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) raise_device_error(SALA_ERR_RANGE);
}

}  // namespace sala
