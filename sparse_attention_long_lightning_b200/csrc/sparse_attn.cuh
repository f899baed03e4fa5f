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
// that a pre-pass writes once, scaled by a power of two per (sequence, KV head)
// so that any bf16 V fits; fp32 accumulation), the online softmax runs per warp
// in registers with a lazily raised reference maximum (rescaling only when a
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
  const int* vexp;   // [B * Hkv]: exponent e of the fp16 copy of v (values times 2^-e)
  const int* vflag;  // [B * Hkv]: 1 when v is outlier-heavy (P V then runs on P's fp16
                     // high and low parts)
  sala_strides sq, sg, so;
  int n_sel, B, T, Hq, Hkv, G;  // T: query rows (q, g, o, idx); keys come by TMA
  float scale_log2;  // softmax scale * log2(e)
  int64_t rows;      // B * Hkv * T
  int64_t qpos0;     // sequence position of query row 0 (row t is position qpos0 + t)
  int nkb;           // key blocks, ceil(Tk / 64): block indices lie in [-1, nkb)
};

// A selected block j takes part in row t iff j >= 0 and its first key is <= t.  (Debug
// builds first check j against [-1, nkb): an index past the keys can only come from a
// corrupted selection; the release rule already skips it as not live.)
__device__ __forceinline__ bool sa_block_live(int j, int64_t t, int nkb) {
  return SALA_IN_BOUNDS(j >= -1 && j < nkb) && j >= 0 && (int64_t)j * kSaBlk <= t;
}

// The first row >= r, in r's class modulo `stride`, of a (sequence, KV head) that this
// variant handles: kPrecise rows belong to heads whose v is outlier-heavy (vflag set),
// the others to the rest.  Whole heads are skipped at once.
template <bool kPrecise>
__device__ __forceinline__ int64_t sa_next_row(int64_t r, int64_t stride, const SaParams& p) {
  while (r < p.rows) {
    const int64_t head = r / p.T;  // b * Hkv + hk
    if ((__ldg(p.vflag + head) != 0) == kPrecise) return r;
    const int64_t next = (head + 1) * p.T;
    r += (next - r + stride - 1) / stride * stride;
  }
  return r;
}

// kPrecise: the variant for heads whose v is outlier-heavy, where P V also takes P's
// fp16 rounding residual; the two variants are launched one after the other, each on its
// own heads, so the common one carries no cost for the other.
template <int D, int NS, bool kPrecise>
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
      const int64_t rstride = (int64_t)kSaGroups * gridDim.x;
      for (int64_t r = sa_next_row<kPrecise>(blockIdx.x + (int64_t)grp * gridDim.x, rstride, p);
           r < p.rows && ok; r = sa_next_row<kPrecise>(r + rstride, rstride, p)) {
        const int64_t t = r % T;
        const int64_t tp = p.qpos0 + t;  // the row's position
        const int hk = (int)((r / T) % p.Hkv);
        const int b = (int)(r / (T * p.Hkv));
        const int32_t* ir = p.idx + r * p.n_sel;
        for (int e = 0; e < p.n_sel; ++e) {
          const int j = __ldg(ir + e);
          if (!sa_block_live(j, tp, p.nkb)) continue;
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
  const int64_t rstride = (int64_t)kSaGroups * gridDim.x;
  for (int64_t r = sa_next_row<kPrecise>(blockIdx.x + (int64_t)grp * gridDim.x, rstride, p);
       r < p.rows; r = sa_next_row<kPrecise>(r + rstride, rstride, p)) {
    const int64_t t = r % T;
    const int64_t tp = p.qpos0 + t;  // the row's position
    const int hk = (int)((r / T) % p.Hkv);
    const int b = (int)(r / (T * p.Hkv));

    // number of live blocks of this row (the producer streams exactly these)
    int nblk = 0;
    {
      const int32_t* ir = p.idx + r * p.n_sel;
      for (int e0 = 0; e0 < p.n_sel; e0 += 32) {
        const int e = e0 + lane;
        const bool live = e < p.n_sel && sa_block_live(__ldg(ir + e), tp, p.nkb);
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
    constexpr bool precise = kPrecise;
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
      // ---- scale; causal mask only where the block reaches past the row's position
      const bool straddle = (int64_t)j * kSaBlk + kSaBlk - 1 > tp;
      const int64_t key0 = (int64_t)j * kSaBlk + wq * 16 + tq * 2;
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float x = sc[nt][c] * p.scale_log2;
          if (straddle && key0 + nt * 8 + (c & 1) > tp) x = -INFINITY;
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
      // P in fp16 (10-bit mantissa), V is the fp16 copy; for outlier-heavy v also P's
      // fp16 rounding residual
      uint32_t pa[4], pl[4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float p0 = exp2f(sc[nt][0] - mu0), p1 = exp2f(sc[nt][1] - mu0);
        const float p2 = exp2f(sc[nt][2] - mu1), p3 = exp2f(sc[nt][3] - mu1);
        l0 += p0 + p1;
        l1 += p2 + p3;
        pa[nt * 2 + 0] = pack_f16x2(p0, p1);
        pa[nt * 2 + 1] = pack_f16x2(p2, p3);
        if constexpr (precise) {
          const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&pa[nt * 2]));
          const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&pa[nt * 2 + 1]));
          pl[nt * 2 + 0] = pack_f16x2(p0 - h0.x, p1 - h0.y);
          pl[nt * 2 + 1] = pack_f16x2(p2 - h1.x, p3 - h1.y);
        }
      }
      // ---- O += P V
#pragma unroll
      for (int pp = 0; pp < kNT / 2; ++pp) {
        mma_f16_16816(oacc[2 * pp], pa, vv[pp][0], vv[pp][1]);
        mma_f16_16816(oacc[2 * pp + 1], pa, vv[pp][2], vv[pp][3]);
      }
      if constexpr (precise) {
#pragma unroll
        for (int pp = 0; pp < kNT / 2; ++pp) {
          mma_f16_16816(oacc[2 * pp], pl, vv[pp][0], vv[pp][1]);
          mma_f16_16816(oacc[2 * pp + 1], pl, vv[pp][2], vv[pp][3]);
        }
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
      // 1 / sum, times 2^e to undo the scale of the fp16 copy of v
      const float inv = Lsum > 0.f ? pow2i(__ldg(p.vexp + b * p.Hkv + hk)) / Lsum : 0.f;
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

// The fp16 copy of v that the P.V MMAs read, written once per call in two launches
// over grid (kVChunks, Hkv, B), each CTA covering rows [x T / kVChunks, (x + 1) T /
// kVChunks) of one (sequence, KV head):
//   v_absmax_kernel    the largest |v| of those rows -> part[(b Hkv + hk) kVChunks + x],
//                      their sum of v^2 -> part_ss[...];
//   to_f16_copy_kernel the (sequence, KV head)'s largest |v| from the partials, its
//                      exponent e (v_operand_exp: v 2^-e below 2^15, the largest above
//                      2^-4, e = 0 whenever fp16 holds the values as they are), the rows
//                      times 2^-e into the contiguous [B, T, Hkv, D] copy, and e itself
//                      (CTA x = 0) into vexp[b Hkv + hk], and vflag[b Hkv + hk] = 1 when
//                      the largest |v| exceeds kSaOutlierRatio x rms(v).  The attention
//                      epilogue multiplies by 2^e.  A non-finite v raises SALA_ERR_RANGE.
constexpr int kVChunks = 128;

__device__ __forceinline__ float bf16x8_absmax(const uint4& u, float m) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k)
    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[k] << 16)),
                       fabsf(__uint_as_float(w[k] & 0xffff0000u))));
  return m;
}

// Largest of `n` non-negative partial maxima (every thread of the CTA gets it); a NaN or
// infinite partial makes the result infinite.  Non-negative floats, +inf included, order
// as their bit patterns.
__device__ __forceinline__ float cta_max_of(const float* part, int n, float* red) {
  float m = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float x = part[i];
    m = x < INFINITY ? fmaxf(m, x) : INFINITY;
  }
  const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = __uint_as_float(mb);
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(256)
v_absmax_kernel(const __nv_bfloat16* __restrict__ x, sala_strides s, int T, int Hkv, int D,
                float* __restrict__ part, float* __restrict__ part_ss) {
  const int hk = blockIdx.y, b = blockIdx.z;
  const int64_t r0 = (int64_t)blockIdx.x * T / kVChunks, r1 = (int64_t)(blockIdx.x + 1) * T / kVChunks;
  const int per_row = D / 8;
  float m = 0.f, ss = 0.f;
  bool nonfinite = false;
  for (int64_t i = r0 * per_row + threadIdx.x; i < r1 * per_row; i += blockDim.x) {
    const int64_t t = i / per_row;
    const int c = (int)(i % per_row);
    const uint4 u = *reinterpret_cast<const uint4*>(x + b * s.b + t * s.t + hk * s.h + 8 * c);
    m = bf16x8_absmax(u, m);
    float f[8];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) ss = fmaf(f[k], f[k], ss);
    // inf or NaN: exponent field all ones in either half of any word
    nonfinite |= ((u.x & 0x7f80u) == 0x7f80u) | ((u.x & 0x7f800000u) == 0x7f800000u) |
                 ((u.y & 0x7f80u) == 0x7f80u) | ((u.y & 0x7f800000u) == 0x7f800000u) |
                 ((u.z & 0x7f80u) == 0x7f80u) | ((u.z & 0x7f800000u) == 0x7f800000u) |
                 ((u.w & 0x7f80u) == 0x7f80u) | ((u.w & 0x7f800000u) == 0x7f800000u);
  }
  __shared__ float red[8], red_ss[8];
  uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(nonfinite ? INFINITY : m));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((threadIdx.x & 31) == 0) {
    red[threadIdx.x >> 5] = __uint_as_float(mb);
    red_ss[threadIdx.x >> 5] = ss;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = 0.f, rs = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      r = fmaxf(r, red[w]);
      rs += red_ss[w];
    }
    part[((int64_t)b * Hkv + hk) * kVChunks + blockIdx.x] = r;
    part_ss[((int64_t)b * Hkv + hk) * kVChunks + blockIdx.x] = rs;
  }
}

// v of a (sequence, KV head) is outlier-heavy when its largest |v| exceeds this many times
// its rms: P's fp16 rounding (2^-11) times such a value can exceed 1e-2 of the output's
// rms, so P V also takes P's low part.
constexpr float kSaOutlierRatio = 16.0f;

__global__ void __launch_bounds__(256)
to_f16_copy_kernel(const __nv_bfloat16* __restrict__ x, sala_strides s, int T, int Hkv, int D,
                   const float* __restrict__ part, const float* __restrict__ part_ss,
                   int* __restrict__ vexp, int* __restrict__ vflag, __half* __restrict__ y) {
  const int hk = blockIdx.y, b = blockIdx.z;
  __shared__ float red[8];
  const float m = cta_max_of(part + ((int64_t)b * Hkv + hk) * kVChunks, kVChunks, red);
  if (!(m < INFINITY)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_device_error(SALA_ERR_RANGE);
  }
  const int e = v_operand_exp(m);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    vexp[(int64_t)b * Hkv + hk] = e;
    double ss = 0.0;
    for (int i = 0; i < kVChunks; ++i) ss += (double)part_ss[((int64_t)b * Hkv + hk) * kVChunks + i];
    const double rms = sqrt(ss / ((double)T * D));
    vflag[(int64_t)b * Hkv + hk] = (m < INFINITY) && (double)m > (double)kSaOutlierRatio * rms;
  }
  const float sc = pow2i(-e);
  const int64_t r0 = (int64_t)blockIdx.x * T / kVChunks, r1 = (int64_t)(blockIdx.x + 1) * T / kVChunks;
  const int per_row = D / 8;
  for (int64_t i = r0 * per_row + threadIdx.x; i < r1 * per_row; i += blockDim.x) {
    const int64_t t = i / per_row;
    const int c = (int)(i % per_row);
    const uint4 u = *reinterpret_cast<const uint4*>(x + b * s.b + t * s.t + hk * s.h + 8 * c);
    uint4 o;
    if (e == 0) {
      o = make_uint4(bf16x2_to_f16x2(u.x), bf16x2_to_f16x2(u.y), bf16x2_to_f16x2(u.z),
                     bf16x2_to_f16x2(u.w));
    } else {
      o = make_uint4(bf16x2_to_f16x2_scaled(u.x, sc), bf16x2_to_f16x2_scaled(u.y, sc),
                     bf16x2_to_f16x2_scaled(u.z, sc), bf16x2_to_f16x2_scaled(u.w, sc));
    }
    *reinterpret_cast<uint4*>(y + (((int64_t)b * T + t) * Hkv + hk) * D + 8 * c) = o;
  }
}

}  // namespace sala
