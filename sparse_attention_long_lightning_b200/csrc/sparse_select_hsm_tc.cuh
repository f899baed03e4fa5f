// sparse_select_hsm_tc.cuh -- per-head softmax-normalised block scores on tcgen05.
//
// The per-head selection variant (MiniCPM-SALA tech-report mirror, section 02 (2): the
// selection score is left open; this variant softmax-normalises each query head's
// scores before the GQA group sums them):
//   s_{h,j}  = (1/sqrt(D)) q_{t,h} . Kbar_j        h in group(hk), n_init <= j <= c - n_local
//   p_{h,j}  = exp(s_{h,j} - m_h) / sum_{j'} exp(s_{h,j'} - m_h),   m_h = max_j s_{h,j}
//   score_j  = sum_{h in group(hk)} p_{h,j}
// written into the fp32 score scratch from which topk_select_kernel picks the top-k.
//
// Design (sm_100a).  An item is R = 128 / G consecutive query rows of one KV head: its
// R x G (query row, head) pairs are the M = 128 rows of the MMAs, so TMEM lane l =
// (row l / G, head l % G) and each consumer thread owns one head of one row.  The A
// operand (q as stored: bf16 is exact) sits in TMEM, so the MMAs of a tile read only the
// block means from shared memory.  The block means times log2(e)/sqrt(D) (one fp32
// rounding: the scores come out in the log2 domain of the exponentials) are split into
// three bf16 parts hi + mid + lo = that value exactly (8 significant bits each).  A
// tile's three parts are stacked as the N = 192 rows of the B operand, so 8 MMAs
// (D = 128) give q.hi, q.mid and q.lo side by side in TMEM and the consumers form
// S = (q.lo + q.mid) + q.hi: the fp32 dot product up to the summation order (fewer,
// wider MMAs: each MMA instruction has a fixed cost that N = 64 products did not cover).
// Every item is scored twice: pass 1 keeps each thread's running maximum and sum of
// exponentials (online, in registers), pass 2 recomputes S, forms
// p = exp2(s - (m + log2 l)), and the G threads of a query row sum their heads' p by a
// butterfly reduce-scatter over the thread's 16 candidates (lane g of the row's group
// ends with the sums of 16 / G of them, or shares one with G / 16 - 1 other lanes when
// G = 32) and store them, coalesced, into the scratch row.
//   producers (warps 17-20): thread l loads lane l's query-head row of the next item
//     and stores it into its TMEM lane (two A buffers), overlapping the current item;
//   copier (warp 21, one thread): TMA of the block-mean tiles (4-stage ring, hi / mid /
//     lo per 64-dim half), running ahead by the ring depth;
//   issuer (warp 16, one thread): the MMAs of each tile into one of 2 TMEM score buffers;
//   consumers (warps 0-15): warps w, w + 4, w + 8, w + 12 read TMEM lane quadrant w % 4,
//     each one quarter (16 candidates) of every tile: tcgen05.ld, buffer release
//     (per-warp arrival), then the pass's arithmetic; at the end of pass 1 the four
//     threads of a lane merge their parts' (max, sum) through shared memory in a fixed
//     order (a bounded mbarrier wait, per item parity), so pass 2 normalises with the
//     row's full sum.
// All waits are bounded: a wait that runs out raises SALA_ERR_TIMEOUT, and the kernel
// drains its copies and MMAs before it frees TMEM and returns.
#pragma once

#include "sparse_select.cuh"

namespace sala {

constexpr int kHtLanes = 128;   // (query row, head) pairs per item = TMEM lanes
constexpr int kHtN = 64;        // candidates per tile
constexpr int kHtPart = kHtN / 4;  // candidates of a tile per consumer thread
constexpr int kHtStages = 4;    // block-mean tile ring
constexpr int kHtAcc = 2;       // TMEM score buffers (3 x kHtN columns each)
constexpr int kHtConsumers = 16; // four warps per TMEM lane quadrant (16 columns each)
constexpr int kHtThreads = kHtConsumers * 32 + 32 + kHtLanes + 32;  // consumers, issuer,
                                                                    // producers, copier
constexpr int kHtCopier = kHtConsumers + 1 + kHtLanes / 32;        // the copier's warp

// 2^x on the transcendental unit (relative error about 2^-22; subnormal results kept)
__device__ __forceinline__ float ht_exp2(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
struct HtSmem {
  static constexpr int kHalfB = kHtN * 128;         // 64 candidates x 64 dims, bf16
  static constexpr int kHalf3 = 3 * kHalfB;         // hi, mid, lo of one 64-dim half
  static constexpr int kStage = (D / 64) * kHalf3;
  static constexpr size_t kB = 0;                                    // [stages]
  static constexpr size_t kBars = kB + kHtStages * size_t(kStage);
  // full[S], stage_free[S], mma_done[A], acc_free[A], a_full[2], a_free[2], drain,
  // merged[4 quadrants][2 item parities]
  static constexpr int kNumBars = 2 * kHtStages + 2 * kHtAcc + 4 + 1 + 8;
  // [2 item parities][4 tile parts][128 lanes] x (max, sum): the four warps of a lane
  // quadrant combine their parts' running softmax state at the end of pass 1
  static constexpr size_t kComb = kBars + kNumBars * 8 + 16;
  static constexpr size_t need = 1024 + kComb + 2 * 4 * kHtLanes * 8;
  // at least half of the SM's shared memory, so that one CTA per SM holds all 512 TMEM
  // columns (a second CTA's allocation would wait for the first to finish)
  static constexpr size_t bytes = need > 120 * 1024 ? need : 120 * 1024;
  static_assert(bytes <= 232448, "fits one CTA per SM");
};

// Walks this CTA's (item, pass, tile) sequence: items in snake order over the long-rows-
// first list, items without candidates skipped, two passes per item.
struct HtCursor {
  int r, u, pass, i;        // round, scoring items so far (A buffer u & 1), pass, tile
  int t0, hk, b, ntiles;    // the current item
  bool valid;
};

struct HtGeom {
  int R, r0, r1, Tq, qpos0, nb, Hkv, hb, nitems, nrounds, n_init, n_local;
  __device__ int item_of(int r) const {
    return r * (int)gridDim.x + ((r & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
  }
  // fills t0 / hk / b / ntiles of item k (k < nitems)
  __device__ void info(int k, HtCursor& c) const {
    const int x = k / hb, rem = k % hb;
    const int ntile_rows = (r1 - r0 + R - 1) / R;
    c.t0 = r0 + (ntile_rows - 1 - x) * R;
    c.hk = rem % Hkv;
    c.b = rem / Hkv;
    const int t_last = qpos0 + min(c.t0 + R, r1) - 1;             // the item's last position
    const int jhi = min(t_last / kSelBlk - n_local, nb - 1);       // its last candidate
    c.ntiles = jhi >= n_init ? (jhi - n_init) / kHtN + 1 : 0;
  }
  // first tile of the first scoring item at or after round r
  __device__ void seek(HtCursor& c, int r) const {
    c.valid = false;
    for (; r < nrounds; ++r) {
      const int k = item_of(r);
      if (k >= nitems) continue;
      info(k, c);
      if (c.ntiles == 0) continue;
      c.r = r;
      c.pass = 0;
      c.i = 0;
      c.valid = true;
      return;
    }
  }
  __device__ void begin(HtCursor& c) const {
    c.u = 0;
    seek(c, 0);
  }
  __device__ void next(HtCursor& c) const {
    if (++c.i < c.ntiles) return;
    c.i = 0;
    if (++c.pass < 2) return;
    ++c.u;
    seek(c, c.r + 1);
  }
};

// Sum of the G lanes' values of one query row, scattered: each step at distance d
// (G / 2, G / 4, .., 1) adds the partner's half of the N values the lane still holds and
// keeps the half selected by (lane & d); lane g of the group ends with the sums of
// entries g * N / G .. (g + 1) * N / G - 1 in s[0 ..].
// When G > N the last steps have one value left: lanes d apart add theirs (both keep
// the sum), so lanes g and g ^ d .. hold the same entry (entry g * N / G rounded down).
template <int G, int N>
__device__ __forceinline__ void ht_reduce_scatter(float (&s)[kHtPart], int lane) {
  if constexpr (G > 1) {
    constexpr int d = G / 2;
    if constexpr (N > 1) {
      constexpr int half = N / 2;
      const bool upper = (lane & d) != 0;
#pragma unroll
      for (int x = 0; x < half; ++x) {
        const float send = upper ? s[x] : s[x + half];
        const float keep = upper ? s[x + half] : s[x];
        s[x] = keep + __shfl_xor_sync(0xffffffffu, send, d);
      }
      ht_reduce_scatter<d, half>(s, lane);
    } else {
      s[0] += __shfl_xor_sync(0xffffffffu, s[0], d);
      ht_reduce_scatter<d, 1>(s, lane);
    }
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kHtThreads, 1)
select_hsm_tc_kernel(const __nv_bfloat16* __restrict__ q, sala_strides sq,
                     const __grid_constant__ CUtensorMap tm_hi,
                     const __grid_constant__ CUtensorMap tm_mid,
                     const __grid_constant__ CUtensorMap tm_lo, float* __restrict__ scores,
                     const HtGeom geo, int rows_pass) {
  using L = HtSmem<D>;
  constexpr int kK = D / 16;  // k-steps
  constexpr uint32_t kId = umma_idesc_bf16(128, 3 * kHtN, false, false);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBars);  // [S] tile landed
  uint64_t* stage_free = full + kHtStages;                       // [S] tile's MMAs done
  uint64_t* mma_done = stage_free + kHtStages;                   // [A] scores ready
  uint64_t* acc_free = mma_done + kHtAcc;                        // [A] scores read
  uint64_t* a_full = acc_free + kHtAcc;                          // [2] q tile landed
  uint64_t* a_free = a_full + 2;                                 // [2] q tile's MMAs done
  uint64_t* drain = a_free + 2;                                  // every MMA done (exit)
  uint64_t* pair = drain + 1;                                    // [4][2] halves merged
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pair + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < kHtStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&stage_free[i], 1);
    }
    for (int i = 0; i < kHtAcc; ++i) {
      mbar_init(&mma_done[i], 1);
      mbar_init(&acc_free[i], kHtConsumers);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], kHtLanes);
      mbar_init(&a_free[i], 1);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&pair[i], 4 * 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  constexpr int kAcols = D / 2;  // TMEM columns of one A buffer (bf16 pairs)
  constexpr uint32_t kCols = 2 * kAcols + kHtAcc * 3 * kHtN <= 256 ? 256 : 512;
  static_assert(2 * kAcols + kHtAcc * 3 * kHtN <= 512, "TMEM columns");
  if (warp == 0) tc_alloc(tmem_slot, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tD = tmem + 2 * kAcols;  // [kHtAcc] x (hi, mid, lo) x kHtN columns

  if (warp == kHtCopier) {
    // ================= copier: block-mean tiles (hi, mid, lo per 64-dim half) by TMA
    if ((tid & 31) == 0) {
      prefetch_tmap(&tm_hi);
      prefetch_tmap(&tm_mid);
      prefetch_tmap(&tm_lo);
      HtCursor tc;
      geo.begin(tc);
      int g_tma = 0;
      bool ok = true;
      while (tc.valid && ok) {
        const int st = g_tma % kHtStages;
        if (*abort_flag ||
            (g_tma >= kHtStages && !mbar_wait(&stage_free[st], ((g_tma / kHtStages) + 1) & 1))) {
          ok = false;
          break;
        }
        uint8_t* dst = smem + L::kB + st * L::kStage;
        const int j0 = geo.n_init + tc.i * kHtN;
        mbar_arrive_expect_tx(&full[st], L::kStage);
        // per 64-dim half: hi, mid, lo (B operand rows 0-63, 64-127, 128-191)
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          uint8_t* h3 = dst + hf * L::kHalf3;
          tma_load_4d(h3, &tm_hi, &full[st], hf * 64, tc.hk, j0, tc.b);
          tma_load_4d(h3 + L::kHalfB, &tm_mid, &full[st], hf * 64, tc.hk, j0, tc.b);
          tma_load_4d(h3 + 2 * L::kHalfB, &tm_lo, &full[st], hf * 64, tc.hk, j0, tc.b);
        }
        ++g_tma;
        geo.next(tc);
      }
      if (!ok) *abort_flag = 1;
      // every copy landed before the CTA releases its shared memory
      for (int x = g_tma > kHtStages ? g_tma - kHtStages : 0; x < g_tma; ++x)
        mbar_wait(&full[x % kHtStages], (x / kHtStages) & 1);
    }
  } else if (warp == kHtConsumers) {
    // ================= issuer: the score MMAs of each tile
    if ((tid & 31) == 0) {
      HtCursor mc;
      geo.begin(mc);
      int g_mma = 0;
      bool ok = true;
      auto desc = [&](uint32_t base, int kk, int half_bytes) {
        return umma_desc_sw128(base + (kk >> 2) * half_bytes + (kk & 3) * 32, 16, 1024);
      };
      while (mc.valid && ok) {
        const int buf = mc.u & 1, st = g_mma % kHtStages, ab = g_mma % kHtAcc;
        if (mc.pass == 0 && mc.i == 0) ok = !*abort_flag && mbar_wait(&a_full[buf], (mc.u >> 1) & 1);
        ok = ok && mbar_wait(&full[st], (g_mma / kHtStages) & 1) &&
             (g_mma < kHtAcc || mbar_wait(&acc_free[ab], ((g_mma / kHtAcc) + 1) & 1));
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = tmem + buf * kAcols;  // A in TMEM: k-step kk at columns 8 kk
        const uint32_t bh = smem_u32(smem + L::kB + st * L::kStage);
        const uint32_t d = tD + 3 * kHtN * ab;
#pragma unroll
        for (int kk = 0; kk < kK; ++kk)
          tc_mma_ts(d, a + 8 * kk, desc(bh, kk, L::kHalf3), kId, kk > 0 ? 1u : 0u);
        tc_commit(&mma_done[ab]);
        tc_commit(&stage_free[st]);
        const bool last_of_item = mc.pass == 1 && mc.i == mc.ntiles - 1;
        if (last_of_item) tc_commit(&a_free[buf]);
        ++g_mma;
        geo.next(mc);
      }
      if (!ok) *abort_flag = 1;
      // wind down: every MMA complete before TMEM is freed
      tc_commit(drain);
      mbar_wait(drain, 0);
    }
  } else if (warp > kHtConsumers) {
    // ================= producers (warps 9-12): lane l's query-head row of each item into its TMEM lane
    const int l = 32 * (warp & 3) + (tid & 31);  // this warp's TMEM lane quadrant is warp % 4
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int rrow = l / G, head = l % G;
    HtCursor c;
    geo.begin(c);
    while (c.valid) {
      const int buf = c.u & 1;
      if (*abort_flag || (c.u >= 2 && !mbar_wait(&a_free[buf], ((c.u - 2) >> 1) & 1))) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int t = c.t0 + rrow;
      const bool in = t < geo.Tq;
      const __nv_bfloat16* qp = q + c.b * sq.b + (int64_t)(in ? t : 0) * sq.t +
                                (int64_t)(c.hk * G + head) * sq.h;
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        uint32_t w[32];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const uint4 v = in ? __ldg(reinterpret_cast<const uint4*>(qp + hf * 64 + 8 * x))
                             : make_uint4(0u, 0u, 0u, 0u);
          w[4 * x] = v.x;
          w[4 * x + 1] = v.y;
          w[4 * x + 2] = v.z;
          w[4 * x + 3] = v.w;
        }
        tc_st32(tmem + buf * kAcols + 32 * hf + lane_off, w);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&a_full[buf]);
      // the next scoring item
      c.pass = 1;
      c.i = c.ntiles - 1;
      geo.next(c);
    }
  } else {
    // ================= consumers: thread (l, part) with l = (row l / G, head l % G)
    const int quad = warp & 3, part = warp >> 2;
    const int l = 32 * quad + (tid & 31);
    const int rrow = l / G, gl = l % G;  // row within the item, lane within the row's group
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    // after the reduce-scatter: `per` sums per lane, shared by `rep` lanes
    constexpr int per = kHtPart / G > 0 ? kHtPart / G : 1;
    constexpr int rep = G / kHtPart > 0 ? G / kHtPart : 1;
    float2* comb = reinterpret_cast<float2*>(smem + L::kComb);  // [parity][part][lane]
    HtCursor c;
    geo.begin(c);
    int g = 0;
    float m = -INFINITY, lsum = 0.f, mp = -INFINITY;
    bool ok = true;
    while (c.valid && ok) {
      const int t = c.t0 + rrow;                      // query row (local)
      const bool live = t < geo.r1;
      const int cblk = (geo.qpos0 + t) / kSelBlk;
      const int jmax = live ? min(cblk - geo.n_local, geo.nb - 1) : geo.n_init - 1;
      if (c.pass == 0 && c.i == 0) {
        m = -INFINITY;
        lsum = 0.f;
      }
      const int ab = g % kHtAcc;
      const bool landed = !*abort_flag && mbar_wait(&mma_done[ab], (g / kHtAcc) & 1);
      if (__any_sync(0xffffffffu, !landed)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sh[kHtPart], sm[kHtPart], sl[kHtPart];  // q.hi, q.mid, q.lo
      const uint32_t col = tD + 3 * kHtN * ab + kHtPart * part + lane_off;
      tc_ld16(col, sh);
      tc_ld16(col + kHtN, sm);
      tc_ld16(col + 2 * kHtN, sl);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&acc_free[ab]);
      const int j0 = geo.n_init + c.i * kHtN + kHtPart * part;  // this part's first candidate
      float s[kHtPart];  // scores, log2 domain (-inf: not a candidate of the row)
#pragma unroll
      for (int x = 0; x < kHtPart; ++x)
        s[x] = (__uint_as_float(sl[x]) + __uint_as_float(sm[x])) + __uint_as_float(sh[x]);
      if (j0 + kHtPart - 1 > jmax) {  // the row's candidates end inside this part
#pragma unroll
        for (int x = 0; x < kHtPart; ++x) s[x] = j0 + x <= jmax ? s[x] : -INFINITY;
      }
      if (c.pass == 0) {
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int x = 0; x < kHtPart; ++x) mx[x & 3] = fmaxf(mx[x & 3], s[x]);
        const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        if (mt > -INFINITY) {
          const float mn = fmaxf(m, mt);
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int x = 0; x < kHtPart; ++x) acc[x & 3] += ht_exp2(s[x] - mn);  // exp2(-inf) = 0
          lsum = lsum * ht_exp2(m - mn) + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
          m = mn;
        }
        if (c.i == c.ntiles - 1) {
          // merge the four parts' (max, sum) of the same lane, in part order (so the
          // four threads compute the same values)
          const int par = c.u & 1;
          comb[(par * 4 + part) * kHtLanes + l] = make_float2(m, lsum);
          mbar_arrive(&pair[quad * 2 + par]);
          const bool merged = mbar_wait(&pair[quad * 2 + par], (c.u >> 1) & 1);
          if (__any_sync(0xffffffffu, !merged)) {  // leave the loop as a whole warp
            ok = false;
            break;
          }
          float2 o[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) o[q4] = comb[(par * 4 + q4) * kHtLanes + l];
          const float ma = fmaxf(fmaxf(o[0].x, o[1].x), fmaxf(o[2].x, o[3].x));
          float la = 0.f;
          if (ma != -INFINITY) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) la += o[q4].y * ht_exp2(o[q4].x - ma);
          }
          // p = exp2(s - ma) / la = exp2(s - mp); -inf marks a row without candidates
          mp = la > 0.f ? ma + log2f(la) : -INFINITY;
        }
      } else {
        // p (exp2(-inf) = 0 for candidates outside the row; all 0 for a row without any)
        if (mp == -INFINITY) {
#pragma unroll
          for (int x = 0; x < kHtPart; ++x) s[x] = 0.f;
        } else {
#pragma unroll
          for (int x = 0; x < kHtPart; ++x) s[x] = ht_exp2(s[x] - mp);
        }
        ht_reduce_scatter<G, kHtPart>(s, l);
        // lane gl of the row holds candidates j0 + (gl / rep) * per .. + per - 1 (the
        // first of each `rep` lanes that share them stores)
        if (live && gl % rep == 0) {
          float* srow = scores + (((int64_t)c.b * geo.Hkv + c.hk) * rows_pass + (t - geo.r0)) *
                                     (int64_t)geo.nb;
          const int jb = j0 + (gl / rep) * per;
#pragma unroll
          for (int x = 0; x < per; ++x)
            if (jb + x <= jmax &&
                SALA_IN_BOUNDS(jb + x - geo.n_init < geo.nb && t - geo.r0 < rows_pass))
              srow[jb + x - geo.n_init] = s[x];
        }
      }
      ++g;
      geo.next(c);
    }
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tc_dealloc(tmem, kCols);
  }
}

}  // namespace sala
