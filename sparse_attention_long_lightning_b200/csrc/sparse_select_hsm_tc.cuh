// sparse_select_hsm_tc.cuh -- per-head softmax-normalised block scores on tcgen05.
//
// The per-head selection variant (MiniCPM-SALA tech-report mirror, section 02 (2): the
// selection score is left open; this variant softmax-normalises each query head's
// scores before the GQA group sums them):
//   s_{h,j}  = (1/sqrt(D)) q_{t,h} . Kbar_j          h in group(hk), n_init <= j <= c - n_local
//   p_{h,j}  = exp(s_{h,j} - m_h) / sum_{j'} exp(s_{h,j'} - m_h),   m_h = max_j s_{h,j}
//   score_j  = sum_{h in group(hk)} p_{h,j}
// written into the same fp32 score scratch as block_scores_hsm_kernel, from which
// topk_select_kernel picks the top-k.
//
// Design (sm_100a).  An item is R = 128 / G consecutive query rows of one KV head: its
// R x G (query row, head) pairs are the M = 128 rows of the MMAs, so TMEM lane l =
// (row l / G, head l % G) and each consumer thread owns one head of one row.  A TMA box
// of q [B, T, Hq, D] with G heads x R rows lands exactly in that order (the A operand,
// q as stored: bf16 is exact).  The block means (fp32) are split into three bf16 parts
// hi + mid + lo = Kbar exactly (8 significant bits each), so
//   S = q.lo + q.mid + q.hi
// (24 MMAs of N = 64 per 64-candidate tile at D = 128) is the fp32 dot product up to
// the accumulation order.  Every item is scored twice: pass 1 keeps each thread's
// running maximum and sum of exponentials (online, in registers: no cross-thread work),
// pass 2 recomputes S, forms p = exp(s - m) / l, and the G threads of a query row sum
// their heads' p by a butterfly reduce-scatter (after which lane g of the row's group
// holds the sums of candidates g * 64/G .. (g + 1) * 64/G - 1 of the tile) and store
// them, coalesced, into the scratch row.
//   issuer (warp 4, one thread): TMA of the items' q tiles (two A buffers) and of the
//     block-mean tiles (3-stage ring, hi / mid / lo), and the MMAs into one of 4 TMEM
//     score buffers, running ahead of the consumers by the ring depth;
//   consumers (warps 0-3): tcgen05.ld of a tile's 64 scores, buffer release (per-warp
//     arrival), then the pass's arithmetic.
// All waits are bounded: a wait that runs out raises SALA_ERR_TIMEOUT, and the kernel
// drains its copies and MMAs before it frees TMEM and returns.
#pragma once

#include "sparse_select.cuh"

namespace sala {

constexpr int kHtLanes = 128;   // (query row, head) pairs per item = TMEM lanes
constexpr int kHtN = 64;        // candidates per tile
constexpr int kHtStages = 3;    // block-mean tile ring
constexpr int kHtAcc = 4;       // TMEM score buffers
constexpr int kHtThreads = kHtLanes + 32;

template <int D>
struct HtSmem {
  static constexpr int kHalfB = kHtN * 128;         // 64 candidates x 64 dims, bf16
  static constexpr int kPartB = (D / 64) * kHalfB;  // one of hi / mid / lo
  static constexpr int kStage = 3 * kPartB;
  static constexpr int kAHalf = kHtLanes * 128;     // 128 lanes x 64 dims, bf16
  static constexpr int kA = (D / 64) * kAHalf;
  static constexpr size_t kB = 0;                                    // [stages]
  static constexpr size_t kAoff = kB + kHtStages * size_t(kStage);   // [2]
  static constexpr size_t kBars = kAoff + 2 * size_t(kA);
  // full[S], stage_free[S], mma_done[A], acc_free[A], a_full[2], a_free[2], drain
  static constexpr int kNumBars = 2 * kHtStages + 2 * kHtAcc + 4 + 1;
  static constexpr size_t bytes = 1024 + kBars + kNumBars * 8 + 16;
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
  int R, r0, r1, qpos0, nb, Hkv, hb, nitems, nrounds, n_init, n_local;
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
// entries g * kHtN / G .. (g + 1) * kHtN / G - 1 in s[0 ..].
template <int G, int N>
__device__ __forceinline__ void ht_reduce_scatter(float (&s)[kHtN], int lane) {
  if constexpr (G > 1) {
    constexpr int d = G / 2, half = N / 2;
    const bool upper = (lane & d) != 0;
#pragma unroll
    for (int x = 0; x < half; ++x) {
      const float send = upper ? s[x] : s[x + half];
      const float keep = upper ? s[x + half] : s[x];
      s[x] = keep + __shfl_xor_sync(0xffffffffu, send, d);
    }
    ht_reduce_scatter<d, half>(s, lane);
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kHtThreads, 1)
select_hsm_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_hi,
                     const __grid_constant__ CUtensorMap tm_mid,
                     const __grid_constant__ CUtensorMap tm_lo, float* __restrict__ scores,
                     const HtGeom geo, int rows_pass, float scale_log2) {
  using L = HtSmem<D>;
  constexpr int kK = D / 16;  // k-steps
  constexpr uint32_t kId = umma_idesc_bf16(128, kHtN, false, false);
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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < kHtStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&stage_free[i], 1);
    }
    for (int i = 0; i < kHtAcc; ++i) {
      mbar_init(&mma_done[i], 1);
      mbar_init(&acc_free[i], kHtLanes / 32);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_free[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(tmem_slot, kHtAcc * kHtN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tD = *tmem_slot;

  if (warp == 4) {
    // ================= issuer: TMA (q tiles, block-mean tiles) and the score MMAs
    if ((tid & 31) == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_hi);
      prefetch_tmap(&tm_mid);
      prefetch_tmap(&tm_lo);
      HtCursor tc, mc;  // TMA cursor (runs ahead), MMA cursor
      geo.begin(tc);
      geo.begin(mc);
      int g_tma = 0, g_mma = 0, a_loads = 0;
      bool ok = true;
      // issue the copies of the tile under the TMA cursor (and its item's q tile first)
      auto tma_step = [&]() -> bool {
        if (tc.pass == 0 && tc.i == 0) {
          const int buf = tc.u & 1;
          if (tc.u >= 2 && !mbar_wait(&a_free[buf], ((tc.u - 2) >> 1) & 1)) return false;
          uint8_t* dst = smem + L::kAoff + buf * L::kA;
          mbar_arrive_expect_tx(&a_full[buf], L::kA);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_4d(dst + hf * L::kAHalf, &tm_q, &a_full[buf], hf * 64, tc.hk * G, tc.t0,
                        tc.b);
          a_loads = tc.u + 1;
        }
        const int st = g_tma % kHtStages;
        if (g_tma >= kHtStages &&
            !mbar_wait(&stage_free[st], ((g_tma / kHtStages) + 1) & 1))
          return false;
        uint8_t* dst = smem + L::kB + st * L::kStage;
        const int j0 = geo.n_init + tc.i * kHtN;
        mbar_arrive_expect_tx(&full[st], L::kStage);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          tma_load_4d(dst + hf * L::kHalfB, &tm_hi, &full[st], hf * 64, tc.hk, j0, tc.b);
          tma_load_4d(dst + L::kPartB + hf * L::kHalfB, &tm_mid, &full[st], hf * 64, tc.hk, j0,
                      tc.b);
          tma_load_4d(dst + 2 * L::kPartB + hf * L::kHalfB, &tm_lo, &full[st], hf * 64, tc.hk,
                      j0, tc.b);
        }
        ++g_tma;
        geo.next(tc);
        return true;
      };
      auto desc = [&](uint32_t base, int kk, int half_bytes) {
        return umma_desc_sw128(base + (kk >> 2) * half_bytes + (kk & 3) * 32, 16, 1024);
      };
      for (int x = 0; x < kHtStages - 1 && tc.valid && ok; ++x) ok = tma_step();
      while (mc.valid && ok) {
        if (tc.valid) ok = tma_step();
        if (!ok) break;
        const int buf = mc.u & 1, st = g_mma % kHtStages, ab = g_mma % kHtAcc;
        if (mc.pass == 0 && mc.i == 0) ok = mbar_wait(&a_full[buf], (mc.u >> 1) & 1);
        ok = ok && mbar_wait(&full[st], (g_mma / kHtStages) & 1) &&
             (g_mma < kHtAcc || mbar_wait(&acc_free[ab], ((g_mma / kHtAcc) + 1) & 1));
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = smem_u32(smem + L::kAoff + buf * L::kA);
        const uint32_t bh = smem_u32(smem + L::kB + st * L::kStage);
        const uint32_t d = tD + kHtN * ab;
        // smallest part first: lo, mid, hi
#pragma unroll
        for (int kk = 0; kk < kK; ++kk)
          tc_mma_ss(d, desc(a, kk, L::kAHalf), desc(bh + 2 * L::kPartB, kk, L::kHalfB), kId,
                    kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kK; ++kk)
          tc_mma_ss(d, desc(a, kk, L::kAHalf), desc(bh + L::kPartB, kk, L::kHalfB), kId, 1u);
#pragma unroll
        for (int kk = 0; kk < kK; ++kk)
          tc_mma_ss(d, desc(a, kk, L::kAHalf), desc(bh, kk, L::kHalfB), kId, 1u);
        tc_commit(&mma_done[ab]);
        tc_commit(&stage_free[st]);
        const bool last_of_item = mc.pass == 1 && mc.i == mc.ntiles - 1;
        if (last_of_item) tc_commit(&a_free[buf]);
        ++g_mma;
        geo.next(mc);
      }
      if (!ok) *abort_flag = 1;
      // wind down: every MMA complete and every copy landed before TMEM is freed
      tc_commit(drain);
      mbar_wait(drain, 0);
      for (int x = g_tma > kHtStages ? g_tma - kHtStages : 0; x < g_tma; ++x)
        mbar_wait(&full[x % kHtStages], (x / kHtStages) & 1);
      for (int x = a_loads > 2 ? a_loads - 2 : 0; x < a_loads; ++x)
        mbar_wait(&a_full[x & 1], (x >> 1) & 1);
    }
  } else {
    // ================= consumers: thread l = (row l / G, head l % G) of the item
    const int l = tid;
    const int rrow = l / G, gl = l % G;  // row within the item, lane within the row's group
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    constexpr int per = kHtN / G;        // candidates each lane stores per tile
    HtCursor c;
    geo.begin(c);
    int g = 0;
    float m = -INFINITY, lsum = 0.f, inv_l = 0.f;
    while (c.valid) {
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
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      uint32_t sv[2][32];
      tc_ld32(tD + kHtN * ab + lane_off, sv[0]);
      tc_ld32(tD + kHtN * ab + 32 + lane_off, sv[1]);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&acc_free[ab]);
      const int j0 = geo.n_init + c.i * kHtN;
      float s[kHtN];
#pragma unroll
      for (int x = 0; x < kHtN; ++x) {
        const bool in = j0 + x <= jmax;
        s[x] = in ? __uint_as_float(sv[x >> 5][x & 31]) * scale_log2 : -INFINITY;
      }
      if (c.pass == 0) {
        float mt = -INFINITY;
#pragma unroll
        for (int x = 0; x < kHtN; ++x) mt = fmaxf(mt, s[x]);
        if (mt > -INFINITY) {
          const float mn = fmaxf(m, mt);
          float acc = 0.f;
#pragma unroll
          for (int x = 0; x < kHtN; ++x) acc += exp2f(s[x] - mn);  // exp2(-inf) = 0
          lsum = lsum * exp2f(m - mn) + acc;                       // 0 on the row's first tile
          m = mn;
        }
        if (c.i == c.ntiles - 1) inv_l = lsum > 0.f ? 1.0f / lsum : 0.f;
      } else {
        // p (0 for candidates outside the row, also when the row has none: m = -inf)
#pragma unroll
        for (int x = 0; x < kHtN; ++x) s[x] = s[x] == -INFINITY ? 0.f : exp2f(s[x] - m) * inv_l;
        ht_reduce_scatter<G, kHtN>(s, l);
        // lane gl of the row holds candidates j0 + gl * per .. j0 + gl * per + per - 1
        if (live) {
          float* srow = scores + (((int64_t)c.b * geo.Hkv + c.hk) * rows_pass + (t - geo.r0)) *
                                     (int64_t)geo.nb;
          const int jb = j0 + gl * per;
#pragma unroll
          for (int x = 0; x < kHtN; ++x)
            if (x < per && jb + x <= jmax) srow[jb + x - geo.n_init] = s[x];
        }
      }
      ++g;
      geo.next(c);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tc_dealloc(*tmem_slot, kHtAcc * kHtN);
  }
}

}  // namespace sala
