// sparse_select_tc.cuh -- block selection on tcgen05, one query row per TMEM lane.
//
// Same selection as sparse_select.cuh (InfLLM-v2 style, MiniCPM-SALA tech-report
// mirror, section 02 (2); summary page, "Prerequisites / Sparse Attention"):
//   score_j = (1/sqrt(D)) (sum_{h in group(hk)} q_{t,h}) . Kbar_j  over the candidates
//   n_init <= j <= c - n_local, top `topk` (larger score first, ties -> smaller j),
//   plus the init blocks and the local window, sorted, -1 padded.
//
// Design (sm_100a).  A work item is 128 consecutive query rows (two query blocks) of
// one KV head; the 128 rows are the M dimension of tcgen05 MMAs, so TMEM lane = query
// row.  CTAs are persistent (one per SM) and take items in a snake order over the
// long-rows-first item list.  Each CTA has two warpgroups:
//   producers (warps 4-7): thread p sums the group's queries of row p in fp32, splits
//     the sum into bf16 high / low parts and stores them to its TMEM lane: the A
//     operand of the NEXT item (two A buffers), so the query reads overlap the scan;
//   issuer (warp 8, one thread): streams 64-candidate tiles of the block means (bf16
//     high / low, written by block_means_kernel) through a 2-stage shared-memory ring
//     by TMA and issues S = qs_lo.Kb_hi + qs_hi.Kb_lo + qs_hi.Kb_hi (24 MMAs of N = 64:
//     the MMA issue, not the data, paces the pipeline) into one of 4 fp32 TMEM score
//     buffers;
//   consumers (warps 0-3): thread r reads its row's 64 scores of a tile, releases the
//     score buffer (per-warp arrival, so the warps run decoupled) and appends the
//     scores above its row threshold to a per-row buffer (shared memory, block order).
// When a buffer could overflow on the next tile, the rows of that warp compact their
// buffers (each thread its own row, in step): the topk-th best is located by bucketing
// the scores' order-preserving integer keys (64 bins per pass, counted with shared
// atomics; the bin holding the boundary is refined until it is resolved), then the
// kept entries are packed in place, which preserves block order.  The threshold becomes the smallest kept score:
// a later candidate with an equal score has a larger block index and loses the tie.
// At the end each row's buffer is compacted to topk and written out as it stands.
#pragma once

#include "sparse_select.cuh"

namespace sala {

constexpr int kStcRows = 128;   // query rows per item (= TMEM lanes = consumer threads)
constexpr int kStcN = 64;       // candidates per tile (per MMA: fewer, wider MMAs per candidate)
constexpr int kStcSub = 32;     // candidates appended between buffer checks
constexpr int kStcCap = 194;    // buffered candidates per row
constexpr int kStcBins = 64;    // histogram bins per compaction pass
constexpr int kStcStages = 2;   // block-mean tile ring
constexpr int kStcAcc = 4;      // TMEM score buffers
constexpr int kStcCoarse = 150;  // entries a compaction during the scan may keep
constexpr int kStcIssuers = 2;  // threads issuing score MMAs (alternate tiles)
constexpr int kStcThreads = 2 * kStcRows + 32 * kStcIssuers;  // consumers, producers, issuers

template <int D>
struct StcSmem {
  static constexpr int kHalfB = kStcN * 128;                 // kStcN rows x 64 dims bf16
  static constexpr int kTileB = (D / 64) * kHalfB;           // one hi or lo tile
  static constexpr int kStage = 2 * kTileB;                  // hi then lo
  static constexpr size_t kB = 0;                                     // [stages]
  static constexpr size_t kBufS = kB + kStcStages * size_t(kStage);   // [entry][row] f32
  static constexpr size_t kBufJ = kBufS + size_t(kStcCap) * kStcRows * 4;  // [entry][row] u16
  // [bin][row % 64] u32, rows r and r + 64 in the low / high 16 bits
  static constexpr size_t kHist = kBufJ + size_t(kStcCap) * kStcRows * 2;
  static constexpr size_t kBars = kHist + size_t(kStcBins) * 64 * 4;
  static constexpr int kNumBars = 2 * kStcStages + 2 * kStcAcc + 4 + 1;
  // full[S], stage_free[S], mma_done[A], acc_free[A], a_full[2], a_free[2], drain;
  // then the tmem slot and the abort flag
  static constexpr size_t bytes = 1024 + kBars + kNumBars * 8 + 8;
  static_assert(bytes <= 232448, "fits one CTA per SM");
};

// Compact one row's m > k buffered entries (shared addresses: sA / jA the scores (f32)
// and block indices (u16), entry e at + e * kStcRows * size; hA the row's 64 histogram
// bins for the rare key refinement, bin b in the 16 bits at `sh16` of the word at
// hA + b * 256), in buffer order.  smin / smax: the smallest and largest buffered score.
// Every entry among the k best (larger score first, ties -> smaller block index) is
// kept; with keep_max == k exactly those are kept, with keep_max > k a coarser cut that
// keeps at most keep_max entries may be taken instead.  Returns the kept count and sets
// *thr to the smallest kept score.
//
// Each score gets a fine index f in [0, 65536) linear in (s - smin), monotone in s.  Up
// to four counting passes of 16 bins (f's bits 15-12, then 11-8 inside the boundary bin,
// and so on), each histogram held in two 64-bit registers of 8-bit counters, locate the
// cell holding the k-th best, stopping as soon as the cut is resolved (or, for a coarse
// cut, small enough).  If the final cell still holds more entries than needed, their
// order-preserving integer keys are bucketed (64 bins in shared memory, refined until
// the boundary is resolved or only equal scores remain, where the earliest = smallest
// block index win).
__device__ __noinline__ int stc_compact(uint32_t sA, uint32_t jA, uint32_t hA, int sh16, int m,
                                        int k, float smin, float smax, int keep_max, float* thr) {
  constexpr uint32_t kSs = kStcRows * 4, kJs = kStcRows * 2, kHs = 64 * 4;  // strides
  constexpr int kU = 8;  // loads in flight per pass
  const float range = smax - smin;
  const float scale = 65536.0f / range;
  const bool linear = range > 0.f && scale <= 3.0e38f;
  auto fine_of = [&](float s) { return linear ? min(65535, (int)((s - smin) * scale)) : 0; };

  // ---- fine-index levels: bin = (f >> sh) & 15 among entries with f >> (sh + 4) == prefix
  int need = k, kept = 0, prefix = 0, cut_sh = 0, c = m;
  bool done = false;
#pragma unroll 1
  for (int sh = 12; sh >= 0; sh -= 4) {
    uint32_t h[4] = {0u, 0u, 0u, 0u};  // bin b in byte b % 4 of h[b / 4] (m <= 255)
    for (int e0 = 0; e0 < m; e0 += kU) {
      float v[kU];
#pragma unroll
      for (int x = 0; x < kU; ++x) v[x] = lds_f32(sA + min(e0 + x, m - 1) * kSs);
#pragma unroll
      for (int x = 0; x < kU; ++x) {
        const int f = fine_of(v[x]);
        const int bin = (f >> sh) & 15;
        const bool in = (e0 + x < m) & ((f >> (sh + 4)) == prefix);
        const uint32_t inc = (uint32_t)in << ((bin & 3) * 8);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] += (bin >> 2) == i ? inc : 0u;
      }
    }
    // bin holding the need-th best, from the top (selects, no branches)
    int above = 0, b = 0, cb_at = 0;
    bool found = false;
#pragma unroll
    for (int bb = 15; bb >= 0; --bb) {
      const int cb = (int)((h[bb >> 2] >> ((bb & 3) * 8)) & 0xffu);
      const bool take = !found & ((above + cb >= need) | (bb == 0));
      b = take ? bb : b;
      cb_at = take ? cb : cb_at;
      above += (!found & !take) ? cb : 0;
      found = found | take;
    }
    need -= above;
    kept += above;
    c = cb_at;
    prefix = prefix * 16 + b;
    if (c == need || kept + c <= keep_max) {  // keep every cell from `prefix` up
      cut_sh = sh;
      done = true;
      break;
    }
  }
  const int fcut = done ? prefix - 1 : prefix;  // keep (f >> cut_sh) > fcut (+ ties below)

  int w = 0;
  float mn = INFINITY;
  if (done) {
    // ---- pack (common path): keep f >> cut_sh > fcut; every store goes to an entry at or
    // below the ones already loaded
    for (int e0 = 0; e0 < m; e0 += kU) {
      float v[kU];
      uint32_t jv[kU];
#pragma unroll
      for (int x = 0; x < kU; ++x) {
        const int e = min(e0 + x, m - 1);
        v[x] = lds_f32(sA + e * kSs);
        jv[x] = lds_u16(jA + e * kJs);
      }
#pragma unroll
      for (int x = 0; x < kU; ++x) {
        const bool keep = (e0 + x < m) & ((fine_of(v[x]) >> cut_sh) > fcut);
        sts_f32_if(keep, sA + w * kSs, v[x]);
        sts_u16_if(keep, jA + w * kJs, jv[x]);
        w += keep ? 1 : 0;
        mn = keep ? fminf(mn, v[x]) : mn;
      }
    }
  } else {
    // ---- the final fine cell holds near-equal scores: bucket their keys
    const uint32_t other = sh16 ? 0x0000ffffu : 0xffff0000u;
    const uint32_t one = 1u << sh16;
    const int fs = prefix;
    uint32_t kl = 0xffffffffu, kh = 0u;
    for (int e = 0; e < m; ++e) {
      const float v = lds_f32(sA + e * kSs);
      if (fine_of(v) == fs) {
        kl = min(kl, order_key(v));
        kh = max(kh, order_key(v));
      }
    }
    int inplay = c;
    while (inplay > need && kl < kh) {
      const uint32_t span = kh - kl;
      const int sh = span < (uint32_t)kStcBins ? 0 : 32 - __clz(span) - 6;  // span >> sh < 64
      const int top = (int)(span >> sh);
      for (int bb = 0; bb <= top; ++bb) red_and_shared(hA + bb * kHs, other);
      for (int e = 0; e < m; ++e) {
        const float v = lds_f32(sA + e * kSs);
        const uint32_t key = order_key(v);
        if (fine_of(v) == fs && key >= kl && key <= kh)
          red_add_shared(hA + ((key - kl) >> sh) * kHs, one);
      }
      int above = 0, b = top;
      for (; b > 0; --b) {
        const int cb = (int)((lds_u32(hA + b * kHs) >> sh16) & 0xffffu);
        if (above + cb >= need) break;
        above += cb;
      }
      need -= above;
      inplay = (int)((lds_u32(hA + b * kHs) >> sh16) & 0xffffu);
      const uint32_t lo = kl + ((uint32_t)b << sh);
      const uint32_t width = (1u << sh) - 1u;
      kh = (kh - lo <= width) ? kh : lo + width;
      kl = lo;
    }
    // keep f > fs; at f == fs keys above kh, then the first `need` keys in [kl, kh]
    int taken = 0;
    for (int e = 0; e < m; ++e) {
      const float v = lds_f32(sA + e * kSs);
      const uint32_t j = lds_u16(jA + e * kJs);
      const int f = fine_of(v);
      const uint32_t key = order_key(v);
      bool keep = f > fs;
      if (!keep && f == fs) {
        if (key > kh) {
          keep = true;
        } else if (key >= kl && taken < need) {
          keep = true;
          ++taken;
        }
      }
      if (keep) {
        sts_f32(sA + w * kSs, v);
        sts_u16(jA + w * kJs, j);
        ++w;
        mn = fminf(mn, v);
      }
    }
  }
  *thr = mn;
  return w;
}

template <int D>
__global__ void __launch_bounds__(kStcThreads, 1)
select_tc_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
                 const __nv_bfloat16* __restrict__ q, int32_t* __restrict__ idx, int T, int qpos0,
                 int nb, int Hkv, int B, int G, sala_strides sq, int topk, int n_init,
                 int n_local) {
  using L = StcSmem<D>;
  constexpr int kK = D / 16;     // k-steps
  constexpr int kAcols = D / 2;  // TMEM columns of one A operand (bf16 pairs)
  constexpr uint32_t kId = umma_idesc_bf16(128, kStcN, false, false);
  constexpr uint32_t kCols = 4 * kAcols + kStcAcc * kStcN <= 256 ? 256 : 512;
  static_assert(4 * kAcols + kStcAcc * kStcN <= 512, "TMEM columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBars);  // [S] tile landed
  uint64_t* stage_free = full + kStcStages;                      // [S] tile's MMAs done
  uint64_t* mma_done = stage_free + kStcStages;                  // [A] scores ready
  uint64_t* acc_free = mma_done + kStcAcc;                       // [A] scores read
  uint64_t* a_full = acc_free + kStcAcc;                         // [2] queries in TMEM
  uint64_t* a_free = a_full + 2;                                 // [2] queries consumed
  uint64_t* drain = a_free + 2;                                  // every MMA done (exit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1) + 1;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int nq2 = (T + kStcRows - 1) / kStcRows;
  const int hb = Hkv * B;
  const int nitems = nq2 * hb;
  const int nrounds = (nitems + (int)gridDim.x - 1) / (int)gridDim.x;
  const int n_sel = n_init + topk + n_local;
  // item of round r for this CTA (snake order over the long-rows-first item list)
  auto item_of = [&](int r) {
    return r * (int)gridDim.x + ((r & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
  };
  struct Item {
    int t0, hk, b, ntiles;
  };
  auto info = [&](int k) {
    Item it;
    const int x = k / hb, rem = k % hb;
    it.t0 = (nq2 - 1 - x) * kStcRows;
    it.hk = rem % Hkv;
    it.b = rem / Hkv;
    const int t_last = qpos0 + min(it.t0 + kStcRows - 1, T - 1);  // the item's last position
    const int jhi = min(t_last / kSelBlk - n_local, nb - 1);  // last candidate of the item
    const int n_item = jhi >= n_init ? jhi - n_init + 1 : 0;
    it.ntiles = n_item > topk ? (n_item + kStcN - 1) / kStcN : 0;  // 0: nothing to score
    return it;
  };

  if (tid == 0) {
    for (int i = 0; i < kStcStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&stage_free[i], 1);
    }
    for (int i = 0; i < kStcAcc; ++i) {
      mbar_init(&mma_done[i], 1);
      mbar_init(&acc_free[i], kStcRows / 32);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], kStcRows);
      mbar_init(&a_free[i], kStcIssuers);
    }
    mbar_init(drain, kStcIssuers);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(tmem_slot, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tD = tmem + 4 * kAcols;  // [kStcAcc] x 32 columns of scores

  if (warp >= 4 && warp < 8) {
    // ================= producers: group-summed queries of the CTA's scoring items
    const int p = tid - kStcRows;
    const uint32_t lane_off = (uint32_t)(32 * (warp - 4)) << 16;
    int u = 0;
    for (int r = 0; r < nrounds; ++r) {
      const int k = item_of(r);
      if (k >= nitems) continue;
      const Item it = info(k);
      if (it.ntiles == 0) continue;
      const int buf = u & 1;
      if (*abort_flag || (u >= 2 && !mbar_wait(&a_free[buf], ((u - 2) >> 1) & 1))) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tA = tmem + buf * 2 * kAcols;
      const int t = it.t0 + p;
      const bool in = t < T;
      const __nv_bfloat16* qp = q + it.b * sq.b + (int64_t)(in ? t : 0) * sq.t +
                                (int64_t)it.hk * G * sq.h;
#pragma unroll 1
      for (int half = 0; half < D / 64; ++half) {
        float acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = 0.f;
        const __nv_bfloat16* base = qp + half * 64;
#pragma unroll 2
        for (int h = 0; h < G; ++h) {
          uint4 w[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            w[c] = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)h * sq.h + 8 * c));
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t ww[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc[8 * c + 2 * i] += __uint_as_float(ww[i] << 16);
              acc[8 * c + 2 * i + 1] += __uint_as_float(ww[i] & 0xffff0000u);
            }
          }
        }
        uint32_t hw[32], lw[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x0 = in ? acc[2 * i] : 0.f, x1 = in ? acc[2 * i + 1] : 0.f;
          const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
          const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
          hw[i] = pack_bf16x2(h0, h1);
          lw[i] = pack_bf16x2(x0 - h0, x1 - h1);
        }
        tc_st32(tA + lane_off + 32 * half, hw);
        tc_st32(tA + kAcols + lane_off + 32 * half, lw);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&a_full[buf]);
      ++u;
    }
  } else if (warp >= 8) {
    // ================= issuers: block-mean tiles by TMA (issuer 0), score MMAs (issuer
    // iss takes the tiles gg with gg % kStcIssuers == iss: its own stages and buffers)
    const int iss = warp - 8;
    if ((tid & 31) == 0) {
      if (iss == 0) {
        prefetch_tmap(&tm_hi);
        prefetch_tmap(&tm_lo);
      }
      int g = 0, u = 0, n_issued = 0;
      bool ok = true;
      // tile i of `it` as global tile gg, into stage gg % S once that stage's previous
      // tile has been scored
      auto issue_tma = [&](const Item& it, int i, int gg) {
        const int st = gg % kStcStages;
        if (gg >= kStcStages && !mbar_wait(&stage_free[st], ((gg / kStcStages) + 1) & 1))
          return false;
        uint8_t* dst = smem + L::kB + st * L::kStage;
        const int j0 = n_init + i * kStcN;
        mbar_arrive_expect_tx(&full[st], L::kStage);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          tma_load_4d(dst + hf * L::kHalfB, &tm_hi, &full[st], hf * 64, it.hk, j0, it.b);
          tma_load_4d(dst + L::kTileB + hf * L::kHalfB, &tm_lo, &full[st], hf * 64, it.hk, j0,
                      it.b);
        }
        n_issued = gg + 1;
        return true;
      };
      auto desc_b = [&](uint32_t base, int kk) {
        return umma_desc_sw128(base + (kk >> 2) * L::kHalfB + (kk & 3) * 32, 16, 1024);
      };
      for (int r = 0; r < nrounds && ok; ++r) {
        const int k = item_of(r);
        if (k >= nitems) continue;
        const Item it = info(k);
        if (it.ntiles == 0) continue;
        const int buf = u & 1;
        const uint32_t tA = tmem + buf * 2 * kAcols;
        ok = !*abort_flag;
        // the first S - 1 tiles; tile i + S - 1 follows the MMAs of tile i below
        for (int x = 0; iss == 0 && x < kStcStages - 1 && x < it.ntiles && ok; ++x)
          ok = issue_tma(it, x, g + x);
        ok = ok && mbar_wait(&a_full[buf], (u >> 1) & 1);
        tc_fence_after();
        for (int i = 0; i < it.ntiles && ok; ++i) {
          const int gg = g + i, st = gg % kStcStages, ab = gg % kStcAcc;
          if (gg % kStcIssuers != iss) {
            // another issuer's tile; issuer 0 still refills the stage of tile gg - 1
            if (iss == 0 && i + kStcStages - 1 < it.ntiles)
              ok = issue_tma(it, i + kStcStages - 1, gg + kStcStages - 1);
            continue;
          }
          ok = mbar_wait(&full[st], (gg / kStcStages) & 1) &&
               (gg < kStcAcc || mbar_wait(&acc_free[ab], ((gg / kStcAcc) + 1) & 1));
          if (!ok) break;
          tc_fence_after();
          const uint32_t bh = smem_u32(smem + L::kB + st * L::kStage), bl = bh + L::kTileB;
          const uint32_t d = tD + kStcN * ab;
#pragma unroll
          for (int kk = 0; kk < kK; ++kk)
            tc_mma_ts(d, tA + kAcols + 8 * kk, desc_b(bh, kk), kId, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kK; ++kk) tc_mma_ts(d, tA + 8 * kk, desc_b(bl, kk), kId, 1u);
#pragma unroll
          for (int kk = 0; kk < kK; ++kk) tc_mma_ts(d, tA + 8 * kk, desc_b(bh, kk), kId, 1u);
          tc_commit(&mma_done[ab]);
          tc_commit(&stage_free[st]);
          // into the stage of tile gg - 1, whose MMAs were issued one tile ago
          if (iss == 0 && i + kStcStages - 1 < it.ntiles)
            ok = issue_tma(it, i + kStcStages - 1, gg + kStcStages - 1);
        }
        if (!ok) break;
        tc_commit(&a_free[buf]);  // the item's queries are free once its MMAs complete
        g += it.ntiles;
        ++u;
      }
      if (!ok) *abort_flag = 1;
      // wind down: every MMA complete and every copy landed before resources are released
      tc_commit(drain);
      if (iss == 0) {
        mbar_wait(drain, 0);
        for (int x = n_issued > kStcStages ? n_issued - kStcStages : 0; x < n_issued; ++x)
          mbar_wait(&full[x % kStcStages], (x / kStcStages) & 1);
      }
    }
  } else if (warp < 4) {
    // ================= consumers: scores, per-row buffers, output
    const int row = tid;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const uint32_t sA = smem_u32(smem + L::kBufS) + row * 4;  // entry e at + e * 512
    const uint32_t jA = smem_u32(smem + L::kBufJ) + row * 2;  // entry e at + e * 256
    const uint32_t hA = smem_u32(smem + L::kHist) + (row & 63) * 4;  // bin b at + b * 256
    const int sh16 = (row >> 6) * 16;
    int g = 0;  // tiles consumed so far: score buffer g % kStcAcc
    for (int r = 0; r < nrounds; ++r) {
      const int k = item_of(r);
      if (k >= nitems) continue;
      const Item it = info(k);
      const int t = it.t0 + row;
      const bool live = t < T;
      const int c = (qpos0 + t) / kSelBlk;  // the row's block
      const int jmax = min(c - n_local, nb - 1);  // last candidate of this row
      const int n_row = jmax >= n_init ? jmax - n_init + 1 : 0;
      const bool buffered = live && n_row > topk;
      int cnt = 0;
      float thr = -INFINITY, smin = INFINITY, smax = -INFINITY;
      bool dead = false;
      for (int i = 0; i < it.ntiles; ++i) {
        const int gg = g + i, ab = gg % kStcAcc;
        const bool landed = !*abort_flag && mbar_wait(&mma_done[ab], (gg / kStcAcc) & 1);
        if (__any_sync(0xffffffffu, !landed)) {
          dead = true;
          break;
        }
        tc_fence_after();
        uint32_t sv[kStcN / kStcSub][kStcSub];
#pragma unroll
        for (int sub = 0; sub < kStcN / kStcSub; ++sub)
          tc_ld32(tD + kStcN * ab + kStcSub * sub + lane_off, sv[sub]);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if ((tid & 31) == 0) mbar_arrive(&acc_free[ab]);  // this warp is done with it
#pragma unroll
        for (int sub = 0; sub < kStcN / kStcSub; ++sub) {
          if (buffered) {
            // scores compared as raw dot products: the 1/sqrt(D) factor preserves the order
            const int j0 = n_init + i * kStcN + kStcSub * sub;
            auto append = [&](int cc, bool in_range) {  // predicated, no branch
              const float sc = __uint_as_float(sv[sub][cc]);
              const bool p = (in_range & (sc > thr)) && SALA_IN_BOUNDS(cnt < kStcCap);
              sts_f32_if(p, sA + cnt * (kStcRows * 4), sc);
              sts_u16_if(p, jA + cnt * (kStcRows * 2), (uint32_t)(j0 + cc));
              cnt += p ? 1 : 0;
              smin = p ? fminf(smin, sc) : smin;
              smax = p ? fmaxf(smax, sc) : smax;
            };
            if (j0 + kStcSub - 1 <= jmax) {
#pragma unroll
              for (int cc = 0; cc < kStcSub; ++cc) append(cc, true);
            } else {
#pragma unroll
              for (int cc = 0; cc < kStcSub; ++cc) append(cc, j0 + cc <= jmax);
            }
          }
          if (__any_sync(0xffffffffu, cnt > kStcCap - kStcSub) && cnt > topk) {
            // a cut that keeps at most kStcCoarse entries (all of the topk best)
            cnt = stc_compact(sA, jA, hA, sh16, cnt, topk, smin, smax, max(kStcCoarse, topk),
                              &thr);
            smin = thr;
          }
        }
      }
      if (dead) {
        *abort_flag = 1;
        break;
      }
      g += it.ntiles;
      if (buffered && cnt > topk)
        cnt = stc_compact(sA, jA, hA, sh16, cnt, topk, smin, smax, topk, &thr);  // exact
      // ---- this thread's row: init blocks, the kept candidates in block order, local window
      if (live && SALA_IN_BOUNDS(min(n_init, c + 1) + (buffered ? cnt : max(n_row, 0)) +
                                     max(0, c - max(n_init, c - n_local + 1) + 1) <=
                                 n_sel)) {
        int32_t* out = idx + (((int64_t)it.b * Hkv + it.hk) * T + t) * n_sel;
        const int n_first = min(n_init, c + 1);
        for (int e = 0; e < n_first; ++e) out[e] = e;
        int pos = n_first;
        if (!buffered) {
          for (int e = 0; e < n_row; ++e) out[pos + e] = n_init + e;
          pos += n_row;
        } else {
          for (int e = 0; e < cnt; ++e) out[pos + e] = (int)lds_u16(jA + e * (kStcRows * 2));
          pos += cnt;
        }
        const int lo = max(n_init, c - n_local + 1);
        for (int j = lo; j <= c; ++j) out[pos++] = j;
        for (int e = pos; e < n_sel; ++e) out[e] = -1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tc_dealloc(tmem, kCols);
  }
}

}  // namespace sala
