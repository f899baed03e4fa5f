// sparse_select.cuh -- InfLLM-v2-style KV block selection.
//
// Each query row picks a few key/value blocks (MiniCPM-SALA tech-report mirror,
// section 02 (2): fine-grained block selection, dense at short length; summary
// page, "Prerequisites / Sparse Attention": sliding window plus global anchors):
//   Kbar_j  = mean of the 64 keys of complete block j            (kernel 1)
//   score_j = (1/sqrt(D)) (sum_{h in group(hk)} q_{t,h}) . Kbar_j  (kernel 2)
//   top-k candidates in [n_init, c - n_local], ties -> smaller j,
//   plus init blocks and the local window, sorted, -1 padded    (kernel 3)
// The group sum of q is exact algebra (sum of dot products = dot of the sum).
// Scores are fp32 (inputs are bf16, so the products are exact and only the
// fp32 sums round).  Rows are processed in passes so the score scratch stays
// bounded (at most 1 GiB) at any sequence length.
#pragma once

#include <climits>

#include "ptx.cuh"

namespace sala {

constexpr int kSelBlk = 64;
constexpr size_t kSelScoreCap = size_t(1) << 30;

// Fused path (scores and top-k in one kernel, no score scratch) for topk <= this.
constexpr int kSelFusedMaxK = 64;  // <= 64: the final ordering holds two indices per lane

struct SelLayout {
  int nb;            // complete blocks
  int rows_pass;     // query rows per pass (score-scratch path)
  size_t kbar_off, kbar_bytes;   // block means, fp32
  size_t khi_off, klo_off;       // block means as bf16 high / low parts
  size_t score_off, score_bytes; // score scratch (topk > kSelFusedMaxK only)
  size_t total_fused, total;
};

inline SelLayout sel_layout(int B, int T, int Hkv, int D) {
  SelLayout L{};
  L.nb = T / kSelBlk;
  const size_t per_row = (size_t)B * Hkv * (size_t)(L.nb > 0 ? L.nb : 1) * 4;
  size_t rp = kSelScoreCap / per_row;
  rp = rp / kSelBlk * kSelBlk;
  if (rp < (size_t)kSelBlk) rp = kSelBlk;
  if (rp > (size_t)T) rp = (size_t)((T + kSelBlk - 1) / kSelBlk * kSelBlk);
  L.rows_pass = (int)(rp > 0 ? rp : kSelBlk);
  const size_t nelem = (size_t)B * (L.nb > 0 ? L.nb : 1) * Hkv * D;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  L.kbar_off = 0;
  L.kbar_bytes = nelem * 4;
  L.khi_off = up(L.kbar_bytes);
  L.klo_off = L.khi_off + up(nelem * 2);
  L.score_off = L.klo_off + up(nelem * 2);
  L.total_fused = L.score_off;
  L.score_bytes = per_row * (size_t)L.rows_pass;
  L.total = L.score_off + L.score_bytes;
  return L;
}

// ---- kernel 1: block means.  grid (nb, Hkv, B), block D threads.
// Writes the fp32 mean and its split into bf16 high and low parts (hi + lo
// carries 16 significant bits: the tensor-core scoring operand).
template <int D>
__global__ void __launch_bounds__(D)
block_means_kernel(const __nv_bfloat16* __restrict__ k, float* __restrict__ kbar,
                   __nv_bfloat16* __restrict__ khi, __nv_bfloat16* __restrict__ klo, int nb,
                   int Hkv, sala_strides sk) {
  const int j = blockIdx.x, hk = blockIdx.y, b = blockIdx.z, d = threadIdx.x;
  const __nv_bfloat16* src = k + b * sk.b + (int64_t)j * kSelBlk * sk.t + hk * sk.h + d;
  float acc = 0.f;
#pragma unroll 8
  for (int s = 0; s < kSelBlk; ++s) acc += __bfloat162float(src[(int64_t)s * sk.t]);
  const float m = acc * (1.0f / kSelBlk);
  const int64_t o = (((int64_t)b * nb + j) * Hkv + hk) * D + d;
  kbar[o] = m;
  const __nv_bfloat16 h = __float2bfloat16_rn(m);
  khi[o] = h;
  klo[o] = __float2bfloat16_rn(m - __bfloat162float(h));
}

// ---- kernel 2: block scores for a 64-row tile.  grid (row tiles, Hkv, B), 256 threads.
constexpr int kScTile = 64;
constexpr int kScLd = kScTile + 4;
template <int D>
constexpr size_t score_smem_bytes() { return size_t(2) * D * kScLd * sizeof(float); }

template <int D>
__global__ void __launch_bounds__(256)
block_scores_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ kbar,
                    float* __restrict__ scores, int nb, int Hkv, int G, sala_strides sq,
                    int r_begin, int r_end, int rows_pass, int n_init, int n_local,
                    float inv_sqrt_d) {
  extern __shared__ float sc_smem[];
  float (*qsT)[kScLd] = reinterpret_cast<float (*)[kScLd]>(sc_smem);            // [D][kScLd]
  float (*kbT)[kScLd] = reinterpret_cast<float (*)[kScLd]>(sc_smem + D * kScLd);  // [D][kScLd]
  const int ntiles = (r_end - r_begin + kScTile - 1) / kScTile;
  const int tile = ntiles - 1 - blockIdx.x;  // long (late) rows first
  const int hk = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int t0 = r_begin + tile * kScTile;
  const int t_last = min(t0 + kScTile, r_end) - 1;
  const int j_hi = min(t_last / kSelBlk - n_local, nb - 1);  // last candidate of the tile
  if (j_hi < n_init) return;

  // group-summed queries, transposed: qsT[d][r]
  for (int e = tid; e < kScTile * D; e += 256) {
    const int r = e / D, d = e % D;
    const int t = t0 + r;
    float acc = 0.f;
    if (t <= t_last) {
      const __nv_bfloat16* qp = q + b * sq.b + (int64_t)t * sq.t + (int64_t)hk * G * sq.h + d;
      for (int h = 0; h < G; ++h) acc += __bfloat162float(qp[(int64_t)h * sq.h]);
    }
    qsT[d][r] = acc;
  }
  const int ty = tid >> 4, tx = tid & 15;
  float* srow_base = scores + ((int64_t)b * Hkv + hk) * rows_pass * (int64_t)nb;
  for (int jt0 = n_init; jt0 <= j_hi; jt0 += kScTile) {
    __syncthreads();  // qsT written / previous kbT consumed
    for (int e = tid; e < kScTile * D; e += 256) {
      const int jj = e / D, d = e % D;
      const int j = jt0 + jj;
      kbT[d][jj] = j <= j_hi ? kbar[(((int64_t)b * nb + j) * Hkv + hk) * D + d] : 0.f;
    }
    __syncthreads();
    float acc[4][4] = {};
#pragma unroll 4
    for (int d = 0; d < D; ++d) {
      const float4 a = *reinterpret_cast<const float4*>(&qsT[d][ty * 4]);
      const float4 c = *reinterpret_cast<const float4*>(&kbT[d][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(av[u], cv[w], acc[u][w]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = t0 + ty * 4 + u;
      if (t > t_last) continue;
      const int jmax = t / kSelBlk - n_local;  // candidates of row t end here
      float* srow = srow_base + (int64_t)(t - r_begin) * nb;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int j = jt0 + tx * 4 + w;
        if (j <= jmax && j <= j_hi) srow[j - n_init] = acc[u][w] * inv_sqrt_d;
      }
    }
  }
}

__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- kernel 3: per-row top-k and index assembly.  One warp per (b, hk, t).
constexpr int kTopkWarps = 8;

__global__ void __launch_bounds__(kTopkWarps * 32)
topk_select_kernel(const float* __restrict__ scores, int32_t* __restrict__ idx, int B, int T,
                   int Hkv, int nb, int r_begin, int r_end, int rows_pass, int topk, int n_init,
                   int n_local) {
  __shared__ uint32_t hist_all[kTopkWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_here = r_end - r_begin;
  const int64_t gw = (int64_t)blockIdx.x * kTopkWarps + warp;
  if (gw >= (int64_t)B * Hkv * rows_here) return;
  const int tr = (int)(gw % rows_here);
  const int hk = (int)((gw / rows_here) % Hkv);
  const int b = (int)(gw / ((int64_t)rows_here * Hkv));
  const int t = r_begin + tr;
  const int c = t / kSelBlk;
  const int n_sel = n_init + topk + n_local;
  int32_t* out = idx + (((int64_t)b * Hkv + hk) * T + t) * n_sel;
  const float* srow = scores + (((int64_t)b * Hkv + hk) * rows_pass + tr) * (int64_t)nb;
  const int jhi = min(c - n_local, nb - 1);
  const int n = jhi >= n_init ? jhi - n_init + 1 : 0;
  uint32_t* hist = hist_all[warp];
  const uint32_t lt_mask = (1u << lane) - 1u;

  // init blocks
  const int n_first = min(n_init, c + 1);
  for (int e = lane; e < n_first; e += 32) out[e] = e;
  int pos = n_first;

  if (n <= topk) {
    for (int e = lane; e < n; e += 32) out[pos + e] = n_init + e;
    pos += n;
  } else {
    uint32_t prefix = 0, pmask = 0;
    int remaining = topk;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int e = lane; e < 256; e += 32) hist[e] = 0;
      __syncwarp();
      for (int e = lane; e < n; e += 32) {
        const uint32_t key = order_key(srow[e]);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncwarp();
      uint32_t local = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) local += hist[lane * 8 + u];
      // counts in bins above this lane's 8 bins
      uint32_t incl = local;  // suffix sum over lanes >= lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += o;
      }
      const uint32_t above = incl - local;
      const bool mine = above < (uint32_t)remaining && (uint32_t)remaining <= incl;
      int bucket = 0, rem_new = 0;
      if (mine) {
        uint32_t cnt = above;
        for (int u = 7; u >= 0; --u) {
          const uint32_t hcount = hist[lane * 8 + u];
          if (cnt + hcount >= (uint32_t)remaining) {
            bucket = lane * 8 + u;
            rem_new = remaining - (int)cnt;
            break;
          }
          cnt += hcount;
        }
      }
      const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
      bucket = __shfl_sync(0xffffffffu, bucket, src);
      remaining = __shfl_sync(0xffffffffu, rem_new, src);
      prefix |= (uint32_t)bucket << shift;
      pmask |= 255u << shift;
      __syncwarp();
    }
    // prefix is the exact key of the topk-th largest; take all keys above it and
    // the first `remaining` equal keys in ascending block order.
    int eq_taken = 0;
    for (int base = 0; base < n; base += 32) {
      const int e = base + lane;
      const uint32_t key = e < n ? order_key(srow[e]) : 0u;
      const bool gt = e < n && key > prefix;
      const bool eq = e < n && key == prefix;
      const uint32_t eq_mask = __ballot_sync(0xffffffffu, eq);
      const bool take = gt || (eq && eq_taken + __popc(eq_mask & lt_mask) < remaining);
      eq_taken += __popc(eq_mask);
      const uint32_t sel = __ballot_sync(0xffffffffu, take);
      if (take) out[pos + __popc(sel & lt_mask)] = n_init + e;
      pos += __popc(sel);
    }
  }
  // local window
  const int lo = max(n_init, c - n_local + 1);
  for (int j = lo + lane; j <= c; j += 32) out[pos + (j - lo)] = j;
  pos += (c >= lo) ? c - lo + 1 : 0;
  for (int e = pos + lane; e < n_sel; e += 32) out[e] = -1;
}

// ---- fused selection (topk <= kSelFusedMaxK): one CTA per (query block, KV
// head, batch).  All 64 rows of a query block share the candidate range
// [n_init, c - n_local], so the CTA streams the candidates' block means through
// shared memory in 64-block tiles and scores them on tensor cores:
//   score = (1/sqrt(D)) * qs . Kbar,  qs = sum over the group of q (fp32),
// with both operands split into bf16 high and low parts and the three leading
// products (lo*hi, hi*lo, hi*hi) accumulated in fp32 (16 significant bits per
// operand: the error is far below the score gaps that decide the selection).
// Each row keeps a candidate buffer in shared memory: a score enters only if
// it beats the row's current threshold (the topk-th best seen so far; later
// candidates lose ties because their block index is larger), and a buffer
// about to overflow is compacted to its topk best by a warp radix select.
constexpr int kSfCap = 256;      // candidate buffer entries per row
constexpr int kSfWarps = 8;
constexpr int kSfThreads = kSfWarps * 32;

template <int D>
struct SfSmem {
  static constexpr int kTileB = kSelBlk * D * 2;                         // 64 means x D bf16
  static constexpr size_t kB = 0;                                         // [stage][hi, lo]
  static constexpr size_t kBufS = kB + 4 * size_t(kTileB);                // [64][cap] f32
  static constexpr size_t kBufJ = kBufS + size_t(kSelBlk) * kSfCap * 4;   // [64][cap] u16
  static constexpr size_t kThr = kBufJ + size_t(kSelBlk) * kSfCap * 2;    // [64] f32
  static constexpr size_t kCnt = kThr + kSelBlk * 4;                      // [64] i32
  static constexpr size_t kHist = kCnt + kSelBlk * 4;                     // [warps][256] u32
  static constexpr size_t bytes = kHist + size_t(kSfWarps) * 256 * 4;
  // the group-summed queries (fp32 [64][D]) are staged in the score buffer first
  static_assert(size_t(kSelBlk) * D * 4 <= size_t(kSelBlk) * kSfCap * 4, "q staging fits");
};

__device__ __forceinline__ float order_key_inv(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Warp radix select over keys held in registers (PER per lane), 8 bits per pass
// from the top.  Finds the boundary of the k largest valid keys: on return, every
// key whose bits under *mask exceed *prefix is among the k largest, and *rem of
// the keys equal to *prefix under *mask are too.  It stops early when the whole
// boundary bucket belongs to the k largest (then *rem equals that bucket's size).
template <int PER>
__device__ __forceinline__ void warp_kth_prefix(const uint32_t (&key)[PER],
                                                const bool (&valid)[PER], int k, uint32_t* hist,
                                                int lane, uint32_t* prefix_out,
                                                uint32_t* mask_out, int* rem) {
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int e = lane; e < 256; e += 32) hist[e] = 0;
    __syncwarp();
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (valid[i] && (key[i] & pmask) == prefix) atomicAdd(&hist[(key[i] >> shift) & 255u], 1u);
    __syncwarp();
    uint32_t hv[8];
    uint32_t local = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      hv[u] = hist[lane * 8 + u];
      local += hv[u];
    }
    uint32_t incl = local;  // suffix sum over lanes >= lane
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
      if (lane + off < 32) incl += o;
    }
    const uint32_t above = incl - local;
    const bool mine = above < (uint32_t)remaining && (uint32_t)remaining <= incl;
    int bucket = 0, rem_new = 0, whole = 0;
    if (mine) {
      uint32_t cntv = above;
#pragma unroll
      for (int u = 7; u >= 0; --u) {
        if (rem_new == 0 && cntv + hv[u] >= (uint32_t)remaining) {
          bucket = lane * 8 + u;
          rem_new = remaining - (int)cntv;
          whole = rem_new == (int)hv[u];
        }
        cntv += hv[u];
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    bucket = __shfl_sync(0xffffffffu, bucket, src);
    remaining = __shfl_sync(0xffffffffu, rem_new, src);
    whole = __shfl_sync(0xffffffffu, whole, src);
    prefix |= (uint32_t)bucket << shift;
    pmask |= 255u << shift;
    __syncwarp();
    if (whole) break;
  }
  *prefix_out = prefix;
  *mask_out = pmask;
  *rem = remaining;
}

// Keeps the k best of the m buffered candidates of one row (larger score first,
// equal scores -> smaller block index) at the front of its buffer.  Returns
// min(m, k); when it compacts, *thr receives the k-th best score.  One warp.
__device__ __forceinline__ int sf_compact(float* bs, uint16_t* bj, int m, int k, uint32_t* hist,
                                          int lane, float* thr) {
  if (m <= k) return m;
  constexpr int PER = kSfCap / 32;
  uint32_t key[PER];
  float sv[PER];
  int jv[PER];
  bool valid[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    valid[i] = e < m;
    sv[i] = valid[i] ? bs[e] : 0.f;
    jv[i] = valid[i] ? (int)bj[e] : 0;
    key[i] = valid[i] ? order_key(sv[i]) : 0u;
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  bool take[PER];
  bool done = false;
  {
    // Fast path: one histogram over 256 value bins between the smallest and the largest
    // score.  The bin is a monotone function of the score, so every bin above the one
    // holding the k-th best is kept whole; inside that boundary bin (usually a few
    // entries) the exact order (larger score, then smaller block) decides.
    float lo = INFINITY, hi = -INFINITY;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (valid[i]) {
        lo = fminf(lo, sv[i]);
        hi = fmaxf(hi, sv[i]);
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    const float scale = 255.0f / (hi - lo);
    if (hi > lo && scale < 1.0e30f) {
      int bin[PER];
#pragma unroll
      for (int i = 0; i < PER; ++i) bin[i] = valid[i] ? min(255, (int)((sv[i] - lo) * scale)) : -1;
      for (int e = lane; e < 256; e += 32) hist[e] = 0;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (bin[i] >= 0) atomicAdd(&hist[bin[i]], 1u);
      __syncwarp();
      uint32_t hv[8];
      uint32_t local = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        hv[u] = hist[lane * 8 + u];
        local += hv[u];
      }
      uint32_t incl = local;  // suffix sum over lanes >= lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += o;
      }
      const uint32_t above = incl - local;
      const bool mine = above < (uint32_t)k && (uint32_t)k <= incl;
      int bucket = 0, rem_b = 0, n_b = 0;
      if (mine) {
        uint32_t cntv = above;
#pragma unroll
        for (int u = 7; u >= 0; --u) {
          if (rem_b == 0 && cntv + hv[u] >= (uint32_t)k) {
            bucket = lane * 8 + u;
            rem_b = k - (int)cntv;
            n_b = (int)hv[u];
          }
          cntv += hv[u];
        }
      }
      const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
      bucket = __shfl_sync(0xffffffffu, bucket, src);
      rem_b = __shfl_sync(0xffffffffu, rem_b, src);
      n_b = __shfl_sync(0xffffffffu, n_b, src);
      if (rem_b == n_b) {
#pragma unroll
        for (int i = 0; i < PER; ++i) take[i] = bin[i] >= bucket;
        done = true;
      } else if (n_b <= 32) {
        // gather the boundary bin into lanes 0..n_b-1 (through the histogram area)
        float* xs = reinterpret_cast<float*>(hist);
        int* xj = reinterpret_cast<int*>(hist) + 32;
        int pos[PER];
        int cnt = 0;
        __syncwarp();  // every lane has read the histogram
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const bool in_b = bin[i] == bucket;
          const uint32_t bm = __ballot_sync(0xffffffffu, in_b);
          pos[i] = cnt + __popc(bm & lt_mask);
          if (in_b) {
            xs[pos[i]] = sv[i];
            xj[pos[i]] = jv[i];
          }
          cnt += __popc(bm);
        }
        __syncwarp();
        const float s_me = lane < n_b ? xs[lane] : -INFINITY;
        const int j_me = lane < n_b ? xj[lane] : 0x7fffffff;
        int rank = 0;
        for (int l2 = 0; l2 < n_b; ++l2) {
          const float s2 = __shfl_sync(0xffffffffu, s_me, l2);
          const int j2 = __shfl_sync(0xffffffffu, j_me, l2);
          rank += (s2 > s_me || (s2 == s_me && j2 < j_me));
        }
        const bool win = lane < n_b && rank < rem_b;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const bool w = __shfl_sync(0xffffffffu, win, bin[i] == bucket ? pos[i] : 0);
          take[i] = bin[i] > bucket || (bin[i] == bucket && w);
        }
        done = true;
      }
    }
  }
  if (!done) {
    // general path (equal scores filling the boundary): radix select on the order keys
    uint32_t prefix = 0, pmask = 0;
    int rem = 0;
    warp_kth_prefix<PER>(key, valid, k, hist, lane, &prefix, &pmask, &rem);
    int n_eq = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      n_eq += __popc(__ballot_sync(0xffffffffu, valid[i] && (key[i] & pmask) == prefix));
#pragma unroll
    for (int i = 0; i < PER; ++i)
      take[i] = valid[i] && ((key[i] & pmask) > prefix || ((key[i] & pmask) == prefix && n_eq == rem));
    if (n_eq != rem) {
      // (pmask is all ones here) exact score ties at the boundary: keep the `rem`
      // smallest block indices among them
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        if (valid[i] && key[i] == prefix) {
          int rank = 0;
          for (int e2 = 0; e2 < m; ++e2) rank += (order_key(bs[e2]) == prefix && (int)bj[e2] < jv[i]);
          take[i] = rank < rem;
        }
      }
    }
  }
  // threshold for later candidates: the smallest kept score
  uint32_t kmin = 0xffffffffu;
#pragma unroll
  for (int i = 0; i < PER; ++i)
    if (take[i]) kmin = min(kmin, key[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
  __syncwarp();  // every lane has read the buffer
  int pos = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const uint32_t sel = __ballot_sync(0xffffffffu, take[i]);
    if (take[i]) {
      const int dst = pos + __popc(sel & lt_mask);  // never beyond the entry's own slot
      bs[dst] = sv[i];
      bj[dst] = (uint16_t)jv[i];
    }
    pos += __popc(sel);
  }
  __syncwarp();
  *thr = order_key_inv(kmin);
  return pos;
}

template <int D>
__global__ void __launch_bounds__(kSfThreads, 1)
select_fused_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ khi,
                    const __nv_bfloat16* __restrict__ klo, int32_t* __restrict__ idx, int T,
                    int nb, int Hkv, int G, sala_strides sq, int topk, int n_init, int n_local,
                    float inv_sqrt_d) {
  using L = SfSmem<D>;
  constexpr int kK = D / 16;
  extern __shared__ __align__(128) uint8_t sf_smem[];
  const int nqb = (T + kSelBlk - 1) / kSelBlk;
  const int c = nqb - 1 - (int)blockIdx.x;  // query block (long rows first)
  const int hk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = c * kSelBlk;
  const int nrows = min(kSelBlk, T - t0);
  const int j_hi = min(c - n_local, nb - 1);
  const int n = j_hi >= n_init ? j_hi - n_init + 1 : 0;  // candidates of every row here
  const int n_sel = n_init + topk + n_local;
  float* bufS = reinterpret_cast<float*>(sf_smem + L::kBufS);
  uint16_t* bufJ = reinterpret_cast<uint16_t*>(sf_smem + L::kBufJ);
  float* thr = reinterpret_cast<float*>(sf_smem + L::kThr);
  int* cnt = reinterpret_cast<int*>(sf_smem + L::kCnt);
  uint32_t* hist = reinterpret_cast<uint32_t*>(sf_smem + L::kHist) + warp * 256;

  if (n > topk) {
    // ---- group-summed queries (fp32, staged in the score buffer) -> bf16 hi / lo
    float* qs = bufS;  // [64][D]
    for (int e = tid; e < kSelBlk * (D / 8); e += kSfThreads) {
      const int r = e / (D / 8), ch = e % (D / 8);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (r < nrows) {
        // 16-byte loads (strides are multiples of 16 bytes), several heads in flight
        const __nv_bfloat16* qp =
            q + b * sq.b + (int64_t)(t0 + r) * sq.t + (int64_t)hk * G * sq.h + ch * 8;
#pragma unroll 8
        for (int h = 0; h < G; ++h) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(qp + (int64_t)h * sq.h));
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] += __uint_as_float(w[i] << 16);
            acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
          }
        }
      }
      float4* dst = reinterpret_cast<float4*>(qs + r * D + ch * 8);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
    if (tid < kSelBlk) {
      thr[tid] = -INFINITY;
      cnt[tid] = 0;
    }
    __syncthreads();
    const int mt = warp >> 1, nh = warp & 1;  // rows 16*mt.., blocks 32*nh.. of each tile
    const int gq = lane >> 2, tq = lane & 3, mat = lane >> 3, rin = lane & 7;
    uint32_t ah[kK][4], al[kK][4];
#pragma unroll
    for (int kk = 0; kk < kK; ++kk) {
#pragma unroll
      for (int rg = 0; rg < 4; ++rg) {
        const int row = 16 * mt + gq + (rg & 1) * 8;
        const int col = kk * 16 + tq * 2 + (rg >> 1) * 8;
        const float2 v = *reinterpret_cast<const float2*>(qs + row * D + col);
        const float h0 = __bfloat162float(__float2bfloat16_rn(v.x));
        const float h1 = __bfloat162float(__float2bfloat16_rn(v.y));
        ah[kk][rg] = pack_bf16x2(h0, h1);
        al[kk][rg] = pack_bf16x2(v.x - h0, v.y - h1);
      }
    }
    __syncthreads();  // qs consumed: the buffer holds candidates from here on

    const int ntiles = (n + kSelBlk - 1) / kSelBlk;
    auto load_tile = [&](int ti) {
      constexpr int kCh = D / 8;  // 16-byte chunks per block mean
      uint8_t* dst0 = sf_smem + L::kB + size_t(2 * (ti & 1)) * L::kTileB;
      for (int e = tid; e < 2 * kSelBlk * kCh; e += kSfThreads) {
        const int hl = e / (kSelBlk * kCh);
        const int rr = e % (kSelBlk * kCh);
        const int row = rr / kCh, ch = rr % kCh;
        const int j = n_init + ti * kSelBlk + row;
        if (j > j_hi) continue;
        const __nv_bfloat16* src =
            (hl ? klo : khi) + (((int64_t)b * nb + j) * Hkv + hk) * D + ch * 8;
        cp_async16(smem_u32(dst0 + hl * L::kTileB + row * (D * 2) + ((ch ^ (row & 7)) << 4)), src);
      }
      cp_async_commit();
    };
    load_tile(0);
    for (int ti = 0; ti < ntiles; ++ti) {
      if (ti + 1 < ntiles) {
        load_tile(ti + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();  // tile ti landed; thresholds / counts of the last compaction visible
      const int jt = n_init + ti * kSelBlk;
      const uint32_t bh = smem_u32(sf_smem + L::kB + size_t(2 * (ti & 1)) * L::kTileB);
      const uint32_t bl = bh + L::kTileB;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < kK; ++kk) {
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          const uint32_t krow = 32 * nh + 16 * np + (mat >> 1) * 8 + rin;
          const uint32_t ch = 2 * kk + (mat & 1);
          const uint32_t off = krow * (D * 2) + ((ch ^ (krow & 7)) << 4);
          uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
          ldsm_x4(bh + off, h0, h1, h2, h3);
          ldsm_x4(bl + off, l0, l1, l2, l3);
          mma_bf16_16816(acc[2 * np], al[kk], h0, h1);
          mma_bf16_16816(acc[2 * np + 1], al[kk], h2, h3);
          mma_bf16_16816(acc[2 * np], ah[kk], l0, l1);
          mma_bf16_16816(acc[2 * np + 1], ah[kk], l2, l3);
          mma_bf16_16816(acc[2 * np], ah[kk], h0, h1);
          mma_bf16_16816(acc[2 * np + 1], ah[kk], h2, h3);
        }
      }
      // ---- append the scores that beat their row's threshold
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = 16 * mt + gq + 8 * hr;
        const float th = thr[row];
        float sv[8];
        int jv[8];
        bool ps[8];
        int cnt_l = 0;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int i = nt * 2 + cc;
            jv[i] = jt + 32 * nh + 8 * nt + tq * 2 + cc;
            sv[i] = acc[nt][2 * hr + cc] * inv_sqrt_d;
            ps[i] = jv[i] <= j_hi && sv[i] > th;
            cnt_l += ps[i];
          }
        }
        // offsets inside the quad of lanes that share this row
        int incl = cnt_l;
        int v = __shfl_up_sync(0xffffffffu, incl, 1, 4);
        if (tq >= 1) incl += v;
        v = __shfl_up_sync(0xffffffffu, incl, 2, 4);
        if (tq >= 2) incl += v;
        const int total = __shfl_sync(0xffffffffu, incl, 3, 4);
        int base = 0;
        if (tq == 0 && total > 0) base = atomicAdd(&cnt[row], total);
        base = __shfl_sync(0xffffffffu, base, 0, 4);
        int pos = base + incl - cnt_l;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (ps[i]) {
            bufS[row * kSfCap + pos] = sv[i];
            bufJ[row * kSfCap + pos] = (uint16_t)jv[i];
            ++pos;
          }
        }
      }
      __syncthreads();  // appends done; this tile's stage may be refilled
      // ---- compact rows whose buffer could overflow on the next tile
      for (int row = warp; row < kSelBlk; row += kSfWarps) {
        const int m = cnt[row];
        if (m > kSfCap - kSelBlk) {
          float th = 0.f;
          const int m2 = sf_compact(bufS + row * kSfCap, bufJ + row * kSfCap, m, topk, hist,
                                    lane, &th);
          if (lane == 0) {
            cnt[row] = m2;
            thr[row] = th;
          }
        }
      }
    }
  }
  // ---- per row: final top-k in block order, init blocks, local window, padding
  for (int row = warp; row < nrows; row += kSfWarps) {
    const int t = t0 + row;
    int32_t* out = idx + (((int64_t)b * Hkv + hk) * T + t) * n_sel;
    const int n_first = min(n_init, c + 1);
    for (int e = lane; e < n_first; e += 32) out[e] = e;
    int pos = n_first;
    if (n <= topk) {
      for (int e = lane; e < n; e += 32) out[pos + e] = n_init + e;
      pos += n;
    } else {
      __syncwarp();
      float th = 0.f;
      const int m = sf_compact(bufS + row * kSfCap, bufJ + row * kSfCap, cnt[row], topk, hist,
                               lane, &th);
      // block order: rank of each kept index among the m <= 64 kept ones
      const uint16_t* bjr = bufJ + row * kSfCap;
      const int ja = lane < m ? (int)bjr[lane] : INT_MAX;
      const int jb = lane + 32 < m ? (int)bjr[lane + 32] : INT_MAX;
      int ra = 0, rb = 0;
#pragma unroll 8
      for (int src = 0; src < 32; ++src) {
        const int xa = __shfl_sync(0xffffffffu, ja, src);
        const int xb = __shfl_sync(0xffffffffu, jb, src);
        ra += (xa < ja) + (xb < ja);
        rb += (xa < jb) + (xb < jb);
      }
      if (lane < m) out[pos + ra] = ja;
      if (lane + 32 < m) out[pos + rb] = jb;
      pos += m;
    }
    const int lo = max(n_init, c - n_local + 1);
    for (int j = lo + lane; j <= c; j += 32) out[pos + (j - lo)] = j;
    pos += (c >= lo) ? c - lo + 1 : 0;
    for (int e = pos + lane; e < n_sel; e += 32) out[e] = -1;
  }
}

}  // namespace sala
