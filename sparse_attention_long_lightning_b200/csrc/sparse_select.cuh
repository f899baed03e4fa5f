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
// The query rows may be a window of the sequence (a shard of it): row t of q and
// idx is position qpos0 + t, which sets its block c and so its candidates; the
// keys (and their block means) cover positions 0 .. Tk - 1.
#pragma once

#include <climits>

#include "ptx.cuh"

namespace sala {

constexpr int kSelBlk = 64;
constexpr size_t kSelScoreCap = size_t(1) << 30;

// Fused path (scores and top-k in one kernel, no score scratch, sparse_select_tc.cuh)
// for topk <= this.
constexpr int kSelFusedMaxK = 64;

struct SelLayout {
  int nb;            // complete blocks
  int rows_pass;     // query rows per pass (score-scratch path)
  size_t kbar_off, kbar_bytes;   // block means, fp32
  size_t khi_off, klo_off;       // block means as bf16 high / low parts
  size_t score_off, score_bytes; // score scratch (topk > kSelFusedMaxK only)
  size_t klo2_off;               // third bf16 part of the means (score-scratch layout only)
  size_t total_fused, total;
};

// T: query rows, Tk: key positions.
inline SelLayout sel_layout(int B, int T, int Tk, int Hkv, int D) {
  SelLayout L{};
  L.nb = Tk / kSelBlk;
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
  L.klo2_off = L.score_off + up(L.score_bytes);
  L.total = L.klo2_off + up(nelem * 2);
  return L;
}

// ---- kernel 1: block means.  grid (nb, Hkv, B), block D threads.
// Writes the fp32 mean and its split into bf16 high and low parts (hi + lo
// carries 16 significant bits: the tensor-core scoring operand); with klo2, the
// parts are those of x = mean * part_scale (one fp32 rounding; 1 leaves the mean as it
// is) and include the third part lo2 = x - hi - lo, so that hi + lo + lo2 is x exactly
// (each remainder is exact in fp32 and has at most 8 significant bits left at the end).
template <int D>
__global__ void __launch_bounds__(D)
block_means_kernel(const __nv_bfloat16* __restrict__ k, float* __restrict__ kbar,
                   __nv_bfloat16* __restrict__ khi, __nv_bfloat16* __restrict__ klo,
                   __nv_bfloat16* __restrict__ klo2, float part_scale, int nb, int Hkv,
                   sala_strides sk) {
  const int j = blockIdx.x, hk = blockIdx.y, b = blockIdx.z, d = threadIdx.x;
  const __nv_bfloat16* src = k + b * sk.b + (int64_t)j * kSelBlk * sk.t + hk * sk.h + d;
  float acc = 0.f;
#pragma unroll 8
  for (int s = 0; s < kSelBlk; ++s) acc += __bfloat162float(src[(int64_t)s * sk.t]);
  const float m = acc * (1.0f / kSelBlk);
  const int64_t o = (((int64_t)b * nb + j) * Hkv + hk) * D + d;
  kbar[o] = m;
  const float x = klo2 ? m * part_scale : m;
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  khi[o] = h;
  const float r1 = x - __bfloat162float(h);
  const __nv_bfloat16 lo = __float2bfloat16_rn(r1);
  klo[o] = lo;
  if (klo2) klo2[o] = __float2bfloat16_rn(r1 - __bfloat162float(lo));
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
                    int qpos0, int r_begin, int r_end, int rows_pass, int n_init, int n_local,
                    float inv_sqrt_d) {
  extern __shared__ float sc_smem[];
  float (*qsT)[kScLd] = reinterpret_cast<float (*)[kScLd]>(sc_smem);            // [D][kScLd]
  float (*kbT)[kScLd] = reinterpret_cast<float (*)[kScLd]>(sc_smem + D * kScLd);  // [D][kScLd]
  const int ntiles = (r_end - r_begin + kScTile - 1) / kScTile;
  const int tile = ntiles - 1 - blockIdx.x;  // long (late) rows first
  const int hk = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int t0 = r_begin + tile * kScTile;
  const int t_last = min(t0 + kScTile, r_end) - 1;
  const int j_hi = min((qpos0 + t_last) / kSelBlk - n_local, nb - 1);  // the tile's last candidate
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
      const int jmax = (qpos0 + t) / kSelBlk - n_local;  // candidates of row t end here
      float* srow = srow_base + (int64_t)(t - r_begin) * nb;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int j = jt0 + tx * 4 + w;
        if (j <= jmax && j <= j_hi && SALA_IN_BOUNDS(j - n_init < nb && t - r_begin < rows_pass))
          srow[j - n_init] = acc[u][w] * inv_sqrt_d;
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
                   int qpos0, int Hkv, int nb, int r_begin, int r_end, int rows_pass, int topk,
                   int n_init, int n_local) {
  __shared__ uint32_t hist_all[kTopkWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_here = r_end - r_begin;
  const int64_t gw = (int64_t)blockIdx.x * kTopkWarps + warp;
  if (gw >= (int64_t)B * Hkv * rows_here) return;
  const int tr = (int)(gw % rows_here);
  const int hk = (int)((gw / rows_here) % Hkv);
  const int b = (int)(gw / ((int64_t)rows_here * Hkv));
  const int t = r_begin + tr;
  const int c = (qpos0 + t) / kSelBlk;  // the row's block
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
  if (!SALA_IN_BOUNDS(pos + max(0, c - lo + 1) <= n_sel)) return;
  for (int j = lo + lane; j <= c; j += 32) out[pos + (j - lo)] = j;
  pos += (c >= lo) ? c - lo + 1 : 0;
  for (int e = pos + lane; e < n_sel; e += 32) out[e] = -1;
}

}  // namespace sala
