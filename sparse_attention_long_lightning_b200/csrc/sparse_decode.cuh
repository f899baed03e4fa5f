// sparse_decode.cuh -- sparse-layer (InfLLM-v2 style, NoPE) decode: one new query per
// sequence attends to the key/value blocks it selects from a KV cache.
//
// The step is row t = p of the prefill computation (MiniCPM-SALA tech-report mirror,
// section 02 (2): each query processes only the key/value blocks it selects; summary
// page, "Prerequisites / Sparse Attention"), for a sequence whose cache holds positions
// 0..p (the new token's key and value are already stored at row p):
//   Kbar_j  = mean of the 64 keys of complete block j, kept in a per-sequence cache that
//             this step extends: when p closes block c = p / 64, Kbar_c is written
//   score_j = sum_{h in group(hk)} q_h . Kbar_j  for n_init <= j <= c - n_local
//   chosen  = the top `topk` (larger score first, ties -> smaller j) + the init blocks +
//             the local window, sorted ascending, -1 padded (the prefill rule)
//   o_h     = softmax over the chosen blocks' keys s <= p of scale * q_h . k_s, times v;
//             y = sigmoid(g) * o
// Four launches, all sized by the batch:
//   sd_score_kernel   one CTA per (candidate chunk, KV head, sequence): the group sum of
//                     q in fp32, then one fp32 dot product per candidate block mean
//                     (coalesced 16-byte loads, warp reductions); chunk 0 also writes the
//                     mean of a block the new token completes
//   sd_topk_kernel    one CTA per (KV head, sequence): CTA radix select over the scores'
//                     order-preserving keys, then a stable compaction in block order
//   sd_attn_kernel    one CTA per (split, KV head, sequence): the split's share of the
//                     chosen blocks, a cp.async ring of K/V tiles, the group's query
//                     heads as the M = 16 operand of m16n8k16 tensor-core MMAs (Q K^T in
//                     bf16; P V as two bf16 MMAs, P's high and low parts, on V as stored,
//                     so any bf16 V is exact), online softmax
//                     per warp, the four warps merged into one partial (max, sum, O)
//   sd_combine_kernel one CTA per (query head, sequence): merges the splits, applies the
//                     gate, writes bf16.
#pragma once

#include "ptx.cuh"
#include "sparse_select.cuh"

namespace sala {

constexpr int kSdBlk = 64;           // keys per block
constexpr int kSdScoreChunk = 512;   // most candidates per score CTA
constexpr int kSdMaxSplit = 16;      // attention splits per (sequence, KV head)
constexpr int kSdAttnWarps = 4;      // 16 keys of a block each
#ifndef SALA_SD_STAGES
#define SALA_SD_STAGES 3
#endif
constexpr int kSdStages = SALA_SD_STAGES;  // K/V tile ring depth of the attention kernel

struct SdParams {
  const __nv_bfloat16* q;   // [B, Hq, D]  (strides sq.b, sq.h)
  const __nv_bfloat16* g;   // [B, Hq, D] or null
  __nv_bfloat16* o;         // [B, Hq, D]
  const __nv_bfloat16* k;   // [B, Tmax, Hkv, D] cache
  const __nv_bfloat16* v;
  float* kbar;              // [B, nbcap, Hkv, D] fp32
  const int32_t* pos;       // [B]
  int32_t* idx;             // [B, Hkv, n_sel]
  float* scores;            // [B, Hkv, nbcap]
  float* part;              // [B, Hkv, nsplit, 16 * (D + 2)]
  sala_strides sq, sg, so, sk, sv;
  int B, Tmax, Hq, Hkv, G, D, nbcap;
  int n_init, topk, n_local, n_sel, nsplit, chunk;
  float scale_log2;         // softmax scale * log2(e)
};

// Position of sequence b, or -1 (and SALA_ERR_RANGE) when it lies outside the cache.
__device__ __forceinline__ int sd_pos(const SdParams& p, int b) {
  const int t = __ldg(p.pos + b);
  if (t < 0 || t >= p.Tmax) {
    if (threadIdx.x == 0) raise_device_error(SALA_ERR_RANGE);
    return -1;
  }
  return t;
}

// ---- scores of the candidate blocks (and the mean of a block the new token closes)
template <int D>
__global__ void __launch_bounds__(256) sd_score_kernel(const SdParams p) {
  constexpr int kPer = D / 32;  // dims per lane
  __shared__ __align__(16) float qs[D];
  const int b = blockIdx.z, hk = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int t = sd_pos(p, b);
  if (t < 0) return;
  const int c = t / kSdBlk;
  if (blockIdx.x == 0 && (t + 1) % kSdBlk == 0) {
    // block c is complete with this token: its mean, summed in key order like the prefill
    for (int d = tid; d < D; d += 256) {
      const __nv_bfloat16* src = p.k + b * p.sk.b + (int64_t)c * kSdBlk * p.sk.t + hk * p.sk.h + d;
      float acc = 0.f;
#pragma unroll 8
      for (int s = 0; s < kSdBlk; ++s) acc += __bfloat162float(src[(int64_t)s * p.sk.t]);
      p.kbar[(((int64_t)b * p.nbcap + c) * p.Hkv + hk) * D + d] = acc * (1.0f / kSdBlk);
    }
  }
  const int jhi = c - p.n_local;                      // last candidate (complete blocks)
  const int j0 = p.n_init + blockIdx.x * p.chunk;
  const int j1 = min(jhi, j0 + p.chunk - 1);
  if (j1 < j0) return;
  for (int d = tid; d < D; d += 256) {
    const __nv_bfloat16* qr = p.q + b * p.sq.b + (int64_t)hk * p.G * p.sq.h + d;
    float acc = 0.f;
    for (int h = 0; h < p.G; ++h) acc += __bfloat162float(qr[(int64_t)h * p.sq.h]);
    qs[d] = acc;
  }
  __syncthreads();
  float qv[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) qv[i] = qs[lane * kPer + i];
  const float* kb = p.kbar + ((int64_t)b * p.nbcap * p.Hkv + hk) * D + lane * kPer;
  float* out = p.scores + ((int64_t)b * p.Hkv + hk) * p.nbcap;
  // four candidates per warp step for memory-level parallelism
  for (int jb = j0 + warp * 4; jb <= j1; jb += 8 * 4) {
    float dot[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = min(jb + u, j1);
      const float* kr = kb + (int64_t)j * p.Hkv * D;
      float a = 0.f;
      if constexpr (kPer == 4) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(kr));
        a = fmaf(qv[0], x.x, fmaf(qv[1], x.y, fmaf(qv[2], x.z, qv[3] * x.w)));
      } else {
        const float2 x = __ldg(reinterpret_cast<const float2*>(kr));
        a = fmaf(qv[0], x.x, qv[1] * x.y);
      }
      dot[u] = a;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int u = 0; u < 4; ++u) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], off);
    if (lane < 4 && jb + lane <= j1) {
      float v = dot[0];
#pragma unroll
      for (int u = 1; u < 4; ++u) v = lane == u ? dot[u] : v;
      out[jb + lane] = v;
    }
  }
}

// ---- top-k of the candidates, written with the init blocks and the local window
constexpr int kSdTopkThreads = 256;
constexpr int kSdTopkStage = 8192;  // candidates staged in shared memory (else read from L2)

// Exclusive prefix sum of one int per thread over the CTA; *total gets the sum.
__device__ __forceinline__ int sd_cta_exscan(int x, int* wbuf, int* total) {
  constexpr int kW = kSdTopkThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) wbuf[warp] = incl;
  __syncthreads();
  int before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kW; ++w) {
    const int v = wbuf[w];
    before += w < warp ? v : 0;
    tot += v;
  }
  __syncthreads();  // wbuf may be reused
  *total = tot;
  return before + incl - x;
}

__global__ void __launch_bounds__(kSdTopkThreads) sd_topk_kernel(const SdParams p) {
  __shared__ float stage[kSdTopkStage];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_rem;
  __shared__ int wbuf[kSdTopkThreads / 32];
  const int b = blockIdx.y, hk = blockIdx.x, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int t = sd_pos(p, b);
  if (t < 0) return;
  const int c = t / kSdBlk;
  const int jhi = c - p.n_local;
  const int n = jhi >= p.n_init ? jhi - p.n_init + 1 : 0;
  int32_t* out = p.idx + ((int64_t)b * p.Hkv + hk) * p.n_sel;
  const float* sc = p.scores + ((int64_t)b * p.Hkv + hk) * p.nbcap + p.n_init;
  const int n_first = min(p.n_init, c + 1);
  for (int e = tid; e < n_first; e += kSdTopkThreads) out[e] = e;
  int pos = n_first;
  if (n <= p.topk) {
    for (int e = tid; e < n; e += kSdTopkThreads) out[pos + e] = p.n_init + e;
    pos += n;
  } else {
    const float* src = sc;
    if (n <= kSdTopkStage) {
      for (int e = tid; e < n; e += kSdTopkThreads) stage[e] = sc[e];
      src = stage;
      __syncthreads();
    }
    // radix select, 8 bits per pass from the top: the topk-th largest key
    uint32_t prefix = 0, pmask = 0;
    int remaining = p.topk;
    for (int shift = 24; shift >= 0; shift -= 8) {
      hist[tid] = 0;
      __syncthreads();
      for (int e = tid; e < n; e += kSdTopkThreads) {
        const uint32_t key = order_key(src[e]);
        if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        uint32_t local = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) local += hist[lane * 8 + u];
        uint32_t incl = local;  // keys in the bins of lanes >= lane
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t o = __shfl_down_sync(0xffffffffu, incl, off);
          if (lane + off < 32) incl += o;
        }
        const uint32_t above = incl - local;
        if (above < (uint32_t)remaining && (uint32_t)remaining <= incl) {
          uint32_t cnt = above;
          for (int u = 7; u >= 0; --u) {
            const uint32_t hc = hist[lane * 8 + u];
            if (cnt + hc >= (uint32_t)remaining) {
              s_prefix = prefix | ((uint32_t)(lane * 8 + u) << shift);
              s_rem = (uint32_t)remaining - cnt;
              break;
            }
            cnt += hc;
          }
        }
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = (int)s_rem;
      pmask |= 255u << shift;
    }
    // keys above `prefix` are in; of the keys equal to it, the first `remaining` in block
    // order.  Each thread owns a contiguous run of candidates: one scan of the counts
    // places every thread's selections.
    const int per = (n + kSdTopkThreads - 1) / kSdTopkThreads;
    const int e0 = min(n, tid * per), e1 = min(n, e0 + per);
    int ngt = 0, neq = 0;
    for (int e = e0; e < e1; ++e) {
      const uint32_t key = order_key(src[e]);
      ngt += key > prefix;
      neq += key == prefix;
    }
    int tot;
    const int gt_before = sd_cta_exscan(ngt, wbuf, &tot);
    const int eq_before = sd_cta_exscan(neq, wbuf, &tot);
    int w = pos + gt_before + min(eq_before, remaining);
    int eq_seen = eq_before;
    for (int e = e0; e < e1; ++e) {
      const uint32_t key = order_key(src[e]);
      bool take = key > prefix;
      if (key == prefix) take = eq_seen++ < remaining;
      if (take) out[w++] = p.n_init + e;
    }
    pos += p.topk;
  }
  const int lo = max(p.n_init, c - p.n_local + 1);
  for (int j = lo + tid; j <= c; j += kSdTopkThreads) out[pos + (j - lo)] = j;
  pos += c >= lo ? c - lo + 1 : 0;
  for (int e = pos + tid; e < p.n_sel; e += kSdTopkThreads) out[e] = -1;
}

// ---- attention over one split of the chosen blocks; partial (max, sum, O) per head row
template <int D>
struct SdAttnSmem {
  static constexpr int kHalf = kSdBlk * 128;        // 64 rows x 64 bf16 columns: 8 KB
  static constexpr int kTile = kSdBlk * D * 2;       // K or V block
  static constexpr int kBuf = 2 * kTile;             // K then V
  static constexpr int kMerge = kSdAttnWarps * 16 * D * 4 + kSdAttnWarps * 32 * 4;
  static_assert(kMerge <= kSdStages * kBuf, "merge area fits in the tile buffers");
  static constexpr size_t bytes = kSdStages * size_t(kBuf) + 128;  // + alignment slack
};

template <int D>
__global__ void __launch_bounds__(kSdAttnWarps * 32) sd_attn_kernel(const SdParams p) {
  using L = SdAttnSmem<D>;
  constexpr int kKSteps = D / 16, kNT = D / 8, kCh = D / 8;  // k-steps, n-tiles, 16-B chunks
  extern __shared__ uint8_t sd_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sd_smem_raw) + 127) &
                                             ~uintptr_t(127));
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int t = sd_pos(p, b);
  if (t < 0) return;
  const int c = t / kSdBlk;
  const int32_t* ir = p.idx + ((int64_t)b * p.Hkv + hk) * p.n_sel;
  float* part = p.part + (((int64_t)b * p.Hkv + hk) * p.nsplit + split) * (16 * (D + 2));
  // chosen blocks are sorted ascending with -1 padding: count the live ones
  int nblk = 0;
  for (int e0 = 0; e0 < p.n_sel; e0 += 32) {
    const int e = e0 + lane;
    nblk += __popc(__ballot_sync(0xffffffffu, e < p.n_sel && __ldg(ir + e) >= 0));
  }
  const int per = (nblk + p.nsplit - 1) / p.nsplit;
  const int sb0 = split * per, sb1 = min(nblk, sb0 + per);
  if (sb0 >= sb1) {
    for (int i = tid; i < 32; i += blockDim.x) part[i] = i < 16 ? -INFINITY : 0.f;
    return;
  }
  // Q fragments: rows = the group's query heads (padded to 16 with zeros)
  uint32_t qa[kKSteps][4];
  {
    const __nv_bfloat16* qr = p.q + b * p.sq.b + (int64_t)(hk * p.G) * p.sq.h;
#pragma unroll
    for (int kk = 0; kk < kKSteps; ++kk)
#pragma unroll
      for (int rg = 0; rg < 4; ++rg) {
        const int row = gq + (rg & 1) * 8;
        const int col = kk * 16 + tq * 2 + (rg >> 1) * 8;
        qa[kk][rg] = row < p.G
                         ? *reinterpret_cast<const uint32_t*>(qr + (int64_t)row * p.sq.h + col)
                         : 0u;
      }
  }
  auto issue = [&](int e) {  // K and V of chosen block e into ring slot (e - sb0) % S
    const int j = __ldg(ir + e);
    if (!SALA_IN_BOUNDS(j >= 0 && j <= c)) return;  // a chosen block lies in [0, c]
    const uint32_t kb = smem_u32(smem + ((e - sb0) % kSdStages) * L::kBuf), vb = kb + L::kTile;
    const __nv_bfloat16* ks = p.k + b * p.sk.b + (int64_t)j * kSdBlk * p.sk.t + hk * p.sk.h;
    const __nv_bfloat16* vs = p.v + b * p.sv.b + (int64_t)j * kSdBlk * p.sv.t + hk * p.sv.h;
    for (int x = tid; x < kSdBlk * kCh; x += blockDim.x) {
      const int r = x / kCh, cc = x % kCh;
      const uint32_t off = (cc >> 3) * L::kHalf + swz128(r, cc & 7);
      cp_async16(kb + off, ks + (int64_t)r * p.sk.t + cc * 8);
      cp_async16(vb + off, vs + (int64_t)r * p.sv.t + cc * 8);
    }
  };
#pragma unroll
  for (int x = 0; x < kSdStages; ++x) {  // one commit group per slot, possibly empty
    if (sb0 + x < sb1) issue(sb0 + x);
    cp_async_commit();
  }

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows gq, gq+8 (log2 domain)
  float oacc[kNT][4];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt) oacc[nt][0] = oacc[nt][1] = oacc[nt][2] = oacc[nt][3] = 0.f;
  for (int e = sb0; e < sb1; ++e) {
    cp_async_wait<kSdStages - 1>();  // block e's group has landed
    __syncthreads();
    const int j = __ldg(ir + e);
    const uint32_t kb = smem_u32(smem + ((e - sb0) % kSdStages) * L::kBuf), vb = kb + L::kTile;
    const bool straddle = j == c && t % kSdBlk != kSdBlk - 1;  // keys past t in this block
    if (straddle) {
      // rows past t may hold anything: zero their V so 0-weights stay 0
      for (int x = tid; x < kSdBlk * kCh; x += blockDim.x) {
        const int r = x / kCh, cc = x % kCh;
        if (j * kSdBlk + r > t)
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(
                           vb + (cc >> 3) * L::kHalf + swz128(r, cc & 7)),
                       "r"(0u)
                       : "memory");
      }
      __syncthreads();
    }
    // ---- S = Q K^T for keys 16*warp .. 16*warp+15
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int mat = lane >> 3, rin = lane & 7;
      const uint32_t krow = warp * 16 + (mat >> 1) * 8 + rin;
#pragma unroll
      for (int kk = 0; kk < kKSteps; ++kk) {
        const uint32_t chunk = 2 * kk + (mat & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + (chunk >> 3) * L::kHalf + swz128(krow, chunk & 7), b0, b1, b2, b3);
        mma_bf16_16816(sc[0], qa[kk], b0, b1);
        mma_bf16_16816(sc[1], qa[kk], b2, b3);
      }
    }
    // ---- V fragments, bf16 as stored (no range limit)
    uint32_t vv[kNT / 2][4];
    {
      const int mat = lane >> 3, rin = lane & 7;
      const uint32_t vrow = warp * 16 + (mat & 1) * 8 + rin;
#pragma unroll
      for (int pp = 0; pp < kNT / 2; ++pp) {
        const uint32_t chunk = 2 * pp + (mat >> 1);
        ldsm_x4_t(vb + (chunk >> 3) * L::kHalf + swz128(vrow, chunk & 7), vv[pp][0], vv[pp][1],
                  vv[pp][2], vv[pp][3]);
      }
    }
    // ---- scale, causal mask, online softmax
    const int key0 = j * kSdBlk + warp * 16 + tq * 2;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float x = sc[nt][cc] * p.scale_log2;
        if (key0 + nt * 8 + (cc & 1) > t) x = -INFINITY;
        sc[nt][cc] = x;
      }
      mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    const float al0 = n0 == -INFINITY ? 1.f : exp2f(m0 - n0);
    const float al1 = n1 == -INFINITY ? 1.f : exp2f(m1 - n1);
    m0 = n0;
    m1 = n1;
    l0 *= al0;
    l1 *= al1;
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      oacc[nt][0] *= al0; oacc[nt][1] *= al0;
      oacc[nt][2] *= al1; oacc[nt][3] *= al1;
    }
    const float mu0 = m0 == -INFINITY ? 0.f : m0, mu1 = m1 == -INFINITY ? 0.f : m1;
    // P as a bf16 high part plus a bf16 low part (the rounding residual): with V in bf16
    // the two P V products carry ~16 significant bits of P and any bf16 V exactly
    uint32_t pa[4], pl[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const float p0 = exp2f(sc[nt][0] - mu0), p1 = exp2f(sc[nt][1] - mu0);
      const float p2 = exp2f(sc[nt][2] - mu1), p3 = exp2f(sc[nt][3] - mu1);
      l0 += p0 + p1;
      l1 += p2 + p3;
      pa[nt * 2 + 0] = pack_bf16x2_hi_lo(p0, p1, pl[nt * 2 + 0]);
      pa[nt * 2 + 1] = pack_bf16x2_hi_lo(p2, p3, pl[nt * 2 + 1]);
    }
#pragma unroll
    for (int pp = 0; pp < kNT / 2; ++pp) {
      mma_bf16_16816(oacc[2 * pp], pa, vv[pp][0], vv[pp][1]);
      mma_bf16_16816(oacc[2 * pp + 1], pa, vv[pp][2], vv[pp][3]);
      mma_bf16_16816(oacc[2 * pp], pl, vv[pp][0], vv[pp][1]);
      mma_bf16_16816(oacc[2 * pp + 1], pl, vv[pp][2], vv[pp][3]);
    }
    __syncthreads();  // block e's slot is free again
    if (e + kSdStages < sb1) issue(e + kSdStages);  // into block e's slot
    cp_async_commit();
  }
  cp_async_wait<0>();

  // ---- merge the four warps' partial states into the split's partial
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();  // every warp is done with the tile buffers
  float* mO = reinterpret_cast<float*>(smem);                       // [warp][16][D]
  float* mML = mO + kSdAttnWarps * 16 * D;                          // [warp][m 16, l 16]
  {
    float* myO = mO + warp * 16 * D;
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      const int col = nt * 8 + tq * 2;
      *reinterpret_cast<float2*>(myO + gq * D + col) = make_float2(oacc[nt][0], oacc[nt][1]);
      *reinterpret_cast<float2*>(myO + (gq + 8) * D + col) = make_float2(oacc[nt][2], oacc[nt][3]);
    }
    if (tq == 0) {
      mML[warp * 32 + gq] = m0;
      mML[warp * 32 + gq + 8] = m1;
      mML[warp * 32 + 16 + gq] = l0;
      mML[warp * 32 + 16 + gq + 8] = l1;
    }
  }
  __syncthreads();
  // thread -> (row, column range): 128 threads, 8 per row
  const int row = tid >> 3;
  const int c0 = (tid & 7) * (D / 8);
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kSdAttnWarps; ++w) M = fmaxf(M, mML[w * 32 + row]);
  float wgt[kSdAttnWarps], Ls = 0.f;
#pragma unroll
  for (int w = 0; w < kSdAttnWarps; ++w) {
    wgt[w] = M == -INFINITY ? 0.f : exp2f(mML[w * 32 + row] - M);
    Ls += wgt[w] * mML[w * 32 + 16 + row];
  }
  if ((tid & 7) == 0) {
    part[row] = M;
    part[16 + row] = Ls;
  }
  float* po = part + 32 + row * D;
  for (int cc = c0; cc < c0 + D / 8; ++cc) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kSdAttnWarps; ++w) a = fmaf(wgt[w], mO[(w * 16 + row) * D + cc], a);
    po[cc] = a;
  }
}

// ---- merge the splits of each (sequence, query head), gate, write bf16
template <int D>
__global__ void __launch_bounds__(D) sd_combine_kernel(const SdParams p) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  if (sd_pos(p, b) < 0) return;
  const int hk = h / p.G, row = h % p.G;
  const float* base = p.part + ((int64_t)b * p.Hkv + hk) * p.nsplit * (16 * (D + 2));
  float M = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, base[s * (16 * (D + 2)) + row]);
  float Ls = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.nsplit; ++s) {
      const float* ps = base + s * (16 * (D + 2));
      const float ms = ps[row];
      if (ms == -INFINITY) continue;  // an empty split carries no O
      const float w = exp2f(ms - M);
      Ls = fmaf(w, ps[16 + row], Ls);
      acc = fmaf(w, ps[32 + row * D + d], acc);
    }
  }
  float y = Ls > 0.f ? acc / Ls : 0.f;
  if (p.g) y *= sigmoidf_(__bfloat162float(p.g[b * p.sg.b + (int64_t)h * p.sg.h + d]));
  if (!(fabsf(y) < INFINITY)) raise_device_error(SALA_ERR_RANGE);  // non-finite input
  p.o[b * p.so.b + (int64_t)h * p.so.h + d] = __float2bfloat16_rn(y);
}

// ---- block means of a filled cache (after a prefill): kbar[b][j][hk] for j < T / 64,
// summed in key order exactly as the prefill selection and the decode step do.
// grid (T / 64, Hkv, B), D threads.
template <int D>
__global__ void __launch_bounds__(D)
sd_block_means_kernel(const __nv_bfloat16* __restrict__ k, sala_strides sk, int nbcap, int Hkv,
                      float* __restrict__ kbar) {
  const int j = blockIdx.x, hk = blockIdx.y, b = blockIdx.z, d = threadIdx.x;
  const __nv_bfloat16* src = k + b * sk.b + (int64_t)j * kSdBlk * sk.t + hk * sk.h + d;
  float acc = 0.f;
#pragma unroll 8
  for (int s = 0; s < kSdBlk; ++s) acc += __bfloat162float(src[(int64_t)s * sk.t]);
  kbar[(((int64_t)b * nbcap + j) * Hkv + hk) * D + d] = acc * (1.0f / kSdBlk);
}

}  // namespace sala
