// sparse_attn_tc.cuh -- block-sparse softmax attention on tcgen05 (head_dim 128).
//
// Same operation as sparse_attn.cuh (InfLLM-v2 style sparse layer, MiniCPM-SALA
// tech-report mirror, section 02 (2) and (4): each query row of KV head hk attends
// to the union of its selected 64-key blocks, keys s <= t, the GQA group shares the
// selection, NoPE, optional sigmoid gate).
//
// Keys as the M dimension.  A row has only G <= 16 query heads, below tcgen05's
// minimum M, so the MMAs are transposed: for every PAIR of selected blocks
// (128 keys)
//     S^T [128 keys x 16 heads]  = K_pair . Q^T          (M = 128, N = 16)
//     O^T [128 dims x 32]       += V^T . P^T              (M = 128, N = 32)
// with K, V used exactly as TMA lands them (128-byte swizzle; V^T is the MN-major
// view of the V tile) and P^T holding the softmax weights split into bf16 high and
// low parts (columns 0-15 and 16-31 of O^T), so the weights keep 2^-16 relative
// precision.  Accumulators live in tensor memory, so the softmax warps hold no
// accumulator registers.
//
// Roles (320 threads): warps 0-7 softmax + epilogue (thread = TMEM lane: a key of the
// pair, later a head dimension; warps w and w+4 share the lanes and take heads 0-7 and
// 8-15), warp 8 TMA producer, warp 9 MMA issuer.  The
// softmax keeps a per-head reference maximum that is raised only when a score
// exceeds it by more than 2^8 (then O^T and the running sums are rescaled); row sums
// accumulate per thread and are reduced once per row.  S^T, P^T, Q and O^T are
// double-buffered; K/V pairs stream through an NS-deep ring.  All waits are bounded.
#pragma once

#include "sparse_attn.cuh"

namespace sala {

constexpr int kStNS = 3;                  // K ring and V ring depth (pairs)
constexpr int kStThreads = 320;          // 8 softmax warps, producer, MMA issuer
constexpr int kStSoft = 256;
constexpr int kStHalf = 128 * 128;        // [128 rows x 64 cols] bf16 slab: 16 KB
constexpr int kStTile = 2 * kStHalf;      // K or V of a pair: d-half 0, d-half 1 (32 KB)
constexpr int kStPBuf = 2 * 32 * 128;     // P^T: two 64-key halves of [32 rows x 128 B]
constexpr int kStQBuf = 2 * 16 * 128;     // Q: two 64-dim halves of [16 heads x 128 B]
constexpr int kStMaxSel = 256;            // selected-block list capacity of one row
constexpr float kStLazy = 8.0f;

struct StSmem {
  static constexpr size_t kKRing = 0;
  static constexpr size_t kVRing = kKRing + size_t(kStNS) * kStTile;
  static constexpr size_t kP = kVRing + size_t(kStNS) * kStTile;
  static constexpr size_t kQ = kP + 2 * kStPBuf;
  static constexpr size_t kList = kQ + 2 * kStQBuf;
  static constexpr size_t kRed = kList + kStMaxSel * 4;     // [4][16] floats
  static constexpr size_t kFlag = kRed + 4 * 16 * 4;        // [16] ints
  static constexpr size_t kBars = kFlag + 64;
  static constexpr int kNumBars = 4 * kStNS + 16;
  static constexpr size_t kSlot = kBars + kNumBars * 8;
  static constexpr size_t bytes = 1024 + kSlot + 16;
};

__device__ __forceinline__ uint64_t st_desc_k(uint32_t base, int kk, uint32_t half_bytes) {
  return umma_desc_sw128(base + (kk >> 2) * half_bytes + (kk & 3) * 32, 16, 1024);
}

__global__ void __launch_bounds__(kStThreads, 1)
sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const SaParams p) {
  constexpr uint32_t kIdQK = umma_idesc_bf16(128, 16, false, false);
  constexpr uint32_t kIdPV = umma_idesc_bf16(128, 32, true, false);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* kring = smem + StSmem::kKRing;
  uint8_t* vring = smem + StSmem::kVRing;
  uint8_t* pbuf = smem + StSmem::kP;
  uint8_t* qbuf = smem + StSmem::kQ;
  int32_t* list = reinterpret_cast<int32_t*>(smem + StSmem::kList);
  float* red = reinterpret_cast<float*>(smem + StSmem::kRed);
  volatile int* flags = reinterpret_cast<volatile int*>(smem + StSmem::kFlag);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + StSmem::kBars);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + kStNS;
  uint64_t* v_full = k_empty + kStNS;
  uint64_t* v_empty = v_full + kStNS;
  uint64_t* q_full = v_empty + kStNS;    // [2]
  uint64_t* q_empty = q_full + 2;        // [2]
  uint64_t* s_full = q_empty + 2;        // [2]
  uint64_t* s_free = s_full + 2;         // [2]
  uint64_t* p_ready = s_free + 2;        // [2]
  uint64_t* p_free = p_ready + 2;        // [2]
  uint64_t* o_full = p_free + 2;         // [2]
  uint64_t* o_free = o_full + 2;         // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + StSmem::kSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStNS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kStSoft / 32);
      mbar_init(&p_ready[i], kStSoft / 32);
      mbar_init(&p_free[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], kStSoft / 32);
    }
    for (int i = 0; i < 8; ++i) flags[i] = 0;  // abort flag, vote slots, block count
    fence_mbar_init();
  }
  if (warp == 9) tc_alloc(tmem_slot, 128);
  // Q rows past the group (G < 16) are never loaded: keep them zero
  for (int i = tid; i < 2 * kStQBuf / 16; i += kStThreads)
    reinterpret_cast<uint4*>(qbuf)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // columns: S^T[2] at 0 / 16 (16 each), O^T[2] at 32 / 64 (32 each)
  const int64_t T = p.T;

  // live blocks of row r, in idx order (each role derives the same sequence)
  auto row_coords = [&](int64_t r, int64_t& t, int& hk, int& b) {
    t = r % T;
    hk = (int)((r / T) % p.Hkv);
    b = (int)(r / (T * p.Hkv));
  };

  if (warp == 8) {
    // ------------------------------------------------------------------ producer
    // lane 0 streams Q and the K ring, lane 1 the V ring, so K can run ahead of V
    if (lane < 2) {
      const bool is_k = lane == 0;
      if (is_k) {
        prefetch_tmap(&tmq);
        prefetch_tmap(&tmk);
      } else {
        prefetch_tmap(&tmv);
      }
      uint32_t it = 0, qrow = 0;
      bool ok = true;
      uint64_t* fullb = is_k ? k_full : v_full;
      uint64_t* emptyb = is_k ? k_empty : v_empty;
      uint8_t* ring = is_k ? kring : vring;
      const CUtensorMap* map = is_k ? &tmk : &tmv;
      for (int64_t r = blockIdx.x; r < p.rows && ok; r += gridDim.x) {
        int64_t t; int hk, b;
        row_coords(r, t, hk, b);
        const int32_t* ir = p.idx + r * p.n_sel;
        int nblk = 0;
        for (int e = 0; e < p.n_sel; ++e) nblk += sa_block_live(__ldg(ir + e), t);
        if (nblk == 0) continue;
        if (is_k) {
          const int qs = qrow & 1;
          if (flags[0] || !mbar_wait(&q_empty[qs], ((qrow >> 1) & 1) ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[qs], 2 * 128 * p.q_box_h);
          tma_load_4d(qbuf + qs * kStQBuf, &tmq, &q_full[qs], 0, hk * p.G, (int)t, b);
          tma_load_4d(qbuf + qs * kStQBuf + 2048, &tmq, &q_full[qs], 64, hk * p.G, (int)t, b);
          ++qrow;
        }
        int e = 0, got = 0;
        while (got < nblk && ok) {
          int jA = -1, jB = -1;
          while (jA < 0) { const int j = __ldg(ir + e++); if (sa_block_live(j, t)) jA = j; }
          ++got;
          if (got < nblk) {
            while (jB < 0) { const int j = __ldg(ir + e++); if (sa_block_live(j, t)) jB = j; }
            ++got;
          } else {
            jB = jA;  // odd tail: repeat a real block; its keys are masked out
          }
          const int s = it % kStNS;
          if (flags[0] || !mbar_wait(&emptyb[s], ((it / kStNS) & 1) ^ 1)) { ok = false; break; }
          uint8_t* st = ring + size_t(s) * kStTile;
          mbar_arrive_expect_tx(&fullb[s], kStTile);
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_4d(st + hf * kStHalf, map, &fullb[s], hf * 64, hk, jA * kSaBlk, b);
            tma_load_4d(st + hf * kStHalf + 8192, map, &fullb[s], hf * 64, hk, jB * kSaBlk, b);
          }
          ++it;
        }
      }
      if (!ok) flags[0] = 1;
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t pr = 0, qrow = 0, orow = 0;
      bool ok = true;
      // the previous pair's P.V, issued after the next pair's Q.K^T
      bool have_prev = false;
      uint32_t pv_pr = 0, pv_orow = 0;
      bool pv_first = false, pv_last = false;
      auto issue_pv = [&]() -> bool {
        const uint32_t pb = pv_pr & 1, ob = pv_orow & 1, vs = pv_pr % kStNS;
        if (!mbar_wait(&v_full[vs], (pv_pr / kStNS) & 1)) return false;
        if (!mbar_wait(&p_ready[pb], (pv_pr >> 1) & 1)) return false;
        if (pv_first && !mbar_wait(&o_free[ob], ((pv_orow >> 1) & 1) ^ 1)) return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(vring + size_t(vs) * kStTile);
        const uint32_t pbb = smem_u32(pbuf + pb * kStPBuf);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma_ss(tmem + 32 + 32 * ob, umma_desc_sw128(vb + kk * 2048, kStHalf, 1024),
                    st_desc_k(pbb, kk, 4096), kIdPV, (pv_first && kk == 0) ? 0u : 1u);
        tc_commit(&v_empty[vs]);
        tc_commit(&p_free[pb]);
        if (pv_last) tc_commit(&o_full[ob]);
        return true;
      };
      for (int64_t r = blockIdx.x; r < p.rows && ok; r += gridDim.x) {
        int64_t t; int hk, b;
        row_coords(r, t, hk, b);
        const int32_t* ir = p.idx + r * p.n_sel;
        int nblk = 0;
        for (int e = 0; e < p.n_sel; ++e) nblk += sa_block_live(__ldg(ir + e), t);
        if (nblk == 0) continue;
        const int npairs = (nblk + 1) >> 1;
        const uint32_t qs = qrow & 1;
        if (flags[0] || !mbar_wait(&q_full[qs], (qrow >> 1) & 1)) { ok = false; break; }
        for (int i = 0; i < npairs; ++i) {
          const uint32_t s = pr % kStNS, sb = pr & 1;
          if (!mbar_wait(&k_full[s], (pr / kStNS) & 1) ||
              !mbar_wait(&s_free[sb], ((pr >> 1) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kb = smem_u32(kring + size_t(s) * kStTile);
          const uint32_t qb = smem_u32(qbuf + qs * kStQBuf);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_ss(tmem + 16 * sb, st_desc_k(kb, kk, kStHalf), st_desc_k(qb, kk, 2048), kIdQK,
                      kk > 0);
          tc_commit(&s_full[sb]);
          tc_commit(&k_empty[s]);
          if (i == npairs - 1) tc_commit(&q_empty[qs]);
          if (have_prev && !issue_pv()) { ok = false; break; }
          have_prev = true;
          pv_pr = pr; pv_orow = orow;
          pv_first = (i == 0); pv_last = (i == npairs - 1);
          ++pr;
        }
        ++qrow;
        ++orow;
      }
      if (ok && have_prev && !issue_pv()) ok = false;
      if (!ok) flags[0] = 1;
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int kl = tid & 127;       // key of the pair (softmax) / head dimension (epilogue)
    const int hh = tid >> 7;        // head half: heads 8*hh .. 8*hh+7
    const int wq = warp & 3;        // TMEM lane quadrant
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    uint32_t pr = 0, orow = 0;
    int vote = 0;                   // cross-warp votes taken so far
    bool ok = true;
    for (int64_t r = blockIdx.x; r < p.rows && ok; r += gridDim.x) {
      int64_t t; int hk, b;
      row_coords(r, t, hk, b);
      // compact the row's live blocks into shared memory (warp 0), count them
      named_bar_sync(1, kStSoft);  // previous row finished reading the list
      if (warp == 0) {
        const int32_t* ir = p.idx + r * p.n_sel;
        int base = 0;
        for (int e0 = 0; e0 < p.n_sel; e0 += 32) {
          const int e = e0 + lane;
          const int j = e < p.n_sel ? __ldg(ir + e) : -1;
          const bool live = e < p.n_sel && sa_block_live(j, t);
          const uint32_t m = __ballot_sync(0xffffffffu, live);
          if (live) list[base + __popc(m & ((1u << lane) - 1u))] = j;
          base += __popc(m);
        }
        if (lane == 0) flags[7] = base;
      }
      named_bar_sync(1, kStSoft);
      const int nblk = flags[7];
      const int npairs = (nblk + 1) >> 1;
      const int d = kl;
      const int h0 = 8 * hh;
      // gate of this thread's dimension for its 8 heads (prefetched)
      uint32_t graw[4] = {};
      if (p.g != nullptr && nblk > 0) {
        const __nv_bfloat16* gr =
            p.g + b * p.sg.b + t * p.sg.t + (int64_t)(hk * p.G + h0) * p.sg.h + d;
#pragma unroll
        for (int h = 0; h < 8; h += 2) {
          const uint16_t a = h0 + h < p.G ? __ldg(reinterpret_cast<const uint16_t*>(gr + (int64_t)h * p.sg.h)) : 0;
          const uint16_t c = h0 + h + 1 < p.G ? __ldg(reinterpret_cast<const uint16_t*>(gr + (int64_t)(h + 1) * p.sg.h)) : 0;
          graw[h >> 1] = (uint32_t)a | ((uint32_t)c << 16);
        }
      }
      __nv_bfloat16* orow_ptr =
          p.o + b * p.so.b + t * p.so.t + (int64_t)(hk * p.G + h0) * p.so.h + d;
      if (nblk == 0) {
        for (int h = 0; h < 8 && h0 + h < p.G; ++h)
          orow_ptr[(int64_t)h * p.so.h] = __float2bfloat16_rn(0.f);
        continue;
      }
      float m_ref[8], l_part[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) { m_ref[h] = -INFINITY; l_part[h] = 0.f; }
      const uint32_t ob = orow & 1;
      const uint32_t t_o = tmem + 32 + 32 * ob + lane_off;
      for (int i = 0; i < npairs && ok; ++i) {
        const uint32_t sb = pr & 1;
        if (!mbar_wait(&s_full[sb], (pr >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[8];
        tc_ld8(tmem + 16 * sb + h0 + lane_off, sv);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        const int jA = list[2 * i];
        const int jB = (2 * i + 1 < nblk) ? list[2 * i + 1] : -1;
        const int64_t key = kl < 64 ? (int64_t)jA * kSaBlk + kl
                                    : (jB >= 0 ? (int64_t)jB * kSaBlk + kl - 64 : INT64_MAX);
        const bool valid = key <= t;
        float x[8];
        bool raise = false;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          x[h] = valid ? __uint_as_float(sv[h]) * p.scale_log2 : -INFINITY;
          raise |= x[h] > m_ref[h] + kStLazy;
        }
        // cross-warp vote: raise the reference maximum if any score needs it.  Three
        // rotating slots; the slot of vote n-2 is cleared before vote n's barrier.
        const int slot = 1 + vote % 3;
        if (tid == 0) flags[1 + (vote + 1) % 3] = 0;
        if (__any_sync(0xffffffffu, raise) && lane == 0) flags[slot] = 1;
        named_bar_sync(1, kStSoft);
        const bool any_raise = flags[slot] != 0;
        ++vote;
        if (any_raise) {
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            float mh = x[h];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mh = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, off));
            if (lane == 0) red[wq * 16 + h0 + h] = mh;
          }
          named_bar_sync(1, kStSoft);
          float alpha[8];
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const int hd = h0 + h;
            const float bm = fmaxf(fmaxf(red[hd], red[16 + hd]), fmaxf(red[32 + hd], red[48 + hd]));
            const float nm = fmaxf(m_ref[h], bm);
            alpha[h] = (nm == -INFINITY || m_ref[h] == -INFINITY) ? 0.f : exp2f(m_ref[h] - nm);
            if (m_ref[h] == nm) alpha[h] = 1.f;
            m_ref[h] = nm;
            l_part[h] *= alpha[h];
          }
          named_bar_sync(1, kStSoft);  // everyone read red[]
          if (i > 0) {
            // rescale this row's partial O^T once the previous pair's P.V has landed
            const uint32_t pp = pr - 1;
            if (!mbar_wait(&p_free[pp & 1], (pp >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            uint32_t ohi[8], olo[8];
            tc_ld8(t_o + h0, ohi);
            tc_ld8(t_o + 16 + h0, olo);
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < 8; ++h) {
              ohi[h] = __float_as_uint(__uint_as_float(ohi[h]) * alpha[h]);
              olo[h] = __float_as_uint(__uint_as_float(olo[h]) * alpha[h]);
            }
            tc_st8(t_o + h0, ohi);
            tc_st8(t_o + 16 + h0, olo);
            tc_wait_st();
            tc_fence_before();
          }
        }
        // P^T (bf16 high / low parts) for this key and these heads
        if (pr >= 2 && !mbar_wait(&p_free[sb], ((pr >> 1) & 1) ^ 1)) { ok = false; break; }
        uint8_t* pt = pbuf + sb * kStPBuf + (kl >> 6) * 4096;
        const int kk = kl & 63;
        const uint32_t col = (uint32_t)(kk & 7) << 1;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const float mu = m_ref[h] == -INFINITY ? 0.f : m_ref[h];
          const float pv = exp2f(x[h] - mu);
          l_part[h] += pv;
          const __nv_bfloat16 hi = __float2bfloat16_rn(pv);
          const __nv_bfloat16 lo = __float2bfloat16_rn(pv - __bfloat162float(hi));
          const uint32_t n0 = h0 + h, n1 = 16 + h0 + h;
          *reinterpret_cast<__nv_bfloat16*>(pt + n0 * 128 + ((((kk >> 3) ^ (n0 & 7)) << 4) | col)) = hi;
          *reinterpret_cast<__nv_bfloat16*>(pt + n1 * 128 + ((((kk >> 3) ^ (n1 & 7)) << 4) | col)) = lo;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_ready[sb]);
        ++pr;
      }
      if (!ok) break;
      // ---- epilogue: row sums, normalise, gate, store
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        float ls = l_part[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        if (lane == 0) red[wq * 16 + h0 + h] = ls;
      }
      named_bar_sync(1, kStSoft);
      float inv_l[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const int hd = h0 + h;
        const float L = red[hd] + red[16 + hd] + red[32 + hd] + red[48 + hd];
        inv_l[h] = L > 0.f ? 1.0f / L : 0.f;
      }
      if (!mbar_wait(&o_full[ob], (orow >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      uint32_t ohi[8], olo[8];
      tc_ld8(t_o + h0, ohi);
      tc_ld8(t_o + 16 + h0, olo);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[ob]);
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        if (h0 + h < p.G) {
          float y = (__uint_as_float(ohi[h]) + __uint_as_float(olo[h])) * inv_l[h];
          if (p.g != nullptr) {
            const uint32_t gbits = (graw[h >> 1] >> (16 * (h & 1))) & 0xffffu;
            y *= sigmoidf_(__uint_as_float(gbits << 16));
          }
          orow_ptr[(int64_t)h * p.so.h] = __float2bfloat16_rn(y);
        }
      }
      ++orow;
    }
    if (!ok) flags[0] = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tc_dealloc(tmem, 128);
  }
}

}  // namespace sala
