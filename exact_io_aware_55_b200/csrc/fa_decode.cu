// Split-KV decode: a few new queries (Nq <= 16) attending over a long KV cache.
//
// The glossary page (chipfoundryservices "flash attention", last section)
// pairs the method with the KV cache at inference.  Each (batch-head) cache is
// cut into splits of whole key tiles (128 keys at d = 128, 256 at d = 64, so
// that a tile of K and V is 64 KB either way); a split is one work item, and the
// persistent CTAs (one per SM) take items round-robin.  Per item the online
// softmax runs over the split's tiles exactly as in the square forward, but
// with the product transposed so that the keys of a tile fill the MMA's M
// dimension (one 128-key MMA per sub-tile) and the (padded) 16 queries its N:
//   S^T = K_j Q^T        keys x 16 fp32 in TMEM      (tcgen05, both K-major)
//   P^T = exp2(S^T * scale * log2 e - m)   thread = key; the max over the
//                        tile's keys is a warp redux and a four-warp exchange
//   O^T += V_j^T P^T     d x 16 fp32 in TMEM          (A = V tile MN-major,
//                        B = P^T written to shared memory as bf16)
// The running sum l is kept per thread (per key lane) and reduced once per
// item.  The running max is rescaled lazily (only when a tile raises it by
// more than 2^8), so O^T is rarely touched between MMAs.  An item ends with
// its normalised O and LSE (natural log): written directly when a head is a
// single item, else as fp32 partials that decode_merge_kernel combines by
// their log-sum-exp, O = sum_s exp(LSE_s - LSE) O_s.
//
// Warps: 0 TMA producer (Q per item, K/V tiles through a ring), 1 MMA issuer
// and TMEM owner, 4-7 softmax (TMEM lane quarter = warp % 4), 8-11 epilogue.
// Causal masking is aligned to the end of the cache: query i of Nq sees keys
// j <= Nk - Nq + i.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr int kDecNq = 16;         // query columns = MMA N (Nq <= 16, rest zero)
constexpr int kDecThreads = 384;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

template <int D>
struct DecShape {
  static constexpr int kSub = (D == 64) ? 2 : 1;          // 128-key sub-tiles per tile
  static constexpr int kTileKeys = 128 * kSub;
  static constexpr int kTileBytes = kTileKeys * D * 2;    // K (or V) of one tile: 32 KB
  static constexpr int kStageBytes = 2 * kTileBytes;      // K then V
  static constexpr int kNS = 3;                           // ring depth: 192 KB
  static constexpr int kQBytes = kDecNq * D * 2;          // 16 query rows
  static constexpr int kPBytes = kDecNq * kTileKeys * 2;  // P^T of one tile
  static constexpr int kChunks = D / 64;                  // 128-byte column chunks (16 KB per sub-tile)
  static constexpr int kKSteps = D / 16;                  // S^T k-steps per sub-tile
  static constexpr int kPvSteps = kTileKeys / 16;         // O^T k-steps per tile
  static constexpr uint32_t kIdS = idesc_bf16(128, kDecNq, false, false);   // S^T = K Q^T
  static constexpr uint32_t kIdO = idesc_bf16(D, kDecNq, true, false);      // O^T = V^T P^T
  static constexpr uint32_t kColS = 0;                    // two S^T buffers of 16 * kSub columns
  static constexpr uint32_t kColO = 32 * kSub;            // two O^T buffers of 16 columns
  static constexpr uint32_t kTmemCols = (kColO + 32 <= 64) ? 64 : 128;
};

template <int NS>
struct DecBarriers {
  uint64_t kv_full[NS], kv_empty[NS];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], pv_done[2];
  uint64_t red[2];
  uint64_t o_full[2], o_free[2];
  uint64_t stats_full[2];
  alignas(16) float red_max[2][4][kDecNq];   // per-warp tile maxima (log2 units)
  alignas(16) float stat_m[2][kDecNq];       // item running max
  alignas(16) float stat_l[2][4][kDecNq];    // item per-warp sums
  uint32_t tmem_base;
  uint32_t abort;
};

template <int D>
constexpr size_t dec_smem_bytes() {
  using S = DecShape<D>;
  return 1024 + size_t(S::kNS) * S::kStageBytes + 2 * S::kQBytes + 2 * S::kPBytes + sizeof(DecBarriers<S::kNS>);
}

__device__ __forceinline__ float redux_max(float x) {
  float y;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// Work item -> (batch-head, first tile, tile count).
struct Item {
  int bh, split, t0, nt;
};
__device__ __forceinline__ Item item_of(const DecodeArgs& a, int item) {
  Item r;
  r.bh = item / a.n_split;
  r.split = item - r.bh * a.n_split;
  r.t0 = r.split * a.tiles_per_split;
  r.nt = min(a.tiles_per_head - r.t0, a.tiles_per_split);
  return r;
}

template <int D>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const DecodeArgs a) {
  using S = DecShape<D>;
  constexpr int NS = S::kNS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem;                               // NS x (K tile, V tile)
  uint8_t* sQ = sKV + NS * S::kStageBytes;           // 2 x Q
  uint8_t* sP = sQ + 2 * S::kQBytes;                 // 2 x P^T
  auto* b = reinterpret_cast<DecBarriers<NS>*>(sP + 2 * S::kPBytes);
  const WaitCtx wc{&b->abort, a.status, FA_WAIT_LIMIT_NS};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = a.BH * a.n_split;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&b->kv_full[s], 1);
      mbar_init(&b->kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b->q_full[i], 1);
      mbar_init(&b->q_empty[i], 1);
      mbar_init(&b->s_full[i], 1);
      mbar_init(&b->s_free[i], 4);
      mbar_init(&b->p_full[i], 4);
      mbar_init(&b->pv_done[i], 1);
      mbar_init(&b->red[i], 4);
      mbar_init(&b->o_full[i], 1);
      mbar_init(&b->o_free[i], 4);
      mbar_init(&b->stats_full[i], 4);
    }
    b->abort = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&b->tmem_base, S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = b->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    const uint64_t pol = policy_evict_first();      // the cache is streamed once
    bool ok = true;
    int g = 0, it = 0;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it) {
      const Item w = item_of(a, item);
      const int qb = it & 1;
      if (it >= 2 && !mbar_wait_warp(&b->q_empty[qb], ((it >> 1) + 1) & 1, wc, WAIT_DEC_Q_EMPTY)) break;
      mbar_arrive_expect_tx_e(&b->q_full[qb], S::kQBytes);
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c)
        tma_load_3d_hint_e(sQ + qb * S::kQBytes + c * (kDecNq * 128), &tmQ, &b->q_full[qb], c * 64, 0, w.bh, pol);
      for (int j = 0; j < w.nt; ++j, ++g) {
        const int s = g % NS;
        if (g >= NS && !mbar_wait_warp(&b->kv_empty[s], ((g / NS) + 1) & 1, wc, WAIT_DEC_KV_EMPTY)) {
          ok = false;
          break;
        }
        const int key0 = (w.t0 + j) * S::kTileKeys;
        uint8_t* st = sKV + s * S::kStageBytes;
        mbar_arrive_expect_tx_e(&b->kv_full[s], S::kStageBytes);
#pragma unroll
        for (int u = 0; u < S::kSub; ++u)
#pragma unroll
          for (int c = 0; c < S::kChunks; ++c) {
            const int off = (u * S::kChunks + c) * 16384;
            tma_load_3d_hint_e(st + off, &tmK, &b->kv_full[s], c * 64, key0 + 128 * u, w.bh, pol);
            tma_load_3d_hint_e(st + S::kTileBytes + off, &tmV, &b->kv_full[s], c * 64, key0 + 128 * u, w.bh, pol);
          }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    const uint64_t dK = sdesc_sw128(smem_u32(sKV), 16, 1024);                   // K tiles, K-major (A)
    const uint64_t dV = sdesc_sw128(smem_u32(sKV + S::kTileBytes), 16384, 1024);// V tiles, MN-major (A of O^T)
    const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);                    // Q, K-major (B)
    const uint64_t dP = sdesc_sw128(smem_u32(sP), 16, 1024);                    // P^T, K-major (B)
    bool ok = true;
    int g = 0, it = 0;
    // O^T(ob) (+)= V^T P^T for the tile with ring index gg.
    auto issue_pv = [&](int gg, int ob, bool first) -> bool {
      const int pb = gg & 1;
      if (first && it >= 2 && !mbar_wait_warp(&b->o_free[ob], ((it >> 1) + 1) & 1, wc, WAIT_DEC_O_FREE)) return false;
      if (!mbar_wait_warp(&b->p_full[pb], (gg >> 1) & 1, wc, WAIT_DEC_P)) return false;
      tc_fence_after();
      const int s = gg % NS;
#pragma unroll
      for (int kt = 0; kt < S::kPvSteps; ++kt) {
        const uint64_t va = uint64_t((s * S::kStageBytes + (kt >> 3) * S::kChunks * 16384 + (kt & 7) * 2048) >> 4);
        const uint64_t pb_off = uint64_t((pb * S::kPBytes + (kt >> 2) * 2048 + (kt & 3) * 32) >> 4);
        mma_f16_ss_e(tmem + S::kColO + 16 * ob, dV + va, dP + pb_off, S::kIdO, (!first || kt > 0) ? 1u : 0u);
      }
      tc_commit_e(&b->pv_done[pb]);
      tc_commit_e(&b->kv_empty[s]);
      return true;
    };
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it) {
      const Item w = item_of(a, item);
      const int qb = it & 1, ob = it & 1;
      if (!mbar_wait_warp(&b->q_full[qb], (it >> 1) & 1, wc, WAIT_DEC_Q)) break;
      for (int j = 0; j < w.nt; ++j, ++g) {
        const int s = g % NS, sb = g & 1;
        if (!mbar_wait_warp(&b->kv_full[s], (g / NS) & 1, wc, WAIT_DEC_KV) ||
            (g >= 2 && !mbar_wait_warp(&b->s_free[sb], ((g >> 1) + 1) & 1, wc, WAIT_DEC_S_FREE))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int u = 0; u < S::kSub; ++u)
#pragma unroll
          for (int ks = 0; ks < S::kKSteps; ++ks) {
            const uint64_t ka = uint64_t((s * S::kStageBytes + (u * S::kChunks + (ks >> 2)) * 16384 + (ks & 3) * 32) >> 4);
            const uint64_t qo = uint64_t((qb * S::kQBytes + (ks >> 2) * 2048 + (ks & 3) * 32) >> 4);
            mma_f16_ss_e(tmem + S::kColS + 16 * (sb * S::kSub + u), dK + ka, dQ + qo, S::kIdS, ks > 0 ? 1u : 0u);
          }
        tc_commit_e(&b->s_full[sb]);
        if (j == w.nt - 1) tc_commit_e(&b->q_empty[qb]);
        if (j > 0 && !issue_pv(g - 1, ob, j == 1)) {
          ok = false;
          break;
        }
      }
      if (!ok || !issue_pv(g - 1, ob, w.nt == 1)) break;
      tc_commit_e(&b->o_full[ob]);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------- softmax
    const int wq = warp & 3;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const float cl = a.c_log2;
    const int Nq = a.Nq, Nk = a.Nk;
    bool ok = true;
    int g = 0, it = 0;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++it) {
      const Item w = item_of(a, item);
      const int ob = it & 1;
      float m_used[kDecNq], l_t[kDecNq];
#pragma unroll
      for (int q = 0; q < kDecNq; ++q) {
        m_used[q] = -INFINITY;
        l_t[q] = 0.0f;
      }
      for (int j = 0; j < w.nt; ++j, ++g) {
        const int sb = g & 1;
        if (!mbar_wait_warp(&b->s_full[sb], (g >> 1) & 1, wc, WAIT_DEC_S)) {
          ok = false;
          break;
        }
        tc_fence_after();
        constexpr int U = S::kSub;
        float s[U][kDecNq];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          uint32_t r[16];
          tmem_ld_x16(lane_base + S::kColS + 16 * (sb * U + u), r);
#pragma unroll
          for (int q = 0; q < kDecNq; ++q) s[u][q] = __uint_as_float(r[q]) * cl;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b->s_free[sb]);
        const int tile0 = (w.t0 + j) * S::kTileKeys;
        if (tile0 + S::kTileKeys > Nk || (a.causal && tile0 + S::kTileKeys - 1 > Nk - Nq)) {
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int key = tile0 + 128 * u + wq * 32 + lane;
#pragma unroll
            for (int q = 0; q < kDecNq; ++q)
              if (key >= Nk || (a.causal && key > Nk - Nq + q)) s[u][q] = -INFINITY;
          }
        }
        // tile maximum per query: warp redux, then the four softmax warps
        float* rm = &b->red_max[g & 1][wq][0];
        {
          float wm[kDecNq];
#pragma unroll
          for (int q = 0; q < kDecNq; ++q) {
            float x = s[0][q];
#pragma unroll
            for (int u = 1; u < U; ++u) x = fmaxf(x, s[u][q]);
            wm[q] = redux_max(x);
          }
          if (lane == 0) {
#pragma unroll
            for (int q = 0; q < kDecNq; q += 4)
              *reinterpret_cast<float4*>(rm + q) = make_float4(wm[q], wm[q + 1], wm[q + 2], wm[q + 3]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&b->red[g & 1]);
        if (!mbar_wait_warp(&b->red[g & 1], (g >> 1) & 1, wc, WAIT_DEC_RED)) {
          ok = false;
          break;
        }
        float mt[kDecNq];
        {
          const float* r0 = &b->red_max[g & 1][0][0];
#pragma unroll
          for (int q = 0; q < kDecNq; q += 4) {
            const float4 x0 = *reinterpret_cast<const float4*>(r0 + q);
            const float4 x1 = *reinterpret_cast<const float4*>(r0 + kDecNq + q);
            const float4 x2 = *reinterpret_cast<const float4*>(r0 + 2 * kDecNq + q);
            const float4 x3 = *reinterpret_cast<const float4*>(r0 + 3 * kDecNq + q);
            mt[q] = fmaxf(fmaxf(x0.x, x1.x), fmaxf(x2.x, x3.x));
            mt[q + 1] = fmaxf(fmaxf(x0.y, x1.y), fmaxf(x2.y, x3.y));
            mt[q + 2] = fmaxf(fmaxf(x0.z, x1.z), fmaxf(x2.z, x3.z));
            mt[q + 3] = fmaxf(fmaxf(x0.w, x1.w), fmaxf(x2.w, x3.w));
          }
        }
        bool need = false;
#pragma unroll
        for (int q = 0; q < kDecNq; ++q) need |= mt[q] > m_used[q] + kRescaleThreshold;
        if (need) {   // uniform: every thread holds the same m_used and mt
          float alpha[kDecNq];
#pragma unroll
          for (int q = 0; q < kDecNq; ++q) {
            const float mn = fmaxf(m_used[q], mt[q]);
            alpha[q] = (mn == -INFINITY) ? 1.0f : ex2_approx(m_used[q] - mn);
            m_used[q] = mn;
            l_t[q] *= alpha[q];
          }
          if (j > 0) {   // O^T holds earlier tiles of this item: rescale it once PV(g-1) is done
            if (!mbar_wait_warp(&b->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, wc, WAIT_DEC_PV)) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint32_t o[16];
            tmem_ld_x16(lane_base + S::kColO + 16 * ob, o);
#pragma unroll
            for (int q = 0; q < kDecNq; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha[q]);
            tmem_st_x16(lane_base + S::kColO + 16 * ob, o);
            tmem_wait_st();
          }
        }
        // P^T into shared memory: B operand, K-major, rows = queries, the
        // tile's keys in 64-key chunks of 128-byte swizzled rows.
        const int pb = g & 1;
        if (g >= 2 && !mbar_wait_warp(&b->pv_done[pb], ((g - 2) >> 1) & 1, wc, WAIT_DEC_PV)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int kk = 128 * u + wq * 32 + lane;
          uint8_t* pbase = sP + pb * S::kPBytes + (kk >> 6) * 2048 + (kk & 7) * 2;
          const int unit = (kk & 63) >> 3;
#pragma unroll
          for (int q = 0; q < kDecNq; ++q) {
            const float p = (s[u][q] == -INFINITY) ? 0.0f : ex2_approx(s[u][q] - m_used[q]);
            l_t[q] += p;
            *reinterpret_cast<__nv_bfloat16*>(pbase + (q >> 3) * 1024 + (q & 7) * 128 + ((unit ^ (q & 7)) << 4)) =
                __float2bfloat16_rn(p);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b->p_full[pb]);
      }
      if (!ok) break;
      // Item done: once its last PV has completed (which also orders these
      // writes after the epilogue's read of this stats buffer two items ago),
      // publish the running max and the per-warp sums.
      if (!mbar_wait_warp(&b->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, wc, WAIT_DEC_PV)) break;
      float lw[kDecNq];
#pragma unroll
      for (int q = 0; q < kDecNq; ++q) lw[q] = warp_sum(l_t[q]);
      if (lane == 0) {
#pragma unroll
        for (int q = 0; q < kDecNq; q += 4) {
          *reinterpret_cast<float4*>(&b->stat_l[ob][wq][q]) = make_float4(lw[q], lw[q + 1], lw[q + 2], lw[q + 3]);
          if (wq == 0)
            *reinterpret_cast<float4*>(&b->stat_m[ob][q]) =
                make_float4(m_used[q], m_used[q + 1], m_used[q + 2], m_used[q + 3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&b->stats_full[ob]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue
    const int wq = warp & 3;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    // O^T row (= output column) held by this thread: M = d = 128 uses every
    // lane; M = 64 puts rows 16w..16w+15 in lanes 0-15 of quarter w.
    const int drow = (D == 128) ? wq * 32 + lane : (lane < 16 ? wq * 16 + lane : -1);
    const int Nq = a.Nq;
    const bool single = a.n_split == 1;
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
      const Item w = item_of(a, item);
      const int ob = it & 1;
      if (!mbar_wait_warp(&b->o_full[ob], (it >> 1) & 1, wc, WAIT_DEC_O) ||
          !mbar_wait_warp(&b->stats_full[ob], (it >> 1) & 1, wc, WAIT_DEC_STATS))
        break;
      tc_fence_after();
      uint32_t o[16];
      tmem_ld_x16(lane_base + S::kColO + 16 * ob, o);
      float L[kDecNq], M[kDecNq];
#pragma unroll
      for (int q = 0; q < kDecNq; ++q) {
        L[q] = b->stat_l[ob][0][q] + b->stat_l[ob][1][q] + b->stat_l[ob][2][q] + b->stat_l[ob][3][q];
        M[q] = b->stat_m[ob][q];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b->o_free[ob]);
      if (drow >= 0) {
#pragma unroll
        for (int q = 0; q < kDecNq; ++q) {
          if (q < Nq) {
            const float val = (L[q] > 0.0f) ? __uint_as_float(o[q]) / L[q] : 0.0f;
            const float lse = (L[q] > 0.0f) ? (M[q] + lg2_approx(L[q])) * kLn2 : -INFINITY;
            if (single) {
              reinterpret_cast<__nv_bfloat16*>(a.o)[(size_t(w.bh) * Nq + q) * D + drow] = __float2bfloat16_rn(val);
              if (drow == 0) a.lse[size_t(w.bh) * Nq + q] = lse;
            } else {
              const size_t part = (size_t(w.bh) * a.n_split + w.split) * Nq + q;
              a.part_o[part * D + drow] = val;
              if (drow == 0) a.part_lse[part] = lse;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

// O = sum_s exp(LSE_s - LSE) O_s with LSE = log sum_s exp(LSE_s).  One block
// per (query, batch-head); thread = (output column, one of kParts interleaved
// subsets of the splits), the subsets summed through shared memory.
constexpr int kMergeThreads = 256;

template <int D>
__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(const DecodeArgs a) {
  constexpr int kParts = kMergeThreads / D;
  __shared__ float red[kMergeThreads / 32];
  __shared__ float acc_s[kParts][D];
  __shared__ float l_s[kParts];
  const int q = blockIdx.x, bh = blockIdx.y;
  const int Nq = a.Nq, ns = a.n_split;
  const int c = threadIdx.x % D, part = threadIdx.x / D;
  const float* pl = a.part_lse + size_t(bh) * ns * Nq + q;            // split stride Nq
  const float* po = a.part_o + (size_t(bh) * ns * Nq + q) * D + c;    // split stride Nq * D
  float m = -INFINITY;
  for (int s = threadIdx.x; s < ns; s += kMergeThreads) m = fmaxf(m, pl[size_t(s) * Nq]);
  m = redux_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kMergeThreads / 32; ++w) m = fmaxf(m, red[w]);
  float L = 0.0f, acc = 0.0f;
  if (m != -INFINITY) {
#pragma unroll 4
    for (int s = part; s < ns; s += kParts) {
      const float wgt = __expf(pl[size_t(s) * Nq] - m);
      L += wgt;
      acc = fmaf(wgt, po[size_t(s) * Nq * D], acc);
    }
  }
  acc_s[part][c] = acc;
  if (c == 0) l_s[part] = L;
  __syncthreads();
  if (part == 0) {
    float at = 0.0f, lt = 0.0f;
#pragma unroll
    for (int p = 0; p < kParts; ++p) {
      at += acc_s[p][c];
      lt += l_s[p];
    }
    reinterpret_cast<__nv_bfloat16*>(a.o)[(size_t(bh) * Nq + q) * D + c] = __float2bfloat16_rn(lt > 0.0f ? at / lt : 0.0f);
    if (c == 0) a.lse[size_t(bh) * Nq + q] = (lt > 0.0f) ? m + __logf(lt) : -INFINITY;
  }
}

template <int D>
cudaError_t launch_decode_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const DecodeArgs& a, int grid, cudaStream_t stream) {
  constexpr size_t smem = dec_smem_bytes<D>();
  static_assert(smem <= 227 * 1024, "shared memory budget");
  auto kern = decode_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kDecThreads, smem, stream>>>(tq, tk, tv, a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.n_split == 1) return e;
  decode_merge_kernel<D><<<dim3(a.Nq, a.BH), kMergeThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const DecodeArgs& a, int d, int grid, cudaStream_t stream) {
  return d == 64 ? launch_decode_t<64>(tq, tk, tv, a, grid, stream)
                 : launch_decode_t<128>(tq, tk, tv, a, grid, stream);
}

}  // namespace fa
