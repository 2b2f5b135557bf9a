// Deterministic dQ pass of the backward (no atomics).
//
// Same method as bwd_kernel (explainers.rudrite.com "flash-attention-anatomy",
// Q&A "How does FlashAttention save memory in the backward pass?": recompute
// S and P tile by tile from Q, K and the saved LSE), organised around the
// query tile instead of the key tile, so that each dQ row is produced by one
// CTA and written once:
//   for every key tile j (up to the diagonal when causal):
//     S  = Q_i K_j^T          -> TMEM [0,128)       (tcgen05, smem x smem)
//     dP = dO_i V_j^T         -> TMEM [128,256)
//     P  = exp2(S * scale * log2e - LSE2_q)          (thread = query row)
//     dS = scale * P o (dP - D_q)   -> TMEM [256,320) as bf16
//     dQ_i += dS K_j          -> TMEM [320,320+d)   (A = dS from TMEM, K MN-major)
//   dQ_i -> bf16 once.
// Because the thread owns a query row, its LSE and D are two scalars.
// Warps: 0 TMA producer (Q_i, dO_i once; K_j, V_j through a ring), 1 MMA
// issuer and TMEM owner, 4-7 and 8-11 two elementwise warpgroups, each
// handling 64 of the 128 keys of a tile and half of dQ's columns.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 384;

template <int D>
struct DqShape {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kChunks = D / 64;
  static constexpr int kNST = (D == 64) ? 4 : 2;             // K/V ring depth
  static constexpr int kKSteps = D / 16;
  static constexpr uint32_t kIdSS = idesc_bf16(128, 128, false, false);   // S, dP
  static constexpr uint32_t kIdDQ = idesc_bf16(128, D, false, true);      // dQ += dS K (K MN-major)
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDS = 256, kColDQ = 320;
  static_assert(kColDQ + D <= 512, "TMEM budget");
};

template <int NST>
struct DqBarriers {
  uint64_t qdo_full;
  uint64_t k_full[NST], v_full[NST], kv_empty[NST];
  uint64_t s_full, dp_full, s_free, dp_free, ds_full, ds_free, final_;
  uint32_t tmem_base;
  uint32_t abort;
};

template <int D>
constexpr size_t dq_smem_bytes() {
  using S = DqShape<D>;
  return 1024 + size_t(2 + 2 * S::kNST) * S::kTileBytes + sizeof(DqBarriers<S::kNST>);
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdArgs args) {
  using S = DqShape<D>;
  constexpr int NST = S::kNST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + S::kTileBytes;
  uint8_t* sK = sdO + S::kTileBytes;
  uint8_t* sV = sK + NST * S::kTileBytes;
  auto* bars = reinterpret_cast<DqBarriers<NST>*>(sV + NST * S::kTileBytes);
  const WaitCtx wc{&bars->abort, args.status, FA_WAIT_LIMIT_NS};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = args.N;
  const int n_kv = (N + kTile - 1) / kTile;
  // Grid: x = query tile (fastest), y = batch-head; causal: a 1-D grid, the
  // heaviest query tiles (the last ones) first across each group of heads.
  int i, bh;                                           // query tile i (the last = heaviest when causal)
  if constexpr (CAUSAL) {
    int rank;
    causal_block_order(int(blockIdx.x), int((args.N + kTile - 1) / kTile), args.BH, args.head_group, rank, bh);
    i = (args.N + kTile - 1) / kTile - 1 - rank;
  } else {
    i = blockIdx.x;
    bh = blockIdx.y;
  }
  const int T = CAUSAL ? min(n_kv, i + 1) : n_kv;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qdo_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->s_free, 8);
    mbar_init(&bars->dp_free, 8);
    mbar_init(&bars->ds_full, 8);
    mbar_init(&bars->ds_free, 1);
    mbar_init(&bars->final_, 1);
    bars->abort = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmdO);
    const uint64_t pol_q = policy_evict_first();
    const uint64_t pol_kv = policy_evict_last();
    mbar_arrive_expect_tx_e(&bars->qdo_full, 2 * S::kTileBytes);
#pragma unroll
    for (int c = 0; c < S::kChunks; ++c) {
      tma_load_3d_hint_e(sQ + c * 16384, &tmQ, &bars->qdo_full, c * 64, i * kTile, bh, pol_q);
      tma_load_3d_hint_e(sdO + c * 16384, &tmdO, &bars->qdo_full, c * 64, i * kTile, bh, pol_q);
    }
    for (int j = 0; j < T; ++j) {
      const int s = j % NST;
      if (j >= NST) {
        if (!mbar_wait_warp(&bars->kv_empty[s], ((j / NST) + 1) & 1, wc, WAIT_DQ_KV_EMPTY)) break;
      }
      mbar_arrive_expect_tx_e(&bars->k_full[s], S::kTileBytes);
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c)
        tma_load_3d_hint_e(sK + s * S::kTileBytes + c * 16384, &tmK, &bars->k_full[s], c * 64, j * kTile, bh, pol_kv);
      mbar_arrive_expect_tx_e(&bars->v_full[s], S::kTileBytes);
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c)
        tma_load_3d_hint_e(sV + s * S::kTileBytes + c * 16384, &tmV, &bars->v_full[s], c * 64, j * kTile, bh, pol_kv);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    const uint64_t dQ_k = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t ddO_k = sdesc_sw128(smem_u32(sdO), 16, 1024);
    const uint64_t dK_k = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dV_k = sdesc_sw128(smem_u32(sV), 16, 1024);
    const uint64_t dK_mn = sdesc_sw128(smem_u32(sK), 16384, 1024);
    constexpr uint64_t kTileD = uint64_t(S::kTileBytes >> 4);
    auto issue_xt = [&](uint32_t d_tmem, uint64_t a, uint64_t b) {   // A B^T over d, both K-major
#pragma unroll
      for (int ks = 0; ks < S::kKSteps; ++ks) {
        const uint64_t off = uint64_t(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
        mma_f16_ss_e(d_tmem, a + off, b + off, S::kIdSS, ks > 0 ? 1u : 0u);
      }
    };
    bool ok = mbar_wait_warp(&bars->qdo_full, 0, wc, WAIT_DQ_QDO) &&
              mbar_wait_warp(&bars->k_full[0], 0, wc, WAIT_DQ_K) && mbar_wait_warp(&bars->v_full[0], 0, wc, WAIT_DQ_V);
    if (ok) {
      tc_fence_after();
      issue_xt(tmem + S::kColS, dQ_k, dK_k);          // S(0)
      tc_commit_e(&bars->s_full);
      issue_xt(tmem + S::kColDP, ddO_k, dV_k);        // dP(0)
      tc_commit_e(&bars->dp_full);
      for (int j = 0; j < T && ok; ++j) {
        const int s = j % NST;
        if (j + 1 < T) {                              // next S once the groups hold S(j) in registers
          const int sn = (j + 1) % NST;
          if (!mbar_wait_warp(&bars->s_free, j & 1, wc, WAIT_DQ_SFREE) ||
              !mbar_wait_warp(&bars->k_full[sn], ((j + 1) / NST) & 1, wc, WAIT_DQ_K)) { ok = false; break; }
          tc_fence_after();
          issue_xt(tmem + S::kColS, dQ_k, dK_k + uint64_t(sn) * kTileD);
          tc_commit_e(&bars->s_full);
        }
        if (!mbar_wait_warp(&bars->ds_full, j & 1, wc, WAIT_DQ_DS)) { ok = false; break; }
        tc_fence_after();
        // dQ += dS K_j: A = dS (TMEM, bf16: keys 0-63 in columns [256,288), 64-127 in [288,320)),
        // B = K_j MN-major (N = d); 16 keys per step.
#pragma unroll
        for (int kt = 0; kt < 8; ++kt)
          mma_f16_ts_e(tmem + S::kColDQ, tmem + S::kColDS + kt * 8, dK_mn + uint64_t(s) * kTileD + uint64_t(kt * 128),
                       S::kIdDQ, (j > 0 || kt > 0) ? 1u : 0u);
        tc_commit_e(&bars->ds_free);
        if (j + 1 < T) {                              // next dP once the groups hold dP(j)
          const int sn = (j + 1) % NST;
          if (!mbar_wait_warp(&bars->dp_free, j & 1, wc, WAIT_DQ_DPFREE) ||
              !mbar_wait_warp(&bars->v_full[sn], ((j + 1) / NST) & 1, wc, WAIT_DQ_V)) { ok = false; break; }
          tc_fence_after();
          issue_xt(tmem + S::kColDP, ddO_k, dV_k + uint64_t(sn) * kTileD);
          tc_commit_e(&bars->dp_full);
        }
        tc_commit_e(&bars->kv_empty[s]);
      }
      tc_commit_e(&bars->final_);
      if (ok) (void)mbar_wait_warp(&bars->final_, 0, wc, WAIT_DQ_FINAL);
    }
  } else if (warp >= 4) {
    // --------------------------------------------------- elementwise groups
    const int h = (warp - 4) >> 2;                    // keys [64h, 64h+64) of every tile
    const int wq = warp & 3;
    const int r = wq * 32 + lane;                     // query row within the tile
    const int q = i * kTile + r;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const size_t srow = size_t(bh) * args.Np + size_t(q);
    const float nl = args.neg_lse2[srow];             // -LSE*log2e (-inf on padded rows)
    const float nd = args.neg_dvec[srow];             // -D
    const float cl = args.c_log2, scale = args.dq_scale;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const bool diag = CAUSAL && (j == i);
      const bool ragged = (j + 1) * kTile > N;
      const int k0 = j * kTile + 64 * h;
      float p[64];
      if (!mbar_wait_warp(&bars->s_full, j & 1, wc, WAIT_DQ_S)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t rr[64];
        tmem_ld_x64(lane_base + S::kColS + 64 * h, rr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free);
        const float2 cc = make_float2(cl, cl), nl2 = make_float2(nl, nl);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float2 x = ffma2(make_float2(__uint_as_float(rr[2 * t]), __uint_as_float(rr[2 * t + 1])), cc, nl2);
          p[2 * t] = ex2_approx(x.x);
          p[2 * t + 1] = ex2_approx(x.y);
        }
      }
      if (diag || ragged) {
        const int lim = CAUSAL ? min(N - 1, q) : (N - 1);
#pragma unroll
        for (int t = 0; t < 64; ++t)
          if (k0 + t > lim) p[t] = 0.0f;
      }
      if (!mbar_wait_warp(&bars->dp_full, j & 1, wc, WAIT_DQ_DP)) { ok = false; break; }
      tc_fence_after();
      uint32_t w[32];
      {
        uint32_t rr[64];
        tmem_ld_x64(lane_base + S::kColDP + 64 * h, rr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->dp_free);
        const float2 nd2 = make_float2(nd, nd), sc2 = make_float2(scale, scale);
        const float2 dps = make_float2(args.dp_scale, args.dp_scale);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float2 dpm = ffma2(make_float2(__uint_as_float(rr[2 * t]), __uint_as_float(rr[2 * t + 1])), dps, nd2);
          const float2 ds = fmul2(fmul2(make_float2(p[2 * t], p[2 * t + 1]), sc2), dpm);
          w[t] = pack_bf16x2(ds.x, ds.y);
        }
      }
      if (j > 0 && !mbar_wait_warp(&bars->ds_free, (j - 1) & 1, wc, WAIT_DQ_DSFREE)) { ok = false; break; }
      tc_fence_after();
      tmem_st_x32(lane_base + S::kColDS + 32 * h, w);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_full);
    }
    // Epilogue: group h stores dQ columns [h*d/2, (h+1)*d/2) of its rows.
    if (ok && mbar_wait_warp(&bars->final_, 0, wc, WAIT_DQ_FINAL)) {
      tc_fence_after();
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(args.dq) + (size_t(bh) * N + q) * D + h * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t rr[32];
        tmem_ld_x32(lane_base + S::kColDQ + h * (D / 2) + c * 32, rr);
        if (q < N) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(rr[8 * u + 0]), __uint_as_float(rr[8 * u + 1]));
            v.y = pack_bf16x2(__uint_as_float(rr[8 * u + 2]), __uint_as_float(rr[8 * u + 3]));
            v.z = pack_bf16x2(__uint_as_float(rr[8 * u + 4]), __uint_as_float(rr[8 * u + 5]));
            v.w = pack_bf16x2(__uint_as_float(rr[8 * u + 6]), __uint_as_float(rr[8 * u + 7]));
            reinterpret_cast<uint4*>(dst + c * 32)[u] = v;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

template <int D, bool CAUSAL>
cudaError_t launch_bwd_dq(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const BwdArgs& a, cudaStream_t stream) {
  constexpr size_t smem = dq_smem_bytes<D>();
  auto kern = bwd_dq_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int n_t = (a.N + kTile - 1) / kTile;
  const dim3 grid = CAUSAL ? dim3(unsigned(n_t) * unsigned(a.BH)) : dim3(n_t, a.BH);
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tdo, a);
  return cudaGetLastError();
}

template cudaError_t launch_bwd_dq<64, false>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                               const CUtensorMap&, const BwdArgs&, cudaStream_t);
template cudaError_t launch_bwd_dq<64, true>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                              const CUtensorMap&, const BwdArgs&, cudaStream_t);
template cudaError_t launch_bwd_dq<128, false>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                                const CUtensorMap&, const BwdArgs&, cudaStream_t);
template cudaError_t launch_bwd_dq<128, true>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                               const CUtensorMap&, const BwdArgs&, cudaStream_t);

}  // namespace fa
