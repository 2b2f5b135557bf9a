// Forward kernel of exact IO-aware attention for sm_100a, d = 64, bf16.
//
// Method (explainers.rudrite.com "flash-attention-anatomy", Q&A "What is
// online softmax and how does tiling keep it exact?"): the same tiled online
// softmax as the d = 128 kernel in fa_fwd.cu (lazy rescaling included), with
// similar warp roles: warp 0 TMA producer, warps 1 and 2 the MMA issuers of Q
// tile 0 and Q tile 1 (warp 1 also owns TMEM), warps 4-11 two softmax
// warpgroups, one per 128-row Q tile.
//
// At d = 64 the two MMAs of a tile take about half as long as its softmax, so
// the kernel is bound by how busy the softmax warps are kept.
//   * P_g has its own TMEM columns [384 + 64g, 448 + 64g) (TMEM: S_0 S_1 at
//     [0,256), O_0 O_1 at [256,384)).  S_g is free as soon as the softmax has
//     loaded it into registers, so the MMA lane issues S_g(j+1) while
//     softmax(j) is still running: the softmax warps never wait for the
//     tensor pipe.  They wait only, before writing P_g(j) or rescaling O_g,
//     for O_g += P_g(j-1) V_(j-1) to have completed.
//   * A CTA takes work items blockIdx.x, blockIdx.x + gridDim.x, ... (an item
//     is a Q-tile pair, or in the tail of an uneven grid one Q tile).  Q is
//     double-buffered and the K/V ring runs on across items, so the loads of
//     item n+1 overlap item n and no start-up or drain separates the items.
// Causal grids launch one item per CTA (their heavy-first order is kept by
// the hardware block scheduler).
#include <cuda_bf16.h>

#include "fwd_tile.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr int kD64Tile = 128 * 64 * 2;   // one 128-row bf16 tile at d = 64
constexpr int kD64NST = 4;               // K/V ring depth
constexpr uint32_t kD64ColO = 256, kD64ColP = 384;
// Exponentials per 8 pairs on the FMA pipe (exp2_fma2) on unmasked tiles: the
// MMA time of a tile is short at d = 64, so more of them leave the MUFU unit
// than at d = 128 (3/8 was the fastest split measured on B200).
constexpr int kEmuPer8 = 3;
// Register split (launch: 384 threads x 168 = 64512): warpgroup 0 keeps 72,
// the softmax warpgroups take 216 each (128 x 72 + 256 x 216 = 64512).
constexpr uint32_t kRegs64WG0 = 72;
constexpr uint32_t kRegs64Softmax = 216;
static_assert(128 * kRegs64WG0 + 256 * kRegs64Softmax <= 384 * 168, "register split exceeds the launch allocation");

struct Fwd64Barriers {
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t k_full[kD64NST];
  uint64_t v_full[kD64NST];
  uint64_t kv_empty[kD64NST];
  uint64_t s_full[kNQT];
  uint64_t s_free[kNQT];    // the softmax holds S_g in registers
  uint64_t p_full[kNQT];
  uint64_t pv_done[kNQT];   // O_g += P_g V has completed
  uint64_t o_final[kNQT];
  uint32_t tmem_base;
  uint32_t abort;
};

constexpr size_t fwd64_smem_bytes() {
  return 1024 /*alignment slack*/ + size_t(2 * kNQT + 2 * kD64NST) * kD64Tile + sizeof(Fwd64Barriers);
}

// Work item w -> (batch-head, Q-tile pair, `only`): only >= 0 means the item
// is Q tile `only` of the pair alone.  Same numbering as fwd_kernel's blocks.
template <bool CAUSAL>
__device__ __forceinline__ void fwd_item(int w, const FwdArgs& a, int n_pairs, int& bh, int& pair, int& only) {
  only = -1;
  if constexpr (CAUSAL) {
    int rank;
    causal_block_order(w, n_pairs, a.BH, a.head_group, rank, bh);
    pair = n_pairs - 1 - rank;
  } else {
    if (w >= a.pair_blocks) {
      const int u = w - a.pair_blocks;
      w = a.pair_blocks + (u >> 1);
      only = u & 1;
    }
    bh = w / n_pairs;
    pair = w - bh * n_pairs;
  }
}

// First query row and number of key tiles of slot g of an item (0 tiles: the
// slot is empty).
template <bool CAUSAL>
__device__ __forceinline__ void fwd_slot(int pair, int only, int g, int N, int n_kv, int& q0, int& T) {
  q0 = pair * (kNQT * kBM) + (only >= 0 ? only : g) * kBM;
  T = (q0 < N && (only < 0 || g == 0)) ? (CAUSAL ? min(n_kv, q0 / kBN + 1) : n_kv) : 0;
}

template <bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    fwd64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const FwdArgs args) {
  constexpr int NST = kD64NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                          // [buffer][slot] tiles
  uint8_t* sK = sQ + 2 * kNQT * kD64Tile;
  uint8_t* sV = sK + NST * kD64Tile;
  auto* bars = reinterpret_cast<Fwd64Barriers*>(sV + NST * kD64Tile);
  const WaitCtx wc{&bars->abort, args.status, FA_WAIT_LIMIT_NS};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = args.N;
  const int n_kv = (N + kBN - 1) / kBN;
  const int n_pairs = (N + kNQT * kBM - 1) / (kNQT * kBM);
  const int pairs = n_pairs * args.BH;
  const int n_items = CAUSAL ? pairs : args.pair_blocks + 2 * (pairs - args.pair_blocks);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->q_full[b], 1);
      mbar_init(&bars->q_empty[b], kNQT);
    }
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], kNQT);
    }
    for (int g = 0; g < kNQT; ++g) {
      mbar_init(&bars->s_full[g], 1);
      mbar_init(&bars->s_free[g], 4);
      mbar_init(&bars->p_full[g], 4);
      mbar_init(&bars->pv_done[g], 1);
      mbar_init(&bars->o_final[g], 1);
    }
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

  if (warp < 4) {
    regs_dec<kRegs64WG0>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    const uint64_t pol_kv = policy_evict_last();
    const uint64_t pol_q = policy_evict_first();
    int kv_c = 0;                      // K/V tiles loaded so far (ring position)
    bool ok = true;
    for (int w = blockIdx.x, n = 0; w < n_items && ok; w += gridDim.x, ++n) {
      int bh, pair, only, q0[kNQT], T[kNQT];
      fwd_item<CAUSAL>(w, args, n_pairs, bh, pair, only);
#pragma unroll
      for (int g = 0; g < kNQT; ++g) fwd_slot<CAUSAL>(pair, only, g, N, n_kv, q0[g], T[g]);
      const int Tmax = max(T[0], T[1]);
      const int qb = n & 1;
      if (n >= 2 && !mbar_wait_warp(&bars->q_empty[qb], ((n >> 1) + 1) & 1, wc, WAIT_FWD_Q_EMPTY)) break;
      mbar_arrive_expect_tx_e(&bars->q_full[qb], ((T[0] > 0) + (T[1] > 0)) * kD64Tile);
#pragma unroll
      for (int g = 0; g < kNQT; ++g)
        if (T[g] > 0)
          tma_load_3d_hint_e(sQ + (qb * kNQT + g) * kD64Tile, &tmQ, &bars->q_full[qb], 0, q0[g], bh, pol_q);
      for (int j = 0; j < Tmax; ++j, ++kv_c) {
        const int s = kv_c % NST;
        if (kv_c >= NST && !mbar_wait_warp(&bars->kv_empty[s], ((kv_c / NST) + 1) & 1, wc, WAIT_FWD_KV_EMPTY)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx_e(&bars->k_full[s], kD64Tile);
        tma_load_3d_hint_e(sK + s * kD64Tile, &tmK, &bars->k_full[s], 0, j * kBN, bh, pol_kv);
        mbar_arrive_expect_tx_e(&bars->v_full[s], kD64Tile);
        tma_load_3d_hint_e(sV + s * kD64Tile, &tmV, &bars->v_full[s], 0, j * kBN, bh, pol_kv);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ----------------------------------------------------------------- MMA
    // One warp per slot: warp 1 issues every MMA of Q tile 0, warp 2 of Q
    // tile 1, so neither softmax warpgroup waits on the other (at an item
    // boundary, or when one runs a tile ahead).  Per K/V tile j of an item:
    // S_g(j+1) once the softmax holds S_g(j), then O_g += P_g(j) V_j.  Both
    // warps release every K/V stage and Q buffer (kv_empty and q_empty count
    // two arrivals).  A warp whose slot has no work on a tile or an item still
    // waits for that tile's (item's) load before releasing it, so its release
    // can never count towards the previous use of the stage (buffer).
    const int g = warp - 1;
    const uint64_t dQ0 = sdesc_sw128(smem_u32(sQ), 16, 1024);       // K-major
    const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);       // K-major
    const uint64_t dV0 = sdesc_sw128(smem_u32(sV), 16384, 1024);    // MN-major
    constexpr uint64_t kTileD = uint64_t(kD64Tile >> 4);
    constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);
    constexpr uint32_t kIdPV = idesc_bf16(128, 64, false, true);
    auto issue_s = [&](int qb, int s) {
      const uint64_t a = dQ0 + uint64_t(qb * kNQT + g) * kTileD, b = dK0 + uint64_t(s) * kTileD;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)   // 16 of the 64 head dims per step
        mma_f16_ss_e(tmem + uint32_t(g * 128), a + uint64_t(ks * 2), b + uint64_t(ks * 2), kIdS, ks > 0 ? 1u : 0u);
    };
    auto issue_pv = [&](int s, bool acc) {
      const uint64_t b = dV0 + uint64_t(s) * kTileD;
#pragma unroll
      for (int kt = 0; kt < 8; ++kt)   // 16 keys per step
        mma_f16_ts_e(tmem + kD64ColO + uint32_t(g * 64), tmem + kD64ColP + uint32_t(g * 64 + kt * 8),
                     b + uint64_t(kt * 128), kIdPV, (acc || kt > 0) ? 1u : 0u);
    };
    int kv_c = 0;                    // K/V tiles walked so far (ring position)
    int n_s = 0;                     // S tiles issued for this slot
    int n_p = 0;                     // P tiles consumed for this slot
    int n = 0;                       // items taken
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x, ++n) {
      int bh, pair, only, q0[kNQT], T[kNQT];
      fwd_item<CAUSAL>(w, args, n_pairs, bh, pair, only);
#pragma unroll
      for (int gg = 0; gg < kNQT; ++gg) fwd_slot<CAUSAL>(pair, only, gg, N, n_kv, q0[gg], T[gg]);
      const int Tmax = max(T[0], T[1]);
      const int Tg = (g == 0) ? T[0] : T[1];
      const int qb = n & 1;
      if (!mbar_wait_warp(&bars->q_full[qb], (n >> 1) & 1, wc, WAIT_FWD_Q)) {
        ok = false;
        break;
      }
      if (Tg > 0) {
        if (!mbar_wait_warp(&bars->k_full[kv_c % NST], (kv_c / NST) & 1, wc, WAIT_FWD_K) ||
            (n_s > 0 && !mbar_wait_warp(&bars->s_free[g], (n_s - 1) & 1, wc, WAIT_FWD_S_FREE))) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_s(qb, kv_c % NST);
        tc_commit_e(&bars->s_full[g]);
        ++n_s;
      }
      for (int j = 0; j < Tmax; ++j, ++kv_c) {
        const int s = kv_c % NST;
        if (j < Tg) {
          if (j + 1 < Tg) {
            const int c1 = kv_c + 1;
            if (!mbar_wait_warp(&bars->s_free[g], (n_s - 1) & 1, wc, WAIT_FWD_S_FREE) ||
                !mbar_wait_warp(&bars->k_full[c1 % NST], (c1 / NST) & 1, wc, WAIT_FWD_K)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(qb, c1 % NST);
            tc_commit_e(&bars->s_full[g]);
            ++n_s;
          }
          if (!mbar_wait_warp(&bars->v_full[s], (kv_c / NST) & 1, wc, WAIT_FWD_V) ||
              !mbar_wait_warp(&bars->p_full[g], n_p & 1, wc, WAIT_FWD_P)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(s, j > 0);
          tc_commit_e(&bars->pv_done[g]);
          ++n_p;
          if (j + 1 == Tg) tc_commit_e(&bars->o_final[g]);
          tc_commit_e(&bars->kv_empty[s]);
        } else {
          // This slot has no work on tile j: release the stage once it is filled.
          if (!mbar_wait_warp(&bars->v_full[s], (kv_c / NST) & 1, wc, WAIT_FWD_V)) {
            ok = false;
            break;
          }
          if (lane == 0) mbar_arrive(&bars->kv_empty[s]);
        }
      }
      if (!ok) break;
      if (Tg > 0) {
        tc_commit_e(&bars->q_empty[qb]);
      } else if (lane == 0) {
        mbar_arrive(&bars->q_empty[qb]);
      }
    }
    // Let the last commits land before the CTA can exit.
    if (ok && n > 0)
      (void)(mbar_wait_warp(&bars->kv_empty[(kv_c - 1) % NST], ((kv_c - 1) / NST) & 1, wc, WAIT_FWD_KV_EMPTY) &&
             mbar_wait_warp(&bars->q_empty[(n - 1) & 1], ((n - 1) >> 1) & 1, wc, WAIT_FWD_Q_EMPTY));
  }
  } else {
    regs_inc<kRegs64Softmax>();
    // ------------------------------------------------------------- softmax
    const int g = (warp - 4) >> 2;
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const uint32_t s_tmem = lane_base + uint32_t(g * 128);
    const uint32_t o_tmem = lane_base + kD64ColO + uint32_t(g * 64);
    const uint32_t p_tmem = lane_base + kD64ColP + uint32_t(g * 64);
    const float c = args.c_log2;
    int n_t = 0;        // S tiles of this slot so far (all items)
    int n_o = 0;        // items this slot has finished
    bool ok = true;
    for (int w = blockIdx.x; w < n_items && ok; w += gridDim.x) {
      int bh, pair, only, q0g, Tg;
      fwd_item<CAUSAL>(w, args, n_pairs, bh, pair, only);
      fwd_slot<CAUSAL>(pair, only, g, N, n_kv, q0g, Tg);
      if (Tg == 0) continue;
      const int qrow = q0g + row;
      float m_ref = -INFINITY;
      float l = 0.0f;
      for (int j = 0; j < Tg; ++j, ++n_t) {
        if (!mbar_wait_warp(&bars->s_full[g], n_t & 1, wc, WAIT_FWD_S)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float sv[128];
        {
          uint32_t r[128];
          tmem_ld_x128(s_tmem, r);
#pragma unroll
          for (int i = 0; i < 128; ++i) sv[i] = __uint_as_float(r[i]);
        }
        // S_g(j) is in registers: the MMA lane may write S_g(j+1).
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[g]);
        const int k0 = j * kBN;
        const bool need_mask = (k0 + kBN > N) || (CAUSAL && k0 + kBN - 1 > q0g);
        if (need_mask) {
          const int lim = CAUSAL ? min(N - 1, qrow) : (N - 1);   // last visible key
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (k0 + i > lim) sv[i] = -INFINITY;
        }
        const float m_tile = row_max128(sv) * c;
        float alpha = 1.0f;
        bool rescale = false;
        if (j == 0) {
          m_ref = m_tile;
        } else if (m_tile > m_ref + kRescaleThresh) {
          alpha = ex2_approx(m_ref - m_tile);
          m_ref = m_tile;
          rescale = true;
        }
        const float neg_m = (m_ref == -INFINITY) ? 0.0f : -m_ref;
        uint32_t pk[64];
        const float row_sum = need_mask ? row_exp128<false, 0, true>(sv, c, neg_m, pk)
                                        : row_exp128<false, kEmuPer8>(sv, c, neg_m, pk);
        // P_g and O_g are free once O_g += P_g(j-1) V_(j-1) has completed (at
        // j = 0 the previous item's last product was awaited by its epilogue).
        if (j > 0 && !mbar_wait_warp(&bars->pv_done[g], (n_t - 1) & 1, wc, WAIT_FWD_PV)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t (&pa)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[0]);
        uint32_t (&pb)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[32]);
        tmem_st_x32(p_tmem, pa);
        tmem_st_x32(p_tmem + 32, pb);
        l = l * alpha + row_sum;
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t r[32];
            tmem_ld_x32(o_tmem + q * 32, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st_x32(o_tmem + q * 32, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[g]);
      }
      // ---------------------------------------------------------- epilogue
      // O_g is read out before this warp's next P arrive, which is what lets
      // the next item's first product overwrite it.
      if (!ok || !mbar_wait_warp(&bars->o_final[g], n_o & 1, wc, WAIT_FWD_O)) {
        ok = false;
        break;
      }
      ++n_o;
      tc_fence_after();
      const float inv = args.o_scale / l;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(args.o) + (size_t(bh) * N + qrow) * 64;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t r[32];
        tmem_ld_x32(o_tmem + q * 32, r);
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
        if (qrow < N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
      if (qrow < N) args.lse[size_t(bh) * N + qrow] = (m_ref + lg2_approx(l)) * kLn2;
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <bool CAUSAL>
cudaError_t launch_fwd64_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a,
                         cudaStream_t stream) {
  constexpr size_t smem = fwd64_smem_bytes();
  static_assert(smem <= 227 * 1024, "d = 64 forward exceeds the shared-memory limit");
  auto kern = fwd64_kernel<CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const unsigned n_pairs = unsigned((a.N + kNQT * kBM - 1) / (kNQT * kBM));
  const unsigned pairs = n_pairs * unsigned(a.BH);
  const unsigned items = CAUSAL ? pairs : unsigned(a.pair_blocks) + 2u * (pairs - unsigned(a.pair_blocks));
  const unsigned grid = (CAUSAL || a.max_ctas <= 0) ? items : min(items, unsigned(a.max_ctas));
  kern<<<dim3(grid), kThreads, smem, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}


}  // namespace

cudaError_t launch_fwd64(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a,
                         bool causal, cudaStream_t stream) {
  return causal ? launch_fwd64_t<true>(tq, tk, tv, a, stream) : launch_fwd64_t<false>(tq, tk, tv, a, stream);
}

}  // namespace fa
