// Forward kernel of exact IO-aware attention for sm_100a: d = 128 (bf16 and
// e4m3).  d = 64 has a kernel of its own, fa_fwd64.cu.
//
// Method (explainers.rudrite.com "flash-attention-anatomy", Q&A "What is
// online softmax and how does tiling keep it exact?"; chipfoundryservices
// glossary "flash attention", "Tiling plus an online softmax removes the round
// trip"): walk the keys in tiles, keep per query row a running maximum m and
// denominator l, rescale the partial output by exp(m_old - m_new) when m grows,
// write only O = acc / l and LSE = m + ln l.  S and P never leave the SM.
//
// B200 mapping (one CTA = two 128-row Q tiles of one (batch, head)):
//   warp 0      TMA producer: both Q tiles once, then K_j / V_j through an
//               NST-deep shared-memory ring (128-byte swizzle, zero fill past N).
//   warp 1      allocates 512 TMEM columns, and one lane issues every
//               tcgen05.mma: S_g = Q_g K_j^T (both operands in shared memory)
//               and O_g += P_g V_j (P from TMEM, V MN-major in shared memory).
//   warps 4-11  two softmax warpgroups, one per Q tile; thread = query row =
//               TMEM lane.  They read S_g from TMEM, mask, update m and l,
//               write P_g back over S_g (bf16 or e4m3), rescale O_g in TMEM when
//               the reference max moves, and run the epilogue.
// TMEM columns: S_0 [0,128) S_1 [128,256) O_0 [256,256+d) O_1 [256+d,256+2d).
// The MMA lane issues S_g(j+1) right after O_g += P_g(j) V_j, so the tensor
// pipe works on one Q tile while the other tile's softmax runs.
//
// Rescaling is lazy: the row's reference max m_ref is replaced only when the
// tile max exceeds it by more than 8 (log2 units), so P <= 2^8.  O, l and LSE
// all use the same m_ref, so the result is the same exact softmax.
#include <cuda_bf16.h>

#include "fwd_tile.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace fa {

namespace {

template <int D, bool FP8>
struct FwdShape {
  static constexpr int kElemBytes = FP8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElemBytes;          // bytes of one head row
  static constexpr int kChunks = kRowBytes / 128;           // 128-byte swizzle chunks per row
  static constexpr int kChunkElems = 128 / kElemBytes;
  static constexpr int kTileBytes = 128 * kRowBytes;        // one 128-row tile
  static constexpr int kNST = (kTileBytes >= 32768) ? 2 : 4;  // K/V ring depth
  static constexpr int kSSteps = kRowBytes / 32;            // MMA K-steps of S = Q K^T (32 B each)
  static constexpr int kPVRows = FP8 ? 32 : 16;             // keys per PV MMA step
  static constexpr int kPVSteps = kBN / kPVRows;
  // Exponentials per 8 on the FMA pipe (exp2_fma2) instead of MUFU, on tiles
  // without masked entries: where the MMA time per tile is shorter (e4m3)
  // the MUFU unit alone would bound the kernel, so more is moved.
  static constexpr int kEmuPer8 = FP8 ? 3 : 2;
  static constexpr uint32_t kIdS = FP8 ? idesc_e4m3(128, 128, false, false) : idesc_bf16(128, 128, false, false);
  static constexpr uint32_t kIdPV = FP8 ? idesc_e4m3(128, D, false, true) : idesc_bf16(128, D, false, true);
  static_assert(kRowBytes % 128 == 0, "head row must be a whole number of 128-byte chunks");
};

template <int NST>
struct FwdBarriers {
  uint64_t q;
  uint64_t k_full[NST];
  uint64_t v_full[NST];
  uint64_t kv_empty[NST];
  uint64_t s_full[kNQT];
  uint64_t p_full[kNQT];
  uint64_t o_final[kNQT];
  uint32_t tmem_base;
  uint32_t abort;
};

template <int D, bool FP8>
constexpr size_t fwd_smem_bytes() {
  using S = FwdShape<D, FP8>;
  return 1024 /*alignment slack*/ + size_t(kNQT + 2 * S::kNST) * S::kTileBytes + sizeof(FwdBarriers<S::kNST>);
}

template <int D, bool CAUSAL, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdArgs args) {
  using S = FwdShape<D, FP8>;
  constexpr int NST = S::kNST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kNQT * S::kTileBytes;
  uint8_t* sV = sK + NST * S::kTileBytes;
  auto* bars = reinterpret_cast<FwdBarriers<NST>*>(sV + NST * S::kTileBytes);
  const WaitCtx wc{&bars->abort, args.status, FA_WAIT_LIMIT_NS};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Grid: x = Q-tile pair (fastest), y = batch-head, so the CTAs resident at
  // any time cover few heads and their K/V tiles are re-read from L2, not HBM.
  // Causal: a 1-D grid, heaviest pairs (the last ones) first across each group
  // of heads.
  const int N = args.N;
  const int n_kv = (N + kBN - 1) / kBN;
  // Non-causal: a 1-D grid over (head, pair) in that order, pair fastest.  The
  // pairs after `pair_blocks` are split, one Q tile per block, so that the last
  // round of an uneven grid runs short single-tile blocks on many SMs instead
  // of full pairs on a few.
  const int n_pairs = (N + kNQT * kBM - 1) / (kNQT * kBM);
  int bh, pair, only = -1;   // only >= 0: this block takes Q tile `only` of its pair alone
  if constexpr (CAUSAL) {
    int rank;
    causal_block_order(int(blockIdx.x), n_pairs, args.BH, args.head_group, rank, bh);
    pair = n_pairs - 1 - rank;
  } else {
    int p = int(blockIdx.x);
    if (p >= args.pair_blocks) {
      const int u = p - args.pair_blocks;
      p = args.pair_blocks + (u >> 1);
      only = u & 1;
    }
    bh = p / n_pairs;
    pair = p - bh * n_pairs;
  }

  int q0[kNQT], T[kNQT];
  int Tmax = 0;
#pragma unroll
  for (int g = 0; g < kNQT; ++g) {
    // a single-tile block runs its tile as Q tile 0; the other slot is empty
    q0[g] = pair * (kNQT * kBM) + (only >= 0 ? only : g) * kBM;
    T[g] = (q0[g] < N && (only < 0 || g == 0)) ? (CAUSAL ? min(n_kv, q0[g] / kBN + 1) : n_kv) : 0;
    Tmax = max(Tmax, T[g]);
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars->q, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int g = 0; g < kNQT; ++g) {
      mbar_init(&bars->s_full[g], 1);
      mbar_init(&bars->p_full[g], 4);
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
    regs_dec<kRegsWG0>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs this loop; elect.sync picks the lane that issues.
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    const uint64_t pol_kv = policy_evict_last();
    const uint64_t pol_q = policy_evict_first();
    int nq = 0;
#pragma unroll
    for (int g = 0; g < kNQT; ++g) nq += (T[g] > 0);
    mbar_arrive_expect_tx_e(&bars->q, nq * S::kTileBytes);
#pragma unroll
    for (int g = 0; g < kNQT; ++g) {
      if (T[g] == 0) continue;
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c)
        tma_load_3d_hint_e(sQ + g * S::kTileBytes + c * 16384, &tmQ, &bars->q, c * S::kChunkElems, q0[g], bh,
                           pol_q);
    }
    for (int j = 0; j < Tmax; ++j) {
      const int s = j % NST;
      if (j >= NST) {
        if (!mbar_wait_warp(&bars->kv_empty[s], ((j / NST) + 1) & 1, wc, WAIT_FWD_KV_EMPTY)) break;
      }
      mbar_arrive_expect_tx_e(&bars->k_full[s], S::kTileBytes);
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c)
        tma_load_3d_hint_e(sK + s * S::kTileBytes + c * 16384, &tmK, &bars->k_full[s], c * S::kChunkElems,
                           j * kBN, bh, pol_kv);
      mbar_arrive_expect_tx_e(&bars->v_full[s], S::kTileBytes);
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c)
        tma_load_3d_hint_e(sV + s * S::kTileBytes + c * 16384, &tmV, &bars->v_full[s], c * S::kChunkElems,
                           j * kBN, bh, pol_kv);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // Warp-uniform: every lane walks the loop and waits; one elected lane
    // issues each tcgen05 instruction (and all commits, so they track its MMAs).
    // Descriptors: a base per operand, then constant byte offsets (>> 4).
    const uint64_t dQ0 = sdesc_sw128(smem_u32(sQ), 16, 1024);       // K-major
    const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);       // K-major
    const uint64_t dV0 = sdesc_sw128(smem_u32(sV), 16384, 1024);    // MN-major
    constexpr uint64_t kTileD = uint64_t(S::kTileBytes >> 4);
    auto issue_s = [&](int g, int s) {
      const uint32_t d_tmem = tmem + uint32_t(g * 128);
      const uint64_t a = dQ0 + uint64_t(g) * kTileD, b = dK0 + uint64_t(s) * kTileD;
#pragma unroll
      for (int ks = 0; ks < S::kSSteps; ++ks) {
        const uint64_t off = uint64_t(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
        if constexpr (FP8)
          mma_f8_ss_e(d_tmem, a + off, b + off, S::kIdS, ks > 0 ? 1u : 0u);
        else
          mma_f16_ss_e(d_tmem, a + off, b + off, S::kIdS, ks > 0 ? 1u : 0u);
      }
    };
    auto issue_pv = [&](int g, int s, bool acc) {
      const uint32_t d_tmem = tmem + uint32_t(kNQT * 128 + g * D);
      const uint32_t p_tmem = tmem + uint32_t(g * 128);
      const uint64_t b = dV0 + uint64_t(s) * kTileD;
#pragma unroll
      for (int kt = 0; kt < S::kPVSteps; ++kt) {
        const uint64_t off = uint64_t((kt * S::kPVRows * 128) >> 4);
        if constexpr (FP8)
          mma_f8_ts_e(d_tmem, p_tmem + kt * 8, b + off, S::kIdPV, (acc || kt > 0) ? 1u : 0u);
        else
          mma_f16_ts_e(d_tmem, p_tmem + kt * 8, b + off, S::kIdPV, (acc || kt > 0) ? 1u : 0u);
      }
    };
    bool ok = mbar_wait_warp(&bars->q, 0, wc, WAIT_FWD_Q) && mbar_wait_warp(&bars->k_full[0], 0, wc, WAIT_FWD_K);
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int g = 0; g < kNQT; ++g) {
        if (T[g] == 0) continue;
        issue_s(g, 0);
        tc_commit_e(&bars->s_full[g]);
      }
      for (int j = 0; j < Tmax && ok; ++j) {
        const int s = j % NST;
        if (!mbar_wait_warp(&bars->v_full[s], (j / NST) & 1, wc, WAIT_FWD_V)) break;
        tc_fence_after();
        bool k_next_ready = false;
#pragma unroll
        for (int g = 0; g < kNQT; ++g) {
          if (j >= T[g] || !ok) continue;
          if (!mbar_wait_warp(&bars->p_full[g], j & 1, wc, WAIT_FWD_P)) {
            ok = false;
            continue;
          }
          tc_fence_after();
          issue_pv(g, s, j > 0);
          if (j + 1 < T[g]) {
            if (!k_next_ready) {
              const int sn = (j + 1) % NST;
              if (!mbar_wait_warp(&bars->k_full[sn], ((j + 1) / NST) & 1, wc, WAIT_FWD_K)) {
                ok = false;
                continue;
              }
              tc_fence_after();
              k_next_ready = true;
            }
            issue_s(g, (j + 1) % NST);
            tc_commit_e(&bars->s_full[g]);
          } else {
            tc_commit_e(&bars->o_final[g]);
          }
        }
        tc_commit_e(&bars->kv_empty[s]);
      }
      // Let the last commit land before the CTA can exit.
      if (ok && Tmax > 0)
        (void)mbar_wait_warp(&bars->kv_empty[(Tmax - 1) % NST], ((Tmax - 1) / NST) & 1, wc, WAIT_FWD_KV_EMPTY);
    }
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------- softmax
    const int g = (warp - 4) >> 2;
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;
    const int q0g = pair * (kNQT * kBM) + (only >= 0 ? only : g) * kBM;
    const int Tg = (q0g < N && (only < 0 || g == 0)) ? (CAUSAL ? min(n_kv, q0g / kBN + 1) : n_kv) : 0;
    const int qrow = q0g + row;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const uint32_t s_tmem = lane_base + uint32_t(g * 128);
    const uint32_t o_tmem = lane_base + uint32_t(kNQT * 128 + g * D);
    const float c = args.c_log2;
    float m_ref = -INFINITY;
    float l = 0.0f;
    bool ok = Tg > 0;
    for (int j = 0; j < Tg; ++j) {
      if (!mbar_wait_warp(&bars->s_full[g], j & 1, wc, WAIT_FWD_S)) {
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
      float row_sum;
      if constexpr (!FP8) {
        uint32_t pk[64];
        row_sum = need_mask ? row_exp128<false, 0, true>(sv, c, neg_m, pk)
                            : row_exp128<false, S::kEmuPer8>(sv, c, neg_m, pk);
        uint32_t (&pa)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[0]);
        uint32_t (&pb)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pk[32]);
        tmem_st_x32(s_tmem, pa);
        tmem_st_x32(s_tmem + 32, pb);
      } else {
        uint32_t pk[32];
        row_sum = need_mask ? row_exp128<true, 0, true>(sv, c, neg_m, pk)
                            : row_exp128<true, S::kEmuPer8>(sv, c, neg_m, pk);
        tmem_st_x32(s_tmem, pk);
      }
      l = l * alpha + row_sum;
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
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
    // ------------------------------------------------------------ epilogue
    if (ok && mbar_wait_warp(&bars->o_final[g], 0, wc, WAIT_FWD_O)) {
      tc_fence_after();
      const float inv = args.o_scale / l;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(args.o) + (size_t(bh) * N + qrow) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
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
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool CAUSAL, bool FP8>
cudaError_t launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a,
                         cudaStream_t stream) {
  constexpr size_t smem = fwd_smem_bytes<D, FP8>();
  auto kern = fwd_kernel<D, CAUSAL, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const unsigned n_pairs = unsigned((a.N + kNQT * kBM - 1) / (kNQT * kBM));
  const unsigned pairs = n_pairs * unsigned(a.BH);
  const unsigned blocks = CAUSAL ? pairs : unsigned(a.pair_blocks) + 2u * (pairs - unsigned(a.pair_blocks));
  kern<<<dim3(blocks), kThreads, smem, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdArgs& a, int d, bool causal, cudaStream_t stream) {
  if (d == 64) return launch_fwd64(tq, tk, tv, a, causal, stream);
  return causal ? launch_fwd_t<128, true, false>(tq, tk, tv, a, stream)
                : launch_fwd_t<128, false, false>(tq, tk, tv, a, stream);
}

cudaError_t launch_fwd_e4m3(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdArgs& a, int d, bool causal, cudaStream_t stream) {
  (void)d;  // d == 128 (checked by the caller)
  return causal ? launch_fwd_t<128, true, true>(tq, tk, tv, a, stream)
                : launch_fwd_t<128, false, true>(tq, tk, tv, a, stream);
}

}  // namespace fa
