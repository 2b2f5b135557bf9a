// Backward kernels of exact IO-aware attention for sm_100a.
//
// Method (explainers.rudrite.com "flash-attention-anatomy", Q&A "How does
// FlashAttention save memory in the backward pass?"; kipu-akw.pages.dev "The
// Real Complexity", recomputation on the backward pass): P is never stored; each
// tile of S and P is recomputed from Q, K and the saved per-row LSE, and the
// gradients follow from the chain rule through O = P V, P = softmax(S),
// S = scale Q K^T:
//   D = rowsum(dO o O), dV = P^T dO, dP = dO V^T, dS = P o (dP - D),
//   dQ = scale dS K, dK = scale dS^T Q.
//
// Three launches on the caller's stream:
//   bwd_pre      -D and -LSE*log2(e) per row (padded to 128-row tiles, -inf on
//                padding rows so their P is exactly 0) and zeroing of the fp32
//                dQ accumulator.
//   bwd_kernel   one CTA per (key tile j, batch-head); K_j, V_j stay in shared
//                memory, dK_j and dV_j accumulate in TMEM, and the CTA walks the
//                query tiles i (from the diagonal when causal):
//                  S^T = K_j Q_i^T      -> TMEM R1       (tcgen05; K from TMEM at
//                  dP^T = V_j dO_i^T    -> TMEM R2        d = 64, else smem)
//                  P^T = exp2(S^T c - LSE2_i)  written back over R1 as bf16
//                  dV_j += P^T dO_i     (A = P^T from TMEM)
//                  dS^T = P^T o (dP^T - D_i) -> shared memory (bf16, swizzled)
//                                       and over the dP^T columns of R2
//                  dK_j += dS^T Q_i     (A = dS^T from TMEM)
//                  d = 128: dQ_i^T = K_j^T dS^T -> TMEM R2 (both operands read
//                           MN-major from the K tile and the dS^T bytes), then
//                           fp32 red.add into the workspace accumulator, one
//                           d-contiguous line per query row
//                  d = 64:  dQ_i = dS K_j -> TMEM R2 (dS read MN-major from the
//                           dS^T bytes, K MN-major), staged in shared memory and
//                           added to the accumulator by one TMA bulk reduction
//                           per 32 columns (shared memory has room for the
//                           staging tiles only at d = 64)
//   bwd_dq_final dQ accumulator -> bf16.
// Warp roles in bwd_kernel: 0 TMA producer, 1 MMA issuer (+TMEM owner),
// 4-7 and 8-11 the two P / dS warpgroups (thread = key row = TMEM lane; each
// handles 64 of the 128 queries of a tile), 12-15 the dQ warpgroup (thread =
// d index of dQ^T at d = 128, query row of dQ at d = 64).  Epilogue: warps 4-7
// store dV, 8-11 dK.
// TMEM columns: dV [0,d) dK [d,2d) R1 [2d,2d+128) R2 [2d+128,2d+256); at d = 64
// the untransposed dQ tile has its own columns [384, 448), and copies of K_j
// and V_j (the A operands of S^T and dP^T) sit in [448, 480) and [480, 512).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 512;
constexpr float kLog2e = 1.4426950408889634f;
// Registers per thread after re-balancing.  Launch: 512 threads x 128 = 65536;
// after: warpgroup 0 (producer, MMA, 2 idle warps) 96, the two P/dS
// warpgroups 136, the dQ warpgroup 144: 128 x (96 + 2 x 136 + 144) = 65536.
constexpr uint32_t kRegsWG0 = 96;
constexpr uint32_t kRegsPdS = 136;
constexpr uint32_t kRegsDQ = 144;
static_assert(128 * (kRegsWG0 + 2 * kRegsPdS + kRegsDQ) <= 512 * 128, "register split exceeds the launch allocation");

// ------------------------------------------------------------- preprocess
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(BwdArgs a, int row_blocks, long long dq_vec4) {
  constexpr int TPR = D / 8;              // threads per row, 8 elements (16 B) each
  constexpr int RPB = 256 / TPR;          // rows per block
  if (int(blockIdx.x) < row_blocks) {
    const int row = blockIdx.x * RPB + threadIdx.x / TPR;   // row in [0, BH*Np)
    const int sub = threadIdx.x % TPR;
    const int bh = row / a.Np;
    const int i = row - bh * a.Np;
    const bool in_range = bh < a.BH;     // always true: BH*Np is a multiple of RPB
    float part = 0.0f;
    if (in_range && i < a.N) {
      const size_t off = (size_t(bh) * a.N + i) * D + sub * 8;
      const uint4 ov = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.o) + off);
      const uint4 gv = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.dO) + off);
      const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
      const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[t]));
        const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[t]));
        part = fmaf(of.x, gf.x, part);
        part = fmaf(of.y, gf.y, part);
      }
    }
#pragma unroll
    for (int m = TPR / 2; m > 0; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
    if (sub == 0 && in_range) {
      const size_t r = size_t(bh) * a.Np + i;
      a.neg_dvec[r] = (i < a.N) ? -part : 0.0f;
      a.neg_lse2[r] = (i < a.N) ? -a.lse[size_t(bh) * a.N + i] * kLog2e : -INFINITY;
    }
  } else {
    const long long stride = (long long)(gridDim.x - row_blocks) * blockDim.x;
    float4* acc = reinterpret_cast<float4*>(a.dq_acc);
    for (long long t = (long long)(blockIdx.x - row_blocks) * blockDim.x + threadIdx.x; t < dq_vec4; t += stride)
      acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ------------------------------------------------------------ dQ finalize
__global__ void __launch_bounds__(256) bwd_dq_final_kernel(const float* __restrict__ acc, __nv_bfloat16* dq,
                                                           long long n8, float scale) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n8; t += stride) {
    const float4 x = reinterpret_cast<const float4*>(acc)[2 * t];
    const float4 y = reinterpret_cast<const float4*>(acc)[2 * t + 1];
    uint4 o;
    o.x = pack_bf16x2(x.x * scale, x.y * scale);
    o.y = pack_bf16x2(x.z * scale, x.w * scale);
    o.z = pack_bf16x2(y.x * scale, y.y * scale);
    o.w = pack_bf16x2(y.z * scale, y.w * scale);
    reinterpret_cast<uint4*>(dq)[t] = o;
  }
}

// ------------------------------------------------------- e4m3 -> bf16
// Every e4m3 value (normal or subnormal, |x| <= 448) is exactly an f16 value
// and, with at most 4 significant bits, exactly a bf16 value: e4m3 -> f16x2
// (hardware cvt) -> f32 -> bf16x2 loses nothing.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t x) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(x));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16x2(f.x, f.y);
}

__global__ void __launch_bounds__(256) widen_e4m3_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                         long long n16) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n16; t += stride) {
    const uint4 x = src[t];
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[2 * k] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w[k] & 0xffffu));
      o[2 * k + 1] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w[k] >> 16));
    }
    dst[2 * t] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * t + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// ---------------------------------------------------------------- main
template <int D>
struct BwdShape {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kChunks = kRowBytes / 128;
  static constexpr int kTileBytes = 128 * kRowBytes;     // one 128-row bf16 tile
  static constexpr int kDsBytes = 128 * 128 * 2;         // dS^T: 128 keys x 128 queries, bf16 (any d)
  static constexpr int kNST = 2;                         // Q/dO ring depth
  static constexpr int kKSteps = kRowBytes / 32;         // K-steps over d (16 elements)
  static constexpr uint32_t kIdSS = idesc_bf16(128, 128, false, false);   // S^T, dP^T
  static constexpr uint32_t kIdKmaj = idesc_bf16(128, D, false, true);    // dV, dK: B MN-major
  // dQ^T = K^T dS^T: M = d (key-tile rows become TMEM lanes = d), N = 128
  // queries, both operands MN-major (the K tile and the dS^T buffer as stored).
  static constexpr uint32_t kIdDQT = idesc_bf16(D, 128, true, true);
  // d = 64: dQ = dS K: M = 128 queries, N = d; A = dS^T bytes read MN-major,
  // B = K tile MN-major.  The fp32 tile is staged (two buffers of 128 rows x
  // 256 bytes, 128-byte swizzled 32-column chunks) for TMA bulk reductions.
  static constexpr bool kTmaDQ = (D == 64);
  static constexpr uint32_t kIdDQ = idesc_bf16(128, D, true, true);
  static constexpr int kStageDQBytes = kTmaDQ ? 128 * D * 4 : 0;
  static_assert(kIdDQ != 0 && kIdDQT != 0, "both dQ forms are defined for every d");
  // d = 64 leaves TMEM columns [384, 512) free: dQ gets its own region there,
  // so the next dP^T does not wait for the dQ warpgroup to read dQ out.
  static constexpr uint32_t kColDQ = kTmaDQ ? 384u : uint32_t(2 * D + 128);
  static constexpr uint32_t kColDV = 0, kColDK = D, kColR1 = 2 * D, kColR2 = 2 * D + 128;
  // d = 64 also leaves [448, 512) free: K_j and V_j are copied there once, as
  // bf16 pairs (lane = key row), and S^T = K Q^T, dP^T = V dO^T take them as
  // the TMEM A operand, so these two products read only Q / dO from shared
  // memory (the shared-memory data path is the busiest unit of this kernel).
  static constexpr bool kTmemKV = (D == 64);
  static constexpr uint32_t kColKt = 448, kColVt = 480;
  // Exponentials per 8 pairs computed on the FMA pipe on fully unmasked tiles.
  // None: measured on B200, moving 2/8 or 3/8 of them off MUFU made this
  // kernel slower (12-20 % at d = 64), the extra FMA-pipe instructions cost
  // more issue slots than the MUFU unit saves here.
  static constexpr int kEmuPer8 = 0;
};

template <int NST>
struct BwdBarriers {
  uint64_t kv_full;
  uint64_t qdo_full[NST];
  uint64_t qdo_empty[NST];
  uint64_t s_ready, dp_ready, p_ready, ds_ready, ds_free, dq_ready, dq_free, final_;
  uint64_t kv_tmem;                          // d = 64: K_j, V_j copied into TMEM (8 warps)
  uint64_t dq_staged[2], dq_stage_free[2];   // TMA-reduced dQ (d = 64)
  uint32_t tmem_base;
  uint32_t abort;
};

template <int D>
constexpr size_t bwd_smem_bytes() {
  using S = BwdShape<D>;
  return size_t(2 + 2 * S::kNST) * S::kTileBytes + S::kDsBytes + 2 * size_t(S::kStageDQBytes) + S::kNST * 1024 +
         sizeof(BwdBarriers<S::kNST>);
}

__device__ __forceinline__ void red_add_f32(float* addr, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(a) : "memory");
}

// DQ = false: deterministic mode; this kernel produces dK and dV only and
// the dQ^T product, its reductions and the dQ warpgroup are skipped (dQ comes
// from bwd_dq_kernel).
template <int D, bool CAUSAL, bool DQ>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
               const __grid_constant__ CUtensorMap tmdQacc, const BwdArgs args) {
  using S = BwdShape<D>;
  constexpr int NST = S::kNST;
  extern __shared__ __align__(1024) uint8_t smem[];
  auto* bars = reinterpret_cast<BwdBarriers<NST>*>(smem + (2 + 2 * NST) * S::kTileBytes + S::kDsBytes +
                                                    2 * S::kStageDQBytes + NST * 1024);
  // The layout relies on a 1024-byte aligned dynamic shared-memory base (the
  // 128-byte swizzle atoms); refuse to run otherwise.
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (threadIdx.x == 0) {
      atomicCAS(&args.status[0], DEVSTATUS_OK, DEVSTATUS_WAIT_TIMEOUT);
      atomicExch(&args.status[1], WAIT_BWD_FINAL);
    }
    return;
  }
  uint8_t* sK = smem;
  uint8_t* sV = sK + S::kTileBytes;
  uint8_t* sQ = sV + S::kTileBytes;                 // NST tiles
  uint8_t* sdO = sQ + NST * S::kTileBytes;          // NST tiles
  uint8_t* sdS = sdO + NST * S::kTileBytes;         // dS^T: rows = keys, 128 queries each
  uint8_t* sdQ = sdS + S::kDsBytes;                 // d = 64: two fp32 dQ staging tiles
  float* sStat = reinterpret_cast<float*>(sdQ + 2 * S::kStageDQBytes);   // per stage: lse2[128], D[128]
  const WaitCtx wc{&bars->abort, args.status, FA_WAIT_LIMIT_NS};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Grid: x = key tile (fastest), y = batch-head, so the CTAs resident at any
  // time cover few heads: their Q/dO tiles and dQ accumulator rows stay in L2.
  // Causal: a 1-D grid, the heaviest key tiles (the first ones) first across
  // each group of heads.
  const int N = args.N;
  const int n_q = (N + kTile - 1) / kTile;
  int bh, j;                                         // key tile j (0 = heaviest when causal)
  if constexpr (CAUSAL) {
    causal_block_order(int(blockIdx.x), n_q, args.BH, args.head_group, j, bh);
  } else {
    bh = blockIdx.y;
    j = blockIdx.x;
  }
  const int i_begin = CAUSAL ? j : 0;
  const int n_iter = n_q - i_begin;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->qdo_full[s], 1);
      mbar_init(&bars->qdo_empty[s], 1 + 8);
    }
    mbar_init(&bars->s_ready, 1);
    mbar_init(&bars->dp_ready, 1);
    mbar_init(&bars->p_ready, 8);
    mbar_init(&bars->ds_ready, 8);
    mbar_init(&bars->ds_free, 1);
    mbar_init(&bars->kv_tmem, 8);
    mbar_init(&bars->dq_ready, 1);
    mbar_init(&bars->dq_free, 4);
    mbar_init(&bars->final_, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->dq_staged[b], 4);
      mbar_init(&bars->dq_stage_free[b], 1);
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
    tma_prefetch_desc(&tmdO);
    const uint64_t pol_q = policy_evict_last();    // Q/dO tiles are re-read by every key tile
    const uint64_t pol_kv = policy_evict_first();  // K/V tiles are read once
    mbar_arrive_expect_tx_e(&bars->kv_full, 2 * S::kTileBytes);
#pragma unroll
    for (int c = 0; c < S::kChunks; ++c) {
      tma_load_3d_hint_e(sK + c * 16384, &tmK, &bars->kv_full, c * 64, j * kTile, bh, pol_kv);
      tma_load_3d_hint_e(sV + c * 16384, &tmV, &bars->kv_full, c * 64, j * kTile, bh, pol_kv);
    }
    for (int it = 0; it < n_iter; ++it) {
      const int s = it % NST;
      const int i = i_begin + it;
      if (it >= NST) {
        if (!mbar_wait_warp(&bars->qdo_empty[s], ((it / NST) + 1) & 1, wc, WAIT_BWD_QDO_EMPTY)) break;
      }
      mbar_arrive_expect_tx_e(&bars->qdo_full[s], 2 * S::kTileBytes + 1024);
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c) {
        tma_load_3d_hint_e(sQ + s * S::kTileBytes + c * 16384, &tmQ, &bars->qdo_full[s], c * 64, i * kTile, bh,
                           pol_q);
        tma_load_3d_hint_e(sdO + s * S::kTileBytes + c * 16384, &tmdO, &bars->qdo_full[s], c * 64, i * kTile, bh,
                           pol_q);
      }
      const size_t srow = size_t(bh) * args.Np + size_t(i) * kTile;
      bulk_load_e(sStat + s * 256, args.neg_lse2 + srow, 512, &bars->qdo_full[s]);
      bulk_load_e(sStat + s * 256 + 128, args.neg_dvec + srow, 512, &bars->qdo_full[s]);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // Warp-uniform: every lane walks the loop and waits; one elected lane
    // issues each tcgen05 instruction and every commit.  Descriptors: a base
    // per operand, then constant byte offsets (>> 4).
    const uint32_t tR1 = tmem + S::kColR1, tR2 = tmem + S::kColR2;
    const uint64_t dK_k = sdesc_sw128(smem_u32(sK), 16, 1024);      // K tile, K-major (A of S^T)
    const uint64_t dV_k = sdesc_sw128(smem_u32(sV), 16, 1024);      // V tile, K-major (A of dP^T)
    const uint64_t dQ_k = sdesc_sw128(smem_u32(sQ), 16, 1024);      // Q stages, K-major (B of S^T)
    const uint64_t ddO_k = sdesc_sw128(smem_u32(sdO), 16, 1024);    // dO stages, K-major (B of dP^T)
    const uint64_t dQ_mn = sdesc_sw128(smem_u32(sQ), 16384, 1024);  // Q stages, MN-major (B of dK)
    const uint64_t ddO_mn = sdesc_sw128(smem_u32(sdO), 16384, 1024);// dO stages, MN-major (B of dV)
    const uint64_t dK_mn = sdesc_sw128(smem_u32(sK), 16384, 1024);  // K tile, MN-major (A of dQ^T)
    const uint64_t ddS_mn = sdesc_sw128(smem_u32(sdS), 16384, 1024);// dS^T, MN-major (B of dQ^T)
    constexpr uint64_t kTileD = uint64_t(S::kTileBytes >> 4);
    // X^T tile = A_tile B_tile^T over d, both K-major (S^T = K Q^T, dP^T = V dO^T).
    // d = 64: A (K or V) from its TMEM copy instead of shared memory.
    auto issue_xt = [&](uint32_t d_tmem, uint64_t a, uint32_t a_tmem, uint64_t b) {
#pragma unroll
      for (int ks = 0; ks < S::kKSteps; ++ks) {
        const uint64_t off = uint64_t(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
        if constexpr (S::kTmemKV)
          mma_f16_ts_e(d_tmem, a_tmem + uint32_t(ks * 8), b + off, S::kIdSS, ks > 0 ? 1u : 0u);
        else
          mma_f16_ss_e(d_tmem, a + off, b + off, S::kIdSS, ks > 0 ? 1u : 0u);
      }
    };
    bool ok = mbar_wait_warp(&bars->kv_full, 0, wc, WAIT_BWD_KV) &&
              mbar_wait_warp(&bars->qdo_full[0], 0, wc, WAIT_BWD_QDO) &&
              (!S::kTmemKV || mbar_wait_warp(&bars->kv_tmem, 0, wc, WAIT_BWD_KV));
    if (ok) {
      tc_fence_after();
      issue_xt(tR1, dK_k, tmem + S::kColKt, dQ_k);     // S^T_0
      tc_commit_e(&bars->s_ready);
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % NST;
        const uint64_t st = uint64_t(s) * kTileD;
        if (DQ && !S::kTmaDQ && it > 0) {       // dP^T reuses R2, where dQ^T was
          if (!mbar_wait_warp(&bars->dq_free, (it - 1) & 1, wc, WAIT_BWD_DQ_FREE)) { ok = false; break; }
          tc_fence_after();
        }
        issue_xt(tR2, dV_k, tmem + S::kColVt, ddO_k + st);   // dP^T_it
        tc_commit_e(&bars->dp_ready);
        if (!mbar_wait_warp(&bars->p_ready, it & 1, wc, WAIT_BWD_P)) { ok = false; break; }
        tc_fence_after();
        // dV += P^T dO: A = P^T (TMEM R1, bf16), B = dO MN-major; 16 queries per step.
        // P^T of queries 0-63 sits in R1 columns [0,32), of queries 64-127 in [96,128).
#pragma unroll
        for (int kt = 0; kt < 8; ++kt)
          mma_f16_ts_e(tmem + S::kColDV, tR1 + kt * 8 + (kt >= 4 ? 64 : 0), ddO_mn + st + uint64_t(kt * 128),
                       S::kIdKmaj, (it > 0 || kt > 0) ? 1u : 0u);
        if (it + 1 < n_iter) {                        // S^T of the next query tile
          const int sn = (it + 1) % NST;
          if (!mbar_wait_warp(&bars->qdo_full[sn], ((it + 1) / NST) & 1, wc, WAIT_BWD_QDO)) { ok = false; break; }
          tc_fence_after();
          issue_xt(tR1, dK_k, tmem + S::kColKt, dQ_k + uint64_t(sn) * kTileD);
          tc_commit_e(&bars->s_ready);
        }
        if (!mbar_wait_warp(&bars->ds_ready, it & 1, wc, WAIT_BWD_DS)) { ok = false; break; }
        tc_fence_after();
        // dK += dS^T Q: A = dS^T from TMEM R2 (bf16; queries 0-63 in columns
        // [0,32), 64-127 in [64,96)), B = Q MN-major; 16 queries per step.
#pragma unroll
        for (int kt = 0; kt < 8; ++kt)
          mma_f16_ts_e(tmem + S::kColDK, tR2 + uint32_t(kt * 8 + (kt >= 4 ? 32 : 0)), dQ_mn + st + uint64_t(kt * 128),
                       S::kIdKmaj, (it > 0 || kt > 0) ? 1u : 0u);
        // dQ^T = K^T dS^T: A = K read MN-major (M = d), B = the dS^T bytes read
        // MN-major (N = queries); 16 keys per step.  The transposed product puts
        // d on the TMEM lanes, so each dQ row update is one coalesced line.
        if constexpr (DQ && S::kTmaDQ) {
          // dQ = dS K: A = the dS^T bytes read MN-major (M = queries), B = K MN-major (N = d),
          // into its own TMEM region once the dQ warpgroup has read the previous tile.
          if (it > 0) {
            if (!mbar_wait_warp(&bars->dq_free, (it - 1) & 1, wc, WAIT_BWD_DQ_FREE)) { ok = false; break; }
            tc_fence_after();
          }
#pragma unroll
          for (int kt = 0; kt < 8; ++kt)
            mma_f16_ss_e(tmem + S::kColDQ, ddS_mn + uint64_t(kt * 128), dK_mn + uint64_t(kt * 128), S::kIdDQ,
                         kt > 0 ? 1u : 0u);
          tc_commit_e(&bars->dq_ready);
        } else if constexpr (DQ) {
#pragma unroll
          for (int kt = 0; kt < 8; ++kt)
            mma_f16_ss_e(tR2, dK_mn + uint64_t(kt * 128), ddS_mn + uint64_t(kt * 128), S::kIdDQT, kt > 0 ? 1u : 0u);
          tc_commit_e(&bars->dq_ready);
        }
        tc_commit_e(&bars->ds_free);
        tc_commit_e(&bars->qdo_empty[s]);
      }
      tc_commit_e(&bars->final_);
      if (ok) (void)mbar_wait_warp(&bars->final_, 0, wc, WAIT_BWD_FINAL);
    }
  }
  } else if (warp < 12) {
    regs_inc<kRegsPdS>();
    // --------------------------------------------------- P / dS groups
    // Two warpgroups; group h handles queries [64h, 64h+64) of every tile.
    const int h = (warp - 4) >> 2;
    const int wq = warp & 3;
    const int c = wq * 32 + lane;                   // key row within the tile
    const int kv = j * kTile + c;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const uint32_t tS = lane_base + S::kColR1 + 64 * h;        // this half's S^T columns
    const uint32_t tP = lane_base + S::kColR1 + 96 * h;        // its P^T (bf16) columns
    const uint32_t tdP = lane_base + S::kColR2 + 64 * h;       // this half's dP^T columns
    const float cl = args.c_log2;
    const bool kv_valid = kv < N;
    const bool kv_tile_full = (j + 1) * kTile <= N;
    uint8_t* ds_row = sdS + h * 16384 + (c >> 3) * 1024 + (c & 7) * 128;
    bool ok = true;
    if constexpr (S::kTmemKV) {
      // Group 0 copies row c of K_j, group 1 row c of V_j, into TMEM: the
      // 128-byte swizzled row holds d = 8u .. 8u+7 in 16-byte unit u ^ (c % 8).
      ok = mbar_wait_warp(&bars->kv_full, 0, wc, WAIT_BWD_KV);
      if (ok) {
        const uint8_t* row = (h == 0 ? sK : sV) + (c >> 3) * 1024 + (c & 7) * 128;
        uint32_t r[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 x = *reinterpret_cast<const uint4*>(row + ((u ^ (c & 7)) << 4));
          r[4 * u] = x.x;
          r[4 * u + 1] = x.y;
          r[4 * u + 2] = x.z;
          r[4 * u + 3] = x.w;
        }
        tmem_st_x32(lane_base + (h == 0 ? S::kColKt : S::kColVt), r);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->kv_tmem);
      }
    }
    for (int it = 0; it < n_iter && ok; ++it) {
      const int s = it % NST;
      const int i = i_begin + it;
      const float* snl = sStat + s * 256 + 64 * h;   // -LSE2 of this half's queries
      const float* snd = snl + 128;                  // -D of this half's queries
      // -LSE2 / -D of this stage arrived by bulk copy on qdo_full; S^T by MMA commit.
      if (!mbar_wait_warp(&bars->qdo_full[s], (it / NST) & 1, wc, WAIT_BWD_QDO)) { ok = false; break; }
      if (!mbar_wait_warp(&bars->s_ready, it & 1, wc, WAIT_BWD_S)) { ok = false; break; }
      tc_fence_after();
      // P^T = exp2(S^T * scale * log2e - LSE2_q); masked and padded entries are 0.
      const bool diag = CAUSAL && (i == j);
      const bool exact = diag || !kv_tile_full || (i + 1) * kTile > N;
      uint32_t pk[32];
      float2 pf[32];                                  // P in fp32, for dS
      {
        uint32_t r[64];
        tmem_ld_x64(tS, r);
        const float2 cc = make_float2(cl, cl);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float4 nl4 = *reinterpret_cast<const float4*>(snl + 4 * (t >> 1));
          const float2 nl = (t & 1) ? make_float2(nl4.z, nl4.w) : make_float2(nl4.x, nl4.y);
          const float2 x = ffma2(make_float2(__uint_as_float(r[2 * t]), __uint_as_float(r[2 * t + 1])), cc, nl);
          float2 p;
          if (!exact && (t & 7) < S::kEmuPer8) {
            p = exp2_fma2(x);
          } else {
            p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if (diag) {
              const int q0 = 64 * h + 2 * t;
              if (c > q0) p.x = 0.0f;
              if (c > q0 + 1) p.y = 0.0f;
            }
            if (!kv_valid) p = make_float2(0.0f, 0.0f);
          }
          pf[t] = p;
          pk[t] = pack_bf16x2(p.x, p.y);
        }
      }
      tmem_st_x32(tP, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready);
      // dS^T row = P^T o (dP^T - D_q) -> shared memory, 128-byte swizzled K-major rows, from
      // the fp32 P (its bf16 copy feeds only dV).  The factor scale of dS is applied once
      // to dK (epilogue) and dQ (finalize) instead.
      if (!mbar_wait_warp(&bars->dp_ready, it & 1, wc, WAIT_BWD_DP)) { ok = false; break; }
      if (it > 0 && !mbar_wait_warp(&bars->ds_free, (it - 1) & 1, wc, WAIT_BWD_DS_FREE)) { ok = false; break; }
      tc_fence_after();
      // 64 queries = 128 bytes = one full row of chunk h, eight 16-byte units;
      // dP^T in two 32-column pieces.  dP - D = dp_scale * dP^T(as computed) - D.
      const float2 dps = make_float2(args.dp_scale, args.dp_scale);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t r[32];
        tmem_ld_x32(tdP + 32 * q, r);
        uint32_t w[16];
#pragma unroll
        for (int t2 = 0; t2 < 16; ++t2) {
          const int t = 16 * q + t2;
          const float4 nd4 = *reinterpret_cast<const float4*>(snd + 4 * (t >> 1));
          const float2 nd = (t & 1) ? make_float2(nd4.z, nd4.w) : make_float2(nd4.x, nd4.y);
          const float2 dpm = ffma2(make_float2(__uint_as_float(r[2 * t2]), __uint_as_float(r[2 * t2 + 1])), dps, nd);
          const float2 ds = fmul2(pf[t], dpm);
          w[t2] = pack_bf16x2(ds.x, ds.y);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4*>(ds_row + (((4 * q + u) ^ (c & 7)) << 4)) =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        // The same bf16 pairs into R2 over dP^T columns already read: the A
        // operand of dK, so dK reads only Q from shared memory.
        tmem_st_x16(tdP + 16 * q, w);
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->ds_ready);
        mbar_arrive(&bars->qdo_empty[s]);           // done with this stage's -LSE2 / -D
      }
    }
    // Epilogue: group 0 stores dV, group 1 stores dK.
    if (ok && mbar_wait_warp(&bars->final_, 0, wc, WAIT_BWD_FINAL)) {
      tc_fence_after();
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(h == 0 ? args.dv : args.dk) + (size_t(bh) * N + kv) * D;
      const uint32_t src = lane_base + (h == 0 ? S::kColDV : S::kColDK);
      const float f = (h == 0) ? 1.0f : args.dk_scale;   // dK = scale * dS^T Q
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t r[32];
        tmem_ld_x32(src + q * 32, r);
        if (kv_valid) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(r[8 * u + 0]) * f, __uint_as_float(r[8 * u + 1]) * f);
            v.y = pack_bf16x2(__uint_as_float(r[8 * u + 2]) * f, __uint_as_float(r[8 * u + 3]) * f);
            v.z = pack_bf16x2(__uint_as_float(r[8 * u + 4]) * f, __uint_as_float(r[8 * u + 5]) * f);
            v.w = pack_bf16x2(__uint_as_float(r[8 * u + 6]) * f, __uint_as_float(r[8 * u + 7]) * f);
            reinterpret_cast<uint4*>(dst + q * 32)[u] = v;
          }
        }
      }
    }
  } else if (DQ && S::kTmaDQ) {
    regs_inc<kRegsDQ>();
    // ------------------------------------------- dQ group, TMA reduction
    // Thread = query row of the dQ tile in TMEM R2 (lane = row, columns = d).
    // Per query tile: load the row, write it into staging buffer it % 2
    // (two 32-column chunks of 128-byte swizzled rows, the layout of the
    // accumulator's tensor map), and lane 0 of warp 12 adds both chunks to the
    // accumulator with TMA bulk reductions.  A staging buffer is reused once
    // the reduction that read it two tiles earlier has finished reading.
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const bool issuer = (warp == 12);
    bool ok = true;
    for (int it = 0; it < n_iter && ok; ++it) {
      const int i = i_begin + it;
      const int b = it & 1;
      if (!mbar_wait_warp(&bars->dq_ready, it & 1, wc, WAIT_BWD_DQ)) { ok = false; break; }
      tc_fence_after();
      uint32_t v[64];
      tmem_ld_x64(lane_base + S::kColDQ, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dq_free);
      if (it >= 2 && !mbar_wait_warp(&bars->dq_stage_free[b], ((it >> 1) + 1) & 1, wc, WAIT_BWD_DQ_FREE)) {
        ok = false;
        break;
      }
      uint8_t* row = sdQ + b * S::kStageDQBytes + r * 128;
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<uint4*>(row + c * 16384 + ((u ^ (r & 7)) << 4)) =
              make_uint4(v[32 * c + 4 * u], v[32 * c + 4 * u + 1], v[32 * c + 4 * u + 2], v[32 * c + 4 * u + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dq_staged[b]);
      if (issuer) {
        if (!mbar_wait_warp(&bars->dq_staged[b], (it >> 1) & 1, wc, WAIT_BWD_DQ)) { ok = false; break; }
        if (lane == 0) {
          tma_reduce_add_3d(&tmdQacc, sdQ + b * S::kStageDQBytes, 0, i * kTile, bh);
          tma_reduce_add_3d(&tmdQacc, sdQ + b * S::kStageDQBytes + 16384, 32, i * kTile, bh);
          bulk_commit_group();
          bulk_wait_group_read<1>();                  // the reduction of tile it - 1 has read its buffer
          if (it >= 1) mbar_arrive(&bars->dq_stage_free[b ^ 1]);
        }
        __syncwarp();
      }
    }
    if (issuer && lane == 0) bulk_wait_group<0>();    // every reduction complete before the CTA ends
  } else if (DQ) {
    regs_inc<kRegsDQ>();
    // ---------------------------------------------------------- dQ group
    // dQ^T tile in TMEM R2: lane = d index, column = query.  With M = d = 128
    // every lane of the warp's quarter holds a d row; with M = 64 the rows sit
    // in the first 16 lanes of each quarter (row m -> lane m % 16 + 32 (m / 16)).
    const int wq = warp & 3;
    const uint32_t lane_base = tmem + (uint32_t(wq * 32) << 16);
    const int dcol = (D == 128) ? (wq * 32 + lane) : (wq * 16 + lane);
    const bool dcol_valid = (D == 128) || (lane < 16);
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int i = i_begin + it;
      if (!mbar_wait_warp(&bars->dq_ready, it & 1, wc, WAIT_BWD_DQ)) { ok = false; break; }
      tc_fence_after();
      uint32_t dqt[128];
      tmem_ld_x64(lane_base + S::kColR2, *reinterpret_cast<uint32_t(*)[64]>(&dqt[0]));
      tmem_ld_x64(lane_base + S::kColR2 + 64, *reinterpret_cast<uint32_t(*)[64]>(&dqt[64]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dq_free);
      // One query row per instruction: the warp's lanes cover consecutive d.
      float* base = args.dq_acc + (size_t(bh) * N + size_t(i) * kTile) * D + dcol;
      const int rows = min(kTile, N - i * kTile);
      if (dcol_valid) {
#pragma unroll
        for (int q = 0; q < 128; ++q)
          if (q < rows) red_add_f32(base + size_t(q) * D, __uint_as_float(dqt[q]));
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

template <int D, bool CAUSAL, bool DQ>
cudaError_t launch_bwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdArgs& a, void* const* events,
                         cudaStream_t stream) {
  // events (optional, cudaEvent_t[4]): recorded before launches 1, 2, 3 and after the last
  auto mark = [&](int i) -> cudaError_t {
    return events ? cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream) : cudaSuccess;
  };
  cudaError_t e = mark(0);
  if (e != cudaSuccess) return e;
  // 1) preprocess + zero the dQ accumulator
  constexpr int RPB = 256 / (D / 8);
  const long long rows = (long long)a.BH * a.Np;
  const int row_blocks = int((rows + RPB - 1) / RPB);
  const long long dq_vec4 = DQ ? (long long)a.BH * a.N * D / 4 : 0;
  const int zero_blocks = DQ ? int(std::min<long long>((dq_vec4 + 255) / 256, 148LL * 8)) : 0;
  bwd_pre_kernel<D><<<row_blocks + zero_blocks, 256, 0, stream>>>(a, row_blocks, dq_vec4);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = mark(1);
  if (e != cudaSuccess) return e;
  // 2) main kernel
  constexpr size_t smem = bwd_smem_bytes<D>();
  auto kern = bwd_kernel<D, CAUSAL, DQ>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int n_t = (a.N + kTile - 1) / kTile;
  const dim3 grid = CAUSAL ? dim3(unsigned(n_t) * unsigned(a.BH)) : dim3(n_t, a.BH);
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tdo, tdq, a);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = mark(2);
  if (e != cudaSuccess) return e;
  if constexpr (!DQ) {
    // 3) deterministic dQ: query-tile-stationary pass, written once as bf16
    e = launch_bwd_dq<D, CAUSAL>(tq, tk, tv, tdo, a, stream);
  } else {
    // 3) dQ -> bf16
    const long long n8 = (long long)a.BH * a.N * D / 8;
    const int fin_blocks = int(std::min<long long>((n8 + 255) / 256, 148LL * 8));
    bwd_dq_final_kernel<<<fin_blocks, 256, 0, stream>>>(a.dq_acc, reinterpret_cast<__nv_bfloat16*>(a.dq), n8,
                                                        a.dq_scale);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = mark(3);
  return e;
}

}  // namespace

cudaError_t launch_widen_e4m3(const void* src, void* dst, long long n16, cudaStream_t stream) {
  if (n16 <= 0) return cudaSuccess;
  const int blocks = int(std::min<long long>((n16 + 255) / 256, 148LL * 8));
  widen_e4m3_kernel<<<blocks, 256, 0, stream>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16);
  return cudaGetLastError();
}

cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                       const CUtensorMap& tdq, const BwdArgs& a, int d, bool causal, bool deterministic,
                       void* const* events, cudaStream_t stream) {
  if (deterministic) {
    if (d == 64) return causal ? launch_bwd_t<64, true, false>(tq, tk, tv, tdo, tdq, a, events, stream)
                               : launch_bwd_t<64, false, false>(tq, tk, tv, tdo, tdq, a, events, stream);
    return causal ? launch_bwd_t<128, true, false>(tq, tk, tv, tdo, tdq, a, events, stream)
                  : launch_bwd_t<128, false, false>(tq, tk, tv, tdo, tdq, a, events, stream);
  }
  if (d == 64) return causal ? launch_bwd_t<64, true, true>(tq, tk, tv, tdo, tdq, a, events, stream)
                             : launch_bwd_t<64, false, true>(tq, tk, tv, tdo, tdq, a, events, stream);
  return causal ? launch_bwd_t<128, true, true>(tq, tk, tv, tdo, tdq, a, events, stream)
                : launch_bwd_t<128, false, true>(tq, tk, tv, tdo, tdq, a, events, stream);
}

}  // namespace fa
