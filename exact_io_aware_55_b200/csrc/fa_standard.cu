// Standard (materialising) attention on the GPU: the baseline the method is
// measured against.
//
// explainers.rudrite.com "flash-attention-anatomy", Q&A "Why is attention
// memory-bound, and how does FlashAttention fix it?": standard attention
// builds the full N x N score matrix S, writes it to HBM, reads it back for the
// softmax, writes the N x N probabilities P, and reads P again for P V.  These
// three kernels do exactly that, each written for B200, so that the
// difference to the fused kernel is the HBM round trip of S and P and not the
// quality of the pieces:
//   std_scores_kernel   S = scale Q K^T, one 128 x 128 tile per CTA
//                       (tcgen05 into TMEM), stored fp32 [BH, N, Np].
//   std_softmax_kernel  one block per row: max and sum over the row of S
//                       (causal: columns j <= i), P = exp(s - max) / sum
//                       stored bf16 [BH, N, Np] (zero where masked or
//                       j >= N), LSE = max + ln sum.
//   std_pv_kernel       O = P V, one 128-row tile per CTA over every key tile
//                       (tcgen05, P and V through a TMA ring).
// Np = N rounded up to 128.  Causal masking is applied in the softmax only;
// both products run over the full square, as a standard implementation does.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace fa {

namespace {

constexpr float kLog2eF = 1.4426950408889634f;
constexpr float kLn2F = 0.69314718055994530942f;

// ------------------------------------------------------------------ scores
struct ScoresBars {
  uint64_t full, done;
  uint32_t tmem_base;
  uint32_t abort;
};

// At least 57 KB so that no more than four CTAs (4 x 128 TMEM columns) share an SM.
template <int D>
constexpr size_t scores_smem_bytes() {
  constexpr size_t need = 1024 + 2 * size_t(128) * D * 2 + sizeof(ScoresBars);
  return need > 57 * 1024 ? need : 57 * 1024;
}

template <int D>
__global__ void __launch_bounds__(128) std_scores_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                         const __grid_constant__ CUtensorMap tmK,
                                                         const StdArgs a) {
  constexpr int kTileBytes = 128 * D * 2;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kId = idesc_bf16(128, 128, false, false);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTileBytes;
  auto* b = reinterpret_cast<ScoresBars*>(smem + 2 * kTileBytes);
  const WaitCtx wc{&b->abort, a.status, FA_WAIT_LIMIT_NS};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x, i = blockIdx.y, bh = blockIdx.z;

  if (threadIdx.x == 0) {
    mbar_init(&b->full, 1);
    mbar_init(&b->done, 1);
    b->abort = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&b->tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = b->tmem_base;

  if (warp == 0) {
    mbar_arrive_expect_tx_e(&b->full, 2 * kTileBytes);
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      tma_load_3d_hint_e(sQ + c * 16384, &tmQ, &b->full, c * 64, i * 128, bh, policy_evict_last());
      tma_load_3d_hint_e(sK + c * 16384, &tmK, &b->full, c * 64, j * 128, bh, policy_evict_last());
    }
    if (mbar_wait_warp(&b->full, 0, wc, WAIT_STD_LOAD)) {
      tc_fence_after();
      const uint64_t dq = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = sdesc_sw128(smem_u32(sK), 16, 1024);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t off = uint64_t(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
        mma_f16_ss_e(tmem, dq + off, dk + off, kId, ks > 0 ? 1u : 0u);
      }
      tc_commit_e(&b->done);
    }
  }
  // epilogue: thread = query row = TMEM lane; 128 fp32 columns
  const int row = i * 128 + warp * 32 + lane;
  if (mbar_wait_warp(&b->done, 0, wc, WAIT_STD_MMA)) {
    tc_fence_after();
    float* dst = a.s + (size_t(bh) * a.N + row) * a.Np + size_t(j) * 128;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld_x32(tmem + (uint32_t(warp * 32) << 16) + c * 32, r);
      if (row < a.N) {
#pragma unroll
        for (int u = 0; u < 8; ++u)
          reinterpret_cast<float4*>(dst + c * 32)[u] =
              make_float4(__uint_as_float(r[4 * u]) * a.scale, __uint_as_float(r[4 * u + 1]) * a.scale,
                          __uint_as_float(r[4 * u + 2]) * a.scale, __uint_as_float(r[4 * u + 3]) * a.scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ----------------------------------------------------------------- softmax
constexpr int kSmThreads = 256;

// (m, l) pairs in log2 units: l is a sum of 2^(x - m).
__device__ __forceinline__ void combine(float& m, float& l, float m2, float l2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;
  l = l * ex2_approx(m - mn) + l2 * ex2_approx(m2 - mn);
  m = mn;
}

__global__ void __launch_bounds__(kSmThreads) std_softmax_kernel(const StdArgs a) {
  __shared__ float red_m[kSmThreads / 32], red_l[kSmThreads / 32];
  const int row = blockIdx.x, bh = blockIdx.y;
  const int N = a.N, Np = a.Np;
  const float* s = a.s + (size_t(bh) * N + row) * Np;
  __nv_bfloat16* p = a.p + (size_t(bh) * N + row) * Np;
  const int lim = a.causal ? row + 1 : N;   // valid columns [0, lim)
  float m = -INFINITY, l = 0.0f;
  for (int c = threadIdx.x * 4; c < lim; c += kSmThreads * 4) {
    const float4 x = *reinterpret_cast<const float4*>(s + c);
    float v[4] = {x.x * kLog2eF, x.y * kLog2eF, x.z * kLog2eF, x.w * kLog2eF};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (c + e >= lim) v[e] = -INFINITY;
    const float m4 = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
    if (m4 > m) {
      l = (m == -INFINITY) ? 0.0f : l * ex2_approx(m - m4);
      m = m4;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) l += (v[e] == -INFINITY) ? 0.0f : ex2_approx(v[e] - m);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    combine(m, l, __shfl_xor_sync(0xffffffffu, m, off), __shfl_xor_sync(0xffffffffu, l, off));
  if ((threadIdx.x & 31) == 0) {
    red_m[threadIdx.x >> 5] = m;
    red_l[threadIdx.x >> 5] = l;
  }
  __syncthreads();
  m = red_m[0];
  l = red_l[0];
#pragma unroll
  for (int w = 1; w < kSmThreads / 32; ++w) combine(m, l, red_m[w], red_l[w]);
  const float inv = 1.0f / l;
  for (int c = threadIdx.x * 4; c < Np; c += kSmThreads * 4) {
    float pv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (c < lim) {
      const float4 x = *reinterpret_cast<const float4*>(s + c);
      const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (c + e < lim) pv[e] = ex2_approx(xs[e] * kLog2eF - m) * inv;
    }
    uint2 w;
    w.x = pack_bf16x2(pv[0], pv[1]);
    w.y = pack_bf16x2(pv[2], pv[3]);
    *reinterpret_cast<uint2*>(p + c) = w;
  }
  if (threadIdx.x == 0) a.lse[size_t(bh) * N + row] = (m + lg2_approx(l)) * kLn2F;
}

// ---------------------------------------------------------------------- PV
constexpr int kPvNS = 3;

template <int D>
struct PvBars {
  uint64_t full[kPvNS], empty[kPvNS];
  uint64_t done;
  uint32_t tmem_base;
  uint32_t abort;
};

template <int D>
constexpr size_t pv_smem_bytes() {
  return 1024 + size_t(kPvNS) * (128 * 128 * 2 + 128 * D * 2) + sizeof(PvBars<D>);
}

template <int D>
__global__ void __launch_bounds__(192, 1) std_pv_kernel(const __grid_constant__ CUtensorMap tmP,
                                                        const __grid_constant__ CUtensorMap tmV,
                                                        const StdArgs a) {
  constexpr int kPBytes = 128 * 128 * 2;
  constexpr int kVBytes = 128 * D * 2;
  constexpr int kStage = kPBytes + kVBytes;
  constexpr uint32_t kId = idesc_bf16(128, D, false, true);   // O = P V, V MN-major
  constexpr uint32_t kCols = D < 32 ? 32 : D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  auto* b = reinterpret_cast<PvBars<D>*>(smem + kPvNS * kStage);
  const WaitCtx wc{&b->abort, a.status, FA_WAIT_LIMIT_NS};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x, bh = blockIdx.y;
  const int T = a.Np / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPvNS; ++s) {
      mbar_init(&b->full[s], 1);
      mbar_init(&b->empty[s], 1);
    }
    mbar_init(&b->done, 1);
    b->abort = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&b->tmem_base, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = b->tmem_base;

  if (warp == 0) {
    const uint64_t pol_p = policy_evict_first(), pol_v = policy_evict_last();
    for (int j = 0; j < T; ++j) {
      const int s = j % kPvNS;
      if (j >= kPvNS && !mbar_wait_warp(&b->empty[s], ((j / kPvNS) + 1) & 1, wc, WAIT_STD_PV_EMPTY)) break;
      uint8_t* st = smem + s * kStage;
      mbar_arrive_expect_tx_e(&b->full[s], kStage);
#pragma unroll
      for (int c = 0; c < 2; ++c)
        tma_load_3d_hint_e(st + c * 16384, &tmP, &b->full[s], j * 128 + c * 64, i * 128, bh, pol_p);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d_hint_e(st + kPBytes + c * 16384, &tmV, &b->full[s], c * 64, j * 128, bh, pol_v);
    }
  } else if (warp == 1) {
    const uint64_t dp = sdesc_sw128(smem_u32(smem), 16, 1024);
    const uint64_t dv = sdesc_sw128(smem_u32(smem + kPBytes), 16384, 1024);
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int s = j % kPvNS;
      if (!mbar_wait_warp(&b->full[s], (j / kPvNS) & 1, wc, WAIT_STD_PV_FULL)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t so = uint64_t((s * kStage) >> 4);
#pragma unroll
      for (int kt = 0; kt < 8; ++kt) {
        const uint64_t ao = uint64_t(((kt >> 2) * 16384 + (kt & 3) * 32) >> 4);
        mma_f16_ss_e(tmem, dp + so + ao, dv + so + uint64_t(kt * 128), kId, (j > 0 || kt > 0) ? 1u : 0u);
      }
      tc_commit_e(&b->empty[s]);
    }
    if (ok) tc_commit_e(&b->done);
  } else {
    // epilogue (warps 2-5 cover the four TMEM lane quarters)
    const int wq = warp & 3;
    const int row = i * 128 + wq * 32 + lane;
    if (mbar_wait_warp(&b->done, 0, wc, WAIT_STD_PV_DONE)) {
      tc_fence_after();
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.o) + (size_t(bh) * a.N + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld_x32(tmem + (uint32_t(wq * 32) << 16) + c * 32, r);
        if (row < a.N) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(r[8 * u + 0]), __uint_as_float(r[8 * u + 1]));
            v.y = pack_bf16x2(__uint_as_float(r[8 * u + 2]), __uint_as_float(r[8 * u + 3]));
            v.z = pack_bf16x2(__uint_as_float(r[8 * u + 4]), __uint_as_float(r[8 * u + 5]));
            v.w = pack_bf16x2(__uint_as_float(r[8 * u + 6]), __uint_as_float(r[8 * u + 7]));
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
    tmem_dealloc(tmem, kCols);
  }
}

template <int D>
cudaError_t launch_standard_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const CUtensorMap& tp, const StdArgs& a, cudaStream_t stream) {
  const int T = a.Np / 128;
  {
    constexpr size_t smem = scores_smem_bytes<D>();
    auto kern = std_scores_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    kern<<<dim3(T, T, a.BH), 128, smem, stream>>>(tq, tk, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  std_softmax_kernel<<<dim3(a.N, a.BH), kSmThreads, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  constexpr size_t smem = pv_smem_bytes<D>();
  static_assert(smem <= 227 * 1024, "shared memory budget");
  auto kern = std_pv_kernel<D>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem))) != cudaSuccess)
    return e;
  kern<<<dim3(T, a.BH), 192, smem, stream>>>(tp, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_standard(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tp, const StdArgs& a, int d, cudaStream_t stream) {
  return d == 64 ? launch_standard_t<64>(tq, tk, tv, tp, a, stream)
                 : launch_standard_t<128>(tq, tk, tv, tp, a, stream);
}

}  // namespace fa
