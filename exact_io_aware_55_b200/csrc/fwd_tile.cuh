// Shared pieces of the forward kernels (fa_fwd.cu: d = 128 and e4m3;
// fa_fwd64.cu: d = 64): tile sizes, the register split of the warp roles and
// the per-row softmax arithmetic on a 128-score row of S.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;        // query rows per Q tile
constexpr int kBN = 128;        // key rows per K/V tile
constexpr int kNQT = 2;         // Q tiles per CTA
constexpr int kThreads = 384;   // 12 warps
constexpr float kRescaleThresh = 8.0f;
// Registers per thread after re-balancing: warpgroup 0 (producer, MMA, two
// idle warps) gives registers to the two softmax warpgroups.  Launch: 384
// threads x 168 = 64512; after: 128 x 80 + 256 x 208 = 63488.
constexpr uint32_t kRegsWG0 = 80;
constexpr uint32_t kRegsSoftmax = 208;
static_assert(128 * kRegsWG0 + 256 * kRegsSoftmax <= 384 * 168, "register split exceeds the launch allocation");
constexpr float kLn2 = 0.69314718055994530942f;

// Row maximum of 128 scores: four independent chains of 3-input max.
__device__ __forceinline__ float row_max128(const float (&sv)[128]) {
  float acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float a = sv[32 * k];
#pragma unroll
    for (int t = 1; t + 1 < 32; t += 2) a = fmax3(a, sv[32 * k + t], sv[32 * k + t + 1]);
    acc[k] = fmaxf(a, sv[32 * k + 31]);
  }
  return fmax3(acc[0], acc[1], fmaxf(acc[2], acc[3]));
}

// p = 2^(s*c - m) for 128 scores; packs P for the PV MMA (bf16 pairs or e4m3
// quads) and returns the fp32 row sum of p.  EMU of every 8 pairs (bf16) or
// quads (e4m3) use the FMA-pipe exponential, the rest MUFU ex2.  MASKED rows
// hold -inf for masked keys: with c = 0 (scale 0) the product -inf * 0 is NaN,
// which max(x, -inf) turns back into -inf (max returns its non-NaN operand),
// so a masked key still gets p = 0.
template <bool FP8, int EMU, bool MASKED = false>
__device__ __forceinline__ float row_exp128(const float (&sv)[128], float c, float neg_m,
                                            uint32_t (&pk)[FP8 ? 32 : 64]) {
  const float2 cc = make_float2(c, c), nm = make_float2(neg_m, neg_m);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  auto ex = [&](float2 x, bool emu) {
    if constexpr (MASKED) x = make_float2(fmaxf(x.x, -INFINITY), fmaxf(x.y, -INFINITY));
    return emu ? exp2_fma2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
  };
  if constexpr (!FP8) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const float2 x = ffma2(make_float2(sv[2 * i], sv[2 * i + 1]), cc, nm);
      const float2 p = ex(x, (i & 7) < EMU);
      acc[i & 3] = fadd2(acc[i & 3], p);
      pk[i] = pack_bf16x2(p.x, p.y);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const bool emu = (i & 7) < EMU;
      const float2 pa = ex(ffma2(make_float2(sv[4 * i], sv[4 * i + 1]), cc, nm), emu);
      const float2 pb = ex(ffma2(make_float2(sv[4 * i + 2], sv[4 * i + 3]), cc, nm), emu);
      acc[(2 * i) & 3] = fadd2(acc[(2 * i) & 3], pa);
      acc[(2 * i + 1) & 3] = fadd2(acc[(2 * i + 1) & 3], pb);
      pk[i] = pack_e4m3x4(pa.x, pa.y, pb.x, pb.y);
    }
  }
  const float2 s01 = fadd2(acc[0], acc[1]), s23 = fadd2(acc[2], acc[3]);
  const float2 s = fadd2(s01, s23);
  return s.x + s.y;
}

}  // namespace
}  // namespace fa
