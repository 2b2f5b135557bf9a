// Internal launch interface between the C ABI (fa_api.cu) and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace fa {

// Codes recorded in the device status "where" word by a bounded wait that ran out.
enum WaitSite : uint32_t {
  WAIT_FWD_Q = 1,
  WAIT_FWD_K = 2,
  WAIT_FWD_V = 3,
  WAIT_FWD_KV_EMPTY = 4,
  WAIT_FWD_S = 5,
  WAIT_FWD_P = 6,
  WAIT_FWD_O = 7,
  WAIT_FWD_S_FREE = 8,
  WAIT_FWD_PV = 9,
  WAIT_FWD_Q_EMPTY = 10,
  WAIT_BWD_KV = 16,
  WAIT_BWD_QDO = 17,
  WAIT_BWD_QDO_EMPTY = 18,
  WAIT_BWD_S = 19,
  WAIT_BWD_DP = 20,
  WAIT_BWD_P = 21,
  WAIT_BWD_DS = 22,
  WAIT_BWD_DS_FREE = 23,
  WAIT_BWD_DQ = 24,
  WAIT_BWD_DQ_FREE = 25,
  WAIT_BWD_FINAL = 26,
  WAIT_DQ_QDO = 32,
  WAIT_DQ_K = 33,
  WAIT_DQ_V = 34,
  WAIT_DQ_KV_EMPTY = 35,
  WAIT_DQ_S = 36,
  WAIT_DQ_DP = 37,
  WAIT_DQ_SFREE = 38,
  WAIT_DQ_DPFREE = 39,
  WAIT_DQ_DS = 40,
  WAIT_DQ_DSFREE = 41,
  WAIT_DQ_FINAL = 42,
  WAIT_DEC_Q = 48,
  WAIT_DEC_Q_EMPTY = 49,
  WAIT_DEC_KV = 50,
  WAIT_DEC_KV_EMPTY = 51,
  WAIT_DEC_S = 52,
  WAIT_DEC_S_FREE = 53,
  WAIT_DEC_P = 54,
  WAIT_DEC_PV = 55,
  WAIT_DEC_RED = 56,
  WAIT_DEC_O = 57,
  WAIT_DEC_O_FREE = 58,
  WAIT_DEC_STATS = 59,
  WAIT_STD_LOAD = 64,
  WAIT_STD_MMA = 65,
  WAIT_STD_PV_EMPTY = 66,
  WAIT_STD_PV_FULL = 67,
  WAIT_STD_PV_DONE = 68,
  WAIT_SELFTEST = 99,
};

struct FwdArgs {
  uint32_t* status;   // device status words (code, where)
  void* o;        // bf16 [BH, N, d]
  float* lse;     // fp32 [BH, N]
  int N;
  int BH;
  float c_log2;   // scale * log2(e), times the q/k descales for e4m3 inputs
  float o_scale;  // factor applied with 1/l to O (1, or the v descale for e4m3)
  int head_group; // causal: heads per ordering group (see causal_block_order)
  int pair_blocks; // non-causal: blocks [0, pair_blocks) take a Q-tile pair each; the
                   // blocks after them take the two tiles of the following pairs one at a time
  int max_ctas;    // d = 64 non-causal: persistent grid size (the SM count); 0 = one item per CTA
};

struct BwdArgs {
  uint32_t* status;   // device status words (code, where)
  const void* o;      // bf16 [BH, N, d]
  const void* dO;     // bf16 [BH, N, d]
  const float* lse;   // fp32 [BH, N]
  void* dq;           // bf16 [BH, N, d]
  void* dk;           // bf16 [BH, N, d]
  void* dv;           // bf16 [BH, N, d]
  float* neg_dvec;    // workspace: -D, fp32 [BH, Np] (0 on padded rows)
  float* neg_lse2;    // workspace: -LSE * log2(e), fp32 [BH, Np] (-inf on padded rows)
  float* dq_acc;      // workspace: fp32 [BH, N, d]
  int N;
  int Np;             // N rounded up to a multiple of 128
  int BH;
  float c_log2;       // scale * log2(e) (times the q and k descales for e4m3 inputs)
  float dp_scale;     // factor on dP = dO V^T as computed (1, or the v descale for e4m3 inputs)
  float dk_scale;     // dK = dk_scale * dS^T Q as computed (scale, or scale * q descale)
  float dq_scale;     // dQ = dq_scale * dS K as computed (scale, or scale * k descale)
  int head_group;     // causal: heads per ordering group (see causal_block_order)
};

// Exact widening of e4m3 bytes to bf16 (every e4m3 value is a bf16 value):
// `n16` groups of 16 elements from `src` to `dst`, grid-stride.  Used by the
// backward of the e4m3 forward to give the bf16 backward kernels the very
// values the forward multiplied.
cudaError_t launch_widen_e4m3(const void* src, void* dst, long long n16, cudaStream_t stream);

// Causal grids are one-dimensional: n_units work units (query-tile pairs,
// key tiles, query tiles) per head, whose cost grows or shrinks linearly with
// the unit.  Block b is mapped to (rank, head) so that, within each group of
// `group` heads, every head's heaviest unit (rank 0) is dispatched first, then
// every head's next one, and so on; groups follow one another.  The light
// units fill the SMs at the end of the grid instead of the heaviest units of
// the last head, and a group's K/V (or Q/dO) stays within an L2-sized budget.
__device__ __forceinline__ void causal_block_order(int b, int n_units, int BH, int group, int& rank, int& head) {
  const int per_group = group * n_units;
  const int g = b / per_group;
  const int r = b - g * per_group;
  const int h0 = g * group;
  const int gsize = min(group, BH - h0);
  rank = r / gsize;
  head = h0 + (r - rank * gsize);
}

struct DecodeArgs {
  uint32_t* status;   // device status words (code, where)
  void* o;            // bf16 [BH, Nq, d]
  float* lse;         // fp32 [BH, Nq]
  float* part_o;      // workspace: fp32 [BH, n_split, Nq, d] (normalised per split)
  float* part_lse;    // workspace: fp32 [BH, n_split, Nq]
  int Nq;
  int Nk;
  int BH;
  int n_split;           // work items per batch-head
  int tiles_per_split;   // 128-key tiles per item (the last item of a head may hold fewer)
  int tiles_per_head;    // ceil(Nk / 128)
  int causal;
  float c_log2;          // scale * log2(e)
};
struct StdArgs {
  uint32_t* status;   // device status words (code, where)
  float* s;           // workspace: fp32 [BH, N, Np] scores (already scaled)
  __nv_bfloat16* p;   // workspace: bf16 [BH, N, Np] probabilities
  void* o;            // bf16 [BH, N, d]
  float* lse;         // fp32 [BH, N]
  int N;
  int Np;             // N rounded up to 128
  int BH;
  int causal;
  float scale;
};
// p map: dims {Np, N, BH}, box {64 columns, 128 rows}.
cudaError_t launch_standard(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tp, const StdArgs& a, int d, cudaStream_t stream);

// q map: box {128 bytes of d, 16 rows}; k, v maps: box {128 bytes, 128 rows}.
cudaError_t launch_decode(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const DecodeArgs& a, int d, int grid, cudaStream_t stream);

// Tensor maps: 3-D views {d, N, BH} of a [BH, N, d] tensor, box {128 bytes, 128 rows, 1},
// 128-byte swizzle, zero fill out of bounds.
cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdArgs& a, int d, bool causal, cudaStream_t stream);
cudaError_t launch_fwd_e4m3(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdArgs& a, int d, bool causal, cudaStream_t stream);
// d = 64 bf16 forward (fa_fwd64.cu); launch_fwd_bf16 forwards d = 64 here.
cudaError_t launch_fwd64(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a,
                         bool causal, cudaStream_t stream);
// tdq: map over the fp32 dQ accumulator (dims {d, N, BH}, box {32 columns,
// 128 rows}); used by the d = 64 kernel's TMA bulk reductions.
// events: optional cudaEvent_t[4] recorded on `stream` before the preprocess,
// before the main kernel, after it, and after the last launch (NULL: none).
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdArgs& a, int d, bool causal,
                       bool deterministic, void* const* events, cudaStream_t stream);
// Deterministic dQ pass (one 128-query tile per CTA, no atomics); defined in
// fa_bwd_dq.cu, launched by launch_bwd after the dK/dV kernel.
template <int D, bool CAUSAL>
cudaError_t launch_bwd_dq(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_watchdog_selftest(uint64_t limit_ns, cudaStream_t stream);

}  // namespace fa
