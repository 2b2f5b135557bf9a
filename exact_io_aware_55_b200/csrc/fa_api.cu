// C ABI of the library (declared in include/fa.h): argument checks, TMA
// tensor-map construction and kernel dispatch.  No allocation, no
// synchronisation (except fa_device_status, which documents it).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "internal.h"
#include "ptx.cuh"

namespace {

// Status words (code, where) written by bounded waits that run out.
__device__ uint32_t g_status_words[2];

__global__ void watchdog_selftest_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    fa::mbar_init(&bar, 1);
    abort_flag = 0u;
    fa::fence_mbar_init();
  }
  __syncthreads();
  const fa::WaitCtx wc{&abort_flag, status, limit_ns};
  // Nobody arrives on `bar`: the wait must end through its time limit.
  (void)fa::mbar_wait_warp(&bar, 0, wc, fa::WAIT_SELFTEST);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

constexpr int kMaxDevices = 64;
std::atomic<int> g_arch_ok[kMaxDevices];  // 0 unknown, 1 sm_100, 2 other
uint32_t* g_status_ptr[kMaxDevices];

// Checks that the current device is an sm_100 part and returns its status
// word address.
fa_status current_device(uint32_t** status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_ARCH;
  int known = g_arch_ok[dev].load(std::memory_order_acquire);
  if (known == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FA_ERR_ARCH;
    void* sp = nullptr;
    if (major == 10 && minor == 0 && cudaGetSymbolAddress(&sp, g_status_words) == cudaSuccess) {
      g_status_ptr[dev] = static_cast<uint32_t*>(sp);
      known = 1;
    } else {
      known = 2;
    }
    g_arch_ok[dev].store(known, std::memory_order_release);
  }
  if (known != 1) return FA_ERR_ARCH;
  *status = g_status_ptr[dev];
  return FA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// 3-D tensor map over a contiguous [BH, N, d] tensor: dims {d, N, BH},
// box {128 bytes of d, box_rows rows, 1 head}, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* map, const void* base, bool e4m3, int d, int N, int BH, unsigned box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int eb = e4m3 ? 1 : 2;
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(d) * eb, cuuint64_t(N) * d * eb};
  cuuint32_t box[3] = {cuuint32_t(128 / eb), cuuint32_t(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over the backward's fp32 dQ accumulator [BH, N, d]: dims
// {d, N, BH}, box {32 columns (128 bytes), 128 rows, 1 head}, 128-byte swizzle.
bool make_map_dq(CUtensorMap* map, void* base, int d, int N, int BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 4, cuuint64_t(N) * d * 4};
  cuuint32_t box[3] = {32u, 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over the standard path's probabilities P [BH, N, Np] bf16:
// dims {Np, N, BH}, box {64 columns, 128 rows, 1 head}, 128-byte swizzle.
bool make_map_p(CUtensorMap* map, const void* base, int Np, int N, int BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(Np), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(Np) * 2, cuuint64_t(N) * Np * 2};
  cuuint32_t box[3] = {64u, 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Shape checks shared by every entry point.  Sets *empty when there is
// nothing to compute.
fa_status check_shape(int B, int H, int N, int d, float scale, int causal, bool* empty) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale >= 0.0f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  if (BH > 65535) return FA_ERR_UNSUPPORTED;  // grid.y limit of the launch shapes
  // Element offsets are computed in 64-bit; per-head rows in 32-bit.
  if (static_cast<long long>(N) * d > (1ll << 31)) return FA_ERR_UNSUPPORTED;
  *empty = (BH == 0 || N == 0);
  return FA_OK;
}

constexpr float kLog2e = 1.4426950408889634f;

size_t padded_rows(int N) { return (static_cast<size_t>(N) + 127) / 128 * 128; }

struct WsLayout {
  size_t dvec_off, lse2_off, dq_off, total;
};
WsLayout ws_layout(long long BH, int N, int d) {
  WsLayout w{};
  const size_t rows = static_cast<size_t>(BH) * padded_rows(N);
  w.dvec_off = 0;
  w.lse2_off = (rows * 4 + 255) / 256 * 256;
  w.dq_off = w.lse2_off + (rows * 4 + 255) / 256 * 256;
  w.total = w.dq_off + static_cast<size_t>(BH) * N * d * 4;
  return w;
}

// Heads per ordering group of the causal grids: as many as keep the group's
// streamed operands (K/V in the forward; Q, dO and the fp32 dQ rows in the
// backward) within 64 MiB of L2.
int head_group(long long bytes_per_head, int BH) {
  const long long budget = 64ll << 20;
  long long g = bytes_per_head > 0 ? budget / bytes_per_head : BH;
  if (g < 1) g = 1;
  if (g > BH) g = BH;
  return static_cast<int>(g);
}

// Causal grids, and the forward's grids, are 1-D with at most
// BH * ceil(N / 128) blocks; that must fit in a signed 32-bit index.
bool grid_fits(long long BH, int N) { return BH * ((static_cast<long long>(N) + 127) / 128) <= 0x7fffffffll; }

// Non-causal forward: blocks take Q-tile pairs.  When the pairs leave a last
// round that fills at most half the SMs, that round's pairs are split into
// single-tile blocks (twice as many, each about half as long), so the tail
// runs on up to all SMs.  Only when every pair has two tiles (an even number
// of 128-row tiles), so that no block is ever empty.
int sm_count();
int fwd_pair_blocks(long long BH, int N) {
  const long long n_qt = (static_cast<long long>(N) + 127) / 128;
  const long long pairs = BH * ((n_qt + 1) / 2);
  const long long sms = sm_count();
  const long long rem = pairs % sms;
  if (n_qt % 2 != 0 || rem == 0 || 2 * rem > sms) return static_cast<int>(pairs);
  return static_cast<int>(pairs - rem);
}

fa_status launch_status(cudaError_t e) { return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH; }

// Split-KV decode plan.  A head's cache is cut into items of whole key tiles
// (128 keys at d = 128, 256 at d = 64: 64 KB of K and V per tile either way);
// one persistent CTA per SM takes items round-robin, so the kernel
// time is about (items per CTA, rounded up) x (tiles per item + a per-item
// cost).  The per-item cost (pipeline refill, the partial result and its
// merge, Nq d fp32 written and read back) is counted as 1/2 + Nq/64 tiles.
// The plan takes the tiles-per-item value with the smallest such cost.  It
// assumes 148 SMs so that the workspace size needs no device query.
constexpr int kDecodeMaxNq = 16;
constexpr int kDecodePlanSMs = 148;
struct DecodePlan {
  int n_split, tiles_per_split, tiles_per_head;
  size_t o_off, lse_off, total;
};
DecodePlan decode_plan(long long BH, int Nq, int Nk, int d) {
  DecodePlan p{};
  const int tile_keys = d == 64 ? 256 : 128;
  const int T = (Nk + tile_keys - 1) / tile_keys;
  p.tiles_per_head = T;
  p.tiles_per_split = T > 0 ? T : 1;
  p.n_split = 1;
  const double per_item = 0.5 + Nq / 64.0;
  double best = -1.0;
  for (int tps = 1; tps <= T; ++tps) {
    const int ns = (T + tps - 1) / tps;
    if ((T + ns - 1) / ns != tps) continue;          // only the balanced length for ns items
    const long long items = BH * ns;
    if (items > (1ll << 30)) continue;                 // item indices stay 32-bit
    const long long rounds = (items + kDecodePlanSMs - 1) / kDecodePlanSMs;
    const double cost = double(rounds) * (tps + per_item);
    if (best < 0.0 || cost < best - 1e-9) {
      best = cost;
      p.tiles_per_split = tps;
      p.n_split = ns;
    }
  }
  const size_t parts = size_t(BH) * p.n_split * Nq;
  p.o_off = 0;
  p.lse_off = (parts * d * 4 + 255) / 256 * 256;
  p.total = p.n_split > 1 ? p.lse_off + (parts * 4 + 255) / 256 * 256 : 0;
  return p;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return kDecodePlanSMs;
  return n > 0 ? n : kDecodePlanSMs;
}

fa_status check_decode(int B, int H, int Nq, int Nk, int d, float scale, int causal, bool* empty) {
  if (B < 0 || H < 0 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale >= 0.0f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Nq > kDecodeMaxNq) return FA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  if (BH > 65535) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(Nk) * d > (1ll << 31)) return FA_ERR_UNSUPPORTED;
  *empty = (BH == 0 || Nq == 0);
  if (!*empty && Nk == 0) return FA_ERR_INVALID_ARG;            // queries with no keys
  if (!*empty && causal && Nk < Nq) return FA_ERR_INVALID_ARG;  // first queries would see no key
  return FA_OK;
}

fa_status fwd_common(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                     float scale, int causal, void* stream, bool e4m3, float qd, float kd, float vd) {
  bool empty = false;
  fa_status st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK) return st;
  if (e4m3 && d != 128) return FA_ERR_UNSUPPORTED;
  if (e4m3 && !(std::isfinite(qd) && std::isfinite(kd) && std::isfinite(vd) && qd > 0 && kd > 0 && vd > 0))
    return FA_ERR_INVALID_ARG;
  if (empty) return FA_OK;
  if (!grid_fits(static_cast<long long>(B) * H, N)) return FA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGNMENT;
  uint32_t* status = nullptr;
  if ((st = current_device(&status)) != FA_OK) return st;
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, e4m3, d, N, BH) || !make_map(&tk, k, e4m3, d, N, BH) || !make_map(&tv, v, e4m3, d, N, BH))
    return FA_ERR_LAUNCH;
  fa::FwdArgs a{};
  a.status = status;
  a.o = o;
  a.lse = lse;
  a.N = N;
  a.BH = BH;
  a.c_log2 = scale * kLog2e * (e4m3 ? qd * kd : 1.0f);
  a.o_scale = e4m3 ? vd : 1.0f;
  a.head_group = head_group(2ll * N * d * (e4m3 ? 1 : 2), BH);
  a.pair_blocks = fwd_pair_blocks(BH, N);
  a.max_ctas = sm_count();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return launch_status(e4m3 ? fa::launch_fwd_e4m3(tq, tk, tv, a, d, causal != 0, s)
                            : fa::launch_fwd_bf16(tq, tk, tv, a, d, causal != 0, s));
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, void* stream) {
  return fwd_common(q, k, v, o, lse, B, H, N, d, scale, causal, stream, false, 1.f, 1.f, 1.f);
}

fa_status fa_fwd_plan(int B, int H, int N, int d, int causal, int* ctas, int* items, int* pair_items) {
  bool empty = false;
  fa_status st = check_shape(B, H, N, d, 1.0f, causal, &empty);
  if (st != FA_OK) return st;
  if (!ctas || !items || !pair_items) return FA_ERR_INVALID_ARG;
  *ctas = *items = *pair_items = 0;
  if (empty) return FA_OK;
  const long long BH = static_cast<long long>(B) * H;
  if (!grid_fits(BH, N)) return FA_ERR_UNSUPPORTED;
  const long long pairs = BH * ((static_cast<long long>(N) + 2 * 128 - 1) / (2 * 128));
  const long long pair_blocks = causal ? pairs : fwd_pair_blocks(BH, N);
  const long long n_items = pair_blocks + 2 * (pairs - pair_blocks);
  // d = 64 non-causal runs persistent CTAs (at most one per SM) over the items
  const long long n_ctas = (d == 64 && !causal) ? std::min<long long>(n_items, sm_count()) : n_items;
  *ctas = static_cast<int>(n_ctas);
  *items = static_cast<int>(n_items);
  *pair_items = static_cast<int>(pair_blocks);
  return FA_OK;
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_descale, float k_descale,
                     float v_descale, void* o, float* lse, int B, int H, int N, int d, float scale, int causal,
                     void* stream) {
  return fwd_common(q8, k8, v8, o, lse, B, H, N, d, scale, causal, stream, true, q_descale, k_descale, v_descale);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  bool empty = false;
  if (check_shape(B, H, N, d, 1.0f, 0, &empty) != FA_OK) return static_cast<size_t>(-1);
  if (empty) return 0;
  return ws_layout(static_cast<long long>(B) * H, N, d).total;
}

namespace {
// e4m3 inputs of the backward of fa_fwd_fp8 (NULL: bf16 inputs)
struct Fp8Inputs {
  const void* q8;
  const void* k8;
  const void* v8;
  float qd, kd, vd;
};
fa_status bwd_common(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                     void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                     void* workspace, size_t workspace_bytes, void* stream, bool deterministic,
                     void* const* events, const Fp8Inputs* fp8 = nullptr);

// Workspace of the e4m3 backward: the bf16 backward's, then the bf16 widening
// of Q, K and V (each 256-byte aligned).
struct Fp8WsLayout {
  size_t q_off, k_off, v_off, total;
};
Fp8WsLayout fp8_ws_layout(long long BH, int N, int d) {
  Fp8WsLayout w{};
  const size_t t = static_cast<size_t>(BH) * N * d * 2;
  const size_t a = (t + 255) / 256 * 256;
  w.q_off = (ws_layout(BH, N, d).total + 255) / 256 * 256;
  w.k_off = w.q_off + a;
  w.v_off = w.k_off + a;
  w.total = w.v_off + t;
  return w;
}
}  // namespace

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                 void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_common(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace, workspace_bytes, stream,
                    false, nullptr);
}

fa_status fa_bwd_events(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                        void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                        void* workspace, size_t workspace_bytes, void* const* events, void* stream) {
  if (!events || !events[0] || !events[1] || !events[2] || !events[3]) return FA_ERR_INVALID_ARG;
  return bwd_common(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace, workspace_bytes, stream,
                    false, events);
}

size_t fa_bwd_fp8_workspace_size(int B, int H, int N, int d) {
  bool empty = false;
  if (check_shape(B, H, N, d, 1.0f, 0, &empty) != FA_OK || d != 128) return static_cast<size_t>(-1);
  if (empty) return 0;
  return fp8_ws_layout(static_cast<long long>(B) * H, N, d).total;
}

fa_status fa_bwd_fp8(const void* q8, const void* k8, const void* v8, float q_descale, float k_descale,
                     float v_descale, const void* o, const void* dO, const float* lse, void* dq, void* dk, void* dv,
                     int B, int H, int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                     void* stream) {
  const Fp8Inputs in{q8, k8, v8, q_descale, k_descale, v_descale};
  return bwd_common(q8, k8, v8, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace, workspace_bytes,
                    stream, false, nullptr, &in);
}

fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const void* dO,
                               const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                               float scale, int causal, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_common(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace, workspace_bytes, stream,
                    true, nullptr);
}

}  // extern "C"

namespace {
fa_status bwd_common(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                     void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                     void* workspace, size_t workspace_bytes, void* stream, bool deterministic,
                     void* const* events, const Fp8Inputs* fp8) {
  bool empty = false;
  fa_status st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK) return st;
  if (fp8 && d != 128) return FA_ERR_UNSUPPORTED;
  if (fp8 && !(std::isfinite(fp8->qd) && std::isfinite(fp8->kd) && std::isfinite(fp8->vd) && fp8->qd > 0 &&
               fp8->kd > 0 && fp8->vd > 0))
    return FA_ERR_INVALID_ARG;
  if (empty) return FA_OK;
  if (causal && !grid_fits(static_cast<long long>(B) * H, N)) return FA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  const int BH = B * H;
  const WsLayout wl = ws_layout(BH, N, d);
  const size_t need = fp8 ? fp8_ws_layout(BH, N, d).total : wl.total;
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dO, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(workspace, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGNMENT;
  uint32_t* status = nullptr;
  if ((st = current_device(&status)) != FA_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (fp8) {
    // The bf16 kernels run on the exact bf16 values of the e4m3 bytes; the
    // descales are folded into the score, dP, dK and dQ factors below.
    const Fp8WsLayout fl = fp8_ws_layout(BH, N, d);
    uint8_t* wsb = static_cast<uint8_t*>(workspace);
    const long long n16 = static_cast<long long>(BH) * N * d / 16;
    void* wq = wsb + fl.q_off;
    void* wk = wsb + fl.k_off;
    void* wv = wsb + fl.v_off;
    if (fa::launch_widen_e4m3(q, wq, n16, cs) != cudaSuccess || fa::launch_widen_e4m3(k, wk, n16, cs) != cudaSuccess ||
        fa::launch_widen_e4m3(v, wv, n16, cs) != cudaSuccess)
      return FA_ERR_LAUNCH;
    q = wq;
    k = wk;
    v = wv;
  }
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map(&tq, q, false, d, N, BH) || !make_map(&tk, k, false, d, N, BH) ||
      !make_map(&tv, v, false, d, N, BH) || !make_map(&tdo, dO, false, d, N, BH))
    return FA_ERR_LAUNCH;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  fa::BwdArgs a{};
  a.status = status;
  a.o = o;
  a.dO = dO;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.neg_dvec = reinterpret_cast<float*>(ws + wl.dvec_off);
  a.neg_lse2 = reinterpret_cast<float*>(ws + wl.lse2_off);
  a.dq_acc = reinterpret_cast<float*>(ws + wl.dq_off);
  a.N = N;
  a.Np = static_cast<int>(padded_rows(N));
  a.BH = BH;
  a.c_log2 = scale * kLog2e * (fp8 ? fp8->qd * fp8->kd : 1.0f);
  a.dp_scale = fp8 ? fp8->vd : 1.0f;
  a.dk_scale = scale * (fp8 ? fp8->qd : 1.0f);
  a.dq_scale = scale * (fp8 ? fp8->kd : 1.0f);
  a.head_group = head_group(8ll * N * d, BH);   // Q, dO (bf16) and the fp32 dQ rows of a head
  CUtensorMap tdq;
  if (!make_map_dq(&tdq, a.dq_acc, d, N, BH)) return FA_ERR_LAUNCH;
  return launch_status(
      fa::launch_bwd(tq, tk, tv, tdo, tdq, a, d, causal != 0, deterministic, events, cs));
}
}  // namespace

extern "C" {

size_t fa_fwd_decode_workspace_size(int B, int H, int Nq, int Nk, int d) {
  bool empty = false;
  if (check_decode(B, H, Nq, Nk, d, 1.0f, 0, &empty) != FA_OK) return static_cast<size_t>(-1);
  if (empty) return 0;
  return decode_plan(static_cast<long long>(B) * H, Nq, Nk, d).total;
}

fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                        int Nk, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                        void* stream) {
  bool empty = false;
  fa_status st = check_decode(B, H, Nq, Nk, d, scale, causal, &empty);
  if (st != FA_OK) return st;
  if (empty) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  const long long BH = static_cast<long long>(B) * H;
  const DecodePlan plan = decode_plan(BH, Nq, Nk, d);
  if (plan.n_split > 1 && (!workspace || workspace_bytes < plan.total)) return FA_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      (workspace && !aligned(workspace, 16)))
    return FA_ERR_ALIGNMENT;
  uint32_t* status = nullptr;
  if ((st = current_device(&status)) != FA_OK) return st;
  CUtensorMap tq, tk, tv;
  const int bh = static_cast<int>(BH);
  if (!make_map(&tq, q, false, d, Nq, bh, 16) || !make_map(&tk, k, false, d, Nk, bh) ||
      !make_map(&tv, v, false, d, Nk, bh))
    return FA_ERR_LAUNCH;
  fa::DecodeArgs a{};
  a.status = status;
  a.o = o;
  a.lse = lse;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.part_o = plan.n_split > 1 ? reinterpret_cast<float*>(ws + plan.o_off) : nullptr;
  a.part_lse = plan.n_split > 1 ? reinterpret_cast<float*>(ws + plan.lse_off) : nullptr;
  a.Nq = Nq;
  a.Nk = Nk;
  a.BH = static_cast<int>(BH);
  a.n_split = plan.n_split;
  a.tiles_per_split = plan.tiles_per_split;
  a.tiles_per_head = plan.tiles_per_head;
  a.causal = causal;
  a.c_log2 = scale * kLog2e;
  const long long items = BH * plan.n_split;
  const int grid = static_cast<int>(items < sm_count() ? items : sm_count());
  return launch_status(fa::launch_decode(tq, tk, tv, a, d, grid, static_cast<cudaStream_t>(stream)));
}

// Standard attention workspace: S fp32 [BH, N, Np] then P bf16 [BH, N, Np].
struct StdLayout {
  size_t p_off, total;
};
StdLayout std_layout(long long BH, int N) {
  const size_t cells = size_t(BH) * N * padded_rows(N);
  StdLayout w{};
  w.p_off = (cells * 4 + 255) / 256 * 256;
  w.total = w.p_off + cells * 2;
  return w;
}

size_t fa_fwd_standard_workspace_size(int B, int H, int N, int d) {
  bool empty = false;
  if (check_shape(B, H, N, d, 1.0f, 0, &empty) != FA_OK) return static_cast<size_t>(-1);
  if (empty) return 0;
  return std_layout(static_cast<long long>(B) * H, N).total;
}

fa_status fa_fwd_standard(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                          int d, float scale, int causal, void* workspace, size_t workspace_bytes, void* stream) {
  bool empty = false;
  fa_status st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK) return st;
  if (empty) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  const long long BH = static_cast<long long>(B) * H;
  const StdLayout w = std_layout(BH, N);
  if (!workspace || workspace_bytes < w.total) return FA_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(workspace, 256))
    return FA_ERR_ALIGNMENT;
  uint32_t* status = nullptr;
  if ((st = current_device(&status)) != FA_OK) return st;
  const int bh = static_cast<int>(BH);
  const int Np = static_cast<int>(padded_rows(N));
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  CUtensorMap tq, tk, tv, tp;
  if (!make_map(&tq, q, false, d, N, bh) || !make_map(&tk, k, false, d, N, bh) || !make_map(&tv, v, false, d, N, bh) ||
      !make_map_p(&tp, ws + w.p_off, Np, N, bh))
    return FA_ERR_LAUNCH;
  fa::StdArgs a{};
  a.status = status;
  a.s = reinterpret_cast<float*>(ws);
  a.p = reinterpret_cast<__nv_bfloat16*>(ws + w.p_off);
  a.o = o;
  a.lse = lse;
  a.N = N;
  a.Np = Np;
  a.BH = bh;
  a.causal = causal;
  a.scale = scale;
  return launch_status(fa::launch_standard(tq, tk, tv, tp, a, d, static_cast<cudaStream_t>(stream)));
}

const char* fa_strerror(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG:
      return "invalid argument (null pointer, negative size, scale negative or not finite, bad causal flag)";
    case FA_ERR_UNSUPPORTED:
      return "unsupported shape (head dimension must be 64 or 128; e4m3 needs 128; decode takes at most 16 queries)";
    case FA_ERR_ALIGNMENT: return "misaligned pointer (tensors need 16-byte, lse 4-byte alignment)";
    case FA_ERR_ARCH: return "current CUDA device is not an sm_100 (B200-class) GPU";
    case FA_ERR_LAUNCH: return "CUDA launch or tensor-map setup failed";
    case FA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case FA_ERR_WORKSPACE: return "backward workspace missing or smaller than fa_bwd_workspace_size()";
    case FA_ERR_SCRATCH_LIMIT:
      return "shape needs more backward scratch than fa_bwd_noalloc's fixed array (fa_bwd_noalloc_max_bytes())";
  }
  return "unknown fa_status";
}

fa_status fa_device_status(void* stream, uint32_t* where) {
  uint32_t* status = nullptr;
  fa_status st = current_device(&status);
  if (st != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t host[2] = {0u, 0u};
  if (cudaMemcpyAsync(host, status, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FA_ERR_LAUNCH;
  if (cudaMemsetAsync(status, 0, sizeof(host), s) != cudaSuccess) return FA_ERR_LAUNCH;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_LAUNCH;
  if (where) *where = host[1];
  return host[0] == 0u ? FA_OK : FA_ERR_DEVICE_TIMEOUT;
}

fa_status fa_get_device_status(void* stream) { return fa_device_status(stream, nullptr); }

fa_status fa_watchdog_selftest(uint32_t limit_us, void* stream) {
  if (limit_us == 0u || limit_us > 1000000u) return FA_ERR_INVALID_ARG;
  uint32_t* status = nullptr;
  fa_status st = current_device(&status);
  if (st != FA_OK) return st;
  watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status,
                                                                             uint64_t(limit_us) * 1000ull);
  return launch_status(cudaGetLastError());
}

int fa_version(void) { return 100; }

}  // extern "C"
