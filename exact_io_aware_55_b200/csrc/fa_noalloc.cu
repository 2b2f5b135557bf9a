// fa_bwd_noalloc: the backward pass with a workspace owned by the library.
//
// Some callers cannot allocate device memory at the point where they run the
// backward: a plugin loaded into a host framework that owns every device
// allocation and hands the plugin no allocator, or a serving loop that
// reserves all of its memory at start-up and must not call cudaMalloc later
// (cudaMalloc may synchronise the device and would break a budget sized in
// advance).  For them this entry point takes the same inputs and outputs as
// fa_bwd but no workspace: the scratch (D, log2-domain LSE and the fp32 dQ
// accumulator) lives in the fixed-size __device__ array below, which every GPU
// that loads this library holds until the process exits.
//
// Every call shares that array and it keeps the last call's contents.  What
// must start at zero (the dQ accumulator) is cleared by the backward's own
// preprocess launch on each call, and everything else in it is overwritten
// before it is read.  Calls whose GPU work overlaps (on different streams, or
// from different host threads without ordering) race on the array.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "fa.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;   // 64 MiB per device

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices];

// The current device must be an sm_100 part (the check fa_bwd makes too):
// on any other GPU the kernels cannot run, and the symbol lookup below would
// fail for the same reason.
fa_status check_arch(int* dev_out) {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return FA_ERR_ARCH;
  }
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return FA_ERR_ARCH;
  }
  if (major != 10 || minor != 0) return FA_ERR_ARCH;
  *dev_out = dev;
  return FA_OK;
}

// Device address of the scratch array on device `dev` (the current one).  The
// symbol's name in host code is only a host-side stand-in; the address comes
// from cudaGetSymbolAddress, once per device, with that device current.  A
// failed lookup leaves no pending error behind.
fa_status scratch_on_device(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return FA_ERR_ARCH;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" {

size_t fa_bwd_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                         int causal, void* stream) {
  // Host-side argument checks first, so that a bad argument is reported as
  // such whatever the shape's size.
  if (!(std::isfinite(scale) && scale >= 0.0f) || (causal != 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need == static_cast<size_t>(-1)) {
    // Invalid shape: let fa_bwd report the precise code without touching the device.
    return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, nullptr, 0, stream);
  }
  if (need > kNoAllocScratchBytes) return FA_ERR_SCRATCH_LIMIT;
  if (need == 0) return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, nullptr, 0, stream);
  int dev = 0;
  fa_status st = check_arch(&dev);
  if (st != FA_OK) return st;
  void* scratch = nullptr;
  if ((st = scratch_on_device(dev, &scratch)) != FA_OK) return st;
  return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, scratch, kNoAllocScratchBytes,
                stream);
}

}  // extern "C"
