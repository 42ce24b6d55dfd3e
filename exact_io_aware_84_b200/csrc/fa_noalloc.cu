// Backward entry point for callers that cannot allocate device memory.
//
// fa_bwd needs scratch space (an fp32 dQ accumulator and two fp32 row
// vectors, see fa_bwd_workspace_size) that its caller normally allocates.
// Some callers cannot call cudaMalloc: a custom operator inside a framework
// or inference engine whose allocator owns all device memory and forbids
// allocations behind its back, or a host loop with a latency budget that
// must not pay cudaMalloc's synchronisation after start-up.  fa_bwd_noalloc
// gives them the same backward with the scratch taken from a fixed array in
// this library's own device memory (kNoAllocScratchBytes, held on every GPU
// that loads the library until the process exits).
#include <cuda_runtime.h>

#include <mutex>

#include "fa.h"

namespace {

// 32 MiB covers, e.g., B*H = 96 heads of N = 1024 at d = 64 (about 26 MB).
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

// Host code sees only a host-side stand-in for this array; its device
// address is looked up below, once per device.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Per-device address of the array.  Only a successful lookup is kept: a
// first call that fails (made during stream capture, or with an earlier
// error pending) leaves the slot empty and a later call tries again.
struct DeviceScratch {
  std::mutex mu;
  void* ptr = nullptr;
};
DeviceScratch g_scratch[kMaxDevices];

void* scratch_address(int dev) {
  DeviceScratch& s = g_scratch[dev];
  std::lock_guard<std::mutex> lock(s.mu);
  if (s.ptr == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess) s.ptr = p;
  }
  return s.ptr;
}

}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                              float scale, int causal, int dtype, void* stream) {
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need == 0 || !q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) {
    // invalid arguments: fa_bwd reports which, before it would touch any
    // workspace; the scratch is not looked up
    return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, nullptr, 0, B, H, N, d, scale, causal, dtype, stream);
  }
  if (need > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;  // problem too large for the fixed scratch
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_NO_DEVICE;
  // The first successful call on a device (with it current) resolves the
  // array's device address; make that first call before any stream capture.
  void* ws = scratch_address(dev);
  if (ws == nullptr) return FA_ERR_CUDA;
  // fa_bwd rewrites all of the scratch it reads (it zeroes the dQ accumulator
  // and recomputes the row vectors), so stale contents from an earlier call
  // do not matter.  Calls that overlap on the GPU share the array and race.
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, ws, kNoAllocScratchBytes, B, H, N, d, scale, causal, dtype,
                stream);
}
