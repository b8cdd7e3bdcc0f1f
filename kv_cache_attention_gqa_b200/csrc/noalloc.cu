// gqa_decode_noalloc: the split-KV decode with its scratch space in a fixed device array that
// the library owns, for callers that cannot allocate device memory themselves.
//
// Who needs it: code that runs where cudaMalloc is not available or not allowed, for example a
// plugin called by a host framework that owns all device memory and hands the plugin only its
// input and output buffers, or a latency-critical loop that must not risk the implicit device
// synchronisation an allocation can cause. Such callers still pass inputs and outputs; the
// decode's workspace (per-piece partial results and a work ticket) lives in g_decode_scratch.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// kNoAllocScratchBytes of it until the process exits. In host code its name is only a host-side
// handle, so the device address is looked up with cudaGetSymbolAddress once per device (with
// that device current) on the first call and cached. A device reset (cudaDeviceReset) frees the
// array and leaves the cached address stale, so the library is not to be used on a device after
// it was reset in the same process (the same holds for its other per-device state). All calls share the array and it keeps the
// last call's contents; the work ticket that must start at zero is cleared on the stream before
// every launch. Calls whose execution overlaps on the GPU (different streams, or different host
// threads on one device) race on the array and must be serialised by the caller.

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace gqa {
namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// Device address of g_decode_scratch on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  static void* addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace gqa

extern "C" gqa_status gqa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         void* o, float* lse, const int32_t* kv_len,
                                         const int32_t* q_pos, int B, int h_q, int h_kv,
                                         int T_max, int d_h, float scale, int window,
                                         gqa_dtype dtype, int num_splits, void* stream) {
  using namespace gqa;
  // gqa_decode's own checks come first, so a request it would refuse gets the same status here
  // (an unsupported shape is UNSUPPORTED, not a too-small scratch array)
  const gqa_status st = decode_check_args(q, k_cache, v_cache, o, B, h_q, h_kv, T_max, d_h, scale,
                                          window, dtype, num_splits, (long long)B * h_kv * T_max);
  if (st != GQA_OK) return st;
  const size_t need = gqa_decode_workspace_size(B, h_q, h_kv, T_max, d_h, dtype, num_splits);
  if (need == 0) return GQA_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return GQA_ERR_WORKSPACE;  // beyond the fixed scratch size
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return GQA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the work ticket (first 256 bytes of the workspace) must be zero when the decode starts
  if (cudaMemsetAsync(scratch, 0, 256, s) != cudaSuccess) return GQA_ERR_CUDA;
  return gqa_decode(q, k_cache, v_cache, o, lse, kv_len, q_pos, B, h_q, h_kv, T_max, d_h, scale,
                    window, dtype, scratch, kNoAllocScratchBytes, num_splits, stream);
}
