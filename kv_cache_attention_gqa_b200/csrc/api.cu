// C ABI of the library (declared in include/gqa.h): host-side argument checks, TMA descriptor
// encoding and dispatch to the kernels. No per-call allocation; no per-request state.

#include <cudaTypedefs.h>
#include <math.h>
#include <atomic>
#include <mutex>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace gqa {

// Sticky device error word (one per device that loads the library). Kernels receive its address.
__device__ unsigned g_device_error_word;

namespace {

constexpr int kMaxDevices = 64;

// Test hook set by gqa_debug_expire_waits: the bf16 prefill, the contiguous bf16 decode and the
// tensor-core MLA decode pass it to their kernels, whose CTA 0 then waits on a barrier that nothing
// signals.
std::atomic<int> g_expire_waits{0};

unsigned* device_error_ptr() {
  static unsigned* ptrs[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return nullptr;
    ptrs[dev] = reinterpret_cast<unsigned*>(p);
  }
  return ptrs[dev];
}

int sm_count() {
  static int cached[kMaxDevices] = {0};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDevices && cached[dev] > 0) return cached[dev];
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDevices) cached[dev] = n;
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Encode a bf16 tensor map over a row-major matrix viewed as (rows, inner) with a 128-byte
// swizzle. Dimensions are listed innermost first, as the driver expects.
bool encode_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  uint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                        const_cast<void*>(base), dims, strides_bytes, box, elem_strides,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// scale: finite and > 0, or exactly 0 for the default 1/sqrt(d_h) (computed in double, then
// rounded once to fp32, so every caller of the C ABI gets the same fp32 value)
bool valid_scale(float s) { return isfinite(s) && s >= 0.f; }
float resolve_scale(float s, int d) { return s == 0.f ? (float)(1.0 / sqrt((double)d)) : s; }

gqa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA; }

}  // namespace

}  // namespace gqa

namespace gqa {
gqa_status decode_check_args(const void* q, const void* k_cache, const void* v_cache, const void* o,
                             int B, int h_q, int h_kv, int T_max, int d_h, float scale, int window,
                             gqa_dtype dtype, int num_splits, long long cache_rows) {
  if (!q || !k_cache || !v_cache || !o) return GQA_ERR_INVALID_ARG;
  if (window < 0) return GQA_ERR_INVALID_ARG;
  if (B <= 0 || h_q <= 0 || h_kv <= 0 || T_max <= 0 || d_h <= 0 || num_splits < 0)
    return GQA_ERR_INVALID_ARG;
  if (h_q % h_kv != 0 || !valid_scale(scale)) return GQA_ERR_INVALID_ARG;
  if (dtype != GQA_BF16 && dtype != GQA_FP32) return GQA_ERR_INVALID_ARG;
  if (B > decode_max_batch()) return GQA_ERR_UNSUPPORTED;
  if (dtype == GQA_FP32 && d_h > 256) return GQA_ERR_UNSUPPORTED;
  if (dtype == GQA_BF16 && d_h != 64 && d_h != 128) return GQA_ERR_UNSUPPORTED;
  if (cache_rows >= (1ll << 31) || (long long)B * h_q >= (1ll << 31)) return GQA_ERR_UNSUPPORTED;
  return GQA_OK;
}
}  // namespace gqa

using namespace gqa;

namespace {
// Shared body of gqa_decode and gqa_decode_paged. A paged call passes block_table != nullptr and
// T_max = max_pages * page_size; k_cache / v_cache are then the page pools.
gqa_status decode_impl(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                       const int32_t* kv_len, const int32_t* q_pos, int B, int h_q, int h_kv,
                       int T_max, int d_h, float scale, int window, gqa_dtype dtype, void* workspace,
                       size_t workspace_bytes, int num_splits, void* stream,
                       const int32_t* block_table, int max_pages, int page_size, int num_pages) {
  using namespace gqa;
  const long long cache_rows =
      block_table ? (long long)num_pages * h_kv * page_size : (long long)B * h_kv * T_max;
  const gqa_status st = decode_check_args(q, k_cache, v_cache, o, B, h_q, h_kv, T_max, d_h, scale,
                                          window, dtype, num_splits, cache_rows);
  if (st != GQA_OK) return st;
  scale = resolve_scale(scale, d_h);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GQA_ERR_WORKSPACE;
  // the workspace check needs no device query when num_splits is given
  if (num_splits > 0 && workspace_bytes < decode_workspace_bytes(B, h_q, h_kv, T_max, d_h, num_splits, 1))
    return GQA_ERR_WORKSPACE;
  const int sms = sm_count();
  if (sms <= 0) return GQA_ERR_CUDA;
  if (workspace_bytes < decode_workspace_bytes(B, h_q, h_kv, T_max, d_h, num_splits, sms))
    return GQA_ERR_WORKSPACE;
  DecodeArgs a;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.o = o;
  a.lse = lse;
  a.kv_len = kv_len;
  a.q_pos = q_pos;
  a.B = B;
  a.h_q = h_q;
  a.h_kv = h_kv;
  a.T_max = T_max;
  a.d_h = d_h;
  a.scale = scale;
  a.window = window;
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  a.num_splits = num_splits;
  a.num_sms = sms;
  a.block_table = block_table;
  a.max_pages = max_pages;
  a.page_size = page_size;
  a.num_pages = num_pages;
  a.expire_wait = g_expire_waits.load(std::memory_order_relaxed);
  a.err = device_error_ptr();
  if (!a.err) return GQA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GQA_FP32) return from_cuda(launch_decode_fp32(a, s));
  // Query rows per TMA box = the kernel's m-tiles x 16: units hold min(r, 32) heads (the decode
  // kernel's heads-per-unit limit), two m-tiles above 16. The box height and the kernel's expected
  // bytes must agree, or its full barriers never complete (the bounded waits then report a timeout).
  const int r = h_q / h_kv;
  const uint32_t qrows = r > 16 ? 32 : 16;
  CUtensorMap maps[3];
  // K/V: rows of d_h elements; a paged pool is (num_pages * h_kv * page_size) rows loaded in
  // 64-row boxes when pages hold a multiple of 64 keys, else in 16-row boxes (one per 16-key
  // sub-tile); a contiguous cache (B * h_kv * T_max) in 64-row boxes
  const uint64_t kdims[2] = {(uint64_t)d_h, (uint64_t)cache_rows};
  const uint64_t qdims[2] = {(uint64_t)d_h, (uint64_t)B * h_q};
  const uint64_t strides[1] = {(uint64_t)d_h * 2};
  const uint32_t box[2] = {64, (block_table && page_size % 64 != 0) ? 16u : 64u};
  const uint32_t qbox[2] = {64, qrows};
  if (!encode_bf16(&maps[2], q, 2, qdims, strides, qbox)) return GQA_ERR_CUDA;
  if (block_table && page_size % 64 != 0 && d_h == 128) {
    // 16-row sub-tiles at d_h = 128: a 3-D view whose third dimension steps over the two 128-byte
    // column chunks of a row, so one box carries a whole 16 x 128 sub-tile (half the copies of
    // two 2-D boxes). Falls back to the 2-D boxes if the driver declines the view.
    const uint64_t dims3[3] = {64, (uint64_t)cache_rows, 2};
    const uint64_t strides3[2] = {(uint64_t)d_h * 2, 128};
    const uint32_t box3[3] = {64, 16, 2};
    if (encode_bf16(&maps[0], k_cache, 3, dims3, strides3, box3) &&
        encode_bf16(&maps[1], v_cache, 3, dims3, strides3, box3)) {
      a.paged_3d = 1;
      return from_cuda(launch_decode_bf16(a, maps, s));
    }
  }
  if (!encode_bf16(&maps[0], k_cache, 2, kdims, strides, box) ||
      !encode_bf16(&maps[1], v_cache, 2, kdims, strides, box))
    return GQA_ERR_CUDA;
  return from_cuda(launch_decode_bf16(a, maps, s));
}
}  // namespace

extern "C" {

const char* gqa_status_string(gqa_status s) {
  switch (s) {
    case GQA_OK: return "GQA_OK";
    case GQA_ERR_INVALID_ARG: return "GQA_ERR_INVALID_ARG";
    case GQA_ERR_UNSUPPORTED: return "GQA_ERR_UNSUPPORTED";
    case GQA_ERR_CUDA: return "GQA_ERR_CUDA";
    case GQA_ERR_DEVICE: return "GQA_ERR_DEVICE";
    case GQA_ERR_WORKSPACE: return "GQA_ERR_WORKSPACE";
  }
  return "GQA_ERR_UNKNOWN";
}

const char* gqa_version(void) { return "gqa-b200 0.2.0 (sm_100a)"; }

gqa_status gqa_debug_expire_waits(int enable) {
  if (enable != 0 && enable != 1) return GQA_ERR_INVALID_ARG;
  g_expire_waits.store(enable, std::memory_order_relaxed);
  return GQA_OK;
}

gqa_status gqa_get_device_error(int* code, void* stream) {
  if (!code) return GQA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GQA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_device_error_word, sizeof(v)) != cudaSuccess) return GQA_ERR_CUDA;
  *code = (int)v;
  if (v != 0) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_device_error_word, &zero, sizeof(zero)) != cudaSuccess)
      return GQA_ERR_CUDA;
    return GQA_ERR_DEVICE;
  }
  return GQA_OK;
}

gqa_status kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                     const int32_t* pos, int B, int h_kv, int S_new, int T_max, int d_h,
                     gqa_dtype dtype, void* stream) {
  if (!k_cache || !v_cache) return GQA_ERR_INVALID_ARG;
  if (S_new > 0 && (!k_new || !v_new || !pos)) return GQA_ERR_INVALID_ARG;  // S_new = 0: no-op
  if (B <= 0 || h_kv <= 0 || S_new < 0 || T_max <= 0 || d_h <= 0) return GQA_ERR_INVALID_ARG;
  if (dtype != GQA_BF16 && dtype != GQA_FP32) return GQA_ERR_INVALID_ARG;
  if (S_new > T_max) return GQA_ERR_INVALID_ARG;
  if (S_new == 0) return GQA_OK;  // nothing to copy
  AppendArgs a;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.k_new = k_new;
  a.v_new = v_new;
  a.pos = pos;
  a.B = B;
  a.h_kv = h_kv;
  a.S_new = S_new;
  a.T_max = T_max;
  a.d_h = d_h;
  a.elem_bytes = dtype == GQA_BF16 ? 2 : 4;
  a.err = device_error_ptr();
  if (!a.err) return GQA_ERR_CUDA;
  return from_cuda(launch_kv_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

gqa_status gqa_prefill(const void* q, const void* k_cache, const void* v_cache, void* o,
                       float* lse, const int32_t* q_start, const int32_t* kv_len,
                       int B, int h_q, int h_kv, int S_q, int T_max, int d_h,
                       float scale, int causal, int window, gqa_dtype dtype, void* stream) {
  if (!q || !k_cache || !v_cache || !o) return GQA_ERR_INVALID_ARG;
  // a window is measured back from each row's own position, so it needs the causal mask
  if (window < 0 || (window > 0 && causal != 1)) return GQA_ERR_INVALID_ARG;
  if (B <= 0 || h_q <= 0 || h_kv <= 0 || S_q <= 0 || T_max <= 0 || d_h <= 0)
    return GQA_ERR_INVALID_ARG;
  if (h_q % h_kv != 0 || !valid_scale(scale)) return GQA_ERR_INVALID_ARG;
  scale = resolve_scale(scale, d_h);
  if (causal != 0 && causal != 1) return GQA_ERR_INVALID_ARG;
  // every host-detectable problem is reported before the first CUDA call
  if (dtype != GQA_BF16 && dtype != GQA_FP32) return GQA_ERR_INVALID_ARG;
  if (dtype == GQA_FP32 && d_h > 256) return GQA_ERR_UNSUPPORTED;
  if (dtype == GQA_BF16) {
    if (d_h != 64 && d_h != 128) return GQA_ERR_UNSUPPORTED;
    if ((long long)B * h_kv * T_max >= (1ll << 31) || (long long)B * h_q * S_q >= (1ll << 31))
      return GQA_ERR_UNSUPPORTED;
  }
  PrefillArgs a;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.o = o;
  a.lse = lse;
  a.q_start = q_start;
  a.kv_len = kv_len;
  a.B = B;
  a.h_q = h_q;
  a.h_kv = h_kv;
  a.S_q = S_q;
  a.T_max = T_max;
  a.d_h = d_h;
  a.scale = scale;
  a.causal = causal;
  a.window = window;
  a.expire_wait = g_expire_waits.load(std::memory_order_relaxed);
  a.err = device_error_ptr();
  if (!a.err) return GQA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GQA_FP32) return from_cuda(launch_prefill_fp32(a, s));
  // TMA views: Q as (d_h, S_q, B*h_q) with box (64, P, H): one box holds the H heads x P
  // positions of a tile, head-major; K, V as rows (B*h_kv*T_max, d_h) with box (64, 128).
  const int H = prefill_heads_per_tile(h_q, h_kv);
  const uint32_t P = (uint32_t)(128 / H);
  CUtensorMap maps[3];
  const uint64_t qdims[3] = {(uint64_t)d_h, (uint64_t)S_q, (uint64_t)B * h_q};
  const uint64_t qstrides[2] = {(uint64_t)d_h * 2, (uint64_t)S_q * d_h * 2};
  const uint32_t qbox[3] = {64, P, (uint32_t)H};
  const uint64_t kdims[2] = {(uint64_t)d_h, (uint64_t)B * h_kv * T_max};
  const uint64_t strides[1] = {(uint64_t)d_h * 2};
  const uint32_t box[2] = {64, 128};
  if (!encode_bf16(&maps[0], q, 3, qdims, qstrides, qbox) ||
      !encode_bf16(&maps[1], k_cache, 2, kdims, strides, box) ||
      !encode_bf16(&maps[2], v_cache, 2, kdims, strides, box))
    return GQA_ERR_CUDA;
  return from_cuda(launch_prefill_bf16(a, maps, sm_count(), s));
}

size_t gqa_prefill_backward_workspace_size(int B, int h_q, int S_q) {
  if (B <= 0 || h_q <= 0 || S_q <= 0) return 0;
  const size_t rows = (size_t)B * h_q * S_q;
  return 2 * ((rows * 4 + 255) / 256 * 256) + 256;  // lse2, D, the work-item counter
}

gqa_status gqa_prefill_backward(const void* q, const void* k_cache, const void* v_cache,
                                const void* o, const void* d_o, const float* lse, void* dq,
                                void* dk, void* dv, const int32_t* q_start, const int32_t* kv_len,
                                int B, int h_q, int h_kv, int S_q, int T_max, int d_h, float scale,
                                int causal, int window, gqa_dtype dtype, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!q || !k_cache || !v_cache || !o || !d_o || !lse || !dq || !dk || !dv) return GQA_ERR_INVALID_ARG;
  if (B <= 0 || h_q <= 0 || h_kv <= 0 || S_q <= 0 || T_max <= 0 || d_h <= 0) return GQA_ERR_INVALID_ARG;
  if (h_q % h_kv != 0 || !valid_scale(scale)) return GQA_ERR_INVALID_ARG;
  scale = resolve_scale(scale, d_h);
  if (causal != 0 && causal != 1) return GQA_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && causal != 1)) return GQA_ERR_INVALID_ARG;
  if (dtype != GQA_BF16 && dtype != GQA_FP32) return GQA_ERR_INVALID_ARG;
  if (dtype == GQA_FP32 && d_h > 256) return GQA_ERR_UNSUPPORTED;
  if (dtype == GQA_BF16 && d_h != 64 && d_h != 128) return GQA_ERR_UNSUPPORTED;
  if ((long long)B * h_kv * T_max >= (1ll << 31) || (long long)B * h_q * S_q >= (1ll << 31))
    return GQA_ERR_UNSUPPORTED;
  const size_t need = gqa_prefill_backward_workspace_size(B, h_q, S_q);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
    return GQA_ERR_WORKSPACE;
  BackwardArgs a;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.o = o;
  a.d_o = d_o;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.q_start = q_start;
  a.kv_len = kv_len;
  a.B = B;
  a.h_q = h_q;
  a.h_kv = h_kv;
  a.S_q = S_q;
  a.T_max = T_max;
  a.d_h = d_h;
  a.scale = scale;
  a.causal = causal;
  a.window = window;
  const size_t half = (need - 256) / 2;
  a.lse2 = reinterpret_cast<float*>(workspace);
  a.drow = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + half);
  a.ticket = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(workspace) + 2 * half);
  a.err = device_error_ptr();
  if (!a.err) return GQA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GQA_FP32) return from_cuda(launch_backward_fp32(a, s));
  // TMA views: Q and dO as (d_h, S_q, B*h_q) with box (64, 64, 1) for the key-stationary dK/dV
  // kernel and (64, P, H) for the query-stationary dQ kernel; K, V as rows with box (64, 128) for
  // dK/dV (its 128 stationary keys) and (64, 64) for dQ (its 64-key blocks).
  const int H = prefill_heads_per_tile(h_q, h_kv);
  const uint32_t P = (uint32_t)(128 / H);
  CUtensorMap maps[8];
  const uint64_t qdims[3] = {(uint64_t)d_h, (uint64_t)S_q, (uint64_t)B * h_q};
  const uint64_t qstrides[2] = {(uint64_t)d_h * 2, (uint64_t)S_q * d_h * 2};
  const uint32_t qbox_rows[3] = {64, 64, 1};
  const uint32_t qbox_tile[3] = {64, P, (uint32_t)H};
  const uint64_t kdims[2] = {(uint64_t)d_h, (uint64_t)B * h_kv * T_max};
  const uint64_t strides[1] = {(uint64_t)d_h * 2};
  const uint32_t box[2] = {64, 128};
  const uint32_t box64[2] = {64, 64};
  if (!encode_bf16(&maps[6], k_cache, 2, kdims, strides, box64) ||
      !encode_bf16(&maps[7], v_cache, 2, kdims, strides, box64) ||
      !encode_bf16(&maps[0], q, 3, qdims, qstrides, qbox_rows) ||
      !encode_bf16(&maps[1], d_o, 3, qdims, qstrides, qbox_rows) ||
      !encode_bf16(&maps[2], k_cache, 2, kdims, strides, box) ||
      !encode_bf16(&maps[3], v_cache, 2, kdims, strides, box) ||
      !encode_bf16(&maps[4], q, 3, qdims, qstrides, qbox_tile) ||
      !encode_bf16(&maps[5], d_o, 3, qdims, qstrides, qbox_tile))
    return GQA_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return GQA_ERR_CUDA;
  return from_cuda(launch_backward_bf16(a, maps, sms, s));
}

size_t gqa_decode_workspace_size(int B, int h_q, int h_kv, int T_max, int d_h, gqa_dtype dtype,
                                 int num_splits) {
  if (B <= 0 || h_q <= 0 || h_kv <= 0 || T_max <= 0 || d_h <= 0 || h_q % h_kv != 0) return 0;
  if (num_splits < 0 || (dtype != GQA_BF16 && dtype != GQA_FP32)) return 0;
  const int sms = num_splits > 0 ? 1 : sm_count();
  if (sms <= 0) return 0;
  return decode_workspace_bytes(B, h_q, h_kv, T_max, d_h, num_splits, sms);
}

gqa_status gqa_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                      const int32_t* kv_len, const int32_t* q_pos,
                      int B, int h_q, int h_kv, int T_max, int d_h, float scale, int window,
                      gqa_dtype dtype, void* workspace, size_t workspace_bytes, int num_splits,
                      void* stream) {
  return decode_impl(q, k_cache, v_cache, o, lse, kv_len, q_pos, B, h_q, h_kv, T_max, d_h, scale,
                     window, dtype, workspace, workspace_bytes, num_splits, stream, nullptr, 0, 0, 0);
}

size_t gqa_mla_decode_workspace_size(int B, int h_q, int T_max, int d_v, gqa_dtype dtype,
                                     int num_splits) {
  if (B <= 0 || h_q <= 0 || T_max <= 0 || d_v <= 0 || num_splits < 0) return 0;
  if (dtype != GQA_BF16 && dtype != GQA_FP32) return 0;
  const int sms = num_splits > 0 ? 1 : sm_count();
  if (sms <= 0) return 0;
  return decode_workspace_bytes(B, h_q, 1, T_max, d_v, num_splits, sms, true, mla_uses_tc(h_q, dtype) != 0);
}

gqa_status gqa_mla_decode(const void* q, const void* cache, void* o, float* lse,
                          const int32_t* kv_len, const int32_t* q_pos, int B, int h_q, int T_max,
                          int d_qk, int d_v, float scale, gqa_dtype dtype, void* workspace,
                          size_t workspace_bytes, int num_splits, void* stream) {
  if (!q || !cache || !o) return GQA_ERR_INVALID_ARG;
  if (B <= 0 || h_q <= 0 || T_max <= 0 || d_qk <= 0 || d_v <= 0 || d_v > d_qk || num_splits < 0)
    return GQA_ERR_INVALID_ARG;
  if (!valid_scale(scale)) return GQA_ERR_INVALID_ARG;
  scale = resolve_scale(scale, d_qk);
  if (dtype != GQA_BF16 && dtype != GQA_FP32) return GQA_ERR_INVALID_ARG;
  if (dtype == GQA_BF16 && !mla_dims_supported_bf16(d_qk, d_v)) return GQA_ERR_UNSUPPORTED;
  if (dtype == GQA_FP32 && (d_qk > 768 || d_v > 512)) return GQA_ERR_UNSUPPORTED;
  if (B > decode_max_batch()) return GQA_ERR_UNSUPPORTED;
  if ((long long)B * T_max >= (1ll << 31) || (long long)B * h_q >= (1ll << 31)) return GQA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GQA_ERR_WORKSPACE;
  const bool tc = mla_uses_tc(h_q, dtype) != 0;
  if (num_splits > 0 && workspace_bytes < decode_workspace_bytes(B, h_q, 1, T_max, d_v, num_splits, 1, true, tc))
    return GQA_ERR_WORKSPACE;
  const int sms = sm_count();
  if (sms <= 0) return GQA_ERR_CUDA;
  if (workspace_bytes < decode_workspace_bytes(B, h_q, 1, T_max, d_v, num_splits, sms, true, tc))
    return GQA_ERR_WORKSPACE;
  DecodeArgs a;
  a.q = q;
  a.k = cache;
  a.v = cache;  // values are the first d_v entries of each cache row
  a.o = o;
  a.lse = lse;
  a.kv_len = kv_len;
  a.q_pos = q_pos;
  a.B = B;
  a.h_q = h_q;
  a.h_kv = 1;
  a.T_max = T_max;
  a.d_h = d_qk;
  a.d_v = d_v;
  a.mla = 1;
  a.mla_tc = tc ? 1 : 0;
  a.expire_wait = g_expire_waits.load(std::memory_order_relaxed);
  a.scale = scale;
  a.window = 0;
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  a.num_splits = num_splits;
  a.num_sms = sms;
  a.err = device_error_ptr();
  if (!a.err) return GQA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GQA_FP32) return from_cuda(launch_decode_fp32(a, s));
  CUtensorMap maps[4];
  const uint64_t cdims[2] = {(uint64_t)d_qk, (uint64_t)B * T_max};
  const uint64_t qdims[2] = {(uint64_t)d_qk, (uint64_t)B * h_q};
  const uint64_t strides[1] = {(uint64_t)d_qk * 2};
  const uint32_t cbox[2] = {64, 64};
  const uint32_t qbox[2] = {64, 16};
  // The tensor-core kernel reads rows as (64 columns, rows, 9 column chunks): one copy brings a
  // tile's chunks (the chunk dimension outermost in shared memory, one 128-byte row per key and
  // chunk) -- 32-key cache tiles, and the query's last 3 chunks of 128 heads.
  const uint64_t cdims3[3] = {64, (uint64_t)B * T_max, (uint64_t)d_qk / 64};
  const uint64_t qdims3[3] = {64, (uint64_t)B * h_q, (uint64_t)d_qk / 64};
  const uint64_t strides3[2] = {(uint64_t)d_qk * 2, 128};
  const uint32_t cbox_tc[3] = {64, 32, (uint32_t)d_qk / 64};
  const uint32_t qbox_tc[3] = {64, 128, 3};
  if (!encode_bf16(&maps[0], cache, 2, cdims, strides, cbox) ||
      !encode_bf16(&maps[1], q, 2, qdims, strides, qbox) ||
      (tc && (!encode_bf16(&maps[2], q, 3, qdims3, strides3, qbox_tc) ||
              !encode_bf16(&maps[3], cache, 3, cdims3, strides3, cbox_tc))))
    return GQA_ERR_CUDA;
  return from_cuda(launch_mla_bf16(a, maps, s));
}

gqa_status gqa_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* o,
                            float* lse, const int32_t* kv_len, const int32_t* q_pos,
                            const int32_t* block_table, int B, int h_q, int h_kv, int num_pages,
                            int page_size, int max_pages, int d_h, float scale, int window,
                            gqa_dtype dtype, void* workspace, size_t workspace_bytes,
                            int num_splits, void* stream) {
  if (!block_table || num_pages <= 0 || page_size <= 0 || max_pages <= 0) return GQA_ERR_INVALID_ARG;
  if (page_size % 16 != 0) return GQA_ERR_UNSUPPORTED;
  const long long T_max = (long long)max_pages * page_size;
  if (T_max >= (1ll << 31)) return GQA_ERR_UNSUPPORTED;
  return decode_impl(q, k_pages, v_pages, o, lse, kv_len, q_pos, B, h_q, h_kv, (int)T_max, d_h,
                     scale, window, dtype, workspace, workspace_bytes, num_splits, stream, block_table,
                     max_pages, page_size, num_pages);
}

gqa_status kv_append_paged(void* k_pages, void* v_pages, const void* k_new, const void* v_new,
                           const int32_t* pos, const int32_t* block_table, int B, int h_kv,
                           int S_new, int num_pages, int page_size, int max_pages, int d_h,
                           gqa_dtype dtype, void* stream) {
  using namespace gqa;
  if (!k_pages || !v_pages) return GQA_ERR_INVALID_ARG;
  if (S_new > 0 && (!k_new || !v_new || !pos || !block_table)) return GQA_ERR_INVALID_ARG;  // S_new = 0: no-op
  if (B <= 0 || h_kv <= 0 || S_new < 0 || d_h <= 0) return GQA_ERR_INVALID_ARG;
  if (num_pages <= 0 || page_size <= 0 || max_pages <= 0) return GQA_ERR_INVALID_ARG;
  if (dtype != GQA_BF16 && dtype != GQA_FP32) return GQA_ERR_INVALID_ARG;
  const long long T_max = (long long)max_pages * page_size;
  if (T_max >= (1ll << 31)) return GQA_ERR_UNSUPPORTED;
  if (S_new > T_max) return GQA_ERR_INVALID_ARG;
  if (S_new == 0) return GQA_OK;  // nothing to copy
  AppendArgs a;
  a.k_cache = k_pages;
  a.v_cache = v_pages;
  a.k_new = k_new;
  a.v_new = v_new;
  a.pos = pos;
  a.B = B;
  a.h_kv = h_kv;
  a.S_new = S_new;
  a.T_max = (int)T_max;
  a.d_h = d_h;
  a.elem_bytes = dtype == GQA_BF16 ? 2 : 4;
  a.block_table = block_table;
  a.max_pages = max_pages;
  a.page_size = page_size;
  a.num_pages = num_pages;
  a.err = device_error_ptr();
  if (!a.err) return GQA_ERR_CUDA;
  return from_cuda(launch_kv_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
