// Internal launcher interface between the C ABI (api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gqa.h"

namespace gqa {

struct AppendArgs {
  void* k_cache;
  void* v_cache;
  const void* k_new;
  const void* v_new;
  const int32_t* pos;
  int B, h_kv, S_new, T_max, d_h;
  int elem_bytes;
  unsigned* err;
  // paged cache (see DecodeArgs); T_max = max_pages * page_size
  const int32_t* block_table = nullptr;
  int max_pages = 0, page_size = 0, num_pages = 0;
};
cudaError_t launch_kv_append(const AppendArgs& a, cudaStream_t s);

struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const int32_t* q_start;
  const int32_t* kv_len;
  int B, h_q, h_kv, S_q, T_max, d_h;
  float scale;
  int causal;
  int window;  // 0: none; W > 0 (causal only): row at position p sees keys p - W < j <= p
  int expire_wait = 0;  // test hook (gqa_debug_expire_waits): one bounded wait runs out
  unsigned* err;
};
// fp32 check mode (scalar FFMA)
cudaError_t launch_prefill_fp32(const PrefillArgs& a, cudaStream_t s);
// bf16 tcgen05 path (sm_100a). tmaps: [0] = Q as a 3-D view (d_h, S_q, B*h_q) with box
// (64, 128 / H, H); [1] = K, [2] = V as 2-D views (d_h, B*h_kv*T_max) with box (64, 128).
cudaError_t launch_prefill_bf16(const PrefillArgs& a, const CUtensorMap* tmaps, int num_sms,
                                cudaStream_t s);
// query heads per prefill tile (H); a tile holds H heads x floor(128 / H) positions
int prefill_heads_per_tile(int h_q, int h_kv);

struct BackwardArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* d_o;
  const float* lse;  // natural-log lse from the forward pass (B, h_q, S_q)
  void* dq;
  void* dk;
  void* dv;
  const int32_t* q_start;
  const int32_t* kv_len;
  int B, h_q, h_kv, S_q, T_max, d_h;
  float scale;
  int causal, window;
  float* lse2;  // workspace: (B*h_q*S_q) base-2 lse
  float* drow;  // workspace: (B*h_q*S_q) rowsum(dO * O)
  int* ticket;  // workspace: the bf16 kernel's work-item counter (reset by its row-term kernel)
  unsigned* err;
};
// bf16 tcgen05 path. tmaps: [0] Q, [1] dO as 3-D views (d_h, S_q, B*h_q) with box (64, 64, 1);
// [2] K, [3] V as 2-D views (d_h, B*h_kv*T_max) with box (64, 128); [4] Q, [5] dO as 3-D views
// with the forward's box (64, 128 / H, H); [6] K, [7] V as 2-D views with box (64, 64).
cudaError_t launch_backward_bf16(const BackwardArgs& a, const CUtensorMap* tmaps, int num_sms,
                                 cudaStream_t s);
cudaError_t launch_backward_fp32(const BackwardArgs& a, cudaStream_t s);

struct DecodeArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const int32_t* kv_len;
  const int32_t* q_pos;
  int B, h_q, h_kv, T_max, d_h;
  float scale;
  void* workspace;
  size_t workspace_bytes;
  int num_splits;  // 0 = automatic chunking, else the number of chunks to cut the keys into
  int num_sms;     // persistent grid size
  int window = 0;  // 0: none; W > 0: the query at q_pos sees keys q_pos - W < j <= q_pos
  unsigned* err;
  // paged cache, or block_table == nullptr for the contiguous (B, h_kv, T_max, d_h) layout:
  // k/v are pools (num_pages, h_kv, page_size, d_h), T_max = max_pages * page_size
  const int32_t* block_table = nullptr;
  int max_pages = 0, page_size = 0, num_pages = 0;
  // paged, d_h = 128, page_size not a multiple of 64: K/V maps are 3-D views (64 columns,
  // num_pages*h_kv*page_size rows with a 256-byte stride, 2 column chunks with a 128-byte stride)
  // with box (64, 16, 2)
  int paged_3d = 0;
  // MLA: one shared cache row per token (k = v = the cache, h_kv = 1), d_h = the query / key row
  // width (576), d_v = the value / output width (the row's first 512 entries); 16 heads per unit
  int mla = 0;
  int d_v = 0;
  // MLA with a multiple of 128 heads (bf16): the tensor-core kernel, 128 heads per unit, each
  // chunk on two CTAs (one per half of the 512 value columns)
  int mla_tc = 0;
  int expire_wait = 0;  // test hook (gqa_debug_expire_waits), contiguous bf16 decode only
};

// The host-side argument checks of gqa_decode (contiguous: cache_rows = B * h_kv * T_max), in
// the order gqa_decode applies them; GQA_OK when the request may proceed to the workspace checks.
gqa_status decode_check_args(const void* q, const void* k_cache, const void* v_cache, const void* o,
                             int B, int h_q, int h_kv, int T_max, int d_h, float scale, int window,
                             gqa_dtype dtype, int num_splits, long long cache_rows);

// Workspace bytes for a decode of this shape (layout in decode.cu).
size_t decode_workspace_bytes(int B, int h_q, int h_kv, int T_max, int d_h, int num_splits,
                              int num_sms, bool mla = false, bool mla_tc = false);
int decode_max_batch();

cudaError_t launch_decode_fp32(const DecodeArgs& a, cudaStream_t s);
// tmaps: [0] = K cache, [1] = V cache as 2-D views (d_h, B*h_kv*T_max) with box (64, 64), or for
// a paged cache (d_h, num_pages*h_kv*page_size) with box (64, 16);
// [2] = queries as (d_h, B*h_q) with box (64, 16 or 32 rows: 32 when r > 16); SWIZZLE_128B.
cudaError_t launch_decode_bf16(const DecodeArgs& a, const CUtensorMap* tmaps, cudaStream_t s);
// MLA (bf16, d_h = 576, d_v = 512): tmaps [0] = the cache as (576, B*T_max) with box (64, 64),
// [1] = the queries as (576, B*h_q) with box (64, 16); when a.mla_tc, [2] the queries and [3]
// the cache as (64, rows, 9 chunks) with strides (1152, 128) bytes and boxes (64, 128, 3) and
// (64, 32, 9); SWIZZLE_128B.
cudaError_t launch_mla_bf16(const DecodeArgs& a, const CUtensorMap* tmaps, cudaStream_t s);
int mla_dims_supported_bf16(int d_qk, int d_v);
// 1 when gqa_mla_decode runs the tensor-core kernel for this head count and dtype
int mla_uses_tc(int h_q, gqa_dtype dtype);

}  // namespace gqa
