// kv_append: copy new K/V rows into the unexpanded cache at per-sequence positions.
//
// A decode (or chunked-prefill) step appends the new tokens' K/V to the cache before attending
// [第三章：MHA 的局限与 MQA、GQA、Flash Attention, section 3.1; MHA/MQA/GQA walkthrough,
// section 4]. The copy is bit-exact and memory-bound: every byte moves once, in 16-byte vectors
// when the row size allows, else in 4- or 2-byte words. On a paged cache each row goes to the
// page the block table names for its logical position.

#include "common.cuh"
#include "internal.h"

namespace gqa {
namespace {

// One thread moves one `Vec` of one row of K and the same of V. Rows are (b, g, t) triples.
template <typename Vec>
__global__ void __launch_bounds__(256) kv_append_kernel(AppendArgs a, int vecs_per_row,
                                                         long long total) {
  // A decode launched as a programmatic dependent of this copy may start its prologue now; it
  // reads the cache only after this grid has completed (griddepcontrol.wait).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const long long row = i / vecs_per_row;
    const int c = (int)(i - row * vecs_per_row);
    const int t = (int)(row % a.S_new);
    const long long bg = row / a.S_new;  // b * h_kv + g
    const int b = (int)(bg / a.h_kv);
    const int p = a.pos[b];
    if (p < 0 || (long long)p + a.S_new > a.T_max) {
      if (t == 0 && c == 0) set_device_error(a.err, GQA_DEVERR_POSITION);
      continue;
    }
    long long dst_row;
    if (a.block_table) {
      // paged: logical position p + t is row (p + t) % page_size of page table[b][(p + t) / page_size]
      const int pt = p + t;
      const int page = a.block_table[(long long)b * a.max_pages + pt / a.page_size];
      if (page < 0 || page >= a.num_pages) {
        if (c == 0) set_device_error(a.err, GQA_DEVERR_PAGE);
        continue;
      }
      const int g = (int)(bg - (long long)b * a.h_kv);
      dst_row = ((long long)page * a.h_kv + g) * a.page_size + pt % a.page_size;
    } else {
      dst_row = bg * a.T_max + p + t;
    }
    const Vec* ks = reinterpret_cast<const Vec*>(a.k_new) + row * vecs_per_row + c;
    const Vec* vs = reinterpret_cast<const Vec*>(a.v_new) + row * vecs_per_row + c;
    Vec* kd = reinterpret_cast<Vec*>(a.k_cache) + dst_row * vecs_per_row + c;
    Vec* vd = reinterpret_cast<Vec*>(a.v_cache) + dst_row * vecs_per_row + c;
    *kd = __ldg(ks);
    *vd = __ldg(vs);
  }
}

template <typename Vec>
cudaError_t launch_typed(const AppendArgs& a, cudaStream_t s) {
  const long long row_bytes = (long long)a.d_h * a.elem_bytes;
  const int vecs_per_row = (int)(row_bytes / sizeof(Vec));
  const long long total = (long long)a.B * a.h_kv * a.S_new * vecs_per_row;
  if (total == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)sms * 8;
  if (blocks > cap) blocks = cap;
  kv_append_kernel<Vec><<<(unsigned)blocks, 256, 0, s>>>(a, vecs_per_row, total);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_append(const AppendArgs& a, cudaStream_t s) {
  const long long row_bytes = (long long)a.d_h * a.elem_bytes;
  const uintptr_t all = (uintptr_t)a.k_cache | (uintptr_t)a.v_cache | (uintptr_t)a.k_new |
                        (uintptr_t)a.v_new;
  if (row_bytes % 16 == 0 && all % 16 == 0) return launch_typed<uint4>(a, s);
  if (row_bytes % 4 == 0 && all % 4 == 0) return launch_typed<uint32_t>(a, s);
  return launch_typed<uint16_t>(a, s);
}

}  // namespace gqa
