// Check-mode prefill: fp32 inputs, scalar FFMA arithmetic, fp32 output, no tensor cores.
//
// Same head-to-group map, absolute-position mask and online softmax as the bf16 tensor-core
// kernel, but with fp32 operands, so indexing, masking and the recurrence can be checked against
// the fp64 oracle at a 1e-5 relative tolerance independently of bf16 rounding.
//
// One warp owns one query row (b, a, i). Lane l holds the d_h elements c = l + 32 e of the query
// and of the running output. For each visible key j (j < min(kv_len[b], q_start[b]+i+1) under the
// causal mask, and j > q_start[b]+i - W under a sliding window of W), the warp forms s_j = scale * q . k_j with a shuffle reduction and applies
// the online-softmax update with a block of one key:
//   m' = max(m, s_j),  l' = e^{m - m'} l + e^{s_j - m'},  u' = e^{m - m'} u + e^{s_j - m'} v_j
// [序列计算与存储, section 在线 softmax], starting from m = -inf, l = 0, u = 0; o = u / l.

#include "common.cuh"
#include "internal.h"

namespace gqa {
namespace {

constexpr int kMaxPerLane = 8;  // d_h <= 256

__global__ void __launch_bounds__(256) prefill_fp32_kernel(PrefillArgs a) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)a.B * a.h_q * a.S_q;
  if (warp >= rows) return;
  const int i = warp % a.S_q;
  const int bh = warp / a.S_q;
  const int head = bh % a.h_q;
  const int b = bh / a.h_q;
  const int r = a.h_q / a.h_kv;
  const int g = head / r;  // g(a) = floor(a / r)
  const int D = a.d_h;

  const float* q = reinterpret_cast<const float*>(a.q) + (long long)warp * D;
  float* o = reinterpret_cast<float*>(a.o) + (long long)warp * D;
  const long long kv_base = ((long long)b * a.h_kv + g) * a.T_max * D;
  const float* kp = reinterpret_cast<const float*>(a.k) + kv_base;
  const float* vp = reinterpret_cast<const float*>(a.v) + kv_base;

  const int kv_len = a.kv_len ? a.kv_len[b] : a.T_max;
  const int q0 = a.q_start ? a.q_start[b] : 0;
  int n_vis = -1, j_lo = 0;
  if (kv_len < 1 || kv_len > a.T_max) {
    if (lane == 0) set_device_error(a.err, GQA_DEVERR_KV_LEN);
  } else if (q0 < 0) {
    if (lane == 0) set_device_error(a.err, GQA_DEVERR_POSITION);
  } else {
    const long long lim = (long long)q0 + i + 1;
    n_vis = a.causal ? (int)(lim < kv_len ? lim : kv_len) : kv_len;
    if (a.window > 0) {
      const long long lo = lim - a.window;  // first key inside the window
      if (lo > 0) j_lo = lo < n_vis ? (int)lo : n_vis;
      n_vis -= j_lo;
    }
  }
  if (n_vis <= 0) {  // invalid request or no visible key: zero row, flagged
    if (n_vis == 0 && lane == 0) set_device_error(a.err, GQA_DEVERR_NO_VISIBLE);
    for (int c = lane; c < D; c += 32) o[c] = 0.f;
    if (a.lse && lane == 0) a.lse[warp] = -INFINITY;
    return;
  }

  float qr[kMaxPerLane], acc[kMaxPerLane];
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    const int c = lane + 32 * e;
    qr[e] = c < D ? q[c] : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j = j_lo; j < j_lo + n_vis; ++j) {
    const float* kj = kp + (long long)j * D;
    const float* vj = vp + (long long)j * D;
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < kMaxPerLane; ++e) {
      const int c = lane + 32 * e;
      if (c < D) part = fmaf(qr[e], kj[c], part);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    const float s = part * a.scale;
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new);  // 0 on the first key (m = -inf)
    const float p = expf(s - m_new);
    l = fmaf(l, alpha, p);
#pragma unroll
    for (int e = 0; e < kMaxPerLane; ++e) {
      const int c = lane + 32 * e;
      if (c < D) acc[e] = fmaf(acc[e], alpha, p * vj[c]);
    }
    m = m_new;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    const int c = lane + 32 * e;
    if (c < D) o[c] = acc[e] * inv;
  }
  if (a.lse && lane == 0) a.lse[warp] = m + logf(l);
}

}  // namespace

cudaError_t launch_prefill_fp32(const PrefillArgs& a, cudaStream_t s) {
  const long long rows = (long long)a.B * a.h_q * a.S_q;
  const long long blocks = (rows * 32 + 255) / 256;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  prefill_fp32_kernel<<<(unsigned)blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace gqa
