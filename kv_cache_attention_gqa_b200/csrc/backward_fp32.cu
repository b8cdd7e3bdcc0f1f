// Check-mode backward: fp32 inputs, scalar FFMA arithmetic, fp32 gradients, no tensor cores.
//
// Same mask, head-to-group map and recomputation from the saved lse as the tcgen05 kernels, so
// the indexing and masking of the backward pass can be checked against the fp64 oracle at a tight
// tolerance, independently of bf16 rounding:
//   p_ij = exp(scale q_i.k_j - lse_i),  dp_ij = dO_i.v_j,  ds_ij = p_ij (dp_ij - D_i),
//   dQ_i = scale sum_j ds_ij k_j,  dK_j = scale sum_{a in group, i} ds_ij q_i,
//   dV_j = sum_{a in group, i} p_ij dO_i
// [序列计算与存储, the paragraph after the 两块算例 listing; 第三章, section 3.5].
//   dq kernel    one warp per query row; lanes split d_h
//   dkdv kernel  one warp per (sequence, KV head, key); it walks every row of every head of the
//                group that sees the key. Keys at or past kv_len get zero gradient.

#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gqa {
namespace {

constexpr int kMaxPerLane = 8;  // d_h <= 256

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__device__ __forceinline__ bool seen(long long key, long long pos, int kv, int causal, int window) {
  return key < kv && (!causal || key <= pos) && (window == 0 || key > pos - window);
}

__global__ void __launch_bounds__(256) rowterm_fp32_kernel(BackwardArgs a) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= (long long)a.B * a.h_q * a.S_q) return;
  const float* o = reinterpret_cast<const float*>(a.o) + row * a.d_h;
  const float* d = reinterpret_cast<const float*>(a.d_o) + row * a.d_h;
  float s = 0.f;
  for (int c = lane; c < a.d_h; c += 32) s = fmaf(o[c], d[c], s);
  s = warp_sum(s);
  if (lane == 0) a.drow[row] = s;
}

__global__ void __launch_bounds__(256) dq_fp32_kernel(BackwardArgs a) {
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (long long)a.B * a.h_q * a.S_q) return;
  const int i = (int)(w % a.S_q);
  const int head = (int)((w / a.S_q) % a.h_q);
  const int b = (int)(w / ((long long)a.S_q * a.h_q));
  const int g = head / (a.h_q / a.h_kv);
  const int D = a.d_h;
  const int kv = a.kv_len ? a.kv_len[b] : a.T_max;
  const int qs = a.q_start ? a.q_start[b] : 0;
  float* dq = reinterpret_cast<float*>(a.dq) + w * D;
  const float lse = a.lse[w];
  if (kv < 1 || kv > a.T_max || qs < 0 || !(lse > -INFINITY)) {
    for (int c = lane; c < D; c += 32) dq[c] = 0.f;
    return;
  }
  const float* q = reinterpret_cast<const float*>(a.q) + w * D;
  const float* dO = reinterpret_cast<const float*>(a.d_o) + w * D;
  const long long kvb = ((long long)b * a.h_kv + g) * a.T_max * D;
  const float* kp = reinterpret_cast<const float*>(a.k) + kvb;
  const float* vp = reinterpret_cast<const float*>(a.v) + kvb;
  const float dr = a.drow[w];
  const long long pos = (long long)qs + i;
  float qr[kMaxPerLane], dor[kMaxPerLane], acc[kMaxPerLane];
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    const int c = lane + 32 * e;
    qr[e] = c < D ? q[c] : 0.f;
    dor[e] = c < D ? dO[c] : 0.f;
    acc[e] = 0.f;
  }
  for (int j = 0; j < kv; ++j) {
    if (!seen(j, pos, kv, a.causal, a.window)) continue;
    const float* kj = kp + (long long)j * D;
    const float* vj = vp + (long long)j * D;
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < kMaxPerLane; ++e) {
      const int c = lane + 32 * e;
      if (c < D) {
        s = fmaf(qr[e], kj[c], s);
        dp = fmaf(dor[e], vj[c], dp);
      }
    }
    s = warp_sum(s);
    dp = warp_sum(dp);
    const float p = expf(s * a.scale - lse);
    const float ds = p * (dp - dr);
#pragma unroll
    for (int e = 0; e < kMaxPerLane; ++e) {
      const int c = lane + 32 * e;
      if (c < D) acc[e] = fmaf(ds, kj[c], acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    const int c = lane + 32 * e;
    if (c < D) dq[c] = acc[e] * a.scale;
  }
}

__global__ void __launch_bounds__(256) dkdv_fp32_kernel(BackwardArgs a) {
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (long long)a.B * a.h_kv * a.T_max) return;
  const int j = (int)(w % a.T_max);
  const int g = (int)((w / a.T_max) % a.h_kv);
  const int b = (int)(w / ((long long)a.T_max * a.h_kv));
  const int D = a.d_h;
  const int r = a.h_q / a.h_kv;
  const int kv = a.kv_len ? a.kv_len[b] : a.T_max;
  const int qs = a.q_start ? a.q_start[b] : 0;
  float* dk = reinterpret_cast<float*>(a.dk) + w * D;
  float* dv = reinterpret_cast<float*>(a.dv) + w * D;
  float kr[kMaxPerLane], vr[kMaxPerLane], ak[kMaxPerLane], av[kMaxPerLane];
  const float* kj = reinterpret_cast<const float*>(a.k) + w * D;
  const float* vj = reinterpret_cast<const float*>(a.v) + w * D;
  const bool live = kv >= 1 && kv <= a.T_max && qs >= 0 && j < kv;
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    const int c = lane + 32 * e;
    kr[e] = live && c < D ? kj[c] : 0.f;
    vr[e] = live && c < D ? vj[c] : 0.f;
    ak[e] = 0.f;
    av[e] = 0.f;
  }
  if (live) {
    for (int hl = 0; hl < r; ++hl) {
      const int head = g * r + hl;
      const long long base = ((long long)b * a.h_q + head) * a.S_q;
      for (int i = 0; i < a.S_q; ++i) {
        if (!seen(j, (long long)qs + i, kv, a.causal, a.window)) continue;
        const float lse = a.lse[base + i];
        if (!(lse > -INFINITY)) continue;
        const float* q = reinterpret_cast<const float*>(a.q) + (base + i) * D;
        const float* dO = reinterpret_cast<const float*>(a.d_o) + (base + i) * D;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < kMaxPerLane; ++e) {
          const int c = lane + 32 * e;
          if (c < D) {
            s = fmaf(q[c], kr[e], s);
            dp = fmaf(dO[c], vr[e], dp);
          }
        }
        s = warp_sum(s);
        dp = warp_sum(dp);
        const float p = expf(s * a.scale - lse);
        const float ds = p * (dp - a.drow[base + i]);
#pragma unroll
        for (int e = 0; e < kMaxPerLane; ++e) {
          const int c = lane + 32 * e;
          if (c < D) {
            av[e] = fmaf(p, dO[c], av[e]);
            ak[e] = fmaf(ds, q[c], ak[e]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    const int c = lane + 32 * e;
    if (c < D) {
      dk[c] = ak[e] * a.scale;
      dv[c] = av[e];
    }
  }
}

}  // namespace

cudaError_t launch_backward_fp32(const BackwardArgs& a, cudaStream_t s) {
  const long long rows = (long long)a.B * a.h_q * a.S_q;
  const long long keys = (long long)a.B * a.h_kv * a.T_max;
  if ((rows * 32 + 255) / 256 > 0x7fffffffLL || (keys * 32 + 255) / 256 > 0x7fffffffLL)
    return cudaErrorInvalidConfiguration;
  if (rows > 0) {
    rowterm_fp32_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dq_fp32_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (keys > 0) dkdv_fp32_kernel<<<(unsigned)((keys * 32 + 255) / 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace gqa
