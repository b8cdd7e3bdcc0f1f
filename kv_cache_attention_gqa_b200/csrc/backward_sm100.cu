// Backward pass of grouped-query attention on sm_100a (bf16 in, fp32 accumulate, bf16 out).
//
// What it computes: the gradients of O_a = softmax(Q_a K_g^T * scale + M) V_g (g = floor(a / r))
// for an upstream gradient dO, recomputing the probabilities from the forward pass's saved
// log-sum-exp instead of storing them [序列计算与存储, the paragraph after the 两块算例 listing;
// 第三章：MHA 的局限与 MQA、GQA、Flash Attention, section 3.5]:
//   P = exp(S - lse),  dV_g += P^T dO_a,  dP = dO_a V_g^T,  D = rowsum(dO_a * O_a),
//   dS = P * (dP - D),  dQ_a = scale dS K_g,  dK_g += scale dS^T Q_a.
// The mask is the forward's: causal by absolute position, length, and an optional sliding window.
//
// Three launches:
//   rowterm   one warp per query row: D = rowsum(dO * O) and the base-2 lse (fp32 workspace).
//   dkdv      one CTA per (sequence, KV head, 128-key block). The keys sit on the 128 TMEM lanes;
//             the CTA walks every query block of every head of the group, so the r heads' shares
//             of dK and dV add up in TMEM (no atomics):
//               S^T  = K Q^T     tcgen05.mma, A = K and B = Q from shared memory (K-major)
//               dP^T = V dO^T    A = V, B = dO from shared memory
//               (4 warps) P^T = 2^(S^T c - lse2), dS^T = P^T (dP^T - D) -> bf16 into TMEM
//               dV  += P^T dO    A = P^T from TMEM, B = dO (MN-major view of the same tile)
//               dK  += dS^T Q    A = dS^T from TMEM, B = Q (MN-major)
//   dq        one CTA per forward tile (H heads x P positions of one group), walking the K/V
//             blocks the tile sees:
//               S = Q K^T, dP = dO V^T (A = Q / dO, B = K / V from shared memory), then dS -> bf16
//               into TMEM, dQ += dS K (A = dS from TMEM, B = K, MN-major view).
// TMEM (512 columns): S [0,128), dP [128,256), accumulators from 256; P / dS (bf16 pairs) alias
// the first 64 columns of S / dP. MMAs issued by one thread execute in order, so the next
// block's S is written only after the accumulating MMAs have read P / dS.
//
// Every tcgen05.ld/st/wait sits behind warp-uniform conditions; every mbarrier wait is bounded
// (2 s of %globaltimer) and sets GQA_DEVERR_TIMEOUT instead of hanging.

#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace gqa {
namespace bw {

constexpr int kBK = 128;  // keys per block (dkdv: the CTA's keys; dq: per K/V block)
constexpr int kBQ = 128;  // query rows per block
constexpr int kThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 elementwise (TMEM lanes)
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kColS = 0, kColDP = 128, kColAcc0 = 256;

struct BArgs {
  const float* lse2;  // (B*h_q*S_q) base-2 log-sum-exp per row (+inf for a row with no key)
  const float* drow;  // (B*h_q*S_q) D = rowsum(dO * O)
  void* dq;
  void* dk;
  void* dv;
  const int32_t* q_start;
  const int32_t* kv_len;
  int B, h_q, h_kv, r, S_q, T_max;
  int H, P, hblocks, n_qt;  // dq tiles: H heads x P positions (as in the forward)
  int n_kb;                 // key blocks per (b, g): ceil(T_max / 128)
  float scale, sl2;         // scale and scale * log2(e)
  int causal, window;
  unsigned* err;
};

// Bounded mbarrier wait shared by all roles: gives up after 2 s (or when another thread of the
// CTA gave up), records GQA_DEVERR_TIMEOUT and returns false.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort,
                                         unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        set_device_error(err, GQA_DEVERR_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool visible(long long key, long long pos, int kv, int causal, int window) {
  return key < kv && (!causal || key <= pos) && (window == 0 || key > pos - window);
}

// ---- K-major / MN-major shared-memory descriptors for a 128-row bf16 tile in 64-column chunks
// (128-byte swizzle, as written by TMA with a 64 x 128 box per chunk).
// K-major (the tile's columns are the contraction): k-th 16-wide step.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int k) {
  return tc::smem_desc(tile + (uint32_t)((k >> 2) * (128 * 128) + (k & 3) * 32), 16, 1024);
}
// MN-major (the tile's rows are the contraction, its columns the N dimension): kk-th 16-row step;
// the 64-column chunks are the leading-dimension stride.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int kk) {
  return tc::smem_desc(tile + (uint32_t)(kk * 2048), 128 * 128, 1024);
}

// =============================================================================================
// rowterm: D = rowsum(dO * O), lse2 = lse * log2(e) (+inf for rows without a visible key)
// =============================================================================================
template <typename T>
__global__ void __launch_bounds__(256) rowterm_kernel(const T* o, const T* d_o, const float* lse,
                                                      float* lse2, float* drow, long long rows, int D) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T* a = o + row * D;
  const T* b = d_o + row * D;
  float s = 0.f;
  for (int c = lane; c < D; c += 32) s = fmaf(static_cast<float>(a[c]), static_cast<float>(b[c]), s);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    drow[row] = s;
    const float l = lse[row];
    lse2[row] = l == -INFINITY || l != l ? INFINITY : l * kLog2e;
  }
}


// Shared memory of the dkdv kernel (D = head dim): K and V blocks, a two-stage ring of Q and dO
// blocks with their rows' lse2 and D, barriers.
template <int D>
struct KvCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kTile = kNch * 128 * 128;  // one 128-row bf16 tile
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTile;
  static constexpr int kOffQ = 2 * kTile;               // + stage * 2 * kTile
  static constexpr int kOffDO = 3 * kTile;              // + stage * 2 * kTile
  static constexpr int kOffStat = 6 * kTile;            // 2 stages x (lse2[128], D[128]) floats
  static constexpr int kOffBar = kOffStat + 2 * 2 * 128 * 4;
  static constexpr int kSmem = (kOffBar + 256 + 1024) > 120 * 1024 ? kOffBar + 256 + 1024 : 120 * 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};
enum { kKvFull = 0, kQFull = 1, kQEmpty = 3, kKvS = 5, kKvP = 6, kKvDone = 7, kKvBars = 8 };

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmdo,
                const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                BArgs a) {
  using C = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kKvBars);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* stat = reinterpret_cast<float*>(smem + C::kOffStat);  // [stage][lse2 128 | D 128]
  const uint32_t sK = smem_u32(smem + C::kOffK), sV = smem_u32(smem + C::kOffV);
  auto sQ = [&](int st) { return smem_u32(smem + C::kOffQ + st * 2 * C::kTile); };
  auto sDO = [&](int st) { return smem_u32(smem + C::kOffDO + st * 2 * C::kTile); };
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- this CTA's keys and the query blocks that see them
  const int per = a.B * a.h_kv;
  const int kb = blockIdx.x / per;
  const int b = (blockIdx.x - kb * per) / a.h_kv;
  const int g = blockIdx.x - kb * per - b * a.h_kv;
  const int k0 = kb * kBK;
  const int kv = a.kv_len ? a.kv_len[b] : a.T_max;
  const int qs = a.q_start ? a.q_start[b] : 0;
  const bool valid = kv >= 1 && kv <= a.T_max && qs >= 0;
  const int n_qb = (a.S_q + kBQ - 1) / kBQ;
  int qb_lo = 0, qb_hi = -1;
  if (valid && k0 < kv) {
    qb_hi = n_qb - 1;
    if (a.causal) {
      const long long first_q = (long long)k0 - qs;  // earliest row that can see key k0
      qb_lo = first_q > 0 ? (int)(first_q / kBQ) : 0;
      if (a.window > 0) {
        const long long k_last = min(k0 + kBK, kv) - 1;
        const long long last_q = k_last + a.window - 1 - qs;  // latest row that can see k_last
        qb_hi = last_q < 0 ? -1 : (int)min((long long)qb_hi, last_q / kBQ);
      }
    }
  }
  const int nq = qb_hi >= qb_lo ? qb_hi - qb_lo + 1 : 0;
  const int n_it = nq * a.r;  // (head, query block) pairs

  if (threadIdx.x == 0) {
    mbar_init(bar(kKvFull), 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(bar(kQFull + st), 1 + 32);  // the TMA arrival plus the producer warp's stat rows
      mbar_init(bar(kQEmpty + st), 1);
    }
    mbar_init(bar(kKvS), 1);
    mbar_init(bar(kKvP), 128);
    mbar_init(bar(kKvDone), 1);
    *abort = 0;
    fence_barrier_init();
    if (!valid && kb == 0 && g == 0)
      set_device_error(a.err, kv < 1 || kv > a.T_max ? GQA_DEVERR_KV_LEN : GQA_DEVERR_POSITION);
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  auto head_of = [&](int it) { return g * a.r + it / nq; };
  auto qblk_of = [&](int it) { return qb_lo + it % nq; };

  if (warp == 0 && n_it > 0) {
    // ------------------------------ producer: TMA + the rows' statistics --------------------
    if (lane == 0) {
      tma_prefetch_desc(&tmq);
      tma_prefetch_desc(&tmdo);
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      const int krow = (b * a.h_kv + g) * a.T_max + k0;
      mbar_arrive_expect_tx(bar(kKvFull), 2 * C::kTile);
      for (int ch = 0; ch < C::kNch; ++ch) {
        tma_load_2d(sK + ch * 128 * 128, &tmk, bar(kKvFull), ch * 64, krow);
        tma_load_2d(sV + ch * 128 * 128, &tmv, bar(kKvFull), ch * 64, krow);
      }
    }
    int last[2] = {-1, -1};
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1, n = it >> 1;
      int ok = 1;
      if (n > 0 && lane == 0) ok = wait_bar(bar(kQEmpty + st), (uint32_t)((n - 1) & 1), abort, a.err);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int h = head_of(it), qb = qblk_of(it);
      const int z = b * a.h_q + h;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(kQFull + st), 2 * C::kTile);
        for (int ch = 0; ch < C::kNch; ++ch) {
          tma_load_3d(sQ(st) + ch * 128 * 128, &tmq, bar(kQFull + st), ch * 64, qb * kBQ, z);
          tma_load_3d(sDO(st) + ch * 128 * 128, &tmdo, bar(kQFull + st), ch * 64, qb * kBQ, z);
        }
      }
      float* sl = stat + st * 256;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = lane * 4 + e;
        const int qi = qb * kBQ + c;
        const long long row = (long long)z * a.S_q + qi;
        sl[c] = qi < a.S_q ? a.lse2[row] : INFINITY;
        sl[128 + c] = qi < a.S_q ? a.drow[row] : 0.f;
      }
      mbar_arrive(bar(kQFull + st));
      last[st] = n;
    }
    if (lane == 0) {  // drain (bounded): no copy may still land in shared memory at exit
      volatile int no_abort = 0;
      wait_bar(bar(kKvFull), 0, &no_abort, a.err);
      for (int st = 0; st < 2; ++st)
        if (last[st] >= 0) wait_bar(bar(kQFull + st), (uint32_t)(last[st] & 1), &no_abort, a.err);
    }
  } else if (warp == 1 && lane == 0 && n_it > 0) {
    // ------------------------------ MMA issuer ---------------------------------------------
    constexpr uint32_t idesc_s = tc::idesc_bf16(128, kBQ, false);  // S^T, dP^T: M keys, N queries
    constexpr uint32_t idesc_acc = tc::idesc_bf16(128, D, true);   // dV, dK: M keys, N = d_h
    bool ok = wait_bar(bar(kKvFull), 0, abort, a.err);
    for (int it = 0; it < n_it && ok; ++it) {
      const int st = it & 1;
      if (!wait_bar(bar(kQFull + st), (uint32_t)((it >> 1) & 1), abort, a.err)) break;
      tc::fence_after_sync();
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        tc::mma_ss(tmem + kColS, desc_kmajor(sK, k), desc_kmajor(sQ(st), k), idesc_s, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        tc::mma_ss(tmem + kColDP, desc_kmajor(sV, k), desc_kmajor(sDO(st), k), idesc_s, k > 0 ? 1u : 0u);
      tc::commit(bar(kKvS));
      if (!wait_bar(bar(kKvP), (uint32_t)(it & 1), abort, a.err)) break;
      tc::fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < kBQ / 16; ++kk) {
        const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
        tc::mma_ts(tmem + kColAcc0, tmem + kColS + kk * 8, desc_mnmajor(sDO(st), kk), idesc_acc, acc);
        tc::mma_ts(tmem + kColAcc0 + D, tmem + kColDP + kk * 8, desc_mnmajor(sQ(st), kk), idesc_acc, acc);
      }
      tc::commit(bar(kQEmpty + st));
    }
    tc::commit(bar(kKvDone));
    volatile int no_abort = 0;
    wait_bar(bar(kKvDone), 0, &no_abort, a.err);
  } else if (warp >= 2) {
    // ------------------------------ elementwise: one key row per thread --------------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // TMEM lane = key k0 + row
    const int key = k0 + row;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int st = it & 1;
      if (ok) ok = wait_bar(bar(kKvS), (uint32_t)(it & 1), abort, a.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      // the stage's statistics: written by the producer warp before its arrivals on the stage's
      // full barrier (already complete here; waiting on it orders the reads after those writes)
      if (ok) ok = wait_bar(bar(kQFull + st), (uint32_t)((it >> 1) & 1), abort, a.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const float* sl = stat + st * 256;
      const int qb = qblk_of(it);
      const long long pos0 = (long long)qs + qb * kBQ;  // position of the block's first row
      const bool need_mask = k0 + kBK > kv || qb * kBQ + kBQ > a.S_q ||
                             (a.causal && (long long)k0 + kBK - 1 > pos0) ||
                             (a.window > 0 && (long long)k0 <= pos0 + kBQ - 1 - a.window);
      tc::fence_after_sync();
#pragma unroll 1
      for (int c = 0; c < kBQ / 32; ++c) {
        uint32_t sv[32], dv[32];
        tc::ld32(lane_addr + kColS + c * 32, sv);
        tc::ld32(lane_addr + kColDP + c * 32, dv);
        tc::wait_ld();
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          float p2[2], d2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int col = c * 32 + x + e;
            const float sc = __uint_as_float(sv[x + e]);
            float p = fast_exp2(fmaf(sc, a.sl2, -sl[col]));
            float ds = p * (__uint_as_float(dv[x + e]) - sl[128 + col]);
            if (need_mask && !(qb * kBQ + col < a.S_q && visible(key, pos0 + col, kv, a.causal, a.window))) {
              p = 0.f;
              ds = 0.f;
            }
            p2[e] = p;
            d2[e] = ds;
          }
          pp[x / 2] = pack_bf16x2(p2[0], p2[1]);
          pd[x / 2] = pack_bf16x2(d2[0], d2[1]);
        }
        tc::st16(lane_addr + kColS + c * 16, pp);   // P^T (bf16 pairs) over S^T's first columns
        tc::st16(lane_addr + kColDP + c * 16, pd);  // dS^T over dP^T's first columns
      }
      tc::wait_st();
      tc::fence_before_sync();
      mbar_arrive(bar(kKvP));
    }
    // ---- epilogue: dV and scale * dK rows -> bf16 (rows past kv_len hold zeros)
    bool have = n_it > 0 && ok;
    if (have) {
      have = wait_bar(bar(kKvDone), 0, abort, a.err);
      have = __all_sync(0xffffffffu, have);
      if (have) tc::fence_after_sync();
    }
    if (key < a.T_max) {
      const long long orow = ((long long)b * a.h_kv + g) * a.T_max + key;
      uint4* dvo = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dv) + orow * D);
      uint4* dko = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dk) + orow * D);
      if (!have) {
        for (int v = 0; v < D / 8; ++v) {
          dvo[v] = make_uint4(0u, 0u, 0u, 0u);
          dko[v] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    if (have) {
      const bool store = key < a.T_max;
      const long long orow = ((long long)b * a.h_kv + g) * a.T_max + key;
      uint4* dvo = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dv) + orow * D);
      uint4* dko = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dk) + orow * D);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32], k[32];
        tc::ld32(lane_addr + kColAcc0 + c * 32, v);
        tc::ld32(lane_addr + kColAcc0 + D + c * 32, k);
        tc::wait_ld();
        uint32_t pv[16], pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          pv[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          pk[i] = pack_bf16x2(__uint_as_float(k[2 * i]) * a.scale, __uint_as_float(k[2 * i + 1]) * a.scale);
        }
        if (store) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            dvo[c * 4 + q] = make_uint4(pv[4 * q], pv[4 * q + 1], pv[4 * q + 2], pv[4 * q + 3]);
            dko[c * 4 + q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}


// Shared memory of the dq kernel: the tile's Q and dO rows, a two-stage ring of K and V blocks.
template <int D>
struct QCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kTile = kNch * 128 * 128;
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kTile;
  static constexpr int kOffK = 2 * kTile;  // + stage * 2 * kTile
  static constexpr int kOffV = 3 * kTile;  // + stage * 2 * kTile
  static constexpr int kOffBar = 6 * kTile;
  static constexpr int kSmem = (kOffBar + 256 + 1024) > 120 * 1024 ? kOffBar + 256 + 1024 : 120 * 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};
enum { kQdQ = 0, kQKvFull = 1, kQKvEmpty = 3, kQS = 5, kQP = 6, kQDone = 7, kQBars = 8 };

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmdo,
              const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
              BArgs a) {
  using C = QCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kQBars);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t sQ = smem_u32(smem + C::kOffQ), sDO = smem_u32(smem + C::kOffDO);
  auto sK = [&](int st) { return smem_u32(smem + C::kOffK + st * 2 * C::kTile); };
  auto sV = [&](int st) { return smem_u32(smem + C::kOffV + st * 2 * C::kTile); };
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- the tile (as in the forward): H heads x P positions of one group, heaviest first
  const int per = a.B * a.h_kv * a.hblocks;
  const int qt = a.n_qt - 1 - (int)(blockIdx.x / per);
  const int rem = blockIdx.x - (blockIdx.x / per) * per;
  const int b = rem / (a.h_kv * a.hblocks);
  const int gh = rem - b * (a.h_kv * a.hblocks);
  const int g = gh / a.hblocks, hb = gh - g * a.hblocks;
  const int q0 = qt * a.P;
  const int nh = min(a.H, a.r - hb * a.H);
  const int kv = a.kv_len ? a.kv_len[b] : a.T_max;
  const int qs = a.q_start ? a.q_start[b] : 0;
  const bool valid = kv >= 1 && kv <= a.T_max && qs >= 0;
  const long long pos_min = (long long)qs + q0;
  const long long pos_max = (long long)qs + min(q0 + a.P, a.S_q) - 1;
  int j0 = 0, nb = 0;
  if (valid) {
    int end = (kv + kBK - 1) / kBK;
    if (a.causal) {
      const long long last_key = pos_max < kv - 1 ? pos_max : (long long)(kv - 1);
      end = (int)(last_key / kBK) + 1;
      if (a.window > 0) {
        const long long lo = pos_min - a.window + 1;
        if (lo > 0) j0 = (int)(lo / kBK);
      }
    }
    nb = end > j0 ? end - j0 : 0;
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(kQdQ), 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(bar(kQKvFull + st), 1);
      mbar_init(bar(kQKvEmpty + st), 1);
    }
    mbar_init(bar(kQS), 1);
    mbar_init(bar(kQP), 128);
    mbar_init(bar(kQDone), 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int row0 = (b * a.h_kv + g) * a.T_max;

  if (warp == 0 && lane == 0 && nb > 0) {
    // ------------------------------ TMA producer ------------------------------------------
    tma_prefetch_desc(&tmq);
    tma_prefetch_desc(&tmdo);
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
    const int zq = b * a.h_q + g * a.r + hb * a.H;
    mbar_arrive_expect_tx(bar(kQdQ), (uint32_t)(2 * C::kNch * a.H * a.P * 128));
    for (int ch = 0; ch < C::kNch; ++ch) {
      tma_load_3d(sQ + ch * 128 * 128, &tmq, bar(kQdQ), ch * 64, q0, zq);
      tma_load_3d(sDO + ch * 128 * 128, &tmdo, bar(kQdQ), ch * 64, q0, zq);
    }
    int last[2] = {-1, -1};
    for (int j = 0; j < nb; ++j) {
      const int st = j & 1, n = j >> 1;
      if (n > 0 && !wait_bar(bar(kQKvEmpty + st), (uint32_t)((n - 1) & 1), abort, a.err)) break;
      mbar_arrive_expect_tx(bar(kQKvFull + st), 2 * C::kTile);
      for (int ch = 0; ch < C::kNch; ++ch) {
        tma_load_2d(sK(st) + ch * 128 * 128, &tmk, bar(kQKvFull + st), ch * 64, row0 + (j0 + j) * kBK);
        tma_load_2d(sV(st) + ch * 128 * 128, &tmv, bar(kQKvFull + st), ch * 64, row0 + (j0 + j) * kBK);
      }
      last[st] = n;
    }
    volatile int no_abort = 0;  // drain (bounded)
    wait_bar(bar(kQdQ), 0, &no_abort, a.err);
    for (int st = 0; st < 2; ++st)
      if (last[st] >= 0) wait_bar(bar(kQKvFull + st), (uint32_t)(last[st] & 1), &no_abort, a.err);
  } else if (warp == 1 && lane == 0 && nb > 0) {
    // ------------------------------ MMA issuer ---------------------------------------------
    constexpr uint32_t idesc_s = tc::idesc_bf16(128, kBK, false);  // S, dP: M rows, N keys
    constexpr uint32_t idesc_acc = tc::idesc_bf16(128, D, true);   // dQ: M rows, N = d_h
    bool ok = wait_bar(bar(kQdQ), 0, abort, a.err);
    for (int j = 0; j < nb && ok; ++j) {
      const int st = j & 1;
      if (!wait_bar(bar(kQKvFull + st), (uint32_t)((j >> 1) & 1), abort, a.err)) break;
      tc::fence_after_sync();
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        tc::mma_ss(tmem + kColS, desc_kmajor(sQ, k), desc_kmajor(sK(st), k), idesc_s, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        tc::mma_ss(tmem + kColDP, desc_kmajor(sDO, k), desc_kmajor(sV(st), k), idesc_s, k > 0 ? 1u : 0u);
      tc::commit(bar(kQS));
      if (!wait_bar(bar(kQP), (uint32_t)(j & 1), abort, a.err)) break;
      tc::fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk)
        tc::mma_ts(tmem + kColAcc0, tmem + kColS + kk * 8, desc_mnmajor(sK(st), kk), idesc_acc,
                   (j > 0 || kk > 0) ? 1u : 0u);
      tc::commit(bar(kQKvEmpty + st));
    }
    tc::commit(bar(kQDone));
    volatile int no_abort = 0;
    wait_bar(bar(kQDone), 0, &no_abort, a.err);
  } else if (warp >= 2) {
    // ------------------------------ elementwise: one query row per thread ------------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // TMEM lane = tile row (head h, position p)
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const int h = row / a.P, p = row - h * a.P;
    const int qi = q0 + p;
    const bool store_row = h < nh && row < a.H * a.P && qi < a.S_q;
    const int head = g * a.r + hb * a.H + h;
    const long long srow = ((long long)b * a.h_q + head) * a.S_q + qi;
    const long long pos = (long long)qs + qi;
    const float lse2 = store_row ? a.lse2[srow] : INFINITY;
    const float dr = store_row ? a.drow[srow] : 0.f;
    bool ok = true;
    for (int j = 0; j < nb; ++j) {
      const int st = j & 1;
      if (ok) ok = wait_bar(bar(kQS), (uint32_t)(j & 1), abort, a.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int key0 = (j0 + j) * kBK;
      const bool need_mask = (a.causal && (long long)key0 + kBK - 1 > pos_min) || key0 + kBK > kv ||
                             (a.window > 0 && (long long)key0 <= pos_max - a.window);
      tc::fence_after_sync();
#pragma unroll 1
      for (int c = 0; c < kBK / 32; ++c) {
        uint32_t sv[32], dv[32];
        tc::ld32(lane_addr + kColS + c * 32, sv);
        tc::ld32(lane_addr + kColDP + c * 32, dv);
        tc::wait_ld();
        uint32_t pd[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          float d2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = key0 + c * 32 + x + e;
            const float pr = fast_exp2(fmaf(__uint_as_float(sv[x + e]), a.sl2, -lse2));
            float ds = pr * (__uint_as_float(dv[x + e]) - dr);
            if (need_mask && !visible(key, pos, kv, a.causal, a.window)) ds = 0.f;
            d2[e] = ds;
          }
          pd[x / 2] = pack_bf16x2(d2[0], d2[1]);
        }
        tc::st16(lane_addr + kColS + c * 16, pd);  // dS (bf16 pairs) over S's first columns
      }
      // K rows that no row of the tile may see -- past kv_len (last block), below every row's
      // window (first block) -- get dS = 0 but may hold anything: zero them before dQ += dS K
      const bool zero_tail = j == nb - 1 && key0 + kBK > kv;
      const bool zero_head = j == 0 && a.window > 0 && (long long)key0 < pos_min - a.window + 1;
      if (zero_tail || zero_head) {
        const long long key = (long long)key0 + row;  // this thread's K row in the block
        if ((zero_tail && key >= kv) || (zero_head && key <= pos_min - a.window)) {
          for (int ch = 0; ch < C::kNch; ++ch)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t addr = sK(st) + ch * 128 * 128 + row * 128 + k * 16;
              asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
            }
        }
        tc::fence_proxy_async_smem();
      }
      tc::wait_st();
      tc::fence_before_sync();
      mbar_arrive(bar(kQP));
    }
    // ---- epilogue: scale * dQ -> bf16
    bool have = nb > 0 && ok;
    if (have) {
      have = wait_bar(bar(kQDone), 0, abort, a.err);
      have = __all_sync(0xffffffffu, have);
      if (have) tc::fence_after_sync();
    }
    uint4* out = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dq) + srow * D);
    if (have) {
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tc::ld32(lane_addr + kColAcc0 + c * 32, v);
        tc::wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * a.scale, __uint_as_float(v[2 * i + 1]) * a.scale);
        if (store_row) {
#pragma unroll
          for (int q = 0; q < 4; ++q) out[c * 4 + q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
    } else if (store_row) {
      for (int v = 0; v < D / 8; ++v) out[v] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}


template <int D>
cudaError_t launch_typed(const BArgs& p, const CUtensorMap* tm, cudaStream_t s) {
  static bool attr_set[64] = {false};  // per device: the shared-memory opt-ins are set once
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, KvCfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, QCfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const long long n1 = (long long)p.n_kb * p.B * p.h_kv;
  const long long n2 = (long long)p.n_qt * p.B * p.h_kv * p.hblocks;
  if (n1 > 0x7fffffffLL || n2 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dkdv_kernel<D><<<(unsigned)n1, kThreads, KvCfg<D>::kSmem, s>>>(tm[0], tm[1], tm[2], tm[3], p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dq_kernel<D><<<(unsigned)n2, kThreads, QCfg<D>::kSmem, s>>>(tm[4], tm[5], tm[2], tm[3], p);
  return cudaGetLastError();
}

}  // namespace bw

cudaError_t launch_backward_bf16(const BackwardArgs& a, const CUtensorMap* tmaps, cudaStream_t s) {
  const long long rows = (long long)a.B * a.h_q * a.S_q;
  if (rows <= 0) return cudaSuccess;
  bw::rowterm_kernel<__nv_bfloat16><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(a.o), reinterpret_cast<const __nv_bfloat16*>(a.d_o), a.lse,
      a.lse2, a.drow, rows, a.d_h);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bw::BArgs p;
  p.lse2 = a.lse2;
  p.drow = a.drow;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.q_start = a.q_start;
  p.kv_len = a.kv_len;
  p.B = a.B;
  p.h_q = a.h_q;
  p.h_kv = a.h_kv;
  p.r = a.h_q / a.h_kv;
  p.S_q = a.S_q;
  p.T_max = a.T_max;
  p.H = prefill_heads_per_tile(a.h_q, a.h_kv);
  p.P = 128 / p.H;
  p.hblocks = (p.r + p.H - 1) / p.H;
  p.n_qt = (a.S_q + p.P - 1) / p.P;
  p.n_kb = (a.T_max + bw::kBK - 1) / bw::kBK;
  p.scale = a.scale;
  p.sl2 = a.scale * bw::kLog2e;
  p.causal = a.causal;
  p.window = a.window;
  p.err = a.err;
  if (a.d_h == 128) return bw::launch_typed<128>(p, tmaps, s);
  if (a.d_h == 64) return bw::launch_typed<64>(p, tmaps, s);
  return cudaErrorInvalidValue;
}

}  // namespace gqa
