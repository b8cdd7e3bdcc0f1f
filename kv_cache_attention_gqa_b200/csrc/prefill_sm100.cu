// bf16 causal grouped-query attention prefill on sm_100a: TMA + tcgen05 (TMEM accumulators).
//
// What it computes: O_a = softmax(Q_a K_{g(a)}^T * scale + M) V_{g(a)} with g(a) = floor(a / r)
// [序列计算与存储, section 分组查询注意力], the causal/length mask by absolute position
// [第 09 章 GQA、MLA 与跨层 KV 共享, section 09.2], evaluated block by block with the online
// softmax state (m, l, u) so the score matrix never reaches memory [序列计算与存储, sections
// 分块注意力 and 在线 softmax].
//
// Work tile. Rows of one tile are (query position, query head) pairs of ONE KV group: H heads
// (H = min(r, 128)) times P = floor(128 / H) consecutive positions, head-major, so every K/V block
// staged in shared memory serves all r heads of the group [MHA/MQA/GQA walkthrough, section 7:
// e.g. 32 positions x 4 heads = 128 rows; the mask still uses each row's own position]. A CTA owns
// two such 128-row sub-tiles (positions q0 .. q0 + 2P) that share every K/V block.
//
// Roles (384 threads):
//   warp 0      TMA producer: the two Q sub-tiles once, then 128-key K and V blocks into a 2-stage
//               ring (cp.async.bulk.tensor, 128-byte swizzle, no multicast).
//   warp 1      allocates 512 TMEM columns and issues the MMAs from one thread:
//               S_t = Q_t K_j^T  (tcgen05.mma kind::f16, A and B from shared memory, K-major),
//               O_t += P_t V_j   (A = P from TMEM, B = V from shared memory, MN-major),
//               ping-ponging the two sub-tiles so one sub-tile's softmax overlaps the other's MMAs.
//   warps 4-7   softmax of sub-tile 0, warps 8-11 of sub-tile 1: one thread per row (TMEM lane).
//               Each reads its score row from TMEM, masks by absolute position, updates (m, l),
//               writes P = 2^(s - m) as bf16 back into the same TMEM columns, and rescales its O
//               row only when the running maximum grew by more than 8 (base 2): between rescales
//               P and l share the stale maximum, which leaves O = u / l unchanged.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256, 256+D), O1 [256+D, 256+2D); P_t aliases the
// first 64 columns of S_t. MMAs issued by one thread execute in order, so S_t of block j+1 is
// written only after O_t += P_t V_j has read P_t.

#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace gqa {
namespace pf {

constexpr int kBM = 128;     // rows per sub-tile (= TMEM lanes)
constexpr int kBN = 128;     // keys per K/V block
constexpr int kStages = 2;   // K/V ring depth
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // base-2 units: P <= 2^8 between rescales
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int kNch = D / 64;                  // 64-column (128-byte) chunks
  static constexpr int kQChunk = kBM * 128;            // bytes of one Q chunk (128 rows)
  static constexpr int kQBytes = kNch * kQChunk;       // one sub-tile of Q
  static constexpr int kKVChunk = kBN * 128;
  static constexpr int kKVBytes = kNch * kKVChunk;     // one K (or V) block
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kStages * kKVBytes;
  // barriers + slack for 1024-byte alignment; at least 120 KiB so that only one CTA (which
  // allocates all 512 TMEM columns) is resident per SM
  static constexpr int kSmem = kOffBar + 256 + 1024 > 120 * 1024 ? kOffBar + 256 + 1024 : 120 * 1024;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
};

struct PArgs {
  void* o;
  float* lse;
  const int32_t* q_start;
  const int32_t* kv_len;
  int B, h_q, h_kv, r, S_q, T_max;
  int H, P, hblocks, n_qt;
  float scale_log2;
  int causal;
  unsigned* err;
};

// barrier indices inside the barrier block
enum {
  kBarQ = 0,
  kBarKFull = 1,    // + stage
  kBarVFull = 3,    // + stage
  kBarKVEmpty = 5,  // + stage
  kBarS = 7,        // + sub-tile
  kBarP = 9,        // + sub-tile
  kBarO = 11,       // + sub-tile
  kBarDone = 13,
  kNumBars = 14
};

// Bounded wait that also gives up as soon as another thread of the CTA has aborted.
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

struct Tile {
  int b, g, hb, q0;  // q0: first query position (index into S_q) of sub-tile 0
  int nh;            // heads of this head block
  int qs, kv;        // q_start[b], kv_len[b]
  int nb;            // K/V blocks to visit
  bool valid;
};

__device__ __forceinline__ Tile make_tile(const PArgs& a) {
  Tile t;
  const int per = a.B * a.h_kv * a.hblocks;
  const int w = blockIdx.x;
  const int qt = a.n_qt - 1 - w / per;  // heaviest (latest positions) first
  const int rem = w - (w / per) * per;
  t.b = rem / (a.h_kv * a.hblocks);
  const int gh = rem - t.b * (a.h_kv * a.hblocks);
  t.g = gh / a.hblocks;
  t.hb = gh - t.g * a.hblocks;
  t.q0 = qt * 2 * a.P;
  t.nh = min(a.H, a.r - t.hb * a.H);
  t.kv = a.kv_len ? a.kv_len[t.b] : a.T_max;
  t.qs = a.q_start ? a.q_start[t.b] : 0;
  t.valid = t.kv >= 1 && t.kv <= a.T_max && t.qs >= 0;
  t.nb = 0;
  if (t.valid) {
    if (a.causal) {
      const int last_row = min(t.q0 + 2 * a.P, a.S_q) - 1;
      const long long pos_max = (long long)t.qs + last_row;
      const long long last_key = pos_max < t.kv - 1 ? pos_max : (long long)(t.kv - 1);
      t.nb = (int)(last_key / kBN) + 1;
    } else {
      t.nb = (t.kv + kBN - 1) / kBN;
    }
  }
  return t;
}

// One thread per row of sub-tile t (warps 4-7: t = 0, warps 8-11: t = 1).
template <int D>
__device__ __forceinline__ void softmax_role(const PArgs& a, const Tile& tile, int warp, int lane,
                                             uint32_t tmem, uint32_t sV, uint64_t* bars,
                                             volatile int* abort) {
  using C = Cfg<D>;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int t = (warp - 4) >> 2;
  const int wq = warp & 3;                   // TMEM lane quarter this warp may access
  const int row = wq * 32 + lane;            // TMEM lane = tile row
  const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
  const uint32_t colS = t == 0 ? C::kColS0 : C::kColS1;
  const uint32_t colO = t == 0 ? C::kColO0 : C::kColO1;
  const int h = row / a.P, p = row - h * a.P;
  const int qi = tile.q0 + t * a.P + p;      // query index into S_q
  const bool store_row = h < tile.nh && row < a.H * a.P && qi < a.S_q;
  const long long pos = (long long)tile.qs + qi;
  const long long pos_min = (long long)tile.qs + tile.q0 + t * a.P;  // smallest position in t
  const int nb = tile.nb;

  float m = -INFINITY, l = 0.f;
  bool ok = true;
  for (int j = 0; j < nb && ok; ++j) {
    if (!wait_bar(bar(kBarS + t), (uint32_t)(j & 1), abort, a.err)) { ok = false; break; }
    tc::fence_after_sync();
    uint32_t sr[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tc::ld32(lane_addr + colS + c * 32, sr[c]);
    tc::wait_ld();
    const int key0 = j * kBN;
    const bool need_mask =
        (a.causal && (long long)key0 + kBN - 1 > pos_min) || key0 + kBN > tile.kv;
    float mx = -INFINITY;
    if (need_mask) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int key = key0 + c * 32 + i;
          const bool vis = key < tile.kv && (!a.causal || key <= pos);
          const float x = vis ? __uint_as_float(sr[c][i]) * a.scale_log2 : -INFINITY;
          sr[c][i] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = __uint_as_float(sr[c][i]) * a.scale_log2;
          sr[c][i] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
    }
    // running maximum with lazy rescaling
    const float m_new = fmaxf(m, mx);
    float m_use = m, alpha = 1.f;
    bool rescale_o = false;
    if (m == -INFINITY) {
      m_use = m_new;  // first block with a visible key: nothing accumulated yet
    } else if (m_new > m + kRescaleThreshold) {
      m_use = m_new;
      alpha = fast_exp2(m - m_new);
      rescale_o = true;
    }
    // P = 2^(x - m_use) as bf16 pairs into the first 64 columns of S_t; row sum in fp32
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float p0 = fast_exp2(__uint_as_float(sr[c][2 * i]) - m_use);
        const float p1 = fast_exp2(__uint_as_float(sr[c][2 * i + 1]) - m_use);
        sum += p0 + p1;
        pk[i] = pack_bf16x2(p0, p1);
      }
      tc::st16(lane_addr + colS + c * 16, pk);
    }
    l = l * alpha + sum;
    m = m_use;
    if (rescale_o) {
      // O_t must hold the result of every earlier block before it is rescaled
      if (!wait_bar(bar(kBarO + t), (uint32_t)((j - 1) & 1), abort, a.err)) { ok = false; }
      if (ok) {
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tc::ld32(lane_addr + colO + c * 32, o);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tc::st32(lane_addr + colO + c * 32, o);
        }
      }
    }
    tc::wait_st();
    if (t == 0 && j == nb - 1 && key0 + kBN > tile.kv) {
      // V rows at or past kv_len get weight 0 but may hold anything (NaN included): zero them in
      // shared memory so 0 * V stays 0. The block's V must have landed first.
      const int s = j & 1;
      if (wait_bar(bar(kBarVFull + s), (uint32_t)((j >> 1) & 1), abort, a.err)) {
        const int first_bad = tile.kv - key0;
        if (row >= first_bad) {
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int ch = 0; ch < C::kNch; ++ch)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t addr = sV + s * C::kKVBytes + ch * C::kKVChunk + row * 128 + i * 16;
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(z.x),
                           "r"(z.y), "r"(z.z), "r"(z.w)
                           : "memory");
            }
        }
        tc::fence_proxy_async_smem();
      } else {
        ok = false;
      }
    }
    tc::fence_before_sync();
    mbar_arrive(bar(kBarP + t));
  }
  if (!ok || nb == 0) {
    if (nb == 0 && store_row) {  // invalid request: zero row
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.o) +
                           (((long long)tile.b * a.h_q + tile.g * a.r + tile.hb * a.H + h) * a.S_q + qi) * D;
      for (int c = 0; c < D; ++c) out[c] = __float2bfloat16_rn(0.f);
      if (a.lse) a.lse[((long long)tile.b * a.h_q + tile.g * a.r + tile.hb * a.H + h) * a.S_q + qi] = -INFINITY;
    }
    return;
  }
  // epilogue: O / l -> bf16 -> global; lse = (m + log2 l) * ln 2
  if (!wait_bar(bar(kBarO + t), (uint32_t)((nb - 1) & 1), abort, a.err)) return;
  tc::fence_after_sync();
  const float inv = 1.f / l;
  const long long orow = ((long long)tile.b * a.h_q + tile.g * a.r + tile.hb * a.H + h) * a.S_q + qi;
  uint4* out = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + orow * D);
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tc::ld32(lane_addr + colO + c * 32, o);
    tc::wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
    if (store_row) {
#pragma unroll
      for (int v = 0; v < 4; ++v)
        out[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    }
  }
  if (store_row && a.lse) a.lse[orow] = (m + __log2f(l)) * kLn2;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_bf16_kernel(const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, PArgs a) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Tile tile = make_tile(a);

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarKVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(kBarS + t), 1);
      mbar_init(bar(kBarP + t), 128);
      mbar_init(bar(kBarO + t), 1);
    }
    mbar_init(bar(kBarDone), 1);
    *abort = 0;
    fence_barrier_init();
    if (!tile.valid) set_device_error(a.err, tile.kv < 1 || tile.kv > a.T_max ? GQA_DEVERR_KV_LEN
                                                                               : GQA_DEVERR_POSITION);
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int nb = tile.nb;

  if (warp == 0 && lane == 0 && nb > 0) {
    // ------------------------------ TMA producer ------------------------------------------
    tma_prefetch_desc(&tmq);
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
    const int zq = tile.b * a.h_q + tile.g * a.r + tile.hb * a.H;  // first head of the block
    const uint32_t qbytes = (uint32_t)(C::kNch * a.H * a.P * 128);
    mbar_arrive_expect_tx(bar(kBarQ), 2 * qbytes);
    for (int t = 0; t < 2; ++t)
      for (int ch = 0; ch < C::kNch; ++ch)
        tma_load_3d(sQ + t * C::kQBytes + ch * C::kQChunk, &tmq, bar(kBarQ), ch * 64,
                    tile.q0 + t * a.P, zq);
    const int row0 = (tile.b * a.h_kv + tile.g) * a.T_max;
    int last_fill[kStages] = {-1, -1};
    bool ok = true;
    for (int j = 0; j < nb && ok; ++j) {
      const int s = j & 1, n = j >> 1;
      if (n > 0 && !wait_bar(bar(kBarKVEmpty + s), (uint32_t)((n - 1) & 1), abort, a.err)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(bar(kBarKFull + s), C::kKVBytes);
      for (int ch = 0; ch < C::kNch; ++ch)
        tma_load_2d(sK + s * C::kKVBytes + ch * C::kKVChunk, &tmk, bar(kBarKFull + s), ch * 64,
                    row0 + j * kBN);
      mbar_arrive_expect_tx(bar(kBarVFull + s), C::kKVBytes);
      for (int ch = 0; ch < C::kNch; ++ch)
        tma_load_2d(sV + s * C::kKVBytes + ch * C::kKVChunk, &tmv, bar(kBarVFull + s), ch * 64,
                    row0 + j * kBN);
      last_fill[s] = n;
    }
    // Drain (bounded, whatever the abort state): no copy may still be landing in shared memory
    // when the CTA exits.
    volatile int no_abort = 0;
    wait_bar(bar(kBarQ), 0, &no_abort, a.err);
    for (int s = 0; s < kStages; ++s) {
      if (last_fill[s] < 0) continue;
      wait_bar(bar(kBarKFull + s), (uint32_t)(last_fill[s] & 1), &no_abort, a.err);
      wait_bar(bar(kBarVFull + s), (uint32_t)(last_fill[s] & 1), &no_abort, a.err);
    }
  } else if (warp == 1 && lane == 0 && nb > 0) {
    // ------------------------------ MMA issuer ---------------------------------------------
    constexpr uint32_t idesc_qk = tc::idesc_bf16(kBM, kBN, false);
    constexpr uint32_t idesc_pv = tc::idesc_bf16(kBM, D, true);
    const uint32_t colS[2] = {C::kColS0, C::kColS1};
    const uint32_t colO[2] = {C::kColO0, C::kColO1};
    auto qk = [&](int t, int s) {  // S_t = Q_t K_s^T, K-major operands, 16 columns per MMA
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (uint32_t)((ks >> 2) * C::kQChunk + (ks & 3) * 32);
        const uint32_t koff = (uint32_t)((ks >> 2) * C::kKVChunk + (ks & 3) * 32);
        const uint64_t ad = tc::smem_desc(sQ + t * C::kQBytes + off, 16, 1024);
        const uint64_t bd = tc::smem_desc(sK + s * C::kKVBytes + koff, 16, 1024);
        tc::mma_ss(tmem + colS[t], ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
      }
    };
    auto pv = [&](int t, int s, bool acc) {  // O_t += P_t V_s; P in TMEM (8 columns per 16 keys)
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk) {
        const uint64_t bd = tc::smem_desc(sV + s * C::kKVBytes + kk * 2048, C::kKVChunk, 1024);
        tc::mma_ts(tmem + colO[t], tmem + colS[t] + kk * 8, bd, idesc_pv,
                   (acc || kk > 0) ? 1u : 0u);
      }
    };
    bool ok = wait_bar(bar(kBarQ), 0, abort, a.err);
    if (ok) ok = wait_bar(bar(kBarKFull + 0), 0, abort, a.err);
    if (ok) {
      tc::fence_after_sync();
      qk(0, 0);
      tc::commit(bar(kBarS + 0));
      qk(1, 0);
      tc::commit(bar(kBarS + 1));
    }
    for (int j = 0; j < nb && ok; ++j) {
      const int s = j & 1;
      const uint32_t ph = (uint32_t)((j >> 1) & 1);
      const int s1 = (j + 1) & 1;
      const uint32_t ph1 = (uint32_t)(((j + 1) >> 1) & 1);
      if (!wait_bar(bar(kBarVFull + s), ph, abort, a.err)) break;
      // sub-tile 0
      if (!wait_bar(bar(kBarP + 0), (uint32_t)(j & 1), abort, a.err)) break;
      tc::fence_after_sync();
      pv(0, s, j > 0);
      tc::commit(bar(kBarO + 0));
      if (j + 1 < nb) {
        if (!wait_bar(bar(kBarKFull + s1), ph1, abort, a.err)) break;
        tc::fence_after_sync();
        qk(0, s1);
        tc::commit(bar(kBarS + 0));
      }
      // sub-tile 1
      if (!wait_bar(bar(kBarP + 1), (uint32_t)(j & 1), abort, a.err)) break;
      tc::fence_after_sync();
      pv(1, s, j > 0);
      tc::commit(bar(kBarO + 1));
      tc::commit(bar(kBarKVEmpty + s));  // K_j and V_j are no longer read
      if (j + 1 < nb) {
        qk(1, s1);
        tc::commit(bar(kBarS + 1));
      }
    }
    // every MMA issued above has completed before TMEM is released
    tc::commit(bar(kBarDone));
    volatile int no_abort = 0;
    wait_bar(bar(kBarDone), 0, &no_abort, a.err);
  } else if (warp >= 4) {
    softmax_role<D>(a, tile, warp, lane, tmem, sV, bars, abort);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pf

cudaError_t launch_prefill_bf16(const PrefillArgs& a, const CUtensorMap* tmaps, int num_sms,
                                cudaStream_t s) {
  (void)num_sms;
  pf::PArgs p;
  p.o = a.o;
  p.lse = a.lse;
  p.q_start = a.q_start;
  p.kv_len = a.kv_len;
  p.B = a.B;
  p.h_q = a.h_q;
  p.h_kv = a.h_kv;
  p.r = a.h_q / a.h_kv;
  p.S_q = a.S_q;
  p.T_max = a.T_max;
  p.H = prefill_heads_per_tile(a.h_q, a.h_kv);
  p.P = pf::kBM / p.H;
  p.hblocks = (p.r + p.H - 1) / p.H;
  p.n_qt = (a.S_q + 2 * p.P - 1) / (2 * p.P);
  p.scale_log2 = a.scale * pf::kLog2e;
  p.causal = a.causal;
  p.err = a.err;
  const long long tiles = (long long)p.n_qt * a.B * a.h_kv * p.hblocks;
  if (tiles <= 0) return cudaSuccess;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  cudaError_t e;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool set128[64] = {false}, set64[64] = {false};
  if (a.d_h == 128) {
    if (dev < 0 || dev >= 64 || !set128[dev]) {
      e = cudaFuncSetAttribute(pf::prefill_bf16_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               pf::Cfg<128>::kSmem);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) set128[dev] = true;
    }
    pf::prefill_bf16_kernel<128><<<(unsigned)tiles, pf::kThreads, pf::Cfg<128>::kSmem, s>>>(
        tmaps[0], tmaps[1], tmaps[2], p);
  } else if (a.d_h == 64) {
    if (dev < 0 || dev >= 64 || !set64[dev]) {
      e = cudaFuncSetAttribute(pf::prefill_bf16_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               pf::Cfg<64>::kSmem);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) set64[dev] = true;
    }
    pf::prefill_bf16_kernel<64><<<(unsigned)tiles, pf::kThreads, pf::Cfg<64>::kSmem, s>>>(
        tmaps[0], tmaps[1], tmaps[2], p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

int prefill_heads_per_tile(int h_q, int h_kv) {
  const int r = h_q / h_kv;
  return r < pf::kBM ? r : pf::kBM;
}

}  // namespace gqa
