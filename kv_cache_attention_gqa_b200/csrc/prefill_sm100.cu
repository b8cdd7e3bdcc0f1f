// bf16 causal grouped-query attention prefill on sm_100a: TMA + tcgen05 (TMEM accumulators).
//
// What it computes: O_a = softmax(Q_a K_{g(a)}^T * scale + M) V_{g(a)} with g(a) = floor(a / r)
// [序列计算与存储, section 分组查询注意力], the causal/length mask by absolute position
// [第 09 章 GQA、MLA 与跨层 KV 共享, section 09.2], evaluated block by block with the online
// softmax state (m, l, u) so the score matrix never reaches memory [序列计算与存储, sections
// 分块注意力 and 在线 softmax]. An optional sliding window W limits row p to keys p - W < j <= p
// [第三章：MHA 的局限与 MQA、GQA、Flash Attention, section 3.7]: K/V blocks below the tile's
// earliest window are never loaded, and the boundary blocks are masked per row.
//
// Work tile. Rows of one tile are (query position, query head) pairs of ONE KV group: H heads
// (H = min(r, 128)) times P = floor(128 / H) consecutive positions, head-major, so every K/V block
// staged in shared memory serves all r heads of the group [MHA/MQA/GQA walkthrough, section 7:
// e.g. 32 positions x 4 heads = 128 rows; the mask still uses each row's own position].
//
// Roles (384 threads, one 128-row tile per CTA):
//   warp 0      TMA producer: the tile's Q rows once, then 128-key K blocks into a 3-deep ring and
//               V blocks into a 2-deep ring (cp.async.bulk.tensor, 128-byte swizzle, no multicast).
//   warp 1      allocates 512 TMEM columns and issues every MMA from one thread:
//               S_j = Q K_j^T  (tcgen05.mma kind::f16, A = Q from TMEM, B = K from shared memory),
//               O  += P_j V_j  (A = P_j from TMEM, B = V from shared memory, MN-major).
//               S is double-buffered: S_{j+2} is issued right after O += P_j V_j, so the scores of
//               the next block are ready when the softmax finishes the current one. Both MMAs read
//               only one operand from shared memory (a 128x128x16 MMA with both operands there
//               would need the whole shared-memory bandwidth).
//   warps 4-11  softmax: two warpgroups serve the same 128 rows (one row per TMEM lane), each
//               taking 64 of every block's 128 score columns. First each copies its 64-column
//               chunk of the Q rows from shared memory into TMEM. Per block each thread reads its
//               half row and masks it by absolute position (one clamped 32-bit bound per row);
//               the two halves meet at a named barrier to share the block's row maximum. Each
//               half then writes
//               P = 2^(s - m) as bf16 into its share of the block's first 64 S columns and
//               rescales its half of the O row only when the running maximum grew by more than 8
//               (base 2): between rescales P and l share the stale maximum, which leaves
//               O = u / l unchanged. The row sums meet once, at the end.
// TMEM columns: S_0 [0,128), S_1 [128,256), O [256, 256+D), Q [256+D, 256+3D/2); P_b aliases the
// first 64 columns of S_b. MMAs issued by one thread execute in order, so S_b of block j+2 is
// written only after O += P_j V_j has read P_j.

#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace gqa {
namespace pf {

constexpr int kBM = 128;     // rows per tile (= TMEM lanes)
constexpr int kBN = 128;     // keys per K/V block
constexpr int kKStages = 3;  // K ring depth (K_j is read two blocks before V_j)
constexpr int kVStages = 2;  // V ring depth
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // base-2 units: P <= 2^8 between rescales
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int kNch = D / 64;                  // 64-column (128-byte) chunks
  static constexpr int kQChunk = kBM * 128;            // bytes of one Q chunk (128 rows)
  static constexpr int kQBytes = kNch * kQChunk;
  static constexpr int kKVChunk = kBN * 128;
  static constexpr int kKVBytes = kNch * kKVChunk;     // one K (or V) block
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffX = kOffV + kVStages * kKVBytes;  // 6 x 128 floats
  static constexpr int kOffBar = kOffX + 6 * 128 * 4;
  // barriers + slack for 1024-byte alignment; at least 120 KiB so that only one CTA (which
  // allocates all 512 TMEM columns) is resident per SM
  static constexpr int kSmem = kOffBar + 256 + 1024 > 120 * 1024 ? kOffBar + 256 + 1024 : 120 * 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColQ = 256 + D;
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
  int window;  // 0: none; W > 0: row at position p also needs key j > p - W (causal only)
  int expire_wait;  // test hook: CTA 0's producer first waits on a barrier that nothing signals
  unsigned* err;
};

// barrier indices inside the barrier block
enum {
  kBarQ = 0,          // Q rows landed in shared memory (TMA)
  kBarQT = 1,         // Q rows copied into TMEM (128 softmax threads)
  kBarKFull = 2,      // + K stage (3)
  kBarKEmpty = 5,     // + K stage
  kBarVFull = 8,      // + V stage (3)
  kBarVEmpty = 11,    // + V stage
  kBarS = 14,         // + S buffer (2): scores of a block are in TMEM
  kBarP = 16,         // + S buffer (2): P of a block is in TMEM
  kBarO = 18,         // O += P V of a block completed
  kBarDone = 19,
  kBarNever = 20,     // never signalled: the test hook's wait on it always runs out
  kNumBars = 21
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
  int b, g, hb, q0;  // q0: first query position (index into S_q) of the tile
  int nh;            // heads of this head block
  int qs, kv;        // q_start[b], kv_len[b]
  int j0;            // first K/V block visited (> 0 only under a sliding window)
  int nb;            // K/V blocks to visit: j0 .. j0 + nb - 1
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
  t.q0 = qt * a.P;
  t.nh = min(a.H, a.r - t.hb * a.H);
  t.kv = a.kv_len ? a.kv_len[t.b] : a.T_max;
  t.qs = a.q_start ? a.q_start[t.b] : 0;
  t.valid = t.kv >= 1 && t.kv <= a.T_max && t.qs >= 0;
  t.nb = 0;
  t.j0 = 0;
  if (t.valid) {
    if (a.causal) {
      const int last_row = min(t.q0 + a.P, a.S_q) - 1;
      const long long pos_max = (long long)t.qs + last_row;
      const long long last_key = pos_max < t.kv - 1 ? pos_max : (long long)(t.kv - 1);
      const int end = (int)(last_key / kBN) + 1;
      if (a.window > 0) {
        // blocks wholly below the earliest row's window are skipped [第三章 §3.7: each query
        // reads only its local window]
        const long long lo = (long long)t.qs + t.q0 - a.window + 1;
        if (lo > 0) t.j0 = (int)(lo / kBN);
      }
      t.nb = end > t.j0 ? end - t.j0 : 0;
    } else {
      t.nb = (t.kv + kBN - 1) / kBN;
    }
  }
  return t;
}

// packed fp32x2 helpers (sm_100): d = a * b + c and s += a, on register pairs
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
      "mov.b64 rc, {%5, %5};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
__device__ __forceinline__ void fadd2(float& s0, float& s1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rs;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rs, {%0, %1};\n\t"
      "add.rn.f32x2 rs, rs, ra;\n\tmov.b64 {%0, %1}, rs;\n\t}"
      : "+f"(s0), "+f"(s1)
      : "f"(a0), "f"(a1));
}

// Two warpgroups share the tile's rows: warps 4-7 take the first half of every block's columns
// (keys 0-63) and warps 8-11 the second half (keys 64-127), so each SM sub-partition runs two
// independent softmax warps. A thread owns one row (its TMEM lane, warp % 4 selects the lane
// quarter) and half of the row's columns; the two halves of a row exchange their block maximum
// through shared memory once per block, and their partial sums at the end.
// kWin: the launch has a sliding window (a.window > 0). Without one, the window code is compiled
// out (its per-element compare in the mask loop costs ~9% of the causal kernel's time).
template <int D, bool kWin>
__device__ __forceinline__ void softmax_role(const PArgs& a, const Tile& tile, int warp, int lane,
                                             uint32_t tmem, uint32_t sQ, uint32_t sV, uint64_t* bars,
                                             float* xbuf, volatile int* abort) {
  using C = Cfg<D>;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int half = (warp - 4) >> 2;           // which 64 columns of each block
  const int wq = warp & 3;
  const int row = wq * 32 + lane;             // TMEM lane = tile row
  const int sm_tid = (warp - 4) * 32 + lane;  // 0..255
  const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
  const int h = row / a.P, p = row - h * a.P;
  const int qi = tile.q0 + p;                 // query index into S_q
  const bool store_row = h < tile.nh && row < a.H * a.P && qi < a.S_q;
  const long long pos = (long long)tile.qs + qi;
  // last key this row may see (length and causal limits in one 32-bit bound for the mask loop)
  const long long kl = a.causal && pos < tile.kv - 1 ? pos : (long long)tile.kv - 1;
  const int key_last = (int)kl;
  const long long pos_min = (long long)tile.qs + tile.q0;  // smallest position in the tile
  const long long pos_max = (long long)tile.qs + min(tile.q0 + a.P, a.S_q) - 1;  // largest
  const int nb = tile.nb;
  const float c = a.scale_log2;
  const int win = kWin ? a.window : 0;
  // last key below this row's window, clamped to the int range (keys are ints)
  const long long wl = pos - win;
  const int win_last = kWin ? (int)(wl < -1 ? -1 : (wl > 0x7fffffffLL ? 0x7fffffffLL : wl)) : -1;
  const long long orow = ((long long)tile.b * a.h_q + tile.g * a.r + tile.hb * a.H + h) * a.S_q + qi;
  constexpr int kOHalf = D / 2;               // O columns (and Q columns) of this half
  float* xmax = xbuf;                         // [2 buffers][2 halves][128 rows]

  // ---- this half of this row of Q: shared memory (128-byte swizzled) -> TMEM (A of Q K^T)
  // tcgen05.ld / st / wait are .sync.aligned: every lane of a warp must execute each of them, so
  // every condition in front of one is made warp-uniform (__all_sync / __any_sync) first.
  bool ok = nb > 0 && wait_bar(bar(kBarQ), 0, abort, a.err);
  ok = __all_sync(0xffffffffu, ok);
  if (ok) {
#pragma unroll
    for (int ch = 0; ch < C::kNch; ++ch) {
      if ((C::kNch == 2 && ch != half) || (C::kNch == 1 && half != 0)) continue;
      uint32_t qr[32];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t addr = swz128(sQ + ch * C::kQChunk, row, k);
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(qr[4 * k]), "=r"(qr[4 * k + 1]), "=r"(qr[4 * k + 2]), "=r"(qr[4 * k + 3])
                     : "r"(addr));
      }
      tc::st32(lane_addr + C::kColQ + ch * 32, qr);
    }
    tc::wait_st();
  }
  tc::fence_before_sync();
  mbar_arrive(bar(kBarQT));

  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < nb; ++j) {
    const int buf = j & 1;
    const uint32_t colS = buf ? C::kColS1 : C::kColS0;
    // After a failed wait the loop keeps running (without touching TMEM or other barriers) so
    // that every softmax thread takes the per-block named barrier the same number of times.
    if (ok) ok = wait_bar(bar(kBarS + buf), (uint32_t)((j >> 1) & 1), abort, a.err);
    ok = __all_sync(0xffffffffu, ok);
    float sr[64];
    float lmx = 0.f;
    const int key0 = (tile.j0 + j) * kBN + half * 64;  // first key of this half
    const bool need_mask = (a.causal && (long long)key0 + 63 > pos_min) || key0 + 64 > tile.kv ||
                           (kWin && (long long)key0 <= pos_max - win);
    if (ok) {
      tc::fence_after_sync();
      uint32_t su[2][32];
      tc::ld32(lane_addr + colS + half * 64, su[0]);
      tc::ld32(lane_addr + colS + half * 64 + 32, su[1]);
      tc::wait_ld();
#pragma unroll
      for (int i = 0; i < 64; ++i) sr[i] = __uint_as_float(su[i >> 5][i & 31]);
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int key = key0 + i;
          const bool vis = key <= key_last && (!kWin || key > win_last);
          sr[i] = vis ? sr[i] : -INFINITY;
        }
      }
      float mx0 = sr[0], mx1 = sr[1];
#pragma unroll
      for (int i = 2; i < 64; i += 2) {
        mx0 = fmaxf(mx0, sr[i]);
        mx1 = fmaxf(mx1, sr[i + 1]);
      }
      lmx = fmaxf(mx0, mx1);
    }
    // block maximum over both halves of the row (double-buffered exchange slot per S buffer)
    xmax[(buf * 2 + half) * 128 + row] = lmx;
    named_barrier_sync(1, 256);
    if (!ok) continue;
    const float mx = fmaxf(xmax[(buf * 2 + half) * 128 + row], xmax[(buf * 2 + (half ^ 1)) * 128 + row]) * c;
    // running maximum with lazy rescaling (both halves take the same decision)
    const float m_new = fmaxf(m, mx);
    float m_use = m, alpha = 1.f;
    bool rescale_o = false;
    if (m == -INFINITY) {
      m_use = m_new;  // first block: nothing accumulated yet
    } else if (m_new > m + kRescaleThreshold) {
      m_use = m_new;
      alpha = fast_exp2(m - m_new);
      rescale_o = true;
    }
    // P = 2^(s c - m_use) as bf16 pairs: this half's keys go to 32 of the first 64 S columns.
    // A row that has seen no visible key yet (only possible under a sliding window) keeps
    // m = -inf; its P is 0, computed against 0 instead of -inf.
    const float m_sub = kWin && m_use == -INFINITY ? 0.f : m_use;
    float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float x0, x1;
        ffma2(x0, x1, sr[cc * 32 + 2 * i], sr[cc * 32 + 2 * i + 1], c, -m_sub);
        const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
        fadd2(sum0, sum1, p0, p1);
        pk[i] = pack_bf16x2(p0, p1);
      }
      tc::st16(lane_addr + colS + half * 32 + cc * 16, pk);
    }
    l = l * alpha + (sum0 + sum1);
    m = m_use;
    // the warp rescales its O rows together when any of its rows needs it (rows that do not
    // need it multiply by alpha = 1)
    if (__any_sync(0xffffffffu, rescale_o && j > 0)) {
      // O must hold every earlier block's contribution before it is rescaled
      if (!wait_bar(bar(kBarO), (uint32_t)((j - 1) & 1), abort, a.err)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc::fence_after_sync();
#pragma unroll
        for (int cc = 0; cc < kOHalf / 32; ++cc) {
          uint32_t o[32];
          tc::ld32(lane_addr + C::kColO + half * kOHalf + cc * 32, o);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tc::st32(lane_addr + C::kColO + half * kOHalf + cc * 32, o);
        }
      }
    }
    tc::wait_st();
    const int bkey0 = (tile.j0 + j) * kBN;
    // V rows at or past kv_len, and (sliding window) rows below the earliest row's window, get
    // weight 0 for every row of the tile but may hold anything (NaN included): zero them in shared
    // memory so 0 * V stays 0 (each half zeroes its own 64-column chunk). The block's V must have
    // landed first.
    const bool zero_tail = j == nb - 1 && bkey0 + kBN > tile.kv;
    const bool zero_head = kWin && j == 0 && (long long)bkey0 < pos_min - win + 1;
    if (ok && (zero_tail || zero_head) && (C::kNch == 2 || half == 0)) {
      const int vs = j % kVStages;
      if (wait_bar(bar(kBarVFull + vs), (uint32_t)((j / kVStages) & 1), abort, a.err)) {
        const long long key = (long long)bkey0 + row;
        if ((zero_tail && key >= tile.kv) || (zero_head && key <= pos_min - win)) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t addr = sV + vs * C::kKVBytes + (C::kNch == 2 ? half : 0) * C::kKVChunk + row * 128 + k * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
          }
        }
        tc::fence_proxy_async_smem();
      } else {
        ok = false;
      }
    }
    tc::fence_before_sync();
    mbar_arrive(bar(kBarP + buf));
  }
  if (nb == 0) {  // invalid request: zero row
    if (store_row) {
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.o) + orow * D;
      for (int cc = half * kOHalf; cc < (half + 1) * kOHalf; ++cc) out[cc] = __float2bfloat16_rn(0.f);
      if (a.lse && half == 0) a.lse[orow] = -INFINITY;
    }
    return;
  }
  // row sum over both halves (every softmax thread reaches this barrier, aborted or not)
  float* xsum = xbuf + 4 * 128;
  xsum[half * 128 + row] = l;
  named_barrier_sync(1, 256);
  l += xsum[(half ^ 1) * 128 + row];
  (void)sm_tid;
  // A tile whose pipeline gave up (a bounded wait ran out; the error word says so) writes zero
  // rows and lse = -inf, without touching TMEM.
  auto zero_rows = [&]() {
    if (!store_row) return;
    uint4* z = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + orow * D + half * kOHalf);
#pragma unroll
    for (int v = 0; v < kOHalf / 8; ++v) z[v] = make_uint4(0u, 0u, 0u, 0u);
    if (a.lse && half == 0) a.lse[orow] = -INFINITY;
  };
  if (!__all_sync(0xffffffffu, ok)) {
    zero_rows();
    return;
  }
  // epilogue: this half of O / l -> bf16 -> global; lse = (m + log2 l) * ln 2
  bool ok_o = wait_bar(bar(kBarO), (uint32_t)((nb - 1) & 1), abort, a.err);
  if (!__all_sync(0xffffffffu, ok_o)) {
    zero_rows();
    return;
  }
  tc::fence_after_sync();
  // A row with no visible key (a sliding window that starts at or past kv_len, or a padding row
  // of the tile) has l = 0: it still takes part in the warp's TMEM loads, and writes zeros.
  const bool empty = kWin && l == 0.f;
  if (empty && store_row && half == 0) set_device_error(a.err, GQA_DEVERR_NO_VISIBLE);
  const float inv = empty ? 0.f : 1.f / l;
  uint4* out = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + orow * D + half * kOHalf);
#pragma unroll
  for (int cc = 0; cc < kOHalf / 32; ++cc) {
    uint32_t o[32];
    tc::ld32(lane_addr + C::kColO + half * kOHalf + cc * 32, o);
    tc::wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = empty ? 0u : pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
    if (store_row) {
#pragma unroll
      for (int v = 0; v < 4; ++v)
        out[cc * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    }
  }
  if (store_row && a.lse && half == 0) a.lse[orow] = empty ? -INFINITY : (m + __log2f(l)) * kLn2;
}

template <int D, bool kWin>
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
  float* xbuf = reinterpret_cast<float*>(smem + C::kOffX);  // softmax max/sum exchange
  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Tile tile = make_tile(a);

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    mbar_init(bar(kBarQT), 256);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kBarS + b), 1);
      mbar_init(bar(kBarP + b), 256);
    }
    mbar_init(bar(kBarO), 1);
    mbar_init(bar(kBarDone), 1);
    mbar_init(bar(kBarNever), 1);
    *abort = 0;
    fence_barrier_init();
    if (!tile.valid) set_device_error(a.err, tile.kv < 1 || tile.kv > a.T_max ? GQA_DEVERR_KV_LEN
                                                                               : GQA_DEVERR_POSITION);
    else if (tile.nb == 0) set_device_error(a.err, GQA_DEVERR_NO_VISIBLE);
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
    int last_k[kKStages], last_v[kVStages];
    for (int s = 0; s < kKStages; ++s) last_k[s] = -1;
    for (int s = 0; s < kVStages; ++s) last_v[s] = -1;
    // Test hook (off unless the host enabled it): CTA 0 first waits on a barrier that nothing
    // signals, so its bounded wait runs out, records GQA_DEVERR_TIMEOUT and aborts the CTA before
    // any copy is issued; every other role then gives up through the abort flag.
    const bool go = !(a.expire_wait && blockIdx.x == 0) || wait_bar(bar(kBarNever), 0, abort, a.err);
    if (go) {
      const int zq = tile.b * a.h_q + tile.g * a.r + tile.hb * a.H;  // first head of the block
      mbar_arrive_expect_tx(bar(kBarQ), (uint32_t)(C::kNch * a.H * a.P * 128));
      for (int ch = 0; ch < C::kNch; ++ch)
        tma_load_3d(sQ + ch * C::kQChunk, &tmq, bar(kBarQ), ch * 64, tile.q0, zq);
    }
    const int row0 = (tile.b * a.h_kv + tile.g) * a.T_max;
    for (int j = 0; j < nb && go; ++j) {
      const int ks = j % kKStages, kn = j / kKStages;
      if (kn > 0 && !wait_bar(bar(kBarKEmpty + ks), (uint32_t)((kn - 1) & 1), abort, a.err)) break;
      mbar_arrive_expect_tx(bar(kBarKFull + ks), C::kKVBytes);
      for (int ch = 0; ch < C::kNch; ++ch)
        tma_load_2d(sK + ks * C::kKVBytes + ch * C::kKVChunk, &tmk, bar(kBarKFull + ks), ch * 64,
                    row0 + (tile.j0 + j) * kBN);
      last_k[ks] = kn;
      const int vs = j % kVStages, vn = j / kVStages;
      if (vn > 0 && !wait_bar(bar(kBarVEmpty + vs), (uint32_t)((vn - 1) & 1), abort, a.err)) break;
      mbar_arrive_expect_tx(bar(kBarVFull + vs), C::kKVBytes);
      for (int ch = 0; ch < C::kNch; ++ch)
        tma_load_2d(sV + vs * C::kKVBytes + ch * C::kKVChunk, &tmv, bar(kBarVFull + vs), ch * 64,
                    row0 + (tile.j0 + j) * kBN);
      last_v[vs] = vn;
    }
    // Drain (bounded, whatever the abort state): no copy may still be landing in shared memory
    // when the CTA exits.
    volatile int no_abort = 0;
    if (go) wait_bar(bar(kBarQ), 0, &no_abort, a.err);
    for (int s = 0; s < kKStages; ++s)
      if (last_k[s] >= 0) wait_bar(bar(kBarKFull + s), (uint32_t)(last_k[s] & 1), &no_abort, a.err);
    for (int s = 0; s < kVStages; ++s)
      if (last_v[s] >= 0) wait_bar(bar(kBarVFull + s), (uint32_t)(last_v[s] & 1), &no_abort, a.err);
  } else if (warp == 1 && lane == 0 && nb > 0) {
    // ------------------------------ MMA issuer ---------------------------------------------
    constexpr uint32_t idesc_qk = tc::idesc_bf16(kBM, kBN, false);
    constexpr uint32_t idesc_pv = tc::idesc_bf16(kBM, D, true);
    auto colS = [](int buf) { return buf ? C::kColS1 : C::kColS0; };
    auto qk = [&](int j, int buf) {  // S_buf = Q K_j^T; Q (A) from TMEM, 8 columns per 16 of d_h
      const int ks = j % kKStages;
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t koff = (uint32_t)((k >> 2) * C::kKVChunk + (k & 3) * 32);
        const uint64_t bd = tc::smem_desc(sK + ks * C::kKVBytes + koff, 16, 1024);
        tc::mma_ts(tmem + colS(buf), tmem + C::kColQ + k * 8, bd, idesc_qk, k > 0 ? 1u : 0u);
      }
    };
    auto pv = [&](int j, int buf) {  // O += P_buf V_j; P (A) from TMEM, 8 columns per 16 keys
      const int vs = j % kVStages;
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk) {
        const uint64_t bd = tc::smem_desc(sV + vs * C::kKVBytes + kk * 2048, C::kKVChunk, 1024);
        tc::mma_ts(tmem + C::kColO, tmem + colS(buf) + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
      }
    };
    bool ok = wait_bar(bar(kBarQT), 0, abort, a.err);
    for (int j = 0; j < 2 && j < nb && ok; ++j) {
      ok = wait_bar(bar(kBarKFull + j % kKStages), (uint32_t)((j / kKStages) & 1), abort, a.err);
      if (!ok) break;
      tc::fence_after_sync();
      qk(j, j & 1);
      tc::commit(bar(kBarS + (j & 1)));
      tc::commit(bar(kBarKEmpty + j % kKStages));
    }
    for (int j = 0; j < nb && ok; ++j) {
      const int buf = j & 1;
      if (!wait_bar(bar(kBarVFull + j % kVStages), (uint32_t)((j / kVStages) & 1), abort, a.err)) break;
      if (!wait_bar(bar(kBarP + buf), (uint32_t)((j >> 1) & 1), abort, a.err)) break;
      tc::fence_after_sync();
      pv(j, buf);
      tc::commit(bar(kBarO));
      tc::commit(bar(kBarVEmpty + j % kVStages));
      const int jn = j + 2;
      if (jn < nb) {
        if (!wait_bar(bar(kBarKFull + jn % kKStages), (uint32_t)((jn / kKStages) & 1), abort, a.err)) break;
        tc::fence_after_sync();
        qk(jn, buf);
        tc::commit(bar(kBarS + buf));
        tc::commit(bar(kBarKEmpty + jn % kKStages));
      }
    }
    // every MMA issued above has completed before TMEM is released
    tc::commit(bar(kBarDone));
    volatile int no_abort = 0;
    wait_bar(bar(kBarDone), 0, &no_abort, a.err);
  } else if (warp >= 4) {
    softmax_role<D, kWin>(a, tile, warp, lane, tmem, sQ, sV, bars, xbuf, abort);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool kWin>
cudaError_t launch_typed(const PArgs& p, const CUtensorMap* tmaps, long long tiles, cudaStream_t s) {
  auto kern = prefill_bf16_kernel<D, kWin>;
  static bool attr_set[64] = {false};  // per device: the shared-memory opt-in is set once
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  kern<<<(unsigned)tiles, kThreads, Cfg<D>::kSmem, s>>>(tmaps[0], tmaps[1], tmaps[2], p);
  return cudaGetLastError();
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
  p.n_qt = (a.S_q + p.P - 1) / p.P;
  p.scale_log2 = a.scale * pf::kLog2e;
  p.causal = a.causal;
  p.window = a.window;
  p.expire_wait = a.expire_wait;
  p.err = a.err;
  const long long tiles = (long long)p.n_qt * a.B * a.h_kv * p.hblocks;
  if (tiles <= 0) return cudaSuccess;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (a.d_h == 128) {
    return a.window > 0 ? pf::launch_typed<128, true>(p, tmaps, tiles, s)
                        : pf::launch_typed<128, false>(p, tmaps, tiles, s);
  }
  if (a.d_h == 64) {
    return a.window > 0 ? pf::launch_typed<64, true>(p, tmaps, tiles, s)
                        : pf::launch_typed<64, false>(p, tmaps, tiles, s);
  }
  return cudaErrorInvalidValue;
}

int prefill_heads_per_tile(int h_q, int h_kv) {
  const int r = h_q / h_kv;
  return r < pf::kBM ? r : pf::kBM;
}

}  // namespace gqa
