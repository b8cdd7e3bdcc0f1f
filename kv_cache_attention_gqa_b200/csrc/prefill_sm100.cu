// bf16 causal grouped-query attention prefill on sm_100a: TMA + tcgen05 (TMEM accumulators).
//
// What it computes: O_a = softmax(Q_a K_{g(a)}^T * scale + M) V_{g(a)} with g(a) = floor(a / r)
// [序列计算与存储, section 分组查询注意力], the causal/length mask by absolute position
// [第 09 章 GQA、MLA 与跨层 KV 共享, section 09.2], evaluated block by block with the online
// softmax state (m, l, u) so the score matrix never reaches memory [序列计算与存储, sections
// 分块注意力 and 在线 softmax]. An optional sliding window W limits row p to keys p - W < j <= p
// [第三章：MHA 的局限与 MQA、GQA、Flash Attention, section 3.7]: K/V blocks below the CTA's
// earliest window are never loaded, and the boundary blocks are masked per row.
//
// Work tiles. Rows of one tile are (query position, query head) pairs of ONE KV group: H heads
// (H = min(r, 128)) times P = floor(128 / H) consecutive positions, head-major, so every K/V block
// staged in shared memory serves all r heads of the group [MHA/MQA/GQA walkthrough, section 7:
// e.g. 32 positions x 4 heads = 128 rows; the mask still uses each row's own position]. Each CTA
// runs two independent online-softmax chains, t = 0 and 1, in one of two modes:
//   pair mode   chain t is tile t of two tiles of the same group and heads at consecutive positions
//               (2P positions); each K/V block is staged once for 256 rows.
//   split mode  (when pairs would leave SMs idle, e.g. 512 new queries over a long cache) the CTA
//               holds one tile and chain t takes the tile's K/V blocks t, t + 2, t + 4, ...; at
//               the end the two partial states (m, l, O) of each row merge inside the CTA:
//               O = (2^(m_0 - M) O_0 + 2^(m_1 - M) O_1) / (2^(m_0 - M) l_0 + 2^(m_1 - M) l_1),
//               M = max(m_0, m_1) [第三章, section 3.5: partial results merge after rescaling].
//
// Roles (384 threads, three warpgroups):
//   warp 0      TMA producer: the Q rows once, then 128-key K blocks into a 3-deep ring and
//               V blocks into a 2-deep ring (cp.async.bulk.tensor, 128-byte swizzle, no multicast).
//   warp 1+t    issues the MMAs of tile t (warp 1 also allocates the 512 TMEM columns):
//               S_t = Q_t K_j^T (tcgen05.mma kind::f16, A = Q_t and B = K_j from shared memory),
//               O_t += P_t V_j  (A = P_t from TMEM, B = V_j from shared memory, MN-major).
//               O_t += P_j V_j is followed at once by S_t = Q_t K_{j+1}^T: MMAs issued by one
//               thread execute in order, so the new scores overwrite P_j only after it was read.
//               The two tiles' chains are independent: while one tile's softmax runs, the tensor
//               core works on the other's MMAs. (A single thread issuing both tiles' MMAs was the
//               bottleneck: an MMA issue returns only when the shallow MMA queue has room, so the
//               thread's waits and commits between batches left the tensor core idle.) Each warp
//               runs its loop as a whole, so its state and the operand descriptors stay uniform,
//               and one elected lane issues a batch of MMAs together with its commits.
//   warp 3      idle (it completes the first warpgroup, whose registers go to the softmax).
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: a warp reaches the TMEM lane
//               quarter warp % 4, so each warpgroup covers the 128 rows of its tile, one row per
//               thread and all 128 columns of each block. Per block a thread loads its
//               scores, masks them by absolute position (one clamped 32-bit bound per row) only on
//               blocks that straddle the diagonal, the length or a window, takes the row maximum,
//               and writes P = 2^(s * scale * log2 e - m) as bf16 over the first 64 columns of the
//               tile's S. It rescales its O row only when the running maximum grew by more than 8
//               (base 2): between rescales P and l share the stale maximum, which leaves
//               O = u / l unchanged. No softmax thread waits on the other tile.
// Registers: the launch gives 168 per thread (3 warps of 168 fill a sub-partition's 16,384); the
// first warpgroup gives back down to 64 and each softmax warpgroup takes 216 (64 + 216 + 216 <=
// 3 x 168), which holds a thread's 128 scores without spilling.
// TMEM columns: tile t holds S_t at [256 t, 256 t + 128) and O_t at [256 t + 128, 256 t + 128 + D).

#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace gqa {
namespace pf {

constexpr int kBM = 128;     // rows per tile (= TMEM lanes)
constexpr int kBN = 128;     // keys per K/V block
constexpr int kTiles = 2;    // tiles per CTA
constexpr int kKStages = 3;  // K ring depth
constexpr int kVStages = 2;  // V ring depth
constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;  // first softmax warp: warps 4-7 serve tile 0, warps 8-11 tile 1
constexpr int kRegsControl = 64;  // per thread, first warpgroup (producer, MMA issuer, idle)
constexpr int kRegsSoftmax = 216; // per thread, softmax warpgroups
constexpr uint32_t kTmemCols = 512;
constexpr int kBarBytes = 512;  // barrier block: the mbarriers, the TMEM address and the abort flag
constexpr float kRescaleThreshold = 8.0f;  // base-2 units: P <= 2^8 between rescales
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static constexpr int kNch = D / 64;                  // 64-column (128-byte) chunks
  static constexpr int kQChunk = kBM * 128;            // bytes of one Q chunk (128 rows)
  static constexpr int kQBytes = kNch * kQChunk;       // one tile's Q rows
  static constexpr int kKVChunk = kBN * 128;
  static constexpr int kKVBytes = kNch * kKVChunk;     // one K (or V) block
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kTiles * kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kKVBytes;
  static constexpr int kOffBar = kOffV + kVStages * kKVBytes;
  // barriers + slack for 1024-byte alignment; at least 120 KiB so that only one CTA (which
  // allocates all 512 TMEM columns) is resident per SM
  static constexpr int kSmem =
      kOffBar + kBarBytes + 1024 > 120 * 1024 ? kOffBar + kBarBytes + 1024 : 120 * 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t colS(int t) { return (uint32_t)(256 * t); }
  static constexpr uint32_t colO(int t) { return (uint32_t)(256 * t + 128); }
};

struct PArgs {
  void* o;
  float* lse;
  const int32_t* q_start;
  const int32_t* kv_len;
  int B, h_q, h_kv, r, S_q, T_max;
  int H, P, hblocks, n_pairs, n_qt;
  int split;  // 1: split mode (one tile per CTA, alternate blocks per chain)
  float scale_log2;
  int causal;
  int window;  // 0: none; W > 0: row at position p also needs key j > p - W (causal only)
  int expire_wait;  // test hook: CTA 0's producer first waits on a barrier that nothing signals
  unsigned* err;
};

// barrier indices inside the barrier block (derived from the ring depths, so they never overlap)
enum : int {
  kBarQ = 0,                                    // + tile: Q rows landed in shared memory (TMA)
  kBarKFull = kBarQ + kTiles,                   // + K stage
  kBarVFull = kBarKFull + kKStages,             // + V stage
  kBarKEmpty = kBarVFull + kVStages,            // + chain * kKStages + K stage: the chain's
                                                //   S = Q K^T on that stage completed
  kBarVEmpty = kBarKEmpty + kTiles * kKStages,  // + chain * kVStages + V stage: its O += P V did
  kBarS = kBarVEmpty + kTiles * kVStages,       // + chain: S_t of the chain's current block is in
                                                //   TMEM
  kBarP = kBarS + kTiles,                       // + chain: P_t of its current block is in TMEM
                                                //   (128 arrivals)
  kBarO = kBarP + kTiles,                       // + chain: O_t += P_t V of its current block done
  kBarDone = kBarO + kTiles,                    // + chain: every MMA of the chain's issuer done
  kBarNever = kBarDone + kTiles,                // never signalled: the test hook's wait runs out
  kBarTurn = kBarNever + 1,                     // + chain: the other chain finished its
                                                //   exponentials (128 arrivals)
  kNumBars = kBarTurn + kTiles
};
static_assert(kNumBars * 8 + 8 <= kBarBytes, "barrier block");

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

// The CTA's work: tiles t = 0, 1 at positions q0 + t P .. q0 + (t + 1) P - 1 of the heads
// hb H .. hb H + nh - 1 of group g.
struct Work {
  int b, g, hb, q0;  // q0: first query position (index into S_q) of tile 0
  int nh;            // heads of this head block
  int qs, kv;        // q_start[b], kv_len[b]
  bool split;        // split mode
  int nq;            // Q tiles loaded (pair mode: tiles with at least one query row; split: 1)
  int nt;            // chains (pair mode: nq; split mode: 2)
  int j0;            // first K/V block of the CTA (> 0 only under a sliding window)
  int nb[kTiles];    // blocks chain t visits: pair mode j0 .. j0 + nb[t] - 1 (nb[0] <= nb[1]);
                     // split mode j0 + t, j0 + t + 2, ... (nb[0] >= nb[1])
  int nbmax;         // K/V blocks the CTA loads
  bool valid;
  // CTA block index (from j0) of chain t's i-th block
  template <bool kSplit>
  __device__ __forceinline__ int blk(int t, int i) const { return kSplit ? 2 * i + t : i; }
  // first query index of the rows of chain t
  template <bool kSplit>
  __device__ __forceinline__ int qrow0(int t, int P) const { return kSplit ? q0 : q0 + t * P; }
};

__device__ __forceinline__ Work make_work(const PArgs& a) {
  Work w;
  const int per = a.B * a.h_kv * a.hblocks;
  const int idx = blockIdx.x;
  // heaviest (latest positions) first
  const int pr = (a.split ? a.n_qt : a.n_pairs) - 1 - idx / per;
  const int rem = idx - (idx / per) * per;
  w.b = rem / (a.h_kv * a.hblocks);
  const int gh = rem - w.b * (a.h_kv * a.hblocks);
  w.g = gh / a.hblocks;
  w.hb = gh - w.g * a.hblocks;
  w.split = a.split != 0;
  w.q0 = pr * (w.split ? 1 : kTiles) * a.P;
  w.nh = min(a.H, a.r - w.hb * a.H);
  w.nq = !w.split && w.q0 + a.P < a.S_q ? 2 : 1;
  w.nt = w.split ? 2 : w.nq;
  w.kv = a.kv_len ? a.kv_len[w.b] : a.T_max;
  w.qs = a.q_start ? a.q_start[w.b] : 0;
  w.valid = w.kv >= 1 && w.kv <= a.T_max && w.qs >= 0;
  w.j0 = 0;
  w.nbmax = 0;
  for (int t = 0; t < kTiles; ++t) w.nb[t] = 0;
  if (!w.valid) return w;
  if (a.causal) {
    if (a.window > 0) {
      // blocks wholly below the earliest row's window are skipped [第三章 §3.7: each query reads
      // only its local window]
      const long long lo = (long long)w.qs + w.q0 - a.window + 1;
      if (lo > 0) w.j0 = (int)(lo / kBN);
    }
    for (int t = 0; t < w.nq; ++t) {
      const int last_row = min(w.q0 + (t + 1) * a.P, a.S_q) - 1;
      const long long pos_max = (long long)w.qs + last_row;
      const long long last_key = pos_max < w.kv - 1 ? pos_max : (long long)(w.kv - 1);
      const int end = (int)(last_key / kBN) + 1;
      w.nb[t] = end > w.j0 ? end - w.j0 : 0;
    }
  } else {
    for (int t = 0; t < w.nq; ++t) w.nb[t] = (w.kv + kBN - 1) / kBN;
  }
  w.nbmax = w.nb[w.nq - 1];
  if (w.split) {  // the tile's blocks alternate between the chains
    w.nb[0] = (w.nbmax + 1) / 2;
    w.nb[1] = w.nbmax / 2;
  }
  return w;
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

// Softmax of chain t: a thread owns one row (its TMEM lane) and all 128 columns of each block.
// kWin: the launch has a sliding window (a.window > 0). Without one, the window code is compiled
// out (its per-element compare in the mask loop costs ~9% of the causal kernel's time).
// tcgen05.ld / st / wait are .sync.aligned: every lane of a warp executes each of them, so every
// condition in front of one is made warp-uniform (__all_sync / __any_sync) first.
// xm: 512 floats of shared memory for the split-mode merge (the unused second Q tile).
template <int D, bool kWin, bool kSplit>
__device__ __forceinline__ void softmax_role(const PArgs& a, const Work& w, int t, int wq, int lane,
                                             uint32_t tmem, uint32_t sV, uint64_t* bars, float* xm,
                                             volatile int* abort) {
  using C = Cfg<D>;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int row = wq * 32 + lane;             // TMEM lane = tile row
  const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
  const uint32_t colS = C::colS(t), colO = C::colO(t);
  const int h = row / a.P, p = row - h * a.P;
  const int qt0 = w.qrow0<kSplit>(t, a.P);    // first query index of this chain's rows
  const int qi = qt0 + p;                     // query index into S_q
  const bool store_row = h < w.nh && row < a.H * a.P && qi < a.S_q;
  const long long pos = (long long)w.qs + qi;
  // last key this row may see (length and causal limits in one 32-bit bound for the mask loop)
  const long long kl = a.causal && pos < w.kv - 1 ? pos : (long long)w.kv - 1;
  const int key_last = (int)kl;
  const long long pos_min = (long long)w.qs + qt0;                        // smallest in the tile
  const long long pos_max = (long long)w.qs + min(qt0 + a.P, a.S_q) - 1;  // largest in the tile
  const long long cta_pos_min = (long long)w.qs + w.q0;                   // smallest in the CTA
  const int nb = w.nb[t];
  const float c = a.scale_log2;
  const int win = kWin ? a.window : 0;
  // last key below this row's window, clamped to the int range (keys are ints)
  const long long wl = pos - win;
  const int win_last = kWin ? (int)(wl < -1 ? -1 : (wl > 0x7fffffffLL ? 0x7fffffffLL : wl)) : -1;
  const long long orow = ((long long)w.b * a.h_q + w.g * a.r + w.hb * a.H + h) * a.S_q + qi;
  __nv_bfloat16* const orow_ptr = reinterpret_cast<__nv_bfloat16*>(a.o) + orow * D;

  // Rows of a chain that gives up (a bounded wait ran out; the error word says so) or has no
  // block to visit are written as zeros with lse = -inf, without touching TMEM. In split mode each
  // chain writes its half of the columns.
  auto zero_rows = [&](int c0, int c1) {
    if (!store_row) return;
    uint4* z = reinterpret_cast<uint4*>(orow_ptr);
    for (int v = c0 / 8; v < c1 / 8; ++v) z[v] = make_uint4(0u, 0u, 0u, 0u);
    if (a.lse && c0 == 0) a.lse[orow] = -INFINITY;
  };
  if (nb == 0 && !kSplit) {
    zero_rows(0, D);
    return;
  }

  bool ok = true;
  float m = -INFINITY, l = 0.f;
  for (int i = 0; i < nb; ++i) {
    const int j = w.blk<kSplit>(t, i);  // block of the CTA (from j0)
    ok = ok && wait_bar(bar(kBarS + t), (uint32_t)(i & 1), abort, a.err);
    if (!__all_sync(0xffffffffu, ok)) {
      ok = false;
      break;
    }
    tc::fence_after_sync();
    float sr[kBN];
#pragma unroll
    for (int q = 0; q < 4; ++q) tc::ld32f(lane_addr + colS + q * 32, sr + q * 32);
    tc::wait_ld();
    const int key0 = (w.j0 + j) * kBN;  // first key of the block
    const bool need_mask = (a.causal && (long long)key0 + kBN - 1 > pos_min) || key0 + kBN > w.kv ||
                           (kWin && (long long)key0 <= pos_max - win);
    if (need_mask) {
#pragma unroll
      for (int k = 0; k < kBN; ++k) {
        const int key = key0 + k;
        const bool vis = key <= key_last && (!kWin || key > win_last);
        sr[k] = vis ? sr[k] : -INFINITY;
      }
    }
    float mx0 = sr[0], mx1 = sr[1], mx2 = sr[2], mx3 = sr[3];
#pragma unroll
    for (int k = 4; k < kBN; k += 4) {
      mx0 = fmaxf(mx0, sr[k]);
      mx1 = fmaxf(mx1, sr[k + 1]);
      mx2 = fmaxf(mx2, sr[k + 2]);
      mx3 = fmaxf(mx3, sr[k + 3]);
    }
    const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c;
    // running maximum with lazy rescaling
    const float m_new = fmaxf(m, mx);
    float m_use = m, alpha = 1.f;
    bool rescale_o = false;
    if (m == -INFINITY) {
      m_use = m_new;  // nothing accumulated yet
    } else if (m_new > m + kRescaleThreshold) {
      m_use = m_new;
      alpha = fast_exp2(m - m_new);
      rescale_o = true;
    }
    // The two chains take turns on the exponential unit, chain 0 first in every round: left to
    // themselves their softmax phases overlap and share the unit, which lengthens both chains.
    // Chain 0 waits for chain 1's previous round, chain 1 for chain 0's current one (only while
    // the other chain still has blocks). The loads and the row maximum run outside the turn.
    const bool take_turn = w.nt == 2 && (t == 0 ? i >= 1 && i - 1 < w.nb[1] : i < w.nb[0]);
    if (take_turn) {
      ok = wait_bar(bar(kBarTurn + t), (uint32_t)((t == 0 ? i - 1 : i) & 1), abort, a.err);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
    }
    // P = 2^(s c - m_use) as bf16 pairs over the first 64 S columns. A row that has seen no
    // visible key yet keeps m = -inf (under a sliding window, or in split mode when the chain's
    // first block lies wholly after the row's position); its P is 0, computed against 0 instead
    // of -inf.
    const float m_sub = m_use == -INFINITY ? 0.f : m_use;
    float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float x0, x1;
        ffma2(x0, x1, sr[cc * 32 + 2 * k], sr[cc * 32 + 2 * k + 1], c, -m_sub);
        const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
        fadd2(sum0, sum1, p0, p1);
        pk[k] = pack_bf16x2(p0, p1);
      }
      tc::st16(lane_addr + colS + cc * 16, pk);
      // the other chain's turn starts halfway through this one's exponentials (the halves
      // overlap a little on the unit, which measured faster than strict alternation)
      if (cc == 1 && w.nt == 2) mbar_arrive(bar(kBarTurn + (t ^ 1)));
    }
    l = l * alpha + (sum0 + sum1);
    m = m_use;
    // the warp rescales its O rows together when any of its rows needs it (rows that do not need
    // it multiply by alpha = 1); O must first hold every earlier block's contribution
    if (__any_sync(0xffffffffu, rescale_o && i > 0)) {
      ok = wait_bar(bar(kBarO + t), (uint32_t)((i - 1) & 1), abort, a.err);
      if (__all_sync(0xffffffffu, ok)) {
        tc::fence_after_sync();
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tc::ld32(lane_addr + colO + cc * 32, o);
          tc::wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tc::st32(lane_addr + colO + cc * 32, o);
        }
      } else {
        ok = false;
      }
    }
    tc::wait_st();
    // V rows at or past kv_len, and (sliding window) rows below the CTA's earliest window, get
    // weight 0 for every row but may hold anything (NaN included), so they are zeroed in shared
    // memory before this chain's O += P V may read them, and 0 * V stays 0. In pair mode both
    // tiles zero them (the two chains' MMAs are not ordered); a second write stores the same zeros.
    const int bkey0 = (w.j0 + j) * kBN;
    const bool zero_tail = bkey0 + kBN > w.kv;
    const bool zero_head = kWin && j == 0 && (long long)bkey0 < cta_pos_min - win + 1;
    if (ok && (zero_tail || zero_head)) {
      const int vs = j % kVStages;
      if (wait_bar(bar(kBarVFull + vs), (uint32_t)((j / kVStages) & 1), abort, a.err)) {
        const long long key = (long long)bkey0 + row;  // thread `row` owns V row `row` of the block
        if (row < kBN && ((zero_tail && key >= w.kv) || (zero_head && key <= cta_pos_min - win))) {
#pragma unroll
          for (int ch = 0; ch < C::kNch; ++ch) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t addr = sV + vs * C::kKVBytes + ch * C::kKVChunk + row * 128 + k * 16;
              asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
            }
          }
        }
        tc::fence_proxy_async_smem();
      } else {
        ok = false;
      }
    }
    tc::fence_before_sync();
    mbar_arrive(bar(kBarP + t));
    if (!__all_sync(0xffffffffu, ok)) {
      ok = false;
      break;
    }
  }
  // the chain's last O += P V has completed
  if (ok && nb > 0) ok = __all_sync(0xffffffffu, wait_bar(bar(kBarO + t), (uint32_t)((nb - 1) & 1), abort, a.err));
  if constexpr (!kSplit) {
    if (!ok) {
      zero_rows(0, D);
      return;
    }
    tc::fence_after_sync();
    // epilogue: O / l -> bf16 -> global; lse = (m + log2 l) * ln 2. A row with no visible key (a
    // sliding window that starts at or past kv_len, or a padding row of the tile) has l = 0: it
    // still takes part in the warp's TMEM loads, and writes zeros.
    const bool empty = kWin && l == 0.f;
    if (empty && store_row) set_device_error(a.err, GQA_DEVERR_NO_VISIBLE);
    const float inv = empty ? 0.f : 1.f / l;
    uint4* out = reinterpret_cast<uint4*>(orow_ptr);
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      tc::ld32(lane_addr + colO + cc * 32, o);
      tc::wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 16; ++k)
        pk[k] = empty ? 0u : pack_bf16x2(__uint_as_float(o[2 * k]) * inv, __uint_as_float(o[2 * k + 1]) * inv);
      if (store_row) {
#pragma unroll
        for (int v = 0; v < 4; ++v)
          out[cc * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    }
    if (store_row && a.lse) a.lse[orow] = empty ? -INFINITY : (m + __log2f(l)) * kLn2;
    return;
  } else {
  // ---- split mode: the two chains of each row meet. Each publishes (m, l), both warpgroups
  // meet at a named barrier (every softmax thread of the CTA reaches it, whatever happened
  // before), and each chain then writes half of the row's columns from both chains' O.
  if (!ok) *abort = 1;
  xm[(t * 2) * 128 + row] = m;
  xm[(t * 2 + 1) * 128 + row] = l;
  tc::fence_before_sync();
  named_barrier_sync(1, 256);
  tc::fence_after_sync();
  const int c0 = t * (D / 2), c1 = c0 + D / 2;
  if (*abort) {
    zero_rows(c0, c1);
    return;
  }
  const float m0 = xm[row], l0 = xm[128 + row], m1 = xm[256 + row], l1 = xm[384 + row];
  const float M = fmaxf(m0, m1);
  const bool empty = M == -INFINITY;  // no visible key in either chain (sliding window)
  if (empty && store_row && t == 0) set_device_error(a.err, GQA_DEVERR_NO_VISIBLE);
  const float f0 = empty || w.nb[0] == 0 ? 0.f : fast_exp2(m0 - M);
  const float f1 = empty || w.nb[1] == 0 ? 0.f : fast_exp2(m1 - M);
  const float L = l0 * f0 + l1 * f1;
  const float inv = empty ? 0.f : 1.f / L;
  const float g0 = f0 * inv, g1 = f1 * inv;
  uint4* out = reinterpret_cast<uint4*>(orow_ptr);
#pragma unroll
  for (int cc = 0; cc < D / 64; ++cc) {
    const int col = c0 + cc * 32;
    uint32_t o0[32], o1[32];
    if (w.nb[0] > 0) tc::ld32(lane_addr + C::colO(0) + col, o0);
    if (w.nb[1] > 0) tc::ld32(lane_addr + C::colO(1) + col, o1);
    tc::wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float v0 = 0.f, v1 = 0.f;
      if (w.nb[0] > 0) {
        v0 = __uint_as_float(o0[2 * k]) * g0;
        v1 = __uint_as_float(o0[2 * k + 1]) * g0;
      }
      if (w.nb[1] > 0) {
        v0 = fmaf(__uint_as_float(o1[2 * k]), g1, v0);
        v1 = fmaf(__uint_as_float(o1[2 * k + 1]), g1, v1);
      }
      pk[k] = empty ? 0u : pack_bf16x2(v0, v1);
    }
    if (store_row) {
#pragma unroll
      for (int v = 0; v < 4; ++v)
        out[col / 8 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    }
  }
  if (store_row && a.lse && t == 0) a.lse[orow] = empty ? -INFINITY : (M + __log2f(L)) * kLn2;
  }
}

__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile("{\n\t.reg .pred q;\n\telect.sync _|q, 0xffffffff;\n\tselp.u32 %0, 1, 0, q;\n\t}" : "=r"(p));
  return p != 0;
}

// MMA issuer of tile t: the whole warp runs the loop; one elected lane issues each batch of MMAs
// and the commits that follow it (a commit tracks the MMAs of the thread that issues it, and a
// converged warp elects the same lane every time). The shared-memory descriptors are built once:
// the start address sits in the low 14 bits (address >> 4, below 2^14 for any shared-memory
// address), so the descriptor of base + offset is the base's descriptor plus offset >> 4.
template <int D, bool kSplit>
__device__ __forceinline__ void mma_role(const PArgs& a, const Work& w, int t, uint32_t tmem,
                                         uint32_t sQ, uint32_t sK, uint32_t sV, uint64_t* bars,
                                         volatile int* abort) {
  using C = Cfg<D>;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  constexpr uint32_t idesc_qk = tc::idesc_bf16(kBM, kBN, false);
  constexpr uint32_t idesc_pv = tc::idesc_bf16(kBM, D, true);
  const int qslot = kSplit ? 0 : t;  // split mode: both chains read the one tile
  const uint64_t dQ = tc::smem_desc(sQ + qslot * C::kQBytes, 16, 1024);
  const uint64_t dK = tc::smem_desc(sK, 16, 1024);
  const uint64_t dV = tc::smem_desc(sV, C::kKVChunk, 1024);
  const uint32_t tS = tmem + C::colS(t), tO = tmem + C::colO(t);
  const int nb = w.nb[t];
  auto wait = [&](int b_, uint32_t parity) {
    return __all_sync(0xffffffffu, wait_bar(bar(b_), parity, abort, a.err));
  };
  // S_t = Q_t K^T: A = Q_t and B = the K stage, both K-major in shared memory, 16 columns of d_h
  // per MMA; then the commits of the scores and of the K stage
  auto qk = [&](int ks) {
    const uint64_t kd = dK + (uint64_t)((ks * C::kKVBytes) >> 4);
    if (elect_one()) {
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        tc::mma_ss(tS, dQ + (uint64_t)(((k >> 2) * C::kQChunk + (k & 3) * 32) >> 4),
                   kd + (uint64_t)(((k >> 2) * C::kKVChunk + (k & 3) * 32) >> 4), idesc_qk, k > 0 ? 1u : 0u);
      tc::commit(bar(kBarS + t));
      tc::commit(bar(kBarKEmpty + t * kKStages + ks));
    }
    __syncwarp();
  };
  // O_t += P_t V: A = P_t from TMEM (8 columns per 16 keys), B = the V stage (MN-major); then the
  // commits of the output and of the V stage
  auto pv = [&](int vs, bool first) {
    const uint64_t vd = dV + (uint64_t)((vs * C::kKVBytes) >> 4);
    if (elect_one()) {
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        tc::mma_ts(tO, tS + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv, (!first || kk > 0) ? 1u : 0u);
      tc::commit(bar(kBarO + t));
      tc::commit(bar(kBarVEmpty + t * kVStages + vs));
    }
    __syncwarp();
  };
  // block j of the CTA sits in K stage j % kKStages (fill j / kKStages) and V stage j % kVStages
  const int jf = w.blk<kSplit>(t, 0);
  bool ok = wait(kBarKFull + jf % kKStages, (uint32_t)((jf / kKStages) & 1)) && wait(kBarQ + qslot, 0);
  if (ok) {
    tc::fence_after_sync();
    qk(jf % kKStages);
  }
  for (int i = 0; i < nb && ok; ++i) {
    const int j = w.blk<kSplit>(t, i), vs = j % kVStages;
    if (!(ok = wait(kBarVFull + vs, (uint32_t)((j / kVStages) & 1)) && wait(kBarP + t, (uint32_t)(i & 1)))) break;
    tc::fence_after_sync();
    pv(vs, i == 0);
    if (i + 1 < nb) {
      const int jn = w.blk<kSplit>(t, i + 1);
      if (!(ok = wait(kBarKFull + jn % kKStages, (uint32_t)((jn / kKStages) & 1)))) break;
      tc::fence_after_sync();
      qk(jn % kKStages);
    }
  }
  // every MMA issued above has completed before TMEM is released
  if (elect_one()) tc::commit(bar(kBarDone + t));
  __syncwarp();
  volatile int no_abort = 0;
  wait_bar(bar(kBarDone + t), 0, &no_abort, a.err);
}

template <int D, bool kWin, bool kSplit>
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
  const Work w = make_work(a);

  if (threadIdx.x == 0) {
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(bar(kBarQ + t), 1);
      mbar_init(bar(kBarS + t), 1);
      mbar_init(bar(kBarP + t), 128);
      mbar_init(bar(kBarO + t), 1);
    }
    for (int s = 0; s < kKStages; ++s) mbar_init(bar(kBarKFull + s), 1);
    for (int s = 0; s < kVStages; ++s) mbar_init(bar(kBarVFull + s), 1);
    for (int i = 0; i < kTiles * kKStages; ++i) mbar_init(bar(kBarKEmpty + i), 1);
    for (int i = 0; i < kTiles * kVStages; ++i) mbar_init(bar(kBarVEmpty + i), 1);
    for (int t = 0; t < kTiles; ++t) mbar_init(bar(kBarDone + t), 1);
    for (int t = 0; t < kTiles; ++t) mbar_init(bar(kBarTurn + t), 128);
    mbar_init(bar(kBarNever), 1);
    *abort = 0;
    fence_barrier_init();
    if (!w.valid) set_device_error(a.err, w.kv < 1 || w.kv > a.T_max ? GQA_DEVERR_KV_LEN
                                                                      : GQA_DEVERR_POSITION);
    else if (w.nb[0] == 0) set_device_error(a.err, GQA_DEVERR_NO_VISIBLE);
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int nbmax = w.nbmax;
  // Whole warpgroups move registers from the control roles to the softmax; each setmaxnreg sits
  // inside its role's branch, so the compiler allocates each branch for its own budget.
  if (warp < kSoftmaxWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (warp == 0 && lane == 0 && nbmax > 0) {
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
      const int zq = w.b * a.h_q + w.g * a.r + w.hb * a.H;  // first head of the block
      for (int t = 0; t < w.nq; ++t) {
        mbar_arrive_expect_tx(bar(kBarQ + t), (uint32_t)(C::kNch * a.H * a.P * 128));
        for (int ch = 0; ch < C::kNch; ++ch)
          tma_load_3d(sQ + t * C::kQBytes + ch * C::kQChunk, &tmq, bar(kBarQ + t), ch * 64,
                      w.q0 + t * a.P, zq);
      }
    }
    const int row0 = (w.b * a.h_kv + w.g) * a.T_max;
    // A stage is refilled once every chain that read its previous block b has released it. Pair
    // mode: tile t reads blocks 0 .. nb[t] - 1, so its release of b is its (b / stages)-th on
    // that stage. Split mode: only chain b % 2 reads b, and the blocks of one chain on one stage
    // are spaced lcm(stages, 2) apart, so it is that chain's (b / lcm)-th release.
    auto released = [&](int empty0, int stages, int j) {
      const int s = j % stages, b = j - stages;
      if (b < 0) return true;
      if constexpr (kSplit) {
        const int period = stages % 2 ? 2 * stages : stages;
        return wait_bar(bar(empty0 + (b % 2) * stages + s), (uint32_t)((b / period) & 1), abort, a.err);
      } else {
        for (int t = 0; t < w.nt; ++t)
          if (b < w.nb[t] && !wait_bar(bar(empty0 + t * stages + s), (uint32_t)((b / stages) & 1), abort, a.err))
            return false;
        return true;
      }
    };
    for (int j = 0; j < nbmax && go; ++j) {
      const int ks = j % kKStages, kn = j / kKStages;
      if (!released(kBarKEmpty, kKStages, j)) break;
      mbar_arrive_expect_tx(bar(kBarKFull + ks), C::kKVBytes);
      for (int ch = 0; ch < C::kNch; ++ch)
        tma_load_2d(sK + ks * C::kKVBytes + ch * C::kKVChunk, &tmk, bar(kBarKFull + ks), ch * 64,
                    row0 + (w.j0 + j) * kBN);
      last_k[ks] = kn;
      const int vs = j % kVStages, vn = j / kVStages;
      if (!released(kBarVEmpty, kVStages, j)) break;
      mbar_arrive_expect_tx(bar(kBarVFull + vs), C::kKVBytes);
      for (int ch = 0; ch < C::kNch; ++ch)
        tma_load_2d(sV + vs * C::kKVBytes + ch * C::kKVChunk, &tmv, bar(kBarVFull + vs), ch * 64,
                    row0 + (w.j0 + j) * kBN);
      last_v[vs] = vn;
    }
    // Drain (bounded, whatever the abort state): no copy may still be landing in shared memory
    // when the CTA exits.
    volatile int no_abort = 0;
    if (go)
      for (int t = 0; t < w.nq; ++t) wait_bar(bar(kBarQ + t), 0, &no_abort, a.err);
    for (int s = 0; s < kKStages; ++s)
      if (last_k[s] >= 0) wait_bar(bar(kBarKFull + s), (uint32_t)(last_k[s] & 1), &no_abort, a.err);
    for (int s = 0; s < kVStages; ++s)
      if (last_v[s] >= 0) wait_bar(bar(kBarVFull + s), (uint32_t)(last_v[s] & 1), &no_abort, a.err);
    } else if ((warp == 1 || warp == 2) && warp - 1 < w.nt && w.nb[warp - 1] > 0) {
      // ------------------------------ MMA issuer of tile t ----------------------------------
      const int t = warp - 1;
      mma_role<D, kSplit>(a, w, t, tmem, sQ, sK, sV, bars, abort);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int t = (warp - kSoftmaxWarp0) >> 2;
    float* xm = reinterpret_cast<float*>(smem + C::kOffQ + C::kQBytes);  // second Q tile (split mode)
    if (t < w.nt) softmax_role<D, kWin, kSplit>(a, w, t, warp & 3, lane, tmem, sV, bars, xm, abort);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool kWin, bool kSplit>
cudaError_t launch_typed(const PArgs& p, const CUtensorMap* tmaps, long long ctas, cudaStream_t s) {
  auto kern = prefill_bf16_kernel<D, kWin, kSplit>;
  static bool attr_set[64] = {false};  // per device: the shared-memory opt-in is set once
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  kern<<<(unsigned)ctas, kThreads, Cfg<D>::kSmem, s>>>(tmaps[0], tmaps[1], tmaps[2], p);
  return cudaGetLastError();
}

}  // namespace pf

cudaError_t launch_prefill_bf16(const PrefillArgs& a, const CUtensorMap* tmaps, int num_sms,
                                cudaStream_t s) {
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
  const int n_qt = (a.S_q + p.P - 1) / p.P;
  p.n_qt = n_qt;
  p.n_pairs = (n_qt + pf::kTiles - 1) / pf::kTiles;
  // Pair mode shares each K/V block between two tiles; when that leaves SMs idle (few tiles, long
  // histories: e.g. 512 new queries over 32768 cached keys gives 64 pairs for 148 SMs), split mode
  // runs one tile per CTA and splits its blocks between the chains instead.
  const long long units = (long long)a.B * a.h_kv * p.hblocks;
  p.split = (long long)p.n_pairs * units < num_sms ? 1 : 0;
  p.scale_log2 = a.scale * pf::kLog2e;
  p.causal = a.causal;
  p.window = a.window;
  p.expire_wait = a.expire_wait;
  p.err = a.err;
  const long long ctas = (long long)(p.split ? n_qt : p.n_pairs) * units;
  if (ctas <= 0) return cudaSuccess;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const bool win = a.window > 0;
  if (a.d_h == 128) {
    if (p.split) return win ? pf::launch_typed<128, true, true>(p, tmaps, ctas, s)
                            : pf::launch_typed<128, false, true>(p, tmaps, ctas, s);
    return win ? pf::launch_typed<128, true, false>(p, tmaps, ctas, s)
               : pf::launch_typed<128, false, false>(p, tmaps, ctas, s);
  }
  if (a.d_h == 64) {
    if (p.split) return win ? pf::launch_typed<64, true, true>(p, tmaps, ctas, s)
                            : pf::launch_typed<64, false, true>(p, tmaps, ctas, s);
    return win ? pf::launch_typed<64, true, false>(p, tmaps, ctas, s)
               : pf::launch_typed<64, false, false>(p, tmaps, ctas, s);
  }
  return cudaErrorInvalidValue;
}

int prefill_heads_per_tile(int h_q, int h_kv) {
  const int r = h_q / h_kv;
  return r < pf::kBM ? r : pf::kBM;
}

}  // namespace gqa
