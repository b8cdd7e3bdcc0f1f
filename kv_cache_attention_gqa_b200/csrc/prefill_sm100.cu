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
//               V blocks into a 2-deep ring (cp.async.bulk.tensor, 128-byte swizzle, each CTA its own copies).
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
// first warpgroup gives back down to 72 and each softmax warpgroup takes 216 (72 + 216 + 216 =
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
constexpr int kRegsControl = 72;  // per thread, first warpgroup (producer, MMA issuers, idle)
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
  int split;    // 1: split mode (one tile per item, alternate blocks per chain)
  int n_items;  // work items (pairs or split tiles over all groups); the grid walks them
  FastDiv div_per, div_gh, div_hb;  // by B h_kv hblocks, h_kv hblocks and hblocks
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
  kBarTurn = kBarNever + 1,                     // chain 0's turn: chain 1 is halfway through a
                                                //   round's exponentials (128 arrivals); then
                                                //   + 1 + (round & 3): chain 1's turn, chain 0
                                                //   halfway through that round (128 arrivals)
  kBarQEmpty = kBarTurn + 5,               // + chain: the chain's last S = Q K^T of an item
                                                //   completed (its Q rows may be replaced)
  kNumBars = kBarQEmpty + kTiles
};
// the barriers, then the TMEM address, the abort flag and the split-mode merge's abort word
static_assert(kNumBars * 8 + 12 <= kBarBytes, "barrier block");

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

// One work item: tiles t = 0, 1 at positions q0 + t P .. q0 + (t + 1) P - 1 of the heads
// hb H .. hb H + nh - 1 of group g.
struct Work {
  int b, g, hb, q0;  // q0: first query position (index into S_q) of tile 0
  int nh;            // heads of this head block
  int qs, kv;        // q_start[b], kv_len[b]
  bool split;        // split mode
  int nq;            // Q tiles loaded (pair mode: tiles with at least one query row; split: 1)
  int nt;            // chains (pair mode: nq; split mode: 2)
  int j0;            // first K/V block of the item (> 0 only under a sliding window)
  int nb[kTiles];    // blocks chain t visits: pair mode j0 .. j0 + nb[t] - 1 (nb[0] <= nb[1]);
                     // split mode j0 + t, j0 + t + 2, ... (nb[0] >= nb[1])
  int nbmax;         // K/V blocks the item loads
  bool valid;
  // nb[t] for a chain index known only at run time. (A run-time index into a struct's array puts
  // the struct in local memory, which the shared-memory carve-out leaves almost no L1 for: the
  // roles' per-item bookkeeping measured over a microsecond per item that way.)
  __device__ __forceinline__ int nbt(int t) const { return t == 0 ? nb[0] : nb[1]; }
  // item block index (from j0) of chain t's i-th block
  template <bool kSplit>
  __device__ __forceinline__ int blk(int t, int i) const { return kSplit ? 2 * i + t : i; }
  // first query index of the rows of chain t
  template <bool kSplit>
  __device__ __forceinline__ int qrow0(int t, int P) const { return kSplit ? q0 : q0 + t * P; }
};

// Item idx: items are numbered heaviest (latest positions) first.
__device__ __forceinline__ Work make_work(const PArgs& a, int idx) {
  Work w;
  const int per = a.B * a.h_kv * a.hblocks;
  const int qd = a.div_per.div(idx);
  const int pr = (a.split ? a.n_qt : a.n_pairs) - 1 - qd;
  const int rem = idx - qd * per;
  w.b = a.div_gh.div(rem);
  const int gh = rem - w.b * (a.h_kv * a.hblocks);
  w.g = a.div_hb.div(gh);
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
#pragma unroll
  for (int t = 0; t < kTiles; ++t) w.nb[t] = 0;
  if (!w.valid) return w;
  if (a.causal) {
    if (a.window > 0) {
      // blocks wholly below the earliest row's window are skipped [第三章 §3.7: each query reads
      // only its local window]
      const long long lo = (long long)w.qs + w.q0 - a.window + 1;
      if (lo > 0) w.j0 = (int)(lo / kBN);
    }
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
      if (t >= w.nq) break;
      const int last_row = min(w.q0 + (t + 1) * a.P, a.S_q) - 1;
      const long long pos_max = (long long)w.qs + last_row;
      const long long last_key = pos_max < w.kv - 1 ? pos_max : (long long)(w.kv - 1);
      const int end = (int)(last_key / kBN) + 1;
      w.nb[t] = end > w.j0 ? end - w.j0 : 0;
    }
  } else {
#pragma unroll
    for (int t = 0; t < kTiles; ++t)
      if (t < w.nq) w.nb[t] = (w.kv + kBN - 1) / kBN;
  }
  w.nbmax = w.nq == 2 ? w.nb[1] : w.nb[0];
  if (w.split) {  // the tile's blocks alternate between the chains
    w.nb[0] = (w.nbmax + 1) / 2;
    w.nb[1] = w.nbmax / 2;
  }
  return w;
}

// In pair mode the grid is persistent: CTA c of G takes items c, 2G - 1 - c, 2G + c, 4G - 1 - c,
// ... (a snake over the heaviest-first order, which evens out the CTAs' total work), and each role
// runs its pipeline straight on from one item into the next: the producer loads the next item's
// rows and blocks while the current item's last blocks are still in the softmax, and no CTA start,
// set-up or drain sits between items (a CTA's start and end measured ~7 us per item, about three
// blocks' worth). Split mode, chosen when the items barely fill the SMs, runs one item per CTA.
__device__ __forceinline__ long long item_of(int it) {
  const long long base = (long long)it * gridDim.x;
  return base + ((it & 1) ? gridDim.x - 1 - blockIdx.x : blockIdx.x);
}

// Running counts over the items a CTA has done so far. Every role derives them from the same
// items, so each role knows the phase of every barrier it waits on.
struct Seq {
  int J;           // K/V blocks loaded
  int ci[kTiles];  // blocks of chain t (phases of its S, P and O barriers)
  int qf[kTiles];  // fills of Q slot q
  // the same with a run-time index (see Work::nbt)
  __device__ __forceinline__ int ci_of(int t) const { return t == 0 ? ci[0] : ci[1]; }
  __device__ __forceinline__ int qf_of(int q) const { return q == 0 ? qf[0] : qf[1]; }
};

__device__ __forceinline__ void advance(Seq& s, const Work& w) {
  s.J += w.nbmax;
#pragma unroll
  for (int t = 0; t < kTiles; ++t) {
    if (t < w.nt) s.ci[t] += w.nb[t];
    // pair mode: slot t holds tile t's rows when chain t runs; split mode: slot 0, both chains
    if (w.split ? t == 0 && w.nbmax > 0 : t < w.nq && w.nb[t] > 0) ++s.qf[t];
  }
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

// Softmax of chain t over the CTA's items: a thread owns one row (its TMEM lane) and all 128
// columns of each block.
// kWin: the launch has a sliding window (a.window > 0). Without one, the window code is compiled
// out (its per-element compare in the mask loop costs ~9% of the causal kernel's time).
// tcgen05.ld / st / wait are .sync.aligned: every lane of a warp executes each of them, so every
// condition in front of one is made warp-uniform (__all_sync / __any_sync) first.
// xm: 512 floats of shared memory for the split-mode merge (the unused second Q tile); xabort: a
// word that a split-mode chain sets before the merge when it gave up, read by both chains after
// the merge's first barrier, so that both take the same path through the barriers.
template <int D, bool kWin, bool kSplit>
__device__ __forceinline__ void softmax_role(const PArgs& a, int t, int wq, int lane, uint32_t tmem,
                                             uint32_t sV, uint64_t* bars, float* xm,
                                             volatile int* xabort, volatile int* abort) {
  using C = Cfg<D>;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int row = wq * 32 + lane;             // TMEM lane = tile row
  const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
  const uint32_t colS = C::colS(t), colO = C::colO(t);
  const int h = row / a.P, p = row - h * a.P;
  const float c = a.scale_log2;
  const int win = kWin ? a.window : 0;
  // running counts over the CTA's items (see Seq): K/V blocks loaded, this chain's blocks, rounds
  // of the other chain this chain's turn waits count (its arrivals), and this chain's arrivals
  int cJ = 0, cI = 0, cT = 0, cA = 0;
  // false once a wait gave up (the error word says so): this chain's rows of the remaining items
  // are written as zeros with lse = -inf, without touching TMEM
  bool ok = true;
  for (int it = 0; !kSplit || it < 1; ++it) {  // split mode: one item per CTA
    const long long item = item_of(it);
    if (item >= a.n_items) break;
    const Work w = make_work(a, (int)item);
    const int J0 = cJ, I0 = cI, T0 = cT, A0 = cA;  // counts before this item
    cJ += w.nbmax;
    if (t < w.nt) cI += w.nbt(t);
    if (w.nt == 2) {
      cT += w.nbt(t ^ 1);
      cA += w.nbt(t);
    }
    if (t >= w.nt) continue;  // pair mode: the item has no second tile
    const int qt0 = w.qrow0<kSplit>(t, a.P);    // first query index of this chain's rows
    const int qi = qt0 + p;                     // query index into S_q
    const bool store_row = h < w.nh && row < a.H * a.P && qi < a.S_q;
    const long long pos = (long long)w.qs + qi;
    // last key this row may see (length and causal limits in one 32-bit bound for the mask loop)
    const long long kl = a.causal && pos < w.kv - 1 ? pos : (long long)w.kv - 1;
    const int key_last = (int)kl;
    const long long pos_min = (long long)w.qs + qt0;                        // smallest in the tile
    const long long pos_max = (long long)w.qs + min(qt0 + a.P, a.S_q) - 1;  // largest in the tile
    const long long item_pos_min = (long long)w.qs + w.q0;                  // smallest in the item
    const int nb = w.nbt(t);
    // last key below this row's window, clamped to the int range (keys are ints)
    const long long wl = pos - win;
    const int win_last = kWin ? (int)(wl < -1 ? -1 : (wl > 0x7fffffffLL ? 0x7fffffffLL : wl)) : -1;
    const long long orow = ((long long)w.b * a.h_q + w.g * a.r + w.hb * a.H + h) * a.S_q + qi;
    __nv_bfloat16* const orow_ptr = reinterpret_cast<__nv_bfloat16*>(a.o) + orow * D;

    // Rows of a chain that gave up or has no block to visit are written as zeros with
    // lse = -inf. In split mode each chain writes its half of the columns.
    auto zero_rows = [&](int c0, int c1) {
      if (!store_row) return;
      uint4* z = reinterpret_cast<uint4*>(orow_ptr);
      for (int v = c0 / 8; v < c1 / 8; ++v) z[v] = make_uint4(0u, 0u, 0u, 0u);
      if (a.lse && c0 == 0) a.lse[orow] = -INFINITY;
    };
    if (!ok) {
      if constexpr (kSplit) zero_rows(t * (D / 2), t * (D / 2) + D / 2);
      else zero_rows(0, D);
      continue;
    }
    if (nb == 0 && !kSplit) {
      zero_rows(0, D);
      continue;
    }

    float m = -INFINITY, l = 0.f;
    for (int i = 0; i < nb; ++i) {
      const int j = w.blk<kSplit>(t, i);  // block of the item (from j0)
      const int gi = I0 + i;              // the chain's block count over the CTA's items
      ok = ok && wait_bar(bar(kBarS + t), (uint32_t)(gi & 1), abort, a.err);
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
      // Pair mode: the two chains take turns on the exponential unit, chain 0 first in every
      // round; left to themselves their softmax phases overlap and share the unit, which
      // lengthens both chains. Within an item chain 1 waits for chain 0's current round and chain
      // 0 for chain 1's previous one. Waits are by phase parity, so a barrier must not complete
      // two phases past the one its waiter asks for. Chain 1 cannot get there on chain 0's
      // barrier (its next round waits for chain 0's next one); chain 0's first round of an item
      // waits for nothing, so chain 0's rounds cycle through four barriers (the K/V rings keep
      // either chain within three rounds of the other: a block is loaded only after both chains
      // released the one two or three before it). Chain 0 waits on a single barrier, which lags
      // a phase when chain 1 runs two rounds behind; the wait then passes at once and chain 0
      // runs on (holding it to chain 1's pace there measured 8% slower on prefill_4k). Split
      // mode takes no turns (4% faster on chunked prefill than taking them). The loads and the
      // row maximum run outside the turn.
      if (!kSplit && w.nt == 2 && (t == 0 ? i >= 1 && i - 1 < w.nb[1] : i < w.nb[0])) {
        const int r = t == 0 ? T0 + i - 1 : T0 + i;  // the other chain's round to wait for
        ok = t == 0 ? wait_bar(bar(kBarTurn), (uint32_t)(r & 1), abort, a.err)
                    : wait_bar(bar(kBarTurn + 1 + (r & 3)), (uint32_t)((r >> 2) & 1), abort, a.err);
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
        if (!kSplit && cc == 1 && w.nt == 2)
          mbar_arrive(bar(t == 0 ? kBarTurn + 1 + ((A0 + i) & 3) : kBarTurn));
      }
      l = l * alpha + (sum0 + sum1);
      m = m_use;
      // the warp rescales its O rows together when any of its rows needs it (rows that do not
      // need it multiply by alpha = 1); O must first hold every earlier block's contribution
      if (__any_sync(0xffffffffu, rescale_o && i > 0)) {
        ok = wait_bar(bar(kBarO + t), (uint32_t)((gi - 1) & 1), abort, a.err);
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
      // V rows at or past kv_len, and (sliding window) rows below the item's earliest window,
      // get weight 0 for every row but may hold anything (NaN included), so they are zeroed in
      // shared memory before this chain's O += P V may read them, and 0 * V stays 0. In pair mode
      // both tiles zero them (the two chains' MMAs are not ordered); a second write stores the
      // same zeros.
      const int bkey0 = (w.j0 + j) * kBN;
      const bool zero_tail = bkey0 + kBN > w.kv;
      const bool zero_head = kWin && j == 0 && (long long)bkey0 < item_pos_min - win + 1;
      if (ok && (zero_tail || zero_head)) {
        const int jg = J0 + j;  // block count over the CTA's items
        const int vs = jg % kVStages;
        if (wait_bar(bar(kBarVFull + vs), (uint32_t)((jg / kVStages) & 1), abort, a.err)) {
          const long long key = (long long)bkey0 + row;  // thread `row` owns V row `row` of the block
          if (row < kBN && ((zero_tail && key >= w.kv) || (zero_head && key <= item_pos_min - win))) {
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
    // the chain's last O += P V of the item has completed
    if (ok && nb > 0)
      ok = __all_sync(0xffffffffu, wait_bar(bar(kBarO + t), (uint32_t)((I0 + nb - 1) & 1), abort, a.err));
    if constexpr (!kSplit) {
      if (!ok) {
        zero_rows(0, D);
        continue;
      }
      tc::fence_after_sync();
      // epilogue: O / l -> bf16 -> global; lse = (m + log2 l) * ln 2. A row with no visible key
      // (a sliding window that starts at or past kv_len, or a padding row of the tile) has l = 0:
      // it still takes part in the warp's TMEM loads, and writes zeros. The next item's first
      // O += P V, which overwrites O, waits for this warpgroup's P of that item, so it comes
      // after these loads.
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
    } else {
      // ---- split mode: the two chains of each row meet. Each publishes (m, l), both warpgroups
      // meet at a named barrier (every softmax thread of the CTA reaches it, whatever happened
      // before), and each chain then writes half of the row's columns from both chains' O.
      if (!ok) *xabort = 1;
      xm[(t * 2) * 128 + row] = m;
      xm[(t * 2 + 1) * 128 + row] = l;
      tc::fence_before_sync();
      named_barrier_sync(1, 256);
      tc::fence_after_sync();
      const int c0 = t * (D / 2), c1 = c0 + D / 2;
      if (*xabort) {  // set before the barrier only, so both chains see the same value
        ok = false;
        zero_rows(c0, c1);
        continue;
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
      // 16 columns at a time (the two chains' values of a chunk are live together)
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        const int col = c0 + cc * 16;
        uint32_t o0[16], o1[16];
        if (w.nb[0] > 0) tc::ld16(lane_addr + C::colO(0) + col, o0);
        if (w.nb[1] > 0) tc::ld16(lane_addr + C::colO(1) + col, o1);
        tc::wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
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
          out[col / 8] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          out[col / 8 + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (store_row && a.lse && t == 0) a.lse[orow] = empty ? -INFINITY : (M + __log2f(L)) * kLn2;
    }
  }
}

using tc::elect_one;

// MMA issuer of tile t over the CTA's items: the whole warp runs the loop; one elected lane issues
// each batch of MMAs and the commits that follow it (a commit tracks the MMAs of the thread that
// issues it, and a converged warp elects the same lane every time). The shared-memory descriptors
// are built once: the start address sits in the low 14 bits (address >> 4, below 2^14 for any
// shared-memory address), so the descriptor of base + offset is the base's descriptor plus
// offset >> 4.
template <int D, bool kSplit>
__device__ __forceinline__ void mma_role(const PArgs& a, int t, uint32_t tmem, uint32_t sQ,
                                         uint32_t sK, uint32_t sV, uint64_t* bars,
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
  auto wait = [&](int b_, uint32_t parity) {
    return __all_sync(0xffffffffu, wait_bar(bar(b_), parity, abort, a.err));
  };
  // S_t = Q_t K^T: A = Q_t and B = the K stage, both K-major in shared memory, 16 columns of d_h
  // per MMA; then the commits of the scores and of the K stage (and, after the item's last one,
  // of the Q rows)
  auto qk = [&](int ks, bool last) {
    const uint64_t kd = dK + (uint64_t)((ks * C::kKVBytes) >> 4);
    if (elect_one()) {
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        tc::mma_ss(tS, dQ + (uint64_t)(((k >> 2) * C::kQChunk + (k & 3) * 32) >> 4),
                   kd + (uint64_t)(((k >> 2) * C::kKVChunk + (k & 3) * 32) >> 4), idesc_qk, k > 0 ? 1u : 0u);
      tc::commit(bar(kBarS + t));
      tc::commit(bar(kBarKEmpty + t * kKStages + ks));
      if (last) tc::commit(bar(kBarQEmpty + t));
    }
    __syncwarp();
  };
  // O_t += P_t V: A = P_t from TMEM (8 columns per 16 keys), B = the V stage (MN-major); then the
  // commits of the output and of the V stage. An item's first one overwrites O_t: the P it waits
  // for comes from the softmax threads that read the previous item's O_t before (pair mode; a
  // split-mode CTA has one item).
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
  Seq sq = {};
  bool ok = true;
  for (int it = 0; ok && (!kSplit || it < 1); ++it) {  // split mode: one item per CTA
    const long long item = item_of(it);
    if (item >= a.n_items) break;
    const Work w = make_work(a, (int)item);
    const Seq s0 = sq;
    advance(sq, w);
    const int nb = t < w.nt ? w.nbt(t) : 0;
    // Pair mode: the blocks of the item this chain does not read (past its tile's last key, or
    // all of them when it has no tile) are taken and released unread, in block order after its
    // own, so that every wait of the chain on a stage is for that stage's next fill. (A chain that
    // skipped a fill could see its stage's earlier phase parity and take a block still in flight.)
    auto pass_over = [&](int j0_, int j1_) {
      for (int j = j0_; j < j1_ && ok; ++j) {
        const int jg = s0.J + j;
        const int ks = jg % kKStages, vs = jg % kVStages;
        ok = wait(kBarKFull + ks, (uint32_t)((jg / kKStages) & 1)) &&
             wait(kBarVFull + vs, (uint32_t)((jg / kVStages) & 1));
        if (ok && elect_one()) {
          mbar_arrive(bar(kBarKEmpty + t * kKStages + ks));
          mbar_arrive(bar(kBarVEmpty + t * kVStages + vs));
        }
        __syncwarp();
      }
    };
    if (nb == 0) {
      if constexpr (!kSplit) pass_over(0, w.nbmax);
      continue;
    }
    // block j of the item is the CTA's block s0.J + j: K stage (s0.J + j) % kKStages (fill
    // (s0.J + j) / kKStages), V stage (s0.J + j) % kVStages
    const int jf = s0.J + w.blk<kSplit>(t, 0);
    ok = wait(kBarKFull + jf % kKStages, (uint32_t)((jf / kKStages) & 1)) &&
         wait(kBarQ + qslot, (uint32_t)(s0.qf_of(qslot) & 1));
    if (!ok) break;
    tc::fence_after_sync();
    qk(jf % kKStages, nb == 1);
    for (int i = 0; i < nb && ok; ++i) {
      const int j = s0.J + w.blk<kSplit>(t, i), vs = j % kVStages;
      if (!(ok = wait(kBarVFull + vs, (uint32_t)((j / kVStages) & 1)) &&
                 wait(kBarP + t, (uint32_t)((s0.ci_of(t) + i) & 1))))
        break;
      tc::fence_after_sync();
      pv(vs, i == 0);
      if (i + 1 < nb) {
        const int jn = s0.J + w.blk<kSplit>(t, i + 1);
        if (!(ok = wait(kBarKFull + jn % kKStages, (uint32_t)((jn / kKStages) & 1)))) break;
        tc::fence_after_sync();
        qk(jn % kKStages, i + 2 == nb);
      }
    }
    if constexpr (!kSplit) pass_over(nb, w.nbmax);
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
  volatile int* xabort = abort + 1;
  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(bar(kBarQ + t), 1);
      mbar_init(bar(kBarS + t), 1);
      mbar_init(bar(kBarP + t), 128);
      mbar_init(bar(kBarO + t), 1);
      mbar_init(bar(kBarQEmpty + t), 1);
    }
    for (int s = 0; s < kKStages; ++s) mbar_init(bar(kBarKFull + s), 1);
    for (int s = 0; s < kVStages; ++s) mbar_init(bar(kBarVFull + s), 1);
    for (int i = 0; i < kTiles * kKStages; ++i) mbar_init(bar(kBarKEmpty + i), 1);
    for (int i = 0; i < kTiles * kVStages; ++i) mbar_init(bar(kBarVEmpty + i), 1);
    for (int t = 0; t < kTiles; ++t) mbar_init(bar(kBarDone + t), 1);
    for (int i = 0; i < 5; ++i) mbar_init(bar(kBarTurn + i), 128);
    mbar_init(bar(kBarNever), 1);
    *abort = 0;
    *xabort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  cta_sync();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // Whole warpgroups move registers from the control roles to the softmax; each setmaxnreg sits
  // inside its role's branch, so the compiler allocates each branch for its own budget.
  if (warp < kSoftmaxWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (warp == 0 && lane == 0) {
    // ------------------------------ TMA producer ------------------------------------------
    tma_prefetch_desc(&tmq);
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
    // A ring stage (or Q slot) is refilled once every chain that read its previous contents has
    // released it. The chains that read each stage's current block (2 bits per stage: chain 0,
    // chain 1) and the parity each chain's empty barrier completes next (1 bit per chain and
    // stage) are kept here: every read of a stage by a chain completes one phase of that chain's
    // empty barrier of the stage, and the producer waits for them in order.
    uint32_t kread = 0, vread = 0, qread = 0;  // readers: 2 bits per stage / slot
    uint32_t kph = 0, vph = 0, qph = 0;        // next parity: bit chain * stages + stage / chain
    int nk = 0, nv = 0, nq0 = 0, nq1 = 0;  // K and V blocks and Q fills issued (for the drain)
    // Test hook (off unless the host enabled it): CTA 0 first waits on a barrier that nothing
    // signals, so its bounded wait runs out, records GQA_DEVERR_TIMEOUT and aborts the CTA before
    // any copy is issued; every other role then gives up through the abort flag.
    bool ok = !(a.expire_wait && blockIdx.x == 0) || wait_bar(bar(kBarNever), 0, abort, a.err);
    // wait for the readers `rd` (2 bits) of a stage on their empty barriers empty0 + chain * n + s
    auto release = [&](uint32_t rd, uint32_t& ph, int empty0, int n, int s) {
      for (int c = 0; c < kTiles; ++c) {
        if (!((rd >> c) & 1u)) continue;
        const int bit = c * n + s;
        if (!wait_bar(bar(empty0 + c * n + s), (ph >> bit) & 1u, abort, a.err)) return false;
        ph ^= 1u << bit;
      }
      return true;
    };
    Seq sq = {};
    for (int it = 0; ok && (!kSplit || it < 1); ++it) {  // split mode: one item per CTA
      const long long item = item_of(it);
      if (item >= a.n_items) break;
      const Work w = make_work(a, (int)item);
      const Seq s0 = sq;
      advance(sq, w);
      if (!w.valid) set_device_error(a.err, w.kv < 1 || w.kv > a.T_max ? GQA_DEVERR_KV_LEN
                                                                        : GQA_DEVERR_POSITION);
      else if (w.nb[0] == 0) set_device_error(a.err, GQA_DEVERR_NO_VISIBLE);
      // the Q rows of every chain that runs (split mode: the one tile both chains read)
      const int zq = w.b * a.h_q + w.g * a.r + w.hb * a.H;  // first head of the block
#pragma unroll
      for (int q = 0; q < (kSplit ? 1 : kTiles); ++q) {
        if (!ok) break;
        const uint32_t rd = kSplit ? (w.nb[0] > 0 ? 1u : 0u) | (w.nb[1] > 0 ? 2u : 0u)
                                   : (q < w.nq && w.nb[q] > 0 ? 1u << q : 0u);
        if (!rd) continue;
        uint32_t prev = (qread >> (2 * q)) & 3u;
        if (!(ok = release(prev, qph, kBarQEmpty, 1, 0))) break;
        qread = (qread & ~(3u << (2 * q))) | (rd << (2 * q));
        mbar_arrive_expect_tx(bar(kBarQ + q), (uint32_t)(C::kNch * a.H * a.P * 128));
        for (int ch = 0; ch < C::kNch; ++ch)
          tma_load_3d(sQ + q * C::kQBytes + ch * C::kQChunk, &tmq, bar(kBarQ + q), ch * 64,
                      w.q0 + q * a.P, zq);
        if (q == 0) ++nq0; else ++nq1;
      }
      const int row0 = (w.b * a.h_kv + w.g) * a.T_max;
      for (int j = 0; j < w.nbmax && ok; ++j) {
        const int jg = s0.J + j;  // block count over the CTA's items
        // chains that release block j: split mode chain j % 2 (its reader); pair mode both, a chain
        // that does not read it (past its tile's last key, or no tile) releasing it unread, so that
        // each chain sees every fill of every stage in order
        const uint32_t rd = kSplit ? 1u << (j & 1) : 3u;
        const int ks = jg % kKStages;
        if (!(ok = release((kread >> (2 * ks)) & 3u, kph, kBarKEmpty, kKStages, ks))) break;
        kread = (kread & ~(3u << (2 * ks))) | (rd << (2 * ks));
        mbar_arrive_expect_tx(bar(kBarKFull + ks), C::kKVBytes);
        for (int ch = 0; ch < C::kNch; ++ch)
          tma_load_2d(sK + ks * C::kKVBytes + ch * C::kKVChunk, &tmk, bar(kBarKFull + ks), ch * 64,
                      row0 + (w.j0 + j) * kBN);
        ++nk;
        const int vs = jg % kVStages;
        if (!(ok = release((vread >> (2 * vs)) & 3u, vph, kBarVEmpty, kVStages, vs))) break;
        vread = (vread & ~(3u << (2 * vs))) | (rd << (2 * vs));
        mbar_arrive_expect_tx(bar(kBarVFull + vs), C::kKVBytes);
        for (int ch = 0; ch < C::kNch; ++ch)
          tma_load_2d(sV + vs * C::kKVBytes + ch * C::kKVChunk, &tmv, bar(kBarVFull + vs), ch * 64,
                      row0 + (w.j0 + j) * kBN);
        ++nv;
      }
    }
    // Drain (bounded, whatever the abort state): no copy may still be landing in shared memory
    // when the CTA exits.
    volatile int no_abort = 0;
    // the last fill of each stage or slot: fill f completes phase f, and blocks 0 .. n - 1 put
    // (n - 1 - s) / stages + 1 fills into stage s
    if (nq0 > 0) wait_bar(bar(kBarQ + 0), (uint32_t)((nq0 - 1) & 1), &no_abort, a.err);
    if (nq1 > 0) wait_bar(bar(kBarQ + 1), (uint32_t)((nq1 - 1) & 1), &no_abort, a.err);
#pragma unroll
    for (int s = 0; s < kKStages; ++s)
      if (nk > s) wait_bar(bar(kBarKFull + s), (uint32_t)(((nk - 1 - s) / kKStages) & 1), &no_abort, a.err);
#pragma unroll
    for (int s = 0; s < kVStages; ++s)
      if (nv > s) wait_bar(bar(kBarVFull + s), (uint32_t)(((nv - 1 - s) / kVStages) & 1), &no_abort, a.err);
    } else if (warp == 1 || warp == 2) {
      // ------------------------------ MMA issuer of tile t ----------------------------------
      mma_role<D, kSplit>(a, warp - 1, tmem, sQ, sK, sV, bars, abort);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int t = (warp - kSoftmaxWarp0) >> 2;
    float* xm = reinterpret_cast<float*>(smem + C::kOffQ + C::kQBytes);  // second Q tile (split mode)
    softmax_role<D, kWin, kSplit>(a, t, warp & 3, lane, tmem, sV, bars, xm, xabort, abort);
  }

  tc::fence_before_sync();
  cta_sync();
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
  const long long items = (long long)(p.split ? n_qt : p.n_pairs) * units;
  if (items <= 0) return cudaSuccess;
  if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  p.n_items = (int)items;
  p.div_per = FastDiv::make((uint32_t)units);
  p.div_gh = FastDiv::make((uint32_t)(a.h_kv * p.hblocks));
  p.div_hb = FastDiv::make((uint32_t)p.hblocks);
  // pair mode: one persistent CTA per SM (it holds all 512 TMEM columns), or one per item when
  // fewer; split mode (chosen when the items barely fill the SMs): one CTA per item
  const long long ctas = p.split || items < num_sms ? items : num_sms;
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
