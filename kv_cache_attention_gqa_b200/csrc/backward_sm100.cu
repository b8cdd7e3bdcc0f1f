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
// Two launches: rowterm, then one persistent grid (one CTA per SM) whose CTAs take work items in
// the order dkdv tiles (heaviest first), then dq tiles (heaviest first): item c for CTA c, then
// items from a ticket counter that rowterm resets, so an SM that finishes early takes the next
// item, as the hardware's CTA scheduler would, without a CTA exit and launch per item (measured:
// the 512-column TMEM release of an exiting CTA took 3.5-5 us after these kernels' epilogues).
// Each dkdv item initialises its barriers and invalidates them at its end; once a CTA draws a dq
// tile, every later ticket is a dq tile too, and it runs them as one pipelined sequence (the next
// tile's loads and first scores overlap the current tile's dQ write-out).
//   rowterm   one warp per query row: D = rowsum(dO * O) and the base-2 lse (fp32 workspace).
//   dkdv      one CTA per (sequence, KV head, 128-key block). The keys sit on the 128 TMEM lanes;
//             the CTA walks every 64-row query block of every head of the group, so the r heads'
//             shares of dK and dV add up in TMEM (no atomics):
//               S^T  = K Q^T     tcgen05.mma, A = K and B = Q from shared memory (K-major)
//               dP^T = V dO^T    A = V, B = dO from shared memory
//               (8 warps: two per TMEM lane quarter, one per 32-column half of the block)
//               P^T = 2^(S^T c - lse2), dS^T = P^T (dP^T - D) -> bf16 into TMEM
//               dV  += P^T dO    A = P^T from TMEM, B = dO (MN-major view of the same tile)
//               dK  += dS^T Q    A = dS^T from TMEM, B = Q (MN-major)
//   dq        one CTA per forward tile (H heads x P positions of one group), walking the 64-key
//             K/V blocks the tile sees:
//               S = Q K^T, dP = dO V^T (A = the tile's Q / dO rows, copied once into TMEM;
//               B = K / V from shared memory), then dS -> bf16 into TMEM, dQ += dS K (A = dS from
//               TMEM, B = K, MN-major view).
// Masks: on blocks that straddle the diagonal, the window or the length, each elementwise thread
// compares indices with one pair of 32-bit bounds fixed for the block: the query columns that see
// its key (dkdv) or the keys its row sees (dq).
// TMEM (512 columns): S double-buffered at [0,64) and [64,128), dP at [128,192) and [192,256),
// accumulators from 256; P / dS (bf16 pairs) are written over the first columns of the scores
// they come from. MMAs issued by one thread execute in order, so a buffer is rewritten only
// after the accumulating MMAs have read its P / dS, and the next block's scores overlap the
// current block's elementwise pass.
//
// Every tcgen05.ld/st/wait sits behind warp-uniform conditions; every mbarrier wait is bounded
// (2 s of %globaltimer) and sets GQA_DEVERR_TIMEOUT instead of hanging.

#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace gqa {
namespace bw {

constexpr int kBK = 128;  // keys of a dkdv CTA (one per TMEM lane)
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kColAcc0 = 256;  // first accumulator column (scores and their bf16 P / dS use [0, 256))

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
  FastDiv div_per, div_gh, div_hb;  // by B*h_kv*hblocks, h_kv*hblocks, hblocks (dq tile numbers)
  int n_items;              // dkdv tiles + dq tiles
  int* ticket;              // items handed out past the first gridDim.x (reset by rowterm)
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

// Packed fp32x2 arithmetic (sm_100): two lanes of work per instruction in the elementwise passes.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
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
                                                      float* lse2, float* drow, long long rows, int D,
                                                      int* ticket) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (ticket && blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0;  // for the next kernel's items
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

// The same for bf16 rows of D = 64 or 128 elements with 16-byte aligned bases: D / 8 lanes per
// row each load 16 bytes of O and of dO, so a warp covers 32 / (D / 8) rows. (One warp per row
// with 2-byte loads ran at under half the DRAM bandwidth that reading O and dO needs.)
template <int D>
__global__ void __launch_bounds__(256) rowterm_vec_kernel(const __nv_bfloat16* o, const __nv_bfloat16* d_o,
                                                          const float* lse, float* lse2, float* drow,
                                                          long long rows, int* ticket) {
  constexpr int kLpr = D / 8;       // lanes per row
  constexpr int kRpw = 32 / kLpr;   // rows per warp
  const int lane = threadIdx.x & 31;
  if (ticket && blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0;  // for the next kernel's items
  const long long row = (((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * kRpw + lane / kLpr;
  const int sub = lane % kLpr;
  float s = 0.f;
  if (row < rows) {
    const uint4 av = __ldg(reinterpret_cast<const uint4*>(o + row * D) + sub);
    const uint4 bv = __ldg(reinterpret_cast<const uint4*>(d_o + row * D) + sub);
    const uint32_t aw[4] = {av.x, av.y, av.z, av.w}, bw_[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[i]));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw_[i]));
      s = fmaf(fa.x, fb.x, s);
      s = fmaf(fa.y, fb.y, s);
    }
  }
#pragma unroll
  for (int off = kLpr / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (sub == 0 && row < rows) {
    drow[row] = s;
    const float l = lse[row];
    lse2[row] = l == -INFINITY || l != l ? INFINITY : l * kLog2e;
  }
}

// Descriptors for tiles of any row count: `chunk` is the byte stride between 64-column chunks
// (rows x 128 B).
__device__ __forceinline__ uint64_t desc_k(uint32_t tile, int k, uint32_t chunk) {
  return tc::smem_desc(tile + (uint32_t)((k >> 2) * chunk + (k & 3) * 32), 16, 1024);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t tile, int kk, uint32_t chunk) {
  return tc::smem_desc(tile + (uint32_t)(kk * 2048), chunk, 1024);
}
using tc::elect_one;
using tc::koff;
using tc::mnoff;

// ---- dkdv: key-stationary dK / dV -------------------------------------------------------------
// Query blocks of 64 rows, so S^T and dP^T are double-buffered in TMEM next to the dV / dK
// accumulators: the MMA warp issues block i+1's S^T / dP^T while eight warps (two per TMEM lane
// quarter, one per 32-query half) turn block i into P^T / dS^T. Each half writes its bf16 pairs
// over the first 16 columns of its own 32, so the halves never touch each other's columns; the
// accumulating MMAs address their A operand per 16-query step accordingly.
// TMEM: S^T[buf] at 64 buf, dP^T[buf] at 128 + 64 buf, dV at 256, dK at 256 + D.
constexpr int kKvBQ = 64;
constexpr int kKvStages = 3;
constexpr int kKvThreads = 320;  // warp 0 TMA + statistics, warp 1 MMA, warps 2-9 elementwise
template <int D>
struct KvCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kKTile = kNch * 128 * 128;     // K or V: 128 rows
  static constexpr int kQChunk = kKvBQ * 128;         // 64 rows x 128 B
  static constexpr int kQTile = kNch * kQChunk;       // Q or dO: 64 rows
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kKTile;
  static constexpr int kOffQ = 2 * kKTile;                        // + stage * 2 * kQTile
  static constexpr int kOffStat = kOffQ + kKvStages * 2 * kQTile;  // stages x (lse2[64], D[64])
  static constexpr int kOffBar = kOffStat + kKvStages * 2 * kKvBQ * 4;
  static constexpr int kSmem = (kOffBar + 256 + 1024) > 120 * 1024 ? kOffBar + 256 + 1024 : 120 * 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};
enum {
  kKvFull = 0,
  kQFull = 1,                    // + stage (3): TMA bytes + the producer warp's 32 stat arrivals
  kQEmpty = kQFull + kKvStages,  // + stage
  kKvS = kQEmpty + kKvStages,    // + buffer (2): S^T, dP^T of a block are in TMEM
  kKvP = kKvS + 2,               // + buffer (2): P^T, dS^T of a block are in TMEM (256 arrivals)
  kKvDone = kKvP + 2,
  kKvBars = kKvDone + 1
};

// One CTA of the dK / dV pass for tile `tile` (sequence, KV head, key block).
template <int D>
__device__ __forceinline__ void dkdv_cta(const CUtensorMap& tmq, const CUtensorMap& tmdo,
                                         const CUtensorMap& tmk, const CUtensorMap& tmv, const BArgs& a,
                                         int tile, uint32_t tmem) {
  using C = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  // the abort flag sits after the barriers (the TMEM address is the kernel's, held across items)
  volatile int* abort = reinterpret_cast<volatile int*>(bars + kKvBars) + 1;
  float* stat = reinterpret_cast<float*>(smem + C::kOffStat);  // [stage][lse2 64 | D 64]
  const uint32_t sK = smem_u32(smem + C::kOffK), sV = smem_u32(smem + C::kOffV);
  auto sQ = [&](int st) { return smem_u32(smem + C::kOffQ + st * 2 * C::kQTile); };
  auto sDO = [&](int st) { return smem_u32(smem + C::kOffQ + st * 2 * C::kQTile + C::kQTile); };
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- this CTA's keys and the query blocks that see them
  const int per = a.B * a.h_kv;
  const int kb = tile / per;
  const int b = (tile - kb * per) / a.h_kv;
  const int g = tile - kb * per - b * a.h_kv;
  const int k0 = kb * kBK;
  const int kv = a.kv_len ? a.kv_len[b] : a.T_max;
  const int qs = a.q_start ? a.q_start[b] : 0;
  const bool valid = kv >= 1 && kv <= a.T_max && qs >= 0;
  const int n_qb = (a.S_q + kKvBQ - 1) / kKvBQ;
  int qb_lo = 0, qb_hi = -1;
  if (valid && k0 < kv) {
    qb_hi = n_qb - 1;
    if (a.causal) {
      const long long first_q = (long long)k0 - qs;  // earliest row that can see key k0
      qb_lo = first_q > 0 ? (int)(first_q / kKvBQ) : 0;
      if (a.window > 0) {
        const long long k_last = min(k0 + kBK, kv) - 1;
        const long long last_q = k_last + a.window - 1 - qs;  // latest row that can see k_last
        qb_hi = last_q < 0 ? -1 : (int)min((long long)qb_hi, last_q / kKvBQ);
      }
    }
  }
  const int nq = qb_hi >= qb_lo ? qb_hi - qb_lo + 1 : 0;
  const int n_it = nq * a.r;  // (head, query block) pairs

  if (threadIdx.x == 0) {
    mbar_init(bar(kKvFull), 1);
    for (int st = 0; st < kKvStages; ++st) {
      mbar_init(bar(kQFull + st), 1 + 32);
      mbar_init(bar(kQEmpty + st), 1);
    }
    for (int bf = 0; bf < 2; ++bf) {
      mbar_init(bar(kKvS + bf), 1);
      mbar_init(bar(kKvP + bf), 256);
    }
    mbar_init(bar(kKvDone), 1);
    *abort = 0;
    fence_barrier_init();
    if (!valid && kb == 0 && g == 0)
      set_device_error(a.err, kv < 1 || kv > a.T_max ? GQA_DEVERR_KV_LEN : GQA_DEVERR_POSITION);
  }
  tc::fence_before_sync();
  cta_sync();
  tc::fence_after_sync();
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
      mbar_arrive_expect_tx(bar(kKvFull), 2 * C::kKTile);
      for (int ch = 0; ch < C::kNch; ++ch) {
        tma_load_2d(sK + ch * 128 * 128, &tmk, bar(kKvFull), ch * 64, krow);
        tma_load_2d(sV + ch * 128 * 128, &tmv, bar(kKvFull), ch * 64, krow);
      }
    }
    int last[kKvStages];
    for (int st = 0; st < kKvStages; ++st) last[st] = -1;
    for (int it = 0; it < n_it; ++it) {
      const int st = it % kKvStages, n = it / kKvStages;
      int ok = 1;
      if (n > 0 && lane == 0) ok = wait_bar(bar(kQEmpty + st), (uint32_t)((n - 1) & 1), abort, a.err);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int h = head_of(it), qb = qblk_of(it);
      const int z = b * a.h_q + h;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(kQFull + st), 2 * C::kQTile);
        for (int ch = 0; ch < C::kNch; ++ch) {
          tma_load_3d(sQ(st) + ch * C::kQChunk, &tmq, bar(kQFull + st), ch * 64, qb * kKvBQ, z);
          tma_load_3d(sDO(st) + ch * C::kQChunk, &tmdo, bar(kQFull + st), ch * 64, qb * kKvBQ, z);
        }
      }
      float* sl = stat + st * 2 * kKvBQ;
#pragma unroll
      for (int e = 0; e < kKvBQ / 32; ++e) {
        const int c = lane * (kKvBQ / 32) + e;
        const int qi = qb * kKvBQ + c;
        const long long row = (long long)z * a.S_q + qi;
        sl[c] = qi < a.S_q ? -a.lse2[row] : -INFINITY;  // stored negated for the fused FMAs
        sl[kKvBQ + c] = qi < a.S_q ? -a.drow[row] : 0.f;
      }
      mbar_arrive(bar(kQFull + st));
      last[st] = n;
    }
    if (lane == 0) {  // drain (bounded): no copy may still land in shared memory at exit
      volatile int no_abort = 0;
      wait_bar(bar(kKvFull), 0, &no_abort, a.err);
      for (int st = 0; st < kKvStages; ++st)
        if (last[st] >= 0) wait_bar(bar(kQFull + st), (uint32_t)(last[st] & 1), &no_abort, a.err);
    }
  } else if (warp == 1 && n_it > 0) {
    // ------------------------------ MMA issuer ---------------------------------------------
    // The whole warp runs the loop (its state and the descriptors stay warp-uniform) and one
    // elected lane issues each batch of MMAs together with its commit. (One thread issuing with
    // descriptors built per MMA spent most of its time between MMAs, not in them.)
    constexpr uint32_t idesc_s = tc::idesc_bf16(128, kKvBQ, false);  // S^T, dP^T: M keys, N queries
    constexpr uint32_t idesc_acc = tc::idesc_bf16(128, D, true);     // dV, dK: M keys, N = d_h
    const uint64_t dK = tc::smem_desc(sK, 16, 1024), dV = tc::smem_desc(sV, 16, 1024);
    auto wait = [&](int b_, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_bar(bar(b_), parity, abort, a.err));
    };
    auto issue_s = [&](int it) {  // S^T and dP^T of block `it` into buffer it & 1
      const int st = it % kKvStages, bf = it & 1;
      const uint64_t dq = tc::smem_desc(sQ(st), 16, 1024), ddo = tc::smem_desc(sDO(st), 16, 1024);
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_ss(tmem + 64 * bf, dK + koff(k, 128 * 128), dq + koff(k, C::kQChunk), idesc_s, k > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_ss(tmem + 128 + 64 * bf, dV + koff(k, 128 * 128), ddo + koff(k, C::kQChunk), idesc_s,
                     k > 0 ? 1u : 0u);
        tc::commit(bar(kKvS + bf));
      }
      __syncwarp();
    };
    bool ok = wait(kKvFull, 0) && wait(kQFull, 0);
    if (ok) {
      tc::fence_after_sync();
      issue_s(0);
    }
    for (int it = 0; it < n_it && ok; ++it) {
      const int st = it % kKvStages, bf = it & 1;
      if (it + 1 < n_it) {  // next block's scores overlap this block's elementwise pass
        const int st1 = (it + 1) % kKvStages;
        if (!(ok = wait(kQFull + st1, (uint32_t)(((it + 1) / kKvStages) & 1)))) break;
        tc::fence_after_sync();
        issue_s(it + 1);
      }
      if (!(ok = wait(kKvP + bf, (uint32_t)((it >> 1) & 1)))) break;
      tc::fence_after_sync();
      const uint64_t ddo_mn = tc::smem_desc(sDO(st), C::kQChunk, 1024);
      const uint64_t dq_mn = tc::smem_desc(sQ(st), C::kQChunk, 1024);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kKvBQ / 16; ++kk) {
          const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
          const uint32_t acol = (uint32_t)(64 * bf + (kk >> 1) * 32 + (kk & 1) * 8);  // half kk/2
          tc::mma_ts(tmem + kColAcc0, tmem + acol, ddo_mn + mnoff(kk), idesc_acc, acc);
          tc::mma_ts(tmem + kColAcc0 + D, tmem + 128 + acol, dq_mn + mnoff(kk), idesc_acc, acc);
        }
        tc::commit(bar(kQEmpty + st));
      }
      __syncwarp();
    }
    if (elect_one()) tc::commit(bar(kKvDone));
    __syncwarp();
    volatile int no_abort = 0;
    wait_bar(bar(kKvDone), 0, &no_abort, a.err);
  } else if (warp >= 2) {
    // ------------------------------ elementwise: one key row, 32 queries per thread ---------
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;     // which 32 queries of each 64-query block
    const int row = quarter * 32 + lane;  // TMEM lane = key k0 + row
    const int key = k0 + row;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int st = it % kKvStages, bf = it & 1;
      if (ok) ok = wait_bar(bar(kKvS + bf), (uint32_t)((it >> 1) & 1), abort, a.err);
      if (ok) ok = wait_bar(bar(kQFull + st), (uint32_t)((it / kKvStages) & 1), abort, a.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const float* sl = stat + st * 2 * kKvBQ + half * 32;
      const int qb = qblk_of(it);
      const int col0 = qb * kKvBQ + half * 32;        // first query (index into S_q) of this half
      const long long pos0 = (long long)qs + col0;
      const bool need_mask = k0 + kBK > kv || col0 + 32 > a.S_q ||
                             (a.causal && (long long)k0 + kBK - 1 > pos0) ||
                             (a.window > 0 && (long long)k0 <= pos0 + 31 - a.window);
      tc::fence_after_sync();
      uint32_t sv[32], dv[32];
      tc::ld32(lane_addr + 64 * bf + 32 * half, sv);
      tc::ld32(lane_addr + 128 + 64 * bf + 32 * half, dv);
      tc::wait_ld();
      // query columns [c_lo, c_hi) of this half that see this key: rows at or past it (causal),
      // within its window, inside S_q; none when the key is past kv_len
      int c_lo = 0, c_hi = 32;
      if (need_mask) {
        const long long rel = (long long)key - pos0;  // column of the row at the key's position
        if (a.causal) c_lo = (int)(rel < 0 ? 0 : (rel > 32 ? 32 : rel));
        long long hi = a.S_q - col0 < 32 ? a.S_q - col0 : 32;
        if (a.window > 0 && rel + a.window < hi) hi = rel + a.window;
        c_hi = key < kv ? (int)(hi < 0 ? 0 : hi) : 0;
      }
      uint32_t pp[16], pd[16];
      const float2 c2 = make_float2(a.sl2, a.sl2);
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        const float2 nl = *reinterpret_cast<const float2*>(sl + x);          // -lse2 of the two rows
        const float2 nd = *reinterpret_cast<const float2*>(sl + kKvBQ + x);  // -D of the two rows
        const float2 arg = fma2(make_float2(__uint_as_float(sv[x]), __uint_as_float(sv[x + 1])), c2, nl);
        float2 p = make_float2(fast_exp2(arg.x), fast_exp2(arg.y));
        float2 ds = mul2(p, add2(make_float2(__uint_as_float(dv[x]), __uint_as_float(dv[x + 1])), nd));
        if (need_mask) {
          if (x < c_lo || x >= c_hi) p.x = ds.x = 0.f;
          if (x + 1 < c_lo || x + 1 >= c_hi) p.y = ds.y = 0.f;
        }
        pp[x / 2] = pack_bf16x2(p.x, p.y);
        pd[x / 2] = pack_bf16x2(ds.x, ds.y);
      }
      tc::st16(lane_addr + 64 * bf + 32 * half, pp);        // P^T over this half's first columns
      tc::st16(lane_addr + 128 + 64 * bf + 32 * half, pd);  // dS^T likewise in dP^T
      tc::wait_st();
      tc::fence_before_sync();
      mbar_arrive(bar(kKvP + bf));
    }
    // ---- epilogue: dV and scale * dK rows -> bf16; each half writes half of the columns
    bool have = n_it > 0 && ok;
    if (have) {
      have = wait_bar(bar(kKvDone), 0, abort, a.err);
      have = __all_sync(0xffffffffu, have);
      if (have) tc::fence_after_sync();
    }
    const long long orow = ((long long)b * a.h_kv + g) * a.T_max + key;
    uint4* dvo = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dv) + orow * D);
    uint4* dko = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dk) + orow * D);
    const bool store = key < a.T_max;
    if (!have) {
      if (store)
        for (int v = half * (D / 16); v < (half + 1) * (D / 16); ++v) {
          dvo[v] = make_uint4(0u, 0u, 0u, 0u);
          dko[v] = make_uint4(0u, 0u, 0u, 0u);
        }
    } else {
#pragma unroll 1
      for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {  // 32-column chunks
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
  // every role is done with the item (copies landed, MMAs complete, TMEM read): its barriers go
  tc::fence_before_sync();
  cta_sync();
  if (threadIdx.x == 0)
    for (int i = 0; i < kKvBars; ++i) mbar_inval(bar(i));
}

// ---- dq: query-stationary dQ on the forward's tiles -------------------------------------------
// K/V blocks of 64 keys, so S and dP are double-buffered in TMEM next to the dQ accumulator: the
// MMA warp issues block j+1's S / dP while eight warps (two per lane quarter, one per 32-key half)
// turn block j into dS. The tile's Q and dO rows are copied into TMEM once and are the A operands
// of S = Q K^T and dP = dO V^T, so those MMAs read only K / V from shared memory.
// TMEM: S[buf] at 64 buf, dP[buf] at 128 + 64 buf, dQ at 256, Q at 256 + D, dO at 256 + 3D/2.
constexpr int kQBK = 64;
constexpr int kQStages = 3;
constexpr int kQThreads = 320;
template <int D>
struct QCfg {
  static constexpr int kNch = D / 64;
  static constexpr int kQTile = kNch * 128 * 128;  // Q or dO: 128 rows
  static constexpr int kKChunk = kQBK * 128;       // 64 rows x 128 B
  static constexpr int kKTile = kNch * kKChunk;    // K or V: 64 rows
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kQTile;
  static constexpr int kOffK = 2 * kQTile;  // + stage * 2 * kKTile (K, then V)
  static constexpr int kOffBar = kOffK + kQStages * 2 * kKTile;
  static constexpr int kSmem = (kOffBar + 256 + 1024) > 120 * 1024 ? kOffBar + 256 + 1024 : 120 * 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};
enum {
  kQdQ = 0,                            // Q / dO of a tile in shared memory (or the end)
  kQT = 1,                             // Q, dO copied into TMEM (256 arrivals)
  kQKvFull = 2,                        // + stage
  kQKvEmpty = kQKvFull + kQStages,     // + stage
  kQS = kQKvEmpty + kQStages,          // + buffer
  kQP = kQS + 2,                       // + buffer (256 arrivals)
  kQDone = kQP + 2,                    // a tile's dQ MMAs complete
  kQdQEmpty = kQDone + 1,              // Q / dO copied into TMEM and the tile number read (257)
  kQAll = kQdQEmpty + 1,               // every MMA of the run complete
  kQBars = kQAll + 1
};

// One dQ tile (as in the forward): H heads x P positions of one group, and the 64-key blocks
// j0 .. j0 + nb - 1 its rows see.
struct DqTile {
  int b, g, hb, q0, nh, kv, qs, j0, nb;
  long long pos_min, pos_max;
};

__device__ __forceinline__ DqTile dq_tile(const BArgs& a, int tile) {
  DqTile t;
  const int per = a.B * a.h_kv * a.hblocks;
  const int qd = a.div_per.div(tile);
  const int qt = a.n_qt - 1 - qd;  // heaviest (latest positions) first
  const int rem = tile - qd * per;
  t.b = a.div_gh.div(rem);
  const int gh = rem - t.b * (a.h_kv * a.hblocks);
  t.g = a.div_hb.div(gh);
  t.hb = gh - t.g * a.hblocks;
  t.q0 = qt * a.P;
  t.nh = min(a.H, a.r - t.hb * a.H);
  t.kv = a.kv_len ? a.kv_len[t.b] : a.T_max;
  t.qs = a.q_start ? a.q_start[t.b] : 0;
  const bool valid = t.kv >= 1 && t.kv <= a.T_max && t.qs >= 0;
  t.pos_min = (long long)t.qs + t.q0;
  t.pos_max = (long long)t.qs + min(t.q0 + a.P, a.S_q) - 1;
  t.j0 = 0;
  t.nb = 0;
  if (valid) {
    int end = (t.kv + kQBK - 1) / kQBK;
    if (a.causal) {
      const long long last_key = t.pos_max < t.kv - 1 ? t.pos_max : (long long)(t.kv - 1);
      end = (int)(last_key / kQBK) + 1;
      if (a.window > 0) {
        const long long lo = t.pos_min - a.window + 1;
        if (lo > 0) t.j0 = (int)(lo / kQBK);
      }
    }
    t.nb = end > t.j0 ? end - t.j0 : 0;
  }
  return t;
}

// The dQ pass from item `item0` on: every item after the first dQ tile is a dQ tile, so the CTA
// takes them all here from the work counter, with its pipelines running on from one tile into the
// next. The producer loads a tile's Q and dO rows as soon as the elementwise warps have copied the
// previous tile's into TMEM (that copy follows the previous tile's last S / dP, the MMAs that read
// them), and its K/V blocks through the ring; the MMA warp issues the new tile's first S and dP
// while the elementwise warps write out the previous tile's dQ; the new tile's first dQ += dS K,
// which overwrites the accumulator, waits for dS that those warps produce after reading it out.
// The producer hands each tile's number to the other roles through `s_items` (two slots), and a
// number past the last item ends the run.
template <int D>
__device__ __forceinline__ void dq_run(const CUtensorMap& tmq, const CUtensorMap& tmdo,
                                       const CUtensorMap& tmk, const CUtensorMap& tmv, const BArgs& a,
                                       int item0, int n_dkdv, uint32_t tmem, volatile int* s_items) {
  using C = QCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  volatile int* abort = reinterpret_cast<volatile int*>(bars + kQBars) + 1;  // after the barriers
  const uint32_t sQ = smem_u32(smem + C::kOffQ), sDO = smem_u32(smem + C::kOffDO);
  auto sK = [&](int st) { return smem_u32(smem + C::kOffK + st * 2 * C::kKTile); };
  auto sV = [&](int st) { return smem_u32(smem + C::kOffK + st * 2 * C::kKTile + C::kKTile); };
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(kQdQ), 1);
    mbar_init(bar(kQdQEmpty), 256 + 1);  // the elementwise threads and the MMA warp's lane
    mbar_init(bar(kQT), 256);
    for (int st = 0; st < kQStages; ++st) {
      mbar_init(bar(kQKvFull + st), 1);
      mbar_init(bar(kQKvEmpty + st), 1);
    }
    for (int bf = 0; bf < 2; ++bf) {
      mbar_init(bar(kQS + bf), 1);
      mbar_init(bar(kQP + bf), 256);
    }
    mbar_init(bar(kQDone), 1);
    mbar_init(bar(kQAll), 1);
    *abort = 0;
    fence_barrier_init();
  }
  tc::fence_before_sync();
  cta_sync();
  tc::fence_after_sync();

  // the tile number of the run's n-th item, or -1 at the end (after its Q/dO barrier phase n)
  auto item_at = [&](int n) { return s_items[n & 1]; };

  if (warp == 0 && lane == 0) {
    // ------------------------------ TMA producer ------------------------------------------
    tma_prefetch_desc(&tmq);
    tma_prefetch_desc(&tmdo);
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
    int item = item0, n = 0, J = 0, nk = 0;  // J: K/V blocks loaded (nk: issued, for the drain)
    bool ok = true;
    while (ok) {
      // the slot of item n held item n - 2; item n - 1's Q/dO rows are in TMEM and its number
      // has been read
      if (n > 0 && !(ok = wait_bar(bar(kQdQEmpty), (uint32_t)((n - 1) & 1), abort, a.err))) break;
      if (item >= a.n_items) {
        s_items[n & 1] = -1;
        mbar_arrive(bar(kQdQ));  // completes phase n with no bytes: the end
        break;
      }
      const int tile = item - n_dkdv;
      const DqTile t = dq_tile(a, tile);
      s_items[n & 1] = tile;
      const int next = (int)gridDim.x + atomicAdd(a.ticket, 1);  // the next item, fetched early
      const int zq = t.b * a.h_q + t.g * a.r + t.hb * a.H;
      mbar_arrive_expect_tx(bar(kQdQ), (uint32_t)(2 * C::kNch * a.H * a.P * 128));
      for (int ch = 0; ch < C::kNch; ++ch) {
        tma_load_3d(sQ + ch * 128 * 128, &tmq, bar(kQdQ), ch * 64, t.q0, zq);
        tma_load_3d(sDO + ch * 128 * 128, &tmdo, bar(kQdQ), ch * 64, t.q0, zq);
      }
      const int row0 = (t.b * a.h_kv + t.g) * a.T_max;
      for (int j = 0; j < t.nb && ok; ++j) {
        const int jg = J + j, st = jg % kQStages, f = jg / kQStages;
        if (f > 0 && !(ok = wait_bar(bar(kQKvEmpty + st), (uint32_t)((f - 1) & 1), abort, a.err))) break;
        mbar_arrive_expect_tx(bar(kQKvFull + st), 2 * C::kKTile);
        for (int ch = 0; ch < C::kNch; ++ch) {
          tma_load_2d(sK(st) + ch * C::kKChunk, &tmk, bar(kQKvFull + st), ch * 64, row0 + (t.j0 + j) * kQBK);
          tma_load_2d(sV(st) + ch * C::kKChunk, &tmv, bar(kQKvFull + st), ch * 64, row0 + (t.j0 + j) * kQBK);
        }
        ++nk;
      }
      J += t.nb;
      ++n;
      item = next;
    }
    // Drain (bounded): no copy may still land in shared memory when the run ends. The Q/dO rows
    // of every item were copied into TMEM before the end (or the run gave up); the K/V fills:
    volatile int no_abort = 0;
    if (!ok && n > 0) wait_bar(bar(kQdQ), (uint32_t)((n - 1) & 1), &no_abort, a.err);
#pragma unroll
    for (int s = 0; s < kQStages; ++s)
      if (nk > s) wait_bar(bar(kQKvFull + s), (uint32_t)(((nk - 1 - s) / kQStages) & 1), &no_abort, a.err);
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ---------------------------------------------
    constexpr uint32_t idesc_s = tc::idesc_bf16(128, kQBK, false);  // S, dP: M rows, N keys
    constexpr uint32_t idesc_acc = tc::idesc_bf16(128, D, true);    // dQ: M rows, N = d_h
    constexpr uint32_t kColQ = kColAcc0 + D, kColDO = kColAcc0 + D + D / 2;
    auto wait = [&](int b_, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_bar(bar(b_), parity, abort, a.err));
    };
    auto issue_s = [&](int jg) {  // the run's block jg: K/V stage jg % 3 into score buffer jg & 1
      const int st = jg % kQStages, bf = jg & 1;
      const uint64_t dk = tc::smem_desc(sK(st), 16, 1024), dv = tc::smem_desc(sV(st), 16, 1024);
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_ts(tmem + 64 * bf, tmem + kColQ + k * 8, dk + koff(k, C::kKChunk), idesc_s, k > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          tc::mma_ts(tmem + 128 + 64 * bf, tmem + kColDO + k * 8, dv + koff(k, C::kKChunk), idesc_s, k > 0 ? 1u : 0u);
        tc::commit(bar(kQS + bf));
      }
      __syncwarp();
    };
    int n = 0, J = 0;  // items, K/V blocks (= score blocks) so far
    bool ok = true;
    while (ok) {
      if (!(ok = wait(kQdQ, (uint32_t)(n & 1)))) break;
      const int tile = item_at(n);
      if (tile < 0) break;
      const DqTile t = dq_tile(a, tile);
      // this tile's Q and dO in TMEM; only then is the release below allowed: it lets the
      // elementwise warps reach the next tile's copy, and this warp must not be two phases of
      // kQT behind when they do
      if (!(ok = wait(kQT, (uint32_t)(n & 1)))) break;
      if (elect_one()) mbar_arrive(bar(kQdQEmpty));
      __syncwarp();
      if (t.nb > 0) {
        if (!(ok = wait(kQKvFull + J % kQStages, (uint32_t)((J / kQStages) & 1)))) break;
        tc::fence_after_sync();
        issue_s(J);
        for (int j = 0; j < t.nb && ok; ++j) {
          const int jg = J + j, st = jg % kQStages, bf = jg & 1;
          if (j + 1 < t.nb) {
            const int jn = jg + 1;
            if (!(ok = wait(kQKvFull + jn % kQStages, (uint32_t)((jn / kQStages) & 1)))) break;
            tc::fence_after_sync();
            issue_s(jn);
          }
          if (!(ok = wait(kQP + bf, (uint32_t)((jg >> 1) & 1)))) break;
          tc::fence_after_sync();
          const uint64_t dk_mn = tc::smem_desc(sK(st), C::kKChunk, 1024);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < kQBK / 16; ++kk)
              tc::mma_ts(tmem + kColAcc0, tmem + (uint32_t)(64 * bf + (kk >> 1) * 32 + (kk & 1) * 8),
                         dk_mn + mnoff(kk), idesc_acc, (j > 0 || kk > 0) ? 1u : 0u);
            tc::commit(bar(kQKvEmpty + st));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) tc::commit(bar(kQDone));  // this tile's dQ is complete
        __syncwarp();
      }
      J += t.nb;
      ++n;
    }
    // every MMA issued above has completed before the run ends
    if (elect_one()) tc::commit(bar(kQAll));
    __syncwarp();
    volatile int no_abort = 0;
    wait_bar(bar(kQAll), 0, &no_abort, a.err);
  } else if (warp >= 2) {
    // ------------------------------ elementwise: one query row, 32 keys per thread ----------
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;     // which 32 keys of each 64-key block
    const int et = (warp - 2) * 32 + lane;  // 0..255, for the K-row zeroing
    const int row = quarter * 32 + lane;  // TMEM lane = tile row (head h, position p)
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const int h = row / a.P, p = row - h * a.P;
    // dQ of the previous tile -> bf16 rows (or zeros when it had no block or gave up)
    auto epilogue = [&](bool have, long long srow, bool store_row) {
      uint4* out = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dq) + srow * D);
      if (have) {
#pragma unroll 1
        for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
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
        for (int v = half * (D / 16); v < (half + 1) * (D / 16); ++v) out[v] = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    int n = 0, J = 0, nd = 0;  // items, K/V blocks, items whose dQ the MMA warp completed
    bool ok = true;
    bool prev = false, prev_blocks = false, prev_store = false;  // the previous tile's epilogue
    long long prev_srow = 0;
    while (true) {
      if (ok) ok = wait_bar(bar(kQdQ), (uint32_t)(n & 1), abort, a.err);
      ok = __all_sync(0xffffffffu, ok);
      const int tile = ok ? item_at(n) : -1;
      if (tile < 0) break;
      const DqTile t = dq_tile(a, tile);
      const int qi = t.q0 + p;
      const bool store_row = h < t.nh && row < a.H * a.P && qi < a.S_q;
      const long long srow = ((long long)t.b * a.h_q + t.g * a.r + t.hb * a.H + h) * a.S_q + qi;
      const long long pos = (long long)t.qs + qi;
      const float lse2 = store_row ? a.lse2[srow] : INFINITY;
      const float dr = store_row ? a.drow[srow] : 0.f;
      // keys [k_first, k_last] this row sees (length, causal and window limits as 32-bit bounds)
      const long long kl = a.causal && pos < t.kv - 1 ? pos : (long long)t.kv - 1;
      const int k_last = (int)kl;
      const long long kf = a.window > 0 ? pos - a.window + 1 : 0;
      const int k_first = kf < 0 ? 0 : (kf > 0x7fffffffLL ? 0x7fffffff : (int)kf);
      // this row of Q (half 0) or dO (half 1): shared memory (128-byte swizzled) -> TMEM. The
      // previous tile's S and dP MMAs, which read these columns, are complete (this warp saw the
      // scores of its last block).
      {
        const uint32_t src = half == 0 ? sQ : sDO;
        const uint32_t dst = lane_addr + kColAcc0 + D + half * (D / 2);
#pragma unroll
        for (int ch = 0; ch < C::kNch; ++ch) {
          uint32_t r[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t addr = swz128(src + ch * 128 * 128, row, k);
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(r[4 * k]), "=r"(r[4 * k + 1]), "=r"(r[4 * k + 2]), "=r"(r[4 * k + 3])
                         : "r"(addr));
          }
          tc::st32(dst + ch * 32, r);
        }
        tc::wait_st();
      }
      tc::fence_before_sync();
      mbar_arrive(bar(kQT));
      mbar_arrive(bar(kQdQEmpty));
      // the previous tile's dQ (the MMA warp can start this tile's scores meanwhile)
      if (prev) {
        bool have = prev_blocks && ok;
        if (have) {
          have = wait_bar(bar(kQDone), (uint32_t)((nd - 1) & 1), abort, a.err);
          have = __all_sync(0xffffffffu, have);
          if (have) tc::fence_after_sync();
          else ok = false;
        }
        epilogue(have, prev_srow, prev_store);
      }
      for (int j = 0; j < t.nb; ++j) {
        const int jg = J + j, st = jg % kQStages, bf = jg & 1;
        if (ok) ok = wait_bar(bar(kQS + bf), (uint32_t)((jg >> 1) & 1), abort, a.err);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const int blk0 = (t.j0 + j) * kQBK;
        const int key0 = blk0 + half * 32;  // first key of this half
        const bool need_mask = (a.causal && (long long)key0 + 31 > t.pos_min) || key0 + 32 > t.kv ||
                               (a.window > 0 && (long long)key0 <= t.pos_max - a.window);
        tc::fence_after_sync();
        uint32_t sv[32], dv[32];
        tc::ld32(lane_addr + 64 * bf + 32 * half, sv);
        tc::ld32(lane_addr + 128 + 64 * bf + 32 * half, dv);
        tc::wait_ld();
        uint32_t pd[16];
        const float2 c2 = make_float2(a.sl2, a.sl2), nl = make_float2(-lse2, -lse2), nd2 = make_float2(-dr, -dr);
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float2 arg = fma2(make_float2(__uint_as_float(sv[x]), __uint_as_float(sv[x + 1])), c2, nl);
          const float2 pr = make_float2(fast_exp2(arg.x), fast_exp2(arg.y));
          float2 ds = mul2(pr, add2(make_float2(__uint_as_float(dv[x]), __uint_as_float(dv[x + 1])), nd2));
          if (need_mask) {
            if (key0 + x < k_first || key0 + x > k_last) ds.x = 0.f;
            if (key0 + x + 1 < k_first || key0 + x + 1 > k_last) ds.y = 0.f;
          }
          pd[x / 2] = pack_bf16x2(ds.x, ds.y);
        }
        tc::st16(lane_addr + 64 * bf + 32 * half, pd);  // dS over this half's first columns of S
        // K rows no row of the tile may see (past kv_len: last block; below every row's window:
        // first block) get dS = 0 but may hold anything: zero them before dQ += dS K
        const bool zero_tail = j == t.nb - 1 && blk0 + kQBK > t.kv;
        const bool zero_head = j == 0 && a.window > 0 && (long long)blk0 < t.pos_min - a.window + 1;
        if ((zero_tail || zero_head) && et < kQBK) {
          const long long key = (long long)blk0 + et;  // this thread's K row of the block
          if ((zero_tail && key >= t.kv) || (zero_head && key <= t.pos_min - a.window)) {
            for (int ch = 0; ch < C::kNch; ++ch)
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const uint32_t addr = sK(st) + ch * C::kKChunk + et * 128 + k * 16;
                asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
              }
          }
          tc::fence_proxy_async_smem();
        }
        tc::wait_st();
        tc::fence_before_sync();
        mbar_arrive(bar(kQP + bf));
      }
      prev = true;
      prev_blocks = t.nb > 0;
      prev_store = store_row;
      prev_srow = srow;
      if (t.nb > 0) ++nd;
      J += t.nb;
      ++n;
    }
    if (prev) {  // the last tile's dQ
      bool have = prev_blocks && ok;
      if (have) {
        have = wait_bar(bar(kQDone), (uint32_t)((nd - 1) & 1), abort, a.err);
        have = __all_sync(0xffffffffu, have);
        if (have) tc::fence_after_sync();
      }
      epilogue(have, prev_srow, prev_store);
    }
  }
  // every role is done (copies landed, MMAs complete, TMEM read): the barriers go
  tc::fence_before_sync();
  cta_sync();
  if (threadIdx.x == 0)
    for (int i = 0; i < kQBars; ++i) mbar_inval(bar(i));
}

// One launch for both passes: the first n_dkdv CTAs run the key-stationary dK / dV pass
// (heaviest key blocks first), the rest the query-stationary dQ pass, which fills the SMs the
// uneven dK / dV CTAs leave idle. Both use 320 threads, the larger of the two shared-memory sizes
// and their own 512 TMEM columns (one CTA per SM).
static_assert(kKvThreads == kQThreads, "one block size for both passes");
template <int D>
struct BwCfg {
  static constexpr int kSmem = KvCfg<D>::kSmem > QCfg<D>::kSmem ? KvCfg<D>::kSmem : QCfg<D>::kSmem;
};

template <int D>
__global__ void __launch_bounds__(kKvThreads, 1)
    backward_kernel(const __grid_constant__ CUtensorMap tmq_rows, const __grid_constant__ CUtensorMap tmdo_rows,
                    const __grid_constant__ CUtensorMap tmk128, const __grid_constant__ CUtensorMap tmv128,
                    const __grid_constant__ CUtensorMap tmq_tile, const __grid_constant__ CUtensorMap tmdo_tile,
                    const __grid_constant__ CUtensorMap tmk64, const __grid_constant__ CUtensorMap tmv64,
                    BArgs a, int n_dkdv) {
  __shared__ uint32_t s_tmem;
  __shared__ int s_next;
  __shared__ int s_items[2];
  const int warp = threadIdx.x >> 5;
  if (warp == 1) {  // all 512 columns, held across the CTA's items
    tc::tmem_alloc(smem_u32(&s_tmem), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  cta_sync();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  for (int item = blockIdx.x; item < a.n_items;) {
    if (item >= n_dkdv) {  // tickets only grow: every later item of this CTA is a dq tile too
      dq_run<D>(tmq_tile, tmdo_tile, tmk64, tmv64, a, item, n_dkdv, tmem, s_items);
      break;
    }
    // the next item's ticket, fetched while this item runs by a thread of the elementwise warps
    // (which wait for the first scores anyway); the item's closing barrier publishes it
    if (threadIdx.x == 64) s_next = (int)gridDim.x + atomicAdd(a.ticket, 1);
    dkdv_cta<D>(tmq_rows, tmdo_rows, tmk128, tmv128, a, item, tmem);
    item = s_next;
    cta_sync();  // every thread has read s_next before the next item writes it
  }
  tc::fence_before_sync();
  cta_sync();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_typed(const BArgs& p, const CUtensorMap* tm, int num_sms, cudaStream_t s) {
  static bool attr_set[64] = {false};  // per device: the shared-memory opt-in is set once
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(backward_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, BwCfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const long long n1 = (long long)p.n_kb * p.B * p.h_kv;
  const long long n2 = (long long)p.n_qt * p.B * p.h_kv * p.hblocks;
  if (n1 + n2 > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (n1 + n2 <= 0) return cudaSuccess;
  BArgs q = p;
  q.n_items = (int)(n1 + n2);
  const long long ctas = n1 + n2 < num_sms ? n1 + n2 : num_sms;  // one CTA per SM
  backward_kernel<D><<<(unsigned)ctas, kKvThreads, BwCfg<D>::kSmem, s>>>(
      tm[0], tm[1], tm[2], tm[3], tm[4], tm[5], tm[6], tm[7], q, (int)n1);
  return cudaGetLastError();
}

}  // namespace bw

cudaError_t launch_backward_bf16(const BackwardArgs& a, const CUtensorMap* tmaps, int num_sms,
                                 cudaStream_t s) {
  const long long rows = (long long)a.B * a.h_q * a.S_q;
  if (rows <= 0) return cudaSuccess;
  const auto* ob = reinterpret_cast<const __nv_bfloat16*>(a.o);
  const auto* dob = reinterpret_cast<const __nv_bfloat16*>(a.d_o);
  const bool vec = ((reinterpret_cast<uintptr_t>(a.o) | reinterpret_cast<uintptr_t>(a.d_o)) & 15u) == 0;
  if (vec && a.d_h == 128) {  // 2 rows per warp, 16 per block
    bw::rowterm_vec_kernel<128><<<(unsigned)((rows + 15) / 16), 256, 0, s>>>(ob, dob, a.lse, a.lse2, a.drow,
                                                                             rows, a.ticket);
  } else if (vec && a.d_h == 64) {  // 4 rows per warp, 32 per block
    bw::rowterm_vec_kernel<64><<<(unsigned)((rows + 31) / 32), 256, 0, s>>>(ob, dob, a.lse, a.lse2, a.drow,
                                                                            rows, a.ticket);
  } else {
    bw::rowterm_kernel<__nv_bfloat16><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(
        ob, dob, a.lse, a.lse2, a.drow, rows, a.d_h, a.ticket);
  }
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
  p.div_per = FastDiv::make((uint32_t)(a.B * a.h_kv * p.hblocks));
  p.div_gh = FastDiv::make((uint32_t)(a.h_kv * p.hblocks));
  p.div_hb = FastDiv::make((uint32_t)p.hblocks);
  p.scale = a.scale;
  p.sl2 = a.scale * bw::kLog2e;
  p.causal = a.causal;
  p.window = a.window;
  p.ticket = a.ticket;
  p.n_items = 0;
  p.err = a.err;
  if (a.d_h == 128) return bw::launch_typed<128>(p, tmaps, num_sms, s);
  if (a.d_h == 64) return bw::launch_typed<64>(p, tmaps, num_sms, s);
  return cudaErrorInvalidValue;
}

}  // namespace gqa
