// Split-KV decode: one new query per sequence attending over its cached K/V.
//
// Work decomposition. A "unit" is (sequence b, KV head g, head block hb): the r query heads that
// read KV head g [序列计算与存储, section 分组查询注意力: g(a) = floor(a / r)] are packed into one
// tile so each cached K/V byte is read from HBM once for all of them [MHA/MQA/GQA walkthrough,
// section 7: one K/V tile serves the group's query rows]. (Groups wider than 32 heads are cut
// into head blocks of 32; each block re-reads the group's K/V.) Unit u has n_b visible keys,
// n_b = min(kv_len[b], q_pos[b] + 1). The visible keys of all units, laid end to end, are cut
// into G equal contiguous ranges, one per CTA (stream-K style), so every CTA streams the same
// number of bytes whatever the per-request lengths are; a range may end inside a unit and the
// next range continues it. This is the "split along history" of the walkthrough's section 9,
// with the split points chosen for balance.
//
// Per piece (the part of one unit inside one CTA's range) the CTA keeps the online-softmax state
// (m, l, u) per query row [序列计算与存储, section 在线 softmax] and produces the normalised
// piece output and its log-sum-exp. A unit that lies inside one range is written directly.
// Otherwise each piece writes a partial to the workspace, and the CTA that finishes the unit's
// last piece merges them: M = max_p lse_p, O = sum_p e^{lse_p - M} o_p / sum_p e^{lse_p - M}
// [第三章：MHA 的局限与 MQA、GQA、Flash Attention, section 3.5: merge with a common maximum].
//
// bf16 kernel: warp-specialised. One producer warp streams 64-key K and V tiles with TMA
// (cp.async.bulk.tensor, 128-byte swizzle, no multicast) into a 4-stage shared-memory ring guarded
// by mbarriers. Four consumer warps per 16-row m-tile each take 16 keys of every tile: scores
// S = Q K^T and the update O += P V run on the tensor cores as m16n8k16 bf16 MMAs with fp32
// accumulators (the r <= 32 query rows of a unit are too few for a 64/128-row tcgen05 tile; the
// kernel is HBM-bound, so the MMA rate is not the limit). Scores use the base-2 exponent with
// scale * log2(e) folded into one multiply.
//
// fp32 kernel (check mode): the same partition, piece bookkeeping and merge, with a scalar core:
// one warp per query head, lanes split d_h, one key per online-softmax step.

#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gqa {
namespace dec {

constexpr int kTile = 64;     // keys per pipeline stage
constexpr int kStages = 4;    // pipeline depth
constexpr int kMaxBatch = 1024;
constexpr int kMinKeysPerRange = 64;
constexpr int kHeadsPerUnitMax = 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Layout {
  int U;           // number of units
  int hpu;         // query heads per unit (head block width)
  int hblocks;     // head blocks per KV head
  size_t cnt_off, lse_off, o_off, total;
};

__host__ __device__ inline Layout make_layout(int B, int h_q, int h_kv, int d_h, int G) {
  Layout L;
  const int r = h_q / h_kv;
  L.hpu = r < kHeadsPerUnitMax ? r : kHeadsPerUnitMax;
  L.hblocks = (r + L.hpu - 1) / L.hpu;
  L.U = B * h_kv * L.hblocks;
  const size_t slots = (size_t)G + L.U;
  L.cnt_off = 0;
  L.lse_off = align_up((size_t)L.U * 4, 256);
  L.o_off = L.lse_off + align_up(slots * L.hpu * 4, 256);
  L.total = L.o_off + slots * L.hpu * d_h * 4;
  return L;
}

// Per-CTA view of the partition, built in shared memory by the prologue.
struct Plan {
  long long* pre;  // pre[b] = sum_{b' < b} n_b' (pre[B] = total), in keys of one unit
  int* nlen;       // n_b
  int UPB;         // units per sequence = h_kv * hblocks
  long long K;     // total keys over all units
  int G;           // effective number of ranges
};

__device__ __forceinline__ long long range_start(const Plan& p, int c) {
  return (long long)c * p.K / p.G;
}
// CTA whose range contains global key position x.
__device__ __forceinline__ int range_of(const Plan& p, long long x) {
  return (int)(((x + 1) * (long long)p.G + p.K - 1) / p.K) - 1;
}

struct Piece {
  int b, g, hb;
  int unit;         // global unit index
  int k0, k1;       // key range inside the unit
  int n;            // unit length
  int c_first, n_pieces;
  long long unit_start;
};

// Locate the piece that starts at global position x (x < K).
__device__ __forceinline__ Piece locate(const Plan& p, int B, int hblocks, long long x,
                                        long long range_end) {
  // largest b with pre[b] * UPB <= x and n_b > 0
  int lo = 0, hi = B;  // invariant: pre[lo]*UPB <= x < pre[hi]*UPB
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.pre[mid] * p.UPB <= x) lo = mid; else hi = mid;
  }
  int b = lo;
  while (p.nlen[b] == 0) ++b;
  Piece pc;
  pc.b = b;
  pc.n = p.nlen[b];
  const long long rel = x - p.pre[b] * p.UPB;
  const int ui = (int)(rel / pc.n);  // g * hblocks + hb
  pc.g = ui / hblocks;
  pc.hb = ui - pc.g * hblocks;
  pc.unit = b * p.UPB + ui;
  pc.unit_start = p.pre[b] * p.UPB + (long long)ui * pc.n;
  pc.k0 = (int)(x - pc.unit_start);
  const long long e = range_end - pc.unit_start;
  pc.k1 = e < pc.n ? (int)e : pc.n;
  pc.c_first = range_of(p, pc.unit_start);
  pc.n_pieces = range_of(p, pc.unit_start + pc.n - 1) - pc.c_first + 1;
  return pc;
}

struct KArgs {
  const void* q;
  const void* k;  // read by the fp32 kernel (the bf16 kernel reads K/V through tensor maps)
  const void* v;
  void* o;
  float* lse;
  const int32_t* kv_len;
  const int32_t* q_pos;
  int B, h_q, h_kv, r, T_max, D;
  int hpu, hblocks;
  float scale;  // natural-log scale; the bf16 core folds log2(e) in
  int G;        // grid size
  int* counters;
  float* part_lse;
  float* part_o;
  unsigned* err;
};

// Prologue: lengths, prefix sums and zero rows for invalid sequences. Run by warp `w0`.
template <typename OutT>
__device__ void build_plan(const KArgs& a, Plan& p, long long* pre, int* nlen, int warp, int lane,
                           int w0) {
  if (warp == w0) {
    long long run = 0;
    for (int base = 0; base < a.B; base += 32) {
      const int b = base + lane;
      int n = 0;
      if (b < a.B) {
        const int kv = a.kv_len ? a.kv_len[b] : a.T_max;
        const int qp = a.q_pos ? a.q_pos[b] : kv - 1;
        if (kv < 1 || kv > a.T_max) {
          if (blockIdx.x == 0) set_device_error(a.err, GQA_DEVERR_KV_LEN);
        } else if (qp < 0) {
          if (blockIdx.x == 0) set_device_error(a.err, GQA_DEVERR_POSITION);
        } else {
          n = qp + 1 < kv ? qp + 1 : kv;
        }
        nlen[b] = n;
      }
      // inclusive warp scan of n
      long long s = n;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long t = __shfl_up_sync(0xffffffffu, s, off);
        if (lane >= off) s += t;
      }
      if (b < a.B) pre[b] = run + s - n;
      run += __shfl_sync(0xffffffffu, s, 31);
    }
    if (lane == 0) pre[a.B] = run;
  }
  __syncthreads();
  p.pre = pre;
  p.nlen = nlen;
  p.UPB = a.h_kv * a.hblocks;
  p.K = pre[a.B] * p.UPB;
  long long g = p.K / kMinKeysPerRange;
  if (g < 1) g = 1;
  p.G = (int)(g < a.G ? g : a.G);

  // CTA 0 writes zero rows (and lse = -inf) for sequences with nothing visible.
  if (blockIdx.x == 0) {
    for (int b = 0; b < a.B; ++b) {
      if (nlen[b] != 0) continue;
      const long long base = (long long)b * a.h_q * a.D;
      for (int e = threadIdx.x; e < a.h_q * a.D; e += blockDim.x)
        reinterpret_cast<OutT*>(a.o)[base + e] = OutT(0.f);
      if (a.lse)
        for (int h = threadIdx.x; h < a.h_q; h += blockDim.x) a.lse[(long long)b * a.h_q + h] = -INFINITY;
    }
  }
}

__device__ __forceinline__ void store_out(float* o, long long i, float v) { o[i] = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16* o, long long i, float v) {
  o[i] = __float2bfloat16_rn(v);
}

template <bool kFast>
__device__ __forceinline__ float exp2_(float x) {
  if constexpr (kFast) return fast_exp2(x);
  else return exp2f(x);
}
template <bool kFast>
__device__ __forceinline__ float log2_(float x) {
  if constexpr (kFast) return __log2f(x);
  else return log2f(x);
}

// Emit one finished element of a piece: either the final output (single-piece unit) or a
// workspace partial. lse2 is the base-2 log-sum-exp of the row (used by the element with col 0).
template <typename OutT>
__device__ __forceinline__ void emit(const KArgs& a, const Piece& pc, int head_local, int col,
                                     float val, float lse2) {
  const int head = pc.g * a.r + pc.hb * a.hpu + head_local;
  if (pc.n_pieces == 1) {
    store_out(reinterpret_cast<OutT*>(a.o), ((long long)pc.b * a.h_q + head) * a.D + col, val);
    if (col == 0 && a.lse) a.lse[(long long)pc.b * a.h_q + head] = lse2 * kLn2;
  } else {
    const int c = blockIdx.x;
    const long long slot = (long long)c + pc.unit;
    a.part_o[(slot * a.hpu + head_local) * a.D + col] = val;
    if (col == 0) a.part_lse[slot * a.hpu + head_local] = lse2;
  }
}

// After every consumer thread has emitted its piece elements: count the piece and, if it was the
// unit's last, merge all partials. `tid`/`nthreads` index the consumer threads; `bar_id` is a named
// barrier over exactly those threads; `flag` is a shared int.
template <typename OutT, bool kFast>
__device__ void finish_unit(const KArgs& a, const Piece& pc, int tid, int nthreads, int bar_id,
                            int* flag) {
  if (pc.n_pieces == 1) return;
  __threadfence();
  named_barrier_sync(bar_id, nthreads);
  if (tid == 0) {
    const int old = atomicAdd(&a.counters[pc.unit], 1);
    __threadfence();
    *flag = (old == pc.n_pieces - 1);
  }
  named_barrier_sync(bar_id, nthreads);
  if (!*flag) return;
  const int nh = min(a.hpu, a.r - pc.hb * a.hpu);
  for (int e = tid; e < nh * a.D; e += nthreads) {
    const int h = e / a.D, col = e - h * a.D;
    float M = -INFINITY;
    for (int p = 0; p < pc.n_pieces; ++p) {
      const long long slot = (long long)pc.c_first + p + pc.unit;
      M = fmaxf(M, __ldcg(&a.part_lse[slot * a.hpu + h]));
    }
    float L = 0.f, acc = 0.f;
    for (int p = 0; p < pc.n_pieces; ++p) {
      const long long slot = (long long)pc.c_first + p + pc.unit;
      const float w = exp2_<kFast>(__ldcg(&a.part_lse[slot * a.hpu + h]) - M);
      L += w;
      acc = fmaf(w, __ldcg(&a.part_o[(slot * a.hpu + h) * a.D + col]), acc);
    }
    const int head = pc.g * a.r + pc.hb * a.hpu + h;
    store_out(reinterpret_cast<OutT*>(a.o), ((long long)pc.b * a.h_q + head) * a.D + col, acc / L);
    if (col == 0 && a.lse) a.lse[(long long)pc.b * a.h_q + head] = (M + log2_<kFast>(L)) * kLn2;
  }
  named_barrier_sync(bar_id, nthreads);
  if (tid == 0) a.counters[pc.unit] = 0;  // leave the workspace ready for the next call
}

// =============================================================================================
// bf16 tensor-core kernel
// =============================================================================================

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// zero the bf16 halves of a packed pair whose key index is >= nvalid
__device__ __forceinline__ uint32_t mask_pair(uint32_t v, int key_lo, int nvalid) {
  const uint32_t lo = key_lo < nvalid ? 0x0000ffffu : 0u;
  const uint32_t hi = key_lo + 1 < nvalid ? 0xffff0000u : 0u;
  return v & (lo | hi);
}

template <int D, int MT>
struct Bf16Cfg {
  static constexpr int kNch = D / 64;                       // 64-column (128-byte) chunks
  static constexpr int kChunkBytes = kTile * 128;           // one chunk of one tile
  static constexpr int kTileBytes = kNch * kChunkBytes;     // K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;        // K + V
  static constexpr int kConsumerWarps = 4 * MT;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kRedStride = D + 8;                  // floats per row of the merge buffer
  static constexpr int kRedBytes = MT * 4 * 16 * kRedStride * 4;
  static constexpr int kStatBytes = MT * 4 * 16 * 4;
  static constexpr size_t kSmem = (size_t)kStages * kStageBytes + kRedBytes + 2 * kStatBytes +
                                  (kMaxBatch + 1) * 8 + kMaxBatch * 4 + 2 * kStages * 8 + 64 +
                                  1024;  // alignment slack
};

template <int D, int MT>
__global__ void __launch_bounds__(Bf16Cfg<D, MT>::kThreads, 1)
    decode_bf16_kernel(const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, KArgs a) {
  using C = Bf16Cfg<D, MT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  float* red = reinterpret_cast<float*>(smem + kStages * C::kStageBytes);
  float* st_m = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(red) + C::kRedBytes);
  float* st_l = st_m + MT * 4 * 16;
  long long* pre = reinterpret_cast<long long*>(st_l + MT * 4 * 16);
  int* nlen = reinterpret_cast<int*>(pre + kMaxBatch + 1);
  uint64_t* bars = reinterpret_cast<uint64_t*>(nlen + kMaxBatch);
  int* flag = reinterpret_cast<int*>(bars + 2 * kStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int producer_warp = C::kConsumerWarps;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);                          // full: producer arrival + tx
      mbar_init(smem_u32(&bars[kStages + s]), C::kConsumerWarps);  // empty: one per consumer warp
    }
    fence_barrier_init();
  }
  Plan plan;
  build_plan<__nv_bfloat16>(a, plan, pre, nlen, warp, lane, producer_warp);
  // (build_plan ends with __syncthreads, which also publishes the barrier init)
  const int c = blockIdx.x;
  if (c >= plan.G || plan.K == 0) return;
  const long long x_begin = range_start(plan, c), x_end = range_start(plan, c + 1);

  if (warp == producer_warp) {
    if (lane == 0) {
      tma_prefetch_desc(&tmk);
      tma_prefetch_desc(&tmv);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (long long x = x_begin; x < x_end && ok;) {
        const Piece pc = locate(plan, a.B, a.hblocks, x, x_end);
        const int row0 = (pc.b * a.h_kv + pc.g) * a.T_max;
        for (int t = pc.k0; t < pc.k1; t += kTile) {
          if (!mbar_wait(smem_u32(&bars[kStages + stage]), phase ^ 1u, a.err)) { ok = false; break; }
          const uint32_t full = smem_u32(&bars[stage]);
          mbar_arrive_expect_tx(full, C::kStageBytes);
          const uint32_t kdst = smem_u32(stage_base + stage * C::kStageBytes);
          const uint32_t vdst = kdst + C::kTileBytes;
#pragma unroll
          for (int ch = 0; ch < C::kNch; ++ch) {
            tma_load_2d(kdst + ch * C::kChunkBytes, &tmk, full, ch * 64, row0 + t);
            tma_load_2d(vdst + ch * C::kChunkBytes, &tmv, full, ch * 64, row0 + t);
          }
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        x = pc.unit_start + pc.k1;
      }
      // Drain: wait (bounded) until the last kStages fills have been consumed, so no copy is in
      // flight into shared memory when the CTA exits. Fill f used stage f % kStages and its
      // consumption completes phase f / kStages of that stage's empty barrier.
      for (int f = issued > kStages ? issued - kStages : 0; f < issued; ++f) {
        if (!mbar_wait(smem_u32(&bars[kStages + f % kStages]), (uint32_t)(f / kStages) & 1u, a.err))
          break;
      }
    }
    return;
  }

  // ------------------------------- consumer warps -------------------------------------------
  const int mt = warp / 4;       // m-tile (16 query rows)
  const int ws = warp % 4;       // key slice inside each 64-key tile
  const int gid = lane >> 2, tq = lane & 3;
  const int ctid = threadIdx.x;  // 0 .. 32 * kConsumerWarps - 1
  const int nct = 32 * C::kConsumerWarps;
  const int mt_tid = ctid - mt * 128;
  const float sl2 = a.scale * kLog2e;
  constexpr int NK = D / 16;  // k-steps of QK^T
  constexpr int NN = D / 8;   // n-tiles of PV

  int stage = 0;
  uint32_t phase = 0;
  for (long long x = x_begin; x < x_end;) {
    const Piece pc = locate(plan, a.B, a.hblocks, x, x_end);
    const int nh = min(a.hpu, a.r - pc.hb * a.hpu);
    // Q fragments for this m-tile (rows = heads of the unit)
    uint32_t qf[NK][4];
    {
      const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                ((long long)pc.b * a.h_q + pc.g * a.r + pc.hb * a.hpu) * D;
      const int r0 = mt * 16 + gid, r1 = r0 + 8;
#pragma unroll
      for (int ks = 0; ks < NK; ++ks) {
        const int cidx = ks * 16 + 2 * tq;
        qf[ks][0] = r0 < nh ? *reinterpret_cast<const uint32_t*>(qb + r0 * D + cidx) : 0u;
        qf[ks][1] = r1 < nh ? *reinterpret_cast<const uint32_t*>(qb + r1 * D + cidx) : 0u;
        qf[ks][2] = r0 < nh ? *reinterpret_cast<const uint32_t*>(qb + r0 * D + cidx + 8) : 0u;
        qf[ks][3] = r1 < nh ? *reinterpret_cast<const uint32_t*>(qb + r1 * D + cidx + 8) : 0u;
      }
    }
    float acc[NN][4];
#pragma unroll
    for (int n = 0; n < NN; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;

    for (int t = pc.k0; t < pc.k1; t += kTile) {
      const int nvalid = min(kTile, pc.k1 - t);
      if (!mbar_wait(smem_u32(&bars[stage]), phase, a.err)) { ok = false; break; }
      const int klo = ws * 16;
      if (klo < nvalid) {
        const uint32_t kb = smem_u32(stage_base + stage * C::kStageBytes);
        const uint32_t vb = kb + C::kTileBytes;
        // ---- S = Q K^T for keys klo .. klo+15 (two n-tiles of 8 keys)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
          const int krow = klo + ((lane >> 4) << 3) + (lane & 7);
#pragma unroll
          for (int ks = 0; ks < NK; ++ks) {
            const int d8 = ks * 2 + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(swz128(kb + (d8 >> 3) * C::kChunkBytes, krow, d8 & 7), b0, b1, b2, b3);
            mma_bf16(sc[0], qf[ks], b0, b1);
            mma_bf16(sc[1], qf[ks], b2, b3);
          }
        }
        // ---- mask, scale (base 2), online softmax update
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int key = klo + 8 * j + 2 * tq + e;
            const bool vis = key < nvalid;
            sc[j][e] = vis ? sc[j][e] * sl2 : -INFINITY;
            sc[j][2 + e] = vis ? sc[j][2 + e] * sl2 : -INFINITY;
            mx0 = fmaxf(mx0, sc[j][e]);
            mx1 = fmaxf(mx1, sc[j][2 + e]);
          }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            sc[j][e] = fast_exp2(sc[j][e] - mn0);
            sc[j][2 + e] = fast_exp2(sc[j][2 + e] - mn1);
            ps0 += sc[j][e];
            ps1 += sc[j][2 + e];
          }
        }
        l0 = fmaf(l0, al0, ps0);
        l1 = fmaf(l1, al1, ps1);
#pragma unroll
        for (int n = 0; n < NN; ++n) {
          acc[n][0] *= al0;
          acc[n][1] *= al0;
          acc[n][2] *= al1;
          acc[n][3] *= al1;
        }
        uint32_t pa[4];
        pa[0] = pack_bf16x2(sc[0][0], sc[0][1]);
        pa[1] = pack_bf16x2(sc[0][2], sc[0][3]);
        pa[2] = pack_bf16x2(sc[1][0], sc[1][1]);
        pa[3] = pack_bf16x2(sc[1][2], sc[1][3]);
        // ---- O += P V (keys klo..klo+15, all d_h columns)
        const bool partial = klo + 16 > nvalid;
        const int vrow = klo + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int key_a = klo + 2 * tq, key_b = klo + 8 + 2 * tq;
#pragma unroll
        for (int n2 = 0; n2 < NN / 2; ++n2) {
          const int d8 = n2 * 2 + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(swz128(vb + (d8 >> 3) * C::kChunkBytes, vrow, d8 & 7), b0, b1, b2, b3);
          if (partial) {
            b0 = mask_pair(b0, key_a, nvalid);
            b1 = mask_pair(b1, key_b, nvalid);
            b2 = mask_pair(b2, key_a, nvalid);
            b3 = mask_pair(b3, key_b, nvalid);
          }
          mma_bf16(acc[2 * n2], pa, b0, b1);
          mma_bf16(acc[2 * n2 + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars[kStages + stage]));
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }
    if (!ok) return;

    // ---- merge the four key slices of this m-tile, normalise, emit
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    float* sm = st_m + mt * 64;
    float* sl = st_l + mt * 64;
    if (tq == 0) {
      sm[ws * 16 + gid] = m0;
      sm[ws * 16 + gid + 8] = m1;
      sl[ws * 16 + gid] = l0;
      sl[ws * 16 + gid + 8] = l1;
    }
    named_barrier_sync(2 + mt, 128);
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      M0 = fmaxf(M0, sm[w * 16 + gid]);
      M1 = fmaxf(M1, sm[w * 16 + gid + 8]);
    }
    float L0 = 0.f, L1 = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      L0 += fast_exp2(sm[w * 16 + gid] - M0) * sl[w * 16 + gid];
      L1 += fast_exp2(sm[w * 16 + gid + 8] - M1) * sl[w * 16 + gid + 8];
    }
    const float f0 = fast_exp2(m0 - M0) / L0, f1 = fast_exp2(m1 - M1) / L1;
    float* rb = red + (mt * 4 + ws) * 16 * C::kRedStride;
#pragma unroll
    for (int n = 0; n < NN; ++n) {
      const int col = n * 8 + 2 * tq;
      *reinterpret_cast<float2*>(rb + gid * C::kRedStride + col) = make_float2(acc[n][0] * f0, acc[n][1] * f0);
      *reinterpret_cast<float2*>(rb + (gid + 8) * C::kRedStride + col) = make_float2(acc[n][2] * f1, acc[n][3] * f1);
    }
    named_barrier_sync(2 + mt, 128);
    const float* r0p = red + (mt * 4) * 16 * C::kRedStride;
    for (int e = mt_tid; e < 16 * D; e += 128) {
      const int row = e / D, col = e - row * D;
      const int hl = mt * 16 + row;
      if (hl >= nh) continue;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) v += r0p[(w * 16 + row) * C::kRedStride + col];
      float lse2 = 0.f;
      if (col == 0) {
        float M = -INFINITY, L = 0.f;
        for (int w = 0; w < 4; ++w) M = fmaxf(M, sm[w * 16 + row]);
        for (int w = 0; w < 4; ++w) L += fast_exp2(sm[w * 16 + row] - M) * sl[w * 16 + row];
        lse2 = M + __log2f(L);
      }
      emit<__nv_bfloat16>(a, pc, hl, col, v, lse2);
    }
    named_barrier_sync(1, nct);  // all m-tiles emitted; shared buffers free again
    finish_unit<__nv_bfloat16, true>(a, pc, ctid, nct, 1, flag);
    x = pc.unit_start + pc.k1;
  }
}

// =============================================================================================
// fp32 check-mode kernel
// =============================================================================================
constexpr int kF32Warps = 4;
constexpr int kF32MaxPerLane = 8;  // d_h <= 256

__global__ void __launch_bounds__(32 * kF32Warps, 1) decode_fp32_kernel(KArgs a) {
  __shared__ long long pre[kMaxBatch + 1];
  __shared__ int nlen[kMaxBatch];
  __shared__ int flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Plan plan;
  build_plan<float>(a, plan, pre, nlen, warp, lane, 0);
  const int c = blockIdx.x;
  if (c >= plan.G || plan.K == 0) return;
  const long long x_begin = range_start(plan, c), x_end = range_start(plan, c + 1);
  const int D = a.D;
  for (long long x = x_begin; x < x_end;) {
    const Piece pc = locate(plan, a.B, a.hblocks, x, x_end);
    const int nh = min(a.hpu, a.r - pc.hb * a.hpu);
    const long long kv_base = ((long long)pc.b * a.h_kv + pc.g) * a.T_max * D;
    const float* kp = reinterpret_cast<const float*>(a.k) + kv_base;
    const float* vp = reinterpret_cast<const float*>(a.v) + kv_base;
    for (int hl = warp; hl < nh; hl += kF32Warps) {
      const int head = pc.g * a.r + pc.hb * a.hpu + hl;
      const float* q = reinterpret_cast<const float*>(a.q) + ((long long)pc.b * a.h_q + head) * D;
      float qr[kF32MaxPerLane], acc[kF32MaxPerLane];
#pragma unroll
      for (int e = 0; e < kF32MaxPerLane; ++e) {
        const int col = lane + 32 * e;
        qr[e] = col < D ? q[col] : 0.f;
        acc[e] = 0.f;
      }
      float m = -INFINITY, l = 0.f;
      for (int j = pc.k0; j < pc.k1; ++j) {
        const float* kj = kp + (long long)j * D;
        const float* vj = vp + (long long)j * D;
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < kF32MaxPerLane; ++e) {
          const int col = lane + 32 * e;
          if (col < D) part = fmaf(qr[e], kj[col], part);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        const float s = part * a.scale;
        const float m_new = fmaxf(m, s);
        const float alpha = expf(m - m_new);
        const float p = expf(s - m_new);
        l = fmaf(l, alpha, p);
#pragma unroll
        for (int e = 0; e < kF32MaxPerLane; ++e) {
          const int col = lane + 32 * e;
          if (col < D) acc[e] = fmaf(acc[e], alpha, p * vj[col]);
        }
        m = m_new;
      }
      const float lse2 = (m + logf(l)) * kLog2e;
      const float inv = 1.f / l;
#pragma unroll
      for (int e = 0; e < kF32MaxPerLane; ++e) {
        const int col = lane + 32 * e;
        if (col < D) emit<float>(a, pc, hl, col, acc[e] * inv, lse2);
      }
    }
    named_barrier_sync(1, 32 * kF32Warps);
    finish_unit<float, false>(a, pc, threadIdx.x, 32 * kF32Warps, 1, &flag);
    x = pc.unit_start + pc.k1;
  }
}

template <int D, int MT>
cudaError_t launch_bf16_typed(const KArgs& ka, const CUtensorMap* tm, int grid, cudaStream_t s) {
  using C = Bf16Cfg<D, MT>;
  auto kern = decode_bf16_kernel<D, MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid, C::kThreads, C::kSmem, s>>>(tm[0], tm[1], ka);
  return cudaGetLastError();
}

KArgs make_kargs(const DecodeArgs& a, bool bf16) {
  const Layout L = make_layout(a.B, a.h_q, a.h_kv, a.d_h, a.num_splits);
  (void)bf16;
  KArgs k;
  k.q = a.q;
  k.k = a.k;
  k.v = a.v;
  k.o = a.o;
  k.lse = a.lse;
  k.kv_len = a.kv_len;
  k.q_pos = a.q_pos;
  k.B = a.B;
  k.h_q = a.h_q;
  k.h_kv = a.h_kv;
  k.r = a.h_q / a.h_kv;
  k.T_max = a.T_max;
  k.D = a.d_h;
  k.hpu = L.hpu;
  k.hblocks = L.hblocks;
  k.scale = a.scale;
  k.G = a.num_splits;
  uint8_t* ws = reinterpret_cast<uint8_t*>(a.workspace);
  k.counters = reinterpret_cast<int*>(ws + L.cnt_off);
  k.part_lse = reinterpret_cast<float*>(ws + L.lse_off);
  k.part_o = reinterpret_cast<float*>(ws + L.o_off);
  k.err = a.err;
  return k;
}

}  // namespace dec

size_t decode_workspace_bytes(int B, int h_q, int h_kv, int d_h, bool bf16, int num_splits) {
  (void)bf16;
  return dec::make_layout(B, h_q, h_kv, d_h, num_splits).total;
}

int decode_heads_per_unit(int h_q, int h_kv, bool bf16) {
  (void)bf16;
  const int r = h_q / h_kv;
  return r < dec::kHeadsPerUnitMax ? r : dec::kHeadsPerUnitMax;
}

int decode_max_batch() { return dec::kMaxBatch; }

cudaError_t launch_decode_fp32(const DecodeArgs& a, cudaStream_t s) {
  const dec::KArgs k = dec::make_kargs(a, false);
  dec::decode_fp32_kernel<<<a.num_splits, 32 * dec::kF32Warps, 0, s>>>(k);
  return cudaGetLastError();
}

cudaError_t launch_decode_bf16(const DecodeArgs& a, const CUtensorMap* tmaps, cudaStream_t s) {
  const dec::KArgs k = dec::make_kargs(a, true);
  const bool two = k.hpu > 16;
  if (a.d_h == 128) {
    return two ? dec::launch_bf16_typed<128, 2>(k, tmaps, a.num_splits, s)
               : dec::launch_bf16_typed<128, 1>(k, tmaps, a.num_splits, s);
  }
  if (a.d_h == 64) {
    return two ? dec::launch_bf16_typed<64, 2>(k, tmaps, a.num_splits, s)
               : dec::launch_bf16_typed<64, 1>(k, tmaps, a.num_splits, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gqa
