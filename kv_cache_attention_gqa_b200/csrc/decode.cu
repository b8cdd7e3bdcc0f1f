// Split-KV decode: one new query per sequence attending over its cached K/V.
//
// Work decomposition. A "unit" is (sequence b, KV head g, head block hb): the r query heads that
// read KV head g [序列计算与存储, section 分组查询注意力: g(a) = floor(a / r)] are packed into one
// tile, so each cached K/V byte is read from HBM once for all of them [MHA/MQA/GQA walkthrough,
// section 7: one K/V tile serves the group's query rows]. (Groups wider than 32 heads are cut into
// head blocks of 32; each block re-reads the group's K/V.) Unit u has n_b visible keys,
// n_b = min(kv_len[b], q_pos[b] + 1). The visible keys of all units, laid end to end, are cut into
// equal chunks of C keys ("split along history" [MHA/MQA/GQA walkthrough, section 9]). A chunk
// may hold the end of one unit and the start of the next; the part of a unit inside a chunk is a
// "piece". CTA c starts with chunk c; when there are more chunks than CTAs, further chunks come
// from an atomic ticket, so a CTA that gets more memory bandwidth takes more of them.
//
// Per piece the CTA keeps the online-softmax state (m, l, u) of each query row
// [序列计算与存储, section 在线 softmax] and produces the normalised piece output o_p and its
// base-2 log-sum-exp. A unit that lies inside one chunk is written to the output directly.
// Otherwise each piece writes a partial to the workspace, and a second kernel, launched as a
// programmatic dependent of the first, merges the partials of each row with a running maximum:
// O = sum_p e^{lse_p - M} o_p / sum_p e^{lse_p - M} [第三章：MHA 的局限与 MQA、GQA、Flash Attention,
// section 3.5: partial results merge after rescaling to a common maximum].
//
// bf16 kernel, warp-specialised. One producer warp takes chunks, writes one small descriptor per
// 64-key tile into shared memory, and streams the tile's K and V (and, on the first tile of a
// piece, the unit's query rows) with TMA (cp.async.bulk.tensor, 128-byte swizzle, each CTA its own copies)
// into a 5-stage (one m-tile) or 4-stage (two) ring guarded by mbarriers. Four consumer warps per
// 16-row m-tile each take 16 keys
// of every tile: S = Q K^T and O += P V run on the tensor cores as m16n8k16 bf16 MMAs with fp32
// accumulators (a unit has at most 32 query rows, too few for a 64/128-row tcgen05 tile, and the
// kernel is bound by HBM, not by the MMA rate). Scores use base-2 exponents with scale * log2(e)
// folded into one multiply.
//
// fp32 kernel (check mode): the same chunks, pieces, partials and merge, with a scalar core (one
// warp per query head, lanes split d_h, one key per online-softmax step).
//
// Also here, on the same plan / pieces / merge:
//   * a paged cache (pools of fixed-size pages and a block table): the partition counts 16- or
//     64-key granules so no loaded sub-tile straddles a page, and the whole producer warp
//     prefetches a window of block-table entries (see the producer);
//   * a sliding window: a unit starts at its window (rounded down to the granule), leading keys
//     before the window are masked per tile;
//   * MLA decode over a latent cache (mla_bf16_kernel): one shared KV "head" whose value is the
//     first 512 entries of each 576-wide cache row.

#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace gqa {
namespace dec {

constexpr int kTile = 64;           // keys per pipeline stage
constexpr int kMaxBatch = 1024;
constexpr int kHeadsPerUnitMax = 32;
constexpr int kMinChunkAuto = 128;  // keys; automatic chunking never goes below this
// Automatic chunking: one chunk per SM. Each chunk boundary costs a piece epilogue (a cross-warp
// merge and a partial write) that stalls the stream for ~2 us, which measured more than the load
// imbalance that finer chunks would remove (decode_8k, B200: one chunk per SM was fastest for
// h_kv = 32, 8 and 1).
constexpr int kChunksPerSm = 1;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Quotient of two non-negative 64-bit integers. When both fit in 32 bits (every workload short of
// 2^32 keys in all) it takes a 32-bit unsigned division, a fraction of the 64-bit routine's
// dependent instructions; the plan and the merge sit on the critical path of every call.
__device__ __forceinline__ long long udiv(long long n, long long d) {
  if ((((unsigned long long)n | (unsigned long long)d) >> 32) == 0)
    return (long long)((unsigned)n / (unsigned)d);
  return n / d;
}

// Workspace:
//   [0, 256)       header: chunk ticket (reset to 0 by the merge kernel), chunk size, chunk count
//   pre_off        int64 pre[B + 1]: prefix sums of the visible lengths (written by CTA 0)
//   nlen_off       int32 nlen[B]
//   lse_off        fp32 partial base-2 log-sum-exp, (n_max + U) slots x hpu
//   o_off          fp32 partial outputs, (n_max + U) slots x hpu x d_h
// A piece of unit u in chunk c uses slot c + u: distinct pieces get distinct slots because chunk
// and unit boundaries are both increasing in the global key position.
struct Header {
  int ticket;
  int chunk;  // C
  int n_chunks;
  int pad;
};

struct Layout {
  int U, hpu, hblocks, n_max;
  size_t pre_off, nlen_off, lse_off, o_off, total;
};

// hpu_max: query heads packed into one unit (32 for the GQA kernels, 16 for MLA); d_h: the width
// of the output and of the partials.
__host__ __device__ inline Layout make_layout(int B, int h_q, int h_kv, int d_h, int n_max,
                                              int hpu_max = kHeadsPerUnitMax) {
  Layout L;
  const int r = h_q / h_kv;
  L.hpu = r < hpu_max ? r : hpu_max;
  L.hblocks = (r + L.hpu - 1) / L.hpu;
  L.U = B * h_kv * L.hblocks;
  L.n_max = n_max;
  const size_t slots = (size_t)n_max + L.U;
  L.pre_off = 256;
  L.nlen_off = L.pre_off + align_up((size_t)(B + 1) * 8, 256);
  L.lse_off = L.nlen_off + align_up((size_t)B * 4, 256);
  L.o_off = L.lse_off + align_up(slots * L.hpu * 4, 256);
  L.total = L.o_off + slots * L.hpu * d_h * 4;
  return L;
}

struct KArgs {
  const void* q;
  const void* k;  // read by the fp32 kernel (the bf16 kernel reads K/V through tensor maps)
  const void* v;
  void* o;
  float* lse;
  const int32_t* kv_len;
  const int32_t* q_pos;
  int B, h_q, h_kv, r, T_max, D;  // D: width of the values, the output and the partials
  int Dqk;                         // width of the query and key rows (= D except for MLA)
  int hpu, hblocks;
  float scale;     // natural-log scale; the bf16 core folds log2(e) in
  int n_max;       // upper bound on the number of chunks (workspace slots)
  int auto_chunk;  // 1: chunks hold at least min_chunk keys
  int min_chunk;   // keys
  int align_units;  // 1: when every unit has the same length, chunks do not straddle units
  int window;      // 0: none; W > 0: the query at q_pos sees keys q_pos - W < j <= q_pos
  Header* hdr;
  long long* pre;
  int* nlen;
  float* part_lse;
  float* part_o;
  unsigned* err;
  // paged cache (block_table != nullptr): K/V live in a pool (num_pages, h_kv, page_size, d_h);
  // position t of sequence b is row t % page_size of page block_table[b * max_pages + t / page_size]
  const int32_t* block_table;
  int max_pages, page_size, num_pages;
  // partition granule in keys: 1 for a contiguous cache; on a paged cache 64 when pages hold a
  // multiple of 64 keys (every tile lies in one page), else 16 (every 16-key sub-tile does)
  int gran;
  int expire_wait;  // test hook: CTA 0's producer first waits on a barrier that nothing signals
};

// Partition view built in shared memory by every CTA.
struct Plan {
  const long long* pre;  // pre[b] = sum_{b' < b} ceil(n_b' / gran): positions count granules
  const int* nlen;       // unit length: visible keys from the granule-aligned window start
  const int* wlo;        // first visible key (0 without a sliding window)
  int gran;
  int UPB;               // units per sequence = h_kv * hblocks
  long long K;           // total keys over all units
  long long C;           // chunk size
  int n_chunks;
};

struct Piece {
  int b, g, hb;
  int unit;
  int k0, k1;    // key range inside the unit
  int n;         // unit length
  int n_pieces;  // pieces of this unit over all chunks
  long long unit_start;  // in granules
  long long end;         // global position (granules) just past this piece
};

// The piece that starts at global key position x, inside a chunk ending at x_end.
__device__ __forceinline__ Piece locate(const Plan& p, int B, int hblocks, long long x,
                                        long long x_end) {
  int lo = 0, hi = B;  // pre[lo]*UPB <= x < pre[hi]*UPB
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.pre[mid] * p.UPB <= x) lo = mid; else hi = mid;
  }
  int b = lo;
  while (p.nlen[b] == 0) ++b;
  Piece pc;
  pc.b = b;
  pc.n = p.nlen[b];
  const long long ng = (pc.n + p.gran - 1) / p.gran;  // unit length in granules
  const long long rel = x - p.pre[b] * p.UPB;
  const int ui = (int)udiv(rel, ng);  // g * hblocks + hb
  pc.g = ui / hblocks;
  pc.hb = ui - pc.g * hblocks;
  pc.unit = b * p.UPB + ui;
  pc.unit_start = p.pre[b] * p.UPB + (long long)ui * ng;
  pc.k0 = (int)((x - pc.unit_start) * p.gran);
  const long long e = x_end - pc.unit_start;  // granules
  pc.end = e < ng ? x_end : pc.unit_start + ng;
  pc.k1 = e < ng ? (int)(e * p.gran) : pc.n;
  pc.n_pieces = (int)(udiv(pc.unit_start + ng - 1, p.C) - udiv(pc.unit_start, p.C)) + 1;
  return pc;
}

// Prologue of every CTA: visible lengths and their prefix sums into shared memory (warp `w0`) and
// the chunk size. CTA 0 also publishes them to the workspace for the merge kernel and writes zero
// rows (lse = -inf) for sequences with no visible key.
template <typename OutT>
__device__ void build_plan(const KArgs& a, Plan& p, long long* pre, int* nlen, int* wlo, int warp,
                           int lane, int w0) {
  // Every thread of the CTA reads the lengths of its share of the sequences in one round of loads
  // (a batch of up to kMaxBatch costs one memory round trip, not one per 32 sequences) ...
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    const int kv = a.kv_len ? a.kv_len[b] : a.T_max;
    const int qp = a.q_pos ? a.q_pos[b] : kv - 1;
    int n = 0, lo = 0;
    if (kv < 1 || kv > a.T_max) {
      if (blockIdx.x == 0) set_device_error(a.err, GQA_DEVERR_KV_LEN);
    } else if (qp < 0) {
      if (blockIdx.x == 0) set_device_error(a.err, GQA_DEVERR_POSITION);
    } else {
      n = qp + 1 < kv ? qp + 1 : kv;
      if (a.window > 0 && qp - a.window + 1 > 0) lo = qp - a.window + 1;
      if (lo >= n) {  // the window starts at or past the last cached key
        if (blockIdx.x == 0) set_device_error(a.err, GQA_DEVERR_NO_VISIBLE);
        n = 0;
        lo = 0;
      }
    }
    // the unit starts at the window start rounded down to the granule; the keys before the
    // window inside that first granule are masked (only on a paged cache, gran > 1)
    if (n > 0) n -= lo / a.gran * a.gran;
    nlen[b] = n;
    wlo[b] = lo;
  }
  cta_sync();
  // ... then one warp turns them into prefix sums in granules, from shared memory (and notes
  // whether every sequence has the same visible length)
  __shared__ int s_same_len;
  if (warp == w0) {
    long long run = 0;
    bool same = true;
    for (int base = 0; base < a.B; base += 32) {
      const int b = base + lane;
      const long long ngr = b < a.B ? (nlen[b] + a.gran - 1) / a.gran : 0;  // granules
      same = same && __all_sync(0xffffffffu, b >= a.B || nlen[b] == nlen[0]);
      long long s = ngr;  // inclusive warp scan
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long t = __shfl_up_sync(0xffffffffu, s, off);
        if (lane >= off) s += t;
      }
      if (b < a.B) pre[b] = run + s - ngr;
      run += __shfl_sync(0xffffffffu, s, 31);
    }
    if (lane == 0) {
      pre[a.B] = run;
      s_same_len = same ? 1 : 0;
    }
  }
  cta_sync();
  p.pre = pre;
  p.nlen = nlen;
  p.wlo = wlo;
  p.gran = a.gran;
  p.UPB = a.h_kv * a.hblocks;
  p.K = pre[a.B] * p.UPB;
  long long C = udiv(p.K + a.n_max - 1, a.n_max);
  if (a.auto_chunk) {
    // at least kMinChunkAuto keys, and at least 16 keys per query row, so the partial written per
    // chunk (hpu x d_h fp32) stays small against the chunk's K/V bytes (2 x C x d_h bf16)
    const long long lo = udiv((long long)a.min_chunk + a.gran - 1, a.gran);
    if (C < lo) C = lo;
  }
  if (C < 1) C = 1;
  if (a.align_units && s_same_len && nlen[0] > 0) {
    // Every unit has the same length N (in granules): cut each into m equal chunks, m dividing N
    // and as large as the chunk bound allows (down to half of it), so that no chunk holds the end
    // of one unit and the start of the next (a second piece costs a CTA its start-up again).
    const long long N = (nlen[0] + a.gran - 1) / a.gran;
    const long long units = (long long)a.B * p.UPB;
    const long long m_hi = udiv(a.n_max, units);
    for (long long m = m_hi; m >= 1 && 2 * m >= m_hi; --m) {
      if (N % m == 0 && N / m >= C) {
        C = N / m;
        break;
      }
    }
  }
  p.C = C;
  p.n_chunks = (int)udiv(p.K + C - 1, C);

  if (blockIdx.x == 0) {
    for (int b = threadIdx.x; b <= a.B; b += blockDim.x) {
      a.pre[b] = pre[b];
      if (b < a.B) a.nlen[b] = nlen[b];
    }
    if (threadIdx.x == 0) {
      a.hdr->chunk = (int)p.C;
      a.hdr->n_chunks = p.n_chunks;
    }
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

// Emit one finished element of a piece: the final output (single-piece unit, slot < 0) or a
// workspace partial. lse2 (base 2) is used by the element with col == 0.
template <typename OutT>
__device__ __forceinline__ void emit(const KArgs& a, int b, int g, int hb, int slot, int hl,
                                     int col, float val, float lse2) {
  if (slot < 0) {
    const int head = g * a.r + hb * a.hpu + hl;
    store_out(reinterpret_cast<OutT*>(a.o), ((long long)b * a.h_q + head) * a.D + col, val);
    if (col == 0 && a.lse) a.lse[(long long)b * a.h_q + head] = lse2 * kLn2;
  } else {
    a.part_o[((long long)slot * a.hpu + hl) * a.D + col] = val;
    if (col == 0) a.part_lse[(long long)slot * a.hpu + hl] = lse2;
  }
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// =============================================================================================
// merge kernel (both dtypes): one warp per (unit, query head) row, running-maximum merge
// =============================================================================================
template <bool kFast>
__device__ __forceinline__ float ex2(float x) {
  if constexpr (kFast) return fast_exp2(x);
  else return exp2f(x);
}

// Running-maximum merge of the partials of one row. Each lane owns kV consecutive columns
// (kV = 4: 16-byte loads; lanes past d_h idle) and keeps kU pieces' loads in flight.
template <typename OutT, bool kFast, int kV, int kU>
__device__ __forceinline__ void merge_row(const KArgs& a, int lane, int unit, int h,
                                          long long c0, long long c1, long long out_base,
                                          long long lse_index, int col_base) {
  const int D = a.D;
  const int col0 = col_base + lane * kV;
  const bool active = col0 < D;
  float M = -INFINITY, L = 0.f;
  float acc[kV];
#pragma unroll
  for (int i = 0; i < kV; ++i) acc[i] = 0.f;
  for (long long c = c0; c <= c1; c += kU) {
    float ls[kU];
    float ov[kU][kV];
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const long long slot = c + j + unit;
      const bool ok = c + j <= c1;
      ls[j] = ok ? __ldcg(&a.part_lse[slot * a.hpu + h]) : -INFINITY;
      const float* src = a.part_o + (slot * a.hpu + h) * D + col0;
      if constexpr (kV == 4) {
        const float4 v4 = (ok && active) ? __ldcg(reinterpret_cast<const float4*>(src))
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
        ov[j][0] = v4.x; ov[j][1] = v4.y; ov[j][2] = v4.z; ov[j][3] = v4.w;
      } else {
#pragma unroll
        for (int i = 0; i < kV; ++i) ov[j][i] = (ok && col0 + i < D) ? __ldcg(src + i) : 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      if (ls[j] == -INFINITY) continue;
      const float Mn = fmaxf(M, ls[j]);
      const float s_old = ex2<kFast>(M - Mn);
      const float w = ex2<kFast>(ls[j] - Mn);
      L = L * s_old + w;
#pragma unroll
      for (int i = 0; i < kV; ++i) acc[i] = acc[i] * s_old + w * ov[j][i];
      M = Mn;
    }
  }
  const float inv = 1.f / L;
  if (active) {
#pragma unroll
    for (int i = 0; i < kV; ++i)
      if (col0 + i < D) store_out(reinterpret_cast<OutT*>(a.o), out_base + col0 + i, acc[i] * inv);
  }
  if (lane == 0 && col_base == 0 && a.lse) a.lse[lse_index] = (M + (kFast ? __log2f(L) : log2f(L))) * kLn2;
}

// Rows wider than 256 (the MLA latent) are merged by one warp per 128-column slice.
__host__ __device__ inline int merge_slices(int D) { return D > 256 ? (D + 127) / 128 : 1; }

// Merge paths by row width, one kernel each so that each carries only its own registers (the
// 8-column path keeps twice the loads in flight): 0 for d <= 128 (4 columns per lane), 1 for
// d <= 256 (8, lane-strided), 2 for wider rows (4 columns per lane, one warp per 128-column slice,
// 8 partials per round so that four blocks fit an SM), 3 the same with 16 partials per round for
// launches small enough to fit one wave anyway (rows with many partials then take fewer rounds).
__host__ __device__ inline int merge_path(int D) { return D % 4 == 0 && D <= 128 ? 0 : D <= 256 ? 1 : 2; }

template <typename OutT, bool kFast, int kPath>
__global__ void __launch_bounds__(256, kPath == 2 ? 4 : 1) merge_kernel(KArgs a) {
  // The row's place (unit, head, output offsets) depends only on the arguments, so it is worked
  // out before the wait (units number fewer than 2^31: B * h_q is below it).
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slices = merge_slices(a.D);
  const long long wid = (long long)blockIdx.x * 8 + warp;
  const long long row = udiv(wid, slices);
  const int slice = (int)(wid - row * slices);
  const int UPB = a.h_kv * a.hblocks;
  const long long rows = (long long)a.B * UPB * a.hpu;
  const int unit = (int)udiv(row, a.hpu), h = (int)(row - (long long)unit * a.hpu);
  const int b = unit / UPB, ui = unit - b * UPB;
  const int g = ui / a.hblocks, hb = ui - g * a.hblocks;
  const int nh = min(a.hpu, a.r - hb * a.hpu);
  // The chunk size and the length and prefix of the block's sequences (its 8 rows span at most
  // 8 of them) are loaded once per block, one round trip, into shared memory: every warp loading
  // its own made a few addresses hot (thousands of warps requesting the same words).
  __shared__ long long s_pre[8];
  __shared__ int s_n[8];
  __shared__ long long s_C;
  const long long row_first = udiv((long long)blockIdx.x * 8, slices);
  const int b_first = (int)udiv(udiv(row_first, a.hpu), UPB);
  pdl_wait();  // the decode grid has completed and its writes are visible
  if (blockIdx.x == 0 && threadIdx.x == 0) a.hdr->ticket = 0;  // ready for the next call
  if (threadIdx.x < 8 && b_first + (int)threadIdx.x < a.B) {
    s_n[threadIdx.x] = __ldcg(&a.nlen[b_first + threadIdx.x]);
    s_pre[threadIdx.x] = __ldcg(&a.pre[b_first + threadIdx.x]);
  }
  if (threadIdx.x == 32) s_C = __ldcg(&a.hdr->chunk);
  __syncthreads();
  if (row >= rows || h >= nh) return;
  const long long C = s_C;
  const int n = s_n[b - b_first];
  const long long pre_b = s_pre[b - b_first];
  if (n == 0) return;
  const long long ng = (n + a.gran - 1) / a.gran;
  const long long P = pre_b * UPB + (long long)ui * ng;
  const long long c0 = udiv(P, C), c1 = udiv(P + ng - 1, C);
  if (c0 == c1) return;  // written directly by the decode kernel
  const int head = g * a.r + hb * a.hpu + h;
  const long long ob = ((long long)b * a.h_q + head) * a.D;
  const long long li = (long long)b * a.h_q + head;
  if constexpr (kPath == 0) merge_row<OutT, kFast, 4, 16>(a, lane, unit, h, c0, c1, ob, li, 0);
  else if constexpr (kPath == 1) merge_row<OutT, kFast, 8, 16>(a, lane, unit, h, c0, c1, ob, li, 0);
  else if constexpr (kPath == 2) merge_row<OutT, kFast, 4, 8>(a, lane, unit, h, c0, c1, ob, li, slice * 128);
  else merge_row<OutT, kFast, 4, 16>(a, lane, unit, h, c0, c1, ob, li, slice * 128);
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
__device__ __forceinline__ uint32_t mask_pair(uint32_t v, int key_lo, int first, int nvalid) {
  const uint32_t lo = key_lo < nvalid && key_lo >= first ? 0x0000ffffu : 0u;
  const uint32_t hi = key_lo + 1 < nvalid && key_lo + 1 >= first ? 0xffff0000u : 0u;
  return v & (lo | hi);
}

// Descriptor of one pipeline stage, written by the producer before it arms the stage.
struct TileMeta {
  int b, g, hb;
  int nvalid;  // valid keys in this tile (1..64)
  int flags;   // kFirst | kLast | kEnd
  int slot;    // partial slot, or -1: write the output directly
  int nh;      // query heads in the unit
  int nskip;   // leading keys of the tile before the sliding window (masked), else 0
};
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

template <int D, int MT>
struct Bf16Cfg {
  // pipeline depth: as many 32 KiB stages as shared memory allows next to the other buffers
  static constexpr int kStages = MT == 1 ? 5 : 4;
  static constexpr int kNch = D / 64;                    // 64-column (128-byte) chunks
  static constexpr int kChunkBytes = kTile * 128;        // one column chunk of one K/V tile
  static constexpr int kTileBytes = kNch * kChunkBytes;  // K (or V) tile
  static constexpr int kSubBytes = kNch * 16 * 128;       // one 16-key sub-tile, all chunks
  static constexpr int kQRows = 16 * MT;
  static constexpr int kQChunkBytes = kQRows * 128;
  static constexpr int kQBytes = kNch * kQChunkBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kConsumerWarps = 4 * MT;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kRedStride = 64 + 4;  // floats per row of the merge buffer (64 columns)
  static constexpr int kRedBytes = MT * 4 * 16 * kRedStride * 4;
  static constexpr int kStatBytes = MT * 4 * 16 * 4;
  static constexpr size_t kSmem = (size_t)kStages * (kStageBytes + kQBytes) + kRedBytes +
                                  2 * kStatBytes + (kMaxBatch + 1) * 8 + 2 * kMaxBatch * 4 +
                                  kStages * sizeof(TileMeta) + (2 * kStages + 1) * 8 + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

// Cache layouts the bf16 kernel reads (template parameter kMode):
//   kContig    (B, h_kv, T_max, d_h), one 64-row box per column chunk and tile
//   kPaged2d   page pools, 2-D boxes: 64 rows when pages hold a multiple of 64 keys, else 16 rows
//              (one box per 16-key sub-tile and column chunk)
//   kPaged3d   page pools with d_h = 128 and 16-row sub-tiles: a 3-D view (64 columns, rows,
//              2 column chunks) loads both chunks of a sub-tile in one box, so a stage takes half
//              as many copies; a sub-tile then sits in shared memory as its own 4 KiB block
//              (chunk-major, 16 rows each) instead of inside 64-row chunk planes
constexpr int kContig = 0, kPaged2d = 1, kPaged3d = 2;

template <int D, int MT, int kMode>
__global__ void __launch_bounds__(Bf16Cfg<D, MT>::kThreads, 1)
    decode_bf16_kernel(const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv,
                       const __grid_constant__ CUtensorMap tmq, KArgs a) {
  using C = Bf16Cfg<D, MT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;                         // C::kStages x (K, V) tiles
  uint8_t* q_base = smem + C::kStages * C::kStageBytes;  // C::kStages x query rows
  float* red = reinterpret_cast<float*>(q_base + C::kStages * C::kQBytes);
  float* st_m = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(red) + C::kRedBytes);
  float* st_l = st_m + MT * 64;
  long long* pre = reinterpret_cast<long long*>(st_l + MT * 64);
  int* nlen = reinterpret_cast<int*>(pre + kMaxBatch + 1);
  int* wlo = nlen + kMaxBatch;
  TileMeta* meta = reinterpret_cast<TileMeta*>(wlo + kMaxBatch);
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta + C::kStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int producer_warp = C::kConsumerWarps;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);                            // full: producer + tx bytes
      mbar_init(smem_u32(&bars[C::kStages + s]), C::kConsumerWarps);  // empty: one per consumer warp
    }
    mbar_init(smem_u32(&bars[2 * C::kStages]), 1);  // never signalled (test hook)
    fence_barrier_init();
  }
  if (warp == producer_warp && lane == 0) {
    tma_prefetch_desc(&tmk);
    tma_prefetch_desc(&tmv);
    tma_prefetch_desc(&tmq);
  }
  // The kernel is launched as a programmatic dependent of the previous kernel on the stream (for
  // example the kv_append that wrote the new token's K/V): everything above overlaps that kernel,
  // and no input (lengths, positions, queries, cache, block table) is read before it completed.
  pdl_wait();
  Plan plan;
  build_plan<__nv_bfloat16>(a, plan, pre, nlen, wlo, warp, lane, producer_warp);
  pdl_launch_dependents();

  if (warp == producer_warp) {
    // Stage bookkeeping of the producer: fill f uses stage f % kStages; its consumption completes
    // phase f / kStages of that stage's empty barrier.
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    const int G = gridDim.x;
    // chunks past the grid are handed out by the atomic ticket; with no more chunks than CTAs
    // (the automatic choice) every CTA has its one chunk and takes no ticket
    const bool dyn = plan.n_chunks > G;
    // Writes the stage's descriptor and arms its full barrier for `kv_bytes` of K/V (+ the query
    // rows on a piece's first tile). Lane 0 only.
    auto arm = [&](const Piece& pc, int t, int slot, int nh, uint32_t kv_bytes, int nskip) -> uint32_t {
      const bool first = t == pc.k0;
      TileMeta m;
      m.b = pc.b;
      m.g = pc.g;
      m.hb = pc.hb;
      m.nvalid = min(kTile, pc.k1 - t);
      m.flags = (first ? kFirst : 0) | (t + kTile >= pc.k1 ? kLast : 0);
      m.slot = slot;
      m.nh = nh;
      m.nskip = t == 0 ? nskip : 0;  // only a unit's first tile starts before the window
      meta[stage] = m;
      const uint32_t full = smem_u32(&bars[stage]);
      mbar_arrive_expect_tx(full, kv_bytes + (first ? C::kQBytes : 0));
      if (first) {
        const uint32_t qdst = smem_u32(q_base + stage * C::kQBytes);
        const int qrow = pc.b * a.h_q + pc.g * a.r + pc.hb * a.hpu;
#pragma unroll
        for (int ch = 0; ch < C::kNch; ++ch)
          tma_load_2d(qdst + ch * C::kQChunkBytes, &tmq, full, ch * 64, qrow);
      }
      return full;
    };
    auto advance = [&]() {
      ++issued;
      if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
    };

    if constexpr (kMode == kContig) {
      if (lane == 0) {
        // Test hook (off unless the host enabled it): CTA 0's producer waits on a barrier that
        // nothing signals; the bounded wait runs out and records GQA_DEVERR_TIMEOUT, no copy is
        // issued, and the consumers' own bounded waits on the first stage then run out too (all
        // at their first tile, so no consumer is left at a named barrier). The rows of CTA 0's
        // chunk are then left unwritten or merged from stale partials.
        if (a.expire_wait && blockIdx.x == 0 && !mbar_wait(smem_u32(&bars[2 * C::kStages]), 0, a.err))
          ok = false;
        // Chunk tickets: CTA c starts with chunk c; later chunks come from an atomic counter whose
        // value is fetched one chunk ahead, so its latency overlaps the current chunk's loads.
        int chunk = blockIdx.x;
        int next = ok && dyn && chunk < plan.n_chunks ? G + atomicAdd(&a.hdr->ticket, 1) : plan.n_chunks;
        for (; ok && chunk < plan.n_chunks;) {
          const long long x1 = min((long long)(chunk + 1) * plan.C, plan.K);
          for (long long x = (long long)chunk * plan.C; x < x1 && ok;) {
            const Piece pc = locate(plan, a.B, a.hblocks, x, x1);
            const int slot = pc.n_pieces == 1 ? -1 : chunk + pc.unit;
            const int nh = min(a.hpu, a.r - pc.hb * a.hpu);
            const int lo = plan.wlo[pc.b];  // contiguous cache: granule 1, the unit starts at lo
            const int row0 = (pc.b * a.h_kv + pc.g) * a.T_max + lo;
            for (int t = pc.k0; t < pc.k1; t += kTile) {
              if (!mbar_wait(smem_u32(&bars[C::kStages + stage]), phase ^ 1u, a.err)) { ok = false; break; }
              const uint32_t full = arm(pc, t, slot, nh, C::kStageBytes, 0);
              const uint32_t kdst = smem_u32(stage_base + stage * C::kStageBytes);
              const uint32_t vdst = kdst + C::kTileBytes;
#pragma unroll
              for (int ch = 0; ch < C::kNch; ++ch) {
                tma_load_2d(kdst + ch * C::kChunkBytes, &tmk, full, ch * 64, row0 + t);
                tma_load_2d(vdst + ch * C::kChunkBytes, &tmv, full, ch * 64, row0 + t);
              }
              advance();
            }
            x = pc.end;
          }
          chunk = next;
          if (chunk < plan.n_chunks) next = G + atomicAdd(&a.hdr->ticket, 1);
        }
      }
    } else {
      // Paged cache: the whole warp runs the loop. Each lane holds the block-table entry of one
      // 16-key sub-tile of a 32-sub-tile window (8 tiles); the next window's entries are loaded
      // when a window starts, so the table's latency is hidden behind 8 tiles of copies instead of
      // sitting between consecutive tiles. Lane 0 takes each tile's four rows by shuffle and
      // issues the copies: one 16-row box per sub-tile (16 rows x 128 B = 2 KiB keeps the 1 KiB
      // swizzle atoms aligned, so the stage has the layout of one 64-row box). Sub-tiles past the
      // tile's valid keys are not loaded (the consumer warp owning such a slice skips it).
      int chunk = blockIdx.x;
      int next = 0;
      if (lane == 0) next = dyn && chunk < plan.n_chunks ? G + atomicAdd(&a.hdr->ticket, 1) : plan.n_chunks;
      next = __shfl_sync(0xffffffffu, next, 0);
      for (; ok && chunk < plan.n_chunks;) {
        const long long x1 = min((long long)(chunk + 1) * plan.C, plan.K);
        for (long long x = (long long)chunk * plan.C; x < x1 && ok;) {
          const Piece pc = locate(plan, a.B, a.hblocks, x, x1);
          const int slot = pc.n_pieces == 1 ? -1 : chunk + pc.unit;
          const int nh = min(a.hpu, a.r - pc.hb * a.hpu);
          const int32_t* bt = a.block_table + (long long)pc.b * a.max_pages;
          // keys are absolute positions koff + t: the unit starts at the window start rounded
          // down to the granule (a multiple of 16), and its first nskip keys are masked
          const int lo = plan.wlo[pc.b];
          const int koff = lo / a.gran * a.gran;
          const int nskip = lo - koff;
          const int s_end = (koff + pc.k1 + 15) >> 4;  // sub-tiles: [(koff + k0) / 16, s_end)
          // raw table entry of sub-tile s (-1 past the piece: never used)
          auto fetch = [&](int s) -> int { return s < s_end ? __ldg(bt + (s << 4) / a.page_size) : -1; };
          // pool row of sub-tile s from its table entry; an entry outside the pool is flagged and
          // replaced by page 0
          auto to_row = [&](int page, int s) -> int {
            if (s >= s_end) return 0;
            if (page < 0 || page >= a.num_pages) {
              set_device_error(a.err, GQA_DEVERR_PAGE);
              page = 0;
            }
            return (page * a.h_kv + pc.g) * a.page_size + (s << 4) % a.page_size;
          };
          int wbase = (koff + pc.k0) >> 4;  // first sub-tile of the current window
          int cur = to_row(fetch(wbase + lane), wbase + lane);
          int nxt = fetch(wbase + 32 + lane);
          for (int t = pc.k0; t < pc.k1; t += kTile) {
            const int s = (koff + t) >> 4;
            if (s >= wbase + 32) {
              wbase += 32;
              cur = to_row(nxt, wbase + lane);
              nxt = fetch(wbase + 32 + lane);
            }
            int prow[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) prow[j] = __shfl_sync(0xffffffffu, cur, (s - wbase + j) & 31);
            int good = 1;
            if (lane == 0) good = mbar_wait(smem_u32(&bars[C::kStages + stage]), phase ^ 1u, a.err) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, good, 0)) { ok = false; break; }
            if (lane == 0) {
              const uint32_t kdst = smem_u32(stage_base + stage * C::kStageBytes);
              const uint32_t vdst = kdst + C::kTileBytes;
              if (kMode == kPaged2d && a.gran == kTile) {
                // pages hold a multiple of 64 keys and tiles start on multiples of 64: the whole
                // tile lies in one page and loads as one 64-row box per column chunk
                const uint32_t full = arm(pc, t, slot, nh, C::kStageBytes, nskip);
#pragma unroll
                for (int ch = 0; ch < C::kNch; ++ch) {
                  tma_load_2d(kdst + ch * C::kChunkBytes, &tmk, full, ch * 64, prow[0]);
                  tma_load_2d(vdst + ch * C::kChunkBytes, &tmv, full, ch * 64, prow[0]);
                }
              } else {
                const int nsub = (min(kTile, pc.k1 - t) + 15) >> 4;
                const uint32_t full = arm(pc, t, slot, nh, (uint32_t)nsub * (C::kStageBytes / 4), nskip);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  if (j >= nsub) break;
                  if constexpr (kMode == kPaged3d) {
                    tma_load_3d(kdst + j * C::kSubBytes, &tmk, full, 0, prow[j], 0);
                    tma_load_3d(vdst + j * C::kSubBytes, &tmv, full, 0, prow[j], 0);
                  } else {
#pragma unroll
                    for (int ch = 0; ch < C::kNch; ++ch) {
                      tma_load_2d(kdst + ch * C::kChunkBytes + j * 2048, &tmk, full, ch * 64, prow[j]);
                      tma_load_2d(vdst + ch * C::kChunkBytes + j * 2048, &tmv, full, ch * 64, prow[j]);
                    }
                  }
                }
              }
            }
            __syncwarp();
            advance();
          }
          x = pc.end;
        }
        chunk = next;
        if (chunk < plan.n_chunks) {
          if (lane == 0) next = G + atomicAdd(&a.hdr->ticket, 1);
          next = __shfl_sync(0xffffffffu, next, 0);
        }
      }
    }

    if (lane == 0) {
      if (ok && mbar_wait(smem_u32(&bars[C::kStages + stage]), phase ^ 1u, a.err)) {
        meta[stage].flags = kEnd;  // tells the consumers to stop
        mbar_arrive(smem_u32(&bars[stage]));
        ++issued;
      }
      // Drain (bounded): wait until the last kStages fills were consumed, so no copy is in flight
      // into shared memory when the CTA exits.
      for (int f = issued > C::kStages ? issued - C::kStages : 0; f < issued; ++f) {
        if (!mbar_wait(smem_u32(&bars[C::kStages + f % C::kStages]), (uint32_t)(f / C::kStages) & 1u, a.err))
          break;
      }
    }
    return;
  }

  // ------------------------------- consumer warps -------------------------------------------
  const int mt = warp / 4;  // m-tile (16 query rows)
  const int ws = warp % 4;  // key slice inside each 64-key tile
  const int gid = lane >> 2, tq = lane & 3;
  const int mt_tid = threadIdx.x - mt * 128;
  const float sl2 = a.scale * kLog2e;
  constexpr int NK = D / 16;  // k-steps of Q K^T
  constexpr int NN = D / 8;   // n-tiles of P V

  // K/V addressing in a stage: chunk planes of 64 rows, or (kPaged3d) one block per 16-key
  // sub-tile, which is this warp's own slice ws
  constexpr bool kSub = kMode == kPaged3d;
  constexpr int kKvChunkStride = kSub ? 16 * 128 : C::kChunkBytes;
  const uint32_t kv_warp_off = kSub ? ws * C::kSubBytes : 0;
  const int kv_row_mask = kSub ? 15 : 63;

  int stage = 0;
  uint32_t phase = 0;
  uint32_t qf[NK][4];
  float acc[NN][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  while (true) {
    // ldmatrix / mma.sync below need the whole warp: leave together if the wait ran out
    if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bars[stage]), phase, a.err))) return;
    const TileMeta m = meta[stage];
    if (m.flags & kEnd) {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars[C::kStages + stage]));
      break;
    }
    const uint32_t kb = smem_u32(stage_base + stage * C::kStageBytes);
    const uint32_t vb = kb + C::kTileBytes;
    if (m.flags & kFirst) {
      // query fragments of this m-tile from the staged query rows (rows = heads of the unit)
      const uint32_t qb = smem_u32(q_base + stage * C::kQBytes);
      const int i = lane >> 3;
      const int qr = mt * 16 + (i & 1) * 8 + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < NK; ++ks) {
        const int d8 = ks * 2 + (i >> 1);
        ldsm_x4(swz128(qb + (d8 >> 3) * C::kQChunkBytes, qr, d8 & 7), qf[ks][0], qf[ks][1],
                qf[ks][2], qf[ks][3]);
      }
#pragma unroll
      for (int n = 0; n < NN; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
    }
    const int nvalid = m.nvalid;
    const int nskip = m.nskip;
    const int klo = ws * 16;
    if (klo < nvalid && klo + 16 > nskip) {
      // ---- S = Q K^T for keys klo .. klo+15 (two n-tiles of 8 keys)
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int krow = klo + ((lane >> 4) << 3) + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < NK; ++ks) {
          const int d8 = ks * 2 + ((lane >> 3) & 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(swz128(kb + kv_warp_off + (d8 >> 3) * kKvChunkStride, krow & kv_row_mask, d8 & 7),
                  b0, b1, b2, b3);
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
          const bool vis = key < nvalid && key >= nskip;
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
      const bool partial = klo + 16 > nvalid || klo < nskip;
      const int vrow = klo + ((lane >> 3) & 1) * 8 + (lane & 7);
      const int key_a = klo + 2 * tq, key_b = klo + 8 + 2 * tq;
#pragma unroll
      for (int n2 = 0; n2 < NN / 2; ++n2) {
        const int d8 = n2 * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(swz128(vb + kv_warp_off + (d8 >> 3) * kKvChunkStride, vrow & kv_row_mask, d8 & 7),
                  b0, b1, b2, b3);
        if (partial) {
          b0 = mask_pair(b0, key_a, nskip, nvalid);
          b1 = mask_pair(b1, key_b, nskip, nvalid);
          b2 = mask_pair(b2, key_a, nskip, nvalid);
          b3 = mask_pair(b3, key_b, nskip, nvalid);
        }
        mma_bf16(acc[2 * n2], pa, b0, b1);
        mma_bf16(acc[2 * n2 + 1], pa, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[C::kStages + stage]));
    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
    if (!(m.flags & kLast)) continue;

    // ---- piece end: merge the four key slices of this m-tile, normalise, emit
    const float l0s = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
    const float l0t = l0s + __shfl_xor_sync(0xffffffffu, l0s, 2);
    const float l1s = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
    const float l1t = l1s + __shfl_xor_sync(0xffffffffu, l1s, 2);
    float* sm = st_m + mt * 64;
    float* sl = st_l + mt * 64;
    // the four lanes of a row hold the same m and l: all store (the same values), so the warp
    // reaches the barrier with no lane-divergent code in front of it
    sm[ws * 16 + gid] = m0;
    sm[ws * 16 + gid + 8] = m1;
    sl[ws * 16 + gid] = l0t;
    sl[ws * 16 + gid + 8] = l1t;
    named_barrier_sync(1 + mt, 128);
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
    const float* r0p = red + (mt * 4) * 16 * C::kRedStride;
    // 64 columns per pass: the four slices' rescaled rows go through shared memory and are summed
#pragma unroll
    for (int pass = 0; pass < D / 64; ++pass) {
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int col = n * 8 + 2 * tq;
        const int nn = pass * 8 + n;
        *reinterpret_cast<float2*>(rb + gid * C::kRedStride + col) =
            make_float2(acc[nn][0] * f0, acc[nn][1] * f0);
        *reinterpret_cast<float2*>(rb + (gid + 8) * C::kRedStride + col) =
            make_float2(acc[nn][2] * f1, acc[nn][3] * f1);
      }
      named_barrier_sync(1 + mt, 128);
      for (int e = mt_tid; e < 16 * 64; e += 128) {
        const int row = e >> 6, c = e & 63;
        const int hl = mt * 16 + row;
        if (hl >= m.nh) continue;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) v += r0p[(w * 16 + row) * C::kRedStride + c];
        const int col = pass * 64 + c;
        float lse2 = 0.f;
        if (col == 0) {  // base-2 log-sum-exp of the piece for this row
          float M = -INFINITY, L = 0.f;
          for (int w = 0; w < 4; ++w) M = fmaxf(M, sm[w * 16 + row]);
          for (int w = 0; w < 4; ++w) L += fast_exp2(sm[w * 16 + row] - M) * sl[w * 16 + row];
          lse2 = M + __log2f(L);
        }
        emit<__nv_bfloat16>(a, m.b, m.g, m.hb, m.slot, hl, col, v, lse2);
      }
      named_barrier_sync(1 + mt, 128);
    }
  }
}

// =============================================================================================
// MLA decode (bf16): every head of a sequence against its shared latent cache rows
// =============================================================================================
// A cache row is [latent C (512) | decoupled rotary key (64)]; the query row of a head is the
// absorbed latent query and its rotary part (576); the value is the row's first 512 entries
// [第 09 章 GQA、MLA 与跨层 KV 共享, section 09.3: Q (C U_K)^T = (Q U_K^T) C^T and
// P (C U_V) = (P C) U_V; 第三章, section 3.4 on the decoupled position key]. A unit is 16 heads
// of one sequence; its keys go through the same split-KV chunks, partials and merge as GQA
// decode. Per 64-key tile (9 column chunks of 64, staged by TMA) eight consumer warps:
//   S   warp w scores keys [8w, 8w+8) for the 16 heads over all 576 columns (m16n8k16);
//   max the row maxima of the eight warps meet in shared memory, so all warps share one running
//       maximum per head; P = 2^(s - m) goes to shared memory as bf16;
//   PV  warp w accumulates latent columns [64w, 64w+64) of O += P V over the 64 keys, reading V
//       as the tile's first eight column chunks.
constexpr int kMlaDqk = 576, kMlaDv = 512, kMlaHeads = 16;
// k-steps of the query kept in registers (9 warps: at most 168 registers each; 16 does not spill)
constexpr int kMlaQReg = 16;
struct MlaCfg {
  static constexpr int kStages = 2;  // also the number of query slots (see the producer)
  static constexpr int kNch = kMlaDqk / 64;              // 9 column chunks of a cache row
  static constexpr int kChunkBytes = kTile * 128;        // 64 rows x 128 B
  static constexpr int kTileBytes = kNch * kChunkBytes;  // 72 KiB
  static constexpr int kQChunkBytes = kMlaHeads * 128;
  static constexpr int kQBytes = kNch * kQChunkBytes;    // 18 KiB
  static constexpr int kConsumerWarps = 8;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kPBytes = kMlaHeads * 128;        // 16 heads x 64 keys, bf16, swizzled
  static constexpr int kRedBytes = 2 * kConsumerWarps * kMlaHeads * 4;
  static constexpr size_t kSmem = (size_t)kStages * (kTileBytes + kQBytes) + kPBytes + kRedBytes +
                                  (kMaxBatch + 1) * 8 + 2 * kMaxBatch * 4 + kStages * sizeof(TileMeta) +
                                  2 * kStages * 8 + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

__global__ void __launch_bounds__(MlaCfg::kThreads, 1)
    mla_bf16_kernel(const __grid_constant__ CUtensorMap tmc, const __grid_constant__ CUtensorMap tmq,
                    KArgs a) {
  using C = MlaCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* q_base = smem + C::kStages * C::kTileBytes;
  uint8_t* p_buf = q_base + C::kStages * C::kQBytes;
  float* red_m = reinterpret_cast<float*>(p_buf + C::kPBytes);  // [warp][head]
  float* red_l = red_m + C::kConsumerWarps * kMlaHeads;
  long long* pre = reinterpret_cast<long long*>(red_l + C::kConsumerWarps * kMlaHeads);
  int* nlen = reinterpret_cast<int*>(pre + kMaxBatch + 1);
  int* wlo = nlen + kMaxBatch;
  TileMeta* meta = reinterpret_cast<TileMeta*>(wlo + kMaxBatch);
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta + C::kStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int producer_warp = C::kConsumerWarps;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[C::kStages + s]), C::kConsumerWarps);
    }
    fence_barrier_init();
  }
  if (warp == producer_warp && lane == 0) {
    tma_prefetch_desc(&tmc);
    tma_prefetch_desc(&tmq);
  }
  pdl_wait();  // launched as a programmatic dependent: no input is read before this
  Plan plan;
  build_plan<__nv_bfloat16>(a, plan, pre, nlen, wlo, warp, lane, producer_warp);
  pdl_launch_dependents();

  if (warp == producer_warp) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      const int G = gridDim.x;
      const bool dyn = plan.n_chunks > G;
      int chunk = blockIdx.x;
      int next = dyn && chunk < plan.n_chunks ? G + atomicAdd(&a.hdr->ticket, 1) : plan.n_chunks;
      // the query rows of a piece stay in one of two slots for all of its tiles; pieces alternate
      // slots, and with two stages the piece two back has been consumed before its slot refills
      int qslot = 0;
      for (; ok && chunk < plan.n_chunks;) {
        const long long x1 = min((long long)(chunk + 1) * plan.C, plan.K);
        for (long long x = (long long)chunk * plan.C; x < x1 && ok; qslot ^= 1) {
          const Piece pc = locate(plan, a.B, a.hblocks, x, x1);
          const int slot = pc.n_pieces == 1 ? -1 : chunk + pc.unit;
          const int nh = min(a.hpu, a.r - pc.hb * a.hpu);
          const int row0 = pc.b * a.T_max + plan.wlo[pc.b];
          const int qrow = pc.b * a.h_q + pc.hb * a.hpu;
          for (int t = pc.k0; t < pc.k1; t += kTile) {
            if (!mbar_wait(smem_u32(&bars[C::kStages + stage]), phase ^ 1u, a.err)) { ok = false; break; }
            const bool first = t == pc.k0;
            TileMeta m;
            m.b = pc.b;
            m.g = qslot;  // MLA has one KV "head": g carries the piece's query slot
            m.hb = pc.hb;
            m.nvalid = min(kTile, pc.k1 - t);
            m.flags = (first ? kFirst : 0) | (t + kTile >= pc.k1 ? kLast : 0);
            m.slot = slot;
            m.nh = nh;
            m.nskip = 0;
            meta[stage] = m;
            const uint32_t full = smem_u32(&bars[stage]);
            mbar_arrive_expect_tx(full, C::kTileBytes + (first ? C::kQBytes : 0));
            const uint32_t kdst = smem_u32(stage_base + stage * C::kTileBytes);
#pragma unroll
            for (int ch = 0; ch < C::kNch; ++ch)
              tma_load_2d(kdst + ch * C::kChunkBytes, &tmc, full, ch * 64, row0 + t);
            if (first) {
              const uint32_t qdst = smem_u32(q_base + qslot * C::kQBytes);
#pragma unroll
              for (int ch = 0; ch < C::kNch; ++ch)
                tma_load_2d(qdst + ch * C::kQChunkBytes, &tmq, full, ch * 64, qrow);
            }
            ++issued;
            if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
          }
          x = pc.end;
        }
        chunk = next;
        if (chunk < plan.n_chunks) next = G + atomicAdd(&a.hdr->ticket, 1);
      }
      if (ok && mbar_wait(smem_u32(&bars[C::kStages + stage]), phase ^ 1u, a.err)) {
        meta[stage].flags = kEnd;
        mbar_arrive(smem_u32(&bars[stage]));
        ++issued;
      }
      for (int f = issued > C::kStages ? issued - C::kStages : 0; f < issued; ++f) {
        if (!mbar_wait(smem_u32(&bars[C::kStages + f % C::kStages]), (uint32_t)(f / C::kStages) & 1u, a.err))
          break;
      }
    }
    return;
  }

  // ------------------------------- consumer warps -------------------------------------------
  const int w = warp;
  const int gid = lane >> 2, tq = lane & 3;
  const float sl2 = a.scale * kLog2e;
  const uint32_t pb = smem_u32(p_buf);
  int stage = 0;
  uint32_t phase = 0;
  float acc[8][4];
  uint32_t qf[kMlaQReg][4];  // the unit's 16 query rows as A fragments, first kMlaQReg k-steps
  uint32_t qb = 0;           // the piece's query slot (the remaining k-steps are read from it)
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  while (true) {
    if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bars[stage]), phase, a.err))) return;
    const TileMeta m = meta[stage];
    if (m.flags & kEnd) {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars[C::kStages + stage]));
      break;
    }
    const uint32_t kb = smem_u32(stage_base + stage * C::kTileBytes);
    if (m.flags & kFirst) {
      qb = smem_u32(q_base + m.g * C::kQBytes);
      const int i = lane >> 3;
      const int qr = (i & 1) * 8 + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < kMlaQReg; ++ks) {
        const int d8q = ks * 2 + (i >> 1);
        ldsm_x4(swz128(qb + (d8q >> 3) * C::kQChunkBytes, qr, d8q & 7), qf[ks][0], qf[ks][1], qf[ks][2],
                qf[ks][3]);
      }
#pragma unroll
      for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
    }
    const int nvalid = m.nvalid, nskip = m.nskip;
    // ---- S = Q K^T for keys [8w, 8w + 8), all 576 columns (36 k-steps, two per ldmatrix of K)
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kp = 0; kp < kMlaDqk / 32; ++kp) {
      const int d8 = 4 * kp + (lane >> 3);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(swz128(kb + (d8 >> 3) * C::kChunkBytes, 8 * w + (lane & 7), d8 & 7), b0, b1, b2, b3);
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const int ks = 2 * kp + s2;
        if (ks < kMlaQReg) {
          mma_bf16(sc, qf[ks < kMlaQReg ? ks : 0], s2 ? b2 : b0, s2 ? b3 : b1);
        } else {
          const int i = lane >> 3;
          const int d8q = ks * 2 + (i >> 1);
          uint32_t qa[4];
          ldsm_x4(swz128(qb + (d8q >> 3) * C::kQChunkBytes, (i & 1) * 8 + (lane & 7), d8q & 7), qa[0], qa[1],
                  qa[2], qa[3]);
          mma_bf16(sc, qa, s2 ? b2 : b0, s2 ? b3 : b1);
        }
      }
    }
    // ---- mask, base-2 scale, the eight warps' row maxima -> one running maximum per head
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int key = 8 * w + 2 * tq + e;
      const bool vis = key < nvalid && key >= nskip;
      sc[e] = vis ? sc[e] * sl2 : -INFINITY;
      sc[2 + e] = vis ? sc[2 + e] * sl2 : -INFINITY;
      mx0 = fmaxf(mx0, sc[e]);
      mx1 = fmaxf(mx1, sc[2 + e]);
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    if (tq == 0) {
      red_m[w * kMlaHeads + gid] = mx0;
      red_m[w * kMlaHeads + gid + 8] = mx1;
    }
    named_barrier_sync(1, 32 * C::kConsumerWarps);
    float t0 = -INFINITY, t1 = -INFINITY;
#pragma unroll
    for (int v = 0; v < C::kConsumerWarps; ++v) {
      t0 = fmaxf(t0, red_m[v * kMlaHeads + gid]);
      t1 = fmaxf(t1, red_m[v * kMlaHeads + gid + 8]);
    }
    const float mn0 = fmaxf(m0, t0), mn1 = fmaxf(m1, t1);  // finite: every tile has a visible key
    const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    const float p00 = fast_exp2(sc[0] - mn0), p01 = fast_exp2(sc[1] - mn0);
    const float p10 = fast_exp2(sc[2] - mn1), p11 = fast_exp2(sc[3] - mn1);
    float ps0 = p00 + p01, ps1 = p10 + p11;
    ps0 += __shfl_xor_sync(0xffffffffu, ps0, 1);
    ps0 += __shfl_xor_sync(0xffffffffu, ps0, 2);
    ps1 += __shfl_xor_sync(0xffffffffu, ps1, 1);
    ps1 += __shfl_xor_sync(0xffffffffu, ps1, 2);
    l0 = fmaf(l0, al0, ps0);  // this warp's share of the row sums (its 8 keys), common maximum
    l1 = fmaf(l1, al1, ps1);
    // P (bf16) into shared memory: row = head, keys 8w + 2tq, +1 are 4 bytes of 16-byte unit w
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(swz128(pb, gid, w) + 4 * tq), "r"(pack_bf16x2(p00, p01)) : "memory");
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(swz128(pb, gid + 8, w) + 4 * tq), "r"(pack_bf16x2(p10, p11)) : "memory");
    named_barrier_sync(2, 32 * C::kConsumerWarps);
    // ---- O[:, 64w .. 64w+64) += P V over the tile's 64 keys
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      acc[n][0] *= al0;
      acc[n][1] *= al0;
      acc[n][2] *= al1;
      acc[n][3] *= al1;
    }
    const bool partial = nvalid < kTile || nskip > 0;
#pragma unroll
    for (int ks = 0; ks < kTile / 16; ++ks) {
      uint32_t pa[4];
      {
        const int i = lane >> 3;
        const int pr = (i & 1) * 8 + (lane & 7);
        ldsm_x4(swz128(pb, pr, ks * 2 + (i >> 1)), pa[0], pa[1], pa[2], pa[3]);
      }
      const int vrow = 16 * ks + ((lane >> 3) & 1) * 8 + (lane & 7);
      const int key_a = 16 * ks + 2 * tq, key_b = key_a + 8;
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {
        const int d8 = 8 * w + n2 * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(swz128(kb + (d8 >> 3) * C::kChunkBytes, vrow, d8 & 7), b0, b1, b2, b3);
        if (partial) {
          b0 = mask_pair(b0, key_a, nskip, nvalid);
          b1 = mask_pair(b1, key_b, nskip, nvalid);
          b2 = mask_pair(b2, key_a, nskip, nvalid);
          b3 = mask_pair(b3, key_b, nskip, nvalid);
        }
        mma_bf16(acc[2 * n2], pa, b0, b1);
        mma_bf16(acc[2 * n2 + 1], pa, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[C::kStages + stage]));
    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
    if (!(m.flags & kLast)) continue;

    // ---- piece end: row sums over the eight warps, normalise, emit latent columns [64w, 64w+64)
    if (tq == 0) {
      red_l[w * kMlaHeads + gid] = l0;
      red_l[w * kMlaHeads + gid + 8] = l1;
    }
    named_barrier_sync(3, 32 * C::kConsumerWarps);
    float L0 = 0.f, L1 = 0.f;
#pragma unroll
    for (int v = 0; v < C::kConsumerWarps; ++v) {
      L0 += red_l[v * kMlaHeads + gid];
      L1 += red_l[v * kMlaHeads + gid + 8];
    }
    const float inv0 = 1.f / L0, inv1 = 1.f / L1;
    const float lse0 = m0 + __log2f(L0), lse1 = m1 + __log2f(L1);
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int col = 64 * w + 8 * n + 2 * tq;
      if (gid < m.nh) {
        emit<__nv_bfloat16>(a, m.b, 0, m.hb, m.slot, gid, col, acc[n][0] * inv0, lse0);
        emit<__nv_bfloat16>(a, m.b, 0, m.hb, m.slot, gid, col + 1, acc[n][1] * inv0, lse0);
      }
      if (gid + 8 < m.nh) {
        emit<__nv_bfloat16>(a, m.b, 0, m.hb, m.slot, gid + 8, col, acc[n][2] * inv1, lse1);
        emit<__nv_bfloat16>(a, m.b, 0, m.hb, m.slot, gid + 8, col + 1, acc[n][3] * inv1, lse1);
      }
    }
  }
}

// =============================================================================================
// MLA decode on the tensor cores (bf16, 128 heads per unit)
// =============================================================================================
// With 128 heads the score and value products are dense enough for tcgen05: the unit's 128
// heads sit on the 128 TMEM lanes (M = 128) and each 32-key tile of latent rows is the B operand
//   S  = Q C^T   (M 128, N 32 keys, K 576)   into TMEM columns [0, 32) and [32, 64) (two halves
//                                            of the contraction, added by the softmax warps)
//   O += P C_v   (M 128, N 256, K 32 keys)   into TMEM columns [64, 320)
// The 512-wide latent accumulator is twice what TMEM holds next to S, so a unit's chunk is run by
// two CTAs, each owning 256 of the latent columns (d_v half); both compute the same S (the same
// bits: the same MMAs on the same inputs), and each writes its half of the piece output.
// TMEM: S [0, 64), O half [64, 320), the query's first 384 columns [320, 512) (the A operand of
// the first 24 k-steps of S); the query's last 192 columns stay in shared memory (the A operand of
// the other 12). P (bf16) goes to shared memory, so the next tile's S overwrites the scores as soon
// as the softmax warps have read them and runs while they compute P. The tiles pass through a
// 4-deep ring of 36 KiB stages, so a tile's copy starts three tiles ahead of its use.
// Warps: 0 TMA producer; 1 issues k-steps 0-17 of S and P V (and owns TMEM); 6 issues k-steps
// 18-35 of S (an MMA issue returns only after tens of cycles, and at N = 32 one issuing thread
// left the tensor pipe mostly idle); 2..5 softmax, one TMEM lane quarter each (warp w reads lanes
// 32 (w % 4) ..), one head per thread.
// Chunks: CTAs 2p and 2p + 1 take chunks p, p + G/2, ... of the same split-KV plan as the other
// decode kernels (with equal-length sequences, chunks that divide each sequence: see the plan);
// partials and the merge kernel are shared with them.
constexpr int kMlaTcHeads = 128;
constexpr int kMlaTcMinChunk = 256;  // keys; the automatic chunking never goes below this
constexpr int kMlaTcKeys = 32;       // keys per tile
struct MlaTcCfg {
  static constexpr int kStages = 4;
  static constexpr int kNch = kMlaDqk / 64;                // 9 column chunks of a latent row
  static constexpr int kChunkBytes = kMlaTcKeys * 128;     // 32 rows x 128 B
  static constexpr int kTileBytes = kNch * kChunkBytes;    // 36 KiB
  static constexpr int kQTmemCh = 6;                       // query chunks held in TMEM (384 columns)
  static constexpr int kQSmemCh = kNch - kQTmemCh;         // 3 in shared memory
  static constexpr int kQChunkBytes = kMlaTcHeads * 128;   // 128 rows x 128 B
  static constexpr int kQBytes = kQSmemCh * kQChunkBytes;  // 48 KiB
  static constexpr int kPBytes = kMlaTcHeads * 128;        // 128 rows of 128 B; a tile's P uses 64 B
  static constexpr int kThreads = 224;
  static constexpr int kKSplit = 18;  // k-steps of S issued by warp 1; warp 6 issues the other 18
  static constexpr uint32_t kColS = 0, kColS2 = 32, kColO = 64, kColQ = 320;
  static constexpr int kHalf = kMlaDv / 2;                 // latent columns per CTA
  enum { kFull = 0, kEmpty = kFull + kStages, kQInfo = kEmpty + kStages, kQFull, kQTmem, kSFull, kSFull2,
         kSFree, kPFull, kPvDone, kPieceDone, kAll, kAll2, kNever, kBars };
  static constexpr size_t kOffQ = (size_t)kStages * kTileBytes;
  static constexpr size_t kOffP = kOffQ + kQBytes;
  static constexpr size_t kOffPre = kOffP + kPBytes;
  static constexpr size_t kOffNlen = kOffPre + (kMaxBatch + 1) * 8;
  static constexpr size_t kOffWlo = kOffNlen + kMaxBatch * 4;
  static constexpr size_t kOffMeta = kOffWlo + kMaxBatch * 4;
  static constexpr size_t kOffBar = kOffMeta + kStages * sizeof(TileMeta);
  static constexpr size_t kSmem = kOffBar + kBars * 8 + 1024;  // + alignment of the base
  static_assert(kSmem + 16 <= 227 * 1024, "shared memory budget");
};

__global__ void __launch_bounds__(MlaTcCfg::kThreads, 1)
    mla_tc_kernel(const __grid_constant__ CUtensorMap tmc, const __grid_constant__ CUtensorMap tmq,
                  KArgs a) {
  using C = MlaTcCfg;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_qrow;  // the current piece's first query row (b * h_q + first head), -1: the end
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  long long* pre = reinterpret_cast<long long*>(smem + C::kOffPre);
  int* nlen = reinterpret_cast<int*>(smem + C::kOffNlen);
  int* wlo = reinterpret_cast<int*>(smem + C::kOffWlo);
  TileMeta* meta = reinterpret_cast<TileMeta*>(smem + C::kOffMeta);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  volatile int* qrow_slot = &s_qrow;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const uint32_t sQ = smem_u32(smem + C::kOffQ), sP = smem_u32(smem + C::kOffP);
  auto sC = [&](int st) { return smem_u32(smem + st * C::kTileBytes); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = blockIdx.x & 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::kFull + s), 1);
      mbar_init(bar(C::kEmpty + s), 1);
    }
    mbar_init(bar(C::kQInfo), 1);
    mbar_init(bar(C::kQFull), 1);
    mbar_init(bar(C::kQTmem), 128);
    mbar_init(bar(C::kSFull), 1);
    mbar_init(bar(C::kSFull2), 1);
    mbar_init(bar(C::kSFree), 128);
    mbar_init(bar(C::kPFull), 128);
    mbar_init(bar(C::kPvDone), 1);
    mbar_init(bar(C::kPieceDone), 1);
    mbar_init(bar(C::kAll), 1);
    mbar_init(bar(C::kAll2), 1);
    mbar_init(bar(C::kNever), 1);  // nothing arrives: the expired-wait test hook waits on it
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmc);
    tma_prefetch_desc(&tmq);
  }
  if (warp == 1) {  // all 512 columns (one CTA per SM: the shared memory sees to that)
    tc::tmem_alloc(smem_u32(&s_tmem), 512);
    tc::tmem_relinquish();
    tc::fence_before_sync();
  }
  pdl_wait();  // launched as a programmatic dependent: no input is read before this
  Plan plan;
  build_plan<__nv_bfloat16>(a, plan, pre, nlen, wlo, warp, lane, 0);  // ends with a CTA barrier
  pdl_launch_dependents();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;
  const int pairs = (int)(gridDim.x >> 1);

  if (warp == 0) {
    // ------------------------------ TMA producer (lane 0) --------------------------------------
    if (lane == 0) {
      int stage = 0, issued = 0, pieces = 0;
      uint32_t phase = 0;
      // test hook: CTA 0 first waits on a barrier that nothing signals, runs out after the bound
      // and gives up (its rows are left unspecified; every other role's first wait runs out too)
      bool ok = !(a.expire_wait && blockIdx.x == 0) || mbar_wait(bar(C::kNever), 0, a.err);
      for (int chunk = (int)(blockIdx.x >> 1); ok && chunk < plan.n_chunks; chunk += pairs) {
        const long long x1 = min((long long)(chunk + 1) * plan.C, plan.K);
        for (long long x = (long long)chunk * plan.C; x < x1 && ok;) {
          const Piece pc = locate(plan, a.B, a.hblocks, x, x1);
          const int slot = pc.n_pieces == 1 ? -1 : chunk + pc.unit;
          const int row0 = pc.b * a.T_max;
          const int qrow = pc.b * a.h_q + pc.hb * kMlaTcHeads;
          const int ntiles = (pc.k1 - pc.k0 + kMlaTcKeys - 1) / kMlaTcKeys;
          // the piece's 128 query rows (contiguous) into L2 now: the softmax warps read their
          // first 384 columns with plain loads once the previous piece is done
          prefetch_l2(reinterpret_cast<const uint8_t*>(a.q) + (long long)qrow * (kMlaDqk * 2),
                      (uint32_t)(kMlaTcHeads * kMlaDqk * 2));
          // tile i of the piece: all 9 column chunks in one 3-D copy (chunk-major in the stage)
          auto issue_tile = [&](int i) -> bool {
            if (!mbar_wait(bar(C::kEmpty + stage), phase ^ 1u, a.err)) return false;
            const int t = pc.k0 + i * kMlaTcKeys;
            TileMeta m;
            m.b = pc.b;
            m.g = 0;
            m.hb = pc.hb;
            m.nvalid = min(kMlaTcKeys, pc.k1 - t);
            m.flags = (i == 0 ? kFirst : 0) | (i == ntiles - 1 ? kLast : 0);
            m.slot = slot;
            m.nh = kMlaTcHeads;
            m.nskip = 0;
            meta[stage] = m;
            mbar_arrive_expect_tx(bar(C::kFull + stage), (uint32_t)C::kTileBytes);
            tma_load_3d(sC(stage), &tmc, bar(C::kFull + stage), 0, row0 + t, 0);
            ++issued;
            if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
            return true;
          };
          // Up to kStages tiles of a later piece go out before its query: the stages they take
          // were held by earlier pieces' tiles, whose consumption needs nothing of this piece.
          const int early = pieces > 0 ? min(C::kStages, ntiles) : 0;
          for (int i = 0; i < early && ok; ++i) ok = issue_tile(i);
          if (!ok) break;
          // The previous piece's MMAs (the last readers of the query buffers) are complete, and
          // every consumer has passed its piece start (so no barrier phase below is skipped).
          if (pieces > 0 && !(ok = mbar_wait(bar(C::kPieceDone), (uint32_t)((pieces - 1) & 1), a.err))) break;
          *qrow_slot = qrow;
          mbar_arrive(bar(C::kQInfo));  // the softmax warps start the query's TMEM copy now
          mbar_arrive_expect_tx(bar(C::kQFull), (uint32_t)C::kQBytes);
          tma_load_3d(sQ, &tmq, bar(C::kQFull), 0, qrow, C::kQTmemCh);
          ++pieces;
          for (int i = early; i < ntiles && ok; ++i) ok = issue_tile(i);
          x = pc.end;
        }
      }
      // Drain (bounded) before the end markers: every copy issued has landed, so none can reach
      // shared memory after the CTA is gone. Fill f of stage f % 4 completes phase f / 4 of its
      // full barrier and no later fill follows the last four; the query rows complete phase
      // pieces - 1 of theirs.
      for (int f = issued > C::kStages ? issued - C::kStages : 0; f < issued; ++f)
        mbar_wait(bar(C::kFull + f % C::kStages), (uint32_t)(f / C::kStages) & 1u, a.err);
      if (pieces > 0) mbar_wait(bar(C::kQFull), (uint32_t)((pieces - 1) & 1), a.err);
      if (ok) {
        // the end: a piece with no rows for the softmax warps, a marker tile for the MMA warp
        if (pieces == 0 || mbar_wait(bar(C::kPieceDone), (uint32_t)((pieces - 1) & 1), a.err)) {
          *qrow_slot = -1;
          mbar_arrive(bar(C::kQInfo));
        }
        if (mbar_wait(bar(C::kEmpty + stage), phase ^ 1u, a.err)) {
          meta[stage].flags = kEnd;
          mbar_arrive(bar(C::kFull + stage));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (one elected lane) ------------------------------
    constexpr uint32_t idesc_s = tc::idesc_bf16(128, kMlaTcKeys, false);  // S: 128 heads x 32 keys
    constexpr uint32_t idesc_o = tc::idesc_bf16(128, C::kHalf, true);     // O: 128 x 256, B MN-major
    auto wait = [&](int b_, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar(b_), parity, a.err));
    };
    auto issue_s = [&](int st) {  // S_a = Q C^T over the tile's columns [0, 288) (query from TMEM)
      const uint64_t dc = tc::smem_desc(sC(st), 16, 1024);
      if (tc::elect_one()) {
#pragma unroll
        for (int k = 0; k < C::kKSplit; ++k)
          tc::mma_ts(tmem + C::kColS, tmem + C::kColQ + k * 8, dc + tc::koff(k, C::kChunkBytes), idesc_s,
                     k > 0 ? 1u : 0u);
        tc::commit(bar(C::kSFull));
      }
      __syncwarp();
    };
    int stage = 0, jg = 0, piece = 0;
    uint32_t phase = 0;
    bool pre_issued = false;  // S of the current tile was issued with the previous tile
    bool ok = true;
    while (ok) {
      if (!(ok = wait(C::kFull + stage, phase))) break;
      const TileMeta m = meta[stage];
      if (m.flags & kEnd) break;
      if (m.flags & kFirst) {
        if (!(ok = wait(C::kQFull, (uint32_t)(piece & 1)) && wait(C::kQTmem, (uint32_t)(piece & 1)))) break;
      }
      if (!pre_issued) {
        if (jg > 0 && !(ok = wait(C::kSFree, (uint32_t)((jg - 1) & 1)))) break;
        tc::fence_after_sync();
        issue_s(stage);
      }
      pre_issued = false;
      const int nstage = stage + 1 == C::kStages ? 0 : stage + 1;
      const uint32_t nphase = stage + 1 == C::kStages ? phase ^ 1u : phase;
      if (!(m.flags & kLast)) {
        // the piece's next tile, if it has landed: its scores overlap this tile's softmax; if
        // not, this tile's P V goes first, so its stage refills sooner
        if (!(ok = wait(C::kSFree, (uint32_t)(jg & 1)))) break;
        int landed = lane == 0 ? (int)mbar_test(bar(C::kFull + nstage), nphase) : 0;
        landed = __shfl_sync(0xffffffffu, landed, 0);
        if (landed) {
          tc::fence_after_sync();
          issue_s(nstage);
          pre_issued = true;
        }
      }
      if (!(ok = wait(C::kPFull, (uint32_t)(jg & 1)))) break;
      tc::fence_after_sync();
      const uint64_t dp = tc::smem_desc(sP, 16, 1024);
      const uint64_t dv = tc::smem_desc(sC(stage) + half * 4 * C::kChunkBytes, C::kChunkBytes, 1024);
      if (tc::elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kMlaTcKeys / 16; ++kk)
          tc::mma_ss(tmem + C::kColO, dp + tc::koff(kk, C::kPBytes), dv + tc::mnoff(kk), idesc_o,
                     ((m.flags & kFirst) && kk == 0) ? 0u : 1u);
        tc::commit(bar(C::kPvDone));
        tc::commit(bar(C::kEmpty + stage));
        if (m.flags & kLast) tc::commit(bar(C::kPieceDone));
      }
      __syncwarp();
      if (m.flags & kLast) ++piece;
      ++jg;
      stage = nstage;
      phase = nphase;
    }
    // every MMA issued above has completed before TMEM is released
    if (tc::elect_one()) tc::commit(bar(C::kAll));
    __syncwarp();
    mbar_wait(bar(C::kAll), 0, a.err);
  } else if (warp == 6) {
    // ------------------------------ second score issuer (one elected lane) ---------------------
    // S_b = Q C^T over the tile's columns [288, 576): an MMA issue returns only after tens of
    // cycles, so at N = 32 one thread issuing all 36 k-steps left the tensor pipe mostly idle; two
    // threads issue half each, into separate accumulators that the softmax warps add.
    constexpr uint32_t idesc_s = tc::idesc_bf16(128, kMlaTcKeys, false);
    auto wait = [&](int b_, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar(b_), parity, a.err));
    };
    int stage = 0, jg = 0, piece = 0;
    uint32_t phase = 0;
    bool ok = true;
    while (ok) {
      if (!(ok = wait(C::kFull + stage, phase))) break;
      const TileMeta m = meta[stage];
      if (m.flags & kEnd) break;
      if (m.flags & kFirst) {
        if (!(ok = wait(C::kQFull, (uint32_t)(piece & 1)) && wait(C::kQTmem, (uint32_t)(piece & 1)))) break;
      }
      if (jg > 0 && !(ok = wait(C::kSFree, (uint32_t)((jg - 1) & 1)))) break;  // S_b(jg - 1) read
      tc::fence_after_sync();
      const uint64_t dc = tc::smem_desc(sC(stage), 16, 1024), dq = tc::smem_desc(sQ, 16, 1024);
      if (tc::elect_one()) {
#pragma unroll
        for (int k = C::kKSplit; k < 4 * C::kQTmemCh; ++k)  // query columns [288, 384) from TMEM
          tc::mma_ts(tmem + C::kColS2, tmem + C::kColQ + k * 8, dc + tc::koff(k, C::kChunkBytes), idesc_s,
                     k > C::kKSplit ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < 4 * C::kQSmemCh; ++k)  // [384, 576) from shared memory
          tc::mma_ss(tmem + C::kColS2, dq + tc::koff(k, C::kQChunkBytes),
                     dc + tc::koff(4 * C::kQTmemCh + k, C::kChunkBytes), idesc_s, 1u);
        tc::commit(bar(C::kSFull2));
      }
      __syncwarp();
      if (m.flags & kLast) ++piece;
      ++jg;
      if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
    }
    if (tc::elect_one()) tc::commit(bar(C::kAll2));
    __syncwarp();
    mbar_wait(bar(C::kAll2), 0, a.err);
  } else {
    // ------------------------------ softmax: one head (TMEM lane) per thread --------------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const int et = (warp - 2) * 32 + lane;  // 0..127, for the V-row zeroing
    const float sl2 = a.scale * kLog2e;
    // this head's query columns [0, 384) -> TMEM, two 64-column chunks per round of loads; the
    // caller has seen every score of the previous piece, so no MMA still reads these columns
    auto copy_query = [&](int qrow) {
      const uint4* qg = reinterpret_cast<const uint4*>(a.q) + (long long)(qrow + row) * (kMlaDqk / 8);
#pragma unroll
      for (int bc = 0; bc < C::kQTmemCh; bc += 2) {
        uint4 v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] = __ldg(qg + bc * 8 + u);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            r[4 * u] = v[8 * c + u].x;
            r[4 * u + 1] = v[8 * c + u].y;
            r[4 * u + 2] = v[8 * c + u].z;
            r[4 * u + 3] = v[8 * c + u].w;
          }
          tc::st32(lane_addr + C::kColQ + (bc + c) * 32, r);
        }
      }
      tc::wait_st();
      tc::fence_before_sync();
      mbar_arrive(bar(C::kQTmem));
    };
    int stage = 0, jg = 0, piece = 0;
    uint32_t phase = 0;
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kQInfo), 0u, a.err));
    int qrow = ok ? *qrow_slot : -1;
    if (qrow >= 0) copy_query(qrow);
    while (qrow >= 0) {
      float m_run = -INFINITY, l_run = 0.f;
      bool last = false;
      TileMeta m;
      while (!last) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kFull + stage), phase, a.err));
        if (!ok) break;
        m = meta[stage];
        const bool first = (m.flags & kFirst) != 0;
        last = (m.flags & kLast) != 0;
        // ---- scores of this tile
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kSFull), (uint32_t)(jg & 1), a.err) &&
                                         mbar_wait(bar(C::kSFull2), (uint32_t)(jg & 1), a.err));
        if (!ok) break;
        tc::fence_after_sync();
        float s[kMlaTcKeys], s2[kMlaTcKeys];
        tc::ld32f(lane_addr + C::kColS, s);
        tc::ld32f(lane_addr + C::kColS2, s2);
        tc::wait_ld();
#pragma unroll
        for (int i = 0; i < kMlaTcKeys; ++i) s[i] += s2[i];
        tc::fence_before_sync();
        mbar_arrive(bar(C::kSFree));  // the next tile's scores may overwrite them
        const int nvalid = m.nvalid;
        float bm = -INFINITY;
#pragma unroll
        for (int i = 0; i < kMlaTcKeys; ++i) {
          s[i] = i < nvalid ? s[i] * sl2 : -INFINITY;
          bm = fmaxf(bm, s[i]);
        }
        // running maximum, raised lazily: the accumulator is rescaled only when the tile's
        // maximum passes the running one by more than 2^8 (P then stays below 2^8); the piece's
        // first tile sets it (its P V overwrites the accumulator)
        float alpha = 1.f;
        const bool raise = first || bm > m_run + 8.f;
        if (raise) {
          alpha = first ? 0.f : fast_exp2(m_run - bm);
          m_run = bm;
        }
        // the previous tile's P V has completed: P may be rewritten and O rescaled
        if (jg > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kPvDone), (uint32_t)((jg - 1) & 1), a.err));
          if (!ok) break;
          tc::fence_after_sync();
        }
        if (__any_sync(0xffffffffu, raise && !first)) {  // `first` is the same for the whole warp
#pragma unroll 1
          for (int c = 0; c < C::kHalf / 32; ++c) {
            float o[32];
            tc::ld32f(lane_addr + C::kColO + c * 32, o);
            tc::wait_ld();
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * alpha);
            tc::st32(lane_addr + C::kColO + c * 32, w);
          }
          tc::wait_st();
        }
        l_run *= alpha;
        float ls = 0.f;
        uint32_t pk[kMlaTcKeys / 2];
#pragma unroll
        for (int i = 0; i < kMlaTcKeys; i += 2) {
          const float p0 = fast_exp2(s[i] - m_run), p1 = fast_exp2(s[i + 1] - m_run);
          ls += p0 + p1;
          pk[i / 2] = pack_bf16x2(p0, p1);
        }
        l_run += ls;
#pragma unroll
        for (int u = 0; u < kMlaTcKeys / 8; ++u)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(swz128(sP, row, u)), "r"(pk[4 * u]),
                       "r"(pk[4 * u + 1]), "r"(pk[4 * u + 2]), "r"(pk[4 * u + 3])
                       : "memory");
        // rows past the piece's last key may hold anything (NaN past a length): their P is 0,
        // but 0 * NaN is NaN, so this CTA's value columns of those rows are zeroed before P V
        if (nvalid < kMlaTcKeys) {
          const int units = (kMlaTcKeys - nvalid) * 4 * 8;  // rows x 4 chunks x 8 16-byte units
          for (int e = et; e < units; e += 128) {
            const int rr = nvalid + e / 32, ch = (e / 8) & 3, u = e & 7;
            const uint32_t addr = sC(stage) + (half * 4 + ch) * C::kChunkBytes + rr * 128 + u * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
          }
        }
        tc::fence_proxy_async_smem();
        tc::fence_before_sync();
        mbar_arrive(bar(C::kPFull));
        ++jg;
        if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      // The next piece's query goes into TMEM first (this piece's scores are all read), so its
      // first scores run while this piece's output is written out.
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kQInfo), (uint32_t)((piece + 1) & 1), a.err));
      const int next = ok ? *qrow_slot : -1;
      if (next >= 0) copy_query(next);
      // ---- piece end: O / l -> the output (one piece) or a partial, this CTA's columns; the
      // next piece's first P V, which overwrites the accumulator, waits for this warp's P
      const bool done = __all_sync(0xffffffffu, mbar_wait(bar(C::kPvDone), (uint32_t)((jg - 1) & 1), a.err));
      if (done) {
        tc::fence_after_sync();
        const float inv = 1.f / l_run;
        const float lse2 = m_run + __log2f(l_run);
        const int head = m.hb * kMlaTcHeads + row;
#pragma unroll 1
        for (int c = 0; c < C::kHalf / 32; ++c) {
          float o[32];
          tc::ld32f(lane_addr + C::kColO + c * 32, o);
          tc::wait_ld();
          const int col = half * C::kHalf + c * 32;
          if (m.slot < 0) {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) +
                                                  ((long long)m.b * a.h_q + head) * kMlaDv + col);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv),
                                  pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                  pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                  pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
          } else {
            // The warp's 32 rows x 32 columns pass through its quarter of the P buffer (free: the
            // piece's last P V has completed; 128-byte rows, 16-byte units swizzled by row), so
            // each store below writes 128 contiguous bytes of 4 rows, not 16 bytes of 32.
            const uint32_t stg = sP + quarter * 4096;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(stg + lane * 128 + ((u ^ (lane & 7)) << 4)),
                           "f"(o[4 * u] * inv), "f"(o[4 * u + 1] * inv), "f"(o[4 * u + 2] * inv), "f"(o[4 * u + 3] * inv)
                           : "memory");
            __syncwarp();
            float* rows = a.part_o + ((long long)m.slot * a.hpu + quarter * 32) * kMlaDv + col;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int r = k * 4 + (lane >> 3), u = lane & 7;
              float4 v;
              asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                           : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                           : "r"(stg + r * 128 + ((u ^ (r & 7)) << 4)));
              *reinterpret_cast<float4*>(rows + (long long)r * kMlaDv + u * 4) = v;
            }
            __syncwarp();
          }
        }
        if (half == 0) {
          if (m.slot < 0) {
            if (a.lse) a.lse[(long long)m.b * a.h_q + head] = lse2 * kLn2;
          } else {
            a.part_lse[(long long)m.slot * a.hpu + row] = lse2;
          }
        }
      }
      if (!done) break;
      qrow = next;
      ++piece;
    }
  }
  // every role is done: copies landed, MMAs complete, TMEM read
  tc::fence_before_sync();
  cta_sync();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// =============================================================================================
// fp32 check-mode kernel
// =============================================================================================
constexpr int kF32Warps = 4;
constexpr int kF32MaxPerLane = 16;  // value / output width <= 512 ...
constexpr int kF32MaxQkPerLane = 24;  // ... query / key width <= 768 (MLA rows: 576)

__global__ void __launch_bounds__(32 * kF32Warps, 1) decode_fp32_kernel(KArgs a) {
  __shared__ long long pre[kMaxBatch + 1];
  __shared__ int nlen[kMaxBatch];
  __shared__ int wlo[kMaxBatch];
  __shared__ int chunk_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Plan plan;
  build_plan<float>(a, plan, pre, nlen, wlo, warp, lane, 0);
  pdl_launch_dependents();
  const int D = a.D;
  for (int iter = 0;; ++iter) {
    cta_sync();
    if (threadIdx.x == 0)
      chunk_s = iter == 0 ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(&a.hdr->ticket, 1);
    cta_sync();
    const int chunk = chunk_s;
    if (chunk >= plan.n_chunks) break;
    const long long x1 = min((long long)(chunk + 1) * plan.C, plan.K);
    for (long long x = (long long)chunk * plan.C; x < x1;) {
      const Piece pc = locate(plan, a.B, a.hblocks, x, x1);
      const int slot = pc.n_pieces == 1 ? -1 : chunk + pc.unit;
      const int nh = min(a.hpu, a.r - pc.hb * a.hpu);
      const int lo = wlo[pc.b];
      const int koff = lo / a.gran * a.gran;  // absolute position of the unit's key 0
      const int jskip = lo - koff;            // keys of the first granule before the window
      const int Dk = a.Dqk;  // query / key row width; values are the first D entries of V's rows
      const long long kv_base = ((long long)pc.b * a.h_kv + pc.g) * a.T_max * Dk;
      const float* kp = reinterpret_cast<const float*>(a.k) + kv_base;
      const float* vp = reinterpret_cast<const float*>(a.v) + kv_base;
      for (int hl = warp; hl < nh; hl += kF32Warps) {
        const int head = pc.g * a.r + pc.hb * a.hpu + hl;
        const float* q = reinterpret_cast<const float*>(a.q) + ((long long)pc.b * a.h_q + head) * Dk;
        float qr[kF32MaxQkPerLane], accv[kF32MaxPerLane];
#pragma unroll
        for (int e = 0; e < kF32MaxQkPerLane; ++e) {
          const int col = lane + 32 * e;
          qr[e] = col < Dk ? q[col] : 0.f;
        }
#pragma unroll
        for (int e = 0; e < kF32MaxPerLane; ++e) accv[e] = 0.f;
        float m = -INFINITY, l = 0.f;
        for (int jr = max(pc.k0, jskip); jr < pc.k1; ++jr) {
          const int j = koff + jr;  // absolute key position
          const float* kj = kp + (long long)j * Dk;
          const float* vj = vp + (long long)j * Dk;
          if (a.block_table) {
            int page = a.block_table[(long long)pc.b * a.max_pages + j / a.page_size];
            if (page < 0 || page >= a.num_pages) {
              if (lane == 0) set_device_error(a.err, GQA_DEVERR_PAGE);
              page = 0;
            }
            const long long row = ((long long)page * a.h_kv + pc.g) * a.page_size + j % a.page_size;
            kj = reinterpret_cast<const float*>(a.k) + row * Dk;
            vj = reinterpret_cast<const float*>(a.v) + row * Dk;
          }
          float part = 0.f;
#pragma unroll
          for (int e = 0; e < kF32MaxQkPerLane; ++e) {
            const int col = lane + 32 * e;
            if (col < Dk) part = fmaf(qr[e], kj[col], part);
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
            if (col < D) accv[e] = fmaf(accv[e], alpha, p * vj[col]);
          }
          m = m_new;
        }
        const float lse2 = (m + logf(l)) * kLog2e;
        const float inv = 1.f / l;
#pragma unroll
        for (int e = 0; e < kF32MaxPerLane; ++e) {
          const int col = lane + 32 * e;
          if (col < D) emit<float>(a, pc.b, pc.g, pc.hb, slot, hl, col, accv[e] * inv, lse2);
        }
      }
      x = pc.end;
    }
  }
}

// =============================================================================================
// host side
// =============================================================================================

template <typename OutT, bool kFast>
cudaError_t launch_merge(const KArgs& ka, cudaStream_t s) {
  const long long rows = (long long)ka.B * ka.h_kv * ka.hblocks * ka.hpu * merge_slices(ka.D);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((rows + 7) / 8));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int path = merge_path(ka.D);
  if (path == 2 && rows <= 2048) path = 3;  // 256 blocks: one wave at two blocks per SM
  void (*kern)(KArgs) = path == 0   ? merge_kernel<OutT, kFast, 0>
                        : path == 1 ? merge_kernel<OutT, kFast, 1>
                        : path == 2 ? merge_kernel<OutT, kFast, 2>
                                    : merge_kernel<OutT, kFast, 3>;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ka);
  if (e != cudaSuccess) {
    // programmatic dependent launch refused (e.g. on a stream that does not support it): fall
    // back to an ordinary launch ordered after the decode kernel
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, kern, ka);
  }
  return e;
}

// Launch `kern` as a programmatic dependent of the previous kernel on the stream (its prologue
// overlaps that kernel; the kernel waits with griddepcontrol.wait before reading any input), or
// as an ordinary launch where the stream does not support it.
template <typename... KParams, typename... Args>
cudaError_t launch_dependent(void (*kern)(KParams...), int grid, int threads, size_t smem, cudaStream_t s,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, kern, args...);
  }
  return e;
}

template <int D, int MT, int kMode>
cudaError_t launch_bf16_typed(const KArgs& ka, const CUtensorMap* tm, int grid, cudaStream_t s) {
  using C = Bf16Cfg<D, MT>;
  auto kern = decode_bf16_kernel<D, MT, kMode>;
  static bool attr_set[64] = {false};  // per device: the shared-memory opt-in is set once
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  e = launch_dependent(kern, grid, C::kThreads, C::kSmem, s, tm[0], tm[1], tm[2], ka);
  if (e != cudaSuccess) return e;
  return launch_merge<__nv_bfloat16, true>(ka, s);
}

int auto_n_max(long long K_max, int sms) {
  long long n = (K_max + kMinChunkAuto - 1) / kMinChunkAuto;
  const long long cap = (long long)kChunksPerSm * (sms > 0 ? sms : 1);
  if (n > cap) n = cap;
  return (int)(n < 1 ? 1 : n);
}

// The tensor-core MLA kernel runs each chunk on two CTAs: at most one chunk per pair of SMs.
int auto_n_max_mla_tc(long long K_max, int sms) {
  long long n = (K_max + kMlaTcMinChunk - 1) / kMlaTcMinChunk;
  const long long cap = sms / 2 > 0 ? sms / 2 : 1;
  if (n > cap) n = cap;
  return (int)(n < 1 ? 1 : n);
}

int mla_heads_per_unit(bool mla, bool mla_tc) {
  return mla ? (mla_tc ? kMlaTcHeads : kMlaHeads) : kHeadsPerUnitMax;
}

KArgs make_kargs(const DecodeArgs& a) {
  const bool auto_chunk = a.num_splits == 0;
  const int r = a.h_q / a.h_kv;
  const int hpu_max = mla_heads_per_unit(a.mla != 0, a.mla_tc != 0);
  const int hpu = r < hpu_max ? r : hpu_max;
  const int d_out = a.d_v > 0 ? a.d_v : a.d_h;
  const long long K_max = (long long)a.B * a.h_kv * ((r + hpu - 1) / hpu) * a.T_max;
  const int n_max = !auto_chunk ? a.num_splits
                    : a.mla_tc  ? auto_n_max_mla_tc(K_max, a.num_sms)
                                : auto_n_max(K_max, a.num_sms);
  const Layout L = make_layout(a.B, a.h_q, a.h_kv, d_out, n_max, hpu_max);
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
  k.r = r;
  k.T_max = a.T_max;
  k.D = d_out;
  k.Dqk = a.d_h;
  k.hpu = L.hpu;
  k.hblocks = L.hblocks;
  k.scale = a.scale;
  k.n_max = n_max;
  k.auto_chunk = auto_chunk ? 1 : 0;
  // at least 16 keys per query row, so the partial written per chunk (hpu x d_out fp32) stays
  // small against the chunk's K/V bytes; the tensor-core MLA kernel is bound by its MMAs instead
  // and wants every pair of SMs busy
  k.min_chunk = a.mla_tc ? kMlaTcMinChunk : (16 * L.hpu > kMinChunkAuto ? 16 * L.hpu : kMinChunkAuto);
  // the compute-bound tensor-core MLA kernel gives up a few idle SMs for chunks that never hold
  // two pieces; the HBM-bound kernels keep every SM streaming
  k.align_units = a.mla_tc && auto_chunk ? 1 : 0;
  k.window = a.window;
  uint8_t* ws = reinterpret_cast<uint8_t*>(a.workspace);
  k.hdr = reinterpret_cast<Header*>(ws);
  k.pre = reinterpret_cast<long long*>(ws + L.pre_off);
  k.nlen = reinterpret_cast<int*>(ws + L.nlen_off);
  k.part_lse = reinterpret_cast<float*>(ws + L.lse_off);
  k.part_o = reinterpret_cast<float*>(ws + L.o_off);
  k.err = a.err;
  k.block_table = a.block_table;
  k.max_pages = a.max_pages;
  k.page_size = a.page_size;
  k.num_pages = a.num_pages;
  k.gran = a.block_table ? (a.page_size % kTile == 0 ? kTile : 16) : 1;
  k.expire_wait = a.block_table || (a.mla && !a.mla_tc) ? 0 : a.expire_wait;
  return k;
}

}  // namespace dec

size_t decode_workspace_bytes(int B, int h_q, int h_kv, int T_max, int d_h, int num_splits,
                              int num_sms, bool mla, bool mla_tc) {
  const int r = h_q / h_kv;
  const int hpu_max = dec::mla_heads_per_unit(mla, mla_tc);
  const int hpu = r < hpu_max ? r : hpu_max;
  const long long K_max = (long long)B * h_kv * ((r + hpu - 1) / hpu) * T_max;
  const int n_max = num_splits != 0 ? num_splits
                    : mla_tc        ? dec::auto_n_max_mla_tc(K_max, num_sms)
                                    : dec::auto_n_max(K_max, num_sms);
  return dec::make_layout(B, h_q, h_kv, d_h, n_max, hpu_max).total;
}

int decode_max_batch() { return dec::kMaxBatch; }

cudaError_t launch_decode_fp32(const DecodeArgs& a, cudaStream_t s) {
  const dec::KArgs k = dec::make_kargs(a);
  dec::decode_fp32_kernel<<<a.num_sms, 32 * dec::kF32Warps, 0, s>>>(k);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return dec::launch_merge<float, false>(k, s);
}

namespace dec {
template <int kMode>
cudaError_t launch_bf16_dispatch(const KArgs& k, const CUtensorMap* tmaps, int grid, cudaStream_t s) {
  const bool two = k.hpu > 16;
  if (k.D == 128) {
    return two ? launch_bf16_typed<128, 2, kMode>(k, tmaps, grid, s)
               : launch_bf16_typed<128, 1, kMode>(k, tmaps, grid, s);
  }
  if constexpr (kMode != kPaged3d) {
    if (k.D == 64) {
      return two ? launch_bf16_typed<64, 2, kMode>(k, tmaps, grid, s)
                 : launch_bf16_typed<64, 1, kMode>(k, tmaps, grid, s);
    }
  }
  return cudaErrorInvalidValue;
}
}  // namespace dec

cudaError_t launch_decode_bf16(const DecodeArgs& a, const CUtensorMap* tmaps, cudaStream_t s) {
  const dec::KArgs k = dec::make_kargs(a);
  if (!a.block_table) return dec::launch_bf16_dispatch<dec::kContig>(k, tmaps, a.num_sms, s);
  return a.paged_3d ? dec::launch_bf16_dispatch<dec::kPaged3d>(k, tmaps, a.num_sms, s)
                    : dec::launch_bf16_dispatch<dec::kPaged2d>(k, tmaps, a.num_sms, s);
}

cudaError_t launch_mla_bf16(const DecodeArgs& a, const CUtensorMap* tmaps, cudaStream_t s) {
  const dec::KArgs k = dec::make_kargs(a);
  if (a.mla_tc) {
    using T = dec::MlaTcCfg;
    static bool tc_attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !tc_attr_set[dev]) {
      e = cudaFuncSetAttribute(dec::mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)T::kSmem);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) tc_attr_set[dev] = true;
    }
    const int pairs = k.n_max < a.num_sms / 2 ? k.n_max : a.num_sms / 2;
    if (pairs < 1) return cudaErrorInvalidConfiguration;
    e = dec::launch_dependent(dec::mla_tc_kernel, 2 * pairs, T::kThreads, T::kSmem, s, tmaps[3], tmaps[2], k);
    if (e != cudaSuccess) return e;
    return dec::launch_merge<__nv_bfloat16, true>(k, s);
  }
  using C = dec::MlaCfg;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(dec::mla_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  e = dec::launch_dependent(dec::mla_bf16_kernel, a.num_sms, C::kThreads, C::kSmem, s, tmaps[0], tmaps[1], k);
  if (e != cudaSuccess) return e;
  return dec::launch_merge<__nv_bfloat16, true>(k, s);
}

int mla_dims_supported_bf16(int d_qk, int d_v) { return d_qk == dec::kMlaDqk && d_v == dec::kMlaDv; }

int mla_uses_tc(int h_q, gqa_dtype dtype) { return dtype == GQA_BF16 && h_q % dec::kMlaTcHeads == 0; }

}  // namespace gqa
