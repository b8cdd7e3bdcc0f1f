/*
 * gqa.h - C ABI of the B200 (sm_100a) causal grouped-query attention library.
 *
 * The operation (all citations name the source page by title and section):
 *
 *   h_q query heads share h_kv K/V heads, h_q divisible by h_kv, r = h_q / h_kv. Query head a
 *   reads K/V head g(a) = floor(a / r); the r heads of one group are adjacent
 *   [序列计算与存储, section 分组查询注意力; 第 09 章 GQA、MLA 与跨层 KV 共享, section 09.2].
 *   h_kv = h_q is MHA, h_kv = 1 is MQA [序列计算与存储, the head-sharing table].
 *
 *   O_a = softmax(Q_a K_{g(a)}^T * scale + M) V_{g(a)}
 *   [序列计算与存储, display equation of section 分组查询注意力; section 分块注意力],
 *   evaluated block by block with an online softmax (running max m, running sum l, rescaled
 *   output u) so the score matrix never reaches memory [序列计算与存储, section 在线 softmax;
 *   第三章：MHA 的局限与 MQA、GQA、Flash Attention, section 3.5].
 *
 *   M masks by absolute position and by length: query row i of sequence b sits at position
 *   q_start[b] + i and sees key j iff j <= q_start[b] + i (causal) and j < kv_len[b]
 *   [第 09 章, section 09.2 on ptr_current_pos; 第三章, section 3.3 on is_causal].
 *
 *   The K/V cache is kept unexpanded as (B, h_kv, T_max, d_h) [序列计算与存储, section 缓存字节].
 *
 * Conventions shared by every entry point:
 *   - All tensors are dense, row-major (C order), with the shapes given per call. Element type is
 *     bf16 (GQA_BF16) or fp32 (GQA_FP32, the check mode: scalar FFMA, no tensor cores).
 *   - Tensor pointers are DEVICE pointers on the current CUDA device. Small integer arrays
 *     (q_start, kv_len, q_pos, pos) are device int32 arrays of length B, or NULL for the default.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Every call is
 *     asynchronous on that stream; the library keeps no per-request state and allocates nothing
 *     per call (tensor-map descriptors are encoded on the host and passed by value).
 *   - Buffers are owned by the caller. The library never frees or retains them after the call.
 *   - The library caches a little per-device state on first use (the device address of its error
 *     word, kernel attributes). A device reset (cudaDeviceReset) invalidates it: after resetting a
 *     device, do not call the library on that device again in the same process.
 *   - Host-detectable argument errors return a status without launching anything. Errors that only
 *     the device can see (a length or position out of range, a query with no visible key) never
 *     trap: the kernel writes zeros for the affected output rows, records the first such error in
 *     a sticky device word, and returns; read it with gqa_get_device_error().
 */
#ifndef GQA_B200_H
#define GQA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GQA_OK = 0,
  GQA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, h_q % h_kv != 0, a scale that is
                              negative, NaN or infinite ...                                        */
  GQA_ERR_UNSUPPORTED = 2, /* a valid request this build does not implement (e.g. bf16 d_h 96)  */
  GQA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (launch, symbol, tensor map)      */
  GQA_ERR_DEVICE = 4,      /* returned by gqa_get_device_error when the device word was set       */
  GQA_ERR_WORKSPACE = 5    /* workspace pointer missing, too small or not 256-byte aligned        */
} gqa_status;

typedef enum {
  GQA_BF16 = 0, /* bf16 in, fp32 accumulate (tcgen05 / mma), bf16 out                        */
  GQA_FP32 = 1  /* check mode: fp32 in, fp32 scalar FFMA arithmetic, fp32 out                 */
} gqa_dtype;

/* Device error codes (the value of the sticky word read by gqa_get_device_error). */
enum {
  GQA_DEVERR_NONE = 0,
  GQA_DEVERR_KV_LEN = 1,      /* kv_len[b] < 1 or kv_len[b] > T_max                               */
  GQA_DEVERR_POSITION = 2,    /* q_start/q_pos < 0, or an append that does not fit in T_max       */
  GQA_DEVERR_NO_VISIBLE = 3,  /* a query row that sees no key (e.g. q_start + i < 0 is impossible,
                                 but kv_len = 0 with a valid position is)                          */
  GQA_DEVERR_TIMEOUT = 4,     /* a bounded pipeline wait ran out (the kernel returned early)      */
  GQA_DEVERR_PAGE = 5         /* a block-table entry outside [0, num_pages) (paged cache)          */
};

/*
 * gqa_prefill - causal (or full) grouped-query attention of S_q new queries over a cache.
 *
 *   q        (B, h_q, S_q, d_h)    queries, already position-encoded.
 *   k_cache  (B, h_kv, T_max, d_h) keys;   only rows j < kv_len[b] are read.
 *   v_cache  (B, h_kv, T_max, d_h) values; only rows j < kv_len[b] are read.
 *   o        (B, h_q, S_q, d_h)    output (written).
 *   lse      (B, h_q, S_q) fp32 or NULL: natural-log sum over visible keys of exp(score * scale)
 *            (the softmax normaliser; written when non-NULL).
 *   q_start  device int32[B] or NULL (= all 0): absolute position of query row 0.
 *   kv_len   device int32[B] or NULL (= all T_max): keys present, 1 <= kv_len[b] <= T_max.
 *   scale    finite and > 0, or 0 for the standard 1/sqrt(d_h) (computed in double precision and
 *            rounded once to fp32). The same rule holds for every call that takes a scale.
 *   causal   1: key j visible to row i iff j <= q_start[b] + i and j < kv_len[b];
 *            0: iff j < kv_len[b].
 *   window   0: no window. W > 0 (requires causal = 1): sliding-window attention, each row reads
 *            only its local window [第三章, section 3.7, the Sliding Window Attention row]: key j
 *            is visible to row i only if also j > q_start[b] + i - W (the W most recent
 *            positions, the row's own included). K/V blocks below a tile's window are not read.
 *            A row whose window holds no cached key is written as zeros, lse = -inf, and sets
 *            GQA_DEVERR_NO_VISIBLE.
 *   dtype    GQA_BF16: d_h in {64, 128}, tcgen05 tensor-core kernel (sm_100a);
 *            GQA_FP32: 1 <= d_h <= 256, scalar check-mode kernel.
 *
 * A chunked prefill over an existing cache is kv_append(...) of the chunk's K/V at position p,
 * then gqa_prefill with q_start[b] = p and kv_len[b] = p + S_q.
 * Errors: INVALID_ARG (nulls, sizes <= 0, h_q % h_kv, scale, an unknown dtype, window < 0 or a
 * window without the causal mask), UNSUPPORTED (bf16 d_h outside {64, 128}, fp32 d_h > 256, or in
 * bf16 B*h_kv*T_max or B*h_q*S_q at or above 2^31 rows), CUDA. Every status but CUDA is decided on
 * the host before any CUDA call.
 */
gqa_status gqa_prefill(const void* q, const void* k_cache, const void* v_cache, void* o,
                       float* lse, const int32_t* q_start, const int32_t* kv_len,
                       int B, int h_q, int h_kv, int S_q, int T_max, int d_h,
                       float scale, int causal, int window, gqa_dtype dtype, void* stream);

/*
 * gqa_mla_decode - multi-head latent attention decode over a latent cache (absorbed form).
 * MLA caches one low-dimensional latent per token, C = X W_D, and K = C W_UK, V = C W_UV; for one
 * head Q (C U_K)^T = (Q U_K^T) C^T and P (C U_V) = (P C) U_V exactly, so a decode step scores
 * the latent cache directly with the absorbed query and up-projects the latent output afterwards
 * [第 09 章, section 09.3]. The full MLA keeps a decoupled position key beside the latent
 * [第三章, section 3.4]; it is the tail of each cache row here. This call computes the attention
 * core: for every head h of sequence b and visible token j,
 *   s_hj = scale * q[b, h, :] . cache[b, j, :],   o[b, h, :] = sum_j softmax_j(s_hj) cache[b, j, :d_v]
 * The projections (q_nope U_K^T, o U_V) are ordinary matrix products left to the caller.
 *
 *   q      (B, h_q, d_qk): [absorbed latent query (d_v) | rotary query part], already rotated.
 *   cache  (B, T_max, d_qk): [latent (d_v) | rotary key part], shared by all heads.
 *   o      (B, h_q, d_v) written (latent output). lse: (B, h_q) fp32 or NULL (natural log).
 *   kv_len, q_pos: as gqa_decode. scale: the model's softmax scale (for absorbed MLA this is
 *          1/sqrt(d_nope + d_rope) of the original heads, not 1/sqrt(d_qk)); 0 selects
 *          1/sqrt(d_qk), which is rarely the right value for a real model.
 *   dtype  GQA_BF16: d_qk = 576 and d_v = 512 (the DeepSeek-V2/V3 latent and rotary widths);
 *          GQA_FP32: d_qk <= 768, d_v <= min(d_qk, 512) (check mode).
 *   workspace: >= gqa_mla_decode_workspace_size(B, h_q, T_max, d_v, dtype, num_splits) bytes,
 *          256-byte aligned, zero-filled before first use, as for gqa_decode (same reuse rules);
 *          the size depends on dtype and h_q because they select the kernel (below).
 *   num_splits: as gqa_decode.
 * Kernels: bf16 with h_q a multiple of 128 runs on the tensor cores (tcgen05): a unit is 128 heads
 * of one sequence, and each chunk of keys runs on two CTAs, one per half of the d_v value columns.
 * With automatic chunking and every sequence at the same visible length, each sequence is cut into
 * equal chunks that divide it (no chunk holds parts of two sequences). Otherwise a unit is 16 heads
 * (m16n8k16 tensor-core MMAs). The fp32 check mode uses 16-head units too.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
size_t gqa_mla_decode_workspace_size(int B, int h_q, int T_max, int d_v, gqa_dtype dtype,
                                     int num_splits);
gqa_status gqa_mla_decode(const void* q, const void* cache, void* o, float* lse,
                          const int32_t* kv_len, const int32_t* q_pos, int B, int h_q, int T_max,
                          int d_qk, int d_v, float scale, gqa_dtype dtype, void* workspace,
                          size_t workspace_bytes, int num_splits, void* stream);

/*
 * gqa_prefill_backward - gradients of gqa_prefill for an upstream gradient dO (training).
 * The pages describe the backward pass as recomputing the local scores from statistics saved in
 * the forward pass, so the probability matrix is never stored [序列计算与存储, the paragraph
 * after the 两块算例 listing; 第三章, section 3.5]. With P = exp(S - lse) recomputed per block:
 *   dV_g = sum over the heads a of group g of P_a^T dO_a,
 *   dS_a = P_a * (dO_a V_g^T - D_a),  D_a = rowsum(dO_a * O_a),
 *   dQ_a = scale * dS_a K_g,  dK_g = scale * sum_a dS_a^T Q_a.
 *
 *   q, o, d_o   (B, h_q, S_q, d_h): the forward's queries and output, and dL/dO.
 *   k_cache, v_cache (B, h_kv, T_max, d_h): the forward's keys and values.
 *   lse         (B, h_q, S_q) fp32: the natural-log lse gqa_prefill returned (required). A row
 *               with lse = -inf (no visible key) gets dQ = 0 and contributes nothing.
 *   dq          (B, h_q, S_q, d_h) written.
 *   dk, dv      (B, h_kv, T_max, d_h) written in full; rows j >= kv_len[b] are zero.
 *   q_start, kv_len, scale, causal, window: exactly as passed to gqa_prefill.
 *   dtype       GQA_BF16 (d_h 64 or 128; tcgen05 kernels, bf16 gradients) or GQA_FP32 (d_h <= 256;
 *               scalar check mode, fp32 gradients). All tensors share the dtype; lse is fp32.
 *   workspace   device memory of at least gqa_prefill_backward_workspace_size(B, h_q, S_q) bytes,
 *               256-byte aligned, no initial contents required (two fp32 values per query row and
 *               a work-item counter). Calls that share a workspace must not overlap on the GPU.
 * Two launches run in order on `stream`: the row term D (with the base-2 lse; it also resets the
 * counter), then one persistent grid whose CTAs take the key-stationary dK/dV tiles (the heads of
 * a group add up in one CTA, no atomics) and then the query-stationary dQ tiles, heaviest first,
 * from the counter.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
size_t gqa_prefill_backward_workspace_size(int B, int h_q, int S_q);
gqa_status gqa_prefill_backward(const void* q, const void* k_cache, const void* v_cache,
                                const void* o, const void* d_o, const float* lse, void* dq,
                                void* dk, void* dv, const int32_t* q_start, const int32_t* kv_len,
                                int B, int h_q, int h_kv, int S_q, int T_max, int d_h, float scale,
                                int causal, int window, gqa_dtype dtype, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * gqa_decode_workspace_size - bytes of device workspace gqa_decode needs for this shape with
 * `num_splits` (0 = the automatic choice gqa_decode makes on the current device).
 * The workspace holds a small header (a work ticket), the per-sequence visible lengths and their
 * prefix sums, and per-piece partial results. It must be zero-filled before its first use; every
 * gqa_decode call that completes leaves the ticket at zero again, so one workspace can be reused,
 * for any shape it is large enough for, without clearing. Returns 0 on invalid arguments.
 */
size_t gqa_decode_workspace_size(int B, int h_q, int h_kv, int T_max, int d_h, gqa_dtype dtype,
                                 int num_splits);

/*
 * gqa_decode - one new query per sequence attending over its cached keys (split-KV decode).
 *
 *   q        (B, h_q, d_h)          the new token's queries.
 *   k_cache, v_cache (B, h_kv, T_max, d_h); rows j < min(kv_len[b], q_pos[b] + 1) are read,
 *            each exactly once from HBM per call.
 *   o        (B, h_q, d_h)          output.  lse: (B, h_q) fp32 or NULL, as in gqa_prefill.
 *   kv_len   device int32[B] or NULL (= all T_max).
 *   q_pos    device int32[B] or NULL (= kv_len[b] - 1: the token's own K/V was appended first,
 *            so it sees every cached key [MHA/MQA/GQA walkthrough, section 4]).
 *   window   0: none; W > 0: sliding window as in gqa_prefill, only keys q_pos[b] - W < j are
 *            visible, and only those are read (the visible keys of a unit start at the window).
 *   workspace, workspace_bytes: caller-owned device memory, >= gqa_decode_workspace_size(...),
 *            256-byte aligned, zero-filled before first use (see above). Calls that share one
 *            workspace must not overlap in time (use one stream, or one workspace per stream).
 *   num_splits: the visible keys of all (sequence, KV head) units, laid end to end, are cut into
 *            at most this many contiguous chunks of equal size; 0 = automatic (one chunk per SM,
 *            at least 128 keys and at least 16 keys per query head in a chunk). Results do not depend on it beyond floating-point
 *            rounding. The call launches two kernels: the split-KV pass over the chunks and a merge
 *            of the rows whose keys fell into more than one chunk.
 *   dtype    GQA_BF16: d_h in {64, 128}; GQA_FP32: 1 <= d_h <= 256 (check mode).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
gqa_status gqa_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                      const int32_t* kv_len, const int32_t* q_pos,
                      int B, int h_q, int h_kv, int T_max, int d_h, float scale, int window,
                      gqa_dtype dtype, void* workspace, size_t workspace_bytes, int num_splits,
                      void* stream);

/*
 * gqa_decode_noalloc - gqa_decode for callers that cannot allocate device memory. (The source
 * pages have no counterpart; this is a library convenience.) Some callers run where cudaMalloc is
 * unavailable or forbidden: a plugin inside a host framework that owns all device memory and hands
 * over only inputs and outputs, or a latency-critical loop that must not risk the synchronisation
 * an allocation can bring. This entry point takes the same arguments as gqa_decode minus the
 * workspace, and uses a fixed 16 MiB scratch array that the library itself holds in device memory
 * (every GPU that loads the library keeps it until the process exits). It allocates nothing.
 *   - Shapes whose workspace (gqa_decode_workspace_size) exceeds 16 MiB are rejected with
 *     GQA_ERR_WORKSPACE; use gqa_decode with your own workspace for those.
 *   - The first call on a device looks up the scratch array's device address and caches it; make
 *     that first call before any stream capture. A device reset (cudaDeviceReset) frees the array
 *     and leaves that address stale: do not call the library on a device after resetting it.
 *   - All calls share the one array, which keeps the previous call's contents; the part that must
 *     start at zero is cleared on `stream` before each launch. Calls that overlap on the GPU (on
 *     different streams or from different host threads) race on the array: serialise them.
 * Errors: as gqa_decode, checked in the same order (so an unsupported shape is UNSUPPORTED even
 * when its workspace would also exceed the scratch array), then WORKSPACE for the size limit.
 */
gqa_status gqa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, void* o,
                              float* lse, const int32_t* kv_len, const int32_t* q_pos,
                              int B, int h_q, int h_kv, int T_max, int d_h, float scale,
                              int window, gqa_dtype dtype, int num_splits, void* stream);

/*
 * kv_append - copy new K/V rows into the cache: cache[b, g, pos[b] + t, :] = new[b, g, t, :]
 * for t < S_new. Bit-exact; no other byte of the cache is written.
 * [第三章, section 3.1: the new token's K/V join the cache; MHA/MQA/GQA walkthrough, section 4].
 *
 *   k_cache, v_cache (B, h_kv, T_max, d_h), written in place.
 *   k_new, v_new     (B, h_kv, S_new, d_h), read.
 *   pos      device int32[B] (required when S_new > 0): first cache row written for sequence b.
 *            S_new = 0 is a no-op; k_new, v_new and pos may then be NULL.
 *            Rows that would fall outside [0, T_max) are not written; the device error word is
 *            set to GQA_DEVERR_POSITION.
 *   dtype    element type of all four tensors (bf16: 2 bytes, fp32: 4 bytes); any d_h >= 1.
 * Errors: INVALID_ARG, CUDA.
 */
gqa_status kv_append(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                     const int32_t* pos, int B, int h_kv, int S_new, int T_max, int d_h,
                     gqa_dtype dtype, void* stream);

/*
 * Paged KV cache. The pages name page metadata and fragmentation as the deployment cost of a
 * cache that grows token by token [第三章, section 3.6; MHA/MQA/GQA walkthrough, section 8, the
 * ledger's note on page metadata]. A paged cache keeps K and V in pools of fixed-size pages
 *   k_pages, v_pages (num_pages, h_kv, page_size, d_h)
 * and a block table (B, max_pages) of int32 page indices: logical position t of sequence b is row
 * t % page_size of page block_table[b * max_pages + t / page_size]. Pages may be shared or in any
 * order; entries for positions a call does not touch are never read. Attention over a paged
 * cache is, by definition, attention over the contiguous cache the pages spell out, so the
 * results equal gqa_decode's on that cache (to floating-point rounding; chunk boundaries fall on
 * multiples of 16 keys here, of 64 when page_size is a multiple of 64).
 *
 * gqa_decode_paged - gqa_decode over a paged cache. T_max is max_pages * page_size.
 *   page_size  a multiple of 16 (every 16-key sub-tile the kernel loads lies inside one page);
 *            a multiple of 64 lets every 64-key tile load as one block (fewer, larger copies).
 *   num_pages * h_kv * page_size must stay below 2^31 (pool rows are addressed with 32 bits).
 *   block_table device int32 (B, max_pages), row-major. An entry outside [0, num_pages) that a
 *            call needs is replaced by page 0 and sets GQA_DEVERR_PAGE (the output is then wrong).
 *   workspace  as gqa_decode, sized by gqa_decode_workspace_size(B, h_q, h_kv,
 *            max_pages * page_size, d_h, dtype, num_splits).
 * Other arguments and errors as gqa_decode.
 */
gqa_status gqa_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* o,
                            float* lse, const int32_t* kv_len, const int32_t* q_pos,
                            const int32_t* block_table, int B, int h_q, int h_kv, int num_pages,
                            int page_size, int max_pages, int d_h, float scale, int window,
                            gqa_dtype dtype, void* workspace, size_t workspace_bytes,
                            int num_splits, void* stream);

/*
 * kv_append_paged - kv_append into a paged cache: new[b, g, t, :] goes to logical position
 * pos[b] + t, i.e. row (pos[b] + t) % page_size of page block_table[b, (pos[b] + t) / page_size].
 * Bit-exact; no other byte of the pools is written.
 *   k_pages, v_pages (num_pages, h_kv, page_size, d_h), written in place; page_size >= 1.
 *   k_new, v_new     (B, h_kv, S_new, d_h).
 *   pos      device int32[B] (with k_new, v_new and block_table, required when S_new > 0; S_new = 0
 *            is a no-op). Sequences whose rows would leave [0, max_pages * page_size) are not
 *            written (GQA_DEVERR_POSITION); rows whose page entry is outside [0, num_pages) are
 *            not written (GQA_DEVERR_PAGE).
 * Errors: INVALID_ARG, CUDA.
 */
gqa_status kv_append_paged(void* k_pages, void* v_pages, const void* k_new, const void* v_new,
                           const int32_t* pos, const int32_t* block_table, int B, int h_kv,
                           int S_new, int num_pages, int page_size, int max_pages, int d_h,
                           gqa_dtype dtype, void* stream);

/*
 * gqa_get_device_error - synchronise `stream`, then read and clear the sticky device error word
 * of the current device. *code receives a GQA_DEVERR_* value. Returns GQA_ERR_DEVICE when the word
 * was non-zero, GQA_OK when it was zero, GQA_ERR_CUDA if the read failed.
 */
gqa_status gqa_get_device_error(int* code, void* stream);

/* Human-readable name of a status. Never NULL. */
const char* gqa_status_string(gqa_status s);

/* Library version string, e.g. "gqa-b200 0.2.0 (sm_100a)". */
const char* gqa_version(void);

/*
 * gqa_debug_expire_waits - failure-detection test hook; never needed in normal use.
 * Every pipeline wait of the kernels is bounded (about 2 s of %globaltimer); when one runs out the
 * kernel records GQA_DEVERR_TIMEOUT and returns instead of spinning, so the context stays usable.
 * With enable = 1, every later bf16 gqa_prefill, contiguous bf16 gqa_decode and tensor-core
 * gqa_mla_decode (bf16, a multiple of 128 heads) on any device makes CTA 0 wait on a barrier that
 * nothing signals, so that bound is reached on purpose: the call takes about 2 s longer, the error
 * word reads GQA_DEVERR_TIMEOUT, prefill writes the rows of the tile that gave up as zeros
 * (lse = -inf), and decode and MLA decode leave the rows of CTA 0's first chunk unspecified. A following call with the hook off is unaffected (a decode workspace stays
 * reusable). enable = 0 (the default) turns it off. Other calls ignore it. Not thread-safe with
 * respect to concurrent launches: set it only while no other thread calls the library.
 * Errors: INVALID_ARG (enable not 0 or 1).
 */
gqa_status gqa_debug_expire_waits(int enable);

#ifdef __cplusplus
}
#endif

#endif /* GQA_B200_H */
