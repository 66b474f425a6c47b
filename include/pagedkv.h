/*
 * pagedkv.h -- C ABI of libpagedkv.so: attention over a block-paged KV cache
 * on NVIDIA B200 (sm_100a).
 *
 * The method (from the pages this library follows):
 *   - "从零构建CUDA推理引擎：Tiny-Infer项目的技术深度解析", section
 *     "分页KV缓存：借鉴操作系统的内存管理": the KV cache is divided into
 *     fixed-size blocks ("pages") and a mapping table turns each logical
 *     position into a physical block, so sequences can share memory and grow.
 *   - same page, section "Flash Attention：内存与计算的重平衡", and
 *     "5 Fun Projects for LLM Inference Engineering", section 2: attention is
 *     computed tile by tile with a running max and running sum (online softmax),
 *     never materialising the full score matrix; the result is exact attention.
 *
 * Layouts (all row-major, bf16 = IEEE bfloat16):
 *   k_cache, v_cache : [NB][Hkv][bs][D]   one (block, kv head) page is contiguous
 *   block_tables     : [B][MB] int32      physical block of logical page p of
 *                                          sequence b; entries past the last
 *                                          used page are never read
 *   context_lens     : [B] int32          number of valid keys of sequence b,
 *                                          including rows just written
 *   slot_mapping     : [T] int64          slot = block * bs + offset; < 0 = skip
 *   Grouped-query heads: query head h reads kv head h / (Hq / Hkv).
 *
 * Conventions:
 *   - Ownership: the caller owns every buffer (device memory unless stated).
 *     The library allocates no device memory; it keeps one static device error
 *     word per device, and the static scratch array of
 *     pkv_paged_attention_split_noalloc.  Workspace for the split-KV path is
 *     otherwise passed in.
 *   - Asynchrony: every call only enqueues kernels on `stream` and returns;
 *     nothing synchronises except pkv_get_device_error.
 *   - Errors: argument checks happen on the host before any launch and return
 *     a status without launching.  A failed launch returns PKV_ERR_CUDA.
 *     Problems only the device can see (a slot or block id outside the pool, a
 *     context length larger than the block table, a wait that ran out) set
 *     the device error word, read with pkv_get_device_error.
 *   - Supported now: dtype PKV_BF16; decode and prefill need bs = 16 and
 *     D in {64, 128}; the cache write takes any
 *     bs and any D that is a multiple of 8.  All pointers 16-byte aligned.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pkv_status {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer      */
  PKV_ERR_UNSUPPORTED = 2,  /* valid but not built: dtype, D, bs, group size   */
  PKV_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed            */
  PKV_ERR_TIMEOUT = 4,      /* device: a bounded wait gave up                  */
  PKV_ERR_BOUNDS = 5,       /* device: slot / block id / length out of range   */
  PKV_ERR_WORKSPACE = 6,    /* workspace missing or smaller than required      */
  PKV_ERR_NO_BLOCKS = 7     /* block allocator: not enough free blocks         */
} pkv_status;

typedef enum pkv_dtype { PKV_BF16 = 0 } pkv_dtype;

/* A cudaStream_t (NULL = the legacy default stream). */
typedef void* pkv_stream_t;

/*
 * kv_cache_write -- scatter new K/V rows into their physical slots.
 * For every token t with s = slot_mapping[t] >= 0 and every kv head h:
 *   k_cache[s / bs][h][s % bs][:] = key[t][h][:]   (and the same for V).
 * A bit copy: the result is exact.  Tiny-Infer page, section
 * "分页KV缓存：借鉴操作系统的内存管理" (logical position -> physical block).
 *   key, value       : device, [T][Hkv][D] bf16; token stride in ELEMENTS
 *                      (>= Hkv*D, a multiple of 8), head stride D
 *   k_cache, v_cache : device, [NB][Hkv][bs][D] bf16, written in place
 *   slot_mapping     : device, [T] int64; < 0 skips the token; >= NB*bs sets
 *                      PKV_ERR_BOUNDS on the device and skips the token
 * T = 0 launches nothing.  Returns PKV_ERR_INVALID_ARG for null pointers,
 * negative sizes or misalignment, PKV_ERR_UNSUPPORTED for D % 8 != 0.
 */
pkv_status pkv_kv_cache_write(const void* key, const void* value,
                              int64_t key_stride_tok, int64_t value_stride_tok,
                              void* k_cache, void* v_cache,
                              const int64_t* slot_mapping, int32_t T,
                              int32_t Hkv, int32_t D, int32_t NB, int32_t bs,
                              pkv_dtype dtype, pkv_stream_t stream);

/*
 * paged_attention -- decode: one query token per sequence against its paged
 * K/V, grouped-query heads, online softmax in one pass over the pages.
 *   out[b][h][:] = sum_j softmax_j(scale * q[b][h] . k_j) v_j over the
 *   context_lens[b] keys of sequence b (0 keys -> a zero row).
 *   out          : device, [B][Hq][D] bf16
 *   q            : device, [B][Hq][D] bf16
 *   block_tables : device, [B][MB] int32; context_lens: device, [B] int32
 *   max_context_len_hint : host upper bound on context_lens (<= 0: MB*bs);
 *                  used only to size the launch, never checked against the
 *                  device values, which are never read on the host
 *   workspace    : device scratch for split-KV partials, or NULL.  With at
 *                  least pkv_paged_attention_workspace_size(...) bytes the
 *                  call may split long contexts across CTAs and merge the
 *                  parts by log-sum-exp; with less it runs one CTA per
 *                  (sequence, head group) and needs none.
 * Same shape limits as the file header; Hq % Hkv == 0.
 */
pkv_status pkv_paged_attention(void* out, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* block_tables,
                               int32_t MB, const int32_t* context_lens,
                               int32_t B, int32_t Hq, int32_t Hkv, int32_t D,
                               int32_t NB, int32_t bs, float scale,
                               int32_t max_context_len_hint, void* workspace,
                               size_t workspace_bytes, pkv_dtype dtype,
                               pkv_stream_t stream);

/* Workspace bytes pkv_paged_attention (or pkv_paged_attention_int8) may use
 * for these sizes on the current device (0 if it would never split). */
size_t pkv_paged_attention_workspace_size(int32_t B, int32_t Hq, int32_t Hkv,
                                          int32_t D, int32_t MB, int32_t bs,
                                          int32_t max_context_len_hint);

/*
 * kv_cache_write_rope -- pkv_kv_cache_write with rotary position embedding
 * applied to K on the way in, so the rotated rows make one trip through
 * memory (the fused-ops page fuses RoPE into the step before it:
 * "Triton融合算子优化：LLM推理性能提升3倍的工程实践", section 3.1).  The pages
 * print no formula; Llama's form (as in the HuggingFace implementation the
 * Tiny-Infer page checks against) is used: element i < D/2 pairs with
 * i + D/2 and turns by pos * rope_base^(-2i/D),
 *   k'[i] = k[i] cos - k[i+D/2] sin,  k'[i+D/2] = k[i+D/2] cos + k[i] sin.
 * The angle is formed and reduced in fp64, sine/cosine and the rotation in
 * fp32, one bf16 rounding at the end.  V rows are copied bit for bit.
 *   positions : device, [T] int64, the absolute position of each token
 *   rope_base : > 1 (10000 for Llama 2, 500000 for Llama 3)
 * Other arguments and errors as pkv_kv_cache_write (D even, 2-byte aligned).
 */
pkv_status pkv_kv_cache_write_rope(const void* key, const void* value,
                                   int64_t key_stride_tok,
                                   int64_t value_stride_tok, void* k_cache,
                                   void* v_cache, const int64_t* slot_mapping,
                                   const int64_t* positions, int32_t T, int32_t Hkv,
                                   int32_t D, int32_t NB, int32_t bs, double rope_base,
                                   pkv_dtype dtype, pkv_stream_t stream);

/*
 * INT8 KV cache.  The Tiny-Infer page (section "推测性解码与INT8量化") names
 * an INT8 KV cache as the way to halve its memory; it fixes neither the scale
 * granularity nor the rounding.  This library's reading: symmetric codes with
 * one fp32 scale per written row (one token's D values of one kv head), the
 * granularity an incremental cache write can fix when the row is written:
 *   amax = max |x|;  inv = 127 / amax;  code = clamp(rint(x * inv), -127, 127);
 *   scale = amax / 127   (fp32, round half to even; amax = 0: codes 0, scale 0)
 * and the row's value is code * scale.  Non-finite inputs give unspecified codes.
 *   k_cache, v_cache : device, [NB][Hkv][bs][D] int8, 16-byte aligned
 *   k_scale, v_scale : device, [NB][Hkv][bs] fp32, 16-byte aligned
 * kv_cache_write_int8: key/value as for pkv_kv_cache_write (bf16, token
 * strides in elements, 2-byte aligned); D in {64, 128, 256}; any bs.  Slots
 * < 0 are skipped; a slot outside the pool sets PKV_ERR_BOUNDS on the device.
 */
pkv_status pkv_kv_cache_write_int8(const void* key, const void* value,
                                   int64_t key_stride_tok,
                                   int64_t value_stride_tok, void* k_cache,
                                   void* v_cache, float* k_scale, float* v_scale,
                                   const int64_t* slot_mapping, int32_t T,
                                   int32_t Hkv, int32_t D, int32_t NB, int32_t bs,
                                   pkv_stream_t stream);

/*
 * paged_attention_int8 -- pkv_paged_attention over the int8 cache: the same
 * workspace (pkv_paged_attention_workspace_size bytes serve either cache) and
 * errors, with split sizes chosen for this kernel; K and
 * V are read as codes and scaled by their row's scale inside the kernel (half
 * the bytes of the bf16 cache, plus 4 bytes per row).  q and out are bf16 as
 * for pkv_paged_attention; D in {64, 128}, bs = 16.  The scores q.k are
 * taken on the tensor cores from the codes directly, with q held per head as
 * a 15-bit fixed-point pair of signed bytes (exact for every element within
 * 2^7 of the head's largest magnitude; smaller ones to 2^-14 of it), so the
 * result differs from attention over code * scale by that rounding of q.
 */
pkv_status pkv_paged_attention_int8(void* out, const void* q, const void* k_cache,
                                    const void* v_cache, const float* k_scale,
                                    const float* v_scale,
                                    const int32_t* block_tables, int32_t MB,
                                    const int32_t* context_lens, int32_t B,
                                    int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                                    int32_t bs, float scale,
                                    int32_t max_context_len_hint, void* workspace,
                                    size_t workspace_bytes, pkv_stream_t stream);

/*
 * paged_attention_window -- pkv_paged_attention under a sliding window: the
 * query (position L_b - 1) attends only to its last `window` keys,
 * max(0, L_b - window) .. L_b - 1.  The inference-lab page lists a
 * sliding-window KV cache among its cache variants ("从零开始的LLM推理优化实
 * 验室：从PyTorch基线到Triton内核的完整实践", section "KV缓存实验与长上下文
 * 优化") without semantics; this is the reading taken.  Pages wholly before the
 * window are never read; the first window page is masked row by row.
 * window >= 1 (else PKV_ERR_INVALID_ARG); any context the block table holds.
 *   workspace: >= pkv_paged_attention_window_workspace_size(...) bytes to let
 *   the call split each window across CTAs, else one CTA per head group.
 */
pkv_status pkv_paged_attention_window(void* out, const void* q, const void* k_cache,
                                      const void* v_cache,
                                      const int32_t* block_tables, int32_t MB,
                                      const int32_t* context_lens, int32_t B,
                                      int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                                      int32_t bs, float scale, int32_t window,
                                      void* workspace, size_t workspace_bytes,
                                      pkv_dtype dtype, pkv_stream_t stream);

size_t pkv_paged_attention_window_workspace_size(int32_t B, int32_t Hq, int32_t Hkv,
                                                 int32_t D, int32_t MB, int32_t bs,
                                                 int32_t window);

/*
 * paged_attention_split -- the split-KV ("flash-decoding") path with an
 * explicit split size.  Split c of sequence b covers logical pages
 * [c*pages_per_split, (c+1)*pages_per_split); each CTA writes its normalised
 * partial o_c and its log-sum-exp, and a second kernel merges
 *   out = sum_c e^{lse_c - M} o_c / sum_c e^{lse_c - M},  M = max_c lse_c.
 * Same result as pkv_paged_attention up to rounding.  The split-KV form is
 * not on the pages; it answers their remark that variable-length batches need
 * padding or bucketing ("Triton融合算子优化：LLM推理性能提升3倍的工程实践",
 * section 六).  pages_per_split >= 1; num_splits = ceil(ceil(max_ctx/bs) /
 * pages_per_split) where max_ctx = max_context_len_hint (<= 0: MB*bs); the
 * device sets PKV_ERR_BOUNDS if a context is longer than that.
 *   workspace: device, >= pkv_split_workspace_size(B, Hq, D, num_splits) bytes.
 */
pkv_status pkv_paged_attention_split(void* out, const void* q,
                                     const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, int32_t MB,
                                     const int32_t* context_lens, int32_t B,
                                     int32_t Hq, int32_t Hkv, int32_t D,
                                     int32_t NB, int32_t bs, float scale,
                                     int32_t max_context_len_hint,
                                     int32_t pages_per_split, void* workspace,
                                     size_t workspace_bytes, pkv_dtype dtype,
                                     pkv_stream_t stream);

/* Workspace bytes of the split path: fp32 partials [B][Hq][C][D] plus fp32
 * log-sum-exp [B][Hq][C], each 256-byte aligned. */
size_t pkv_split_workspace_size(int32_t B, int32_t Hq, int32_t D,
                                int32_t num_splits);

/*
 * paged_attention_split_noalloc -- pkv_paged_attention_split for callers that
 * cannot allocate device memory: an engine plugin whose enqueue hook must not
 * allocate, a serving loop that cannot take the device-wide synchronisation a
 * cudaMalloc may cause, or a process whose device memory is already reserved
 * in full by another allocator.  The pages have no counterpart of this call;
 * it exists for those callers only.
 *   Same arguments and result as pkv_paged_attention_split without the
 *   workspace: the split partials go to one static device array of
 *   PKV_NOALLOC_SCRATCH_BYTES that the library holds on every GPU that loads
 *   it, until the process exits.  The caller still owns out and every input.
 *   - A request whose partials need more than PKV_NOALLOC_SCRATCH_BYTES
 *     (pkv_split_workspace_size(B, Hq, D, num_splits)) returns
 *     PKV_ERR_WORKSPACE and launches nothing.
 *   - The array comes into being when the library's device code is loaded
 *     on a GPU.  With lazy module loading (the CUDA default) that happens at
 *     the library's first call on that device, and it costs an allocation and
 *     a synchronisation there: make any other library call, or one warm-up
 *     call of this one, first, and the hot path never pays it.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and keeps it for the life of the process; make
 *     that first call before any stream capture.  Calls after a device reset
 *     (cudaDeviceReset, or a reset of the primary context) are unsupported:
 *     the kept address no longer names the array.
 *   - Nothing is allocated or freed by this call, by the library or through
 *     any library routine.
 *   - Every call shares the one array and leaves its partials in it; every
 *     partial the merge reads is written first by the same call, so nothing
 *     needs clearing.  Calls that overlap on the GPU (other streams, other
 *     host threads) race on the array: serialise them.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (8u << 20) /* 8 MiB per GPU */

pkv_status pkv_paged_attention_split_noalloc(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int32_t MB, const int32_t* context_lens,
    int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t NB, int32_t bs,
    float scale, int32_t max_context_len_hint, int32_t pages_per_split,
    pkv_dtype dtype, pkv_stream_t stream);

/*
 * paged_attention_prefill -- causal chunked prefill over the paged cache.
 * Sequence b has a chunk of Q_b = query_start_loc[b+1] - query_start_loc[b]
 * new queries, which are the LAST Q_b of its context_lens[b] positions; their
 * K/V must already be in the cache (written by pkv_kv_cache_write).  Query i
 * sits at position L_b - Q_b + i and attends to keys 0 .. L_b - Q_b + i.
 * Runs on the tcgen05 tensor cores with TMEM accumulators: S = Q K^T and
 * O += P V are bf16 MMAs with fp32 accumulation, P rounded to bf16.
 * Tiny-Infer page, sections "Flash Attention：内存与计算的重平衡" and
 * "分页KV缓存：借鉴操作系统的内存管理".
 *   out             : device, [sumQ][Hq][D] bf16
 *   q               : device, [sumQ][Hq][D] bf16
 *   query_start_loc : device, [B+1] int32, query_start_loc[0] = 0
 *   max_q_len       : host upper bound on Q_b (sizes the launch)
 * Needs D in {64, 128}, bs = 16, Hq / Hkv <= 128 (else
 * PKV_ERR_UNSUPPORTED); scale may have either sign but must be finite (else
 * PKV_ERR_INVALID_ARG).
 */
pkv_status pkv_paged_attention_prefill(
    void* out, const void* q, const int32_t* query_start_loc,
    const void* k_cache, const void* v_cache, const int32_t* block_tables,
    int32_t MB, const int32_t* context_lens, int32_t B, int32_t sumQ,
    int32_t max_q_len, int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
    int32_t bs, float scale, pkv_dtype dtype, pkv_stream_t stream);

/*
 * paged_attention_prefill_window -- pkv_paged_attention_prefill under a
 * sliding window: query i of sequence b (position p = L_b - Q_b + i) sees
 * keys max(0, p - window + 1) .. p (the reading of the inference-lab page's
 * sliding-window cache, as for pkv_paged_attention_window).  Key tiles below
 * every row's window are skipped; edge tiles are masked per row.  window >= 1.
 */
pkv_status pkv_paged_attention_prefill_window(
    void* out, const void* q, const int32_t* query_start_loc,
    const void* k_cache, const void* v_cache, const int32_t* block_tables,
    int32_t MB, const int32_t* context_lens, int32_t B, int32_t sumQ,
    int32_t max_q_len, int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
    int32_t bs, float scale, int32_t window, pkv_dtype dtype, pkv_stream_t stream);

/*
 * paged_attention_int8_window -- pkv_paged_attention_int8 under a sliding
 * window of `window` keys (>= 1): the query at position L-1 sees keys
 * L-window .. L-1, as pkv_paged_attention_window does over the bf16 cache
 * (the inference-lab page's sliding-window cache, section "KV缓存实验与长上下文
 * 优化", over the Tiny-Infer page's INT8 cache, section "推测性解码与INT8量化").
 * Same workspace as pkv_paged_attention_window
 * (pkv_paged_attention_window_workspace_size bytes serve either cache); errors as
 * pkv_paged_attention_int8.  Pages wholly before the window are never read.
 */
pkv_status pkv_paged_attention_int8_window(void* out, const void* q, const void* k_cache,
                                           const void* v_cache, const float* k_scale,
                                           const float* v_scale,
                                           const int32_t* block_tables, int32_t MB,
                                           const int32_t* context_lens, int32_t B,
                                           int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                                           int32_t bs, float scale, int32_t window,
                                           void* workspace, size_t workspace_bytes,
                                           pkv_stream_t stream);

/*
 * Shared blocks and copy-on-write.  Sequences that share a prefix (parallel
 * sampling from one prompt) can point their block tables at the same
 * physical blocks and copy a block only when one of them is about to write
 * into it -- the vLLM-style block copying the Tiny-Infer page plans for its
 * paged cache (section "分页KV缓存：借鉴操作系统的内存管理").
 *
 * pkv_block_allocator_*: host-only bookkeeping of which physical blocks are
 * in use and by how many holders (no device memory, no CUDA calls; one mutex
 * per allocator, so host threads may share one).  A fresh allocator hands out
 * the lowest ids first.  Every call is all-or-nothing: on an error nothing
 * changes.
 *   create(num_blocks, &a)          num_blocks >= 0; destroy(a) frees it.
 *   alloc(a, n, ids)                n fresh blocks, refcount 1, written to ids
 *                                   (host array of n); PKV_ERR_NO_BLOCKS if
 *                                   fewer than n are free.
 *   share(a, ids, n)                refcount + 1 for each (all must be live).
 *   release(a, ids, n)              refcount - 1 for each; blocks reaching 0
 *                                   are free again (ids may repeat).
 *   cow(a, id, &new_id, &copy)      before writing into block id: if it is
 *                                   shared, new_id is a fresh block for the
 *                                   writer, id loses one holder, copy = 1 and
 *                                   the caller must pkv_copy_blocks(id ->
 *                                   new_id) before writing; if private,
 *                                   new_id = id and copy = 0.
 *   num_free(a), refcount(a, id)    queries (refcount -1: id outside the pool).
 */
typedef struct pkv_block_allocator pkv_block_allocator;
pkv_status pkv_block_allocator_create(int32_t num_blocks, pkv_block_allocator** out);
void pkv_block_allocator_destroy(pkv_block_allocator* a);
pkv_status pkv_block_allocator_alloc(pkv_block_allocator* a, int32_t n, int32_t* ids);
pkv_status pkv_block_allocator_share(pkv_block_allocator* a, const int32_t* ids, int32_t n);
pkv_status pkv_block_allocator_release(pkv_block_allocator* a, const int32_t* ids, int32_t n);
pkv_status pkv_block_allocator_cow(pkv_block_allocator* a, int32_t id, int32_t* new_id,
                                   int32_t* must_copy);
int32_t pkv_block_allocator_num_free(pkv_block_allocator* a);
int32_t pkv_block_allocator_refcount(pkv_block_allocator* a, int32_t id);

/*
 * hbm_read_probe -- measurement utility, not part of the attention path:
 * reads `bytes` (a multiple of 16) of device memory at `buf` (16-byte
 * aligned) once, in chunks of chunk_bytes moved by bulk copies into shared
 * memory (as decode moves pages), 96 KB in flight per CTA, chunk c by CTA
 * c % nsink.  chunk_bytes divides 98304 and lies in [4096, 32768].  CTA i
 * writes to sink[i] (device, nsink words) the XOR of the first four 32-bit
 * words of each of its chunks.  Timed by the caller, it gives the read-only
 * bandwidth that HBM-bound decode is compared with, and how it depends on
 * the size of each copy.  One launch.
 */
pkv_status pkv_hbm_read_probe(const void* buf, size_t bytes, int32_t chunk_bytes, uint32_t* sink,
                              int32_t nsink, pkv_stream_t stream);

/*
 * copy_blocks -- for each (src, dst) pair in `pairs` (device, [n][2] int32)
 * copy block src to block dst, bit for bit, in both pools (k_cache and
 * v_cache; for the INT8 cache call once for the codes and once for the
 * scales).  block_bytes: bytes of one block of one pool (Hkv*bs*D*elem),
 * a multiple of 16; pools 16-byte aligned.  A dst must not also be a src in
 * the same call, nor appear twice (the pairs run concurrently).  A block id outside [0, NB) sets PKV_ERR_BOUNDS on the
 * device and that pair is skipped.  One launch (none if n = 0).
 */
pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, size_t block_bytes,
                           const int32_t* pairs, int32_t n, int32_t NB,
                           pkv_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word (0 = none, else a pkv_status value recorded by a kernel).
 */
pkv_status pkv_get_device_error(pkv_stream_t stream, int32_t* err_out);

/* Number of kernels the last successful call on this host thread launched. */
int32_t pkv_last_launch_count(void);

/* Static text for a status code. */
const char* pkv_status_string(pkv_status status);

/*
 * Self-test of the bounded waits: launches one CTA that waits on a barrier
 * nothing will complete, with a limit of timeout_us microseconds; the kernel
 * then records PKV_ERR_TIMEOUT in the device error word and returns, leaving
 * the context usable.  For tests of the failure path; hangs nothing.
 */
pkv_status pkv_selftest_wait_timeout(uint32_t timeout_us, pkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
