/*
 * pagedkv.h -- C ABI of libpagedkv: paged-KV-cache attention on B200 (sm_100a).
 *
 * Sources (four web pages on paged KV caches and FlashAttention, cited by title
 * and section):
 *   [KVFA]  "大模型推理优化：KV Cache与FlashAttention实战"
 *   [FAPKV] "Flash Attention与Paged KV Cache优化大模型计算效率"
 *   [KV3X]  "大模型推理优化实战：KV Cache + Flash Attention，让 Token 生成快 3 倍"
 *   [SYS]   "LLM推理系统优化：KV缓存管理与动态批处理技术"
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller (e.g. torch
 *   allocations).  The library allocates no device memory on any call path and
 *   keeps no pointer after a call returns.
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and returns an int status: PKV_OK (0) or a negative
 *   PKV_ERR_* code.  Host-side argument errors are reported before anything is
 *   launched.  No C++ exception crosses the ABI.
 * - Device-side checks (block-table entries, slots, context lengths against
 *   the sizes passed in) never fault: an offending access is skipped, its
 *   output is left unspecified, and a device status word records the first
 *   error; pkv_get_device_status() reads and clears it.
 * - Layouts (token-major pages; [FAPKV] §3.2 stores a page as
 *   (page_size, d_model)):
 *     k_pages, v_pages   [num_pages][page_size][num_kv_heads][head_dim]
 *                        (slot s = page * page_size + offset is row s of the
 *                        pool viewed as [num_pages*page_size][num_kv_heads*head_dim])
 *     k_scales, v_scales [num_pages][page_size][num_kv_heads] fp16 (INT8 pools)
 *     block_tables       int32 [num_seqs][max_pages_per_seq]; entry j of row b
 *                        is the physical page of logical page j of sequence b;
 *                        entries past ceil(context_len / page_size) are never read
 *     context_lens       int32 [num_seqs]
 *   All tensors are dense and row-major as shown.
 * - Grouped-query attention: query head h reads KV head h / (num_q_heads /
 *   num_kv_heads) (contiguous groups, the repeat_interleave of [SYS] §2.1).
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle type as cudaStream_t / CUstream, without the CUDA headers. */
typedef struct CUstream_st* pkv_stream_t;

typedef enum {
    PKV_F32 = 0,   /* float32 */
    PKV_BF16 = 1,  /* bfloat16 */
    PKV_F16 = 2,   /* IEEE float16 */
    PKV_I8 = 3     /* int8 codes with one fp16 scale per (token, KV head) */
} pkv_dtype;

enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = -1,   /* null pointer, non-positive size, mismatched shape */
    PKV_ERR_UNSUPPORTED = -2,   /* valid but not implemented (dtype combo, head_dim) */
    PKV_ERR_WORKSPACE = -3,     /* workspace missing or too small */
    PKV_ERR_CUDA = -4,          /* a CUDA runtime call failed (launch, device query) */
    PKV_ERR_DEVICE_RANGE = -5,  /* device saw an out-of-range page, slot or length */
    PKV_ERR_DEVICE_TIMEOUT = -6, /* a bounded device wait gave up (pipeline stalled) */
    PKV_ERR_OUT_OF_PAGES = -7    /* block manager: not enough free pages (nothing changed) */
};

/* Static description of a status code (thread-safe, never NULL). */
const char* pkv_error_string(int code);

/*
 * Cache append (slot-mapping scatter): the new K/V rows of `num_tokens` tokens
 * go into their pages.  Row t of k (and of v), num_kv_heads*head_dim elements,
 * is copied to slot slot_mapping[t] of k_pages (and v_pages).  This is the
 * paged form of appending the current token's key/value to the cache
 * ([KV3X] "KV Cache 的工作原理": the cache grows by the new k, v every step;
 * [FAPKV] §3.2: fixed-size pages found through a page table).
 *
 *   k, v           [num_tokens][num_kv_heads][head_dim] of `dtype`
 *   slot_mapping   int64 [num_tokens]; slot = page * page_size + offset;
 *                  a negative slot skips the row (padding).  Slots must be
 *                  distinct (duplicates: which row lands is unspecified).
 *   dtype          any pkv_dtype; the copy is bytewise (bit-exact).  For
 *                  PKV_I8 the per-row scales are copied too:
 *   k_scale, v_scale          fp16 [num_tokens][num_kv_heads] (PKV_I8 only)
 *   k_scale_pages, v_scale_pages fp16 pools [num_pages][page_size][num_kv_heads]
 * Device check: slot >= num_pages*page_size is skipped and recorded.
 */
int pkv_kv_cache_write(const void* k, const void* v, const int64_t* slot_mapping,
                       int64_t num_tokens, void* k_pages, void* v_pages,
                       int num_kv_heads, int head_dim, int page_size, int64_t num_pages,
                       pkv_dtype dtype, const void* k_scale, const void* v_scale,
                       void* k_scale_pages, void* v_scale_pages, pkv_stream_t stream);

/*
 * Cache append with INT8 quantisation fused in: each (token, KV head) row of
 * k and v (head_dim elements of src_dtype: PKV_BF16, PKV_F16 or PKV_F32) is
 * quantised symmetrically to 8 bits with one fp16 scale per row ([SYS] §3.2
 * "量化压缩的工程实践" with bits = 8 and one group per row: a = max|x|,
 * scale = fp16(a / 127) rounded to nearest even, code =
 * clamp(round_half_even(x / scale), -127, 127) in IEEE fp32; a zero scale or
 * a NaN element gives code 0) and written to slot slot_mapping[t] of the INT8
 * pools and of the fp16 scale pools.
 *
 *   k, v           [num_tokens][num_kv_heads][head_dim], head_dim 64 or 128
 *   k_pages, v_pages           int8 [num_pages][page_size][num_kv_heads][head_dim]
 *   k_scale_pages, v_scale_pages fp16 [num_pages][page_size][num_kv_heads]
 *   slot_mapping   int64 [num_tokens], as for pkv_kv_cache_write
 * Codes and scales are bit-identical to the definition above (deterministic).
 */
int pkv_kv_cache_write_quant(const void* k, const void* v, pkv_dtype src_dtype,
                             const int64_t* slot_mapping, int64_t num_tokens, void* k_pages,
                             void* v_pages, void* k_scale_pages, void* v_scale_pages,
                             int num_kv_heads, int head_dim, int page_size, int64_t num_pages,
                             pkv_stream_t stream);

/*
 * Decode attention: one query token per sequence attends all context_lens[b]
 * cached keys of its sequence (no mask; the query is the last token of the
 * context):  out[b][h] = softmax(scale * q[b][h] . K_b^T) V_b  ([KVFA] §2.1,
 * [KV3X] "KV Cache 的工作原理"), with K_b, V_b gathered page by page through
 * block_tables[b] ([FAPKV] §3.2).  Computed tile by tile with the online
 * softmax recurrence (running max, running sum, rescale of the accumulator by
 * exp(m_old - m_new); [KV3X] "Flash Attention 的分块计算原理", read with the
 * division by the running sum done once at the end), fp32 softmax state
 * ([KVFA] §6 mixed precision) and the output rounded once to q_dtype.
 *
 *   q            [num_seqs][num_q_heads][head_dim] of q_dtype
 *   out          same shape and dtype as q
 *   q_dtype/kv_dtype: (BF16,BF16), (F16,F16), (BF16,I8), (F16,I8), (F32,F32)
 *   k_scales, v_scales: fp16 [num_pages][page_size][num_kv_heads], required
 *                iff kv_dtype == PKV_I8 (dequantised value = code * scale,
 *                the symmetric 8-bit group quantisation of [SYS] §3.2 with one
 *                group per (token, KV head) row)
 *   head_dim     64 or 128; page_size a multiple of 16 (any >= 1 for F32)
 *   num_splits   0 = let the library partition long contexts (split-KV); n > 0
 *                = at most n partitions per sequence.  Partitions are whole
 *                16-token chunks; each writes a normalised partial output and
 *                its log-sum-exp into `workspace`, and a second kernel merges
 *                them (out = sum_p exp(lse_p - lse) o_p).
 *   workspace    device scratch of at least pkv_decode_workspace_size(...)
 *                bytes for the same arguments (may be NULL when that is 0);
 *                owned by the caller, contents need no initialisation, must
 *                not be used by another call in flight at the same time.
 * context_lens[b] == 0 yields a zero output row.
 */
int pkv_paged_attention_decode(const void* q, const void* k_pages, const void* v_pages,
                               const int32_t* block_tables, const int32_t* context_lens,
                               float scale, void* out, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int page_size,
                               int max_pages_per_seq, int64_t num_pages, pkv_dtype q_dtype,
                               pkv_dtype kv_dtype, const void* k_scales, const void* v_scales,
                               void* workspace, size_t workspace_bytes, int num_splits,
                               pkv_stream_t stream);

/*
 * Decode with local (sliding-window) attention: as pkv_paged_attention_decode,
 * but with window > 0 the query (at position context_lens[b]-1) attends only
 * its last `window` keys (the window_size of the local-attention call in [KVFA]
 * §5.1); window <= 0 is the plain call.  Same workspace size.
 */
int pkv_paged_attention_decode_ex(const void* q, const void* k_pages, const void* v_pages,
                                  const int32_t* block_tables, const int32_t* context_lens,
                                  float scale, void* out, int num_seqs, int num_q_heads,
                                  int num_kv_heads, int head_dim, int page_size,
                                  int max_pages_per_seq, int64_t num_pages, pkv_dtype q_dtype,
                                  pkv_dtype kv_dtype, const void* k_scales, const void* v_scales,
                                  void* workspace, size_t workspace_bytes, int num_splits, int window,
                                  pkv_stream_t stream);

/* Workspace bytes pkv_paged_attention_decode needs for these arguments (0 when
 * no sequence can be split).  Pure host function, no CUDA call. */
size_t pkv_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int page_size, int max_pages_per_seq, pkv_dtype kv_dtype,
                                 int num_splits);

/* Number of partitions per sequence and the partition length in tokens that
 * the decode call will use for these arguments (num_splits as above). */
int pkv_decode_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                    int page_size, int max_pages_per_seq, pkv_dtype kv_dtype, int num_splits,
                    int* splits_out, int* split_tokens_out);

/*
 * Prefill with local (sliding-window) attention: as pkv_paged_attention_prefill,
 * but with window > 0 a query row at absolute position pos attends keys
 * max(0, pos-window+1) .. pos (causal) or .. context_len-1 (non-causal);
 * window <= 0 is the plain call.
 */
int pkv_paged_attention_prefill_ex(const void* q, const void* k_pages, const void* v_pages,
                                   const int32_t* block_tables, const int32_t* q_start,
                                   const int32_t* context_lens, int causal, float scale,
                                   void* out, int num_seqs, int total_q, int max_q_len,
                                   int num_q_heads, int num_kv_heads, int head_dim,
                                   int page_size, int max_pages_per_seq, int64_t num_pages,
                                   pkv_dtype dtype, int window, pkv_stream_t stream);

/*
 * Decode attention without any device allocation by the caller.  The pages
 * have no counterpart: this is a convenience for callers that cannot allocate
 * device memory on demand (a server that reserved all HBM for its KV-cache
 * pool at start-up, a plain-C host without a device allocator, a decode loop
 * that must not risk a synchronising cudaMalloc).  Same arguments and results
 * as pkv_paged_attention_decode, minus the workspace: the split-KV scratch is
 * a fixed array of PKV_NOALLOC_SCRATCH_BYTES inside the library, held by
 * every GPU that loads the library until the process exits.
 *   - Returns PKV_ERR_WORKSPACE, before launching anything, when these
 *     arguments need more scratch than that (pkv_decode_workspace_size() >
 *     PKV_NOALLOC_SCRATCH_BYTES); a smaller num_splits lowers the need.
 *   - The first call on each device that needs scratch looks up the array's
 *     device address (cudaGetSymbolAddress); make that first call before any
 *     stream capture.
 *   - All calls share the one array: calls that overlap on the GPU (several
 *     streams or host threads) race on it and must be serialised by the caller.
 *     Its contents persist between calls; no part of it needs to start zeroed.
 *   - The looked-up address is kept for the life of the process.  A
 *     cudaDeviceReset (or anything else that destroys the device's primary
 *     context) unloads the array with the module, so that address, like the
 *     cached address of the device status word, is stale afterwards: do not
 *     call into the library on a device after resetting it in this process.
 * The library allocates no device memory on this path either.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (48u * 1024u * 1024u)
int pkv_paged_attention_decode_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       float scale, void* out, int num_seqs, int num_q_heads,
                                       int num_kv_heads, int head_dim, int page_size,
                                       int max_pages_per_seq, int64_t num_pages, pkv_dtype q_dtype,
                                       pkv_dtype kv_dtype, const void* k_scales,
                                       const void* v_scales, int num_splits, pkv_stream_t stream);

/*
 * Chunked prefill attention.  Query rows are packed: rows q_start[b] ..
 * q_start[b+1]-1 are the n_b = q_start[b+1]-q_start[b] new tokens of sequence
 * b, sitting at absolute positions context_lens[b]-n_b .. context_lens[b]-1
 * (the chunk follows the cached prefix; bottom-right alignment).  With
 * causal != 0, row r attends keys 0 .. context_lens[b]-n_b+r; otherwise all
 * context_lens[b] keys.  The chunk's own K/V must already be in the pool
 * (pkv_kv_cache_write first).  Prompt processing with FlashAttention-style
 * tiling ([FAPKV] §2.1 and §4.1, [KVFA] §3.1), reading K/V through the page
 * table; prefix pages may be shared by several sequences' block tables
 * (refcounted prompt sharing, [KVFA] §4.1 "零拷贝共享").
 *
 *   q, out     [total_q][num_q_heads][head_dim], dtype PKV_BF16 or PKV_F16
 *   q_start    int32 [num_seqs + 1], q_start[0] = 0, nondecreasing,
 *              q_start[num_seqs] = total_q
 *   max_q_len  >= every n_b (sizes the launch grid)
 *   scale      the softmax scale, finite and > 0 (1/sqrt(head_dim) on the
 *              pages); anything else is PKV_ERR_INVALID_ARG
 *   head_dim   64 or 128; page_size a multiple of 16
 *   q, out, k_pages, v_pages 16-byte aligned (else PKV_ERR_INVALID_ARG)
 * n_b > context_lens[b] is recorded as a device range error.
 */
int pkv_paged_attention_prefill(const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* block_tables, const int32_t* q_start,
                                const int32_t* context_lens, int causal, float scale,
                                void* out, int num_seqs, int total_q, int max_q_len,
                                int num_q_heads, int num_kv_heads, int head_dim,
                                int page_size, int max_pages_per_seq, int64_t num_pages,
                                pkv_dtype dtype, pkv_stream_t stream);

/*
 * Host-side block manager for the paged pool (pure host code, thread-safe, no
 * CUDA call).  GPU memory is cut into fixed-size pages handed out on demand
 * and released whole ([KVFA] §4.1 块级内存池); sequences that share a prompt
 * share its pages with reference counts ([KVFA] §4.1 零拷贝共享, [SYS] §3.1);
 * each sequence's page table maps logical to physical pages ([FAPKV] §3.2) and
 * freeing a sequence deletes its table entry (the leak fix of [FAPKV] §5.2).
 *   create:   num_pages physical pages of page_size tokens, at most
 *             max_pages_per_seq pages per sequence; NULL on bad arguments.
 *   add_sequence: a new empty sequence; its id is written to *seq_id_out.
 *   fork:     a child sequence sharing every page of the parent (refcount + 1).
 *   append:   reserve slots for num_tokens new tokens at the end of `seq`
 *             (slots_out[num_tokens], slot = page * page_size + offset, ready for
 *             pkv_kv_cache_write).  If the last page is shared and not full it is
 *             first replaced by a private page (copy-on-write): the pair is
 *             returned in copy_src[0] / copy_dst[0] (arrays of >= 1 entry) with
 *             *num_copies = 1, and the caller must run pkv_copy_pages before
 *             writing.  PKV_ERR_OUT_OF_PAGES (or INVALID_ARG past
 *             max_pages_per_seq) leaves the manager unchanged.
 *   free_sequence: drop the sequence's page references and delete its entry;
 *             pages whose count reaches zero return to the free pool.  Freeing an
 *             unknown or already freed id is PKV_ERR_INVALID_ARG.
 *   block_tables: export int32 [num_seqs][max_pages_per_seq] tables (-1 past
 *             the last page) and context lengths for the attention calls.
 */
typedef struct pkv_block_manager pkv_block_manager;
pkv_block_manager* pkv_bm_create(int64_t num_pages, int page_size, int max_pages_per_seq);
void pkv_bm_destroy(pkv_block_manager* bm);
int pkv_bm_add_sequence(pkv_block_manager* bm, int64_t* seq_id_out);
int pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t* child_out);
int pkv_bm_append(pkv_block_manager* bm, int64_t seq, int num_tokens, int64_t* slots_out,
                  int32_t* copy_src, int32_t* copy_dst, int* num_copies);
int pkv_bm_free_sequence(pkv_block_manager* bm, int64_t seq);
int pkv_bm_block_tables(pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs,
                        int32_t* table_out, int32_t* context_lens_out);
int64_t pkv_bm_num_free_pages(pkv_block_manager* bm);
int pkv_bm_page_refcount(pkv_block_manager* bm, int32_t page);   /* or PKV_ERR_INVALID_ARG */
int pkv_bm_num_sequences(pkv_block_manager* bm);

/*
 * Device copy of whole pages for copy-on-write: page src[i] of the K and V
 * pools is copied to page dst[i] (page_bytes = page_size * num_kv_heads *
 * head_dim * element size; for INT8 pools call it again on the scale pools
 * with their page size in bytes).  src/dst are device int32 arrays of
 * num_copies entries; an out-of-range page is skipped and recorded in the
 * device status word.  Bit-exact.
 */
int pkv_copy_pages(void* k_pages, void* v_pages, const int32_t* src, const int32_t* dst,
                   int num_copies, int64_t page_bytes, int64_t num_pages, pkv_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device.  Returns PKV_OK, PKV_ERR_DEVICE_RANGE, PKV_ERR_DEVICE_TIMEOUT
 * or PKV_ERR_CUDA.  If `detail` is not NULL it receives the first offending
 * value recorded (page, slot or length), or -1.
 */
int pkv_get_device_status(pkv_stream_t stream, int64_t* detail);

/*
 * Self-test of the device time-out path (no counterpart on the pages).  Launches
 * one thread that waits, with the bounded mbarrier wait the prefill kernel uses
 * (1 s of %globaltimer), on a barrier that nothing ever completes.  The wait runs
 * out, PKV_ERR_DEVICE_TIMEOUT is recorded in the device status word and the
 * kernel returns; the context stays usable.  Read the result with
 * pkv_get_device_status.  Returns PKV_OK once launched.
 */
int pkv_selftest_wait_timeout(pkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
