// C ABI of libpagedkv (declared in include/pagedkv.h): argument validation,
// the split-KV partitioner and the device status word; the kernels live in
// scatter.cu, decode.cu and prefill.cu.
#include <cmath>
#include <cstdint>
#include <mutex>
#include <set>
#include <utility>

#include "pkv_kernels.h"

namespace pkv {

// One status word per device (every device that loads the library gets its
// own copy of this variable).  Kernels record the first out-of-range index or
// timed-out wait here instead of faulting.
__device__ DeviceStatus g_status;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kChunk = 16;
#ifndef PKV_SPLIT_MAX_CHUNKS
#define PKV_SPLIT_MAX_CHUNKS 128  // longest automatic partition: 128 chunks of 16 tokens (2048)
#endif

DeviceStatus* status_ptr() {
    static std::mutex mu;
    static DeviceStatus* ptrs[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<DeviceStatus*>(p);
    }
    return ptrs[dev];
}

int sm_count() {
    int dev = 0, v = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v;
}

int elem_bytes(pkv_dtype t) {
    switch (t) {
    case PKV_F32: return 4;
    case PKV_BF16:
    case PKV_F16: return 2;
    case PKV_I8: return 1;
    }
    return 0;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Plan {
    int splits;            // partitions per sequence the workspace must hold
    int chunks_per_split;  // partition length in 16-token chunks
};

// Split-KV partitioner.  Partitions are whole 16-token chunks (and whole pages
// when a page holds several chunks).  Automatic choice: partitions of at most
// 2048 tokens, halved while the grid would hold fewer than 12 CTAs per SM, but
// not below 512 tokens unless it would not even fill one wave (3 CTAs per SM),
// and never below 256.  The numbers are measured balances: longer partitions
// mean fewer CTAs (less per-CTA set-up, fewer partials to merge) but a longer
// tail.  The 2048-token ceiling beat both 1024 and 4096 on every bench decode
// workload (Llama-2-7B/70B shapes, 131k-token contexts in bf16 and INT8), which
// the fill rule leaves untouched; at batch 16 of the Llama-2-7B shapes the
// 12-per-SM target (1024-token partitions) is 6% faster than stopping at two
// waves of two, and at batch 4 256-token partitions lose 2.7% against 512.
Plan plan_decode(int num_seqs, int num_kv_heads, int page_size, int max_pages_per_seq,
                 pkv_dtype kv_dtype, int num_splits) {
    const int64_t max_tokens = static_cast<int64_t>(max_pages_per_seq) * page_size;
    const int max_chunks = static_cast<int>((max_tokens + kChunk - 1) / kChunk);
    if (kv_dtype == PKV_F32 || max_chunks <= 0) return {1, max_chunks > 0 ? max_chunks : 1};
    int cps;
    if (num_splits > 0) {
        const int s = num_splits < max_chunks ? num_splits : max_chunks;
        cps = (max_chunks + s - 1) / s;
    } else {
        const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads;
        const int64_t sms = sm_count();
        cps = PKV_SPLIT_MAX_CHUNKS;
        for (;;) {
            const int64_t ctas = units * ((max_chunks + cps - 1) / cps);
            if (!((cps > 32 && ctas < 12 * sms) || (cps > 16 && ctas < 3 * sms))) break;
            cps /= 2;
        }
    }
    const int page_chunks = page_size / kChunk > 1 ? page_size / kChunk : 1;
    cps = (cps + page_chunks - 1) / page_chunks * page_chunks;
    return {(max_chunks + cps - 1) / cps, cps};
}

size_t workspace_bytes_for(const Plan& pl, int num_seqs, int num_q_heads, int head_dim) {
    if (pl.splits <= 1) return 0;
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * pl.splits;
    const size_t o_bytes = (rows * head_dim * sizeof(float) + 255) / 256 * 256;
    return o_bytes + rows * sizeof(float);
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA; }

}  // namespace

DeviceStatus* device_status_ptr() { return status_ptr(); }

cudaError_t ensure_dynamic_smem(const void* kernel, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<const void*, int>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kernel, dev})) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert({kernel, dev});
    return e;
}

}  // namespace pkv

using namespace pkv;

extern "C" {

const char* pkv_error_string(int code) {
    switch (code) {
    case PKV_OK: return "success";
    case PKV_ERR_INVALID_ARG: return "invalid argument (null pointer, bad size or shape, misalignment)";
    case PKV_ERR_UNSUPPORTED: return "unsupported configuration (dtype combination, head_dim, page_size or group size)";
    case PKV_ERR_WORKSPACE: return "workspace missing or smaller than pkv_decode_workspace_size()";
    case PKV_ERR_CUDA: return "a CUDA runtime call failed";
    case PKV_ERR_DEVICE_RANGE: return "device saw an out-of-range page, slot or length (access skipped)";
    case PKV_ERR_DEVICE_TIMEOUT: return "a bounded device wait gave up";
    case PKV_ERR_OUT_OF_PAGES: return "the block manager has no free page left";
    default: return "unknown pagedkv status";
    }
}

int pkv_kv_cache_write(const void* k, const void* v, const int64_t* slot_mapping, int64_t num_tokens,
                       void* k_pages, void* v_pages, int num_kv_heads, int head_dim, int page_size,
                       int64_t num_pages, pkv_dtype dtype, const void* k_scale, const void* v_scale,
                       void* k_scale_pages, void* v_scale_pages, pkv_stream_t stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || page_size <= 0 || num_pages <= 0)
        return PKV_ERR_INVALID_ARG;
    const int eb = elem_bytes(dtype);
    if (!eb) return PKV_ERR_INVALID_ARG;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !slot_mapping || !k_pages || !v_pages || !aligned(slot_mapping, 8)) return PKV_ERR_INVALID_ARG;
    if (dtype == PKV_I8 && (!k_scale || !v_scale || !k_scale_pages || !v_scale_pages)) return PKV_ERR_INVALID_ARG;
    if (num_tokens > 0xffffffffLL) return PKV_ERR_UNSUPPORTED;
    DeviceStatus* st = status_ptr();
    if (!st) return PKV_ERR_CUDA;
    auto s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t num_slots = num_pages * page_size;
    const int64_t row_bytes = static_cast<int64_t>(num_kv_heads) * head_dim * eb;
    int rc = from_cuda(launch_kv_scatter(k, v, slot_mapping, num_tokens, k_pages, v_pages, row_bytes,
                                         num_slots, st, s));
    if (rc == PKV_OK && dtype == PKV_I8)
        rc = from_cuda(launch_kv_scatter(k_scale, v_scale, slot_mapping, num_tokens, k_scale_pages,
                                         v_scale_pages, static_cast<int64_t>(num_kv_heads) * 2, num_slots,
                                         st, s));
    return rc;
}

int pkv_kv_cache_write_quant(const void* k, const void* v, pkv_dtype src_dtype, const int64_t* slot_mapping,
                             int64_t num_tokens, void* k_pages, void* v_pages, void* k_scale_pages,
                             void* v_scale_pages, int num_kv_heads, int head_dim, int page_size,
                             int64_t num_pages, pkv_stream_t stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || page_size <= 0 || num_pages <= 0)
        return PKV_ERR_INVALID_ARG;
    if (src_dtype != PKV_BF16 && src_dtype != PKV_F16 && src_dtype != PKV_F32) return PKV_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !slot_mapping || !k_pages || !v_pages || !k_scale_pages || !v_scale_pages ||
        !aligned(slot_mapping, 8) || !aligned(k_scale_pages, 2) || !aligned(v_scale_pages, 2))
        return PKV_ERR_INVALID_ARG;
    if (num_tokens > 0xffffffffLL) return PKV_ERR_UNSUPPORTED;
    DeviceStatus* st = status_ptr();
    if (!st) return PKV_ERR_CUDA;
    return from_cuda(launch_kv_quant_scatter(k, v, src_dtype, slot_mapping, num_tokens, num_kv_heads, head_dim,
                                             k_pages, v_pages, k_scale_pages, v_scale_pages,
                                             num_pages * page_size, st, reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_decode_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int page_size,
                    int max_pages_per_seq, pkv_dtype kv_dtype, int num_splits, int* splits_out,
                    int* split_tokens_out) {
    (void)num_q_heads;
    (void)head_dim;
    if (num_seqs < 0 || num_kv_heads <= 0 || page_size <= 0 || max_pages_per_seq <= 0 || num_splits < 0)
        return PKV_ERR_INVALID_ARG;
    const Plan pl = plan_decode(num_seqs, num_kv_heads, page_size, max_pages_per_seq, kv_dtype, num_splits);
    if (splits_out) *splits_out = pl.splits;
    if (split_tokens_out) *split_tokens_out = pl.chunks_per_split * kChunk;
    return PKV_OK;
}

size_t pkv_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                 int page_size, int max_pages_per_seq, pkv_dtype kv_dtype,
                                 int num_splits) {
    if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || page_size <= 0 ||
        max_pages_per_seq <= 0 || num_splits < 0)
        return 0;
    const Plan pl = plan_decode(num_seqs, num_kv_heads, page_size, max_pages_per_seq, kv_dtype, num_splits);
    return workspace_bytes_for(pl, num_seqs, num_q_heads, head_dim);
}

int pkv_paged_attention_decode(const void* q, const void* k_pages, const void* v_pages,
                               const int32_t* block_tables, const int32_t* context_lens, float scale,
                               void* out, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int page_size, int max_pages_per_seq, int64_t num_pages, pkv_dtype q_dtype,
                               pkv_dtype kv_dtype, const void* k_scales, const void* v_scales,
                               void* workspace, size_t workspace_bytes, int num_splits,
                               pkv_stream_t stream) {
    return pkv_paged_attention_decode_ex(q, k_pages, v_pages, block_tables, context_lens, scale, out, num_seqs,
                                         num_q_heads, num_kv_heads, head_dim, page_size, max_pages_per_seq,
                                         num_pages, q_dtype, kv_dtype, k_scales, v_scales, workspace,
                                         workspace_bytes, num_splits, 0, stream);
}

int pkv_paged_attention_decode_ex(const void* q, const void* k_pages, const void* v_pages,
                                  const int32_t* block_tables, const int32_t* context_lens, float scale,
                                  void* out, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                  int page_size, int max_pages_per_seq, int64_t num_pages, pkv_dtype q_dtype,
                                  pkv_dtype kv_dtype, const void* k_scales, const void* v_scales,
                                  void* workspace, size_t workspace_bytes, int num_splits, int window,
                                  pkv_stream_t stream) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || page_size <= 0 ||
        max_pages_per_seq <= 0 || num_pages <= 0 || num_splits < 0 || !std::isfinite(scale))
        return PKV_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads) return PKV_ERR_INVALID_ARG;
    if (num_seqs == 0) return PKV_OK;
    if (!q || !k_pages || !v_pages || !block_tables || !context_lens || !out) return PKV_ERR_INVALID_ARG;
    const bool combo_ok = (q_dtype == PKV_F32 && kv_dtype == PKV_F32) ||
                          ((q_dtype == PKV_BF16 || q_dtype == PKV_F16) && (kv_dtype == q_dtype || kv_dtype == PKV_I8));
    if (!combo_ok) return PKV_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (kv_dtype == PKV_I8 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (q_dtype != PKV_F32 && page_size % kChunk) return PKV_ERR_UNSUPPORTED;
    if (num_q_heads / num_kv_heads > 16) return PKV_ERR_UNSUPPORTED;
    if (kv_dtype == PKV_I8 && (!k_scales || !v_scales || !aligned(k_scales, 4) || !aligned(v_scales, 4)))
        return PKV_ERR_INVALID_ARG;
    if (!aligned(q, 4) || !aligned(out, 4) || !aligned(k_pages, 16) || !aligned(v_pages, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4))
        return PKV_ERR_INVALID_ARG;
    if (static_cast<int64_t>(max_pages_per_seq) * page_size > (1LL << 30)) return PKV_ERR_UNSUPPORTED;

    const Plan pl = plan_decode(num_seqs, num_kv_heads, page_size, max_pages_per_seq, kv_dtype, num_splits);
    const size_t need = workspace_bytes_for(pl, num_seqs, num_q_heads, head_dim);
    if (need && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return PKV_ERR_WORKSPACE;
    DeviceStatus* st = status_ptr();
    if (!st) return PKV_ERR_CUDA;

    DecodeParams p{};
    p.q = q;
    p.k_pages = k_pages;
    p.v_pages = v_pages;
    p.k_scales = static_cast<const __half*>(k_scales);
    p.v_scales = static_cast<const __half*>(v_scales);
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.out = out;
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * pl.splits;
    p.o_part = need ? static_cast<float*>(workspace) : nullptr;
    p.lse_part = need ? reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                 (rows * head_dim * sizeof(float) + 255) / 256 * 256)
                      : nullptr;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.page_size = page_size;
    p.max_pages_per_seq = max_pages_per_seq;
    p.num_pages = num_pages;
    p.chunks_per_split = pl.chunks_per_split;
    p.max_splits = pl.splits;
    p.window = window > 0 ? window : 0;
    p.status = st;
    return from_cuda(launch_decode(p, q_dtype, kv_dtype, reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_paged_attention_prefill(const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* block_tables, const int32_t* q_start,
                                const int32_t* context_lens, int causal, float scale, void* out,
                                int num_seqs, int total_q, int max_q_len, int num_q_heads, int num_kv_heads,
                                int head_dim, int page_size, int max_pages_per_seq, int64_t num_pages,
                                pkv_dtype dtype, pkv_stream_t stream) {
    return pkv_paged_attention_prefill_ex(q, k_pages, v_pages, block_tables, q_start, context_lens, causal, scale,
                                          out, num_seqs, total_q, max_q_len, num_q_heads, num_kv_heads, head_dim,
                                          page_size, max_pages_per_seq, num_pages, dtype, 0, stream);
}

int pkv_selftest_wait_timeout(pkv_stream_t stream) {
    DeviceStatus* st = status_ptr();
    if (!st) return PKV_ERR_CUDA;
    return from_cuda(launch_wait_timeout_selftest(st, reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_paged_attention_prefill_ex(const void* q, const void* k_pages, const void* v_pages,
                                   const int32_t* block_tables, const int32_t* q_start,
                                   const int32_t* context_lens, int causal, float scale, void* out,
                                   int num_seqs, int total_q, int max_q_len, int num_q_heads, int num_kv_heads,
                                   int head_dim, int page_size, int max_pages_per_seq, int64_t num_pages,
                                   pkv_dtype dtype, int window, pkv_stream_t stream) {
    if (num_seqs < 0 || total_q < 0 || max_q_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
        head_dim <= 0 || page_size <= 0 || max_pages_per_seq <= 0 || num_pages <= 0 || !std::isfinite(scale) ||
        !(scale > 0.f))
        return PKV_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads) return PKV_ERR_INVALID_ARG;
    if (num_seqs == 0 || total_q == 0 || max_q_len == 0) return PKV_OK;
    if (!q || !k_pages || !v_pages || !block_tables || !q_start || !context_lens || !out)
        return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_BF16 && dtype != PKV_F16) return PKV_ERR_UNSUPPORTED;
    if ((head_dim != 64 && head_dim != 128) || page_size % kChunk) return PKV_ERR_UNSUPPORTED;
    // q and the pools are TMA tensor-map bases; out is written with 16-byte stores
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16))
        return PKV_ERR_INVALID_ARG;
    DeviceStatus* st = status_ptr();
    if (!st) return PKV_ERR_CUDA;
    PrefillParams p{};
    p.q = q;
    p.k_pages = k_pages;
    p.v_pages = v_pages;
    p.block_tables = block_tables;
    p.q_start = q_start;
    p.context_lens = context_lens;
    p.out = out;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.causal = causal ? 1 : 0;
    p.num_seqs = num_seqs;
    p.total_q = total_q;
    p.max_q_len = max_q_len;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.page_size = page_size;
    p.max_pages_per_seq = max_pages_per_seq;
    p.num_pages = num_pages;
    p.window = window > 0 ? window : 0;
    p.status = st;
    return from_cuda(launch_prefill(p, dtype, reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_get_device_status(pkv_stream_t stream, int64_t* detail) {
    if (detail) *detail = -1;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return PKV_ERR_CUDA;
    DeviceStatus h{};
    if (cudaMemcpyFromSymbol(&h, g_status, sizeof h) != cudaSuccess) return PKV_ERR_CUDA;
    if (h.code == 0) return PKV_OK;
    const DeviceStatus zero{};
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof zero) != cudaSuccess) return PKV_ERR_CUDA;
    if (detail) *detail = h.detail;
    return h.code;
}

}  // extern "C"
