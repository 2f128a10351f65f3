// Host-side launch interfaces between api.cu and the kernel translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv_common.cuh"

namespace pkv {

// Device address of this device's status word (set up on first use).
DeviceStatus* device_status_ptr();

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device).
cudaError_t ensure_dynamic_smem(const void* kernel, int bytes);

// ---- cache append -----------------------------------------------------------
// Row t (row_bytes bytes) of src_k/src_v goes to row slots[t] of dst_k/dst_v.
cudaError_t launch_kv_scatter(const void* src_k, const void* src_v, const int64_t* slots,
                              int64_t num_tokens, void* dst_k, void* dst_v, int64_t row_bytes,
                              int64_t num_slots, DeviceStatus* status, cudaStream_t stream);

// Quantise-on-write: rows of head_dim (64 or 128) elements of src_dtype
// (bf16/f16/f32) become int8 codes + one fp16 scale per (token, head) row.
cudaError_t launch_kv_quant_scatter(const void* src_k, const void* src_v, pkv_dtype src_dtype,
                                    const int64_t* slots, int64_t num_tokens, int num_kv_heads, int head_dim,
                                    void* k_pages, void* v_pages, void* k_scales, void* v_scales,
                                    int64_t num_slots, DeviceStatus* status, cudaStream_t stream);

// ---- decode ------------------------------------------------------------------
struct DecodeParams {
    const void* q;
    const void* k_pages;
    const void* v_pages;
    const __half* k_scales;
    const __half* v_scales;
    const int32_t* block_tables;
    const int32_t* context_lens;
    void* out;
    float* o_part;     // [num_seqs][num_q_heads][max_splits][head_dim]
    float* lse_part;   // [num_seqs][num_q_heads][max_splits], log2 domain
    float scale_log2;  // softmax scale * log2(e)
    int num_seqs, num_q_heads, num_kv_heads, head_dim, page_size, max_pages_per_seq;
    int64_t num_pages;
    int chunks_per_split;  // 16-token chunks per partition
    int max_splits;        // partitions the workspace holds (1 = no workspace)
    int window;            // > 0: only the last `window` keys are attended (local attention)
    DeviceStatus* status;
};

cudaError_t launch_decode(const DecodeParams& p, pkv_dtype q_dtype, pkv_dtype kv_dtype,
                          cudaStream_t stream);

// ---- prefill -------------------------------------------------------------------
struct PrefillParams {
    const void* q;
    const void* k_pages;
    const void* v_pages;
    const int32_t* block_tables;
    const int32_t* q_start;
    const int32_t* context_lens;
    void* out;
    float scale_log2;
    int causal;
    int num_seqs, total_q, max_q_len, num_q_heads, num_kv_heads, head_dim, page_size;
    int max_pages_per_seq;
    int64_t num_pages;
    int window;            // > 0: a query at pos sees keys pos-window+1 .. pos only
    DeviceStatus* status;
};

cudaError_t launch_prefill(const PrefillParams& p, pkv_dtype dtype, cudaStream_t stream);
// One bounded mbarrier wait that nothing completes (records PKV_ERR_DEVICE_TIMEOUT).
cudaError_t launch_wait_timeout_selftest(DeviceStatus* st, cudaStream_t stream);

}  // namespace pkv
