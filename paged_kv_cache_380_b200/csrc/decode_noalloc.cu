// Decode attention for callers that cannot allocate device memory.
//
// pkv_paged_attention_decode needs a caller-provided scratch buffer (the
// split-KV workspace) whenever long contexts are split into partitions.  Some
// callers cannot produce one on demand: an inference server that carved all of
// HBM into its KV-cache pool at start-up and forbids later allocations, a
// plain-C host with no device allocator of its own, or a latency-critical
// decode loop where a cudaMalloc/cudaFree could synchronise the device.  This
// entry point takes the same arguments minus the workspace and uses a fixed
// scratch array compiled into the library instead, so it allocates nothing.
//
// The array (PKV_NOALLOC_SCRATCH_BYTES per GPU) is a file-scope __device__
// variable: every GPU that loads the library holds it until the process
// exits.  Its device address is looked up once per device with
// cudaGetSymbolAddress, on the first call that needs it, with that device
// current (host code cannot use the variable's name as a device pointer).
// All calls share the array, so calls that overlap on the GPU (other streams,
// other host threads) race on it.  Nothing in it has to start at zero: each
// call writes every partial it later reads.
#include <cstdint>
#include <mutex>

#include "pkv_kernels.h"

namespace pkv {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[PKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_decode_scratch on the current device, looked up once per device.
cudaError_t scratch_address(void** out) {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace pkv

extern "C" int pkv_paged_attention_decode_noalloc(
    const void* q, const void* k_pages, const void* v_pages, const int32_t* block_tables,
    const int32_t* context_lens, float scale, void* out, int num_seqs, int num_q_heads, int num_kv_heads,
    int head_dim, int page_size, int max_pages_per_seq, int64_t num_pages, pkv_dtype q_dtype,
    pkv_dtype kv_dtype, const void* k_scales, const void* v_scales, int num_splits, pkv_stream_t stream) {
    const size_t need = pkv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, page_size,
                                                  max_pages_per_seq, kv_dtype, num_splits);
    if (need > PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0 && pkv::scratch_address(&scratch) != cudaSuccess) return PKV_ERR_CUDA;
    return pkv_paged_attention_decode(q, k_pages, v_pages, block_tables, context_lens, scale, out, num_seqs,
                                      num_q_heads, num_kv_heads, head_dim, page_size, max_pages_per_seq,
                                      num_pages, q_dtype, kv_dtype, k_scales, v_scales, scratch,
                                      need > 0 ? PKV_NOALLOC_SCRATCH_BYTES : 0, num_splits, stream);
}
