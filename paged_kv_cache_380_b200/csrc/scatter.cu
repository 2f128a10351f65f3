// Cache append: slot-mapping scatter of new K/V rows into their pages.
//
// The paged form of the per-step cache growth of "大模型推理优化实战：KV Cache +
// Flash Attention，让 Token 生成快 3 倍" ("KV Cache 的工作原理": the new k, v are
// appended to the cache every step) with the page table of "Flash Attention与
// Paged KV Cache优化大模型计算效率" §3.2: row t of the new K/V goes to slot
// slot_mapping[t] = page * page_size + offset of the pool.  A pure byte copy,
// so it is bit-exact for every dtype.
//
// HBM-bound: every thread moves U vectors of VEC bytes, issuing all U loads
// before the U stores so each SM keeps tens of KB in flight; the grid is a
// multiple of the SM count and grid-strides over (tensor, token, vector).
#include "pkv_kernels.h"

namespace pkv {
namespace {

template <int VEC> struct Vec;
template <> struct Vec<16> { using T = uint4; };
template <> struct Vec<8> { using T = uint2; };
template <> struct Vec<4> { using T = uint32_t; };
template <> struct Vec<2> { using T = uint16_t; };
template <> struct Vec<1> { using T = uint8_t; };

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

template <int VEC>
__global__ void __launch_bounds__(kThreads)
kv_scatter_kernel(const uint8_t* __restrict__ src_k, const uint8_t* __restrict__ src_v,
                  const int64_t* __restrict__ slots, uint32_t num_tokens,
                  uint8_t* __restrict__ dst_k, uint8_t* __restrict__ dst_v, uint32_t row_vecs,
                  int64_t num_slots, DeviceStatus* status) {
    using V = typename Vec<VEC>::T;
    const uint64_t per_tensor = static_cast<uint64_t>(num_tokens) * row_vecs;
    const uint64_t total = 2 * per_tensor;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    const uint64_t row_bytes = static_cast<uint64_t>(row_vecs) * VEC;
    for (uint64_t base = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
         base < total; base += stride * kUnroll) {
        V val[kUnroll];
        uint8_t* dst[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint64_t item = base + u * stride;
            dst[u] = nullptr;
            if (item < total) {
                const bool is_v = item >= per_tensor;
                const uint64_t w = is_v ? item - per_tensor : item;
                uint32_t t, j;
                if (per_tensor <= 0xffffffffull) {   // 32-bit division when it fits
                    t = static_cast<uint32_t>(w) / row_vecs;
                    j = static_cast<uint32_t>(w) - t * row_vecs;
                } else {
                    t = static_cast<uint32_t>(w / row_vecs);
                    j = static_cast<uint32_t>(w - static_cast<uint64_t>(t) * row_vecs);
                }
                const int64_t s = __ldg(slots + t);
                if (s >= num_slots) {
                    if (j == 0 && !is_v) record_error(status, PKV_ERR_DEVICE_RANGE, s);
                } else if (s >= 0) {
                    const uint8_t* src = (is_v ? src_v : src_k) + t * row_bytes + j * VEC;
                    val[u] = __ldg(reinterpret_cast<const V*>(src));
                    dst[u] = (is_v ? dst_v : dst_k) + static_cast<uint64_t>(s) * row_bytes + j * VEC;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
            if (dst[u]) *reinterpret_cast<V*>(dst[u]) = val[u];
    }
}

int sm_count() {
    static int n = [] {
        int dev = 0, v = 148;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        return v;
    }();
    return n;
}

}  // namespace

cudaError_t launch_kv_scatter(const void* src_k, const void* src_v, const int64_t* slots,
                              int64_t num_tokens, void* dst_k, void* dst_v, int64_t row_bytes,
                              int64_t num_slots, DeviceStatus* status, cudaStream_t stream) {
    if (num_tokens == 0) return cudaSuccess;
    const uintptr_t align = reinterpret_cast<uintptr_t>(src_k) | reinterpret_cast<uintptr_t>(src_v) |
                            reinterpret_cast<uintptr_t>(dst_k) | reinterpret_cast<uintptr_t>(dst_v) |
                            static_cast<uintptr_t>(row_bytes);
    int vec = 16;
    while (vec > 1 && (align % vec)) vec >>= 1;
    const uint64_t row_vecs = static_cast<uint64_t>(row_bytes) / vec;
    const uint64_t total = 2 * static_cast<uint64_t>(num_tokens) * row_vecs;
    const uint64_t want = (total + kThreads * kUnroll - 1) / (kThreads * kUnroll);
    const uint64_t cap = static_cast<uint64_t>(sm_count()) * 8;
    const unsigned blocks = static_cast<unsigned>(want < cap ? want : cap);
    const auto* sk = static_cast<const uint8_t*>(src_k);
    const auto* sv = static_cast<const uint8_t*>(src_v);
    auto* dk = static_cast<uint8_t*>(dst_k);
    auto* dv = static_cast<uint8_t*>(dst_v);
    const uint32_t T = static_cast<uint32_t>(num_tokens);
    const uint32_t rv = static_cast<uint32_t>(row_vecs);
    switch (vec) {
    case 16: kv_scatter_kernel<16><<<blocks, kThreads, 0, stream>>>(sk, sv, slots, T, dk, dv, rv, num_slots, status); break;
    case 8: kv_scatter_kernel<8><<<blocks, kThreads, 0, stream>>>(sk, sv, slots, T, dk, dv, rv, num_slots, status); break;
    case 4: kv_scatter_kernel<4><<<blocks, kThreads, 0, stream>>>(sk, sv, slots, T, dk, dv, rv, num_slots, status); break;
    case 2: kv_scatter_kernel<2><<<blocks, kThreads, 0, stream>>>(sk, sv, slots, T, dk, dv, rv, num_slots, status); break;
    default: kv_scatter_kernel<1><<<blocks, kThreads, 0, stream>>>(sk, sv, slots, T, dk, dv, rv, num_slots, status); break;
    }
    return cudaGetLastError();
}

}  // namespace pkv
