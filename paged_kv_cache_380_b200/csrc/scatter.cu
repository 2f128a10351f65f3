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
// before the U stores so each SM keeps tens of KB in flight; the grid is the
// number of CTAs that can be resident at once (one wave: a partial second wave
// cost a quarter of the bandwidth) and grid-strides over (tensor, token, vector).
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

// Quantise-on-write: one warp per (token, KV head, K or V) row.  Symmetric
// 8-bit quantisation of "LLM推理系统优化：KV缓存管理与动态批处理技术" §3.2 with one
// group per row: a = max|x| (NaN ignored), scale = fp16(a / 127) rounded to
// nearest even, code = clamp(rint(x / scale), -127, 127) with the division in
// IEEE fp32 and ties to even; a zero scale (or a NaN element) gives code 0.
template <typename T, int E>
__global__ void __launch_bounds__(256)
kv_quant_scatter_kernel(const T* __restrict__ src_k, const T* __restrict__ src_v, const int64_t* __restrict__ slots,
                        uint32_t num_tokens, int num_kv_heads, int8_t* __restrict__ kp, int8_t* __restrict__ vp,
                        __half* __restrict__ ks, __half* __restrict__ vs, int64_t num_slots, DeviceStatus* status) {
    constexpr int D = 32 * E;
    const uint64_t rows = static_cast<uint64_t>(num_tokens) * num_kv_heads * 2;
    const int lane = threadIdx.x & 31;
    const uint64_t warps = static_cast<uint64_t>(gridDim.x) * (blockDim.x >> 5);
    for (uint64_t w = (static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; w < rows; w += warps) {
        const bool is_v = w & 1;
        const uint64_t th = w >> 1;                      // token * num_kv_heads + head
        const uint32_t t = static_cast<uint32_t>(th / num_kv_heads);
        const int head = static_cast<int>(th - static_cast<uint64_t>(t) * num_kv_heads);
        const int64_t s = __ldg(slots + t);
        if (s < 0) continue;
        if (s >= num_slots) {
            if (lane == 0 && head == 0 && !is_v) record_error(status, PKV_ERR_DEVICE_RANGE, s);
            continue;
        }
        const T* src = (is_v ? src_v : src_k) + th * D + lane * E;
        float x[E];
#pragma unroll
        for (int i = 0; i < E; ++i) x[i] = static_cast<float>(src[i]);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < E; ++i) a = fmaxf(a, fabsf(x[i]));
#pragma unroll
        for (int off = 16; off; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        const __half s16 = __float2half_rn(__fdiv_rn(a, 127.f));
        const float sc = __half2float(s16);
        int8_t q[E];
#pragma unroll
        for (int i = 0; i < E; ++i) {
            float r = sc != 0.f ? rintf(__fdiv_rn(x[i], sc)) : 0.f;
            if (r != r) r = 0.f;
            q[i] = static_cast<int8_t>(fminf(fmaxf(r, -127.f), 127.f));
        }
        const uint64_t row = static_cast<uint64_t>(s) * num_kv_heads + head;
        int8_t* dst = (is_v ? vp : kp) + row * D + lane * E;
#pragma unroll
        for (int i = 0; i < E; ++i) dst[i] = q[i];
        if (lane == 0) (is_v ? vs : ks)[row] = s16;
    }
}

// CTAs of `kernel` (256 threads, no dynamic shared memory) resident on the whole GPU.
template <typename K>
unsigned resident_ctas(K kernel) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    return static_cast<unsigned>(per_sm * sm_count());
}

}  // namespace

cudaError_t launch_kv_quant_scatter(const void* src_k, const void* src_v, pkv_dtype src_dtype,
                                    const int64_t* slots, int64_t num_tokens, int num_kv_heads, int head_dim,
                                    void* k_pages, void* v_pages, void* k_scales, void* v_scales,
                                    int64_t num_slots, DeviceStatus* status, cudaStream_t stream) {
    if (num_tokens == 0) return cudaSuccess;
    const uint64_t rows = static_cast<uint64_t>(num_tokens) * num_kv_heads * 2;
    const uint64_t want = (rows + 7) / 8;
    static const unsigned cap = resident_ctas(kv_quant_scatter_kernel<__nv_bfloat16, 4>);
    const unsigned blocks = static_cast<unsigned>(want < cap ? want : cap);
    auto* kp = static_cast<int8_t*>(k_pages);
    auto* vp = static_cast<int8_t*>(v_pages);
    auto* ks = static_cast<__half*>(k_scales);
    auto* vs = static_cast<__half*>(v_scales);
    const uint32_t T = static_cast<uint32_t>(num_tokens);
#define PKV_QUANT_LAUNCH(TYPE, E)                                                                         \
    kv_quant_scatter_kernel<TYPE, E><<<blocks, 256, 0, stream>>>(static_cast<const TYPE*>(src_k),          \
                                                                 static_cast<const TYPE*>(src_v), slots, T, \
                                                                 num_kv_heads, kp, vp, ks, vs, num_slots, status)
    const int E = head_dim / 32;
    if (src_dtype == PKV_BF16) {
        if (E == 4) PKV_QUANT_LAUNCH(__nv_bfloat16, 4); else PKV_QUANT_LAUNCH(__nv_bfloat16, 2);
    } else if (src_dtype == PKV_F16) {
        if (E == 4) PKV_QUANT_LAUNCH(__half, 4); else PKV_QUANT_LAUNCH(__half, 2);
    } else {
        if (E == 4) PKV_QUANT_LAUNCH(float, 4); else PKV_QUANT_LAUNCH(float, 2);
    }
#undef PKV_QUANT_LAUNCH
    return cudaGetLastError();
}

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
    static const unsigned cap[5] = {resident_ctas(kv_scatter_kernel<1>), resident_ctas(kv_scatter_kernel<2>),
                                    resident_ctas(kv_scatter_kernel<4>), resident_ctas(kv_scatter_kernel<8>),
                                    resident_ctas(kv_scatter_kernel<16>)};
    const unsigned c = cap[vec == 16 ? 4 : vec == 8 ? 3 : vec == 4 ? 2 : vec == 2 ? 1 : 0];
    const unsigned blocks = static_cast<unsigned>(want < c ? want : c);
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
