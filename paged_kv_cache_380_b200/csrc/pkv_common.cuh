// Shared device-side definitions of libpagedkv (sm_100a only).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pagedkv.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libpagedkv is written for sm_100a (B200) only"
#endif

namespace pkv {

// Device status word: [0] = first error code (0 = none), [1..2] = detail
// (64-bit offending value).  One per device, lives in api.cu; kernels get its
// address as an argument.
struct DeviceStatus {
    int code;
    int pad;
    long long detail;
};

__device__ __forceinline__ void record_error(DeviceStatus* st, int code, long long detail) {
    if (atomicCAS(&st->code, 0, code) == 0) {
        atomicExch(reinterpret_cast<unsigned long long*>(&st->detail),
                   static_cast<unsigned long long>(detail));
    }
}

// Iteration cap for every spin wait on an mbarrier: far above any legitimate
// wait (each probe of try_wait may itself suspend for a while), low enough
// that a stalled pipeline gives up within about a second.
constexpr uint32_t kSpinLimit = 1u << 22;

template <typename T> struct DType;
template <> struct DType<__nv_bfloat16> { static constexpr pkv_dtype value = PKV_BF16; };
template <> struct DType<__half> { static constexpr pkv_dtype value = PKV_F16; };
template <> struct DType<float> { static constexpr pkv_dtype value = PKV_F32; };
template <> struct DType<int8_t> { static constexpr pkv_dtype value = PKV_I8; };

template <typename T> __device__ __forceinline__ T from_float(float x);
template <> __device__ __forceinline__ __nv_bfloat16 from_float(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ __half from_float(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ float from_float(float x) { return x; }

// Pack two floats into a 32-bit pair of 16-bit values (low half = a).
template <typename T> __device__ __forceinline__ uint32_t pack2(float a, float b);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Unpack a 32-bit pair of 16-bit values (low half first) to two floats.
template <typename T> __device__ __forceinline__ float2 unpack2(uint32_t v);
template <> __device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
template <> __device__ __forceinline__ float2 unpack2<__half>(uint32_t v) {
    return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

__host__ __device__ constexpr inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace pkv
