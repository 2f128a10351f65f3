// Chunked-prefill attention over a paged KV cache (causal, bottom-right).
//
// Query rows q_start[b] .. q_start[b+1]-1 of sequence b sit at absolute
// positions ctx-n .. ctx-1; row r attends keys 0 .. ctx-n+r (causal) or all
// ctx keys.  FlashAttention-style tiling ("Flash Attention与Paged KV Cache优化
// 大模型计算效率" §2.1: tiles of Q and K/V staged on chip, softmax computed
// per tile; "大模型推理优化实战：KV Cache + Flash Attention，让 Token 生成快 3 倍",
// "Flash Attention 的分块计算原理": online max/sum with rescaling), K/V tiles
// gathered through the block table.
//
// This version runs the two contractions with warp-level mma.sync (16 query
// rows per warp, 64-key tiles, cp.async double buffering).
#include <cmath>
#include <type_traits>

#include "pkv_kernels.h"
#include "pkv_ptx.cuh"

namespace pkv {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int BM = 64, BN = 64, HD = 128, kRowB = HD * 2, kUnits = kRowB / 16;
constexpr int kThreads = 128;
constexpr int kTileB = BN * kRowB;   // one K or V tile
constexpr int kSmem = BM * kRowB + 4 * kTileB;

template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value)
        ptx::mma_bf16_16816(d, a0, a1, a2, a3, b0, b1);
    else
        ptx::mma_f16_16816(d, a0, a1, a2, a3, b0, b1);
}

__device__ __forceinline__ uint32_t swz(int r, int u) { return r * kRowB + ((u ^ (r & 7)) << 4); }

template <typename T>
__global__ void __launch_bounds__(kThreads) prefill_mma_kernel(const PrefillParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
    const int mt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int Hq = p.num_q_heads, Hkv = p.num_kv_heads, kvh = h / (Hq / Hkv), ps = p.page_size;
    const int q0 = __ldg(p.q_start + b), n = __ldg(p.q_start + b + 1) - q0;
    const int ctx = __ldg(p.context_lens + b);
    const int r0 = mt * BM;
    if (r0 >= n) return;
    if (n > ctx || ctx > p.max_pages_per_seq * ps) {
        if (mt == 0 && h == 0 && tid == 0) record_error(p.status, PKV_ERR_DEVICE_RANGE, ctx);
        return;
    }
    const int last_row = min(r0 + BM, n) - 1;
    const int max_key = p.causal ? ctx - n + last_row : ctx - 1;
    const int n_tiles = max_key / BN + 1;

    const uint32_t sQ = ptx::smem_u32(smem);
    const uint32_t sKV = sQ + BM * kRowB;   // [buf][K|V]
    const uint8_t* kpool = static_cast<const uint8_t*>(p.k_pages);
    const uint8_t* vpool = static_cast<const uint8_t*>(p.v_pages);
    const int32_t* bt = p.block_tables + static_cast<size_t>(b) * p.max_pages_per_seq;

    // Q tile (rows past the chunk are zero-filled)
    {
        const uint8_t* q = static_cast<const uint8_t*>(p.q);
        for (int x = tid; x < BM * kUnits; x += kThreads) {
            const int r = x / kUnits, u = x % kUnits;
            const bool ok = r0 + r < n;
            const size_t off = (static_cast<size_t>(q0 + r0 + r) * Hq + h) * kRowB + u * 16;
            ptx::cp_async16(sQ + swz(r, u), ok ? q + off : q, ok ? 16u : 0u);
        }
    }
    auto load_tile = [&](int j) {
        const uint32_t sK = sKV + (j & 1) * 2 * kTileB, sV = sK + kTileB;
        for (int x = tid; x < BN * kUnits; x += kThreads) {
            const int r = x / kUnits, u = x % kUnits;
            const int key = j * BN + r;
            bool ok = key < ctx;
            int page = 0;
            if (ok) {
                page = __ldg(bt + key / ps);
                if (page < 0 || page >= p.num_pages) {
                    if (u == 0) record_error(p.status, PKV_ERR_DEVICE_RANGE, page);
                    ok = false;
                }
            }
            const size_t off = ((static_cast<size_t>(page) * ps + key % ps) * Hkv + kvh) * kRowB + u * 16;
            ptx::cp_async16(sK + swz(r, u), ok ? kpool + off : kpool, ok ? 16u : 0u);
            ptx::cp_async16(sV + swz(r, u), ok ? vpool + off : vpool, ok ? 16u : 0u);
        }
    };
    load_tile(0);
    ptx::cp_async_commit();

    uint32_t qa[HD / 16][4];
    float o[HD / 8][4];
#pragma unroll
    for (int dt = 0; dt < HD / 8; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
    const int row_a = r0 + warp * 16 + g, row_b = row_a + 8;
    const int lim_a = p.causal ? ctx - n + row_a : ctx - 1;
    const int lim_b = p.causal ? ctx - n + row_b : ctx - 1;

    for (int j = 0; j < n_tiles; ++j) {
        if (j + 1 < n_tiles) {
            load_tile(j + 1);
            ptx::cp_async_commit();
            ptx::cp_async_wait<1>();
        } else {
            ptx::cp_async_wait<0>();
        }
        __syncthreads();
        if (j == 0) {
            const int r = warp * 16 + (lane & 15);
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
                ptx::ldmatrix_x4(sQ + swz(r, 2 * kk + (lane >> 4)), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
        }
        const uint32_t sK = sKV + (j & 1) * 2 * kTileB, sV = sK + kTileB;

        float s[BN / 8][4];
#pragma unroll
        for (int nt = 0; nt < BN / 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < BN / 16; ++np) {
                const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int u = 2 * kk + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ptx::ldmatrix_x4(sK + swz(r, u), b0, b1, b2, b3);
                mma16816<T>(s[2 * np], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
                mma16816<T>(s[2 * np + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
            }
        }
        // mask + online softmax (rows row_a, row_b)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < BN / 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = j * BN + nt * 8 + 2 * c + (e & 1);
                const int lim = (e < 2) ? lim_a : lim_b;
                s[nt][e] = key <= lim ? s[nt][e] * p.scale_log2 : -INFINITY;
                mx[e >> 1] = fmaxf(mx[e >> 1], s[nt][e]);
            }
        }
        float corr[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(kFull, mx[i], 1));
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(kFull, mx[i], 2));
            const float m_new = fmaxf(m_r[i], mx[i]);
            // a row whose keys are all masked so far keeps m = -inf: use 0 as its shift
            const float shift = m_new == -INFINITY ? 0.f : m_new;
            corr[i] = ptx::ex2(m_r[i] - shift);
            m_r[i] = m_new;
            mx[i] = shift;
        }
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < BN / 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s[nt][e] = ptx::ex2(s[nt][e] - mx[e >> 1]);
                rs[e >> 1] += s[nt][e];
            }
        }
        l_r[0] = l_r[0] * corr[0] + rs[0];
        l_r[1] = l_r[1] * corr[1] + rs[1];
#pragma unroll
        for (int dt = 0; dt < HD / 8; ++dt) {
            o[dt][0] *= corr[0]; o[dt][1] *= corr[0];
            o[dt][2] *= corr[1]; o[dt][3] *= corr[1];
        }
        // O += P V
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t a0 = pack2<T>(s[2 * kk][0], s[2 * kk][1]);
            const uint32_t a1 = pack2<T>(s[2 * kk][2], s[2 * kk][3]);
            const uint32_t a2 = pack2<T>(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            const uint32_t a3 = pack2<T>(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int dp = 0; dp < HD / 16; ++dp) {
                const int r = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                const int u = 2 * dp + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ptx::ldmatrix_x4_trans(sV + swz(r, u), b0, b1, b2, b3);
                mma16816<T>(o[2 * dp], a0, a1, a2, a3, b0, b1);
                mma16816<T>(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        l_r[i] += __shfl_xor_sync(kFull, l_r[i], 1);
        l_r[i] += __shfl_xor_sync(kFull, l_r[i], 2);
    }
    T* out = static_cast<T*>(p.out);
    const float inv_a = 1.f / l_r[0], inv_b = 1.f / l_r[1];
#pragma unroll
    for (int dt = 0; dt < HD / 8; ++dt) {
        const int d = dt * 8 + 2 * c;
        if (row_a < n)
            *reinterpret_cast<uint32_t*>(out + (static_cast<size_t>(q0 + row_a) * Hq + h) * HD + d) =
                pack2<T>(o[dt][0] * inv_a, o[dt][1] * inv_a);
        if (row_b < n)
            *reinterpret_cast<uint32_t*>(out + (static_cast<size_t>(q0 + row_b) * Hq + h) * HD + d) =
                pack2<T>(o[dt][2] * inv_b, o[dt][3] * inv_b);
    }
}

template <typename T>
cudaError_t run(const PrefillParams& p, cudaStream_t stream) {
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(prefill_mma_kernel<T>), kSmem);
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(p.max_q_len, BM), p.num_q_heads, p.num_seqs);
    prefill_mma_kernel<T><<<grid, kThreads, kSmem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p, pkv_dtype dtype, cudaStream_t stream) {
    if (p.max_q_len <= 0 || p.num_seqs <= 0) return cudaSuccess;
    return dtype == PKV_BF16 ? run<__nv_bfloat16>(p, stream) : run<__half>(p, stream);
}

}  // namespace pkv
