// Decode attention over a paged KV cache: one query token per sequence.
//
// What is computed: out[b][h] = softmax(scale * q[b][h] . K_b^T) V_b over all
// context_lens[b] cached tokens ("大模型推理优化：KV Cache与FlashAttention实战"
// §2.1; "大模型推理优化实战：KV Cache + Flash Attention，让 Token 生成快 3 倍",
// "KV Cache 的工作原理"), K_b/V_b read page by page through the block table
// ("Flash Attention与Paged KV Cache优化大模型计算效率" §3.2), query head h using
// KV head h / G ("LLM推理系统优化：KV缓存管理与动态批处理技术" §2.1, GQA).  The
// softmax is evaluated tile by tile with the online recurrence of the page
// "KV Cache + Flash Attention，让 Token 生成快 3 倍" ("Flash Attention 的分块计算
// 原理": running max m, running sum l, accumulator rescaled by exp(m_old -
// m_new)); the division by l happens once at the end (the printed loop divides
// inside the loop as well, which double-normalises; the plain reading is the
// standard recurrence).  Softmax state and accumulators are fp32 ("大模型推理优化：
// KV Cache与FlashAttention实战" §6), exponentials in base 2 with log2(e) folded
// into the scale.
//
// B200 design (HBM-bound: every K/V byte is read once, ~1-8 flop per byte):
//  * CTA = (partition, KV head, sequence); its WARPS warps take the
//    partition's 16-token chunks round-robin, each warp with a private
//    STAGES-deep cp.async ring (16-byte copies, zero-filled past the context)
//    so ~100 KB per SM is in flight.  Page tiles land XOR-swizzled (16-byte
//    unit u of row r at u ^ (r & 7)) so ldmatrix reads are bank-conflict free.
//  * All G query heads of the KV head share each K/V tile.  Both contractions
//    run on the tensor cores with the context as the M dimension, so no group
//    size wastes rows:  S^T[16 tok x 8 heads] = K[16 x D] . Q^T and
//    O^T[D x 8 heads] += V^T[D x 16 tok] . P^T; P^T's fragments come from S^T's
//    accumulator by an 8x8 movmatrix transpose.  Max/sum across the chunk use
//    warp shuffles.
//  * INT8 pages (one fp16 scale per token and KV head, the symmetric
//    quantisation of "LLM推理系统优化" §3.2): codes are widened exactly to the
//    MMA type in registers; the key scale multiplies the score of its token,
//    the value scale multiplies that token's probability before P.V.  The
//    d-axis is permuted consistently in Q and K (and in V and the output) so
//    that each thread's ldmatrix bytes form whole MMA fragments.
//  * Long contexts are split into partitions of whole chunks (split-KV); each
//    CTA writes its normalised partial and log-sum-exp, and a second kernel
//    merges them: lse = log2 sum 2^lse_p, out = sum_p 2^(lse_p - lse) o_p.
#include <cmath>
#include <type_traits>

#include "pkv_kernels.h"
#include "pkv_ptx.cuh"

namespace pkv {
namespace {

constexpr int kChunk = 16;            // tokens per pipeline stage of one warp
constexpr unsigned kFull = 0xffffffffu;

// int8 code pair (bytes a, b of w, each offset by 128 through w ^ 0x80808080)
// -> fp16x2 holding 1152 + code, exact, in one byte permute: the offset byte
// u = code + 128 becomes the low mantissa byte of the fp16 number 1024 + u
// (exponent pattern 0x64).
__device__ __forceinline__ uint32_t s8pair_biased(uint32_t w_biased, uint32_t sel_a, uint32_t sel_b) {
    return __byte_perm(w_biased, 0x64646464u, sel_a | 0x40u | (sel_b << 8) | 0x4000u);
}
// Both operands stay biased, which saves a subtraction per code pair:
//  * keys: sum_d q_d (k_d + 1152) = sum_d q_d k_d + 1152 sum_d q_d, so each score
//    accumulator starts from -1152 sum_d q_d (of the fp16 q the MMAs see) and the bias
//    cancels inside the fp32 accumulation (measured: the same error against the oracle
//    as subtracting 1152 from every code, also for all-positive queries);
//  * values: sum_t p_t (v_t + 1152) = sum_t p_t v_t + 1152 sum_t p_t, and sum_t p_t
//    comes from one more MMA per chunk against a matrix of ones (the same fp16 P
//    operand, p <= 1), accumulated and rescaled with O and subtracted at the end.
constexpr float kCodeBias = 1152.f;
constexpr uint32_t kOnePair = 0x3C003C00u;    // fp16x2 (1, 1)

template <typename QT>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    if constexpr (std::is_same<QT, __nv_bfloat16>::value)
        ptx::mma_bf16_16816(d, a0, a1, a2, a3, b0, b1);
    else
        ptx::mma_f16_16816(d, a0, a1, a2, a3, b0, b1);
}

template <typename QT, typename KVT, int HD, int NT, int WARPS, int STAGES>
struct DecodeCfg {
    static constexpr bool kInt8 = std::is_same<KVT, int8_t>::value;
    static constexpr int kRowBytes = HD * static_cast<int>(sizeof(KVT));
    static constexpr int kUnits = kRowBytes / 16;
    static constexpr int kTile = kChunk * kRowBytes;
    static constexpr int kScaleBytes = kInt8 ? 2 * kChunk * 4 : 0;
    static constexpr int kStage = 2 * kTile + kScaleBytes;
    static constexpr int kPipe = WARPS * STAGES * kStage;
    static constexpr int kMerge = WARPS * 8 * NT * (HD + 2) * 4;
    static constexpr int kSmem = kPipe > kMerge ? kPipe : kMerge;
    static constexpr int kDT = HD / 16;   // 16-wide d tiles (MMA k-steps for QK, M tiles for PV)
    // Lazy rescale: probabilities are taken against a reference max that may lag the
    // running max by up to 2^kRescale (P <= 256 in the bf16 / fp16 MMA operand).  The
    // INT8 path multiplies P by the value scale in fp16, so it keeps P <= 1 there.
    static constexpr float kRescale = kInt8 ? 0.f : 8.f;
    static_assert(kUnits >= 8, "rows must span at least 128 bytes for the swizzle");
    static_assert(!kInt8 || HD == 128, "INT8 pages need head_dim 128");
};

template <typename QT, typename KVT, int HD, int NT, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32)
decode_mma_kernel(const DecodeParams p) {
    using Cfg = DecodeCfg<QT, KVT, HD, NT, WARPS, STAGES>;
    // INT8 pages run the MMAs in fp16 (codes widen to fp16, offset by 1152, in one byte
    // permute per pair after one XOR per four codes)
    using MT = typename std::conditional<Cfg::kInt8, __half, QT>::type;
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    // KV heads vary fastest: the CTAs of one token range for all KV heads run side by
    // side, so a token's K/V rows (all heads contiguous in the page) are read together
    const int kvh = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
    const int Hq = p.num_q_heads, Hkv = p.num_kv_heads, G = Hq / Hkv, ps = p.page_size;

    const int ctx = __ldg(p.context_lens + b);
    if (ctx < 0 || ctx > p.max_pages_per_seq * ps) {
        if (split == 0 && kvh == 0 && threadIdx.x == 0) record_error(p.status, PKV_ERR_DEVICE_RANGE, ctx);
        return;
    }
    QT* out = static_cast<QT*>(p.out);
    const size_t head0 = static_cast<size_t>(b) * Hq + static_cast<size_t>(kvh) * G;
    if (ctx == 0) {
        if (split == 0)
            for (int i = threadIdx.x; i < G * HD; i += WARPS * 32) out[head0 * HD + i] = from_float<QT>(0.f);
        return;
    }
    // keys k_lo .. ctx-1 are attended (k_lo > 0 only with a local-attention window)
    const int k_lo = (p.window > 0 && ctx > p.window) ? ctx - p.window : 0;
    const int c_lo = k_lo / kChunk;
    const int n_chunks = ceil_div(ctx, kChunk) - c_lo;
    const int nsplit = ceil_div(n_chunks, p.chunks_per_split);
    if (split >= nsplit) return;
    const int c_begin = c_lo + split * p.chunks_per_split;
    const int c_end = min(c_begin + p.chunks_per_split, c_lo + n_chunks);
    const int n_mine = (c_end - c_begin > warp) ? ceil_div(c_end - c_begin - warp, WARPS) : 0;

    // ---- query fragments (B operand of S^T = K . Q^T), kept in registers ----
    uint32_t qf[NT][Cfg::kDT][2];
    {
        const QT* q = static_cast<const QT*>(p.q);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int n = nt * 8 + g;
            const QT* qrow = q + (head0 + n) * HD;
#pragma unroll
            for (int kk = 0; kk < Cfg::kDT; ++kk) {
                const int d0 = Cfg::kInt8 ? kk * 16 + 4 * c : kk * 16 + 2 * c;
                const int d1 = Cfg::kInt8 ? d0 + 2 : d0 + 8;
                qf[nt][kk][0] = n < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + d0)) : 0u;
                qf[nt][kk][1] = n < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + d1)) : 0u;
            }
        }
    }
    // INT8 pages: q goes to fp16 for the MMA.  Each head is first scaled by a power
    // of two (exact) so that its largest |q| stays below 2^15; the inverse factor
    // multiplies that head's scores.  qinv[nt][h] is the factor of head 2c + h.
    float qinv[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) qinv[nt][0] = qinv[nt][1] = 1.f;
    if constexpr (Cfg::kInt8) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float mq = 0.f;
#pragma unroll
            for (int kk = 0; kk < Cfg::kDT; ++kk)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float2 v = unpack2<QT>(qf[nt][kk][i]);
                    mq = fmaxf(mq, fmaxf(fabsf(v.x), fabsf(v.y)));
                }
            mq = fmaxf(mq, __shfl_xor_sync(kFull, mq, 1));
            mq = fmaxf(mq, __shfl_xor_sync(kFull, mq, 2));
            const int e = ((__float_as_int(mq) >> 23) & 0xff) - 127;      // floor(log2(max |q|))
            const float f = e >= 15 ? __int_as_float((127 + 14 - e) << 23) : 1.f;
#pragma unroll
            for (int kk = 0; kk < Cfg::kDT; ++kk)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float2 v = unpack2<QT>(qf[nt][kk][i]);
                    qf[nt][kk][i] = pack2<__half>(v.x * f, v.y * f);
                }
            const float inv = 1.f / f;                                    // exact: a power of two
            qinv[nt][0] = __shfl_sync(kFull, inv, (2 * c) * 4);
            qinv[nt][1] = __shfl_sync(kFull, inv, (2 * c + 1) * 4);
        }
    }
    // INT8 pages: keys widen to 1152 + code, so every score of head n carries 1152 sum_d q_nd;
    // the accumulators start from minus that (of the fp16 q the MMAs see).
    float kbias[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) kbias[nt][0] = kbias[nt][1] = 0.f;
    if constexpr (Cfg::kInt8) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float sq = 0.f;
#pragma unroll
            for (int kk = 0; kk < Cfg::kDT; ++kk)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float2 v = unpack2<__half>(qf[nt][kk][i]);
                    sq += v.x + v.y;
                }
            sq += __shfl_xor_sync(kFull, sq, 1);
            sq += __shfl_xor_sync(kFull, sq, 2);
            kbias[nt][0] = -kCodeBias * __shfl_sync(kFull, sq, (2 * c) * 4);
            kbias[nt][1] = -kCodeBias * __shfl_sync(kFull, sq, (2 * c + 1) * 4);
        }
    }

    // ---- per-warp cp.async ring ----
    // Everything per lane that does not change from chunk to chunk is computed once:
    // the shared-memory destination of each of the lane's 16-byte copies, their byte
    // offsets from the chunk's first pool row, and the chunk-relative token row.  Per
    // chunk only the pool row (read with the page indices, 32 chunks at a time) and
    // the context test change.
    uint8_t* ring = smem + warp * STAGES * Cfg::kStage;
    const uint32_t ring_s = ptx::smem_u32(ring);
    const uint8_t* kpool = static_cast<const uint8_t*>(p.k_pages);
    const uint8_t* vpool = static_cast<const uint8_t*>(p.v_pages);
    const int32_t* bt = p.block_tables + static_cast<size_t>(b) * p.max_pages_per_seq;
    constexpr int NI = kChunk * Cfg::kUnits / 32;          // 16-byte copies per lane per tensor
    uint32_t cp_dst[NI];
    int32_t cp_off[NI], cp_row[NI];
#pragma unroll
    for (int k = 0; k < NI; ++k) {
        const int x = lane + 32 * k, r = x / Cfg::kUnits, u = x % Cfg::kUnits;
        cp_row[k] = r;
        cp_dst[k] = r * Cfg::kRowBytes + ((u ^ (r & 7)) << 4);
        cp_off[k] = r * Hkv * Cfg::kRowBytes + u * 16;
    }
    const int sc_row = lane & 15;                           // INT8 scale copies: token row of this lane
    int64_t first_row_reg = 0;                              // pool row of chunk (i & ~31) + lane, or -1
    int issue_slot = 0;

    auto issue = [&](int i) {
        if (i < n_mine) {
            if ((i & 31) == 0) {        // first pool rows of my next 32 chunks, one per lane
                const int j = i + lane;
                int64_t fr = 0;
                if (j < n_mine) {
                    const int tok = (c_begin + warp + j * WARPS) * kChunk;
                    const int page = __ldg(bt + tok / ps);
                    fr = (page >= 0 && page < p.num_pages) ? static_cast<int64_t>(page) * ps + tok % ps : -1;
                    if (fr < 0) record_error(p.status, PKV_ERR_DEVICE_RANGE, page);
                }
                first_row_reg = fr;
            }
            const int64_t frow = __shfl_sync(kFull, first_row_reg, i & 31);
            const int rem = frow < 0 ? 0 : ctx - (c_begin + warp + i * WARPS) * kChunk;   // valid rows
            const int64_t row0 = (frow < 0 ? 0 : frow) * Hkv + kvh;
            const uint8_t* kb = kpool + row0 * Cfg::kRowBytes;
            const uint8_t* vb = vpool + row0 * Cfg::kRowBytes;
            const uint32_t sK = ring_s + issue_slot * Cfg::kStage;
            const uint32_t sV = sK + Cfg::kTile;
#pragma unroll
            for (int k = 0; k < NI; ++k) {
                const bool ok = cp_row[k] < rem;
                ptx::cp_async16(sK + cp_dst[k], ok ? kb + cp_off[k] : kpool, ok ? 16u : 0u);
                ptx::cp_async16(sV + cp_dst[k], ok ? vb + cp_off[k] : vpool, ok ? 16u : 0u);
            }
            if constexpr (Cfg::kInt8) {   // lanes 0-15: key scales, 16-31: value scales
                const bool ok = sc_row < rem;
                const __half* sc = lane < 16 ? p.k_scales : p.v_scales;
                const uintptr_t a = reinterpret_cast<uintptr_t>(sc + (row0 + static_cast<int64_t>(sc_row) * Hkv));
                ptx::cp_async4(sV + Cfg::kTile + lane * 4,
                               ok ? reinterpret_cast<const void*>(a & ~uintptr_t(3)) : static_cast<const void*>(sc),
                               ok ? 4u : 0u);
            }
            issue_slot = issue_slot + 1 == STAGES ? 0 : issue_slot + 1;
        }
        ptx::cp_async_commit();
    };

    float m[NT][2], l[NT][2], o[NT][Cfg::kDT][4];
    float osum[NT][4];   // INT8: sum over tokens of the fp16 P operand, per head (bias of O)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        m[nt][0] = m[nt][1] = -INFINITY;
        l[nt][0] = l[nt][1] = 0.f;
        osum[nt][0] = osum[nt][1] = osum[nt][2] = osum[nt][3] = 0.f;
#pragma unroll
        for (int dt = 0; dt < Cfg::kDT; ++dt) o[nt][dt][0] = o[nt][dt][1] = o[nt][dt][2] = o[nt][dt][3] = 0.f;
    }

#pragma unroll
    for (int i = 0; i < STAGES - 1; ++i) issue(i);

    int use_slot = 0;
    for (int i = 0; i < n_mine; ++i) {
        issue(i + STAGES - 1);
        ptx::cp_async_wait<STAGES - 1>();
        __syncwarp();
        const uint32_t sK = ring_s + use_slot * Cfg::kStage;
        const uint32_t sV = sK + Cfg::kTile;
        const int tok0 = (c_begin + warp + i * WARPS) * kChunk;

        // ---- S^T = K . Q^T  (16 tokens x 8 heads per n-tile) ----
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            s[nt][0] = s[nt][2] = kbias[nt][0];
            s[nt][1] = s[nt][3] = kbias[nt][1];
        }
        {
            const int r = lane & 15;
            if constexpr (!Cfg::kInt8) {
#pragma unroll
                for (int kk = 0; kk < Cfg::kDT; ++kk) {
                    const int u = 2 * kk + (lane >> 4);
                    uint32_t a0, a1, a2, a3;
                    ptx::ldmatrix_x4(sK + r * Cfg::kRowBytes + ((u ^ (r & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma16816<QT>(s[nt], a0, a1, a2, a3, qf[nt][kk][0], qf[nt][kk][1]);
                }
            } else {
#pragma unroll
                for (int U = 0; U < Cfg::kUnits; U += 2) {
                    const int u = U + (lane >> 4);
                    uint32_t w0, w1, w2, w3;
                    ptx::ldmatrix_x4(sK + r * Cfg::kRowBytes + ((u ^ (r & 7)) << 4), w0, w1, w2, w3);
                    w0 ^= 0x80808080u; w1 ^= 0x80808080u; w2 ^= 0x80808080u; w3 ^= 0x80808080u;
                    // w0: rows 0-7 unit U, w1: rows 8-15 unit U, w2/w3: unit U+1
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma16816<MT>(s[nt], s8pair_biased(w0, 0, 1), s8pair_biased(w1, 0, 1), s8pair_biased(w0, 2, 3),
                                     s8pair_biased(w1, 2, 3), qf[nt][U][0], qf[nt][U][1]);
                        mma16816<MT>(s[nt], s8pair_biased(w2, 0, 1), s8pair_biased(w3, 0, 1), s8pair_biased(w2, 2, 3),
                                     s8pair_biased(w3, 2, 3), qf[nt][U + 1][0], qf[nt][U + 1][1]);
                    }
                }
            }
        }

        // ---- online softmax over this chunk (base 2) ----
        float ks_a = 1.f, ks_b = 1.f, vs_a = 1.f, vs_b = 1.f;
        if constexpr (Cfg::kInt8) {
            // Scales were copied as the aligned 4-byte word holding them; the
            // half is the parity of the element index (slot * Hkv + kvh).  With
            // page_size a multiple of 16 that parity is kvh's for even Hkv and
            // (row + kvh)'s for odd Hkv.
            const uint8_t* sS = ring + use_slot * Cfg::kStage + 2 * Cfg::kTile;
            auto scale_at = [&](int base, int row) {
                const uint32_t w = *reinterpret_cast<const uint32_t*>(sS + base + row * 4);
                const int odd = ((Hkv & 1) ? (row + kvh) : kvh) & 1;
                return __half2float(__ushort_as_half(static_cast<unsigned short>(odd ? (w >> 16) : (w & 0xffffu))));
            };
            ks_a = scale_at(0, g); ks_b = scale_at(0, g + 8);
            vs_a = scale_at(64, g); vs_b = scale_at(64, g + 8);
        }
        const bool va = tok0 + g < ctx && tok0 + g >= k_lo, vb = tok0 + g + 8 < ctx && tok0 + g + 8 >= k_lo;
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float x[4];
            x[0] = va ? s[nt][0] * (p.scale_log2 * ks_a * qinv[nt][0]) : -INFINITY;
            x[1] = va ? s[nt][1] * (p.scale_log2 * ks_a * qinv[nt][1]) : -INFINITY;
            x[2] = vb ? s[nt][2] * (p.scale_log2 * ks_b * qinv[nt][0]) : -INFINITY;
            x[3] = vb ? s[nt][3] * (p.scale_log2 * ks_b * qinv[nt][1]) : -INFINITY;
            float pr[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float mx = fmaxf(x[h], x[2 + h]);
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
                // m is a reference max: the accumulator is rescaled only when the chunk's
                // max exceeds it by more than kRescale (finite: every chunk holds an
                // attended token; the first chunk always rescales from -inf)
                if (mx > m[nt][h] + Cfg::kRescale) {
                    const float corr = ptx::ex2(m[nt][h] - mx);
                    m[nt][h] = mx;
                    l[nt][h] *= corr;
#pragma unroll
                    for (int dt = 0; dt < Cfg::kDT; ++dt) {
                        o[nt][dt][h] *= corr;
                        o[nt][dt][2 + h] *= corr;
                    }
                    if constexpr (Cfg::kInt8) {
                        osum[nt][h] *= corr;
                        osum[nt][2 + h] *= corr;
                    }
                }
                pr[h] = ptx::ex2(x[h] - m[nt][h]);
                pr[2 + h] = ptx::ex2(x[2 + h] - m[nt][h]);
                l[nt][h] += pr[h] + pr[2 + h];
            }
            // P^T fragments (B operand of O^T += V^T . P^T) via 8x8 transposes
            pb[nt][0] = ptx::movmatrix_trans(pack2<MT>(pr[0] * vs_a, pr[1] * vs_a));
            pb[nt][1] = ptx::movmatrix_trans(pack2<MT>(pr[2] * vs_b, pr[3] * vs_b));
        }

        // ---- O^T += V^T . P^T ----
        if constexpr (!Cfg::kInt8) {
            const int r = (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
            for (int dt = 0; dt < Cfg::kDT; ++dt) {
                const int u = 2 * dt + ((lane >> 3) & 1);
                uint32_t a0, a1, a2, a3;
                ptx::ldmatrix_x4_trans(sV + r * Cfg::kRowBytes + ((u ^ (r & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816<QT>(o[nt][dt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
        } else {
            const int r = (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int U = 0; U < Cfg::kUnits; U += 2) {
                const int u = U + (lane >> 4);
                uint32_t w0, w1, w2, w3;
                ptx::ldmatrix_x4_trans(sV + r * Cfg::kRowBytes + ((u ^ (r & 7)) << 4), w0, w1, w2, w3);
                w0 ^= 0x80808080u; w1 ^= 0x80808080u; w2 ^= 0x80808080u; w3 ^= 0x80808080u;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma16816<MT>(o[nt][U], s8pair_biased(w0, 0, 2), s8pair_biased(w0, 1, 3), s8pair_biased(w1, 0, 2),
                                 s8pair_biased(w1, 1, 3), pb[nt][0], pb[nt][1]);
                    mma16816<MT>(o[nt][U + 1], s8pair_biased(w2, 0, 2), s8pair_biased(w2, 1, 3),
                                 s8pair_biased(w3, 0, 2), s8pair_biased(w3, 1, 3), pb[nt][0], pb[nt][1]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                mma16816<MT>(osum[nt], kOnePair, kOnePair, kOnePair, kOnePair, pb[nt][0], pb[nt][1]);
        }
        __syncwarp();
        use_slot = use_slot + 1 == STAGES ? 0 : use_slot + 1;
    }
    ptx::cp_async_wait<0>();
    if constexpr (Cfg::kInt8) {
        // O accumulated (v + 1152) p: subtract 1152 sum_t p_t (rows of osum are all equal)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int dt = 0; dt < Cfg::kDT; ++dt)
#pragma unroll
                for (int i = 0; i < 4; ++i) o[nt][dt][i] -= kCodeBias * osum[nt][i & 1];
    }

    // ---- merge the warps' partial softmax states ----
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float x = l[nt][h];
            x += __shfl_xor_sync(kFull, x, 4);
            x += __shfl_xor_sync(kFull, x, 8);
            x += __shfl_xor_sync(kFull, x, 16);
            l[nt][h] = x;
        }
    __syncthreads();
    constexpr int NH = 8 * NT;
    float* sm_m = reinterpret_cast<float*>(smem);
    float* sm_l = sm_m + WARPS * NH;
    float* sm_o = sm_l + WARPS * NH;
    if (g == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                sm_m[warp * NH + nt * 8 + 2 * c + h] = m[nt][h];
                sm_l[warp * NH + nt * 8 + 2 * c + h] = l[nt][h];
            }
    }
    __syncthreads();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int n = nt * 8 + 2 * c + h;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < WARPS; ++w) M = fmaxf(M, sm_m[w * NH + n]);
            const float f = (m[nt][h] == -INFINITY) ? 0.f : ptx::ex2(m[nt][h] - M);
            float* dst = sm_o + (warp * NH + n) * HD;
#pragma unroll
            for (int dt = 0; dt < Cfg::kDT; ++dt) {
                const int d_lo = Cfg::kInt8 ? dt * 16 + 2 * g : dt * 16 + g;
                const int d_hi = Cfg::kInt8 ? d_lo + 1 : d_lo + 8;
                dst[d_lo] = o[nt][dt][h] * f;
                dst[d_hi] = o[nt][dt][2 + h] * f;
            }
        }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * HD; idx += WARPS * 32) {
        const int n = idx / HD, d = idx % HD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) M = fmaxf(M, sm_m[w * NH + n]);
        float L = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const float mw = sm_m[w * NH + n];
            L += (mw == -INFINITY) ? 0.f : sm_l[w * NH + n] * ptx::ex2(mw - M);
            acc += sm_o[(w * NH + n) * HD + d];
        }
        const float val = acc / L;
        if (nsplit == 1) {
            out[(head0 + n) * HD + d] = from_float<QT>(val);
        } else {
            const size_t row = (head0 + n) * p.max_splits + split;
            p.o_part[row * HD + d] = val;
            if (d == 0) p.lse_part[row] = M + __log2f(L);
        }
    }
}

// Merge of the split-KV partials: one CTA per (sequence, query head), its 8
// warps striding over the partitions (each warp reads whole 512-byte partial
// rows, four in flight), then a shared-memory sum across the warps.  Weights
// 2^(lse_p - max) against the global max of the partitions' log2-sum-exps.
constexpr int kCombineWarps = 8;

template <typename QT, int HD>
__global__ void __launch_bounds__(kCombineWarps * 32) decode_combine_kernel(const DecodeParams p) {
    __shared__ float sm_max[kCombineWarps];
    __shared__ float sm_w[kCombineWarps];
    __shared__ float sm_acc[kCombineWarps][HD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x;                                   // b * Hq + h
    const int b = gw / p.num_q_heads;
    const int ctx = __ldg(p.context_lens + b);
    if (ctx <= 0 || ctx > p.max_pages_per_seq * p.page_size) return;
    const int k_lo = (p.window > 0 && ctx > p.window) ? ctx - p.window : 0;
    const int ns = ceil_div(ceil_div(ctx, kChunk) - k_lo / kChunk, p.chunks_per_split);
    if (ns <= 1) return;
    const float* lse = p.lse_part + static_cast<size_t>(gw) * p.max_splits;
    const float* op = p.o_part + static_cast<size_t>(gw) * p.max_splits * HD;
    float M = -INFINITY;
    for (int s = threadIdx.x; s < ns; s += kCombineWarps * 32) M = fmaxf(M, lse[s]);
#pragma unroll
    for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
    if (lane == 0) sm_max[warp] = M;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) M = fmaxf(M, sm_max[w]);
    constexpr int E = HD / 32;
    float acc[E];
#pragma unroll
    for (int j = 0; j < E; ++j) acc[j] = 0.f;
    float wsum = 0.f;
#pragma unroll 4
    for (int s = warp; s < ns; s += kCombineWarps) {
        const float w = ptx::ex2(lse[s] - M);
        wsum += w;
        const float* src = op + static_cast<size_t>(s) * HD + lane * E;
        if constexpr (E == 4) {
            const float4 v = *reinterpret_cast<const float4*>(src);
            acc[0] += w * v.x; acc[1] += w * v.y; acc[2] += w * v.z; acc[3] += w * v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2*>(src);
            acc[0] += w * v.x; acc[1] += w * v.y;
        }
    }
#pragma unroll
    for (int j = 0; j < E; ++j) sm_acc[warp][lane * E + j] = acc[j];
    if (lane == 0) sm_w[warp] = wsum;
    __syncthreads();
    if (threadIdx.x < HD) {
        float a = 0.f, wt = 0.f;
#pragma unroll
        for (int w = 0; w < kCombineWarps; ++w) {
            a += sm_acc[w][threadIdx.x];
            wt += sm_w[w];
        }
        static_cast<QT*>(p.out)[static_cast<size_t>(gw) * HD + threadIdx.x] = from_float<QT>(a / wt);
    }
}

// fp32 pages and queries (small problems; CUDA-core path with exact-ish fp32
// arithmetic): one warp per query head, lanes across head_dim.
template <int HD>
__global__ void __launch_bounds__(128) decode_f32_kernel(const DecodeParams p) {
    const int kvh = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Hq = p.num_q_heads, Hkv = p.num_kv_heads, G = Hq / Hkv, ps = p.page_size;
    const int ctx = __ldg(p.context_lens + b);
    if (ctx < 0 || ctx > p.max_pages_per_seq * ps) {
        if (kvh == 0 && threadIdx.x == 0) record_error(p.status, PKV_ERR_DEVICE_RANGE, ctx);
        return;
    }
    constexpr int E = HD / 32;
    const float* q = static_cast<const float*>(p.q);
    const float* kp = static_cast<const float*>(p.k_pages);
    const float* vp = static_cast<const float*>(p.v_pages);
    float* out = static_cast<float*>(p.out);
    const int32_t* bt = p.block_tables + static_cast<size_t>(b) * p.max_pages_per_seq;
    for (int n = warp; n < G; n += 4) {
        const size_t h = static_cast<size_t>(b) * Hq + static_cast<size_t>(kvh) * G + n;
        float qv[E], acc[E];
#pragma unroll
        for (int j = 0; j < E; ++j) { qv[j] = q[h * HD + lane + 32 * j]; acc[j] = 0.f; }
        float mx = -INFINITY, l = 0.f;
        const int k_lo = (p.window > 0 && ctx > p.window) ? ctx - p.window : 0;
        for (int t = k_lo; t < ctx; ++t) {
            const int page = __ldg(bt + t / ps);
            if (page < 0 || page >= p.num_pages) {
                if (lane == 0) record_error(p.status, PKV_ERR_DEVICE_RANGE, page);
                continue;
            }
            const size_t row = ((static_cast<size_t>(page) * ps + t % ps) * Hkv + kvh) * HD;
            float dot = 0.f;
#pragma unroll
            for (int j = 0; j < E; ++j) dot = fmaf(qv[j], __ldg(kp + row + lane + 32 * j), dot);
#pragma unroll
            for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(kFull, dot, off);
            const float x = dot * p.scale_log2;
            const float m_new = fmaxf(mx, x);
            const float corr = exp2f(mx - m_new);
            const float pr = exp2f(x - m_new);
            l = l * corr + pr;
#pragma unroll
            for (int j = 0; j < E; ++j) acc[j] = fmaf(pr, __ldg(vp + row + lane + 32 * j), acc[j] * corr);
            mx = m_new;
        }
#pragma unroll
        for (int j = 0; j < E; ++j) out[h * HD + lane + 32 * j] = ctx > 0 ? acc[j] / l : 0.f;
    }
}

#ifndef PKV_DECODE_WARPS
#define PKV_DECODE_WARPS 4
#endif
constexpr int kWarps = PKV_DECODE_WARPS;    // warps per CTA, each with its own cp.async ring
// Ring depth (16-token chunks), measured per KV type: with 16-bit pages two stages
// (64 KB of ring per CTA) let three CTAs share an SM, which beats the deeper ring of
// two resident CTAs by 2-6% on the decode workloads; int8 pages (4 KB per stage, and
// register-limited to four CTAs per SM) run best with three.
template <typename KVT>
constexpr int stages_for() { return std::is_same<KVT, int8_t>::value ? 3 : 2; }

template <typename QT, typename KVT, int HD, int NT>
cudaError_t run_mma(const DecodeParams& p, cudaStream_t stream) {
    constexpr int kStages = stages_for<KVT>();
    using Cfg = DecodeCfg<QT, KVT, HD, NT, kWarps, kStages>;
    auto kern = decode_mma_kernel<QT, KVT, HD, NT, kWarps, kStages>;
    cudaError_t e0 = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), Cfg::kSmem);
    if (e0 != cudaSuccess) return e0;
    dim3 grid(p.num_kv_heads, p.max_splits, p.num_seqs);
    kern<<<grid, kWarps * 32, Cfg::kSmem, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || p.max_splits == 1) return e;
    decode_combine_kernel<QT, HD><<<p.num_seqs * p.num_q_heads, kCombineWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename QT, typename KVT, int HD>
cudaError_t run_nt(const DecodeParams& p, cudaStream_t stream) {
    const int G = p.num_q_heads / p.num_kv_heads;
    if (G <= 8) return run_mma<QT, KVT, HD, 1>(p, stream);
    return run_mma<QT, KVT, HD, 2>(p, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, pkv_dtype q_dtype, pkv_dtype kv_dtype,
                          cudaStream_t stream) {
    if (q_dtype == PKV_F32) {
        dim3 grid(p.num_kv_heads, p.num_seqs);
        if (p.head_dim == 128) decode_f32_kernel<128><<<grid, 128, 0, stream>>>(p);
        else decode_f32_kernel<64><<<grid, 128, 0, stream>>>(p);
        return cudaGetLastError();
    }
    const bool bf = q_dtype == PKV_BF16;
    if (kv_dtype == PKV_I8)
        return bf ? run_nt<__nv_bfloat16, int8_t, 128>(p, stream) : run_nt<__half, int8_t, 128>(p, stream);
    if (p.head_dim == 128)
        return bf ? run_nt<__nv_bfloat16, __nv_bfloat16, 128>(p, stream) : run_nt<__half, __half, 128>(p, stream);
    return bf ? run_nt<__nv_bfloat16, __nv_bfloat16, 64>(p, stream) : run_nt<__half, __half, 64>(p, stream);
}

}  // namespace pkv
