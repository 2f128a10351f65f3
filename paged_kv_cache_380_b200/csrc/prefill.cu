// Chunked-prefill attention over a paged KV cache on the 5th-generation tensor
// cores (tcgen05 + TMEM), operands staged by TMA.
//
// What is computed: query rows q_start[b] .. q_start[b+1]-1 of sequence b sit
// at absolute positions ctx-n .. ctx-1 (bottom-right alignment: the chunk
// follows the cached prefix); row r attends keys 0 .. ctx-n+r when causal,
// else all ctx keys; out = softmax(scale * q K^T) V.  FlashAttention-style
// tiling ("Flash Attention与Paged KV Cache优化大模型计算效率" §2.1: Q and K/V
// tiles staged on chip, 128x128 tiles; §4.1: prompt processing with
// FlashAttention) with the online softmax of "大模型推理优化实战：KV Cache +
// Flash Attention，让 Token 生成快 3 倍" ("Flash Attention 的分块计算原理"),
// K/V read page by page through the block table.
//
// B200 design, one CTA per (128-row query tile, query head, sequence), 12 warps:
//  * warps 0-2 = TMA producers: the Q tile once (two 64-column SW128 boxes), then
//    per 128-key tile one 16-row box per page group and 64-column half for K and
//    for V (lane pairs of the three warps split the 16 boxes of a tile), into
//    rings of 3 K stages and 2 V stages (mbarrier expect_tx).
//  * warp 3 = MMA issuer (one thread): S_j = Q K_j^T (M=128, N=128, K=128, bf16
//    -> fp32 in TMEM, three S/P buffers) and O += P_j V_j with P read from TMEM
//    (the TS form) and V as an MN-major operand.  S runs two tiles ahead of PV
//    (S_0 S_1 | PV_0 S_2 | PV_1 S_3 ...), so the softmax of tile i+1 never waits
//    for P_i.  One tcgen05.commit per MMA group (each commit costs tensor-pipe
//    time): "S_j done" also frees K stage j, "PV_i done" also frees P buffer i
//    and the V stage PV_i read.
//  * warps 4-11 = softmax: one TMEM lane (query row) per thread, two warps per
//    row quarter taking 64 columns each (row max and row sum exchanged in
//    shared memory); tcgen05.ld of the S half-row, masking, max, 2^(s*scale -
//    m) with the scale folded into one FFMA, row sum, P packed to bf16 pairs
//    and tcgen05.st back over the S columns; one P-ready arrival per warp.  The
//    accumulator is rescaled only when a row's running max grows by more than
//    2^8 (P <= 256 otherwise), which keeps O's TMEM round trip off most tiles;
//    the final division by the row sum makes any consistent reference max exact.
//  * Heaviest (longest causal) query tiles are launched first.
//  * Every mbarrier wait polls (test_wait) and is bounded in time; on time-out
//    the CTA records PKV_ERR_DEVICE_TIMEOUT, raises an abort flag so every role
//    leaves its loop, waits (bounded) for its own async work and frees TMEM.
#include <cuda.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "pkv_kernels.h"
#include "pkv_ptx.cuh"

namespace pkv {
namespace {

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int KST = 3, VST = 2, NSB = 3;        // K stages, V stages, S/P TMEM buffers
constexpr int kProducerWarps = 3;               // TMA issue is split over three warps
constexpr int kMmaWarp = kProducerWarps;
constexpr int kSoftmaxWarp0 = kMmaWarp + 1;
constexpr int kSoftmaxWarps = 8;                // two warps per TMEM lane quarter, 64 columns each
constexpr int kThreads = (kSoftmaxWarp0 + kSoftmaxWarps) * 32;   // 12 warps = 3 warpgroups
constexpr int kAtom = BN * 128;                 // one 64-column SW128 half of a 128-row tile
constexpr int kTile = 2 * kAtom;                // 32 KB
constexpr int kSmemQ = 0;
constexpr int kSmemK = kSmemQ + kTile;
constexpr int kSmemV = kSmemK + KST * kTile;
constexpr int kSmemRed = kSmemV + VST * kTile;   // row-max / row-sum exchange between warp pairs
constexpr int kRedBytes = (2 * 2 * BM + 2 * BM) * 4;
constexpr int kSmemBar = kSmemRed + kRedBytes;
constexpr int kNumBars = 1 + KST + VST + 3 * NSB + 1;
constexpr int kSmemBytes = kSmemBar + kNumBars * 8 + 16 + 1024;   // + TMEM addr, abort flag, alignment
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = NSB * 128;           // O accumulator columns 384..511
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bound of every mbarrier wait (1 s)
constexpr float kRescaleThreshold = 8.0f;       // log2 units: rescale when the max grows by > 2^8

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}

// sm_100 shared-memory matrix descriptor: start, leading and stride byte
// offsets (>> 4), version 1, SWIZZLE_128B layout.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: D fp32, A/B bf16 (fmt 1) or f16 (fmt 0),
// N and M as given, B K-major (0) or MN-major (1).
template <typename T>
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int b_mn_major) {
    constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | (static_cast<uint32_t>(b_mn_major) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// mbarrier addresses, all in one array after the tiles.  Every tcgen05.commit costs
// tensor-pipe time, so each MMA group signals exactly one barrier: s_done(b) =
// "S in buffer b is ready and K stage b is free" (K stages and S buffers share
// the ring index), pv_done(b) = "O is updated, P buffer b and the V stage that
// PV read are free".
struct Bars {
    uint32_t base;
    __device__ __forceinline__ uint32_t q_full() const { return base; }
    __device__ __forceinline__ uint32_t k_full(int i) const { return base + 8 * (1 + i); }
    __device__ __forceinline__ uint32_t v_full(int i) const { return base + 8 * (1 + KST + i); }
    __device__ __forceinline__ uint32_t s_done(int i) const { return base + 8 * (1 + KST + VST + i); }
    __device__ __forceinline__ uint32_t p_full(int i) const { return base + 8 * (1 + KST + VST + NSB + i); }
    __device__ __forceinline__ uint32_t pv_done(int i) const { return base + 8 * (1 + KST + VST + 2 * NSB + i); }
    __device__ __forceinline__ uint32_t mma_done() const { return base + 8 * (1 + KST + VST + 3 * NSB); }
};

// Bounded wait that also gives up as soon as another role raised the abort flag.
// It polls with the non-blocking test_wait: the pipeline is latency-bound, and a
// thread suspended inside try_wait resumes measurably later than a polling one
// (13% of the prefill time on a 128-row causal workload).  The bound is 1 s of
// %globaltimer, after which the CTA records PKV_ERR_DEVICE_TIMEOUT.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         DeviceStatus* st) {
    if (ptx::mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (;;) {
        if (ptx::mbar_test_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
    *abort_flag = 1;
    record_error(st, PKV_ERR_DEVICE_TIMEOUT, static_cast<long long>(bar));
    return false;
}

// One S tile: S[buffer SB] = Q K[stage SB]^T (K stages and S buffers share the index).
template <typename T, int SB>
__device__ __forceinline__ void mma_s(uint32_t sbase, const Bars& bars) {
    static_assert(KST == NSB, "K stage and S buffer share one ring index");
    constexpr uint32_t id_s = idesc_f16<T>(BM, BN, 0);
    const uint32_t kbase = sbase + kSmemK + SB * kTile;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
        ptx::tc_mma_ss(SB * 128, sdesc(sbase + kSmemQ + off, 16, 1024), sdesc(kbase + off, 16, 1024), id_s,
                       kk > 0 ? 1u : 0u);
    }
    ptx::tc_commit(bars.s_done(SB));
}
// One PV tile: O (+)= P[buffer PB] V[stage VS]; ACC = false only for the first tile.
template <typename T, int PB, int VS, bool ACC>
__device__ __forceinline__ void mma_pv(uint32_t sbase, const Bars& bars) {
    constexpr uint32_t id_o = idesc_f16<T>(BM, HD, 1);
    const uint32_t vbase = sbase + kSmemV + VS * kTile;
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk)
        ptx::tc_mma_ts(kOCol, PB * 128 + kk * 8, sdesc(vbase + kk * 2048, kAtom, 1024), id_o,
                       (ACC || kk > 0) ? 1u : 0u);
    ptx::tc_commit(bars.pv_done(PB));
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int num_qt = gridDim.z;
    const int qt = num_qt - 1 - static_cast<int>(blockIdx.z);   // heaviest tiles first
    const int h = blockIdx.x, b = blockIdx.y;
    const int Hq = p.num_q_heads, Hkv = p.num_kv_heads, kvh = h / (Hq / Hkv), ps = p.page_size;
    const int q0 = __ldg(p.q_start + b), n = __ldg(p.q_start + b + 1) - q0;
    const int ctx = __ldg(p.context_lens + b);
    const int r0 = qt * BM;
    if (r0 >= n) return;                                        // whole CTA, before any barrier
    if (n > ctx || ctx > p.max_pages_per_seq * ps || q0 < 0 || q0 + n > p.total_q) {
        if (threadIdx.x == 0) record_error(p.status, PKV_ERR_DEVICE_RANGE, ctx);
        return;
    }
    const int last_row = min(r0 + BM, n) - 1;
    const int max_key = p.causal ? ctx - n + last_row : ctx - 1;
    const int min_lim = p.causal ? ctx - n + r0 : ctx - 1;      // every row of the tile sees keys <= this
    // Local attention (window w > 0): a row at position pos sees keys pos-w+1 .. pos,
    // so the tile's key range starts at the first row's lower bound, and keys below
    // the last row's lower bound need the lower-edge mask.
    const int w = p.window;
    const int key_lo = w > 0 ? max(0, ctx - n + r0 - w + 1) : 0;
    const int lo_mask = w > 0 ? max(0, ctx - n + last_row - w + 1) : 0;
    const int t_first = key_lo / BN;
    const int n_tiles = max_key / BN + 1 - t_first;
    auto tile_of = [&](int j) { return t_first + j; };

    const Bars bars{sbase + kSmemBar};
    // Page indices, 4 tiles (32 groups of 16 keys) per batch: lane i of batch k holds the
    // physical page of group i%8 of tile 4k + i/8 (loaded by the producer warp only).
    const int32_t* bt = p.block_tables + static_cast<size_t>(b) * p.max_pages_per_seq;
    auto load_pages = [&](int k) -> int {
        const int key0 = tile_of(4 * k + (lane >> 3)) * BN + 16 * (lane & 7);
        return key0 < ctx ? __ldg(bt + key0 / ps) : -1;
    };
    int pg_cur = 0, pg_next = 0;
    if (warp < kProducerWarps) {
        pg_cur = load_pages(0);
        pg_next = load_pages(1);
    }
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmemBar + kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmemBar + kNumBars * 8 + 8);

    if (threadIdx.x == 0) {
        ptx::mbar_init(bars.q_full(), 1);
        for (int i = 0; i < KST; ++i) ptx::mbar_init(bars.k_full(i), kProducerWarps);
        for (int i = 0; i < VST; ++i) ptx::mbar_init(bars.v_full(i), kProducerWarps);
        for (int i = 0; i < NSB; ++i) {
            ptx::mbar_init(bars.s_done(i), 1);
            ptx::mbar_init(bars.p_full(i), kSoftmaxWarps);
            ptx::mbar_init(bars.pv_done(i), 1);
        }
        ptx::mbar_init(bars.mma_done(), 1);
        *abort_flag = 0;
        ptx::fence_mbarrier_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    // All 512 columns are allocated, so the allocation starts at lane 0, column 0
    // and the MMAs use constant TMEM addresses; anything else is reported.
    const uint32_t tmem = 0;
    if (threadIdx.x == 0 && *tmem_slot != 0u) {
        *abort_flag = 1;
        record_error(p.status, PKV_ERR_CUDA, static_cast<long long>(*tmem_slot));
    }

    if (warp < kProducerWarps) {
        // ------------------------------ TMA producers ------------------------------
        // A tile is 8 page groups x 2 column halves = 16 boxes per tensor; producer
        // warp w issues the boxes of groups w, w+3, w+6 (one box per lane), because a
        // single issuing warp cannot keep enough 2 KB boxes in flight.  K runs up to KST
        // tiles ahead; V is issued one tile behind K so that waiting for a free V
        // stage never delays the next K tile.  Page indices come from register
        // batches loaded four tiles ahead (pg_cur / pg_next).
        if (warp == 0 && lane == 0) {
            ptx::prefetch_tmap(&tm_q);
            ptx::prefetch_tmap(&tm_k);
            ptx::prefetch_tmap(&tm_v);
            ptx::mbar_arrive_expect_tx(bars.q_full(), kTile);
            ptx::tma_load_3d(sbase + kSmemQ, &tm_q, bars.q_full(), 0, h, q0 + r0);
            ptx::tma_load_3d(sbase + kSmemQ + kAtom, &tm_q, bars.q_full(), 64, h, q0 + r0);
        }
        const int my_group = warp + kProducerWarps * (lane >> 1);   // lane pair -> one page group
        const int my_half = lane & 1;
        const bool my_lane = my_group < 8;
        // TMA row (slot) of my page group in tile t, or -1 (past the context / bad page)
        auto row_of = [&](int t, int pg_word) -> int {
            const int page = __shfl_sync(0xffffffffu, pg_word, (t & 3) * 8 + (my_group & 7));
            const int key0 = tile_of(t) * BN + 16 * my_group;
            if (!my_lane || key0 >= ctx) return -1;
            if (page < 0 || page >= p.num_pages) {
                if (my_half == 0) record_error(p.status, PKV_ERR_DEVICE_RANGE, page);
                return -1;
            }
            return page * ps + key0 % ps;
        };
        auto issue = [&](bool is_k, int t, int row) -> bool {
            const int nst = is_k ? KST : VST, st = t % nst;
            const unsigned nbox = __popc(__ballot_sync(0xffffffffu, row >= 0));
            bool ok = true;
            // a K stage is free once S of the tile KST back is done, a V stage once
            // PV of the tile VST back is done
            if (t >= nst) {
                const int prev = t - nst;
                ok = wait_bar(is_k ? bars.s_done(prev % NSB) : bars.pv_done(prev % NSB), (prev / NSB) & 1,
                              abort_flag, p.status);
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) return false;
            const uint32_t bar = is_k ? bars.k_full(st) : bars.v_full(st);
            if (lane == 0) ptx::mbar_arrive_expect_tx(bar, nbox * 16 * 128);
            __syncwarp();
            if (row >= 0) {
                const uint32_t dst = sbase + (is_k ? kSmemK : kSmemV) + st * kTile + my_half * kAtom + my_group * 2048;
                ptx::tma_load_3d(dst, is_k ? &tm_k : &tm_v, bar, 64 * my_half, kvh, row);
            }
            return true;
        };
        int row_prev = -1;
        for (int t = 0; t <= n_tiles; ++t) {
            int row = -1;
            if (t < n_tiles) {
                if (t > 0 && (t & 3) == 0) {
                    pg_cur = pg_next;
                    pg_next = load_pages(t / 4 + 1);
                }
                row = row_of(t, pg_cur);
                if (!issue(true, t, row)) break;
            }
            if (t >= 1 && !issue(false, t - 1, row_prev)) break;
            row_prev = row;
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------ MMA issuer ------------------------------
        // S runs two tiles ahead of PV (S_0 S_1 | PV_0 S_2 | PV_1 S_3 | ...), so the
        // softmax of tile i+1 never waits for P_i.  The ring slots are template
        // arguments of the issue helpers and the TMEM base is 0, so every MMA
        // operand is a constant.
        if (lane == 0) {
            bool ok = wait_bar(bars.q_full(), 0, abort_flag, p.status);
            auto issue_s = [&](int j) {
                if (!wait_bar(bars.k_full(j % KST), (j / KST) & 1, abort_flag, p.status)) return false;
                if (j >= NSB && !wait_bar(bars.pv_done(j % NSB), ((j / NSB) - 1) & 1, abort_flag, p.status))
                    return false;
                ptx::tc_fence_after();
                switch (j % 3) {
                    case 0: mma_s<T, 0>(sbase, bars); break;
                    case 1: mma_s<T, 1>(sbase, bars); break;
                    default: mma_s<T, 2>(sbase, bars); break;
                }
                return true;
            };
            auto issue_pv = [&](int i) {
                if (!wait_bar(bars.p_full(i % NSB), (i / NSB) & 1, abort_flag, p.status)) return false;
                if (!wait_bar(bars.v_full(i % VST), (i / VST) & 1, abort_flag, p.status)) return false;
                ptx::tc_fence_after();
                switch (i == 0 ? -1 : i % 6) {
                    case -1: mma_pv<T, 0, 0, false>(sbase, bars); break;
                    case 0: mma_pv<T, 0, 0, true>(sbase, bars); break;
                    case 1: mma_pv<T, 1, 1, true>(sbase, bars); break;
                    case 2: mma_pv<T, 2, 0, true>(sbase, bars); break;
                    case 3: mma_pv<T, 0, 1, true>(sbase, bars); break;
                    case 4: mma_pv<T, 1, 0, true>(sbase, bars); break;
                    default: mma_pv<T, 2, 1, true>(sbase, bars); break;
                }
                return true;
            };
            ok = ok && issue_s(0) && (n_tiles < 2 || issue_s(1));
            for (int i = 0; i < n_tiles && ok; ++i) {
                ok = issue_pv(i);
                if (ok && i + 2 < n_tiles) ok = issue_s(i + 2);
            }
            // drain: every tcgen05 op issued by this thread completes before TMEM is freed
            ptx::tc_commit(bars.mma_done());
            ptx::mbar_wait(bars.mma_done(), 0, kSpinLimit);
        }
    } else {
        // ------------------------------ softmax + epilogue ------------------------------
        // Warp w reaches TMEM lanes 32*(w%4)..+31 (its quarter of the rows); the two
        // warps of a quarter split the 128 columns of S (and of O) into halves and
        // exchange row maxima (and finally row sums) through shared memory.
        const int quarter = warp & 3, hf = (warp - kSoftmaxWarp0) >> 2;
        const int row = quarter * 32 + lane;                        // TMEM lane == tile row
        const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
        const int c0 = hf * 64;                                     // this warp's S / O columns
        float* red = reinterpret_cast<float*>(smem + kSmemRed);     // [2 bufs][2 halves][BM]
        float* lsum = red + 2 * 2 * BM;                             // [2 halves][BM]
        const int lim = min(p.causal ? ctx - n + r0 + row : ctx - 1, ctx - 1);
        const int row_lo = w > 0 ? max(0, ctx - n + r0 + row - w + 1) : 0;     // this row's first key
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int bj = j % NSB;
            ok = wait_bar(bars.s_done(bj), (j / NSB) & 1, abort_flag, p.status);
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t r[64];
            {
                uint32_t (&r0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
                uint32_t (&r1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
                ptx::tmem_ld32(trow + bj * 128 + c0, r0);
                ptx::tmem_ld32(trow + bj * 128 + c0 + 32, r1);
            }
            ptx::tc_wait_ld();
            float x[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(r[c]);
            const int jt = tile_of(j);
            if (jt * BN + BN - 1 > min_lim || jt * BN < lo_mask) {  // diagonal / last / window edge
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const int key = jt * BN + c0 + c;
                    if (key > lim || key < row_lo) x[c] = -INFINITY;
                }
            }
            float mh = x[0];
#pragma unroll
            for (int c = 1; c < 64; ++c) mh = fmaxf(mh, x[c]);
            float* rb = red + (j & 1) * 2 * BM;
            rb[hf * BM + row] = mh;
            named_bar_sync(1 + quarter, 64);
            // -inf only for a row that sees no key of this tile (possible with a window)
            const float mt = fmaxf(mh, rb[(1 - hf) * BM + row]) * sl2;
            if (j == 0) {
                m_ref = mt;
            } else if (__any_sync(0xffffffffu, mt > m_ref + kRescaleThreshold)) {
                const float m_new = fmaxf(m_ref, mt);
                const float corr = ptx::ex2(m_ref - m_new);
                l *= corr;
                m_ref = m_new;
                const int pj = j - 1;
                ok = wait_bar(bars.pv_done(pj % NSB), (pj / NSB) & 1, abort_flag, p.status);
                if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                ptx::tc_fence_after();
#pragma unroll
                for (int c32 = 0; c32 < 2; ++c32) {
                    uint32_t o[32];
                    ptx::tmem_ld32(trow + kOCol + c0 + c32 * 32, o);
                    ptx::tc_wait_ld();
                    uint32_t w0[16], w1[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        w0[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
                        w1[i] = __float_as_uint(__uint_as_float(o[16 + i]) * corr);
                    }
                    ptx::tmem_st16(trow + kOCol + c0 + c32 * 32, w0);
                    ptx::tmem_st16(trow + kOCol + c0 + c32 * 32 + 16, w1);
                }
                ptx::tc_wait_st();
            }
            const float neg = m_ref == -INFINITY ? 0.f : -m_ref;      // no key seen yet: all p are 0
            float rs = 0.f;
#pragma unroll
            for (int c16 = 0; c16 < 2; ++c16) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int c = c16 * 32 + 2 * i;
                    const float ya = fmaf(x[c], sl2, neg), yb = fmaf(x[c + 1], sl2, neg);
                    const float a = ptx::ex2(ya), bb = ptx::ex2(yb);
                    rs += a + bb;
                    pk[i] = pack2<T>(a, bb);
                }
                ptx::tmem_st16(trow + bj * 128 + hf * 32 + c16 * 16, pk);
            }
            l += rs;
            ptx::tc_wait_st();
            if (ctx < (jt + 1) * BN) {
                // V rows past the context (tail of the last page, or never loaded) must be
                // finite zeros: P is 0 there but 0 * NaN would poison O.
                const int vs = j % VST;
                ok = wait_bar(bars.v_full(vs), (j / VST) & 1, abort_flag, p.status);
                if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
                const int first = ctx - jt * BN;                    // first invalid row of the tile
                uint4* vt = reinterpret_cast<uint4*>(smem + kSmemV + vs * kTile);
                const int tid = threadIdx.x - kSoftmaxWarp0 * 32;
                for (int idx = tid; idx < 2 * (BN - first) * 8; idx += kSoftmaxWarps * 32) {
                    const int half = idx / ((BN - first) * 8), rem = idx % ((BN - first) * 8);
                    vt[(half * kAtom + (first + rem / 8) * 128) / 16 + rem % 8] = make_uint4(0, 0, 0, 0);
                }
                ptx::fence_proxy_async_smem();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bars.p_full(bj));      // one arrival per warp
        }
        // epilogue: O / l -> out (each warp writes its 64 output columns)
        if (ok) {
            const int pj = n_tiles - 1;
            ok = wait_bar(bars.pv_done(pj % NSB), (pj / NSB) & 1, abort_flag, p.status);
        }
        lsum[hf * BM + row] = l;
        named_bar_sync(1 + quarter, 64);
        if (__all_sync(0xffffffffu, ok)) {
            ptx::tc_fence_after();
            const float inv = 1.f / (l + lsum[(1 - hf) * BM + row]);
            const bool store = r0 + row < n;
            T* out = static_cast<T*>(p.out) + (static_cast<size_t>(q0 + r0 + row) * Hq + h) * HD + c0;
#pragma unroll
            for (int c32 = 0; c32 < 2; ++c32) {
                uint32_t o[32];
                ptx::tmem_ld32(trow + kOCol + c0 + c32 * 32, o);
                ptx::tc_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack2<T>(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
                if (store) {
                    uint4* dst = reinterpret_cast<uint4*>(out + c32 * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0 && lane == 0 && *abort_flag) {
        // let in-flight TMA writes land before the shared memory is handed to another CTA
        for (int t = 0; t < KST; ++t) ptx::mbar_wait(bars.k_full(t), 0, kSpinLimit >> 4);
    }
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(*tmem_slot, kTmemCols);
    }
}

// ---- host: tensor maps through the driver entry point -------------------------

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
    static EncodeTiled fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiled>(nullptr);
        return reinterpret_cast<EncodeTiled>(f);
    }();
    return fn;
}

// 3-D map over a [rows][heads][128] tensor of 16-bit elements, box {64, 1, box_rows}, SW128.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t heads, uint64_t rows,
              uint32_t box_rows) {
    EncodeTiled enc = encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {HD, heads, rows};
    const cuuint64_t strides[2] = {HD * 2, heads * HD * 2};
    const cuuint32_t box[3] = {64, 1, box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
cudaError_t run(const PrefillParams& p, cudaStream_t stream) {
    const CUtensorMapDataType dt =
        std::is_same<T, __nv_bfloat16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tq, tk, tv;
    const uint64_t pool_rows = static_cast<uint64_t>(p.num_pages) * p.page_size;
    if (!make_map(&tq, p.q, dt, p.num_q_heads, p.total_q, BM) ||
        !make_map(&tk, p.k_pages, dt, p.num_kv_heads, pool_rows, 16) ||
        !make_map(&tv, p.v_pages, dt, p.num_kv_heads, pool_rows, 16))
        return cudaErrorInvalidValue;
    dim3 grid(p.num_q_heads, p.num_seqs, ceil_div(p.max_q_len, BM));
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(prefill_tc_kernel<T>), kSmemBytes);
    if (e != cudaSuccess) return e;
    prefill_tc_kernel<T><<<grid, kThreads, kSmemBytes, stream>>>(p, tq, tk, tv);
    return cudaGetLastError();
}

}  // namespace

namespace {
// One thread waits, with the prefill kernel's own bounded wait, on an mbarrier
// that nothing ever arrives on: after kWaitLimitNs it records
// PKV_ERR_DEVICE_TIMEOUT and the kernel returns.  Exercises the time-out path
// without any fault or hang.
__global__ void wait_timeout_selftest_kernel(DeviceStatus* st) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_u32(&bar), 1);
        abort_flag = 0;
        ptx::fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) wait_bar(ptx::smem_u32(&bar), 0, &abort_flag, st);
}
}  // namespace

cudaError_t launch_wait_timeout_selftest(DeviceStatus* st, cudaStream_t stream) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(st);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillParams& p, pkv_dtype dtype, cudaStream_t stream) {
    if (p.max_q_len <= 0 || p.num_seqs <= 0 || p.total_q <= 0) return cudaSuccess;
    return dtype == PKV_BF16 ? run<__nv_bfloat16>(p, stream) : run<__half>(p, stream);
}

}  // namespace pkv
