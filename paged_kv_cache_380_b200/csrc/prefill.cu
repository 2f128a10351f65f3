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
// B200 design.  A persistent kernel: one CTA of 12 warps per SM walks work units
// (128-row query tile, pair of query heads, sequence), heaviest first.  The two
// query heads of a pair read the same KV head (grouped-query attention,
// "LLM推理系统优化：KV缓存管理与动态批处理技术" §2.1), so they share the causal
// mask, the key range and every K/V tile: each tile is loaded once and feeds two
// S tiles and two PV tiles.  The two query tiles ("A" and "B") form a ping-pong:
// while the softmax of one runs on the CUDA cores, the tensor pipe works on the
// other.  The rings, barrier phases and key-tile count run on across units.
//  * TMEM (512 columns): S_A | S_B | O_A | O_B, 128 columns each.  P (bf16)
//    overwrites the first half of its own S tile.
//  * warp 0 = K producer, warp 1 = V producer: per 128-key tile, one 16-row TMA
//    box per page group and 64-column half (one box per lane), into rings of 3
//    K stages and 2 V stages; one barrier per load step carries K tile t and V
//    tile t-1.  Warp 0 also loads each unit's two Q tiles.
//  * warp 2 = MMA issuer (one thread), per key tile j:
//        PV_A(j)  S_A(j+1)  PV_B(j)  S_B(j+1)
//    S = Q K^T (M=128, N=128, both operands K-major in shared memory), PV = P V
//    with P read from TMEM (the TS form) and V as an MN-major operand.  Issuing
//    S_X(j+1) right behind PV_X(j) is what lets P alias S: tcgen05 MMAs of one
//    thread execute in issue order.  Each commit signals one barrier: "S_B(j)
//    done" also frees K stage j, "PV_B(j) done" also frees V stage j.
//  * warps 4-7 = softmax of tile A, warps 8-11 = softmax of tile B: one TMEM
//    lane (query row) per thread, all 128 columns of its row.  tcgen05.ld of
//    the S row, masking, row max, 2^(s*scale - m) with the scale folded into one
//    FFMA, row sum, P packed to bf16 pairs and tcgen05.st over the S columns;
//    one arrival per warp when the first 64 keys' P is stored (P.V over them
//    starts while the other 64 are computed) and one when all of P is.  The accumulator is rescaled only when a
//    row's running max grows by more than 2^8 (P <= 256 otherwise); the final
//    division by the row sum makes any consistent reference max exact.  The same
//    warps write a unit's output after the next unit's first key tile.
//  * Heads of a group that cannot be paired (an odd group size) run one tile
//    per unit through the same code (NT = 1).
//  * Every mbarrier wait is bounded in time (a waiting thread suspends in
//    try_wait); on time-out the CTA records PKV_ERR_DEVICE_TIMEOUT, raises an
//    abort flag so every role leaves its loop, waits (bounded) for its own async
//    work and frees TMEM.
#include <cuda.h>

#include <cmath>
#include <cstring>
#include <type_traits>

#include "pkv_kernels.h"
#include "pkv_ptx.cuh"

namespace pkv {
namespace {

constexpr int BM = 128, BN = 128;               // query rows / keys per tile
constexpr int KST = 3, VST = 2;                 // K stages, V stages
constexpr int kKWarp = 0, kVWarp = 1, kMmaWarp = 2, kSoftWarp0 = 4;
constexpr int kThreads = 12 * 32;               // 3 warpgroups
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 256;                 // O of tile X at 256 + 128 X; S/P of tile X at 128 X
constexpr int kAtom = BM * 128;                 // one 64-column SW128 atom of a 128-row tile (16 KB)
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // bound of every mbarrier wait (1 s)
constexpr float kRescaleThreshold = 8.0f;       // log2 units: rescale when the max grows by > 2^8

// Shared-memory layout of the CTA for head_dim HD and NT query tiles.
template <int HD, int NT>
struct Layout {
    static constexpr int NH = HD / 64;          // 64-column atoms per row
    static constexpr int kTile = NH * kAtom;    // one 128-row tile of HD columns
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + NT * kTile;
    static constexpr int kV = kK + KST * kTile;
    static constexpr int kBar = kV + VST * kTile;
    static constexpr int kNumBars = 25;
    static constexpr int kPend = kBar + kNumBars * 8 + 16;  // after the TMEM address and abort flag
    static constexpr int kEnd = kPend + 8 * 32;             // a pending epilogue's unit, per softmax warp
    // The CTA holds all of TMEM, so only one may run per SM: ask for more than
    // half of the SM's shared memory even when the tiles need less.
    static constexpr int kSmem = kEnd + 1024 > 120 * 1024 ? kEnd + 1024 : 120 * 1024;
};

// mbarriers, all in one array after the tiles.
struct Bars {
    uint32_t base;
    __device__ __forceinline__ uint32_t at(int i) const { return base + 8 * i; }
    __device__ __forceinline__ uint32_t q_full() const { return at(0); }
    // load step t (slot t % KST): K tile t and V tile t-1 landed (one arrival from each producer warp)
    __device__ __forceinline__ uint32_t kv_full(int s) const { return at(1 + s); }
    // S_X(j) done (and, for the last tile, K stage s free), one barrier per K stage
    __device__ __forceinline__ uint32_t s_full(int x, int s) const { return at(1 + KST + VST + x * KST + s); }
    __device__ __forceinline__ uint32_t p_full(int x) const { return at(1 + 3 * KST + VST + x); }
    // PV of the last tile done: V stage s free
    __device__ __forceinline__ uint32_t pv_done(int s) const { return at(3 + 3 * KST + VST + s); }
    __device__ __forceinline__ uint32_t o_full(int x) const { return at(3 + 3 * KST + 2 * VST + x); }
    __device__ __forceinline__ uint32_t mma_done() const { return at(5 + 3 * KST + 2 * VST); }
    // a unit's O has been read by its epilogue (the next unit's first P.V may overwrite it),
    // and the unit's epilogue staging area is drained (the V producer may refill it); both
    // alternate by unit parity so that a waiter one unit behind is never two phases late
    __device__ __forceinline__ uint32_t o_read(int uc) const { return at(6 + 3 * KST + 2 * VST + (uc & 1)); }
    __device__ __forceinline__ uint32_t stage_free(int uc) const { return at(8 + 3 * KST + 2 * VST + (uc & 1)); }
    // P of tile x's first 64 keys is in place (P.V over them may start); phase per key tile
    __device__ __forceinline__ uint32_t p_half(int x) const { return at(10 + 3 * KST + 2 * VST + x); }
};
static_assert(10 + 3 * KST + 2 * VST + 2 == 25, "barrier count");

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

// Each thread of the warp writes 32 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Orders the uses of registers written by a tcgen05.ld after the tcgen05.wait::ld
// that precedes this call (the compiler sees the registers as rewritten here).
__device__ __forceinline__ void reg_fence32(uint32_t* r) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

// 64 consecutive fp32 columns of this thread's TMEM lane into v (waits for the load).
__device__ __forceinline__ void load_half(uint32_t taddr, float (&v)[64]) {
    uint32_t r[64];
    ptx::tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    ptx::tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
    ptx::tc_wait_ld();
    reg_fence32(&r[0]);
    reg_fence32(&r[32]);
#pragma unroll
    for (int c = 0; c < 64; ++c) v[c] = __uint_as_float(r[c]);
}
// Scores of keys outside lo .. lim (key of column c is key0 + c) become -inf; without a
// window only the upper bound can cut (one compare per element).
__device__ __forceinline__ void mask_half(float (&v)[64], int key0, int lim, int lo, bool window) {
    const int hi = lim - key0, lw = lo - key0;
    if (!window) {
#pragma unroll
        for (int c = 0; c < 64; ++c) v[c] = c > hi ? -INFINITY : v[c];
    } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) v[c] = (c > hi || c < lw) ? -INFINITY : v[c];
    }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Two lanes of packed fp32 arithmetic (one instruction for both).
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^y for the two lanes of y in fp32 on the SFU (which evaluates 4 exponentials per
// clock per sub-partition whatever their width, so a packed bf16 form saves no SFU
// time), both added to sum; returns the pair rounded to T and packed (low half =
// first lane).
template <typename T>
__device__ __forceinline__ uint32_t exp2_pair(uint64_t y, uint64_t& sum) {
    float y0, y1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(y));
    const float e0 = ptx::ex2(y0), e1 = ptx::ex2(y1);
    sum = fadd2(sum, f2pack(e0, e1));
    return pack2<T>(e0, e1);
}

#ifndef PKV_PREFILL_MMA_SLEEP
#define PKV_PREFILL_MMA_SLEEP 1
#endif

// Bounded wait that also gives up as soon as another role raised the abort flag.
// kSleep: the thread waits inside try_wait, suspended until the phase completes
// (or a hardware time slice ends), so a waiting warp takes no issue slots from
// the working warps of its sub-partition.  Otherwise it polls with the
// non-blocking test_wait.  The bound is 1 s of %globaltimer, after which the CTA
// records PKV_ERR_DEVICE_TIMEOUT.
template <bool kSleep = true>
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         DeviceStatus* st) {
    auto probe = [&] { return kSleep ? ptx::mbar_try_wait(bar, parity) : ptx::mbar_test_wait(bar, parity); };
    if (probe()) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (;;) {
        if (probe()) return true;
        if (*abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
    *abort_flag = 1;
    record_error(st, PKV_ERR_DEVICE_TIMEOUT, static_cast<long long>(bar));
    return false;
}

// Every lane of the warp waits (measured faster than one polling lane and a
// broadcast); the result is made warp-uniform.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int lane, volatile int* abort_flag,
                                          DeviceStatus* st) {
    (void)lane;
    const bool ok = wait_bar(bar, parity, abort_flag, st);
    return __all_sync(0xffffffffu, ok);
}

// One work unit: a 128-row query tile of NT query heads (h0 ..) of sequence b.
// Units are numbered with the query-tile index varying slowest and reversed, so
// that lower numbers are the longer (later, more keys) tiles.
struct Unit {
    int h0, b, kvh, q0, n, ctx, r0;
    int t_first, n_tiles;            // 128-key tiles t_first .. t_first + n_tiles - 1
    int min_lim, lo_mask;            // masking bounds shared by the tile's rows
    bool valid;
};

// The three per-sequence values a unit needs, loaded one unit ahead of their use
// so that each role's walk over its units never waits on them.
struct UnitLoad {
    int q0, q1, ctx;
};
// A read-only global load kept where it is written (volatile): issued a unit ahead, its
// latency is hidden behind the current unit instead of being moved next to its use.
__device__ __forceinline__ int ld_early(const int* ptr) {
    int v;
    asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(v) : "l"(ptr));
    return v;
}
template <int NT>
__device__ __forceinline__ UnitLoad unit_load(const PrefillParams& p, int u, int num_units) {
    if (u >= num_units) return UnitLoad{0, 0, 0};
    const int b = (u / (p.num_q_heads / NT)) % p.num_seqs;
    return UnitLoad{ld_early(p.q_start + b), ld_early(p.q_start + b + 1), ld_early(p.context_lens + b)};
}

template <int NT>
__device__ __forceinline__ Unit unit_of(const PrefillParams& p, int u, int num_qt, const UnitLoad& ld, bool report) {
    Unit w{};
    const int hp_count = p.num_q_heads / NT;
    const int hp = u % hp_count, rest = u / hp_count;
    w.b = rest % p.num_seqs;
    const int qt = num_qt - 1 - rest / p.num_seqs;
    w.h0 = hp * NT;
    w.kvh = w.h0 / (p.num_q_heads / p.num_kv_heads);
    w.q0 = ld.q0;
    w.n = ld.q1 - ld.q0;
    w.ctx = ld.ctx;
    w.r0 = qt * BM;
    w.valid = false;
    if (w.r0 >= w.n) return w;
    if (w.n > w.ctx || w.ctx > p.max_pages_per_seq * p.page_size || w.q0 < 0 || w.q0 + w.n > p.total_q) {
        if (report) record_error(p.status, PKV_ERR_DEVICE_RANGE, w.ctx);
        return w;
    }
    const int last_row = min(w.r0 + BM, w.n) - 1;
    const int max_key = p.causal ? w.ctx - w.n + last_row : w.ctx - 1;
    w.min_lim = p.causal ? w.ctx - w.n + w.r0 : w.ctx - 1;   // every row of the tile sees keys <= this
    // Local attention (window ww > 0): a row at position pos sees keys pos-ww+1 .. pos
    // (pos-ww+1 .. ctx-1 without the causal mask), so the tile's key range starts at
    // the first row's lower bound, and keys below the last row's lower bound need
    // the lower-edge mask.
    const int ww = p.window;
    const int key_lo = ww > 0 ? max(0, w.ctx - w.n + w.r0 - ww + 1) : 0;
    w.lo_mask = ww > 0 ? max(0, w.ctx - w.n + last_row - ww + 1) : 0;
    w.t_first = key_lo / BN;
    w.n_tiles = max_key / BN + 1 - w.t_first;
    w.valid = true;
    return w;
}

// The MMA issuer.  One code path serves every ring slot: a slot only moves the
// shared-memory start address, i.e. adds a constant to the low word of the
// descriptor (the address field holds addr >> 4 in 14 bits, and shared memory
// ends below 256 KB, so the sum never carries out of it).  One compact loop keeps
// the issuing thread's instruction stream small.
template <typename T, int HD, int NT>
struct Issuer {
    using L = Layout<HD, NT>;
    uint64_t dq[NT];                 // Q of each tile
    uint64_t dk, dv;                 // K and V stage 0
    Bars bars;
    volatile int* abort_flag;
    DeviceStatus* status;

    __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
        return wait_bar<PKV_PREFILL_MMA_SLEEP != 0>(bar, parity, abort_flag, status);
    }
    // S_x = Q_x K[stage ks]^T, then one commit: "S_x done" (+ K stage free for the last tile).
    __device__ __forceinline__ void s(int x, int ks) const {
        constexpr uint32_t id = idesc_f16<T>(BM, BN, 0);
        const uint64_t a = dq[x], b = dk + static_cast<uint64_t>((ks * L::kTile) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kAtom + (kk & 3) * 32) >> 4);
            ptx::tc_mma_ss(static_cast<uint32_t>(x * 128), a + off, b + off, id, kk > 0 ? 1u : 0u);
        }
        ptx::tc_commit(bars.s_full(x, ks));
    }
    // O_x (+)= P_x V[stage vs] over keys 64 h .. 64 h + 63; the first key tile of a unit
    // overwrites O.
    __device__ __forceinline__ void pv(int x, int vs, bool acc, int h) const {
        constexpr uint32_t id = idesc_f16<T>(BM, HD, 1);
        const uint64_t b = dv + static_cast<uint64_t>((vs * L::kTile) >> 4);
#pragma unroll
        for (int k = 0; k < BN / 32; ++k) {
            const int kk = h * (BN / 32) + k;
            ptx::tc_mma_ts(kOCol + x * 128, static_cast<uint32_t>(x * 128 + kk * 8), b + static_cast<uint64_t>((kk * 2048) >> 4),
                           id, (acc || kk > 0) ? 1u : 0u);
        }
    }
    // One unit of n key tiles, global tiles g0 .. g0+n-1: S_A(0) [S_B(0)], then per key
    // tile j: PV_A(j) S_A(j+1) [PV_B(j) S_B(j+1)], each PV in two halves of 64 keys released
    // by their own barrier.  Five barrier probes per key tile (the K/V step, then each
    // half of P_A and of P_B): each probe costs the tensor pipe about as much as two MMAs
    // when nothing is queued behind it.
    // uc = units this CTA has issued before (the Q, O-ready and O-read barriers' phase).
    __device__ bool unit(int g0, int n, int uc) const {
        if (!wait(bars.q_full(), uc & 1)) return false;
        if (g0 == 0 && !wait(bars.kv_full(0), 0)) return false;   // later units: waited by the last step
        ptx::tc_fence_after();
        for (int x = 0; x < NT; ++x) s(x, g0 % KST);
        for (int j = 0; j < n; ++j) {
            const int g = g0 + j, vs = g % VST, ks1 = (g + 1) % KST;
            const bool more = j + 1 < n;
            // load step g+1 holds V tile g (for PV) and K tile g+1 (for the next S).  It is
            // probed first: it has normally landed long before, and the tensor pipe idles from
            // P_A ready until the first P.V is issued, so nothing but that wait sits there.
            if (!wait(bars.kv_full(ks1), ((g + 1) / KST) & 1)) return false;
            // the unit's first P.V overwrites O: the previous unit's epilogue must have read it
            if (j == 0 && uc > 0 && !wait(bars.o_read(uc - 1), ((uc - 1) >> 1) & 1)) return false;
            // P.V over a tile's first 64 keys starts while its softmax finishes the other 64
            if (!wait(bars.p_half(0), g & 1)) return false;
            ptx::tc_fence_after();
            pv(0, vs, j > 0, 0);
            if (!wait(bars.p_full(0), g & 1)) return false;
            ptx::tc_fence_after();
            pv(0, vs, true, 1);
            if (NT == 1) ptx::tc_commit(bars.pv_done(vs));
            if (!more) ptx::tc_commit(bars.o_full(0));
            if (more) s(0, ks1);
            if (NT == 2) {
                if (!wait(bars.p_half(1), g & 1)) return false;
                ptx::tc_fence_after();
                pv(1, vs, j > 0, 0);
                if (!wait(bars.p_full(1), g & 1)) return false;
                ptx::tc_fence_after();
                pv(1, vs, true, 1);
                ptx::tc_commit(bars.pv_done(vs));
                if (!more) ptx::tc_commit(bars.o_full(1));
                if (more) s(1, ks1);
            }
        }
        return true;
    }
};

// Persistent: one CTA per SM walks the work units u = blockIdx.x, + gridDim.x, ...
// (heaviest first).  The rings, the barriers' phases and the key-tile count g run
// on across units, so the next unit's Q and first K/V tiles load while the current
// unit finishes, and its first S MMAs overlap the current unit's epilogue.
template <typename T, int HD, int NT>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const PrefillParams p, int num_qt, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    using L = Layout<HD, NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_units = (p.num_q_heads / NT) * p.num_seqs * num_qt;
    const int Hq = p.num_q_heads, ps = p.page_size;

    const Bars bars{sbase + L::kBar};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + L::kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBar + L::kNumBars * 8 + 8);

    if (threadIdx.x == 0) {
        ptx::mbar_init(bars.q_full(), 1);
        for (int i = 0; i < KST; ++i) {
            ptx::mbar_init(bars.kv_full(i), 2);
            for (int x = 0; x < 2; ++x) ptx::mbar_init(bars.s_full(x, i), 1);
        }
        for (int i = 0; i < VST; ++i) ptx::mbar_init(bars.pv_done(i), 1);
        for (int x = 0; x < 2; ++x) {
            ptx::mbar_init(bars.p_full(x), 4);                  // one arrival per softmax warp
            ptx::mbar_init(bars.p_half(x), 4);
            ptx::mbar_init(bars.o_full(x), 1);
            ptx::mbar_init(bars.o_read(x), 4 * NT);             // one arrival per softmax warp
            ptx::mbar_init(bars.stage_free(x), 4 * NT);
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
    if (threadIdx.x == 0 && *tmem_slot != 0u) {
        *abort_flag = 1;
        record_error(p.status, PKV_ERR_CUDA, static_cast<long long>(*tmem_slot));
    }

    if (warp == kKWarp || warp == kVWarp) {
        // ------------------------------ TMA producers ------------------------------
        // Load step t carries K tile t (K warp) and V tile t-1 (V warp: V runs one tile
        // behind K) on kv_full(t % KST); t counts key tiles across all units of this
        // CTA.  A key tile is 8 page groups of 16 rows x NH column atoms: one box per
        // lane.  The K warp also loads each unit's Q tiles, once the previous unit's
        // last S MMA has read them.
        const bool is_k = warp == kKWarp;
        const int nst = is_k ? KST : VST;
        const CUtensorMap* map = is_k ? &tm_k : &tm_v;
        const uint32_t ring = sbase + (is_k ? L::kK : L::kV);
        const int group = lane / L::NH, half = lane % L::NH;
        const bool my_lane = group < 8;
        if (lane == 0) {
            ptx::prefetch_tmap(map);
            if (is_k) ptx::prefetch_tmap(&tm_q);
            else ptx::mbar_arrive(bars.kv_full(0));             // step 0 carries no V tile
        }
        int g = 0, uc = 0;
        int end_g[2] = {-8, -8};            // last key tile of the units with uc parity 0 / 1
        bool ok = true;
        UnitLoad ld = unit_load<NT>(p, blockIdx.x, num_units);
        for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
            const Unit w = unit_of<NT>(p, u, num_qt, ld, is_k && lane == 0);
            ld = unit_load<NT>(p, u + gridDim.x, num_units);
            if (!w.valid) continue;
            if (is_k) {
                if (uc > 0) {
                    // Q buffers free: the previous unit's last S MMA (of the last tile) is done
                    const int gl = g - 1;
                    ok = warp_wait(bars.s_full(NT - 1, gl % KST), (gl / KST) & 1, lane, abort_flag, p.status);
                    if (!ok) break;
                }
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(bars.q_full(), NT * L::kTile);
                    for (int x = 0; x < NT; ++x)
                        for (int a = 0; a < L::NH; ++a)
                            ptx::tma_load_3d(sbase + L::kQ + x * L::kTile + a * kAtom, &tm_q, bars.q_full(), 64 * a,
                                             w.h0 + x, w.q0 + w.r0);
                }
            }
            const int32_t* bt = p.block_tables + static_cast<size_t>(w.b) * p.max_pages_per_seq;
            for (int j = 0; j < w.n_tiles; ++j, ++g) {
                const int key0 = (w.t_first + j) * BN + 16 * group;
                const int pg = (my_lane && key0 < w.ctx) ? __ldg(bt + key0 / ps) : -1;
                const int st = g % nst;
                if (g >= nst) {
                    // a K stage is free once S of the last tile KST key tiles back is done,
                    // a V stage once PV of the last tile VST key tiles back is done
                    const int prev = g - nst;
                    ok = warp_wait(is_k ? bars.s_full(NT - 1, st) : bars.pv_done(st), (prev / nst) & 1, lane,
                                   abort_flag, p.status);
                    // a V stage that held a unit's last tile is that unit's epilogue staging
                    // area until its epilogue has drained it
                    for (int e = 0; e < 2 && ok && !is_k; ++e)
                        if (end_g[e] == prev) {
                            const int ue = uc - 1 - ((uc - 1 - e) & 1);   // the unit with parity e
                            ok = warp_wait(bars.stage_free(ue), (ue >> 1) & 1, lane, abort_flag, p.status);
                        }
                    if (!ok) break;
                }
                int row = -1;
                if (my_lane && key0 < w.ctx) {
                    if (pg < 0 || pg >= p.num_pages) {
                        if (half == 0) record_error(p.status, PKV_ERR_DEVICE_RANGE, pg);
                    } else {
                        row = pg * ps + key0 % ps;
                    }
                }
                const unsigned nbox = __popc(__ballot_sync(0xffffffffu, row >= 0));
                const uint32_t full = bars.kv_full((is_k ? g : g + 1) % KST);
                if (lane == 0) ptx::mbar_arrive_expect_tx(full, nbox * 16 * 128);
                __syncwarp();
                if (row >= 0)
                    ptx::tma_load_3d(ring + st * L::kTile + half * kAtom + group * 2048, map, full, 64 * half, w.kvh,
                                     row);
            }
            end_g[uc & 1] = g - 1;
            ++uc;
        }
        // The step after the last tile carries no K tile.  Like a K tile, its arrival waits
        // until the step KST back on the same barrier has been consumed (the S MMA of tile
        // g - KST is done): otherwise it could land while that earlier step still waits for
        // its V tile (the V warp may lag behind an epilogue's staging area) and would
        // complete that step's phase without it.
        if (ok && is_k) {
            if (g >= KST)
                ok = warp_wait(bars.s_full(NT - 1, g % KST), ((g - KST) / KST) & 1, lane, abort_flag, p.status);
            if (ok && lane == 0) ptx::mbar_arrive(bars.kv_full(g % KST));
        }
        if (*abort_flag && lane == 0) {
            // let the copies this warp issued land before the CTA's shared memory is released
            const int last = is_k ? g : g + 1;
            for (int v = max(0, last - KST); v < last; ++v)
                ptx::mbar_wait(bars.kv_full(v % KST), (v / KST) & 1, kSpinLimit >> 4);
            if (is_k && uc > 0) ptx::mbar_wait(bars.q_full(), (uc - 1) & 1, kSpinLimit >> 4);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            Issuer<T, HD, NT> mma;
            for (int x = 0; x < NT; ++x) mma.dq[x] = sdesc(sbase + L::kQ + x * L::kTile, 16, 1024);
            mma.dk = sdesc(sbase + L::kK, 16, 1024);
            mma.dv = sdesc(sbase + L::kV, kAtom, 1024);
            mma.bars = bars;
            mma.abort_flag = abort_flag;
            mma.status = p.status;
            int g = 0, uc = 0;
            UnitLoad ld = unit_load<NT>(p, blockIdx.x, num_units);
            for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
                const Unit w = unit_of<NT>(p, u, num_qt, ld, false);
                ld = unit_load<NT>(p, u + gridDim.x, num_units);
                if (!w.valid) continue;
                if (!mma.unit(g, w.n_tiles, uc)) break;
                g += w.n_tiles;
                ++uc;
            }
            // drain: every tcgen05 op issued by this thread completes before TMEM is freed
            ptx::tc_commit(bars.mma_done());
            ptx::mbar_wait(bars.mma_done(), 0, kSpinLimit);
        }
    } else if (warp >= kSoftWarp0 && warp < kSoftWarp0 + 4 * NT) {
        // ------------------------------ softmax + epilogue ------------------------------
        const int x = (warp - kSoftWarp0) >> 2;                  // query tile (head h0 + x)
        const int quarter = warp & 3;                            // TMEM lanes this warp reaches
        const int row = quarter * 32 + lane;                     // TMEM lane == tile row
        const uint32_t trow = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tS = trow + x * 128, tO = trow + kOCol + x * 128;
        const float sl2 = p.scale_log2;
        int g = 0, uc = 0;
        bool ok = true;
        // A unit's epilogue runs once the next unit's first key tile is through softmax (or
        // after the last unit), so that it overlaps the next unit's first MMAs instead of
        // delaying them: it waits for the unit's last P.V (o_full), reads O into registers,
        // lets the issuer overwrite O (o_read), then writes O / l out through the V stage of
        // the unit's last key tile and releases that stage to the V producer (stage_free).
        // Every P.V of the unit is done once o_full of its last tile has fired (commits track
        // all earlier MMAs), so that V stage is no longer read.
        // The pending unit's parameters wait in shared memory (warp-uniform; kept out of the
        // registers the softmax needs), its row sum in l_pend.
        struct Pending {
            int q0, n, r0, h0, g_last, uc;
        };
        Pending* pend_s = reinterpret_cast<Pending*>(smem + L::kPend) + (warp - kSoftWarp0);
        float l_pend = 0.f;
        bool pending = false;
        auto epilogue = [&]() -> bool {
            __syncwarp();
            const Pending e = *pend_s;
            if (!warp_wait(bars.o_full(NT - 1), e.uc & 1, lane, abort_flag, p.status)) return false;
            ptx::tc_fence_after();
            // O / l is read into registers (packed to T), then the issuer may overwrite O
            // (o_read) while the rows leave a column chunk at a time (each warp 32 rows x CW
            // columns; 16-byte chunk c of a row at position c ^ (row % CCH), conflict-free) as
            // whole row segments.
            uint32_t ob[HD / 2];
            const float inv = 1.f / l_pend;
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(tO + 32 * c, o);
                ptx::tc_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    ob[16 * c + i] = pack2<T>(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bars.o_read(e.uc));
            constexpr int CW = L::kTile / 512;                        // columns per chunk (64 or 32)
            constexpr int RB = CW * 2, CCH = RB / 16;                  // bytes and 16-byte chunks per row
            uint8_t* stage = smem + L::kV + (e.g_last % VST) * L::kTile + (warp - kSoftWarp0) * 32 * RB;
            T* out = static_cast<T*>(p.out);
#pragma unroll
            for (int c0 = 0; c0 < HD; c0 += CW) {
#pragma unroll
                for (int cc = 0; cc < CCH; ++cc) {
                    const int k = c0 / 2 + 4 * cc;
                    *reinterpret_cast<uint4*>(stage + lane * RB + ((cc ^ (lane % CCH)) * 16)) =
                        make_uint4(ob[k], ob[k + 1], ob[k + 2], ob[k + 3]);
                }
                __syncwarp();
#pragma unroll
                for (int it = 0; it < CCH; ++it) {
                    const int idx = it * 32 + lane, rr = idx / CCH, cc = idx % CCH;
                    const int tr = e.r0 + quarter * 32 + rr;              // row within the chunk
                    const uint4 val = *reinterpret_cast<const uint4*>(stage + rr * RB + ((cc ^ (rr % CCH)) * 16));
                    if (tr < e.n)
                        *reinterpret_cast<uint4*>(out + (static_cast<size_t>(e.q0 + tr) * Hq + e.h0 + x) * HD + c0 +
                                                  cc * 8) = val;
                }
                __syncwarp();
            }
            if (lane == 0) ptx::mbar_arrive(bars.stage_free(e.uc));
            return true;
        };
        UnitLoad ld = unit_load<NT>(p, blockIdx.x, num_units);
        for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
            const Unit w = unit_of<NT>(p, u, num_qt, ld, false);
            ld = unit_load<NT>(p, u + gridDim.x, num_units);
            if (!w.valid) continue;
            const int pos = w.ctx - w.n + w.r0 + row;
            const int lim = p.causal ? min(pos, w.ctx - 1) : w.ctx - 1;
            const int row_lo = p.window > 0 ? max(0, pos - p.window + 1) : 0;   // this row's first key
            float m_ref = -INFINITY, l = 0.f;
            for (int j = 0; j < w.n_tiles; ++j, ++g) {
                ok = warp_wait(bars.s_full(x, g % KST), (g / KST) & 1, lane, abort_flag, p.status);
                if (!ok) break;
                ptx::tc_fence_after();
                // Two passes over the row in 64-column halves (one compact loop body each; S
                // is read from TMEM twice, which costs a few dozen cycles): the row max, then
                // P = 2^(s * scale - m) written back over the first half of the S columns.
                const int jt = w.t_first + j;
                const bool masked = jt * BN + BN - 1 > w.min_lim || jt * BN < w.lo_mask;   // diagonal / last / window edge
                float mc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    #pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    float v[64];
                    load_half(tS + 64 * hh, v);
                    if (masked) mask_half(v, jt * BN + 64 * hh, lim, row_lo, p.window > 0);
                    // four independent max chains keep the reduction's latency short
    #pragma unroll
                    for (int c = 0; c < 64; c += 8) {
    #pragma unroll
                        for (int k = 0; k < 4; ++k) mc[k] = max3(mc[k], v[c + 2 * k], v[c + 2 * k + 1]);
                    }
                }
                // -inf only for a row that sees no key of this tile (possible with a window)
                const float mt = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])) * sl2;
                if (j == 0) {
                    m_ref = mt;
                } else if (__any_sync(0xffffffffu, mt > m_ref + kRescaleThreshold)) {
                    // S_X(j) completed after PV_X(j-1) (same issuer, in order), so O_X is settled
                    const float m_new = fmaxf(m_ref, mt);
                    const float corr = m_new == -INFINITY ? 1.f : ptx::ex2(m_ref - m_new);
                    l *= corr;
                    m_ref = m_new;
    #pragma unroll 1
                    for (int c = 0; c < HD / 16; ++c) {
                        uint32_t o[16];
                        tmem_ld16(tO + 16 * c, o);
                        ptx::tc_wait_ld();
    #pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
                        ptx::tmem_st16(tO + 16 * c, o);
                    }
                }
                if (x == 0 && w.ctx < (jt + 1) * BN) {
                    // V rows past the context (tail of the last page, or never loaded) must be
                    // finite zeros: P is 0 there but 0 * NaN would poison O.  Tile A's warps do it
                    // before either half of P_A(j) is released (PV_A(j) runs before PV_B(j)).
                    const int vs = g % VST;
                    ok = warp_wait(bars.kv_full((g + 1) % KST), ((g + 1) / KST) & 1, lane, abort_flag, p.status);
                    if (!ok) break;
                    const int first = w.ctx - jt * BN;                  // first invalid row of the tile
                    uint4* vt = reinterpret_cast<uint4*>(smem + L::kV + vs * L::kTile);
                    const int tid = threadIdx.x - kSoftWarp0 * 32, per = (BN - first) * 8;
                    for (int idx = tid; idx < L::NH * per; idx += 128) {
                        const int a = idx / per, rem = idx % per;
                        vt[(a * kAtom + (first + rem / 8) * 128) / 16 + rem % 8] = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                const float neg = m_ref == -INFINITY ? 0.f : -m_ref;      // no key seen yet: all p are 0
                // one packed FMA per key pair, one SFU exponential per key
                const uint64_t sc2 = f2pack(sl2, sl2), ng2 = f2pack(neg, neg);
                uint64_t sum2[2] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
    #pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    float v[64];
                    load_half(tS + 64 * hh, v);
                    if (masked) mask_half(v, jt * BN + 64 * hh, lim, row_lo, p.window > 0);
                    uint32_t pk[32];
    #pragma unroll
                    for (int i = 0; i < 32; ++i)
                        pk[i] = exp2_pair<T>(ffma2(f2pack(v[2 * i], v[2 * i + 1]), sc2, ng2), sum2[i & 1]);
                    // P column c holds keys 2c, 2c+1: half hh goes to columns 32 hh .. 32 hh + 31,
                    // which hold scores this thread has already read
                    tmem_st32(tS + 32 * hh, pk);
                    if (hh == 0) {
                        // the first 64 keys' P is in place: P.V over them may start
                        ptx::tc_wait_st();
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(bars.p_half(x));
                    }
                }
                {
                    float a0, a1, b0, b1;
                    asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(sum2[0]));
                    asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(sum2[1]));
                    l += (a0 + a1) + (b0 + b1);
                }
                ptx::tc_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bars.p_full(x));       // one arrival per warp
                if (j == 0 && pending) {
                    ok = epilogue();
                    if (!ok) break;
                    pending = false;
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) *pend_s = Pending{w.q0, w.n, w.r0, w.h0, g - 1, uc};
            l_pend = l;
            pending = true;
            ++uc;
        }
        if (ok && pending) epilogue();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
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

// 3-D map over a [rows][heads][hd] tensor of 16-bit elements, box {64, 1, box_rows}, SW128.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t hd, uint64_t heads, uint64_t rows,
              uint32_t box_rows) {
    EncodeTiled enc = encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {hd, heads, rows};
    const cuuint64_t strides[2] = {hd * 2, heads * hd * 2};
    const cuuint32_t box[3] = {64, 1, box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int HD, int NT>
cudaError_t run(const PrefillParams& p, cudaStream_t stream) {
    using L = Layout<HD, NT>;
    const CUtensorMapDataType dt =
        std::is_same<T, __nv_bfloat16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tq, tk, tv;
    const uint64_t pool_rows = static_cast<uint64_t>(p.num_pages) * p.page_size;
    if (!make_map(&tq, p.q, dt, HD, p.num_q_heads, p.total_q, BM) ||
        !make_map(&tk, p.k_pages, dt, HD, p.num_kv_heads, pool_rows, 16) ||
        !make_map(&tv, p.v_pages, dt, HD, p.num_kv_heads, pool_rows, 16))
        return cudaErrorInvalidValue;
    // one persistent CTA per SM (at most one per work unit)
    const int num_qt = ceil_div(p.max_q_len, BM);
    const long long units = static_cast<long long>(p.num_q_heads / NT) * p.num_seqs * num_qt;
    if (units > 0x7fffffffLL) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = static_cast<int>(units < sms ? units : sms);
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(prefill_tc_kernel<T, HD, NT>), L::kSmem);
    if (e != cudaSuccess) return e;
    prefill_tc_kernel<T, HD, NT><<<grid, kThreads, L::kSmem, stream>>>(p, num_qt, tq, tk, tv);
    return cudaGetLastError();
}

template <typename T, int HD>
cudaError_t run_hd(const PrefillParams& p, cudaStream_t stream) {
    // pair the heads of a group when the group size is even
    return (p.num_q_heads / p.num_kv_heads) % 2 == 0 ? run<T, HD, 2>(p, stream) : run<T, HD, 1>(p, stream);
}

template <typename T>
cudaError_t run_t(const PrefillParams& p, cudaStream_t stream) {
    return p.head_dim == 64 ? run_hd<T, 64>(p, stream) : run_hd<T, 128>(p, stream);
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
    return dtype == PKV_BF16 ? run_t<__nv_bfloat16>(p, stream) : run_t<__half>(p, stream);
}

}  // namespace pkv
