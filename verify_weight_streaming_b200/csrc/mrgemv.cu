// mrgemv_bf16: multi-row bf16 GEMV with fp32 output for m <= 16 rows.
//
// The multi-row GEMV of Strata PR #109 ("What", router bullet): the weight is
// read from HBM once per call and shared by all m rows, and every row's
// accumulators follow exactly the order of the single-row call.  The
// nx_batchscale_kat.nx note states the test this has to pass: per-row cost must
// fall with m because the weight bytes are not re-streamed per row.
//
// Design (B200):
//  * grid = one CTA per SM (at most n; two per SM for large blocks under
//    PDL); CTA b owns the contiguous column block [b*n/G, (b+1)*n/G) of Wt,
//    i.e. a contiguous run of weight rows.
//  * The block streams through a ring of shared-memory slots, one column group
//    (up to CG columns x k) per slot, with cp.async.bulk global->shared copies
//    counted on an mbarrier (no tensor map; each copy lands in its own CTA).
//    Group g is consumed by column warp g % CWG from slot g % S; when slots
//    are refilled, S is a multiple of CWG, so each slot has a single consumer
//    warp that waits for the slot's successive uses in order.  The first
//    pass of the ring is requested before griddepcontrol.wait (up to 64 KB
//    of it for blocks over 96 KB, the rest right after A), so under
//    programmatic dependent launch the weight streams while the previous
//    kernel runs.
//  * KW x CWG warps per CTA, at most 16.  More warps than k-slices work on
//    separate column groups in parallel.  One more warp, where the SM has
//    room, runs the same code once at kernel start without storing anything,
//    to bring it into the instruction cache (the warm warp).
//  * Fused router (router_gemv_topk): every logit is also stored as a flagged
//    64-bit word; CTA r polls row r's words and selects its top-k.
//  * A (m rows, bf16) is staged once in shared memory by a bulk copy issued
//    after the grid-dependency wait; rows m..MB-1 are zero.
//  * The k loop reads shared memory with loads the compiler may schedule
//    freely (their addresses pass through a volatile move after the slot's
//    barrier wait, and every accumulator is pinned before the slot is
//    released), and advances every chain with fma.rn.f32.bf16 on the bf16
//    operands as they are in shared memory (one rounding in fp32: the same
//    bits as an fp32 FMA of the converted values, with no conversions).
//  * Lanes split k in 4-element chunks: chunk q belongs to lane q % 32 of the
//    k-slice that holds it.  KW warps split k into contiguous slices; KW is a
//    function of k alone.  Each lane keeps one fp32 accumulator per (row,
//    column), updated in ascending k.  Rows run in buckets of 1, 2, 4, 8 or
//    16 (a bucket's spare rows are zero).
//  * Reduction: a fixed xor-butterfly over the 32 lanes
//    (bit 16, 8, 4, 2, 1; realised as a reduce-scatter so each lane finishes a
//    share of the values), then the KW slices in slice order.  The tree of
//    every output element is the same for every m, every row position and
//    every column grouping, so row i is bitwise identical at every m.
//  * Every wait on data is an mbarrier wait bounded in time.  The GEMV warps
//    meet at two named barriers (after A is staged, and before the k-slice
//    sum), which every one of them reaches whether or not a wait ran out.
#include "common.cuh"
#include "topk_core.cuh"

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

namespace mr {
namespace gemv {

// Warps per CTA at most (512 threads, so at most 128 registers each: a CTA
// of fewer warps then leaves room on its SM for the next launch's CTA), and
// the unroll of the k loop: two steps, except for 8-column groups of 4 or more
// rows and for 16 rows, whose accumulators leave few registers for a second
// step (measured: one step is faster there, two elsewhere), and except in the
// fused router's kernels, whose code is fetched cold in each window of a
// sequence of window sizes: one step, half the loop's code, made the window
// sequence 1-3% faster (same box) though a repeated m = 1 window is 0.1 us
// slower.  None of this changes an output's arithmetic: a lane's chain and
// the reduction order are fixed by k.
constexpr int kWarpsMax = 16;
__host__ __device__ constexpr int warps_max(int, int) { return kWarpsMax; }
__host__ __device__ constexpr int q_unroll(int MB, int CG, bool fused = false) {
    return (fused || (CG >= 8 && MB >= 4) || MB >= 16) ? 1 : 2;
}

constexpr int kMaxRows = 16;
// Fused router: each logit is also stored as one 64-bit word, the flag
// kTagReady in the high half and the logit's bits in the low half, in a tag
// array of the workspace that is all zero between calls.  A 64-bit store is
// single-copy atomic, so a word that carries the flag carries its logit too.
constexpr uint32_t kTagReady = 1u;
#ifndef MR_FUSED_P
#define MR_FUSED_P 16   // logits per lane per segment in the fused selection
#endif

struct Params {
    const uint16_t *A;
    int64_t lda;
    const uint16_t *Wt;
    int64_t ldw;
    float *C;
    int64_t ldc;
    int m, n, k;
    int G;          // CTAs
    int KW;         // warps splitting k (function of k only)
    int CWG;        // column-group warps per CTA
    int S;          // ring slots
    uint32_t a_bytes;     // shared bytes reserved for A (MB rows)
    uint32_t slot_bytes;  // CG * k * 2
    int sigmoid;          // store 1 / (1 + exp(-c)) instead of c (MR_GEMV_SIGMOID)
    // Fused router (top-k of each row after the GEMV), unused otherwise.
    int topk;
    int32_t *idx;
    float *val;
    int64_t ldo;
    uint64_t *tags;       // m x n tagged logits, row stride n (zero between calls)
};

// k-slice split: a function of k alone (never of m), so the reduction tree of
// an output element is fixed by k.
#ifndef MR_GEMV_MIN_CHUNKS
#define MR_GEMV_MIN_CHUNKS 4   // 4-element chunks per lane per k-slice, at least
#endif
#ifndef MR_GEMV_EVEN_LANES
#define MR_GEMV_EVEN_LANES 1   // every lane of a slice gets the same number of chunks
#endif
#ifndef MR_GEMV_KW_MAX
#define MR_GEMV_KW_MAX 4
#endif
// Weight bytes a CTA requests before the dependency wait when its block is
// larger than MR_GEMV_PREWAIT_SPLIT (smaller blocks are requested whole).
#ifndef MR_GEMV_PREWAIT_BYTES
#define MR_GEMV_PREWAIT_BYTES 65536u
#endif
#ifndef MR_GEMV_PREWAIT_SPLIT
#define MR_GEMV_PREWAIT_SPLIT 98304u
#endif
__host__ __device__ inline int k_warps(int k) {
    const int q = k / 4;
    int best = 1;
    for (int kw = 2; kw <= MR_GEMV_KW_MAX; kw *= 2) {
        if (q % kw != 0 || q / kw < 32 * MR_GEMV_MIN_CHUNKS) break;
        if (MR_GEMV_EVEN_LANES && (q / kw) % 32 != 0) break;
        best = kw;
    }
    return best;
}

// The shared expert's scalar gate: logistic of the GEMV output, with CUDA's
// expf and an IEEE divide.
__device__ __forceinline__ float gate_out(const Params &p, float c) {
    return p.sigmoid ? 1.0f / (1.0f + expf(-c)) : c;
}

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t *a) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(a) : "memory");
    return v;
}

// Output of logit (r, col): to C, and in the fused router (where C may be
// null) also as a tagged word with a GPU-scope relaxed store.
template <bool FUSED>
__device__ __forceinline__ void store_logit(const Params &p, int r, int col, float v) {
    if (!FUSED || p.C) p.C[(int64_t)r * p.ldc + col] = v;
    if constexpr (FUSED)
        asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p.tags + (int64_t)r * p.n + col),
                     "l"(((uint64_t)kTagReady << 32) | __float_as_uint(v))
                     : "memory");
}

// Top-k of one row of tagged logits, taken by one warp in segments of 32 * P
// words: each segment's words are re-read until all carry the flag (bounded
// by kWaitLimitNs; false if it runs out), then keyed and merged like
// router_topk's rows.  `out`: lane t holds the rank-t key.
// With `synthetic` the row is not read: word j is taken to be a ready
// logit that grows with j, which runs the selection's common path (used to
// bring the code into the instruction cache).
template <int P>
__device__ __forceinline__ bool tagged_topk(const uint64_t *row, int n, int K, int lane, uint64_t *scratch,
                                            uint64_t &out, bool synthetic) {
    const uint64_t t0 = globaltimer_ns();
    uint64_t run = 0ull;
    for (int base = 0; base < n; base += 32 * P) {
        uint64_t w[P];
        if (synthetic) {
#pragma unroll
            for (int i = 0; i < P; ++i)
                w[i] = ((uint64_t)kTagReady << 32) | (0x3F800000u + (uint32_t)(base + lane + 32 * i));
        } else {
#pragma unroll
            for (int i = 0; i < P; ++i) {
                const int j = base + lane + 32 * i;
                w[i] = j < n ? ld_relaxed_u64(row + j) : ((uint64_t)kTagReady << 32);
            }
        }
        for (int spin = 0;; ++spin) {
            bool ready = true;
#pragma unroll
            for (int i = 0; i < P; ++i) ready = ready && (uint32_t)(w[i] >> 32) == kTagReady;
            if (__all_sync(0xffffffffu, ready)) break;
            if ((spin & 15) == 15 && __any_sync(0xffffffffu, globaltimer_ns() - t0 > kWaitLimitNs)) return false;
#pragma unroll
            for (int i = 0; i < P; ++i)
                if ((uint32_t)(w[i] >> 32) != kTagReady) w[i] = ld_relaxed_u64(row + base + lane + 32 * i);
        }
        uint64_t keys[P];
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const int j = base + lane + 32 * i;
            keys[i] = j < n ? topk::make_key(__uint_as_float((uint32_t)w[i]), (uint32_t)j) : 0ull;
        }
        run = topk::warp_topk_merge<P>(keys, run, K, lane, scratch);
    }
    out = run;
    return true;
}


// 8-byte load from shared memory by 32-bit shared address (always LDS, never
// a generic load).  Not volatile: the compiler may schedule it like any
// load, so its address must come from launder() after the wait that makes
// the data valid (that dependence keeps it below the wait).
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

// The same value, through an instruction the compiler cannot see through or
// move across other volatile asm (the barrier waits): loads whose addresses
// derive from it stay after the wait that precedes it.
__device__ __forceinline__ uint32_t launder(uint32_t x) {
    uint32_t y;
    asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x) : "memory");
    return y;
}

// acc = fma(a_h, w_h, acc) with a_h, w_h the bf16 in half H (0 low, 1 high) of
// a and w, multiplied and added in one rounding to nearest in fp32.  A bf16
// converts to fp32 exactly and the product of two bf16 is exact in fp32, so
// this is bit for bit the fp32 FMA of the converted operands, without the
// conversions.
template <int H>
__device__ __forceinline__ void fma_bf16(float &acc, uint32_t a, uint32_t w) {
    if constexpr (H == 0)
        asm("{\n\t.reg .b16 al, ah, wl, wh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {wl, wh}, %2;\n\t"
            "fma.rn.f32.bf16 %0, al, wl, %0;\n\t}"
            : "+f"(acc) : "r"(a), "r"(w));
    else
        asm("{\n\t.reg .b16 al, ah, wl, wh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {wl, wh}, %2;\n\t"
            "fma.rn.f32.bf16 %0, ah, wh, %0;\n\t}"
            : "+f"(acc) : "r"(a), "r"(w));
}

// Reduce-scatter over the warp: level D pairs lanes that differ in bit D (16,
// 8, 4, 2, 1 in that order).  While more than one value is left, the lane with
// bit D clear keeps the lower half and its partner the upper half; with one
// value left both partners add (a + b == b + a, so both hold the same bits).
template <int CNT, int D>
struct ReduceScatter {
    static __device__ __forceinline__ void run(float *v, int lane, int &base) {
        if constexpr (CNT >= 2) {
            constexpr int H = CNT / 2;
            const bool up = (lane & D) != 0;
#pragma unroll
            for (int i = 0; i < H; ++i) {
                const float send = up ? v[i] : v[i + H];
                const float keep = up ? v[i + H] : v[i];
                const float recv = __shfl_xor_sync(0xffffffffu, send, D);
                v[i] = __fadd_rn(keep, recv);
            }
            if (up) base += H;
            if constexpr (D > 1) ReduceScatter<H, D / 2>::run(v, lane, base);
        } else {
            v[0] = __fadd_rn(v[0], __shfl_xor_sync(0xffffffffu, v[0], D));
            if constexpr (D > 1) ReduceScatter<1, D / 2>::run(v, lane, base);
        }
    }
};

// Values per lane after the reduce-scatter of V values, and the mask of lane
// bits that were butterfly (replicating) levels.
template <int V>
struct Scatter {
    static constexpr int kPerLane = V >= 32 ? V / 32 : 1;
    static constexpr int kReplMask = V >= 32 ? 0 : (32 / V) - 1;
};

// Floats of k-slice partials: [groups][KW][MB x CG] when k is split over warps.
__host__ __device__ inline size_t red_floats(int KW, int ng_max, int MB, int CG) {
    return KW > 1 ? (size_t)ng_max * KW * MB * CG : 0;
}

// Most column groups any CTA of the launch owns.
__host__ __device__ inline int ng_max_of(int n, int G, int CG) {
    const int cols_max = (n + G - 1) / G;
    return (cols_max + CG - 1) / CG;
}

struct Smem {
    uint16_t *a;          // [MB][k]
    uint8_t *ring;        // S slots
    uint64_t *chunk_full; // [S] first pass: one barrier per up-front copy chunk
    uint64_t *full;       // [S] refills: slot s's uses 1, 2, ...
    uint64_t *empty;      // [S]
    uint64_t *a_full;     // [1] A has landed (A staged by a bulk copy)
    float *red;           // [groups][KW][MB x CG] k-slice partials (KW > 1)
};

// One column group: NC (power of two) columns of this warp's k-slice.  With
// `warm` the group's code runs over whatever the slot holds, with no barrier
// wait or arrival and no store: it only brings the instructions into the
// instruction cache.
template <int MB, int NC, int CGMAX, bool FUSED>
__device__ __forceinline__ bool do_group(const Params &p, const Smem &sm, int g, int ncol,
                                         int col0, int slice, int lane, int q_begin, int q_end,
                                         int chunk_groups, bool warm) {
    const int k = p.k;
    const int slot = g % p.S;
    // The first S groups come in up-front copy chunks (one barrier each,
    // phase 0); group g >= S is the refill of its slot, use g / S, counted on
    // the slot's refill barrier from phase 0.
    const uint64_t *bar = g < p.S ? &sm.chunk_full[g / chunk_groups] : &sm.full[slot];
    const uint32_t par = g < p.S ? 0u : (uint32_t)(g / p.S - 1) & 1u;
    if (!warm && !mbar_wait_bounded(smem_u32(bar), par, MR_DEVERR_GEMV_TIMEOUT)) return false;

    const uint32_t w_s = launder(smem_u32(sm.ring + (size_t)slot * p.slot_bytes));
    const uint32_t a_s = launder(smem_u32(sm.a));
    const uint32_t row_b = (uint32_t)k * 2u;
    // acc[r][j]: one fp32 chain per (row, column), over this lane's k
    // positions in ascending order.
    float acc[MB][NC];
#pragma unroll
    for (int r = 0; r < MB; ++r)
#pragma unroll
        for (int j = 0; j < NC; ++j) acc[r][j] = 0.0f;

    // Operands come from shared memory through lds64 (non-volatile, so the
    // compiler schedules the loads ahead of the FMAs that use them): four k
    // positions of every row of A and every column of the group.  At each of
    // the four positions, in order, every (row, column) chain advances by one
    // mixed-precision FMA, so consecutive FMAs are independent of each other.
    auto a_at = [&](int r, int qq) { return lds64(a_s + (uint32_t)r * row_b + 8u * (uint32_t)qq); };
    auto w_at = [&](int j, int qq) { return lds64(w_s + (uint32_t)j * row_b + 8u * (uint32_t)qq); };
#pragma unroll (q_unroll(MB, CGMAX, FUSED))
    for (int q = q_begin + lane; q < q_end; q += 32) {
        uint2 wr[NC], ar[MB];
#pragma unroll
        for (int j = 0; j < NC; ++j) wr[j] = w_at(j, q);
#pragma unroll
        for (int r = 0; r < MB; ++r) ar[r] = a_at(r, q);
#pragma unroll
        for (int r = 0; r < MB; ++r)
#pragma unroll
            for (int j = 0; j < NC; ++j) fma_bf16<0>(acc[r][j], ar[r].x, wr[j].x);  // k = 4q
#pragma unroll
        for (int r = 0; r < MB; ++r)
#pragma unroll
            for (int j = 0; j < NC; ++j) fma_bf16<1>(acc[r][j], ar[r].x, wr[j].x);  // 4q + 1
#pragma unroll
        for (int r = 0; r < MB; ++r)
#pragma unroll
            for (int j = 0; j < NC; ++j) fma_bf16<0>(acc[r][j], ar[r].y, wr[j].y);  // 4q + 2
#pragma unroll
        for (int r = 0; r < MB; ++r)
#pragma unroll
            for (int j = 0; j < NC; ++j) fma_bf16<1>(acc[r][j], ar[r].y, wr[j].y);  // 4q + 3
    }
    // Every accumulator is final before the slot is released: the empty
    // volatile asm consumes them all, and volatile asm keeps its order, so no
    // load of the slot (nor the FMAs that use it) can sink below the release.
#pragma unroll
    for (int r = 0; r < MB; ++r)
#pragma unroll
        for (int j = 0; j < NC; ++j) asm volatile("" ::"f"(acc[r][j]));
    // This warp no longer reads the slot.
    __syncwarp();
    if (lane == 0 && !warm) mbar_arrive(smem_u32(&sm.empty[slot]));

    constexpr int V = MB * NC;
    float v[V];
#pragma unroll
    for (int r = 0; r < MB; ++r)
#pragma unroll
        for (int j = 0; j < NC; ++j) v[r * NC + j] = acc[r][j];
    int base = 0;
    ReduceScatter<V, 16>::run(v, lane, base);
    constexpr int PL = Scatter<V>::kPerLane;

    // The warm pass stores nothing: the GEMV warps may already be using the
    // partials' shared memory.
    if ((lane & Scatter<V>::kReplMask) == 0 && !warm) {
        if (p.KW > 1) {
            // Partials of this k-slice for group g; the slices are summed, in
            // slice order, after every group of the CTA is done.
            float *red = sm.red + ((size_t)g * p.KW + slice) * (MB * CGMAX);
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int idx = base + i;
                red[(idx / NC) * CGMAX + idx % NC] = v[i];
            }
        } else {
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                const int idx = base + i;
                const int r = idx / NC, j = idx % NC;
                if (r < p.m && j < ncol) store_logit<FUSED>(p, r, col0 + j, gate_out(p, v[i]));
            }
        }
    }
    return true;
}

template <int MB, int NC, int CGMAX, bool FUSED>
__device__ __forceinline__ bool run_group(const Params &p, const Smem &sm, int g, int ncol,
                                          int col0, int slice, int lane, int q_begin, int q_end,
                                          int chunk_groups, bool warm) {
    if constexpr (NC > 1) {
        if (ncol <= NC / 2)
            return run_group<MB, NC / 2, CGMAX, FUSED>(p, sm, g, ncol, col0, slice, lane, q_begin, q_end,
                                                       chunk_groups, warm);
    }
    return do_group<MB, NC, CGMAX, FUSED>(p, sm, g, ncol, col0, slice, lane, q_begin, q_end, chunk_groups, warm);
}

template <int MB, int CG, bool FUSED>
__global__ void __launch_bounds__(kWarpsMax * 32, 1) gemv_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int k = p.k;

    // Column block of this CTA.
    const int c_begin = (int)(((int64_t)blockIdx.x * p.n) / p.G);
    const int c_end = (int)(((int64_t)(blockIdx.x + 1) * p.n) / p.G);
    const int ncols = c_end - c_begin;
    const int ng = (ncols + CG - 1) / CG;

    Smem sm;
    sm.a = reinterpret_cast<uint16_t *>(smem_raw);
    sm.ring = smem_raw + p.a_bytes;
    sm.chunk_full = reinterpret_cast<uint64_t *>(sm.ring + (size_t)p.S * p.slot_bytes);
    sm.full = sm.chunk_full + p.S;
    sm.empty = sm.full + p.S;
    uint64_t *misc = sm.empty + p.S;  // 6 words: A's barrier and spare words
    sm.a_full = misc;
    sm.red = reinterpret_cast<float *>(misc + 6);

    // Groups per copy chunk when no slot is refilled (0 when slots are refilled).
    const int chunk_groups = (int)max(1u, (32768u + p.slot_bytes - 1) / p.slot_bytes);
    // First-pass chunks requested before the dependency wait: all of them,
    // except that a block larger than MR_GEMV_PREWAIT_SPLIT requests only
    // MR_GEMV_PREWAIT_BYTES before the wait and the rest after A's copy, so
    // that A does not queue behind the whole block (this CTA's copies are
    // served in order, at ~44 GB/s per SM when every SM streams: 100 KB ahead
    // of A delayed it by ~2 us).
    const int first_chunks = (min(ng, p.S) + chunk_groups - 1) / chunk_groups;
    const bool split_prewait = (size_t)ncols * (size_t)k * 2u > MR_GEMV_PREWAIT_SPLIT;
    const int prewait_chunks =
        split_prewait ? min(first_chunks, max(1, (int)(MR_GEMV_PREWAIT_BYTES / ((size_t)chunk_groups * p.slot_bytes))))
                      : first_chunks;
    const int first = min(ng, p.S);

    auto issue_chunk = [&](int c) {
        const uint32_t row_bytes = (uint32_t)k * 2u;
        const int g0 = c * chunk_groups;
        const int g1 = min(g0 + chunk_groups, first);
        const int cc0 = c_begin + g0 * CG;
        const int nc = min((g1 - g0) * CG, c_end - cc0);
        const uint32_t bar = smem_u32(&sm.chunk_full[c]);
        const uint32_t dst = smem_u32(sm.ring + (size_t)g0 * p.slot_bytes);
        mbar_arrive_expect_tx(bar, row_bytes * (uint32_t)nc);
        if (p.ldw == k) {
            bulk_g2s(dst, p.Wt + (int64_t)cc0 * k, row_bytes * (uint32_t)nc, bar);
        } else {
            for (int j = 0; j < nc; ++j)
                bulk_g2s(dst + j * row_bytes, p.Wt + (int64_t)(cc0 + j) * p.ldw, row_bytes, bar);
        }
    };

    auto issue_group = [&](int g) {
        const int slot = g % p.S;
        const int gc0 = c_begin + g * CG;
        const int nc = min(CG, c_end - gc0);
        const uint32_t row_bytes = (uint32_t)k * 2u;
        const uint32_t bar = smem_u32(&sm.full[slot]);
        const uint32_t dst = smem_u32(sm.ring + (size_t)slot * p.slot_bytes);
        mbar_arrive_expect_tx(bar, row_bytes * (uint32_t)nc);
        if (p.ldw == k) {
            bulk_g2s(dst, p.Wt + (int64_t)gc0 * k, row_bytes * (uint32_t)nc, bar);
        } else {
            for (int j = 0; j < nc; ++j)
                bulk_g2s(dst + j * row_bytes, p.Wt + (int64_t)(gc0 + j) * p.ldw, row_bytes, bar);
        }
    };

    if (tid == 0) {
        for (int s = 0; s < p.S; ++s) {
            mbar_init(smem_u32(&sm.chunk_full[s]), 1);
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.empty[s]), (uint32_t)p.KW);
        }
        mbar_init(smem_u32(sm.a_full), 1);
        fence_mbar_init();
        // The whole first pass of the ring (min(ng, S) groups) is requested
        // now, before the wait for the previous kernel, in chunks of whole
        // groups of >= 32 KB each (small bulk copies stream below HBM
        // bandwidth: ~2.6 TB/s for 4 KB copies, ~6.2 TB/s for 16 KB, ~7 TB/s
        // for 32-64 KB).  The weight does not depend on the previous kernel.
        for (int c = 0; c < prewait_chunks; ++c) issue_chunk(c);
    }
    // The weight stream is in flight; the next kernel may start launching.
    grid_launch_dependents();

    const int slice = warp % p.KW;
    const int cw = warp / p.KW;
    const int q_total = k / 4;
    const int q_begin = (int)(((int64_t)slice * q_total) / p.KW);
    const int q_end = (int)(((int64_t)(slice + 1) * q_total) / p.KW);
    constexpr int kQStep = 32 * q_unroll(MB, CG, FUSED);  // one unrolled step of the k loop

    // The GEMV warps are 0 .. KW * CWG - 1.  A launch with fewer than 16 of
    // them has one more warp, which runs the code below once at kernel start
    // ("warm"): the first group for one unrolled step of the k loop and the
    // k-slice sum, over whatever shared memory holds, with no barrier wait
    // or arrival and no global store, then exits.  It fetches the GEMV's
    // instructions into the SM's instruction cache while the GEMV warps wait
    // for the previous kernel and for A.  (A kernel's code starts cold when
    // other kernels ran on the SM in between; measured at 1-2 us a call.)
    // The GEMV warps run the same code (the same instructions) once, for real.
    const int gemv_warps = p.KW * p.CWG;
    const bool warm_warp = warp >= gemv_warps;
    bool failed = false;
#pragma unroll 1
    for (int pass = warm_warp ? 0 : 1; pass < (warm_warp ? 1 : 2); ++pass) {
        const bool warm = pass == 0;
        if (!warm) {
            // A may be produced by the previous kernel on the stream.
            grid_dependency_wait();

            // Stage A (bf16) in shared memory with one bulk copy (per row if
            // strided); rows m..MB-1 are zero.  Under programmatic dependent
            // launch the weight was requested while the previous kernel ran
            // and has mostly landed by now.  (Per-thread cp.async copies of A
            // measured slower: up to 3 us for 16 rows of 2560, since every
            // CTA reads the same A lines.)
            if (tid == 0) {
                const uint32_t row_bytes = (uint32_t)k * 2u;
                const uint32_t bar = smem_u32(sm.a_full);
                mbar_arrive_expect_tx(bar, row_bytes * (uint32_t)p.m);
                if (p.lda == k) {
                    bulk_g2s(smem_u32(sm.a), p.A, row_bytes * (uint32_t)p.m, bar);
                } else {
                    for (int r = 0; r < p.m; ++r)
                        bulk_g2s(smem_u32(sm.a + (size_t)r * k), p.A + (int64_t)r * p.lda, row_bytes, bar);
                }
                for (int c = prewait_chunks; c < first_chunks; ++c) issue_chunk(c);
            }
            {
                const int chunks = k / 8;  // 16-byte chunks per row
                for (int e = p.m * chunks + tid; e < MB * chunks; e += gemv_warps * 32)
                    *reinterpret_cast<uint4 *>(sm.a + (size_t)(e / chunks) * k + 8 * (e % chunks)) =
                        make_uint4(0u, 0u, 0u, 0u);
            }
            // The GEMV warps only (named barrier 1; the warm warp has left).
            asm volatile("bar.sync 1, %0;" ::"r"(gemv_warps * 32) : "memory");
            failed = !mbar_wait_bounded(smem_u32(sm.a_full), 0u, MR_DEVERR_GEMV_TIMEOUT);
        }

        for (int g = warm ? 0 : cw; g < ng && !failed; g += p.CWG) {
            const int col0 = c_begin + g * CG;
            const int ncol = min(CG, c_end - col0);
            if (!run_group<MB, CG, CG, FUSED>(p, sm, g, ncol, col0, slice, lane, q_begin,
                                               warm ? min(q_end, q_begin + kQStep) : q_end, chunk_groups, warm)) {
                failed = true;
                break;
            }
            if (warm) break;
            // Refill the slot with group g + S once every slice has released
            // it.  The whole warp waits (a lone lane in try_wait beside
            // warp-mates suspended on another barrier can stall for the
            // suspend time limit); lane 0 then issues the copies.
            if (slice == 0 && g + p.S < ng) {
                const int slot = g % p.S;
                const uint32_t par = (uint32_t)(g / p.S) & 1u;
                if (!mbar_wait_bounded(smem_u32(&sm.empty[slot]), par, MR_DEVERR_GEMV_TIMEOUT)) {
                    failed = true;
                    break;
                }
                if (lane == 0) issue_group(g + p.S);
                __syncwarp();
            }
        }

        if (p.KW > 1) {
            // Sum the k-slices of every output in slice order and store C;
            // one barrier for the CTA instead of one handshake per group.
            __syncwarp();
            // Named barrier 2 over the GEMV warps: each of them gets here
            // (a failed wait only ends its group loop), so it cannot hang.
            if (!warm) asm volatile("bar.sync 2, %0;" ::"r"(gemv_warps * 32) : "memory");
            constexpr int VCG = MB * CG;
            for (int e = warm ? lane : tid; e < ng * VCG; e += gemv_warps * 32) {
                const int g = e / VCG, rem = e % VCG;
                const int r = rem / CG, col = c_begin + g * CG + rem % CG;
                if (r < p.m && col < c_end) {
                    const float *src = sm.red + (size_t)g * p.KW * VCG + rem;
                    float acc = src[0];
                    for (int sl = 1; sl < p.KW; ++sl) acc = __fadd_rn(acc, src[(size_t)sl * VCG]);
                    if (!warm) store_logit<FUSED>(p, r, col, gate_out(p, acc));
                }
            }
        }
    }
    // The warm warp goes on to warm the fused router's selection where this
    // CTA selects a row.
    if (warm_warp && !(FUSED && (int)blockIdx.x < p.m)) return;

    if constexpr (FUSED) {
        // Router top-k in the same launch, with no fence, counter or barrier
        // across CTAs: CTA b selects rows b, b + G, ... with one warp per row.
        // The warp polls the row's tagged words (GPU-scope relaxed loads,
        // bounded) until every one carries the flag, which it does once the
        // CTA that owns its column has stored it; it then selects the top-k
        // under the router's total order, writes idx / val, and zeroes the
        // row's words for the next call (the next kernel on the stream starts
        // storing only after this one has completed).  Only the <= m CTAs
        // that select wait, each after storing its own columns, so the other
        // CTAs always run to completion.
        // The warm warp runs the selection once on synthetic words.
        const int nwarps = gemv_warps;
        // 64 keys of 16-byte aligned scratch per warp after the k-slice partials.
        const uintptr_t tk0 = reinterpret_cast<uintptr_t>(sm.red + red_floats(p.KW, ng_max_of(p.n, p.G, CG), MB, CG));
        uint64_t *tk = reinterpret_cast<uint64_t *>((tk0 + 15u) & ~(uintptr_t)15u) + warp * 64;
        for (int r = warm_warp ? 0 : (int)blockIdx.x + warp * p.G; r < p.m; r += nwarps * p.G) {
            uint64_t *row = p.tags + (int64_t)r * p.n;
            uint64_t best = 0ull;
            if (!tagged_topk<MR_FUSED_P>(row, p.n, p.topk, lane, tk, best, warm_warp)) {
                if (lane == 0) record_error(MR_DEVERR_GEMV_TIMEOUT);
                return;
            }
            if (warm_warp) return;
            if (lane < p.topk) {
                const uint32_t j = topk::key_index(best);
                p.idx[(int64_t)r * p.ldo + lane] = (int32_t)j;
                if (p.val) {
                    bool exact;
                    const float v = topk::key_value(best, exact);
                    p.val[(int64_t)r * p.ldo + lane] = exact ? v : __uint_as_float((uint32_t)ld_relaxed_u64(row + j));
                }
            }
            __syncwarp();
            for (int j = lane; j < p.n; j += 32) row[j] = 0ull;
        }
    }
}

// ---------------------------------------------------------------- host side

using KernelFn = void (*)(const Params);

// Columns per group (one ring slot holds one group): at most 64 fp32
// accumulators per lane (MB x CG), and slots of about 20 KB for long rows, so
// that a CTA's whole weight block can be in flight at once (8 columns of a
// 2560-element row would make 40 KB slots and force slot refills).
#ifndef MR_GEMV_CG8_MAX_K
#define MR_GEMV_CG8_MAX_K 1536
#endif
inline int col_group_rt(int MB, int k) { return (MB <= 8 && k <= MR_GEMV_CG8_MAX_K) ? 8 : 4; }

template <bool FUSED>
KernelFn kernel_for_mb(int MB, int CG) {
    switch (MB) {
        case 1:  // the fused router has no one-row bucket (see row_bucket)
            if constexpr (!FUSED) return CG == 8 ? gemv_kernel<1, 8, false> : gemv_kernel<1, 4, false>;
            return nullptr;
        case 2: return CG == 8 ? gemv_kernel<2, 8, FUSED> : gemv_kernel<2, 4, FUSED>;
        case 4: return CG == 8 ? gemv_kernel<4, 8, FUSED> : gemv_kernel<4, 4, FUSED>;
        case 8: return CG == 8 ? gemv_kernel<8, 8, FUSED> : gemv_kernel<8, 4, FUSED>;
        default: return gemv_kernel<16, 4, FUSED>;
    }
}

KernelFn kernel_for(int MB, int CG, bool fused) {
    return fused ? kernel_for_mb<true>(MB, CG) : kernel_for_mb<false>(MB, CG);
}

// Row bucket of a call: the kernel instance for the smallest bucket that
// holds m rows.  The fused router runs one row in the 2-row kernel: in a
// sequence of router windows (m = 1, 2, 4, 8, 16) a one-row fused kernel made
// the sequence slower (1.06 against 1.02 us a row), while the plain GEMV at
// m = 1 is 8-11% faster with its one-row kernel.
int row_bucket(int m, bool fused) {
    return (m == 1 && !fused) ? 1 : m <= 2 ? 2 : m <= 4 ? 4 : m <= 8 ? 8 : 16;
}

std::mutex g_attr_mutex;
bool g_attr_done[64] = {};

cudaError_t ensure_attributes(int device) {
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    if (device >= 0 && device < 64 && g_attr_done[device]) return cudaSuccess;
    const int optin = mr_host::max_smem_optin();
    const int mbs[] = {1, 2, 4, 8, 16};
    for (int mb : mbs)
        for (int cg = 4; cg <= 8; cg += 4)
            for (int fused = 0; fused < 2; ++fused) {
                const KernelFn fn = kernel_for(mb, cg, fused != 0);
                if (!fn) continue;
                cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
                if (e != cudaSuccess) return e;
        }
    if (device >= 0 && device < 64) g_attr_done[device] = true;
    return cudaSuccess;
}

// Whether one more warp per CTA (the warm warp) keeps the CTAs per SM the
// launch relies on: as many as without it, or at least two (this launch's CTA
// beside the next launch's, or the two CTAs per SM of a split plan).  Asked of
// the occupancy calculator once per (device, kernel, warps, shared memory).
bool warm_warp_fits(KernelFn fn, int gemv_warps, size_t smem) {
    if (gemv_warps >= kWarpsMax) return false;
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess) return false;
    static std::mutex mu;
    static std::map<std::tuple<int, const void *, int, size_t>, bool> cache;
    const auto key = std::make_tuple(device, reinterpret_cast<const void *>(fn), gemv_warps, smem);
    std::lock_guard<std::mutex> lock(mu);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int without = 0, with = 0;
    bool fits = false;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&without, fn, gemv_warps * 32, smem) == cudaSuccess &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&with, fn, (gemv_warps + 1) * 32, smem) == cudaSuccess)
        fits = with >= 1 && with >= std::min(without, 2);
    cache[key] = fits;
    return fits;
}

}  // namespace gemv
}  // namespace mr

namespace mr {
namespace gemv {

struct Plan {
    int MB, CG, KW, G, CWG, S;
    uint32_t a_bytes, slot_bytes;
    size_t smem;
};

// Launch plan for (m, n, k) on a device with `sms` SMs and `optin` bytes of
// opt-in shared memory per block.  Ring invariant: either every column group
// of a CTA has its own slot (S >= groups, no refills), or S is a multiple of
// CWG so that slot s is only ever consumed by column warp s % CWG, which waits
// for the slot's uses strictly in order (a parity wait is then never more
// than one phase ahead of the barrier).
mr_status make_plan(int m, int n, int k, uint32_t flags, int sms, int optin, Plan &pl, bool fused = false) {
    if (m < 1 || n < 1 || k < 8 || sms < 1 || optin < 1) return MR_ERR_INVALID_ARG;
    if (k % 8 != 0) return MR_ERR_MISALIGNED;
    if (m > kMaxRows) return MR_ERR_UNSUPPORTED;
    pl.MB = row_bucket(m, fused);
    pl.CG = col_group_rt(pl.MB, k);
    pl.KW = k_warps(k);
    pl.G = std::min(sms, n);
    constexpr size_t kPdlBudget = 110 * 1024;  // shared memory per CTA for two CTAs per SM
    int warps_cap = warps_max(pl.MB, pl.CG);
    bool split = false;
    if ((flags & MR_GEMV_PDL) && pl.MB <= 4 && n >= 2 * sms &&
        (size_t)((n + sms - 1) / sms) * k * 2 + (size_t)pl.MB * k * 2 > kPdlBudget) {
        // A weight block too large for two CTAs per SM (the 31 MB sweep
        // weight): two CTAs per SM each take half of it through a ring within
        // the co-residency budget, so that when one exits the next call's CTA
        // starts streaming in its place (3-4% faster at m <= 4; with 8 or 16
        // rows A leaves too little room for the ring, and one CTA per SM with
        // all of the shared memory is faster).
        pl.G = std::min(2 * sms, n);
        warps_cap = 8;
        split = true;
    }
    const int ng_max = ng_max_of(n, pl.G, pl.CG);
    const int cwg0 = std::max(1, std::min(ng_max, std::max(1, warps_cap / pl.KW)));
    pl.a_bytes = (uint32_t)(((size_t)pl.MB * k * 2 + 127) / 128 * 128);
    pl.slot_bytes = (uint32_t)pl.CG * (uint32_t)k * 2u;
    const size_t red_bytes = red_floats(pl.KW, ng_max, pl.MB, pl.CG) * sizeof(float);
    const size_t topk_bytes = fused ? (size_t)warps_max(pl.MB, pl.CG) * 64 * 8 + 16 : 0;
    const size_t fixed = topk_bytes + pl.a_bytes + 24 * (size_t)ng_max + 48 + red_bytes + 64;
    const size_t budget = (flags & MR_GEMV_PDL) ? std::min<size_t>(kPdlBudget, (size_t)optin) : (size_t)optin;
    auto slots_for = [&](size_t b) -> int {
        if (b <= fixed) return 0;
        return (int)std::min<size_t>((size_t)ng_max, (b - fixed) / pl.slot_bytes);
    };
    int s_max = slots_for(budget);
    if (s_max < 1) s_max = slots_for((size_t)optin);
    if (s_max < 1) return MR_ERR_UNSUPPORTED;
    if (s_max < ng_max && budget < (size_t)optin && !split) {
        // The block does not fit the co-residency budget, so slots would be
        // refilled (a second DRAM round trip per refill).  Streaming depth
        // matters more than overlapping the next launch: take the full shared
        // memory.
        s_max = std::max(s_max, slots_for((size_t)optin));
    }
    if (s_max >= ng_max) {
        pl.S = ng_max;
        pl.CWG = cwg0;
    } else {
        // Each consumer warp gets at least two slots when the budget allows.
        pl.CWG = std::max(1, std::min(cwg0, s_max / 2));
        pl.S = (s_max / pl.CWG) * pl.CWG;
    }
    pl.smem = topk_bytes + pl.a_bytes + (size_t)pl.S * pl.slot_bytes + 24 * (size_t)pl.S + 48 + red_bytes;
    if (pl.smem > (size_t)optin) return MR_ERR_UNSUPPORTED;
    return MR_OK;
}

}  // namespace gemv
}  // namespace mr

extern "C" mr_status mrgemv_bf16_plan(int32_t m, int32_t n, int32_t k, uint32_t flags, int32_t sm_count,
                                      int32_t smem_optin, int32_t *out) {
    if (!out) return MR_ERR_INVALID_ARG;
    if (flags & ~(MR_GEMV_PDL | MR_GEMV_SIGMOID)) return MR_ERR_INVALID_ARG;
    mr::gemv::Plan pl;
    const mr_status st = mr::gemv::make_plan(m, n, k, flags, sm_count, smem_optin, pl);
    if (st != MR_OK) return st;
    out[0] = pl.G;
    out[1] = pl.KW * pl.CWG * 32;
    out[2] = (int32_t)pl.smem;
    out[3] = pl.S;
    out[4] = pl.KW;
    out[5] = pl.CWG;
    out[6] = pl.MB;
    out[7] = pl.CG;
    return MR_OK;
}

namespace mr {
namespace gemv {

struct FusedArgs {
    int topk;
    int32_t *idx;
    float *val;
    int64_t ldo;
    uint64_t *tags;
};

// Validate and plan a launch without touching the device or any stream:
// every argument error is found here, before anything is enqueued.  `fused`
// adds the router top-k of every row.
mr_status prepare(const void *A, int64_t lda, const void *Wt, int64_t ldw, float *C, int64_t ldc, int32_t m,
                  int32_t n, int32_t k, uint32_t flags, const FusedArgs *fused, Params &p, Plan &pl) {
    if (!A || !Wt || (!C && !fused)) return MR_ERR_INVALID_ARG;
    if (m < 1 || n < 1 || k < 1) return MR_ERR_INVALID_ARG;
    if (lda < k || ldw < k || ldc < n) return MR_ERR_INVALID_ARG;
    if (flags & ~(MR_GEMV_PDL | MR_GEMV_SIGMOID)) return MR_ERR_INVALID_ARG;
    if (fused && (flags & MR_GEMV_SIGMOID)) return MR_ERR_INVALID_ARG;
    if (k % 8 != 0 || lda % 8 != 0 || ldw % 8 != 0) return MR_ERR_MISALIGNED;
    if (((uintptr_t)A & 15u) || ((uintptr_t)Wt & 15u) || ((uintptr_t)C & 3u)) return MR_ERR_MISALIGNED;
    if (m > kMaxRows) return MR_ERR_UNSUPPORTED;

    const int sms = mr_host::sm_count();
    const int optin = mr_host::max_smem_optin();
    if (sms <= 0 || optin <= 0) return MR_ERR_CUDA;
    const mr_status st = make_plan(m, n, k, flags, sms, optin, pl, fused != nullptr);
    if (st != MR_OK) return st;

    p = Params{};
    p.A = static_cast<const uint16_t *>(A);
    p.lda = lda;
    p.Wt = static_cast<const uint16_t *>(Wt);
    p.ldw = ldw;
    p.C = C;
    p.ldc = ldc;
    p.m = m;
    p.n = n;
    p.k = k;
    p.G = pl.G;
    p.KW = pl.KW;
    p.CWG = pl.CWG;
    p.S = pl.S;
    p.a_bytes = pl.a_bytes;
    p.slot_bytes = pl.slot_bytes;
    p.sigmoid = (flags & MR_GEMV_SIGMOID) ? 1 : 0;
    if (fused) {
        p.topk = fused->topk;
        p.idx = fused->idx;
        p.val = fused->val;
        p.ldo = fused->ldo;
        p.tags = fused->tags;
    }
    return MR_OK;
}

// Launch a prepared plan on `stream`.
mr_status enqueue(const Params &p, const Plan &pl, uint32_t flags, bool fused, void *stream) {
    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) return mr_host::cuda_status(e);
    e = ensure_attributes(device);
    if (e != cudaSuccess) return mr_host::cuda_status(e);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.G);
    // One warm warp beside the GEMV warps when the SM has room for it.
    const KernelFn fn = kernel_for(pl.MB, pl.CG, fused);
    if (!fn) return MR_ERR_UNSUPPORTED;
    const int warps = p.KW * p.CWG + (warm_warp_fits(fn, p.KW * p.CWG, pl.smem) ? 1 : 0);
    cfg.blockDim = dim3((unsigned)(warps * 32));
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (flags & MR_GEMV_PDL) ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, fn, p);
    return mr_host::cuda_status(e);
}

mr_status launch(const void *A, int64_t lda, const void *Wt, int64_t ldw, float *C, int64_t ldc, int32_t m,
                 int32_t n, int32_t k, uint32_t flags, void *stream, const FusedArgs *fused) {
    Params p;
    Plan pl;
    const mr_status st = prepare(A, lda, Wt, ldw, C, ldc, m, n, k, flags, fused, p, pl);
    if (st != MR_OK) return st;
    return enqueue(p, pl, flags, fused != nullptr, stream);
}

// The fused router's own checks (top-k arguments and workspace), then the
// GEMV's; nothing is enqueued.  On success p and pl describe the launch.
mr_status prepare_router(const void *A, int64_t lda, const void *Wt, int64_t ldw, float *logits, int64_t ldl,
                         int32_t m, int32_t n, int32_t k, int32_t topk, int32_t *idx, float *val, int64_t ldo,
                         void *workspace, size_t workspace_bytes, uint32_t flags, bool two_launch, Params &p,
                         Plan &pl);

}  // namespace gemv
}  // namespace mr

extern "C" mr_status mrgemv_bf16_ex(const void *A, int64_t lda, const void *Wt, int64_t ldw,
                                    float *C, int64_t ldc, int32_t m, int32_t n, int32_t k,
                                    uint32_t flags, void *stream) {
    return mr::gemv::launch(A, lda, Wt, ldw, C, ldc, m, n, k, flags, stream, nullptr);
}

// Workspace layout: a reserved head block, the tag array (m x n words) at
// offset MR_ROUTER_TICKET_BYTES, and -- when the caller passes no logits --
// the two-launch form's fp32 logits in the last m * n * 4 bytes (rounded down
// to 256), so that calls of any m * n up to the size the workspace was made
// for never put logits where another call's tags are.
namespace {
size_t align256(size_t b) { return (b + 255u) & ~(size_t)255u; }
}  // namespace

extern "C" size_t router_gemv_topk_workspace_bytes(int32_t m, int32_t n, int32_t logits_provided) {
    if (m < 1 || n < 1) return 0;
    const size_t mn = (size_t)m * (size_t)n;
    return MR_ROUTER_TICKET_BYTES + align256(mn * 8u) + (logits_provided ? 0 : align256(mn * sizeof(float)));
}

namespace mr {
namespace gemv {

mr_status prepare_router(const void *A, int64_t lda, const void *Wt, int64_t ldw, float *logits, int64_t ldl,
                         int32_t m, int32_t n, int32_t k, int32_t topk, int32_t *idx, float *val, int64_t ldo,
                         void *workspace, size_t workspace_bytes, uint32_t flags, bool two_launch, Params &p,
                         Plan &pl) {
    if (!idx || !workspace) return MR_ERR_INVALID_ARG;
    if (m < 1 || n < 1 || topk < 1 || topk > n || ldo < topk) return MR_ERR_INVALID_ARG;
    if (topk > 32) return MR_ERR_UNSUPPORTED;
    if (((uintptr_t)workspace & 255u) || ((uintptr_t)idx & 3u) || ((uintptr_t)val & 3u)) return MR_ERR_MISALIGNED;
    if (workspace_bytes < router_gemv_topk_workspace_bytes(m, n, logits != nullptr)) return MR_ERR_INVALID_ARG;
    float *C = logits;
    int64_t ldc = ldl;
    if (!C) {
        const size_t off = (workspace_bytes - (size_t)m * (size_t)n * sizeof(float)) & ~(size_t)255u;
        C = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + off);
        ldc = n;
    }
    uint64_t *tags = reinterpret_cast<uint64_t *>(static_cast<uint8_t *>(workspace) + MR_ROUTER_TICKET_BYTES);
    const FusedArgs fa = {topk, idx, val, ldo, tags};
    const mr_status st = prepare(A, lda, Wt, ldw, C, ldc, m, n, k, flags, &fa, p, pl);
    // The fused form stores the workspace logits only as tagged words.
    if (st == MR_OK && !logits && !two_launch) p.C = nullptr;
    return st;
}

}  // namespace gemv
}  // namespace mr

namespace mr {
namespace gemv {

// The fused launch, or (MR_ROUTER_TWO_LAUNCH) the GEMV kernel then the top-k
// kernel on the same logits; every argument is checked before either.
mr_status launch_router(const Params &p, const Plan &pl, uint32_t flags, void *stream) {
    const uint32_t gemv_flags = flags & ~MR_ROUTER_TWO_LAUNCH;
    if (!(flags & MR_ROUTER_TWO_LAUNCH)) return enqueue(p, pl, gemv_flags, true, stream);
    const mr_status st = enqueue(p, pl, gemv_flags, false, stream);
    if (st != MR_OK) return st;
    return router_topk_ex(p.C, p.ldc, p.m, p.n, p.topk, p.idx, p.val, p.ldo, 0, stream);
}

}  // namespace gemv
}  // namespace mr

extern "C" mr_status router_gemv_topk(const void *A, int64_t lda, const void *Wt, int64_t ldw, float *logits,
                                      int64_t ldl, int32_t m, int32_t n, int32_t k, int32_t topk, int32_t *idx,
                                      float *val, int64_t ldo, void *workspace, size_t workspace_bytes,
                                      uint32_t flags, void *stream) {
    if (flags & ~(MR_GEMV_PDL | MR_ROUTER_TWO_LAUNCH)) return MR_ERR_INVALID_ARG;
    mr::gemv::Params p;
    mr::gemv::Plan pl;
    const mr_status st = mr::gemv::prepare_router(A, lda, Wt, ldw, logits, ldl, m, n, k, topk, idx, val, ldo,
                                                  workspace, workspace_bytes, flags & ~MR_ROUTER_TWO_LAUNCH,
                                                  (flags & MR_ROUTER_TWO_LAUNCH) != 0, p, pl);
    if (st != MR_OK) return st;
    return mr::gemv::launch_router(p, pl, flags, stream);
}

extern "C" mr_status mrgemv_bf16(const void *A, int64_t lda, const void *Wt, int64_t ldw, float *C,
                                 int64_t ldc, int32_t m, int32_t n, int32_t k, void *stream) {
    return mrgemv_bf16_ex(A, lda, Wt, ldw, C, ldc, m, n, k, 0u, stream);
}

// ---------------------------------------------------------------------------
// router_gemv_topk_noalloc: router_gemv_topk for callers that cannot provide a
// workspace because they cannot allocate device memory -- for example a host
// whose device memory is all owned by its own pool and accounting, or a
// plug-in that is not allowed to call cudaMalloc.  The scratch (ticket block,
// then the logits when the caller passes none) is one file-scope device array
// of fixed size that every GPU loading this library holds until the process
// exits.
// ---------------------------------------------------------------------------

namespace mr {
namespace gemv {

constexpr size_t kNoAllocScratchBytes = 256u * 1024u;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void *g_scratch_ptr[64] = {};

// The array's device address, looked up once per device with that device
// current.  (In host code `g_noalloc_scratch` names a host-side stand-in, not
// device memory, so it must never be passed to a kernel directly.)
mr_status noalloc_scratch(void **out) {
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= 64) return MR_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[device]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MR_ERR_CUDA;
        g_scratch_ptr[device] = ptr;
    }
    *out = g_scratch_ptr[device];
    return MR_OK;
}

}  // namespace gemv
}  // namespace mr

// With no logits passed, m * n values take 12 bytes each (a tagged word and
// an fp32 logit); a multiple of 64 keeps both arrays whole 256-byte blocks.
extern "C" size_t router_gemv_topk_noalloc_max_logits(void) {
    return (mr::gemv::kNoAllocScratchBytes - MR_ROUTER_TICKET_BYTES) / 12u / 64u * 64u;
}

extern "C" mr_status router_gemv_topk_noalloc(const void *A, int64_t lda, const void *Wt, int64_t ldw,
                                              float *logits, int64_t ldl, int32_t m, int32_t n, int32_t k,
                                              int32_t topk, int32_t *idx, float *val, int64_t ldo, uint32_t flags,
                                              void *stream) {
    if (m < 1 || n < 1) return MR_ERR_INVALID_ARG;
    if (router_gemv_topk_workspace_bytes(m, n, logits != nullptr) > mr::gemv::kNoAllocScratchBytes)
        return MR_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    mr_status st = mr::gemv::noalloc_scratch(&scratch);
    if (st != MR_OK) return st;
    // Every argument is checked before anything is put on the stream.
    if (flags & ~(MR_GEMV_PDL | MR_ROUTER_TWO_LAUNCH)) return MR_ERR_INVALID_ARG;
    mr::gemv::Params p;
    mr::gemv::Plan pl;
    const bool two_launch = (flags & MR_ROUTER_TWO_LAUNCH) != 0;
    st = mr::gemv::prepare_router(A, lda, Wt, ldw, logits, ldl, m, n, k, topk, idx, val, ldo, scratch,
                                  mr::gemv::kNoAllocScratchBytes, flags & ~MR_ROUTER_TWO_LAUNCH, two_launch, p, pl);
    if (st != MR_OK) return st;
    // The array keeps whatever the last call left (a call that failed on the
    // device may leave tagged words behind); the tags must start at zero.
    if (!two_launch && cudaMemsetAsync(p.tags, 0, (size_t)m * (size_t)n * 8u, static_cast<cudaStream_t>(stream)) !=
                           cudaSuccess)
        return MR_ERR_CUDA;
    return mr::gemv::launch_router(p, pl, flags, stream);
}
