// gemm_f16: C[M,N] = A[M,K] . Wt[N,K]^T on the sm_100a tensor cores.
//
// The prompt-chunk GEMM of the "opus r35 track A" audit (section 2, gemm_f16
// tiles): a family of tile shapes, a selector that is aware of padded tail
// tiles (M % 128 in 1..64), and outputs that are bitwise identical whatever
// tile is chosen.  Rebuilt for B200:
//
//  * persistent CTAs (one per SM) walk the 128 x BN output tiles; 7 warps:
//    warps 0 and 6 issue TMA loads, warp 1 owns the tensor memory and issues
//    tcgen05.mma from one elected thread, warps 2..5 drain the accumulator
//    (tcgen05.ld) and store the tile.  Two accumulator buffers in tensor
//    memory let one tile's epilogue run under the next tile's MMAs;
//  * A and Wt k-blocks of 64 K-elements (one 128-byte swizzle atom per row)
//    are loaded by TMA, each CTA for itself, into a ring of shared-memory stages,
//    full/empty mbarriers between the producers and the MMA thread.  Each
//    ring step (barrier wait, TMA or MMA issue, commit) costs a few hundred
//    cycles of latency: two producer warps alternate stages, and the tiles
//    up to BN = 128, whose MMAs are short, put two k-blocks in a stage;
//  * tcgen05.mma.cta_group::1.kind::f16 with M = 128, N = BN, K = 16,
//    accumulating fp32 in tensor memory.  Every tile runs the same sequence of
//    K steps (16 at a time, ascending, zero padding past K), with no split-K
//    or stream-K, so an output element's bits depend on its row of A, its row
//    of Wt and K only;
//  * epilogue: fp32 -> f16 / bf16 with round-to-nearest-even (CUDA's
//    conversion intrinsics), or fp32, stored with the row / column tails masked.
//  * every wait is bounded; a wait that runs out sets MR_DEVERR_GEMM_TIMEOUT
//    and the CTA still frees its tensor memory before it exits.
#include "common.cuh"

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

namespace mr {
namespace gemm {

constexpr int BK = 64;           // K elements per k-block (128 bytes of 16-bit data)
constexpr int kMaxBM = 128;      // rows per tile (MMA M): 128, or 64 for tail-heavy M
__host__ __device__ constexpr uint32_t a_bytes_for(int bm) { return (uint32_t)bm * BK * 2; }

// Threads of a CTA: warps 0 and 6 producers (alternate ring stages), warp 1
// MMA issue, warps 2-5 epilogue.
constexpr int kThreads = 224;
constexpr int kProducers = 2;

struct TileDesc {
    int bm;         // rows per tile: 128, or 64 (tcgen05 M = 64: half of each lane quarter)
    int bn;
    int stages;     // k-block slots of shared memory
    int acc_cols;   // tensor-memory columns per accumulator buffer (power of two >= bn)
    int kpb;        // k-blocks per ring stage (one barrier wait and one commit each)
    const char *name;
    bool pair = false;  // two CTAs per tile (cta_group::2): bm = 256, 128 rows per CTA
};

// Tiles up to BN = 128 take two k-blocks per ring stage: their MMAs are short
// (the operand reads from shared memory bound them), so one barrier round trip
// and one commit per k-block would leave the tensor pipe idle between stages.
// The wider tiles keep one, since two 40-48 KB k-blocks per stage would leave
// only two stages in flight.
constexpr TileDesc kTiles[] = {
    {128, 32, 8, 32, 2, "128x32"},   {128, 64, 8, 64, 2, "128x64"},   {128, 96, 7, 128, 2, "128x96"},
    {128, 128, 6, 128, 2, "128x128"}, {128, 192, 5, 256, 1, "128x192"}, {128, 256, 4, 256, 1, "128x256"},
    {64, 128, 8, 128, 2, "64x128"},   {64, 256, 5, 256, 1, "64x256"},
    {256, 256, 7, 256, 1, "256x256", true},
    {256, 128, 9, 128, 1, "256x128", true},
    {64, 32, 12, 32, 2, "64x32"},     {64, 64, 12, 64, 2, "64x64"},
};
constexpr int kNumTiles = sizeof(kTiles) / sizeof(kTiles[0]);

// The barriers (2 per k-block slot, 4 for the accumulators) and the tensor
// memory address take the 256 bytes after the ring: at most 13 slots.
__host__ __device__ constexpr uint32_t smem_bytes_for(int bm, int bn, int stages) {
    return (uint32_t)stages * (a_bytes_for(bm) + (uint32_t)bn * BK * 2) + 1024 /*align*/ + 256 /*barriers*/;
}

// ---- tcgen05 / TMA PTX wrappers --------------------------------------------

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Shared-memory matrix descriptor, K-major operand, 128-byte swizzle:
// start address >> 4 (bits 0-13), leading byte offset (unused for swizzled
// K-major, 16 B), stride byte offset = 1024 B between 8-row swizzle atoms
// (bits 32-45), descriptor version 1 (bits 46-47), layout 128B swizzle = 2
// (bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(16u >> 4) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// One lane of a converged warp (the one elect.sync picks); the MMA issue
// branch is taken by exactly one thread.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// ---- CTA-pair (cta_group::2) helpers -------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of the same offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}

// Every thread of both CTAs: arrive (release) and wait (acquire) on the cluster barrier.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// One MMA for the pair: M = 256 (128 rows of A from each CTA's shared
// memory), N columns (N / 2 rows of Wt from each CTA), K = 16; the
// accumulator's rows 128v..128v+127 land in CTA v's tensor memory.
__device__ __forceinline__ void mma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on the barrier at this offset in both CTAs of the pair once every
// tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    const uint16_t both = 0x3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"(both)
        : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on a
// barrier of either CTA of the pair (cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                                 uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar_cluster)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- epilogue stores -----------------------------------------------------

template <int OUT>
__device__ __forceinline__ void store16(void *C, int64_t ldc, int row, int col, int N, const uint32_t (&r)[16]) {
    if constexpr (OUT == MR_F32) {
        float *dst = static_cast<float *>(C) + (int64_t)row * ldc + col;
        if (col + 16 <= N) {
#pragma unroll
            for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<uint4 *>(dst + i) = make_uint4(r[i], r[i + 1], r[i + 2], r[i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (col + i < N) dst[i] = __uint_as_float(r[i]);
        }
    } else {
        uint32_t h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float lo = __uint_as_float(r[2 * i]), hi = __uint_as_float(r[2 * i + 1]);
            if constexpr (OUT == MR_F16) {
                const __half2 v = __floats2half2_rn(lo, hi);
                h[i] = *reinterpret_cast<const uint32_t *>(&v);
            } else {
                const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
                h[i] = *reinterpret_cast<const uint32_t *>(&v);
            }
        }
        uint16_t *dst = static_cast<uint16_t *>(C) + (int64_t)row * ldc + col;
        if (col + 16 <= N) {
            *reinterpret_cast<uint4 *>(dst) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4 *>(dst + 8) = make_uint4(h[4], h[5], h[6], h[7]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (col + i < N) dst[i] = (uint16_t)((i & 1) ? (h[i >> 1] >> 16) : (h[i >> 1] & 0xFFFFu));
        }
    }
}

// ---- the kernel --------------------------------------------------------------

// Up to MAXG weight matrices ("groups") that share A, each with its own
// tensor map and output.  A tile covers either BN columns of one group
// (P == 1, tn_per_group tiles per group) or P whole groups of N columns each
// (P > 1, BN == P * N, N a multiple of 16).
template <int MAXG>
struct GemmArgs {
    CUtensorMap tmA;
    CUtensorMap tmB[MAXG];
    void *C[MAXG];
    int64_t ldc;
    int M, N, K;
    int G, P, tn_per_group, ntn;
    int raster;     // 0: N-slots fastest; R > 0: bands of R N-slots run down all row tiles
    uint32_t idesc;
};

// Tile t of the persistent walk -> (row tile, N-slot).  raster == 0 walks the
// N-slots of a row tile before the next row tile; raster R > 0 walks bands of
// R N-slots down every row tile (the column-band order of the audit's SLC
// swizzle study).  Only the order changes, never a tile's arithmetic.
__device__ __forceinline__ void tile_coords(int t, int ntm, int ntn, int raster, int &mt, int &nt) {
    if (raster <= 0) {
        mt = t / ntn;
        nt = t % ntn;
        return;
    }
    const int band = t / (ntm * raster);
    const int n0 = band * raster;
    const int width = min(raster, ntn - n0);
    const int r = t - band * ntm * raster;
    mt = r / width;
    nt = n0 + r % width;
}

template <int BM, int BN, int STAGES, int ACC_COLS, int KPB, int OUT, int MAXG>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmArgs<MAXG> args) {
    constexpr uint32_t kABytes = a_bytes_for(BM);
    const CUtensorMap &tmA = args.tmA;
    const int M = args.M, N = args.N, K = args.K, G = args.G, P = args.P;
    const int64_t ldc = args.ldc;
    const uint32_t idesc = args.idesc;
    // Persistent: CTA b takes tiles b, b + gridDim.x, ... (N-tile slots fastest).
    // Two accumulator buffers of ACC_COLS tensor-memory columns each: the
    // epilogue drains tile i from one while the MMAs of tile i+1 fill the other.
    constexpr uint32_t kBBytes = (uint32_t)BN * BK * 2;
    constexpr uint32_t kTmemCols = 2 * ACC_COLS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + STAGES * kABytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(gbase + STAGES * (kABytes + kBBytes));
    // Ring of NST stages of KPB k-blocks each (k-block slot j of stage s is
    // slot s * KPB + j of the A and B regions).  Producer p issues the stages
    // it with it % kProducers == p.  Its previous stage was it - kProducers,
    // whose wait saw stage it - kProducers - NST released; with NST >=
    // kProducers that covers stage it - 2 NST, so a wait on a slot is never
    // more than one phase ahead of the barrier.
    constexpr int NST = STAGES / KPB;
    static_assert(NST >= kProducers, "ring too short for the producer warps");
    static_assert((2 * STAGES + 4) * 8 + 4 <= 256, "barriers exceed their 256 bytes");
    static_assert(smem_bytes_for(BM, BN, STAGES) <= 232448, "ring exceeds the opt-in shared memory");
    uint64_t *full = bars;                    // [NST] TMA -> MMA
    uint64_t *empty = bars + STAGES;          // [NST] MMA -> TMA
    uint64_t *acc_full = bars + 2 * STAGES;   // [2] MMA -> epilogue
    uint64_t *acc_empty = bars + 2 * STAGES + 2;  // [2] epilogue -> MMA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ntn = args.ntn;
    const int ntm = (M + BM - 1) / BM;
    const int ntiles = ntm * ntn;
    const int nkb = (K + BK - 1) / BK;
    const int nst = (nkb + KPB - 1) / KPB;   // ring stages per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&acc_full[b]), 1);
            mbar_init(smem_u32(&acc_empty[b]), 4);  // one arrival per epilogue warp
        }
        fence_mbar_init();
        prefetch_tmap(&tmA);
        if (MAXG == 1) prefetch_tmap(&args.tmB[0]);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // The producer and MMA warps run their loops as whole warps (every lane
    // waits on the same barrier) and let one lane issue: a lone lane spinning
    // in try_wait beside warp-mates parked elsewhere can stall for the
    // suspend limit.
    if (warp == 0 || warp == 6) {
        // Producers: stage `it` counts across tiles, so slots and phases
        // continue from one tile to the next.
        const uint32_t pidx = warp == 0 ? 0u : 1u;
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            int mt, slot;
            tile_coords(t, ntm, ntn, args.raster, mt, slot);
            const int m0 = mt * BM;
            // Groups of this tile and the B rows each contributes.
            const int g0 = P > 1 ? slot * P : slot / args.tn_per_group;
            const int ng = P > 1 ? min(P, G - g0) : 1;
            const int n0 = P > 1 ? 0 : (slot % args.tn_per_group) * BN;
            const uint32_t b_rows = P > 1 ? (uint32_t)N : (uint32_t)BN;
            const uint32_t kb_bytes = kABytes + (uint32_t)ng * b_rows * BK * 2;
            for (int ks = 0; ks < nst; ++ks, ++it) {
                if (it % kProducers != pidx) continue;
                const uint32_t s = it % NST;
                const uint32_t par = ((it / NST) & 1u) ^ 1u;
                const int nsub = KPB == 1 ? 1 : min(KPB, nkb - ks * KPB);
                ok = mbar_wait_bounded(smem_u32(&empty[s]), par, MR_DEVERR_GEMM_TIMEOUT);
                if (!ok) break;
                if (lane == 0) {
                    const uint32_t fb = smem_u32(&full[s]);
                    mbar_arrive_expect_tx(fb, (uint32_t)nsub * kb_bytes);
#pragma unroll
                    for (int sub = 0; sub < KPB; ++sub) {
                        if (sub >= nsub) break;
                        const int kb = ks * KPB + sub;
                        const uint32_t slot_kb = s * KPB + (uint32_t)sub;
                        tma_load_2d(sA + slot_kb * kABytes, &tmA, kb * BK, m0, fb);
                        for (int j = 0; j < ng; ++j)
                            tma_load_2d(sB + slot_kb * kBBytes + (uint32_t)j * b_rows * BK * 2, &args.tmB[g0 + j],
                                        kb * BK, n0, fb);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // Descriptors of slot 0; a slot's descriptor adds its byte offset >> 4
        // to the start-address field (shared addresses stay below 2^18).
        const uint64_t adesc0 = sw128_desc(sA), bdesc0 = sw128_desc(sB);
        // One lane issues every MMA and every commit: tcgen05.commit tracks
        // only the tcgen05 operations of the thread that issues it.
        const bool leader = elect_one();
        uint32_t it = 0, ti = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++ti) {
            const uint32_t b = ti & 1u;
            // Wait until the epilogue has drained this buffer's previous tile.
            ok = mbar_wait_bounded(smem_u32(&acc_empty[b]), ((ti >> 1) & 1u) ^ 1u, MR_DEVERR_GEMM_TIMEOUT);
            if (!ok) break;
            tc_fence_after();
            const uint32_t acc = tmem + b * ACC_COLS;
            for (int ks = 0; ks < nst; ++ks, ++it) {
                const uint32_t s = it % NST;
                const uint32_t par = (it / NST) & 1u;
                const int nsub = KPB == 1 ? 1 : min(KPB, nkb - ks * KPB);
                ok = mbar_wait_bounded(smem_u32(&full[s]), par, MR_DEVERR_GEMM_TIMEOUT);
                if (!ok) break;
                tc_fence_after();
                __syncwarp();
                if (leader) {
                    // K steps of 16 in ascending order: every tile and every
                    // stage grouping issues the same MMA sequence.
#pragma unroll
                    for (int sub = 0; sub < KPB; ++sub) {
                        if (sub >= nsub) break;
                        const uint32_t slot_kb = s * KPB + (uint32_t)sub;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint64_t ad = adesc0 + (uint64_t)((slot_kb * kABytes + kk * 32) >> 4);
                            const uint64_t bd = bdesc0 + (uint64_t)((slot_kb * kBBytes + kk * 32) >> 4);
                            mma_f16(acc, ad, bd, idesc, (ks | sub | kk) != 0 ? 1u : 0u);
                        }
                    }
                    mma_commit(smem_u32(&empty[s]));
                }
                __syncwarp();
            }
            if (ok && leader) mma_commit(smem_u32(&acc_full[b]));
            __syncwarp();
        }
    } else {
        // Epilogue warps 2..5: warp w reads tensor-memory lanes 32*(w%4) .. +31.
        const int q = warp & 3;
        uint32_t ti = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++ti) {
            const uint32_t b = ti & 1u;
            int mt, slot;
            tile_coords(t, ntm, ntn, args.raster, mt, slot);
            const int m0 = mt * BM;
            const int g0 = P > 1 ? slot * P : slot / args.tn_per_group;
            const int n0 = P > 1 ? 0 : (slot % args.tn_per_group) * BN;
            // M = 128: tensor-memory lane 32q + l holds row 32q + l of the tile.
            // M = 64: lanes 32q .. 32q + 15 hold rows 16q .. 16q + 15 (the
            // first half of each lane quarter); lanes 16..31 of the warp
            // read unused lanes and store nothing.
            const int row = BM == 128 ? m0 + 32 * q + lane : (lane < 16 ? m0 + 16 * q + lane : M);
            if (!mbar_wait_bounded(smem_u32(&acc_full[b]), (ti >> 1) & 1u, MR_DEVERR_GEMM_TIMEOUT)) break;
            tc_fence_after();
            const uint32_t acc = tmem + b * ACC_COLS + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
            for (int c = 0; c < BN / 16; ++c) {
                uint32_t r[16];
                tmem_ld16(acc + (uint32_t)(c * 16), r);
                // Column c*16 of the tile: group and column within the group.
                const int g = P > 1 ? g0 + (c * 16) / N : g0;
                const int col = P > 1 ? (c * 16) % N : n0 + c * 16;
                if (row < M && col < N && g < G) store16<OUT>(args.C[g], ldc, row, col, N, r);
            }
            // This warp's lanes of the buffer are read: let the MMAs reuse it.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---- the CTA-pair kernel: 256 x PBN tiles on two SMs (cta_group::2) --------
//
// A cluster of two CTAs computes a 256 x PBN output tile (PBN = 128 or 256)
// with one tcgen05.mma.cta_group::2 per K step of 16: CTA v loads rows
// 128v..128v+127 of the tile's A block and rows v*PBN/2 .. (v+1)*PBN/2 - 1 of
// its Wt block (columns of the output) into its own shared memory, and CTA
// v's tensor memory receives rows 128v..128v+127 of the accumulator.  At
// PBN = 256 each CTA streams 32 KB per k-block instead of the 48 KB a
// 128 x 256 tile needs; at PBN = 128, 24 KB instead of the 32 KB of a
// 128 x 128 tile with the same output per SM.  (A 256 x 64 pair measured
// 17-19 us on the one-wave chunk shapes against 13-15 us for the best tile,
// and was left out.)  The leader (rank 0)
// issues every MMA from one elected thread and waits on its own full
// barriers, which count the TMA bytes of both CTAs (the peer's loads signal
// the leader's barrier; no load is multicast); its commits arrive on the
// barriers of both CTAs.  Both CTAs' epilogue warps release an accumulator
// buffer on the leader's barrier.  The K sequence is that of every other
// tile, so the bits are too.
constexpr int kPairRows = 256;       // output rows per tile (128 per CTA)

// Ring stages of the pair kernel: k-blocks of 16 KB of A and PBN / 2 rows of
// Wt per CTA, as many as fit beside the barriers.
__host__ __device__ constexpr int pair_stages(int pbn) { return pbn >= 256 ? 7 : 9; }
__host__ __device__ constexpr uint32_t pair_smem_bytes(int pbn) {
    return (uint32_t)pair_stages(pbn) * (a_bytes_for(128) + (uint32_t)(pbn / 2) * BK * 2) + 1024 + 256;
}

template <int PBN, int OUT, int MAXG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmArgs<MAXG> args) {
    static_assert(PBN == 128 || PBN == 256, "pair tile width");
    constexpr int BMH = kPairRows / 2;                 // A rows per CTA
    constexpr int BNH = PBN / 2;                       // Wt rows per CTA
    constexpr uint32_t kAB = (uint32_t)BMH * BK * 2;   // 16 KB
    constexpr uint32_t kBB = (uint32_t)BNH * BK * 2;   // 8 or 16 KB (multiples of the 1 KB swizzle atom)
    constexpr int NST = pair_stages(PBN);
    static_assert(NST >= kProducers, "ring too short for the producer warps");
    static_assert(pair_smem_bytes(PBN) <= 232448, "pair ring exceeds the opt-in shared memory");
    static_assert((2 * NST + 4) * 8 + 4 <= 256, "barriers exceed their 256 bytes");
    constexpr uint32_t ACC_COLS = PBN;
    constexpr uint32_t kTmemCols = 2 * ACC_COLS;
    const CUtensorMap &tmA = args.tmA;
    const int M = args.M, N = args.N, K = args.K;
    const int64_t ldc = args.ldc;
    const uint32_t idesc = args.idesc;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + NST * kAB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(gbase + NST * (kAB + kBB));
    uint64_t *full = bars;                  // [NST] TMA (both CTAs) -> MMA; used in the leader
    uint64_t *empty = bars + NST;           // [NST] MMA -> this CTA's producers
    uint64_t *acc_full = bars + 2 * NST;    // [2] MMA -> this CTA's epilogue
    uint64_t *acc_empty = bars + 2 * NST + 2;  // [2] both epilogues -> MMA; used in the leader
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * NST + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ntn = args.ntn;
    const int ntm = (M + kPairRows - 1) / kPairRows;
    const int ntiles = ntm * ntn;
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
    const int nkb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int st = 0; st < NST; ++st) {
            mbar_init(smem_u32(&full[st]), 1);
            mbar_init(smem_u32(&empty[st]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&acc_full[b]), 1);
            mbar_init(smem_u32(&acc_empty[b]), 8);  // four epilogue warps in each CTA
        }
        fence_mbar_init();
        prefetch_tmap(&tmA);
        if (MAXG == 1) prefetch_tmap(&args.tmB[0]);
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 6) {
        // Producers of this CTA's halves; the leader's thread also arms the
        // leader's full barrier with the bytes of both CTAs.
        const uint32_t pidx = warp == 0 ? 0u : 1u;
        uint32_t it = 0;
        bool ok = true;
        for (int t = pair; t < ntiles && ok; t += npairs) {
            int mt, slot;
            tile_coords(t, ntm, ntn, args.raster, mt, slot);
            const int m0 = mt * kPairRows + (int)rank * BMH;
            const int g = slot / args.tn_per_group;
            const int n0 = (slot % args.tn_per_group) * PBN + (int)rank * BNH;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                if (it % kProducers != pidx) continue;
                const uint32_t st = it % NST;
                const uint32_t par = ((it / NST) & 1u) ^ 1u;
                ok = mbar_wait_bounded(smem_u32(&empty[st]), par, MR_DEVERR_GEMM_TIMEOUT);
                if (!ok) break;
                if (lane == 0) {
                    const uint32_t fb = map_to_rank(smem_u32(&full[st]), 0u);
                    if (leader) mbar_arrive_expect_tx(smem_u32(&full[st]), 2u * (kAB + kBB));
                    tma_load_2d_pair(sA + st * kAB, &tmA, kb * BK, m0, fb);
                    tma_load_2d_pair(sB + st * kBB, &args.tmB[g], kb * BK, n0, fb);
                }
                __syncwarp();
            }
        }
        // Tail: wait until the MMAs have released the last fill of every stage
        // this producer wrote, so that no commit arrives on this CTA's
        // barriers after it exits.
        for (uint32_t j = it > (uint32_t)NST ? it - NST : 0u; j < it && ok; ++j) {
            if (j % kProducers != pidx) continue;
            ok = mbar_wait_bounded(smem_u32(&empty[j % NST]), (j / NST) & 1u, MR_DEVERR_GEMM_TIMEOUT);
        }
    } else if (warp == 1) {
        if (leader) {
            const uint64_t adesc0 = sw128_desc(sA), bdesc0 = sw128_desc(sB);
            const bool issuer = elect_one();
            uint32_t it = 0, ti = 0;
            bool ok = true;
            for (int t = pair; t < ntiles && ok; t += npairs, ++ti) {
                const uint32_t b = ti & 1u;
                ok = mbar_wait_bounded(smem_u32(&acc_empty[b]), ((ti >> 1) & 1u) ^ 1u, MR_DEVERR_GEMM_TIMEOUT);
                if (!ok) break;
                tc_fence_after();
                const uint32_t acc = tmem + b * ACC_COLS;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const uint32_t st = it % NST;
                    ok = mbar_wait_bounded(smem_u32(&full[st]), (it / NST) & 1u, MR_DEVERR_GEMM_TIMEOUT);
                    if (!ok) break;
                    tc_fence_after();
                    __syncwarp();
                    if (issuer) {
                        // K steps of 16 in ascending order, as in every tile.
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint64_t ad = adesc0 + (uint64_t)((st * kAB + kk * 32) >> 4);
                            const uint64_t bd = bdesc0 + (uint64_t)((st * kBB + kk * 32) >> 4);
                            mma_f16_pair(acc, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                        mma_commit_pair(smem_u32(&empty[st]));
                    }
                    __syncwarp();
                }
                if (ok && issuer) mma_commit_pair(smem_u32(&acc_full[b]));
                __syncwarp();
            }
        }
    } else {
        // Epilogue warps 2..5 of both CTAs: warp w reads tensor-memory lanes
        // 32*(w%4) .. +31 of this CTA's half, rows 128 * rank + 32 * (w%4) ...
        const int q = warp & 3;
        uint32_t ti = 0;
        for (int t = pair; t < ntiles; t += npairs, ++ti) {
            const uint32_t b = ti & 1u;
            int mt, slot;
            tile_coords(t, ntm, ntn, args.raster, mt, slot);
            const int g = slot / args.tn_per_group;
            const int n0 = (slot % args.tn_per_group) * PBN;
            const int row = mt * kPairRows + (int)rank * BMH + 32 * q + lane;
            if (!mbar_wait_bounded(smem_u32(&acc_full[b]), (ti >> 1) & 1u, MR_DEVERR_GEMM_TIMEOUT)) break;
            tc_fence_after();
            const uint32_t acc = tmem + b * ACC_COLS + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
            for (int c = 0; c < PBN / 16; ++c) {
                uint32_t r[16];
                tmem_ld16(acc + (uint32_t)(c * 16), r);
                const int col = n0 + c * 16;
                if (row < M && col < N) store16<OUT>(args.C[g], ldc, row, col, N, r);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_u32(&acc_empty[b]), 0u));
        }
    }

    // Neither CTA frees tensor memory or exits while its pair may still use it.
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// ---- host side -------------------------------------------------------------

constexpr int kMaxGroups = 64;

template <int MAXG>
using KernelFn = void (*)(const GemmArgs<MAXG>);

template <int T, int OUT, int MAXG>
constexpr KernelFn<MAXG> kernel_of() {
    return gemm_kernel<kTiles[T].bm, kTiles[T].bn, kTiles[T].stages, kTiles[T].acc_cols, kTiles[T].kpb, OUT, MAXG>;
}

template <int OUT, int MAXG>
KernelFn<MAXG> pick_out(int t) {
    if (kTiles[t].pair)
        return kTiles[t].bn == 128 ? gemm_pair_kernel<128, OUT, MAXG> : gemm_pair_kernel<256, OUT, MAXG>;
    switch (t) {
        case 0: return kernel_of<0, OUT, MAXG>();
        case 1: return kernel_of<1, OUT, MAXG>();
        case 2: return kernel_of<2, OUT, MAXG>();
        case 3: return kernel_of<3, OUT, MAXG>();
        case 4: return kernel_of<4, OUT, MAXG>();
        case 5: return kernel_of<5, OUT, MAXG>();
        case 6: return kernel_of<6, OUT, MAXG>();
        case 10: return kernel_of<10, OUT, MAXG>();
        case 11: return kernel_of<11, OUT, MAXG>();
        default: return kernel_of<7, OUT, MAXG>();
    }
}

// Dynamic shared memory of tile t's kernel.
uint32_t tile_smem_bytes(int t) {
    const TileDesc &td = kTiles[t];
    return td.pair ? pair_smem_bytes(td.bn) : smem_bytes_for(td.bm, td.bn, td.stages);
}

// Clusters of two CTAs of the pair kernel that fit on the device at once
// (both SMs of a pair must sit in one GPC), or 0 when the query fails.
int max_pairs(int device) {
    static std::mutex m;
    static int cached[64] = {};
    std::lock_guard<std::mutex> lock(m);
    if (device < 0 || device >= 64) return 0;
    if (cached[device] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = pair_smem_bytes(256);  // the largest pair ring: one CTA per SM for all widths
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<256, MR_F16, 1>, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            return 0;
        }
        cached[device] = n;
    }
    return cached[device];
}

template <int MAXG>
KernelFn<MAXG> kernel_for(int tile, int out) {
    if (out == MR_F16) return pick_out<MR_F16, MAXG>(tile);
    if (out == MR_BF16) return pick_out<MR_BF16, MAXG>(tile);
    return pick_out<MR_F32, MAXG>(tile);
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_mutex;
bool g_attr_done[64] = {};

cudaError_t init_device(int device) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (device >= 0 && device < 64 && !g_attr_done[device]) {
        for (int t = 0; t < kNumTiles; ++t)
            for (int out = 0; out < 3; ++out) {
                const int smem = (int)tile_smem_bytes(t);
                cudaError_t e = cudaFuncSetAttribute(kernel_for<1>(t, out),
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
                if (e != cudaSuccess) return e;
                e = cudaFuncSetAttribute(kernel_for<kMaxGroups>(t, out), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
                if (e != cudaSuccess) return e;
            }
        g_attr_done[device] = true;
    }
    return cudaSuccess;
}

bool encode_operand(CUtensorMap *map, const void *ptr, int64_t rows, int64_t cols, int64_t ld, int dtype,
                    int box_rows) {
    const CUtensorMapDataType dt =
        dtype == MR_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and B
// formats (bits 7-9, 10-12: 0 = f16, 1 = bf16), both K-major (bits 15, 16 = 0),
// N >> 3 (bits 17-22), M >> 4 (bits 24-28).
uint32_t make_idesc(int in_dtype, int bm, int bn) {
    const uint32_t fmt = in_dtype == MR_BF16 ? 1u : 0u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(bm >> 4) << 24);
}

// Tile selection: estimated time = waves x k-blocks x the tile's time per
// k-block, a wave being one tile on every active SM.  The per-k-block times
// are measured: every tile timed on the 48 prompt-chunk shapes (M = 150..2048,
// N = 512..6144, K = 2560, operands from HBM) runs at a near-constant cost per
// wave, and these are those costs / 40 k-blocks.  Narrow tiles are cheap per
// wave (two k-blocks per ring stage, short MMAs) but need more waves; wide
// tiles reuse each A stage over more columns but run longer per wave.  Row
// tails count as whole tiles, so an M with a small M % 128 pays for the
// padding it creates, and a 64-row tile (half the padding, tcgen05 M = 64)
// wins where that padding costs a wave (the audit's tail-tile rule,
// restated as waves over 148 SMs); the narrow N = 96 projections favour
// spreading tiles over SMs.
// Groups packed per tile of width bn: a tile holds whole groups when N
// divides bn and is a multiple of 16 (so no 16-column chunk straddles two
// groups); otherwise 1 (a group spans ceil(N / bn) tiles).
int pack_factor(int bn, int N, int G, bool pair = false) {
    if (!pair && G > 1 && N < bn && bn % N == 0 && N % 16 == 0) return bn / N;
    return 1;
}

int64_t n_slots(int bn, int N, int G, int P) {
    return P > 1 ? (int64_t)((G + P - 1) / P) : (int64_t)G * ((N + bn - 1) / bn);
}

int select_tile_grouped(int M, int N, int K, int G, int sms, int pairs) {
    if (M < 1 || N < 1 || K < 1 || G < 1 || sms < 1) return -1;
    // ns per k-block of one tile: 128 x (32, 64, 96, 128, 192, 256), then
    // 64 x (128, 256).  The 64-row tiles measured 0.78x the 128 x 128 and
    // 0.85x the 128 x 256 per-wave cost in the same all-tiles study, and are
    // placed at those ratios.
    // The 256 x 256 pair tile runs one tile per two SMs; it measured 0.96x
    // the 128 x 256 tile's cost per wave (a wave of pairs covers the same
    // output area as a wave of 128 x 256 tiles).  The 256 x 128 pair costs
    // 0.85x the 128 x 128 tile per wave (215 ns a k-block), and the 64 x 32
    // and 64 x 64 tiles 0.91x and 0.93x the 128 x 32 tile (one-wave shapes):
    // with these the rule picks the fastest of the twelve tiles on 47 of the
    // 48 chunk shapes.
    const double kb_ns[kNumTiles] = {175.0, 193.0, 225.0, 254.0, 338.0, 438.0, 198.0, 372.0, 420.0, 215.0, 159.0, 163.0};
    const int64_t nkb = (K + BK - 1) / BK;
    int best = -1;
    double best_t = 1e300;
    for (int t = 0; t < kNumTiles; ++t) {
        const int bn = kTiles[t].bn;
        const bool pair = kTiles[t].pair;
        if (pair && pairs < 1) continue;
        // A pair tile holds one group: with several groups narrower than the
        // tile, its spare columns are work the packed one-CTA tiles avoid
        // (the 36 projections of N = 96 at M = 512: 13.1 us on 256 x 128
        // against 12.4 us on 128 x 96).
        if (pair && G > 1 && N < bn) continue;
        const int P = pack_factor(bn, N, G, pair);
        const int bm = kTiles[t].bm;
        const int64_t tiles = (int64_t)((M + bm - 1) / bm) * n_slots(bn, N, G, P);
        const int64_t slots = pair ? pairs : sms;
        const int64_t waves = (tiles + slots - 1) / slots;
        const double t_est = (double)waves * (double)nkb * kb_ns[t];
        if (t_est < best_t * 0.999) {
            best_t = t_est;
            best = t;
        }
    }
    return best;
}

int select_tile(int M, int N, int K, int sms, int pairs) { return select_tile_grouped(M, N, K, 1, sms, pairs); }

// Validate, encode the tensor maps and launch one grouped GEMM.
template <int MAXG>
mr_status launch(const void *A, int64_t lda, const void *const *Wts, int64_t ldw, void *const *Cs, int64_t ldc,
                 int32_t M, int32_t N, int32_t K, int32_t G, int32_t in_dtype, int32_t out_dtype, int32_t tile_id,
                 int32_t raster, void *stream) {
    if (!A || !Wts || !Cs) return MR_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 1 || G < 1 || G > MAXG) return MR_ERR_INVALID_ARG;
    if (lda < K || ldw < K || ldc < N) return MR_ERR_INVALID_ARG;
    if (in_dtype != MR_F16 && in_dtype != MR_BF16) return MR_ERR_INVALID_ARG;
    if (out_dtype != MR_F16 && out_dtype != MR_BF16 && out_dtype != MR_F32) return MR_ERR_INVALID_ARG;
    if (tile_id < -1 || tile_id >= kNumTiles) return MR_ERR_INVALID_ARG;
    if (raster < 0 || raster > 64) return MR_ERR_INVALID_ARG;
    for (int g = 0; g < G; ++g)
        if (!Wts[g] || !Cs[g]) return MR_ERR_INVALID_ARG;
    if (K % 8 != 0 || lda % 8 != 0 || ldw % 8 != 0 || ldc % 8 != 0) return MR_ERR_MISALIGNED;
    if ((uintptr_t)A & 15u) return MR_ERR_MISALIGNED;
    for (int g = 0; g < G; ++g)
        if (((uintptr_t)Wts[g] & 15u) || ((uintptr_t)Cs[g] & 15u)) return MR_ERR_MISALIGNED;

    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) return mr_host::cuda_status(e);
    e = init_device(device);
    if (e != cudaSuccess) return MR_ERR_CUDA;
    const int sms = mr_host::sm_count() > 0 ? mr_host::sm_count() : 148;
    const int pairs = max_pairs(device);
    const int t = tile_id >= 0 ? tile_id : select_tile_grouped(M, N, K, G, sms, pairs);
    if (t < 0) return MR_ERR_INVALID_ARG;
    const TileDesc &td = kTiles[t];
    if (td.pair && pairs < 1) return MR_ERR_UNSUPPORTED;

    GemmArgs<MAXG> args;
    memset(&args, 0, sizeof(args));
    args.P = pack_factor(td.bn, N, G, td.pair);
    args.tn_per_group = (N + td.bn - 1) / td.bn;
    args.ntn = (int)n_slots(td.bn, N, G, args.P);
    args.M = M;
    args.N = N;
    args.K = K;
    args.G = G;
    args.ldc = ldc;
    args.raster = raster;
    args.idesc = make_idesc(in_dtype, td.bm, td.bn);
    // The pair tile's CTAs each load 128 rows of A and bn / 2 rows of Wt.
    if (!encode_operand(&args.tmA, A, M, K, lda, in_dtype, td.pair ? td.bm / 2 : td.bm)) return MR_ERR_CUDA;
    const int b_rows = args.P > 1 ? N : (td.pair ? td.bn / 2 : td.bn);
    for (int g = 0; g < G; ++g) {
        if (!encode_operand(&args.tmB[g], Wts[g], N, K, ldw, in_dtype, b_rows)) return MR_ERR_CUDA;
        args.C[g] = Cs[g];
    }

    const int64_t ntiles = (int64_t)args.ntn * ((M + td.bm - 1) / td.bm);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = td.pair ? dim3((unsigned)(2 * std::min<int64_t>(ntiles, pairs)))
                          : dim3((unsigned)std::min<int64_t>(ntiles, sms));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = tile_smem_bytes(t);
    cfg.stream = static_cast<cudaStream_t>(stream);
    e = cudaLaunchKernelEx(&cfg, kernel_for<MAXG>(t, out_dtype), args);
    return mr_host::cuda_status(e);
}

}  // namespace gemm
}  // namespace mr

extern "C" int32_t gemm_f16_num_tiles(void) { return mr::gemm::kNumTiles; }

extern "C" const char *gemm_f16_tile_name(int32_t tile_id) {
    if (tile_id < 0 || tile_id >= mr::gemm::kNumTiles) return nullptr;
    return mr::gemm::kTiles[tile_id].name;
}

namespace mr {
namespace gemm {
// SMs and CTA pairs of the current device (148 and 74 when no device answers).
void device_slots(int &sms, int &pairs) {
    sms = mr_host::sm_count();
    if (sms <= 0) sms = 148;
    int device = 0;
    pairs = (cudaGetDevice(&device) == cudaSuccess && init_device(device) == cudaSuccess) ? max_pairs(device) : 0;
    if (pairs <= 0) pairs = sms / 2;
}
}  // namespace gemm
}  // namespace mr

extern "C" int32_t gemm_f16_select_tile(int32_t M, int32_t N, int32_t K) {
    int sms, pairs;
    mr::gemm::device_slots(sms, pairs);
    return mr::gemm::select_tile(M, N, K, sms, pairs);
}

extern "C" mr_status gemm_f16_ex(const void *A, int64_t lda, const void *Wt, int64_t ldw, void *C, int64_t ldc,
                                 int32_t M, int32_t N, int32_t K, int32_t in_dtype, int32_t out_dtype, int32_t tile_id,
                                 int32_t raster, void *stream) {
    const void *w[1] = {Wt};
    void *c[1] = {C};
    if (!Wt || !C) return MR_ERR_INVALID_ARG;
    return mr::gemm::launch<1>(A, lda, w, ldw, c, ldc, M, N, K, 1, in_dtype, out_dtype, tile_id, raster, stream);
}

extern "C" mr_status gemm_f16(const void *A, int64_t lda, const void *Wt, int64_t ldw, void *C, int64_t ldc,
                              int32_t M, int32_t N, int32_t K, int32_t in_dtype, int32_t out_dtype, int32_t tile_id,
                              void *stream) {
    return gemm_f16_ex(A, lda, Wt, ldw, C, ldc, M, N, K, in_dtype, out_dtype, tile_id, 0, stream);
}

extern "C" mr_status gemm_f16_grouped(const void *A, int64_t lda, const void *const *Wts, int64_t ldw, void *const *Cs,
                                      int64_t ldc, int32_t M, int32_t N, int32_t K, int32_t G, int32_t in_dtype,
                                      int32_t out_dtype, int32_t tile_id, void *stream) {
    if (G > mr::gemm::kMaxGroups) return MR_ERR_UNSUPPORTED;
    return mr::gemm::launch<mr::gemm::kMaxGroups>(A, lda, Wts, ldw, Cs, ldc, M, N, K, G, in_dtype, out_dtype,
                                                  tile_id, 0, stream);
}

extern "C" int32_t gemm_f16_grouped_select_tile(int32_t M, int32_t N, int32_t K, int32_t G) {
    int sms, pairs;
    mr::gemm::device_slots(sms, pairs);
    return mr::gemm::select_tile_grouped(M, N, K, G, sms, pairs);
}
