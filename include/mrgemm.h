/*
 * mrgemm.h -- C ABI of the weight-streaming multi-row matmul library
 * (libmrgemm.so, sm_100a / B200).
 *
 * The library computes C[m,n] = A[m,k] . W[k,n] with the weight read from HBM
 * once per call and shared by every row (the question the nx_batchscale_kat.nx
 * note asks of a matmul path), the multi-row router GEMV and top-10 of Strata
 * PR #109 ("What", router bullet), and the tiled f16/bf16 GEMM for prompt
 * chunks of the "opus r35 track A" audit (section 2, gemm_f16 tiles).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.   Matrices are row-major with an explicit row stride in ELEMENTS.
 *           The weight is passed k-contiguous as Wt[n][k]: row j of Wt is
 *           column j of the logical W[k,n].  Logically C = A . W throughout.
 * Memory.   Every pointer is a device pointer owned by the caller; the
 *           library allocates no device memory per call.  Outputs are
 *           written only by kernels, never by the host.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *           default stream).  Calls are asynchronous on that stream and never
 *           synchronise, except mr_poll_errors.
 * Errors.   Arguments are validated on the host before any launch; on an
 *           error nothing is launched and no output is touched.  No C++
 *           exception crosses the ABI.  The entry points are re-entrant and
 *           thread-safe.
 * Device.   Every wait inside a kernel is bounded in time; a wait that runs
 *           out records a bit in a per-device error word (read it with
 *           mr_poll_errors) and the kernel returns without completing.
 * Numerics. Inputs are exact 16-bit floats, products are accumulated in fp32
 *           in a fixed order, and there is no split-K or stream-K: the bits of
 *           an output element depend only on its row of A, its row of Wt and
 *           k -- not on m, on the other rows, or on the tile shape chosen.
 */
#ifndef MRGEMM_H
#define MRGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mr_status {
    MR_OK = 0,
    MR_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, stride < row length */
    MR_ERR_MISALIGNED = 2,    /* pointer not 16-byte aligned, or k / stride not a multiple of 8 */
    MR_ERR_UNSUPPORTED = 3,   /* size beyond what this build handles (documented per call) */
    MR_ERR_CUDA = 4,          /* a CUDA runtime call failed (no device, launch error, ...) */
    MR_ERR_TIMEOUT = 5        /* a bounded device wait ran out (see mr_poll_errors) */
} mr_status;

/* Element types. */
enum { MR_F16 = 0, MR_BF16 = 1, MR_F32 = 2 };

/* Bits of the per-device error word returned by mr_poll_errors. */
#define MR_DEVERR_GEMV_TIMEOUT   0x1u   /* mrgemv_bf16: a weight stage never arrived */
#define MR_DEVERR_GEMM_TIMEOUT   0x2u   /* gemm_f16: a TMA / MMA pipeline wait ran out */
#define MR_DEVERR_TOPK_TIMEOUT   0x4u   /* router_topk: a wait ran out */
#define MR_DEVERR_SELFTEST       0x8u   /* mr_selftest_wait_timeout fired as intended */

/* Flags for mrgemv_bf16_ex. */
#define MR_GEMV_PDL 0x1u
#define MR_GEMV_SIGMOID 0x2u
/*
 * MR_GEMV_SIGMOID: store 1 / (1 + exp(-c)) for every output c (CUDA's expf,
 * IEEE division): the shared expert's scalar gate of Strata PR #109 ("What":
 * one multi-row GEMV with n = 1 plus a sigmoid), here in the same launch.
 * Not accepted by router_gemv_topk.
 */
/*
 * MR_GEMV_PDL: launch with programmatic dependent launch.  The kernel starts
 * streaming its weight into shared memory BEFORE the previous kernel on the
 * stream has finished, and waits for that kernel only before it reads A.
 * Use it only when the weight is not written by the kernel just before on the
 * same stream (static weights are the normal case); A and C keep ordinary
 * stream order.  Outputs are bitwise identical with and without the flag.
 */

/*
 * mrgemv_bf16 -- multi-row bf16 GEMV, fp32 output.
 *
 * The multi-row GEMV of Strata PR #109 ("What", router bullet: one multi-row
 * GEMV that reads the weight once with per-token accumulators in exactly the
 * single-row order) and the "m>1 packed path" of the nx_batchscale_kat.nx note.
 *
 *   C[i][j] = sum_p A[i][p] * Wt[j][p]   for i < m, j < n, p < k
 *
 * A  : m rows of k bf16, row stride lda (>= k) elements, device.
 * Wt : n rows of k bf16, row stride ldw (>= k) elements, device.
 * C  : m rows of n fp32, row stride ldc (>= n) elements, device (written).
 * 1 <= m <= 16 per call (larger m: call in groups of rows, each row's bits
 * are unchanged); n >= 1; 8 <= k, k % 8 == 0; lda, ldw % 8 == 0; A and Wt
 * 16-byte aligned; k no larger than the per-CTA shared memory allows
 * (k <= 4096 is always accepted) -- else MR_ERR_UNSUPPORTED.
 * Every weight byte is read from HBM once per call.  Row i's result is
 * bitwise identical for every m and every position of the row in A.
 */
mr_status mrgemv_bf16(const void *A, int64_t lda, const void *Wt, int64_t ldw,
                      float *C, int64_t ldc, int32_t m, int32_t n, int32_t k,
                      void *stream);

/* As mrgemv_bf16, with MR_GEMV_* flags (0 gives exactly mrgemv_bf16). */
mr_status mrgemv_bf16_ex(const void *A, int64_t lda, const void *Wt, int64_t ldw,
                         float *C, int64_t ldc, int32_t m, int32_t n, int32_t k,
                         uint32_t flags, void *stream);

/*
 * mrgemv_bf16_plan -- the launch plan mrgemv_bf16_ex would use for (m, n, k,
 * flags) on a device with sm_count SMs and smem_optin bytes of opt-in shared
 * memory per block (pure host arithmetic, no CUDA call).  out[8] receives:
 * grid CTAs, threads of the GEMV warps per CTA, dynamic shared bytes, weight
 * ring slots, warps splitting k, column-group warps, row bucket (m rounded up
 * to 1/2/4/8/16), columns per group.  At launch, where the occupancy
 * calculator allows, a CTA gets one more warp that only fetches the code
 * ahead (it stores nothing and changes no output bit).  Size errors are
 * reported as by mrgemv_bf16.
 */
mr_status mrgemv_bf16_plan(int32_t m, int32_t n, int32_t k, uint32_t flags, int32_t sm_count,
                           int32_t smem_optin, int32_t *out);

/*
 * router_gemv_topk -- the router in one launch: the multi-row GEMV of
 * mrgemv_bf16 followed by the per-row top-k of router_topk.  The two steps of
 * Strata PR #109 ("What", router bullet: one multi-row GEMV plus one multi-row
 * top-10 launch) are fused: every logit is also stored as a 64-bit word
 * (a ready flag and the logit's bits) in the workspace's tag array, and CTA r
 * (one warp per row) polls row r's words until all carry the flag, selects
 * its top-k and zeroes the words again.  No counter, fence or grid-wide
 * barrier is involved.  idx / val are bitwise the outputs of mrgemv_bf16 then
 * router_topk on the same inputs.
 *
 * A, Wt, m, n, k, lda, ldw, flags : as mrgemv_bf16_ex.
 * logits : NULL, or m rows of n fp32 (row stride ldl >= n) that receive the
 *          GEMV output.  When NULL the logits live in the workspace.
 * topk, idx, val, ldo : as router_topk (val may be NULL).
 * workspace : device memory, 256-byte aligned, of at least
 *          router_gemv_topk_workspace_bytes(m, n, logits != NULL) bytes:
 *          a 256-byte head block (MR_ROUTER_TICKET_BYTES, reserved), the tag
 *          array of m * n 64-bit words, and -- when logits is NULL -- room
 *          for the two-launch form's logits in its last m * n * 4 bytes.
 *          Zero it before the first call: every completed fused call leaves
 *          the tag array zero again (after a device error, zero it again).
 *          Calls that share a workspace must pass the same workspace_bytes,
 *          at least the size for the largest m * n among them.  Calls that
 *          may run at the same time (other streams) need separate workspaces.
 */
#define MR_ROUTER_TICKET_BYTES 256u
/*
 * MR_ROUTER_TWO_LAUNCH (flag of router_gemv_topk / _noalloc): run the window
 * as the GEMV kernel followed by the router_topk kernel (programmatic
 * dependent launch) instead of one fused launch: the same outputs, bit for
 * bit, from one call.  The logits go to `logits`, or to the last m * n * 4
 * bytes of the workspace (rounded down to 256); the tag array is not used.
 */
#define MR_ROUTER_TWO_LAUNCH 0x4u
mr_status router_gemv_topk(const void *A, int64_t lda, const void *Wt, int64_t ldw,
                           float *logits, int64_t ldl, int32_t m, int32_t n, int32_t k,
                           int32_t topk, int32_t *idx, float *val, int64_t ldo,
                           void *workspace, size_t workspace_bytes, uint32_t flags,
                           void *stream);

/* Workspace bytes router_gemv_topk needs (0 for invalid sizes). */
size_t router_gemv_topk_workspace_bytes(int32_t m, int32_t n, int32_t logits_provided);

/*
 * router_gemv_topk_noalloc -- router_gemv_topk without a workspace argument,
 * for callers that cannot allocate device memory (a host whose device memory
 * all belongs to its own pool and accounting, a plug-in that may not call
 * cudaMalloc) and so cannot hand in a workspace.  The pages have no
 * counterpart: this is a convenience of this library.
 *
 * Arguments and outputs are those of router_gemv_topk.  The scratch it needs
 * (the workspace layout of router_gemv_topk) is a fixed 256 KiB device array
 * inside the library, held by every GPU that loads the library until the
 * process exits.  With logits == NULL, m * n may not exceed
 * router_gemv_topk_noalloc_max_logits() (21824 values, e.g. 16 x 1364);
 * sizes whose workspace does not fit are rejected with MR_ERR_UNSUPPORTED
 * before anything runs.
 * The call allocates nothing: its first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current, so make
 * that first call before any stream capture.  Each fused call clears the tag
 * array on `stream` (cudaMemsetAsync of m * n * 8 bytes; not with
 * MR_ROUTER_TWO_LAUNCH, which uses no tags) and then launches.  Every call shares the one
 * array, so calls that overlap on the GPU (other streams, or overlapping
 * launches) race and must not be issued.
 */
mr_status router_gemv_topk_noalloc(const void *A, int64_t lda, const void *Wt, int64_t ldw,
                                   float *logits, int64_t ldl, int32_t m, int32_t n, int32_t k,
                                   int32_t topk, int32_t *idx, float *val, int64_t ldo,
                                   uint32_t flags, void *stream);

/* Largest m * n router_gemv_topk_noalloc accepts when logits is NULL. */
size_t router_gemv_topk_noalloc_max_logits(void);

/*
 * router_topk -- per-row top-k of fp32 logits, one CTA per row.
 *
 * The multi-row top-10 launch of Strata PR #109 ("What", router bullet: the
 * kernel takes blockIdx.x = token).  Order: value descending; equal values
 * (-0.0 equals +0.0) by index ascending; a NaN ranks above +inf.  The result
 * is unique under this total order.
 *
 * logits : m rows of n fp32, row stride ldl (>= n) elements, device.
 * idx    : m rows of topk int32 (row stride ldo >= topk), written in rank order.
 * val    : NULL, or m rows of topk fp32 (row stride ldo): the logits at idx,
 *          bit for bit.
 * 1 <= m <= 2^31-1; 1 <= n; 1 <= topk <= min(n, 32).
 */
mr_status router_topk(const float *logits, int64_t ldl, int32_t m, int32_t n,
                      int32_t topk, int32_t *idx, float *val, int64_t ldo,
                      void *stream);

/*
 * router_topk_ex -- router_topk on a shard of columns: the logits are columns
 * [index_base, index_base + n) of a wider row, and every index written is
 * index_base + the column's position in `logits`.  Ties still go to the lower
 * (global) index.  0 <= index_base and index_base + n <= 2^31 - 1; other
 * arguments as router_topk (index_base 0 gives exactly router_topk).
 *
 * The column split of the router across G devices: each device streams its
 * own N/G columns of the weight with A replicated, takes the top-k of its
 * shard, and the G lists are merged (router_topk_merge).  The global top-k
 * lies in the union of the shards' top-k lists, so the merge is exact.  The
 * pages place experts and layers on a second card (Strata PR #109,
 * "Measured" and the release comment); this is that placement for the
 * router's columns.
 */
mr_status router_topk_ex(const float *logits, int64_t ldl, int32_t m, int32_t n,
                         int32_t topk, int32_t *idx, float *val, int64_t ldo,
                         int32_t index_base, void *stream);

/*
 * router_topk_merge -- per-row top-k of candidate (value, index) pairs, under
 * the order of router_topk: value descending, equal values by index
 * ascending, -0.0 equal to +0.0, a NaN above +inf.
 *
 * Row r has `groups` lists of `per_group` pairs; list g of row r is
 *   cand_val[g * ld_group + r * ld_row + t], cand_idx[...]   (t < per_group)
 * (e.g. the [groups][m][per_group] block an all-gather of every shard's
 * router_topk_ex output yields: ld_row = per_group, ld_group = m * per_group).
 * The indices of a row must be distinct; an index < 0 marks an empty entry
 * and is skipped.  idx / val (row stride ldo >= topk) receive the best topk
 * pairs in rank order, the values bit for bit; where a row has fewer than
 * topk non-empty pairs the remaining entries are index -1, value NaN.
 * 1 <= topk <= 32; groups * per_group <= 65536 (MR_ERR_UNSUPPORTED above).
 */
mr_status router_topk_merge(const float *cand_val, const int32_t *cand_idx, int32_t m,
                            int32_t groups, int32_t per_group, int64_t ld_row,
                            int64_t ld_group, int32_t topk, int32_t *idx, float *val,
                            int64_t ldo, void *stream);

/*
 * cast_f32_bf16 -- fp32 -> bf16, round to nearest even, for `rows` rows of
 * `cols` values in one launch: the bf16 cast of the verify window's rows in
 * Strata PR #109 ("What": one call, the rows are contiguous), which feeds the
 * bf16 A of mrgemv_bf16.  NaN stays NaN; overflow rounds to infinity.
 *
 * X : rows x cols fp32, row stride ldx (>= cols) elements, 4-byte aligned.
 * Y : rows x cols bf16, row stride ldy (>= cols) elements, 2-byte aligned.
 * Rows of 8k elements with 16-byte aligned rows take a vectorised path.
 */
mr_status cast_f32_bf16(const float *X, int64_t ldx, void *Y, int64_t ldy, int32_t rows, int32_t cols,
                        void *stream);

/*
 * gemm_f16 -- tiled GEMM on the tcgen05 tensor cores (TMA -> shared memory
 * -> tcgen05.mma with the accumulator in tensor memory), fp32 accumulate.
 *
 * The gemm_f16<TM,TN,SG> prompt-chunk GEMM of the "opus r35 track A" audit
 * (section 2: tiles for M = 150..2048, the M % 128 tail-tile rule, bitwise
 * parity across tiles), rebuilt for sm_100a.
 *
 *   C[i][j] = sum_p A[i][p] * Wt[j][p]     (fp32 accumulate, then out_dtype)
 *
 * A  : M rows of K elements of in_dtype (MR_F16 or MR_BF16), stride lda.
 * Wt : N rows of K elements of in_dtype, stride ldw.
 * C  : M rows of N elements of out_dtype (MR_F16, MR_BF16 or MR_F32), stride ldc;
 *      16-bit outputs are rounded to nearest even.
 * tile_id : -1 selects with gemm_f16_select_tile; 0 .. gemm_f16_num_tiles()-1
 *      forces a tile.  The family: 128 x {32, 64, 96, 128, 192, 256} (MMA
 *      M = 128), 64 x {128, 256} (MMA M = 64, half the padding of a tail
 *      tile), 256 x 256 and 256 x 128 computed by a cluster of two CTAs on
 *      two SMs (tcgen05.mma.cta_group::2, M = 256), then 64 x {32, 64}, in
 *      that order (ids 0 to 11).  Every tile gives the same bits
 *      (fixed K order, K steps of 16, no split-K).
 * M, N >= 1; K >= 8, K % 8 == 0; lda, ldw, ldc % 8 == 0; A, Wt, C 16-byte aligned.
 */
mr_status gemm_f16(const void *A, int64_t lda, const void *Wt, int64_t ldw,
                   void *C, int64_t ldc, int32_t M, int32_t N, int32_t K,
                   int32_t in_dtype, int32_t out_dtype, int32_t tile_id,
                   void *stream);

/*
 * gemm_f16_ex -- gemm_f16 with a tile order: raster 0 is the default (a row
 * tile's N tiles, then the next row tile); raster R in 1..64 walks bands of R
 * N tiles down every row tile, the column-band order of the audit's SLC
 * swizzle study ("opus r35 track A", section 2, SLC swizzle).  Outputs are
 * bitwise identical for every raster; only the order of tiles, and so the
 * reuse of operands in L2, changes.
 */
mr_status gemm_f16_ex(const void *A, int64_t lda, const void *Wt, int64_t ldw,
                      void *C, int64_t ldc, int32_t M, int32_t N, int32_t K,
                      int32_t in_dtype, int32_t out_dtype, int32_t tile_id, int32_t raster,
                      void *stream);

/*
 * gemm_f16_grouped -- G GEMMs that share A in one launch: for g < G,
 *   Cs[g][i][j] = sum_p A[i][p] * Wts[g][j][p]
 * The 36 independent N = 96 projections of one prompt chunk in the
 * "opus r35 track A" audit (section 2, Walbe table: N = 96, K = 2560, 36
 * calls) are this shape.  Each output has exactly the bits gemm_f16 gives for
 * (A, Wts[g]) with any tile: every tile runs the same K sequence.  When N is a
 * multiple of 16 that divides the tile width, one tile covers several groups
 * (for N = 96, two groups per 192-column tile), so A is streamed once for
 * them.
 *
 * Wts, Cs : HOST arrays of G device pointers (Wts[g]: N rows of K elements,
 *           stride ldw; Cs[g]: M rows of N elements, stride ldc).
 * 1 <= G <= 64 (MR_ERR_UNSUPPORTED above); other arguments as gemm_f16.
 */
mr_status gemm_f16_grouped(const void *A, int64_t lda, const void *const *Wts, int64_t ldw,
                           void *const *Cs, int64_t ldc, int32_t M, int32_t N, int32_t K,
                           int32_t G, int32_t in_dtype, int32_t out_dtype, int32_t tile_id,
                           void *stream);

/* The tile gemm_f16_grouped picks for (M, N, K, G) when tile_id is -1. */
int32_t gemm_f16_grouped_select_tile(int32_t M, int32_t N, int32_t K, int32_t G);

/* Number of tile shapes gemm_f16 can run. */
int32_t gemm_f16_num_tiles(void);

/* "BMxBN" name of a tile id (e.g. "128x96"), or NULL when out of range. */
const char *gemm_f16_tile_name(int32_t tile_id);

/*
 * The tile gemm_f16 picks for (M, N, K) when tile_id is -1: a host-side
 * integer cost model over the machine's SM count -- padded tail tiles
 * (M % 128 in 1..64 wastes up to half a tile), wave quantisation, and the
 * narrow-N case (N = 96).  Returns -1 for invalid sizes.
 */
int32_t gemm_f16_select_tile(int32_t M, int32_t N, int32_t K);

/*
 * mr_poll_errors -- synchronise `stream`, then read and clear the error word
 * of the current device.  *device_flags receives MR_DEVERR_* bits (0 when all
 * waits completed).  Returns MR_ERR_TIMEOUT if any bit was set, MR_ERR_CUDA if
 * the synchronisation failed, else MR_OK.  device_flags may be NULL.
 */
mr_status mr_poll_errors(void *stream, uint32_t *device_flags);

/*
 * mr_selftest_wait_timeout -- launch one CTA that waits on an mbarrier which
 * nothing will ever complete, bounded by limit_us microseconds (1..1000000).
 * The wait runs out, sets MR_DEVERR_SELFTEST, and the kernel returns
 * normally: it exercises the bounded-wait path without faulting the GPU.
 */
mr_status mr_selftest_wait_timeout(int32_t limit_us, void *stream);

/* Human-readable name of a status code. */
const char *mr_status_str(mr_status status);

/* Library version string. */
const char *mr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MRGEMM_H */
