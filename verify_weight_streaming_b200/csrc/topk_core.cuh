// Warp-level top-k under the total order of the router selection: value
// descending, equal values by index ascending, -0.0 equal to +0.0, any NaN
// above +inf.  Shared by router_topk and the fused router kernel.
#pragma once

#include <stdint.h>

namespace mr {
namespace topk {

// 64-bit key whose unsigned order is the total order: the high word maps the
// float to an unsigned integer increasing with its value (sign-magnitude
// flip, -0.0 folded onto +0.0, every NaN mapped to the maximum); the low word
// is 0xFFFFFFFF - index, so the lower index of two equal values has the
// larger key.  0 is never a key (it would need index 0xFFFFFFFF) and marks an
// empty entry.
__device__ __forceinline__ uint64_t make_key(float v, uint32_t idx) {
    uint32_t b = __float_as_uint(v);
    uint32_t hi;
    if (v != v) {
        hi = 0xFFFFFFFFu;
    } else {
        if ((b & 0x7FFFFFFFu) == 0u) b = 0u;
        hi = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    }
    return ((uint64_t)hi << 32) | (uint64_t)(0xFFFFFFFFu - idx);
}

__device__ __forceinline__ uint32_t key_index(uint64_t key) { return 0xFFFFFFFFu - (uint32_t)key; }

// The logit a key was made from, bit for bit, except where make_key merged
// values: a zero key stands for +0.0 or -0.0 and the maximal key for any NaN.
// `exact` is false for those two, and the caller must re-read the value.
__device__ __forceinline__ float key_value(uint64_t key, bool &exact) {
    const uint32_t hi = (uint32_t)(key >> 32);
    exact = hi != 0x80000000u && hi != 0xFFFFFFFFu;
    const uint32_t b = (hi & 0x80000000u) ? (hi & 0x7FFFFFFFu) : ~hi;
    return __uint_as_float(b);
}

// Row loads: plain, or (CG) cached in L2 only, for rows other CTAs of the
// same grid have just written (an L1 line cached earlier could be stale).
template <bool CG>
__device__ __forceinline__ float load_row(const float *x, int j) {
    if constexpr (CG) return __ldcg(x + j);
    return x[j];
}

// Value to report for a selected key: decoded from the key when that is
// exact, else re-read from the row.
template <bool CG = false>
__device__ __forceinline__ float selected_value(uint64_t key, const float *x) {
    bool exact;
    const float v = key_value(key, exact);
    return exact ? v : load_row<CG>(x, (int)key_index(key));
}

// Sort L keys descending (insertion network, compile-time indices).
template <int L>
__device__ __forceinline__ void sort_desc(uint64_t (&x)[L]) {
#pragma unroll
    for (int i = 1; i < L; ++i)
#pragma unroll
        for (int j = i; j > 0; --j) {
            const uint64_t a = x[j - 1], b = x[j];
            const bool sw = b > a;
            x[j - 1] = sw ? b : a;
            x[j] = sw ? a : b;
        }
}

// K rounds of warp-wide maximum over the lanes' heads (each lane's keys
// sorted descending).  Lane t receives the t-th largest key (0 if fewer exist).
template <int L>
__device__ __forceinline__ uint64_t warp_select(uint64_t (&x)[L], int K, int lane) {
    uint64_t mine = 0;
#pragma unroll 1
    for (int t = 0; t < K; ++t) {
        const uint32_t hi = (uint32_t)(x[0] >> 32), lo = (uint32_t)x[0];
        const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
        const uint32_t mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
        const bool win = (hi == mhi) && (lo == mlo);
#pragma unroll
        for (int i = 0; i < L - 1; ++i) x[i] = win ? x[i + 1] : x[i];
        if (win) x[L - 1] = 0;
        if (lane == t) mine = ((uint64_t)mhi << 32) | mlo;
    }
    return mine;
}

// Running top-K of elements [begin, end) of a row taken by one warp in
// segments of 32*P elements starting at `begin` and stepping `stride`
// segments; `run` is the warp's running list (lane t holds rank t).
template <int P>
__device__ __forceinline__ uint64_t warp_topk_segments(const float *x, int n, int K, int lane, int seg0,
                                                       int seg_stride, uint64_t run) {
    for (int seg = seg0; (int64_t)seg * 32 * P < n; seg += seg_stride) {
        const int base = seg * 32 * P;
        uint64_t keys[P + 1];
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const int j = base + lane + 32 * i;
            keys[i] = j < n ? make_key(x[j], (uint32_t)j) : 0ull;
        }
        keys[P] = run;
        sort_desc(keys);
        run = warp_select(keys, K, lane);
    }
    return run;
}

// Rank of `key` among the 32 lanes' keys: how many lanes hold a larger key.
// Keys are unique, so nonzero keys get distinct ranks.
__device__ __forceinline__ int warp_rank(uint64_t key, int lane) {
    int r = 0;
#pragma unroll
    for (int s = 1; s < 32; ++s) {
        const uint64_t o = __shfl_sync(0xffffffffu, key, (lane + s) & 31);
        r += o > key ? 1 : 0;
    }
    return r;
}

// Top-K (K <= 32) of one chunk of up to 32*P keys held P per lane, merged
// with a running list `run` (lane t holds rank t, 0 = empty).  Fast path:
// tau = the K-th largest lane maximum (every one of the top K keys is >= tau,
// because the K lanes with the largest maxima each hold a key >= tau); the
// keys >= tau are gathered through `scratch` (64 keys of shared memory per
// warp) and, when there are at most 32, ranked with shuffles in one pass.
// Otherwise (heavy ties) it falls back to K rounds of warp-wide maximum.
// Returns the new running list (lane t holds rank t).
template <int P>
__device__ __forceinline__ uint64_t warp_topk_merge(uint64_t (&key)[P], uint64_t run, int K, int lane,
                                                    uint64_t *scratch) {
    // Lane maximum by a pairwise tree (short dependency chain).
    uint64_t t[P];
#pragma unroll
    for (int i = 0; i < P; ++i) t[i] = key[i];
#pragma unroll
    for (int w = 1; w < P; w <<= 1)
#pragma unroll
        for (int i = 0; i + w < P; i += 2 * w) t[i] = t[i + w] > t[i] ? t[i + w] : t[i];
    const uint64_t mx = t[0] > run ? t[0] : run;
    const int r0 = warp_rank(mx, lane);
    const unsigned who = __ballot_sync(0xffffffffu, r0 == K - 1 && mx != 0ull);
    // Fewer than K nonzero lane maxima: every nonzero key is a candidate.
    const uint64_t tau = who ? __shfl_sync(0xffffffffu, mx, __ffs(who) - 1) : 1ull;
    int c = (run >= tau && run != 0ull) ? 1 : 0;
#pragma unroll
    for (int i = 0; i < P; ++i) c += (key[i] >= tau && key[i] != 0ull) ? 1 : 0;
    int pos = c;  // inclusive prefix sum of the counts over lanes
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, pos, d);
        if (lane >= d) pos += o;
    }
    const int total = __shfl_sync(0xffffffffu, pos, 31);
    if (total <= 32) {
        pos -= c;
        if (c) {
            if (run >= tau && run != 0ull) scratch[pos++] = run;
#pragma unroll
            for (int i = 0; i < P; ++i)
                if (key[i] >= tau && key[i] != 0ull) scratch[pos++] = key[i];
        }
        scratch[32 + lane] = 0ull;
        __syncwarp();
        const uint64_t cand = lane < total ? scratch[lane] : 0ull;
        const int r = warp_rank(cand, lane);
        __syncwarp();
        if (cand != 0ull && r < K) scratch[32 + r] = cand;
        __syncwarp();
        const uint64_t out = lane < K ? scratch[32 + lane] : 0ull;
        __syncwarp();
        return out;
    }
    // Slow path: sort each lane's keys and take K rounds of the warp maximum.
    uint64_t all[P + 1];
#pragma unroll
    for (int i = 0; i < P; ++i) all[i] = key[i];
    all[P] = run;
    sort_desc(all);
    return warp_select(all, K, lane);
}

// Running top-K of x[0, n) taken by one warp in chunks of 32*P elements
// (chunks seg0, seg0 + seg_stride, ...), merged into `run`.
template <int P, bool CG = false>
__device__ __forceinline__ uint64_t warp_topk_fast(const float *x, int n, int K, int lane, int seg0,
                                                   int seg_stride, uint64_t run, uint64_t *scratch) {
    for (int seg = seg0; (int64_t)seg * 32 * P < n; seg += seg_stride) {
        const int base = seg * 32 * P;
        float v[P];
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const int j = base + lane + 32 * i;
            v[i] = j < n ? load_row<CG>(x, j) : 0.0f;
        }
        uint64_t keys[P];
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const int j = base + lane + 32 * i;
            keys[i] = j < n ? make_key(v[i], (uint32_t)j) : 0ull;
        }
        run = warp_topk_merge<P>(keys, run, K, lane, scratch);
    }
    return run;
}

}  // namespace topk
}  // namespace mr
