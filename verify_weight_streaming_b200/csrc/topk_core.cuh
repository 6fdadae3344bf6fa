// Warp-level top-k under the total order of the router selection: value
// descending, equal values by index ascending, -0.0 equal to +0.0, any NaN
// above +inf.  Shared by router_topk, router_topk_merge and the fused router
// kernel.
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
__device__ __forceinline__ uint32_t order_word(float v) {
    const uint32_t b = __float_as_uint(v);
    // b ^ 0x80000000 for a clear sign bit (b | 0x80000000), ~b for a set one
    uint32_t hi = b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
    hi = (b == 0x80000000u) ? 0x80000000u : hi;  // -0.0 onto +0.0
    hi = (v != v) ? 0xFFFFFFFFu : hi;            // every NaN to the maximum
    return hi;
}

__device__ __forceinline__ uint64_t make_key(float v, uint32_t idx) {
    return ((uint64_t)order_word(v) << 32) | (uint64_t)(0xFFFFFFFFu - idx);
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

// Value to report for a selected key: decoded from the key when that is
// exact, else re-read from the row.
__device__ __forceinline__ float selected_value(uint64_t key, const float *x) {
    bool exact;
    const float v = key_value(key, exact);
    return exact ? v : x[key_index(key)];
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

// The heavy-tie fallback of warp_topk_merge: sort each lane's L keys and
// take K rounds of the warp-wide maximum.  Kept out of line: inlined, its
// sorting network is scheduled into the common path and slows it by about
// half although it never runs there.
template <int L>
struct KeySet {
    uint64_t k[L];
};
template <int L>
__device__ __noinline__ uint64_t select_rounds(KeySet<L> all, int K, int lane) {
    sort_desc(all.k);
    return warp_select(all.k, K, lane);
}

// Top-K (K <= 32) of one chunk of up to 32*P keys held P per lane, merged
// with a running list `run` (lane t holds rank t, 0 = empty).  `scratch`:
// 64 keys of shared memory for this warp, 16-byte aligned.
//  1. tau = the K-th largest lane maximum of the keys' high words (the
//     largest value that at least K lanes reach): every one of the top K keys
//     has a high word >= tau, since the K lanes that reach tau each hold one.
//     The lane maxima are exchanged through shared memory (broadcast reads),
//     not shuffles.
//  2. The keys with a high word >= tau are the candidates; each lane's count
//     is prefix-summed over the lanes bit by bit (one ballot per bit) and the
//     candidates are stored to consecutive slots of `scratch`.
//  3. When there are at most 32, lane t takes candidate t and ranks it by
//     comparing with all of them (broadcast reads again); the rank-r key is
//     written to slot 32 + r.  Otherwise (heavy ties) select_rounds.
// Returns the new running list (lane t holds rank t).
template <int P>
__device__ __forceinline__ uint64_t warp_topk_merge(uint64_t (&key)[P], uint64_t run, int K, int lane,
                                                    uint64_t *scratch) {
    static_assert(P + 1 <= 31, "one mask bit per key");
    uint32_t hi[P + 1], t[P + 1];
#pragma unroll
    for (int i = 0; i < P; ++i) hi[i] = (uint32_t)(key[i] >> 32);
    hi[P] = (uint32_t)(run >> 32);
#pragma unroll
    for (int i = 0; i <= P; ++i) t[i] = hi[i];
#pragma unroll
    for (int w = 1; w < P + 1; w <<= 1)
#pragma unroll
        for (int i = 0; i + w < P + 1; i += 2 * w) t[i] = max(t[i], t[i + w]);
    const uint32_t mx = t[0];
    uint32_t *s32 = reinterpret_cast<uint32_t *>(scratch);
    s32[lane] = mx;
    __syncwarp();
    int g0 = 0, g1 = 0, g2 = 0, g3 = 0;  // lanes whose maximum is >= this lane's
    const uint4 *q = reinterpret_cast<const uint4 *>(s32);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint4 w = q[j];
        g0 += w.x >= mx ? 1 : 0;
        g1 += w.y >= mx ? 1 : 0;
        g2 += w.z >= mx ? 1 : 0;
        g3 += w.w >= mx ? 1 : 0;
    }
    const int ge = (g0 + g1) + (g2 + g3);
    // An empty key has a zero high word and no real key does: tau >= 1.
    const uint32_t tau = max(__reduce_max_sync(0xffffffffu, ge >= K ? mx : 0u), 1u);
    uint32_t msk = 0;
#pragma unroll
    for (int i = 0; i <= P; ++i) msk |= (hi[i] >= tau ? 1u : 0u) << i;
    const uint32_t c = (uint32_t)__popc(msk);
    const unsigned below = (1u << lane) - 1u;
    int pos = 0, total = 0;
#pragma unroll
    for (int b = 0; (1 << b) <= P + 1; ++b) {
        const unsigned bb = __ballot_sync(0xffffffffu, (c >> b) & 1u);
        pos += __popc(bb & below) << b;
        total += __popc(bb) << b;
    }
    if (total <= 32) {
        __syncwarp();  // every lane has read the maxima
        int slot = pos;
#pragma unroll
        for (int i = 0; i <= P; ++i) {
            const uint32_t take = (msk >> i) & 1u;
            const uint32_t addr = (uint32_t)__cvta_generic_to_shared(scratch + slot);
            asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q st.shared.u64 [%0], %1;\n\t}" ::"r"(addr),
                         "l"(i < P ? key[i] : run), "r"(take)
                         : "memory");
            slot += (int)take;
        }
        scratch[32 + lane] = 0ull;
        __syncwarp();
        const uint64_t cand = lane < total ? scratch[lane] : 0ull;
        int r0 = 0, r1 = 0, r2 = 0, r3 = 0;  // candidates larger than this lane's
        const ulonglong2 *q2 = reinterpret_cast<const ulonglong2 *>(scratch);
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
            const ulonglong2 a = q2[j], b = q2[j + 1];
            r0 += (2 * j + 0 < total && a.x > cand) ? 1 : 0;
            r1 += (2 * j + 1 < total && a.y > cand) ? 1 : 0;
            r2 += (2 * j + 2 < total && b.x > cand) ? 1 : 0;
            r3 += (2 * j + 3 < total && b.y > cand) ? 1 : 0;
        }
        const int r = (r0 + r1) + (r2 + r3);
        __syncwarp();
        if (cand != 0ull && r < K) scratch[32 + r] = cand;
        __syncwarp();
        const uint64_t out = lane < K ? scratch[32 + lane] : 0ull;
        __syncwarp();
        return out;
    }
    KeySet<P + 1> all;
#pragma unroll
    for (int i = 0; i < P; ++i) all.k[i] = key[i];
    all.k[P] = run;
    return select_rounds<P + 1>(all, K, lane);
}

// Running top-K of x[0, n) taken by one warp in chunks of 32*P elements
// (chunks seg0, seg0 + seg_stride, ...), merged into `run`.
// With `synthetic` the row is not read: element j is taken to be (float)j,
// which runs the common path of the selection on distinct values (used to
// bring the code into the instruction cache ahead of the real call).
template <int P>
__device__ __forceinline__ uint64_t warp_topk_fast(const float *x, int n, int K, int lane, int seg0,
                                                   int seg_stride, uint64_t run, uint64_t *scratch,
                                                   bool synthetic = false) {
    for (int seg = seg0; (int64_t)seg * 32 * P < n; seg += seg_stride) {
        const int base = seg * 32 * P;
        float v[P];
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const int j = base + lane + 32 * i;
            v[i] = j < n ? (synthetic ? (float)j : x[j]) : 0.0f;
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
