// pk_merge.cuh -- merging the per-slice Top-k lists of a pair (shared by the
// merge kernel and the attention kernel that merges before it gathers).
//
// Keys are 64-bit (ord(score) << 32 | ~id): larger is better, real keys are
// distinct, 0 is padding.  Lists arrive sorted descending.
#pragma once

#include "pk_internal.cuh"

namespace pk {

typedef unsigned long long u64;

// Output rank r of pair bh: the key's id (-1 for padding) and score.
__device__ __forceinline__ void emit_topk(int32_t *out_idx, float *out_score, int bh, int k, int r, u64 x)
{
    const bool live = x != 0ull;
    out_idx[(size_t)bh * k + r] = live ? (int32_t)(0xffffffffu - (uint32_t)(x & 0xffffffffu)) : -1;
    if (out_score) out_score[(size_t)bh * k + r] = live ? unord_f32((uint32_t)(x >> 32)) : 0.0f;
}

// One warp: the top 128 of two descending lists of at most 128 keys each
// (element 32 j + lane in register j; missing keys are 0), descending, into
// a.  max(A[i], B[127 - i]) over i is the top half of A and B together and is
// bitonic (a falling sequence against a rising one), so seven half-cleaner
// stages sort it: strides 64 and 32 inside a lane's registers, 16 .. 1 across
// lanes by shuffles.
__device__ __forceinline__ void warp_merge128(u64 (&a)[4], const u64 (&b)[4])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const u64 y = __shfl_sync(kFull, b[3 - j], 31 - lane);
        a[j] = a[j] > y ? a[j] : y;
    }
#pragma unroll
    for (int s = 2; s >= 1; s >>= 1) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            if ((j & s) == 0) {
                const u64 x = a[j], y = a[j + s];
                a[j] = x > y ? x : y;
                a[j + s] = x > y ? y : x;
            }
        }
    }
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool upper = (lane & s) == 0;       // keeps the larger key of the pair
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const u64 y = __shfl_xor_sync(kFull, a[j], s);
            a[j] = upper ? (a[j] > y ? a[j] : y) : (a[j] < y ? a[j] : y);
        }
    }
}

// Keys warp_merge_tree needs in its buffer for ns lists.
__host__ __device__ inline int64_t warp_tree_keys(int ns) { return (int64_t)((ns + 1) / 2 + (ns + 3) / 4) * 128; }

// Top k (k <= 128) of ns >= 2 descending lists (list s: k keys at
// src + s stride; from global memory through L2 when global_src) by a tree
// of warp merges: warp w of NW takes merges w, w + NW, .. of a level and
// fetches its next pair before merging the current one.  buf holds
// warp_tree_keys(ns) keys of shared memory; returns the merged list (in
// buf).  All NW warps of the block call it.
template <int NW>
__device__ const u64 *warp_merge_tree(const u64 *src, size_t stride, bool global_src, int ns, int k, u64 *buf)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    u64 *dst = buf, *alt = buf + (size_t)((ns + 1) / 2) * 128;
    auto fetch = [&](const u64 *list, int len, u64 (&v)[4]) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int e = 32 * j + lane;
            v[j] = (list && e < len) ? (global_src ? __ldcg(list + e) : list[e]) : 0ull;
        }
    };
    while (ns > 1) {
        const int np = (ns + 1) / 2;
        u64 a[4], b[4], na[4], nb[4];
        int m = warp;
        if (m < np) {
            fetch(src + (size_t)(2 * m) * stride, k, a);
            fetch(2 * m + 1 < ns ? src + (size_t)(2 * m + 1) * stride : nullptr, k, b);
        }
        while (m < np) {
            const int mn = m + NW;
            if (mn < np) {                        // in flight while this pair merges
                fetch(src + (size_t)(2 * mn) * stride, k, na);
                fetch(2 * mn + 1 < ns ? src + (size_t)(2 * mn + 1) * stride : nullptr, k, nb);
            }
            warp_merge128(a, b);
            u64 *o = dst + (size_t)m * 128;
#pragma unroll
            for (int j = 0; j < 4; j++) o[32 * j + lane] = a[j];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                a[j] = na[j];
                b[j] = nb[j];
            }
            m = mn;
        }
        __syncthreads();
        src = dst;
        dst = alt;
        alt = const_cast<u64 *>(src);
        stride = 128;
        global_src = false;
        ns = np;
    }
    return src;
}

}  // namespace pk
