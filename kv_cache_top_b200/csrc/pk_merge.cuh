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

// Two independent warp_merge128 calls, stage by stage (the two dependency
// chains interleave): top 128 of a and b into a, of c and d into c.
__device__ __forceinline__ void warp_merge128x2(u64 (&a)[4], const u64 (&b)[4], u64 (&c)[4], const u64 (&d)[4])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const u64 y = __shfl_sync(kFull, b[3 - j], 31 - lane);
        const u64 z = __shfl_sync(kFull, d[3 - j], 31 - lane);
        a[j] = a[j] > y ? a[j] : y;
        c[j] = c[j] > z ? c[j] : z;
    }
#pragma unroll
    for (int s = 2; s >= 1; s >>= 1) {
#pragma unroll
        for (int j = 0; j < 4; j++) {
            if ((j & s) == 0) {
                const u64 x = a[j], y = a[j + s], u = c[j], w = c[j + s];
                a[j] = x > y ? x : y;
                a[j + s] = x > y ? y : x;
                c[j] = u > w ? u : w;
                c[j + s] = u > w ? w : u;
            }
        }
    }
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool upper = (lane & s) == 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const u64 y = __shfl_xor_sync(kFull, a[j], s);
            const u64 z = __shfl_xor_sync(kFull, c[j], s);
            a[j] = upper ? (a[j] > y ? a[j] : y) : (a[j] < y ? a[j] : y);
            c[j] = upper ? (c[j] > z ? c[j] : z) : (c[j] < z ? c[j] : z);
        }
    }
}

// Keys warp_merge_tree needs in its buffer for ns lists.
__host__ __device__ inline int64_t warp_tree_keys(int ns) { return (int64_t)((ns + 1) / 2 + (ns + 3) / 4) * 128; }

// Top k (k <= 128) of ns >= 2 descending lists (list s: k keys at
// src + s stride; from global memory through L2 when global_src) by a tree
// of 4-way warp merges: warp w of NW takes groups w, w + NW, .. of four lists
// of a level (two merges side by side, then one), so a level quarters the
// number of lists.  buf holds warp_tree_keys(ns) keys of shared memory;
// returns the merged list (in buf).  All NW warps of the block call it.
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
    auto list = [&](int i) -> const u64 * { return i < ns ? src + (size_t)i * stride : nullptr; };
    while (ns > 1) {
        // groups of 4 lists per warp: two merges side by side, then one
        const int ng = (ns + 3) / 4;
        for (int m = warp; m < ng; m += NW) {
            u64 a[4], b[4], c[4], d[4];
            fetch(list(4 * m), k, a);
            fetch(list(4 * m + 1), k, b);
            fetch(list(4 * m + 2), k, c);
            fetch(list(4 * m + 3), k, d);
            warp_merge128x2(a, b, c, d);
            warp_merge128(a, c);
            u64 *o = dst + (size_t)m * 128;
#pragma unroll
            for (int j = 0; j < 4; j++) o[32 * j + lane] = a[j];
        }
        __syncthreads();
        src = dst;
        dst = alt;
        alt = const_cast<u64 *>(src);
        stride = 128;
        global_src = false;
        k = 128 < k ? 128 : k;
        ns = ng;
    }
    return src;
}

}  // namespace pk
