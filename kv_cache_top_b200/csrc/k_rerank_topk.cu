// k_rerank_topk.cu -- 4-bit RSQ-IP rerank of the candidates and the Top-k.
//
// Estimate (ParisKV slides, "Stage II estimates the raw attention score from
// 4-bit codes", Eqs. 7-10):
//     <k_i, q>^ = ||q|| sum_b w_{i,b} sum_j sigma_{i,b,j} l_{t_{i,b,j}} q~_{b,j}
// read from the key's 128-byte summary record; "key-only factors are
// precomputed, so GPU ranking needs no full-precision keys".
//
// Work is split by candidate slices (not key ranges), so every CTA reranks
// the same number of records wherever the candidates sit.  A CTA stages its
// candidate ids in shared memory, then each warp keeps 16 record loads in
// flight (8 lanes x 16 B per record, fully coalesced); after one
// pair-exchange each lane owns two blocks (16 coordinates) with their
// weights.  The signed level of a nibble comes from a 16-entry shared table
// (at most 16 distinct words per request: no bank conflicts), q~ stays in
// registers.
//
// Scores never leave the chip: the CTA turns (score, id) into 64-bit keys
// ordered by score desc then id asc, radix-selects its Top-k, sorts it and
// writes it; the last CTA of the pair (ticket counter, no spin-wait) merges the
// per-slice lists into the final sorted Top-k (README: "reranks those
// candidates with a fused 4-bit approximate inner-product kernel and selects
// the final Top-k KV indices").
#include "pk_internal.cuh"

namespace pk {

constexpr int kRrThreads = 256;
constexpr int kRrWarps = kRrThreads / 32;

typedef unsigned long long u64;

struct RrShared {
    u64 tmp[kMaxTopk];
    uint32_t hist[256];
    uint32_t ws[kRrWarps + 1];
    u64 red[kRrWarps];
    uint32_t sh[4];
    uint32_t cnt;
    u64 tau;
    float slev[16];
    int last;
};

// Keep the k largest of keys[0..count) (count > k) in keys[0..k), any order;
// return the smallest kept key.  All threads of the block must call it.
__device__ u64 block_topk_shrink(RrShared &sm, u64 *keys, int count, int k)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    u64 prefix = 0, mask = 0;
    int need = k;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kRrThreads) sm.hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < count; i += kRrThreads) {
            const u64 x = keys[i];
            if ((x & mask) == prefix) atomicAdd(&sm.hist[(x >> shift) & 0xffu], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t hc[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                hc[i] = sm.hist[255 - 8 * lane - i];
                sum += hc[i];
            }
            uint32_t incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t run = incl - sum;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                if (run < (uint32_t)need && run + hc[i] >= (uint32_t)need) {
                    sm.sh[0] = 255 - 8 * lane - i;
                    sm.sh[1] = run;
                    sm.sh[2] = hc[i];
                }
                run += hc[i];
            }
        }
        __syncthreads();
        const uint32_t d = sm.sh[0], above = sm.sh[1], inbin = sm.sh[2];
        need -= (int)above;
        prefix |= (u64)d << shift;
        mask |= (u64)0xffu << shift;
        __syncthreads();
        if ((int)inbin == need) break;
    }
    if (tid == 0) sm.sh[3] = 0;
    __syncthreads();
    for (int i = tid; i < count; i += kRrThreads) {
        const u64 x = keys[i];
        if ((x & mask) >= prefix) {
            const uint32_t pos = atomicAdd(&sm.sh[3], 1u);
            if (pos < (uint32_t)kMaxTopk) sm.tmp[pos] = x;   // exactly k reach here
        }
    }
    __syncthreads();
    u64 mn = ~0ull;
    for (int i = tid; i < k; i += kRrThreads) {
        const u64 x = sm.tmp[i];
        keys[i] = x;
        mn = x < mn ? x : mn;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const u64 y = __shfl_xor_sync(kFull, mn, o);
        mn = y < mn ? y : mn;
    }
    if (lane == 0) sm.red[warp] = mn;
    __syncthreads();
    if (tid == 0) {
        u64 m = sm.red[0];
        for (int w = 1; w < kRrWarps; w++) m = sm.red[w] < m ? sm.red[w] : m;
        sm.tau = m;
    }
    __syncthreads();
    return sm.tau;
}

// Sort keys[0..k) descending into sm.tmp[0..p2) (zero-padded).
__device__ void block_sort_desc(RrShared &sm, const u64 *keys, int k)
{
    const int tid = threadIdx.x;
    int p2 = 1;
    while (p2 < k) p2 <<= 1;
    for (int i = tid; i < p2; i += kRrThreads) sm.tmp[i] = (i < k) ? keys[i] : 0ull;
    __syncthreads();
    for (int kk = 2; kk <= p2; kk <<= 1) {
        for (int j = kk >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < p2; i += kRrThreads) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const u64 x = sm.tmp[i], y = sm.tmp[ixj];
                    const bool desc = (i & kk) == 0;
                    if (desc ? (x < y) : (x > y)) {
                        sm.tmp[i] = y;
                        sm.tmp[ixj] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
}

__device__ __forceinline__ u64 make_key(float est, int32_t idx)
{
    return ((u64)ord_f32(__fadd_rn(est, 0.0f)) << 32) | (u64)(0xffffffffu - (uint32_t)idx);
}

// dot of one block's 8 nibbles (one u32) with 8 coordinates of q~
__device__ __forceinline__ float block_dot(const float *slev, uint32_t nib, const float *q)
{
    float d = 0.0f;
#pragma unroll
    for (int jj = 0; jj < 8; jj++) d = fmaf(slev[(nib >> (4 * jj)) & 0xfu], q[jj], d);
    return d;
}

__global__ void __launch_bounds__(kRrThreads, 2) k_rerank_topk(RerankArgs a)
{
    extern __shared__ __align__(16) unsigned char s_dyn[];
    __shared__ RrShared sm;
    u64 *keys = reinterpret_cast<u64 *>(s_dyn);                         // [slice]
    int32_t *ids = reinterpret_cast<int32_t *>(s_dyn + (size_t)a.slice * sizeof(u64));
    const int bh = blockIdx.y, sl = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.topk;
    const int64_t m0 = (int64_t)sl * a.slice;
    const int count = (int)min((int64_t)a.slice, a.C - m0);

    if (tid < 16) sm.slev[tid] = (tid & 8) ? -a.lv.lev[tid & 7] : a.lv.lev[tid & 7];
    const int32_t *cand = a.cand + (size_t)bh * a.stride + m0;
    for (int i = tid; i < count; i += kRrThreads) ids[i] = cand[i];
    const int q8 = lane & 7, sub = lane >> 3;
    float qr[16];
#pragma unroll
    for (int i = 0; i < 16; i++) qr[i] = a.qt[(size_t)bh * kD + 16 * q8 + i];
    const float qnorm = a.qnorm[bh];
    const uint8_t *rec = a.rec + (size_t)bh * a.stride * kRecBytes;
    float *dest = a.dbg_est ? a.dbg_est + (size_t)bh * a.C + m0 : nullptr;
    __syncthreads();

    const bool odd = (q8 & 1) != 0;
    // software pipeline: the next 16 records of the warp are in flight while
    // the current 16 are decoded
    const int step = kRrWarps * 16;
    uint4 vn[4];
    int32_t idn[4];
#pragma unroll
    for (int u = 0; u < 4; u++) {
        const int r = warp * 16 + 4 * u + sub;
        idn[u] = ids[r < count ? r : 0];
        vn[u] = __ldg(reinterpret_cast<const uint4 *>(rec + (size_t)idn[u] * kRecBytes) + q8);
    }
    for (int r0 = warp * 16; r0 < count; r0 += step) {
        uint4 v[4];
        int32_t id[4];
#pragma unroll
        for (int u = 0; u < 4; u++) {
            v[u] = vn[u];
            id[u] = idn[u];
        }
        if (r0 + step < count) {
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int r = r0 + step + 4 * u + sub;
                idn[u] = ids[r < count ? r : 0];
                vn[u] = __ldg(reinterpret_cast<const uint4 *>(rec + (size_t)idn[u] * kRecBytes) + q8);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; u++) {
            // even lane of a pair: nibble words of blocks 4g..4g+3; odd lane: their
            // weights.  Swap halves so lane q8 owns blocks 2 q8, 2 q8 + 1.
            const uint32_t r0v = __shfl_xor_sync(kFull, odd ? v[u].x : v[u].z, 1);
            const uint32_t r1v = __shfl_xor_sync(kFull, odd ? v[u].y : v[u].w, 1);
            const uint32_t nib0 = odd ? r0v : v[u].x, nib1 = odd ? r1v : v[u].y;
            const float w0 = __uint_as_float(odd ? v[u].z : r0v);
            const float w1 = __uint_as_float(odd ? v[u].w : r1v);
            const float d0 = block_dot(sm.slev, nib0, qr);
            const float d1 = block_dot(sm.slev, nib1, qr + 8);
            float part = fmaf(w0, d0, w1 * d1);
            part += __shfl_xor_sync(kFull, part, 1);
            part += __shfl_xor_sync(kFull, part, 2);
            part += __shfl_xor_sync(kFull, part, 4);
            const int r = r0 + 4 * u + sub;
            if (q8 == 0 && r < count) {
                const float est = qnorm * part;
                keys[r] = make_key(est, id[u]);
                if (dest) dest[r] = est;
            }
        }
    }
    __syncthreads();

    // ---- Top-k of the slice
    const int have = min(count, k);
    if (count > k) block_topk_shrink(sm, keys, count, k);
    block_sort_desc(sm, keys, have);
    u64 *part = a.partial + ((size_t)bh * a.max_slices + sl) * a.topk_cap;
    for (int i = tid; i < k; i += kRrThreads) part[i] = (i < have) ? sm.tmp[i] : 0ull;
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.last = (atomicAdd(&a.tickets[(size_t)bh * 2 + 1], 1u) == (unsigned)(a.nslices - 1));
    __syncthreads();
    if (!sm.last) return;
    __threadfence();

    // ---- last CTA of the pair: merge the per-slice lists (keys[] is reused)
    const int cap = a.slice;                   // room in keys[] (>= 2k by construction)
    int cnt = 0;
    u64 tau = 0ull;
    const int64_t total = (int64_t)a.nslices * k;
    for (int64_t e0 = 0; e0 < total; e0 += cap - k) {
        const int64_t e1 = min(total, e0 + (cap - k));
        if (tid == 0) sm.cnt = (uint32_t)cnt;
        __syncthreads();
        for (int64_t e = e0 + tid; e < e1; e += kRrThreads) {
            const int64_t j = e / k, r = e - j * k;
            const u64 x = __ldcg(a.partial + ((size_t)bh * a.max_slices + j) * a.topk_cap + r);
            if (x != 0ull && x > tau) keys[atomicAdd(&sm.cnt, 1u)] = x;
        }
        __syncthreads();
        cnt = (int)sm.cnt;
        if (cnt > k) {
            tau = block_topk_shrink(sm, keys, cnt, k);
            cnt = k;
        }
    }
    const int got = min(cnt, k);
    if (got != k && tid == 0) devchk(a.dev_err, nullptr, DEVCHK_CAND_COUNT, got);
    block_sort_desc(sm, keys, got);
    for (int i = tid; i < k; i += kRrThreads) {
        const u64 x = sm.tmp[i];
        const bool live = i < got;
        a.out_idx[(size_t)bh * k + i] = live ? (int32_t)(0xffffffffu - (uint32_t)(x & 0xffffffffu)) : -1;
        if (a.out_score) a.out_score[(size_t)bh * k + i] = live ? unord_f32((uint32_t)(x >> 32)) : 0.0f;
    }
    if (tid == 0) a.tickets[(size_t)bh * 2 + 1] = 0u;
}

size_t rerank_smem(int slice) { return (size_t)slice * (sizeof(u64) + sizeof(int32_t)); }

cudaError_t launch_rerank_topk(const RerankArgs &a, int bh, cudaStream_t s)
{
    static int attr_max = 0;
    const size_t smem = rerank_smem(a.slice);
    if ((int)smem > attr_max) {
        cudaError_t e = cudaFuncSetAttribute(k_rerank_topk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)rerank_smem(kMaxSlice));
        if (e != cudaSuccess) return e;
        attr_max = (int)rerank_smem(kMaxSlice);
    }
    k_rerank_topk<<<dim3(a.nslices, bh), kRrThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace pk
