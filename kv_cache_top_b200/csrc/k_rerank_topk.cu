// k_rerank_topk.cu -- candidate compaction, 4-bit RSQ-IP rerank and Top-k.
//
// Candidates (ParisKV slides, Sec. 4.2.2 and Sec. 4.3: keep C = ceil(beta n)
// keys by S): keys with S > s*, plus the lowest-id keys with S = s* up to the
// chunk's quota computed by the collision scan; slots are in ascending id
// order across the whole pair.
//
// Estimate (slides, "Stage II estimates the raw attention score from 4-bit
// codes", Eqs. 7-10):
//     <k_i, q>^ = ||q|| sum_b w_{i,b} sum_j sigma_{i,b,j} l_{t_{i,b,j}} q~_{b,j}
// read from the key's 128-byte summary record.  Eight lanes share a record
// (one coalesced 128 B load); after one pair-exchange each lane owns two
// blocks (16 coordinates) with their weights, so every lane does the same
// amount of decode work; q~ stays in registers.
//
// Scores never leave the chip: each CTA keeps a running Top-k of
// (score, id) keys in shared memory (radix select on 64-bit keys whose order
// is score desc, then id asc), writes its Top-k, and the last CTA of the pair
// merges the per-chunk lists into the final sorted Top-k (README: "reranks
// those candidates with a fused 4-bit approximate inner-product kernel and
// selects the final Top-k KV indices").
#include "pk_internal.cuh"

namespace pk {

constexpr int kRrThreads = 256;
constexpr int kRrWarps = kRrThreads / 32;
constexpr int kWin = 4 * kRrThreads;   // keys per compaction window
constexpr int kCap = 4096;             // running Top-k buffer (64-bit keys)

typedef unsigned long long u64;

struct RrSmem {
    u64 buf[kCap];
    u64 tmp[kMaxTopk];
    int32_t cand[kWin];
    uint32_t hist[256];
    uint32_t ws[kRrWarps + 1];
    u64 red[kRrWarps];
    uint32_t sh[4];
    uint32_t cnt;
    u64 tau;
    float lev[kL];
    int last;
};

// Keep the k largest of buf[0..count) (count > k) in buf[0..k), any order;
// return the smallest kept key.  All threads of the block must call it.
__device__ u64 block_topk_shrink(RrSmem &sm, int count, int k)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    u64 prefix = 0, mask = 0;
    int need = k;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kRrThreads) sm.hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < count; i += kRrThreads) {
            const u64 x = sm.buf[i];
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
        const u64 x = sm.buf[i];
        if ((x & mask) >= prefix) {
            const uint32_t pos = atomicAdd(&sm.sh[3], 1u);
            if (pos < (uint32_t)kMaxTopk) sm.tmp[pos] = x;   // exactly k reach here
        }
    }
    __syncthreads();
    u64 mn = ~0ull;
    for (int i = tid; i < k; i += kRrThreads) {
        const u64 x = sm.tmp[i];
        sm.buf[i] = x;
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
        sm.cnt = (uint32_t)k;
    }
    __syncthreads();
    return sm.tau;
}

// Sort buf[0..k) descending into tmp[0..p2) (zero-padded).
__device__ void block_sort_desc(RrSmem &sm, int k)
{
    const int tid = threadIdx.x;
    int p2 = 1;
    while (p2 < k) p2 <<= 1;
    for (int i = tid; i < p2; i += kRrThreads) sm.tmp[i] = (i < k) ? sm.buf[i] : 0ull;
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

__global__ void __launch_bounds__(kRrThreads) k_rerank_topk(RerankArgs a)
{
    __shared__ RrSmem sm;
    const int bh = blockIdx.y, chunk = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.topk;

    const int64_t lo = (int64_t)chunk * a.chunk;
    const int64_t hi = min(lo + a.chunk, a.n);
    const uint2 info = a.chunk_info[(size_t)bh * a.max_chunks + chunk];
    const uint32_t slot0 = info.x, quota = info.y;
    const int sstar = a.sstar[bh];
    const float qnorm = a.qnorm[bh];
    const int q8 = lane & 7;
    float qr[16];
#pragma unroll
    for (int i = 0; i < 16; i++) qr[i] = a.qt[(size_t)bh * kD + 16 * q8 + i];
    if (tid < kL) sm.lev[tid] = a.lv.lev[tid];
    if (tid == 0) {
        sm.cnt = 0;
        sm.tau = 0ull;
    }
    const uint8_t *S = a.S + (size_t)bh * a.n_cap;
    const uint8_t *rec = a.rec + (size_t)bh * a.n_cap * kRecBytes;
    int32_t *dcand = a.dbg_cand ? a.dbg_cand + (size_t)bh * a.C + slot0 : nullptr;
    float *dest = a.dbg_est ? a.dbg_est + (size_t)bh * a.C + slot0 : nullptr;
    __syncthreads();

    uint32_t carry_gt = 0, carry_eq = 0;
    for (int64_t wbase = lo; wbase < hi; wbase += kWin) {
        // ---- ordered compaction of this window's candidates
        const int64_t i0 = wbase + 4 * tid;
        uint32_t sv[4];
        bool valid[4];
        if (i0 + 3 < hi) {
            const uint32_t w4 = *reinterpret_cast<const uint32_t *>(S + i0);
#pragma unroll
            for (int u = 0; u < 4; u++) {
                sv[u] = (w4 >> (8 * u)) & 0xffu;
                valid[u] = true;
            }
        } else {
#pragma unroll
            for (int u = 0; u < 4; u++) {
                valid[u] = (i0 + u) < hi;
                sv[u] = valid[u] ? S[i0 + u] : 0u;
            }
        }
        uint32_t gtc = 0, eqc = 0;
#pragma unroll
        for (int u = 0; u < 4; u++) {
            gtc += (valid[u] && (int)sv[u] > sstar) ? 1u : 0u;
            eqc += (valid[u] && (int)sv[u] == sstar) ? 1u : 0u;
        }
        uint32_t tot;
        const uint32_t ex = block_excl_scan<kRrThreads>((gtc << 16) | eqc, sm.ws, &tot);
        const uint32_t first = carry_gt + min(carry_eq, quota);
        uint32_t gtb = carry_gt + (ex >> 16), eqb = carry_eq + (ex & 0xffffu);
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const bool is_gt = valid[u] && (int)sv[u] > sstar;
            const bool is_eq = valid[u] && (int)sv[u] == sstar;
            if (is_gt || (is_eq && eqb < quota)) {
                const uint32_t slot = gtb + min(eqb, quota);
                sm.cand[slot - first] = (int32_t)(i0 + u);
                if (dcand && (int64_t)slot0 + slot < a.C) dcand[slot] = (int32_t)(i0 + u);
            }
            gtb += is_gt ? 1u : 0u;
            eqb += is_eq ? 1u : 0u;
        }
        carry_gt += tot >> 16;
        carry_eq += tot & 0xffffu;
        const int wcount = (int)(carry_gt + min(carry_eq, quota) - first);
        __syncthreads();

        // ---- rerank: 4 candidates per warp step, 8 lanes per record
        const u64 tau = sm.tau;
        for (int r0 = warp * 4; r0 < wcount; r0 += kRrWarps * 4) {
            const int r = r0 + (lane >> 3);
            const bool ok = r < wcount;
            const int32_t idx = ok ? sm.cand[r] : (int32_t)lo;
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(rec + (size_t)idx * kRecBytes) + q8);
            const bool odd = (q8 & 1) != 0;
            const uint32_t r0v = __shfl_xor_sync(kFull, odd ? v.x : v.z, 1);
            const uint32_t r1v = __shfl_xor_sync(kFull, odd ? v.y : v.w, 1);
            const uint32_t nib0 = odd ? r0v : v.x, nib1 = odd ? r1v : v.y;
            const float w0 = __uint_as_float(odd ? v.z : r0v);
            const float w1 = __uint_as_float(odd ? v.w : r1v);
            float d0 = 0.0f, d1 = 0.0f;
#pragma unroll
            for (int jj = 0; jj < 8; jj++) {
                const uint32_t n0 = (nib0 >> (4 * jj)) & 0xfu, n1 = (nib1 >> (4 * jj)) & 0xfu;
                const float l0 = __uint_as_float(__float_as_uint(sm.lev[n0 & 7u]) ^ ((n0 & 8u) << 28));
                const float l1 = __uint_as_float(__float_as_uint(sm.lev[n1 & 7u]) ^ ((n1 & 8u) << 28));
                d0 = fmaf(l0, qr[jj], d0);
                d1 = fmaf(l1, qr[8 + jj], d1);
            }
            float part = fmaf(w0, d0, w1 * d1);
            part += __shfl_xor_sync(kFull, part, 1);
            part += __shfl_xor_sync(kFull, part, 2);
            part += __shfl_xor_sync(kFull, part, 4);
            const float est = qnorm * part;
            if (ok && q8 == 0) {
                if (dest && (int64_t)slot0 + first + r < a.C) dest[first + r] = est;
                const u64 key = make_key(est, idx);
                if (key > tau) sm.buf[atomicAdd(&sm.cnt, 1u)] = key;
            }
        }
        __syncthreads();
        const int cnt = (int)sm.cnt;
        if (cnt > kCap - kWin) block_topk_shrink(sm, cnt, k);
    }
    if (tid == 0 && (int64_t)slot0 + carry_gt + min(carry_eq, quota) > a.C)
        devchk(a.dev_err, nullptr, DEVCHK_CAND_COUNT, (long long)slot0);
    {
        const int cnt = (int)sm.cnt;
        if (cnt > k) block_topk_shrink(sm, cnt, k);
        const int have = min((int)sm.cnt, k);
        block_sort_desc(sm, have);
        u64 *part = a.partial + ((size_t)bh * a.max_chunks + chunk) * a.topk_cap;
        for (int i = tid; i < k; i += kRrThreads) part[i] = (i < have) ? sm.tmp[i] : 0ull;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.last = (atomicAdd(&a.tickets[(size_t)bh * 2 + 1], 1u) == (unsigned)(a.nchunks - 1));
    __syncthreads();
    if (!sm.last) return;
    __threadfence();

    // ---- last CTA of the pair: merge the per-chunk Top-k lists
    if (tid == 0) {
        sm.cnt = 0;
        sm.tau = 0ull;
    }
    __syncthreads();
    const int64_t total = (int64_t)a.nchunks * k;
    for (int64_t e0 = 0; e0 < total; e0 += kWin) {
        const u64 tau = sm.tau;
        for (int u = 0; u < 4; u++) {
            const int64_t e = e0 + u * kRrThreads + tid;
            if (e < total) {
                const int64_t j = e / k, r = e - j * k;
                const u64 x = __ldcg(a.partial + ((size_t)bh * a.max_chunks + j) * a.topk_cap + r);
                if (x != 0ull && x > tau) sm.buf[atomicAdd(&sm.cnt, 1u)] = x;
            }
        }
        __syncthreads();
        const int cnt = (int)sm.cnt;
        if (cnt > kCap - kWin) block_topk_shrink(sm, cnt, k);
    }
    const int cnt = (int)sm.cnt;
    if (cnt > k) block_topk_shrink(sm, cnt, k);
    const int have = min((int)sm.cnt, k);
    if (have != k && tid == 0) devchk(a.dev_err, nullptr, DEVCHK_CAND_COUNT, have);
    block_sort_desc(sm, have);
    for (int i = tid; i < k; i += kRrThreads) {
        const u64 x = sm.tmp[i];
        const bool live = i < have;
        a.out_idx[(size_t)bh * k + i] = live ? (int32_t)(0xffffffffu - (uint32_t)(x & 0xffffffffu)) : -1;
        if (a.out_score) a.out_score[(size_t)bh * k + i] = live ? unord_f32((uint32_t)(x >> 32)) : 0.0f;
    }
    if (tid == 0) a.tickets[(size_t)bh * 2 + 1] = 0u;
}

}  // namespace pk

namespace pk {
cudaError_t launch_rerank_topk(const RerankArgs &a, int bh, cudaStream_t s)
{
    k_rerank_topk<<<dim3(a.nchunks, bh), kRrThreads, 0, s>>>(a);
    return cudaGetLastError();
}
}  // namespace pk
