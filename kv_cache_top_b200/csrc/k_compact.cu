// k_compact.cu -- the candidate set of each pair, in ascending key order.
//
// Candidates (ParisKV slides, Sec. 4.2.2 "choose the top-beta keys by S_i"
// and Sec. 4.3 "rerank C = ceil(beta n)"): every key with S > s*, then the
// lowest-id keys with S = s* until C are taken.  The collision scan already
// fixed, per chunk of keys, the first output slot and how many of the chunk's
// S = s* keys it keeps; here each CTA streams its chunk of S (16 bytes per
// thread per window) and writes its candidates with one block-wide scan per
// window, so the list comes out ordered with no global synchronisation.
#include "pk_internal.cuh"

namespace pk {

constexpr int kCpThreads = 256;
constexpr int kCpWin = 16 * kCpThreads;

__global__ void __launch_bounds__(kCpThreads) k_compact(CompactArgs a)
{
    __shared__ uint32_t s_ws[kCpThreads / 32 + 1];
    const int bh = blockIdx.y, chunk = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t lo = (int64_t)chunk * a.chunk;
    const int64_t hi = min(lo + a.chunk, a.n);
    const uint2 info = a.chunk_info[(size_t)bh * a.max_chunks + chunk];
    const uint32_t slot0 = info.x, quota = info.y;
    const int sstar = a.sstar[bh];
    const uint8_t *S = a.S + (size_t)bh * a.stride;
    int32_t *out = a.cand + (size_t)bh * a.stride + slot0;
    int32_t *dbg = a.dbg_cand ? a.dbg_cand + (size_t)bh * a.C + slot0 : nullptr;
    const int64_t room = a.C - (int64_t)slot0;   // slots this chunk may write

    uint32_t carry_gt = 0, carry_eq = 0;
    for (int64_t wbase = lo; wbase < hi; wbase += kCpWin) {
        const int64_t i0 = wbase + 16 * tid;
        uint8_t sv[16];
        if (i0 + 15 < hi) {
            const uint4 v = *reinterpret_cast<const uint4 *>(S + i0);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 16; u++) sv[u] = (uint8_t)(w[u >> 2] >> (8 * (u & 3)));
        } else {
#pragma unroll
            for (int u = 0; u < 16; u++) sv[u] = (i0 + u < hi) ? S[i0 + u] : (uint8_t)0;
        }
        uint32_t gtc = 0, eqc = 0;
#pragma unroll
        for (int u = 0; u < 16; u++) {
            const bool in = i0 + u < hi;
            gtc += (in && (int)sv[u] > sstar) ? 1u : 0u;
            eqc += (in && (int)sv[u] == sstar) ? 1u : 0u;
        }
        uint32_t tot;
        const uint32_t ex = block_excl_scan<kCpThreads>((gtc << 16) | eqc, s_ws, &tot);
        uint32_t gtb = carry_gt + (ex >> 16), eqb = carry_eq + (ex & 0xffffu);
#pragma unroll
        for (int u = 0; u < 16; u++) {
            const bool in = i0 + u < hi;
            const bool is_gt = in && (int)sv[u] > sstar;
            const bool is_eq = in && (int)sv[u] == sstar;
            if (is_gt || (is_eq && eqb < quota)) {
                const uint32_t slot = gtb + min(eqb, quota);
                if ((int64_t)slot < room) {
                    out[slot] = (int32_t)(i0 + u);
                    if (dbg) dbg[slot] = (int32_t)(i0 + u);
                }
            }
            gtb += is_gt ? 1u : 0u;
            eqb += is_eq ? 1u : 0u;
        }
        carry_gt += tot >> 16;
        carry_eq += tot & 0xffffu;
    }
    if (tid == 0 && (int64_t)carry_gt + min(carry_eq, quota) > room)
        devchk(a.dev_err, nullptr, DEVCHK_CAND_COUNT, (long long)slot0);
}

cudaError_t launch_compact(const CompactArgs &a, int nchunks, int bh, cudaStream_t s)
{
    k_compact<<<dim3(nchunks, bh), kCpThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace pk
