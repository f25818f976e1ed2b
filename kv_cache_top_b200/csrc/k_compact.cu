// k_compact.cu -- the candidate set of each pair, in ascending key order.
//
// Candidates (ParisKV slides, Sec. 4.2.2: the keys with the largest collision
// scores S_i; Sec. 4.3: a budget of C = ceil(beta n) of them are reranked):
// every key with S > s*, then the
// lowest-id keys with S = s* until C are taken.  The collision scan already
// fixed, per chunk of keys, the first output slot and how many of the chunk's
// S = s* keys it keeps; here each CTA loads its whole chunk of S at once (up
// to 8 x 16 bytes per thread, each thread a contiguous run of keys), turns
// every 16 bytes into 16-bit masks of "S > s*" and "S = s*", and places the
// candidates with one block-wide scan: no per-key branches.  The ids are
// staged in shared memory in output order and stored by consecutive threads
// (chunks with more than kCpStage candidates store them from each thread).
//
// Byte-parallel compares: scores are <= 96 < 128, so for a byte s,
// s > t  <=>  bit 7 of s + (127 - t) is set, and s >= t <=> bit 7 of
// s + (128 - t); neither sum reaches 256, so the four bytes of a word never
// carry into each other.
#include "pk_internal.cuh"

namespace pk {

constexpr int kCpThreads = 256;
constexpr int kCpMaxU = 8;    // 16-byte groups per thread: chunk <= 32768 keys
constexpr int kCpStage = 4096;   // candidates of a chunk staged in shared memory for coalesced stores

// bit-7 flags of the 4 bytes -> 4-bit mask (bit i = byte i)
__device__ __forceinline__ uint32_t gather4(uint32_t flags) { return (flags * 0x00204081u) >> 28; }

__device__ __forceinline__ void masks16(uint4 v, uint32_t add_gt, uint32_t add_ge, uint32_t &gt,
                                        uint32_t &eq)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    gt = 0;
    eq = 0;
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const uint32_t g = (w[q] + add_gt) & 0x80808080u;
        const uint32_t e = (w[q] + add_ge) & ~g & 0x80808080u;
        gt |= gather4(g) << (4 * q);
        eq |= gather4(e) << (4 * q);
    }
}

__global__ void __launch_bounds__(kCpThreads) k_compact(CompactArgs a)
{
    __shared__ uint32_t s_ws[kCpThreads / 32 + 1];
    __shared__ int32_t s_ids[kCpStage];
    const int bh = blockIdx.y, chunk = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t lo = (int64_t)chunk * a.chunk;
    const int64_t hi = min(lo + a.chunk, a.n);
    pdl_wait();                                   // S, s* and chunk slots come from the scan
    const uint2 info = a.chunk_info[(size_t)bh * a.max_chunks + chunk];
    const uint32_t slot0 = info.x, quota = info.y;
    const uint32_t sstar = (uint32_t)a.sstar[bh];
    const uint32_t add_gt = 0x01010101u * (127u - sstar), add_ge = 0x01010101u * (128u - sstar);
    const uint8_t *S = a.S + (size_t)bh * a.stride;
    const int U = a.groups;                             // 16-byte groups per thread
    const int64_t t0 = lo + (int64_t)16 * U * tid;      // this thread's first key

    uint32_t gtm[kCpMaxU], eqm[kCpMaxU];
    uint4 v[kCpMaxU];
#pragma unroll
    for (int u = 0; u < kCpMaxU; u++) {
        v[u] = make_uint4(0, 0, 0, 0);
        if (u < U && t0 + 16 * u < hi) v[u] = *reinterpret_cast<const uint4 *>(S + t0 + 16 * u);
    }
    uint32_t ngt = 0, neq = 0;
#pragma unroll
    for (int u = 0; u < kCpMaxU; u++) {
        gtm[u] = eqm[u] = 0;
        if (u < U) {
            const int64_t k0 = t0 + 16 * u;
            masks16(v[u], add_gt, add_ge, gtm[u], eqm[u]);
            const int64_t left = hi - k0;                 // keys of this group inside the chunk
            const uint32_t keep = left >= 16 ? 0xffffu : (left <= 0 ? 0u : ((1u << left) - 1u));
            gtm[u] &= keep;
            eqm[u] &= keep;
            ngt += __popc(gtm[u]);
            neq += __popc(eqm[u]);
        }
    }
    uint32_t tot;
    const uint32_t ex = block_excl_scan<kCpThreads>((ngt << 16) | neq, s_ws, &tot);
    uint32_t gtb = ex >> 16, eqb = ex & 0xffffu;      // before this thread, within the chunk
    int32_t *out = a.cand + (size_t)bh * a.stride + slot0;
    int32_t *dbg = a.dbg_cand ? a.dbg_cand + (size_t)bh * a.C + slot0 : nullptr;
    const int64_t room = a.C - (int64_t)slot0;
    // the chunk's candidates: every S > s* key and its first `quota` ties
    const uint32_t n_out = (tot >> 16) + min(tot & 0xffffu, quota);
    const bool stage = n_out <= (uint32_t)kCpStage;   // else each thread stores its own ids
    uint32_t slot = gtb + min(eqb, quota);
#pragma unroll
    for (int u = 0; u < kCpMaxU; u++) {
        if (u >= U) break;
        uint32_t e = eqm[u];
        const uint32_t allow = eqb < quota ? quota - eqb : 0u;    // ties this group may still take
        if ((uint32_t)__popc(e) > allow)   // keep the lowest `allow` ties
            e = allow ? (e & (((1u << __fns(e, 0, (int)allow)) << 1) - 1u)) : 0u;
        eqb += __popc(eqm[u]);
        uint32_t m = gtm[u] | e;
        const int32_t k0 = (int32_t)(t0 + 16 * u);
        while (m) {
            const int bit = __ffs(m) - 1;
            if (stage) {
                s_ids[slot] = k0 + bit;
            } else if ((int64_t)slot < room) {
                out[slot] = k0 + bit;
                if (dbg) dbg[slot] = k0 + bit;
            }
            slot++;
            m &= m - 1;
        }
    }
    if (tid == kCpThreads - 1 && (int64_t)slot > room)
        devchk(a.dev_err, nullptr, DEVCHK_CAND_COUNT, (long long)slot0);
    if (stage) {                                  // consecutive threads store consecutive slots
        __syncthreads();
        const uint32_t lim = room <= 0 ? 0u : ((int64_t)n_out < room ? n_out : (uint32_t)room);
        for (uint32_t i = tid; i < lim; i += kCpThreads) {
            out[i] = s_ids[i];
            if (dbg) dbg[i] = s_ids[i];
        }
    }
    pdl_trigger();
}

cudaError_t launch_compact(const CompactArgs &a, int nchunks, int bh, cudaStream_t s)
{
    return launch_pdl(k_compact, dim3(nchunks, bh), dim3(kCpThreads), 0, s, a);
}

}  // namespace pk
