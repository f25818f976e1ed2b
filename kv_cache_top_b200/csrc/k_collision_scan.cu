// k_collision_scan.cu -- multi-tier collision counting and the integer Top-C
// threshold.
//
// S_i = sum_b bonus_b[code_{i,b}]  (ParisKV slides, "Stage I uses multi-tier
// collision votes to prune keys", App. B.2.1 Eq. 15), an integer in [0, 96].
// "Small integer scores allow histogram and prefix-scan selection instead of a
// full sort" (same frame): each CTA histograms the S of its chunk, and the
// last CTA of a pair to finish (ticket counter, no spin-wait) finds the
// threshold s* = max{s : #{S >= s} >= C}, and for every chunk the first slot of
// its candidates and how many of its S = s* keys it keeps (lower ids first),
// so the compaction kernel can place candidates in ascending id order without
// any further global synchronisation.
//
// Hot loop: 16 B of codes per key read with 128-bit streaming loads,
// double-buffered in registers (the next iteration's codes are in flight
// while the current ones are scored); the 16
// bonus tables (4 bits x 256 centres = one 32-bit register per lane per
// block) live in registers and are read with warp shuffles, which have no
// bank conflicts whatever the codes are.  Lane l's word of block b holds the
// bonus of centre 32 t + l in the 4 bits starting at bit 4 t + r(l), rotated
// by r(l) = (l >> 3) & 3, so a code byte c is used as it is: its low 5 bits
// pick the lane (the shuffle ignores higher bits), and bits 3..7 of c, i.e.
// 4 (c >> 5) + r(c & 31), are exactly the rotate amount that brings the
// bonus to bit 0 (a wrap-mode funnel shift ignores bits above 4) -- one shift
// of the code word per code.  Two extracted bonuses (each <= 6) are added
// before one mask, since their sum still fits in the low nibble.
#include "pk_internal.cuh"

namespace pk {

constexpr int kScanThreads = 256;
constexpr int kScanUnroll = 4;
constexpr int kHistPad = 104;

// Code byte 3 of every 32-bit code word (blocks 3, 7, 11 and 15) is looked up
// in a byte table in shared memory instead of the register tables: one shift
// and an LDS.U8 (at most two distinct words per bank: a 256-byte table spans
// 64 words), against a shuffle, two shifts, a rotate and half an add and a
// mask on the register path.  The split moves work from the integer ALU
// pipe, which bounds the all-register scan, to the load/store pipe; moving
// two or three bytes per word instead measured slower (bank conflicts and
// register spills at 4 CTAs per SM).
__device__ __forceinline__ uint32_t collision_score(const uint32_t (&tab)[kB], const uint8_t *btab, uint4 c)
{
    uint32_t s = 0;
    const uint32_t wds[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const uint32_t w = wds[q];
        // bytes 0..2: register tables by shuffles
        const uint32_t v0 = __shfl_sync(kFull, tab[4 * q + 0], (int)w);
        const uint32_t v1 = __shfl_sync(kFull, tab[4 * q + 1], (int)(w >> 8));
        const uint32_t v2 = __shfl_sync(kFull, tab[4 * q + 2], (int)(w >> 16));
        const uint32_t x0 = __funnelshift_r(v0, v0, w >> 3);
        const uint32_t x1 = __funnelshift_r(v1, v1, w >> 11);
        const uint32_t x2 = __funnelshift_r(v2, v2, w >> 19);
        // byte 3: the block's byte table in shared memory
        const uint32_t l3 = btab[256 * (4 * q + 3) + (w >> 24)];
        s += ((x0 + x1) & 0xfu) + (x2 & 0xfu) + l3;
    }
    return s;
}

__global__ void __launch_bounds__(kScanThreads, 4) k_collision_scan(ScanArgs a)
{
    const int bh = blockIdx.y, chunk = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kScanThreads / 32;
    __shared__ uint32_t s_hist[NW][kHistPad];
    __shared__ uint32_t s_cum[kHistPad];
    __shared__ uint32_t s_ws[NW + 1];
    __shared__ int s_last;
    __shared__ __align__(16) uint8_t s_btab[kB][kNC];   // bonus of (block, centre) for blocks 3, 7, 11, 15

    for (int i = tid; i < NW * kHistPad; i += kScanThreads) (&s_hist[0][0])[i] = 0u;

    pdl_wait();                                   // bonus tables come from the query preparation
    uint32_t tab[kB];
    const uint32_t *bp = a.bonus_packed + (size_t)bh * kB * 32;
#pragma unroll
    for (int b = 0; b < kB; b++) tab[b] = bp[b * 32 + lane];
    {   // byte tables of blocks 3, 7, 11, 15 (warps 3 and 7 build them): lane
        // l's word of block b holds the bonus of centre 32 t + l in bits 4 t..
        // after undoing its rotation by r(l)
        const uint32_t rl = (uint32_t)(lane >> 3) & 3u;
#pragma unroll
        for (int b = 0; b < kB; b++) {
            if ((b & 3) != 3 || (b & (NW - 1)) != warp) continue;
            const uint32_t plain = __funnelshift_r(tab[b], tab[b], rl);
#pragma unroll
            for (int t = 0; t < 8; t++) s_btab[b][32 * t + lane] = (uint8_t)((plain >> (4 * t)) & 0xfu);
        }
    }
    __syncthreads();

    const int64_t lo = (int64_t)chunk * a.chunk;
    const int64_t hi = min(lo + a.chunk, a.n);
    const int64_t cnt = hi - lo;
    const uint4 *codes = reinterpret_cast<const uint4 *>(a.codes + ((size_t)index_pair(bh, a.kvg) * a.n_cap + lo) * kB);
    uint8_t *S = a.S + (size_t)bh * a.n_cap + lo;
    uint8_t *dS = a.dbg_S ? a.dbg_S + (size_t)bh * a.n + lo : nullptr;

    // every lane runs every iteration (the shuffles need the full warp);
    // lanes past the end of the chunk compute on a zero code and store
    // nothing.  Offsets within the chunk are 32-bit (a chunk is < 2^31 keys),
    // and iterations that lie wholly inside the chunk skip the per-key checks.
    const uint32_t ucnt = (uint32_t)cnt;
    uint32_t *hw = s_hist[warp];
    // the next iteration's codes load while this one is scored (registers
    // double-buffered), so a warp always has a load in flight
    const uint32_t step = (uint32_t)NW * 32 * kScanUnroll;
    auto load = [&](uint32_t b, uint4 (&c)[kScanUnroll]) {
        if (b - lane + 32 * kScanUnroll <= ucnt) {
#pragma unroll
            for (int u = 0; u < kScanUnroll; u++) c[u] = __ldcs(codes + b + u * 32);
        } else {
#pragma unroll
            for (int u = 0; u < kScanUnroll; u++) {
                const uint32_t i = b + u * 32;
                c[u] = (i < ucnt) ? __ldcs(codes + i) : make_uint4(0, 0, 0, 0);
            }
        }
    };
    uint4 c[kScanUnroll], cn[kScanUnroll];
    uint32_t base = (uint32_t)warp * 32 * kScanUnroll + lane;
    if (base < ucnt + lane) load(base, c);
    for (; base < ucnt + lane; base += step) {
        const bool full = base - lane + 32 * kScanUnroll <= ucnt;
        if (base + step < ucnt + lane) load(base + step, cn);
        uint32_t sc[kScanUnroll];
#pragma unroll
        for (int u = 0; u < kScanUnroll; u++) sc[u] = collision_score(tab, &s_btab[0][0], c[u]);
        if (full) {
#pragma unroll
            for (int u = 0; u < kScanUnroll; u++) {
                S[base + u * 32] = (uint8_t)sc[u];
                atomicAdd(&hw[sc[u]], 1u);
            }
            if (dS) {
#pragma unroll
                for (int u = 0; u < kScanUnroll; u++) dS[base + u * 32] = (uint8_t)sc[u];
            }
        } else {
#pragma unroll
            for (int u = 0; u < kScanUnroll; u++) {
                const uint32_t i = base + u * 32;
                if (i < ucnt) {
                    S[i] = (uint8_t)sc[u];
                    if (dS) dS[i] = (uint8_t)sc[u];
                    atomicAdd(&hw[sc[u]], 1u);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kScanUnroll; u++) c[u] = cn[u];
    }
    __syncthreads();

    // chunk histogram -> suffix counts cum[s] = #{S >= s}, s = 0..97
    uint32_t hv = 0;
    if (tid < kBins) {
#pragma unroll
        for (int w = 0; w < NW; w++) hv += s_hist[w][tid];
    }
    if (tid < kHistPad) s_cum[tid] = (tid < kBins) ? hv : 0u;
    __syncthreads();
    // suffix sum by a reversed exclusive scan over 256 threads
    {
        const int s = kScanThreads - 1 - tid;   // thread tid handles bin s (descending)
        const uint32_t v = (s < kBins) ? s_cum[s] : 0u;
        uint32_t tot;
        const uint32_t ex = block_excl_scan<kScanThreads>(v, s_ws, &tot);
        if (s < kCum) a.chunk_cum[((size_t)bh * a.max_chunks + chunk) * kCum + s] = ex + v;
    }
    if (tid < kBins && hv) atomicAdd(&a.head_hist[(size_t)bh * kBins + tid], hv);

    __threadfence();
    __syncthreads();
    pdl_trigger();
    if (tid == 0) s_last = (atomicAdd(&a.tickets[(size_t)bh * 2 + 0], 1u) == (unsigned)(a.nchunks - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---- last CTA of this pair: threshold and per-chunk candidate slots
    uint32_t H = 0;
    if (tid < kBins) H = __ldcg(&a.head_hist[(size_t)bh * kBins + tid]);
    if (a.dbg_hist && tid < kBins) a.dbg_hist[(size_t)bh * kBins + tid] = H;
    int64_t cumH;
    {
        const int s = kScanThreads - 1 - tid;
        const uint32_t v = (s < kBins) ? __ldcg(&a.head_hist[(size_t)bh * kBins + s]) : 0u;
        uint32_t tot;
        const uint32_t ex = block_excl_scan<kScanThreads>(v, s_ws, &tot);
        cumH = (int64_t)(ex + v);           // #{S >= s} for s = 255 - tid
        // s* = largest s with #{S >= s} >= C  (cum is non-increasing in s)
        const int pred = (s < kCum) && (cumH >= a.C);
        const int nsat = __syncthreads_count(pred);
        if (tid == 0) s_last = nsat - 1;    // reuse as s*
    }
    __syncthreads();
    const int sstar = s_last;
    if (tid == 0) {
        a.sstar[bh] = sstar;
        if (a.dbg_sstar) a.dbg_sstar[bh] = sstar;
        a.tickets[(size_t)bh * 2 + 0] = 0u;
    }
    // gt_total = #{S > s*}, ties to take t = C - gt_total (1 <= t <= #{S = s*})
    __shared__ uint32_t s_gt_total;
    if (kScanThreads - 1 - tid == sstar + 1) s_gt_total = (uint32_t)cumH;   // s* + 1 <= 97
    __syncthreads();
    const int64_t ties = a.C - (int64_t)s_gt_total;
    uint32_t carry_eq = 0, carry_slot = 0;
    for (int j0 = 0; j0 < a.nchunks; j0 += kScanThreads) {
        const int j = j0 + tid;
        uint32_t gt = 0, eq = 0;
        if (j < a.nchunks) {
            const uint32_t *cj = a.chunk_cum + ((size_t)bh * a.max_chunks + j) * kCum;
            const uint32_t c0 = __ldcg(cj + sstar), c1 = __ldcg(cj + sstar + 1);
            gt = c1;
            eq = c0 - c1;
        }
        uint32_t tot_eq;
        const uint32_t ex_eq = carry_eq + block_excl_scan<kScanThreads>(eq, s_ws, &tot_eq);
        const int64_t room = ties - (int64_t)ex_eq;
        const uint32_t quota = room <= 0 ? 0u : (room >= (int64_t)eq ? eq : (uint32_t)room);
        uint32_t tot_slot;
        const uint32_t ex_slot = carry_slot + block_excl_scan<kScanThreads>(gt + quota, s_ws, &tot_slot);
        if (j < a.nchunks) a.chunk_info[(size_t)bh * a.max_chunks + j] = make_uint2(ex_slot, quota);
        carry_eq += tot_eq;
        carry_slot += tot_slot;
    }
}

}  // namespace pk

namespace pk {
cudaError_t launch_collision_scan(const ScanArgs &a, int bh, cudaStream_t s)
{
    return launch_pdl(k_collision_scan, dim3(a.nchunks, bh), dim3(kScanThreads), 0, s, a);
}
}  // namespace pk
