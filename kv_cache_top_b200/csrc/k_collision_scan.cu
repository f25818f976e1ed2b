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
#include "pk_launch.cuh"

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

// Chunk `chunk` of unit `unit`: thread tid < kBins holds hv = #{S = tid} in
// the chunk.  Writes the chunk's suffix counts #{S >= s}, s = 0..97, and adds
// the counts into the unit's histogram.  All kScanThreads threads call it.
__device__ __forceinline__ void chunk_suffix(const ScanArgs &a, int unit, int chunk, uint32_t hv, uint32_t *s_cum,
                                             uint32_t *s_ws)
{
    const int tid = threadIdx.x;
    if (tid < kHistPad) s_cum[tid] = (tid < kBins) ? hv : 0u;
    __syncthreads();
    // suffix sum by a reversed exclusive scan over the threads
    const int s = kScanThreads - 1 - tid;   // thread tid handles bin s (descending)
    const uint32_t v = (s < kBins) ? s_cum[s] : 0u;
    uint32_t tot;
    const uint32_t ex = block_excl_scan<kScanThreads>(v, s_ws, &tot);
    if (s < kCum) a.chunk_cum[((size_t)unit * a.max_chunks + chunk) * kCum + s] = ex + v;
    if (tid < kBins && hv) atomicAdd(&a.head_hist[(size_t)unit * kBins + tid], hv);
}

// The last CTA of a unit to finish its chunk: the threshold s* = largest s
// with #{S >= s} >= C, and for every chunk the first slot of its candidates
// and how many of its S = s* keys it keeps (lower ids first).  All threads
// call it; s_int and s_u32 are one shared word each.
__device__ __forceinline__ void unit_threshold(const ScanArgs &a, int unit, uint32_t *s_ws, int *s_int, uint32_t *s_u32)
{
    const int tid = threadIdx.x;
    uint32_t H = 0;
    if (tid < kBins) H = __ldcg(&a.head_hist[(size_t)unit * kBins + tid]);
    if (a.dbg_hist && tid < kBins) a.dbg_hist[(size_t)unit * kBins + tid] = H;
    int64_t cumH;
    {
        const int s = kScanThreads - 1 - tid;
        const uint32_t v = (s < kBins) ? __ldcg(&a.head_hist[(size_t)unit * kBins + s]) : 0u;
        uint32_t tot;
        const uint32_t ex = block_excl_scan<kScanThreads>(v, s_ws, &tot);
        cumH = (int64_t)(ex + v);           // #{S >= s} for s = 255 - tid
        // s* = largest s with #{S >= s} >= C  (cum is non-increasing in s)
        const int pred = (s < kCum) && (cumH >= a.C);
        const int nsat = __syncthreads_count(pred);
        if (tid == 0) *s_int = nsat - 1;
    }
    __syncthreads();
    const int sstar = *s_int;
    if (tid == 0) {
        a.sstar[unit] = sstar;
        if (a.dbg_sstar) a.dbg_sstar[unit] = sstar;
    }
    // gt_total = #{S > s*}, ties to take t = C - gt_total (1 <= t <= #{S = s*})
    if (kScanThreads - 1 - tid == sstar + 1) *s_u32 = (uint32_t)cumH;   // s* + 1 <= 97
    __syncthreads();
    const int64_t ties = a.C - (int64_t)*s_u32;
    uint32_t carry_eq = 0, carry_slot = 0;
    for (int j0 = 0; j0 < a.nchunks; j0 += kScanThreads) {
        const int j = j0 + tid;
        uint32_t gt = 0, eq = 0;
        if (j < a.nchunks) {
            const uint32_t *cj = a.chunk_cum + ((size_t)unit * a.max_chunks + j) * kCum;
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
        if (j < a.nchunks) a.chunk_info[(size_t)unit * a.max_chunks + j] = make_uint2(ex_slot, quota);
        carry_eq += tot_eq;
        carry_slot += tot_slot;
    }
    __syncthreads();                          // s_ws, s_int, s_u32 free for the next unit
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

    // chunk histogram -> suffix counts
    uint32_t hv = 0;
    if (tid < kBins) {
#pragma unroll
        for (int w = 0; w < NW; w++) hv += s_hist[w][tid];
    }
    chunk_suffix(a, bh, chunk, hv, s_cum, s_ws);

    __threadfence();
    __syncthreads();
    pdl_trigger();
    if (tid == 0) s_last = (atomicAdd(&a.tickets[(size_t)bh * 2 + 0], 1u) == (unsigned)(a.nchunks - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // ---- last CTA of this pair: threshold and per-chunk candidate slots
    __shared__ uint32_t s_gt_total;
    unit_threshold(a, bh, s_ws, &s_last, &s_gt_total);
    if (tid == 0) a.tickets[(size_t)bh * 2 + 0] = 0u;
}

// ---------------------------------------------------------------------------
// One warp's versions of chunk_suffix and unit_threshold, so that the G units
// of a pair run side by side, one warp each.  Lane l holds bins 4 l .. 4 l + 3;
// the suffix over lanes is a shuffle-down scan.

// inclusive suffix sum over lanes: the sum of t over lanes >= this lane
__device__ __forceinline__ uint32_t warp_suffix_incl(uint32_t t)
{
    const int lane = threadIdx.x & 31;
    uint32_t x = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(kFull, x, o);
        if (lane + o < 32) x += y;
    }
    return x;
}

// inclusive prefix sum over lanes
__device__ __forceinline__ uint32_t warp_prefix_incl(uint32_t t)
{
    const int lane = threadIdx.x & 31;
    uint32_t x = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// chunk_suffix for one unit by one warp: hist[w * wstride + s] = #{S = s} of
// warp w's keys, w < nw.
__device__ __forceinline__ void warp_chunk_suffix(const ScanArgs &a, int unit, int chunk, const uint32_t *hist,
                                                  int wstride, int nw)
{
    const int lane = threadIdx.x & 31;
    uint32_t h[4], t = 0;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const int s = 4 * lane + k;
        h[k] = 0u;
        if (s < kBins)
            for (int w = 0; w < nw; w++) h[k] += hist[w * wstride + s];
        t += h[k];
    }
    uint32_t c = warp_suffix_incl(t) - t;        // #{S >= 4 lane + 4}
    uint32_t *out = a.chunk_cum + ((size_t)unit * a.max_chunks + chunk) * kCum;
#pragma unroll
    for (int k = 3; k >= 0; k--) {
        const int s = 4 * lane + k;
        c += h[k];
        if (s < kCum) out[s] = c;
        if (s < kBins && h[k]) atomicAdd(&a.head_hist[(size_t)unit * kBins + s], h[k]);
    }
}

// unit_threshold for one unit by one warp
__device__ __forceinline__ void warp_unit_threshold(const ScanArgs &a, int unit)
{
    const int lane = threadIdx.x & 31;
    uint32_t h[4], t = 0;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const int s = 4 * lane + k;
        h[k] = (s < kBins) ? __ldcg(&a.head_hist[(size_t)unit * kBins + s]) : 0u;
        if (a.dbg_hist && s < kBins) a.dbg_hist[(size_t)unit * kBins + s] = h[k];
        t += h[k];
    }
    uint32_t cum[4];
    {
        uint32_t c = warp_suffix_incl(t) - t;
#pragma unroll
        for (int k = 3; k >= 0; k--) { c += h[k]; cum[k] = c; }
    }
    // s* = largest s with #{S >= s} >= C: the number of such s, less one
    int nsat = 0;
#pragma unroll
    for (int k = 0; k < 4; k++) nsat += (4 * lane + k < kCum) && ((int64_t)cum[k] >= a.C);
    const int sstar = __reduce_add_sync(kFull, (unsigned)nsat) - 1;
    if (lane == 0) {
        a.sstar[unit] = sstar;
        if (a.dbg_sstar) a.dbg_sstar[unit] = sstar;
    }
    // gt_total = #{S > s*} = cum[s* + 1], from the lane that holds bin s* + 1
    const int s1 = sstar + 1, k1 = s1 & 3;
    const uint32_t mine = k1 == 0 ? cum[0] : k1 == 1 ? cum[1] : k1 == 2 ? cum[2] : cum[3];
    const uint32_t gt_total = __shfl_sync(kFull, mine, s1 >> 2);
    const int64_t ties = a.C - (int64_t)gt_total;
    uint32_t carry_eq = 0, carry_slot = 0;
    for (int j0 = 0; j0 < a.nchunks; j0 += 32) {
        const int j = j0 + lane;
        uint32_t gt = 0, eq = 0;
        if (j < a.nchunks) {
            const uint32_t *cj = a.chunk_cum + ((size_t)unit * a.max_chunks + j) * kCum;
            const uint32_t c0 = __ldcg(cj + sstar), c1 = __ldcg(cj + sstar + 1);
            gt = c1;
            eq = c0 - c1;
        }
        const uint32_t in_eq = warp_prefix_incl(eq);
        const int64_t room = ties - (int64_t)(carry_eq + in_eq - eq);
        const uint32_t quota = room <= 0 ? 0u : (room >= (int64_t)eq ? eq : (uint32_t)room);
        const uint32_t in_slot = warp_prefix_incl(gt + quota);
        if (j < a.nchunks)
            a.chunk_info[(size_t)unit * a.max_chunks + j] = make_uint2(carry_slot + in_slot - (gt + quota), quota);
        carry_eq += __shfl_sync(kFull, in_eq, 31);
        carry_slot += __shfl_sync(kFull, in_slot, 31);
    }
}

// ---------------------------------------------------------------------------
// Per-query-head retrieval: one pass over a pair's codes scores it for all G
// query heads of the pair (units pair G + g).  The G bonus tables are packed
// into one table per (block, centre) in shared memory -- NP words, byte g of
// word p holding the bonus of head 4p + g -- so one lookup per code yields the
// bonuses of every head, and summing the 16 words of a key gives every head's
// S in its own byte (S <= 96: no carry between bytes).  Then each head's S,
// histogram, suffix counts and threshold go through the same steps as the
// single-query scan, one warp per head.  The prep writes the packed table
// ([pairs][16][256][NP] words), so the CTA loads it with 16-byte loads.
template <int NP>
__global__ void __launch_bounds__(kScanThreads, 4) k_collision_scan_heads(ScanArgs a)
{
    const int pair = blockIdx.y, chunk = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kScanThreads / 32;
    const int G = a.kvg;
    const int u0 = pair * G;                      // the pair's first query unit
    extern __shared__ __align__(16) uint32_t s_dyn[];
    uint32_t *ptab = s_dyn;                       // [kB * kNC][NP]
    uint32_t *s_hist = s_dyn + kB * kNC * NP;     // [NW][G][kHistPad]
    __shared__ int s_last;

    for (int i = tid; i < NW * G * kHistPad; i += kScanThreads) s_hist[i] = 0u;
    pdl_wait();                                   // bonus tables come from the query preparation
    {   // the pair's packed table, written so by the query preparation
        const uint4 *src = reinterpret_cast<const uint4 *>(a.bonus_bytes + (size_t)pair * kB * kNC * 4 * NP);
        uint4 *dst = reinterpret_cast<uint4 *>(ptab);
        constexpr int kVec = kB * kNC * NP / 4;
        uint4 v[kVec / kScanThreads];
#pragma unroll
        for (int u = 0; u < kVec / kScanThreads; u++) v[u] = __ldcg(src + tid + u * kScanThreads);
#pragma unroll
        for (int u = 0; u < kVec / kScanThreads; u++) dst[tid + u * kScanThreads] = v[u];
    }
    __syncthreads();

    const int64_t lo = (int64_t)chunk * a.chunk;
    const int64_t hi = min(lo + a.chunk, a.n);
    const uint32_t ucnt = (uint32_t)(hi - lo);
    const uint4 *codes = reinterpret_cast<const uint4 *>(a.codes + ((size_t)pair * a.n_cap + lo) * kB);
    uint8_t *S0 = a.S + (size_t)u0 * a.n_cap + lo;
    uint32_t *hw = s_hist + warp * G * kHistPad;
    constexpr int U = kScanUnroll;                // keys per lane per iteration
    const uint32_t step = (uint32_t)NW * 32 * U;
    // the next iteration's codes load while this one is scored
    auto load = [&](uint32_t b, uint4 (&c)[U]) {
#pragma unroll
        for (int u = 0; u < U; u++) {
            const uint32_t i = b + u * 32;
            c[u] = (i < ucnt) ? __ldcs(codes + i) : make_uint4(0, 0, 0, 0);
        }
    };
    uint4 c[U], cn[U];
    uint32_t base = (uint32_t)warp * 32 * U + lane;
    if (base < ucnt + lane) load(base, c);
    for (; base < ucnt + lane; base += step) {
        if (base + step < ucnt + lane) load(base + step, cn);
#pragma unroll
        for (int u = 0; u < U; u++) {
            const uint32_t i = base + u * 32;
            uint32_t acc[NP];
#pragma unroll
            for (int p = 0; p < NP; p++) acc[p] = 0u;
            const uint32_t wds[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
#pragma unroll
            for (int q = 0; q < 4; q++) {
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const uint32_t e = (uint32_t)(256 * (4 * q + k)) + ((wds[q] >> (8 * k)) & 0xffu);
                    if (NP == 1) {
                        acc[0] += ptab[e];
                    } else {
                        const uint2 v = reinterpret_cast<const uint2 *>(ptab)[e];
                        acc[0] += v.x;
                        acc[NP - 1] += v.y;
                    }
                }
            }
            if (i < ucnt) {
                for (int g = 0; g < G; g++) {
                    const uint32_t sg = (acc[g >> 2] >> (8 * (g & 3))) & 0xffu;
                    S0[(size_t)g * a.n_cap + i] = (uint8_t)sg;
                    atomicAdd(&hw[g * kHistPad + sg], 1u);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; u++) c[u] = cn[u];
    }
    __syncthreads();

    for (int g = warp; g < G; g += NW) warp_chunk_suffix(a, u0 + g, chunk, s_hist + g * kHistPad, G * kHistPad, NW);
    __threadfence();
    __syncthreads();
    pdl_trigger();
    if (tid == 0) s_last = (atomicAdd(&a.tickets[(size_t)u0 * 2 + 0], 1u) == (unsigned)(a.nchunks - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int g = warp; g < G; g += NW) warp_unit_threshold(a, u0 + g);
    if (tid == 0) a.tickets[(size_t)u0 * 2 + 0] = 0u;
}

}  // namespace pk

namespace pk {
cudaError_t launch_collision_scan(const ScanArgs &a, int bh, cudaStream_t s)
{
    return launch_pdl(k_collision_scan, dim3(a.nchunks, bh), dim3(kScanThreads), 0, s, a);
}

size_t scan_heads_smem(int np, int G) { return ((size_t)kB * kNC * np + (size_t)(kScanThreads / 32) * G * kHistPad) * 4; }

cudaError_t launch_collision_scan_heads(const ScanArgs &a, int pairs, cudaStream_t s)
{
    static std::atomic<int> set1[kMaxDevices], set2[kMaxDevices];
    if (a.kvg <= 4) {
        const cudaError_t e = dyn_smem_limit(k_collision_scan_heads<1>, (int)scan_heads_smem(1, 4), set1);
        if (e != cudaSuccess) return e;
        return launch_pdl(k_collision_scan_heads<1>, dim3(a.nchunks, pairs), dim3(kScanThreads),
                          scan_heads_smem(1, a.kvg), s, a);
    }
    const cudaError_t e = dyn_smem_limit(k_collision_scan_heads<2>, (int)scan_heads_smem(2, kMaxGroup), set2);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_collision_scan_heads<2>, dim3(a.nchunks, pairs), dim3(kScanThreads),
                      scan_heads_smem(2, a.kvg), s, a);
}
}  // namespace pk
