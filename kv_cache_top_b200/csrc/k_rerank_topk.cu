// k_rerank_topk.cu -- 4-bit RSQ-IP rerank of the candidates and the Top-k.
//
// Estimate (ParisKV slides, Sec. 4.2.3 Eqs. 7-10):
//     <k_i, q>^ = ||q|| sum_b w_{i,b} sum_j sigma_{i,b,j} l_{t_{i,b,j}} q~_{b,j}
// read from the key's 128-byte summary record: every factor that depends on
// the key alone is stored at encode time, so scoring a candidate touches no
// full-precision key.
//
// Work is split by candidate slices (not key ranges), so every CTA reranks
// the same number of records wherever the candidates sit; a CTA has 256 or
// 128 threads, whichever one-wave split loads the busiest SM with fewer
// records.  A CTA stages its candidate ids in shared memory (in the slots
// that later hold the keys); each warp streams its records into a
// private multi-stage shared-memory ring with asynchronous 16-byte copies
// (several stages in flight per warp, no registers held), and four lanes
// decode a record, each taking one 32-byte group (the nibbles of 4 blocks and
// their 4 weights, 32 coordinates) with no exchange.  The signed level of a
// nibble comes from a 16-entry shared table (at most 16 distinct words per
// request: no bank conflicts), addressed by one byte permute per coordinate;
// q~ stays in registers.  The kernel is issue-bound, so the layout minimises
// instructions per record.
//
// Scores never leave the chip: the CTA turns (score, id) into 64-bit keys
// ordered by score desc then id asc, selects its slice's Top-k set in one
// counting pass over value-linear bins (radix select as the fallback), and
// writes it sorted; a merge kernel (one CTA per pair) merges the sorted
// per-slice lists into the final Top-k with a tree of pairwise merges
// (bitonic warp merges in registers for k <= 128, merge-path runs in shared
// memory otherwise)
// (README, pipeline step 2: one fused kernel scores the candidates with the
// 4-bit inner-product estimate and picks the final Top-k ids).
#include "pk_internal.cuh"
#include "pk_launch.cuh"
#include "pk_merge.cuh"

namespace pk {

constexpr int kRrThreads = 256;                  // the merge CTA; a rerank CTA has NT = 256 or 128
constexpr int kRrWarps = kRrThreads / 32;

// Signed level x query coordinate, one 16-entry table per coordinate j:
//     tab[tab_index(j, c)] = sigma(c) l_{c & 7} q~_j,   sigma(c) = -1 iff c & 8,
// placed so that coordinates j and j + 64 (read at once by the two halves of a
// warp) sit in opposite halves of the 32 banks: entry (j, c) is word
// 32 (j & 63) + 16 (j >> 6) + c.
__host__ __device__ constexpr int tab_index(int j, int c) { return 32 * (j & 63) + 16 * (j >> 6) + c; }

struct RrShared {
    union {
        u64 tmp[kMaxTopk];        // the select's kept keys (after the decode)
        float tab[kD * 16];       // the decode's lookup tables
    };
    uint32_t hist[2][256];
    u64 red[2][kRrWarps];
    uint32_t sh[4];
    uint32_t cnt;
    uint32_t bcnt;
    int last;
};
static_assert(sizeof(u64) * kMaxTopk == sizeof(float) * kD * 16, "tab and tmp share storage");

// Warp-aggregated append: every lane with `want` gets a distinct slot of
// *ctr (one shared-memory atomic per warp instead of one per lane).
__device__ __forceinline__ uint32_t warp_append(uint32_t *ctr, bool want)
{
    const int lane = threadIdx.x & 31;
    const uint32_t bal = __ballot_sync(kFull, want);
    if (!bal) return 0u;
    const int leader = __ffs(bal) - 1;
    uint32_t base = 0;
    if (lane == leader) base = atomicAdd(ctr, (uint32_t)__popc(bal));
    base = __shfl_sync(kFull, base, leader);
    return base + (uint32_t)__popc(bal & ((1u << lane) - 1u));
}

// One warp sorts up to 32 keys (one per lane, missing ones = 0) descending;
// returns the lane's key at its rank (rank = lane).
__device__ __forceinline__ u64 warp_sort32_desc(u64 x)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const u64 y = __shfl_xor_sync(kFull, x, j);
            const bool lower = (lane & j) == 0, desc = (lane & k) == 0;
            const bool keep_max = (lower == desc);
            x = keep_max ? (x > y ? x : y) : (x < y ? x : y);
        }
    }
    return x;
}

// Keep the k largest of keys[0..count) (count > k; keys distinct) in
// sm.tmp[0..k), any order; returns the smallest kept key.  Radix select, most
// significant digit first, starting at the highest bit where the keys differ
// (scores of one query share sign and exponent, so leading digits would put
// every key in one bin); histogram increments are aggregated per warp over
// lanes that hit the same bin.  Once the bin holding the k-th key has at most
// 32 keys, one warp sorts that bin and finishes.  All threads of the block
// must call it (NT threads).
template <int NT>
__device__ u64 block_topk_select(RrShared &sm, const u64 *keys, int count, int k)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    u64 lo = ~0ull, hi = 0ull;
    for (int i = tid; i < count; i += NT) {
        const u64 x = keys[i];
        lo = x < lo ? x : lo;
        hi = x > hi ? x : hi;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const u64 a = __shfl_xor_sync(kFull, lo, o), b = __shfl_xor_sync(kFull, hi, o);
        lo = a < lo ? a : lo;
        hi = b > hi ? b : hi;
    }
    if (lane == 0) {
        sm.red[0][warp] = lo;
        sm.red[1][warp] = hi;
    }
    for (int i = tid; i < 2 * 256; i += NT) (&sm.hist[0][0])[i] = 0u;
    if (tid == 0) {
        sm.sh[3] = 0;
        sm.bcnt = 0;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < (NT / 32); w++) {
        lo = sm.red[0][w] < lo ? sm.red[0][w] : lo;
        hi = sm.red[1][w] > hi ? sm.red[1][w] : hi;
    }
    const int hb = 63 - __clzll((long long)(lo ^ hi));      // highest differing bit
    u64 mask = (hb >= 63) ? 0ull : ~((2ull << hb) - 1ull);   // bits above hb: common to all keys
    u64 prefix = hi & mask;
    int need = k;
    int pass = 0;
    uint32_t inbin = 0;
    u64 bmask = 0, bprefix = 0;         // the boundary bin (valid when it is small)
    for (int top = hb; top >= 0; top -= 8, pass ^= 1) {
        const int width = top + 1 < 8 ? top + 1 : 8;
        const int shift = top + 1 - width;
        const uint32_t dmask = (1u << width) - 1u;
        uint32_t *H = sm.hist[pass];
        for (int base = 0; base < count; base += NT) {
            const int i = base + tid;
            bool act = false;
            uint32_t bin = 0xffffffffu;
            if (i < count) {
                const u64 x = keys[i];
                act = (x & mask) == prefix;
                if (act) bin = (uint32_t)(x >> shift) & dmask;
            }
            const uint32_t grp = __match_any_sync(kFull, bin);
            if (act && lane == __ffs(grp) - 1) atomicAdd(&H[bin], (uint32_t)__popc(grp));
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t hc[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                hc[i] = H[255 - 8 * lane - i];
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
                H[255 - 8 * lane - i] = 0u;     // ready for the pass after next
            }
        }
        __syncthreads();
        const uint32_t d = sm.sh[0], above = sm.sh[1];
        inbin = sm.sh[2];
        need -= (int)above;
        bprefix = prefix | ((u64)d << shift);
        bmask = mask | ((u64)dmask << shift);
        // keys strictly above the boundary bin stay in the (prefix, mask) test below
        if ((int)inbin == need || inbin <= 32u) break;
        prefix = bprefix;
        mask = bmask;
    }
    // keys in bins above the boundary bin: (x & mask) == prefix and x's digit > d,
    // i.e. (x & bmask) > bprefix; they are all kept.  Keys of the boundary bin
    // go to a side list when the bin is small.
    const bool small = (int)inbin != need;
    u64 mn = ~0ull;
    for (int base = 0; base < count; base += NT) {
        const int i = base + tid;
        u64 x = 0;
        bool above = false, inb = false;
        if (i < count) {
            x = keys[i];
            const u64 xm = x & bmask;
            // bmask covers mask, so (x & bmask) orders keys by their selected prefix
            above = small ? (xm > bprefix) : (xm >= bprefix);
            inb = small && xm == bprefix;
        }
        const uint32_t pos = warp_append(&sm.sh[3], above);
        if (above) {
            if (pos < (uint32_t)kMaxTopk) sm.tmp[pos] = x;
            mn = x < mn ? x : mn;
        }
        const uint32_t bpos = warp_append(&sm.bcnt, inb);
        if (inb && bpos < 32u) reinterpret_cast<u64 *>(sm.hist[pass ^ 1])[bpos] = x;
    }
    __syncthreads();
    if (small && warp == 0) {
        // sort the boundary bin (<= 32 keys) and keep its `need` best
        const uint32_t nb = sm.bcnt;
        u64 x = (lane < (int)nb) ? reinterpret_cast<const u64 *>(sm.hist[pass ^ 1])[lane] : 0ull;
        x = warp_sort32_desc(x);
        const uint32_t base = sm.sh[3];
        if (lane < need && base + lane < (uint32_t)kMaxTopk) sm.tmp[base + lane] = x;
        if (lane < need) mn = x < mn ? x : mn;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const u64 y = __shfl_xor_sync(kFull, mn, o);
        mn = y < mn ? y : mn;
    }
    __syncthreads();
    if (lane == 0) sm.red[0][warp] = mn;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < (NT / 32); w++) mn = sm.red[0][w] < mn ? sm.red[0][w] : mn;
    return mn;
}

// Keep the k largest of keys[0..count) (k < count <= kSelPer NT; keys
// distinct) in sm.tmp[0..k), any order, in one counting pass; [vmin, vmax]
// is the range of the keys' scores (the caller tracks it).  Scores of one
// query span both signs and a few octaves, so bits of the key spread them
// poorly; instead bin b(v) = min(255, floor((v - vmin) 256 / (vmax - vmin)))
// of the score v, which never decreases as the key grows, so every key in a
// bin above the boundary bin is kept.  The upper tail is sparse, so the bin
// holding the k-th key usually has a few keys; one warp sorts it.  Keys are
// held in registers, each warp histograms into its own 256 counters (hist:
// 1 KB of free scratch per warp), and placement is one block scan.  Returns
// false -- with nothing written to sm.tmp -- when the scores are all equal or
// the boundary bin holds more than 32 keys that must be split; the caller
// then runs the radix select.  All threads of the block call it.
template <int NT>
__device__ bool block_topk_select_linear(RrShared &sm, const u64 *keys, int count, int k, uint32_t *hist,
                                         float vmin, float vmax)
{
    constexpr int kPer = kSelPer;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    u64 x[kPer];
#pragma unroll
    for (int u = 0; u < kPer; u++) {
        const int i = tid + u * NT;
        x[u] = (i < count) ? keys[i] : 0ull;
    }
    uint32_t *wh = hist + warp * 256;             // this warp's own counters
#pragma unroll
    for (int i = 0; i < 8; i++) wh[lane + 32 * i] = 0u;
    __syncwarp();
    const float range = vmax - vmin;
    const float scale = 256.0f / range;
    if (!(range > 0.0f) || !(range < INFINITY) || !(scale < INFINITY)) {
        __syncthreads();
        return false;
    }
    auto bin_of = [&](u64 key) {
        const float v = unord_f32((uint32_t)(key >> 32));
        return min(255, (int)((v - vmin) * scale));
    };
#pragma unroll
    for (int u = 0; u < kPer; u++)
        if (tid + u * NT < count) atomicAdd(&wh[bin_of(x[u])], 1u);
    __syncthreads();
    // thread tid takes the BPT = 256 / NT bins 255 - BPT tid - i (i < BPT),
    // highest first: keys in higher bins by an exclusive scan of its sum
    static_assert(NT == 128 || NT == 256, "one or two bins per thread");
    constexpr int BPT = 256 / NT;
    uint32_t hb[BPT], hv = 0;
#pragma unroll
    for (int i = 0; i < BPT; i++) {
        hb[i] = 0u;
#pragma unroll
        for (int w = 0; w < (NT / 32); w++) hb[i] += hist[w * 256 + 255 - BPT * tid - i];
        hv += hb[i];
    }
    uint32_t tot;
    uint32_t above = block_excl_scan<NT>(hv, reinterpret_cast<uint32_t *>(&sm.hist[0][0]), &tot);
#pragma unroll
    for (int i = 0; i < BPT; i++) {
        if (above < (uint32_t)k && above + hb[i] >= (uint32_t)k) {
            sm.sh[0] = 255 - BPT * tid - i;
            sm.sh[1] = above;
            sm.sh[2] = hb[i];
        }
        above += hb[i];
    }
    if (tid == 0) {
        sm.sh[3] = 0u;
        sm.bcnt = 0u;
    }
    __syncthreads();
    const int bstar = (int)sm.sh[0];
    const int need = k - (int)sm.sh[1];
    const int inbin = (int)sm.sh[2];
    const bool small = inbin != need;          // the boundary bin must be split
    if (small && inbin > 32) {
        __syncthreads();
        return false;
    }
    u64 *side = reinterpret_cast<u64 *>(&sm.hist[1][0]);   // <= 32 keys
    // positions by one block scan of per-thread counts (kept keys in the
    // high half, boundary-bin keys in the low half), then plain stores
    uint32_t keepm = 0, inbm = 0;
#pragma unroll
    for (int u = 0; u < kPer; u++) {
        const bool live = tid + u * NT < count;
        const int bq = live ? bin_of(x[u]) : -1;
        if (live && (small ? bq > bstar : bq >= bstar)) keepm |= 1u << u;
        if (live && small && bq == bstar) inbm |= 1u << u;
    }
    uint32_t tot2;
    const uint32_t ex2 = block_excl_scan<NT>(((uint32_t)__popc(keepm) << 16) | (uint32_t)__popc(inbm),
                                                     reinterpret_cast<uint32_t *>(&sm.hist[0][0]), &tot2);
    uint32_t pos = ex2 >> 16, bp = ex2 & 0xffffu;
#pragma unroll
    for (int u = 0; u < kPer; u++) {
        if (keepm & (1u << u)) sm.tmp[pos++] = x[u];
        if (inbm & (1u << u)) side[bp++] = x[u];
    }
    if (tid == 0) sm.sh[3] = tot2 >> 16;
    __syncthreads();
    if (small && warp == 0) {
        u64 y = (lane < inbin) ? side[lane] : 0ull;
        y = warp_sort32_desc(y);
        const uint32_t base = sm.sh[3];
        if (lane < need) sm.tmp[base + lane] = y;
    }
    __syncthreads();
    return true;
}

__device__ __forceinline__ u64 make_key(float est, int32_t idx)
{
    return ((u64)ord_f32(__fadd_rn(est, 0.0f)) << 32) | (u64)(0xffffffffu - (uint32_t)idx);
}

// Descending rank of every key of v[0..m) (keys distinct): rank(x) =
// #{y in v : y > x}.  Every thread walks the whole list in step (broadcast
// shared-memory reads), so the pass costs m / blockDim compares per key and
// no barrier; it sorts and selects at once for small m.
template <int NT, typename Emit>
__device__ __forceinline__ void rank_by_count(const u64 *v, int m, Emit emit)
{
    for (int i0 = 0; i0 < m; i0 += NT) {
        const int i = i0 + (int)threadIdx.x;
        const u64 x = (i < m) ? v[i] : ~0ull;
        int r = 0;
#pragma unroll 4
        for (int j = 0; j < m; j++) r += (v[j] > x) ? 1 : 0;
        if (i < m) emit(r, x);
    }
}

// <v_b, q~_b> of one block from its 8 nibbles (one u32: byte i holds
// coordinates 2i and 2i + 1 in its low and high nibble).  lo / hi hold, per
// byte, 64 h + 4 x the low / high nibble (h = this lane's half of the warp),
// i.e. the byte offset of the entry inside the two-table slot of a coordinate
// pair; one byte permute per coordinate yields the address, and the 8 table
// entries are summed in a fixed order.  `tb` points at the slot of the
// block's first coordinate (tab + 32 x 8 bb words for block bb of the half).
__device__ __forceinline__ float block_dot(const float *tb, uint32_t nib, uint32_t hmask)
{
    const uint32_t lo = ((nib << 2) & 0x3c3c3c3cu) | hmask, hi = ((nib >> 2) & 0x3c3c3c3cu) | hmask;
    const char *base = reinterpret_cast<const char *>(tb);
    float x[8];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t o0 = __byte_perm(lo, 0u, 0x4440u + i), o1 = __byte_perm(hi, 0u, 0x4440u + i);
        x[2 * i] = *reinterpret_cast<const float *>(base + 128 * (2 * i) + o0);
        x[2 * i + 1] = *reinterpret_cast<const float *>(base + 128 * (2 * i + 1) + o1);
    }
    return ((x[0] + x[1]) + (x[2] + x[3])) + ((x[4] + x[5]) + (x[6] + x[7]));
}


// Merge of the per-slice Top-k lists of one pair into its final sorted
// Top-k.  Each list arrives sorted descending (zero = padding; real keys are
// distinct).  Lists of at most 128 keys merge by a tree of warp merges in
// registers (warp_merge_tree).  Otherwise, when the lists fit in shared
// memory, a tree of pairwise merges halves their number per level, each
// merge keeping its k best.  A level splits every merge's outputs into runs, about one per
// thread; a run starts at the co-rank of its first output d (merge path: the
// first d outputs are A[0..i) and B[0..d-i) for the i found by binary
// search) and merges sequentially from there, so a level costs one barrier
// whatever the score distribution.
// Larger inputs run in rounds of radix select that keep the best k seen.

// Lists s = 0..ns-1 of k keys at src + s k; returns the buffer holding the
// merged list (k keys).  src needs ns k keys, dst (ns + 1) / 2 k keys.  All
// NT threads of the block call it.
template <int NT>
__device__ const u64 *merge_tree(u64 *src, u64 *dst, int ns, int k)
{
    while (ns > 1) {
        const int np = (ns + 1) / 2;
        // about one run of R consecutive outputs per thread
        const int R = max(1, (np * k + NT - 1) / NT);
        const int rpm = (k + R - 1) / R;          // runs per merge
        for (int t = threadIdx.x; t < np * rpm; t += NT) {
            const int m = t / rpm, d0 = (t - m * rpm) * R, d1 = min(k, d0 + R);
            const u64 *A = src + (size_t)(2 * m) * k;
            u64 *out = dst + (size_t)m * k;
            if (2 * m + 1 >= ns) {
                for (int d = d0; d < d1; d++) out[d] = A[d];     // odd list out: carried up
            } else {
                const u64 *B = A + k;
                int lo = 0, hi = d0;              // d0 < k: the co-rank i is in [0, d0]
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (A[mid] > B[d0 - 1 - mid]) lo = mid + 1;
                    else hi = mid;
                }
                int i = lo, j = d0 - lo;
                u64 x = A[i], y = B[j];
                for (int d = d0; d < d1; d++) {   // sequential merge of the run
                    if (x > y) {
                        out[d] = x;
                        x = (++i < k) ? A[i] : 0ull;
                    } else {
                        out[d] = y;
                        y = (++j < k) ? B[j] : 0ull;
                    }
                }
            }
        }
        __syncthreads();
        u64 *t = src;
        src = dst;
        dst = t;
        ns = np;
    }
    return src;
}

// Per-warp ring of record stages.  The gather is latency-bound (random
// 128-byte records), so the ring is as deep as shared memory allows at the
// CTA's occupancy: 4 stages at 256 threads (2 CTAs per SM), 3 at 128 (4 per
// SM); stages - 1 of them are in flight while one is decoded.
__host__ __device__ constexpr int rr_stages(int nt) { return nt == 256 ? 4 : 3; }
constexpr int kRrStep = 16;                        // records per warp stage
constexpr int kRecSlot = 128;                      // shared-memory record slot, no padding
__host__ __device__ constexpr size_t rr_ring_bytes(int nt)
{
    return (size_t)(nt / 32) * rr_stages(nt) * kRrStep * kRecSlot;
}
// Byte offset of 16-byte chunk c of slot j in a stage: chunks are XOR-swizzled
// by the slot index, so 8 lanes reading (or writing) chunk c of 8 consecutive
// slots, or 8 chunks of one slot, hit 8 different 16-byte bank groups.
__device__ __forceinline__ int slot_off(int j, int c) { return j * kRecSlot + 16 * (c ^ (j & 7)); }

// NT = 256 (2 CTAs per SM) or 128 (4 CTAs per SM): the host takes the size
// whose one-wave split of the candidates loads the SMs more evenly.
template <int NT>
__global__ void __launch_bounds__(NT, 512 / NT) k_rerank_topk(RerankArgs a)
{
    constexpr int NW = NT / 32;
    extern __shared__ __align__(16) unsigned char s_dyn[];
    __shared__ RrShared sm;
    unsigned char *ring_all = s_dyn;                                   // [warps][stages][16][144]
    // [slice]: the candidate ids (low 32 bits) until a record is decoded, then its key
    u64 *keys = reinterpret_cast<u64 *>(s_dyn + rr_ring_bytes(NT));
    const int bh = blockIdx.y, sl = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.topk;
    const int64_t m0 = (int64_t)sl * a.slice;
    const int count = (int)min((int64_t)a.slice, a.C - m0);

    pdl_wait();                                   // candidates come from the compaction
    const int32_t *cand = a.cand + (size_t)bh * a.stride + m0;
    {   // count <= kSelPer NT: every id load of the thread in flight at once
        int32_t cv[kSelPer];
#pragma unroll
        for (int u = 0; u < kSelPer; u++) cv[u] = (tid + u * NT < count) ? cand[tid + u * NT] : 0;
#pragma unroll
        for (int u = 0; u < kSelPer; u++)
            if (tid + u * NT < count) keys[tid + u * NT] = (u64)(uint32_t)cv[u];
    }
    {   // the lookup tables: entry e of tab holds (j, c) with c = e & 15,
        // j = 64 ((e >> 4) & 1) + (e >> 5); one fp32 product each
        const float *qt = a.qt + (size_t)bh * kD;
#pragma unroll
        for (int u = 0; u < (kD * 16) / NT; u++) {
            const int e = tid + u * NT, c = e & 15, j = 64 * ((e >> 4) & 1) + (e >> 5);
            const float l = a.lv.lev[c & 7];
            sm.tab[e] = __fmul_rn((c & 8) ? -l : l, qt[j]);
        }
    }
    const int rr = lane & 15, half = lane >> 4;        // record of the step, half of it (8 blocks)
    const uint32_t hmask = half ? 0x40404040u : 0u;    // this half's tables: +64 bytes in each slot
    // this lane's four 16-byte chunks (nibbles, weights, nibbles, weights) of its record slot
    const int off0 = slot_off(rr, 4 * half), off1 = slot_off(rr, 4 * half + 1);
    const int off2 = slot_off(rr, 4 * half + 2), off3 = slot_off(rr, 4 * half + 3);
    const float qnorm = a.qnorm[bh];
    float vlo = INFINITY, vhi = -INFINITY;        // range of this lane's scores (the select's bins)
    const uint8_t *rec = a.rec + (size_t)index_pair(bh, a.kvg) * a.stride * kRecBytes;
    float *dest = a.dbg_est ? a.dbg_est + (size_t)bh * a.C + m0 : nullptr;
    __syncthreads();

    // Each warp streams its own records (warp w takes steps w, w + 8, ...,
    // 16 records per step) through a private ring of kRrStages shared-memory
    // stages: the copies of the next stages are in flight while one stage is
    // decoded.  Copies are coalesced: lane l moves 16-byte pieces l, l+32,
    // l+64, l+96 of the step's 2 KB.
    constexpr int kRrStages = rr_stages(NT);
    unsigned char *ring = ring_all + (size_t)warp * kRrStages * kRrStep * kRecSlot;
    const int nsteps = (count + kRrStep - 1) / kRrStep;
    auto issue = [&](int step_local, int stage) {
        const int r0 = (warp + step_local * NW) * kRrStep;
        if (r0 < count) {
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const int piece = lane + 32 * u;
                const int j = piece >> 3, c = piece & 7;
                const int r = r0 + j;
                if (r < count) {                      // keys[r] still holds the id: r is decoded later
                    const int32_t id = (int32_t)(uint32_t)keys[r];
                    cp_async16(ring + (size_t)stage * kRrStep * kRecSlot + slot_off(j, c),
                               rec + (size_t)id * kRecBytes + 16 * c);
                }
            }
        }
        cp_async_commit();                            // always one group per call
    };
    const int my_steps = (nsteps > warp) ? (nsteps - warp + NW - 1) / NW : 0;
#pragma unroll
    for (int s = 0; s < kRrStages - 1; s++) issue(s, s);
    for (int t = 0; t < my_steps; t++) {
        cp_async_wait<kRrStages - 2>();               // step t has landed (this lane's pieces)
        __syncwarp();                                 // ... and every lane's
        const int stage = t % kRrStages;
        const int r0 = (warp + t * NW) * kRrStep;
        const unsigned char *st = ring + (size_t)stage * kRrStep * kRecSlot;
        {
            // lanes rr and rr + 16 take the two halves (8 blocks each) of record rr
            const uint4 n0 = *reinterpret_cast<const uint4 *>(st + off0);
            const uint4 w0 = *reinterpret_cast<const uint4 *>(st + off1);
            const uint4 n1 = *reinterpret_cast<const uint4 *>(st + off2);
            const uint4 w1 = *reinterpret_cast<const uint4 *>(st + off3);
            float part = __fmul_rn(__uint_as_float(w0.x), block_dot(sm.tab + 256 * 0, n0.x, hmask));
            part = fmaf(__uint_as_float(w0.y), block_dot(sm.tab + 256 * 1, n0.y, hmask), part);
            part = fmaf(__uint_as_float(w0.z), block_dot(sm.tab + 256 * 2, n0.z, hmask), part);
            part = fmaf(__uint_as_float(w0.w), block_dot(sm.tab + 256 * 3, n0.w, hmask), part);
            part = fmaf(__uint_as_float(w1.x), block_dot(sm.tab + 256 * 4, n1.x, hmask), part);
            part = fmaf(__uint_as_float(w1.y), block_dot(sm.tab + 256 * 5, n1.y, hmask), part);
            part = fmaf(__uint_as_float(w1.z), block_dot(sm.tab + 256 * 6, n1.z, hmask), part);
            part = fmaf(__uint_as_float(w1.w), block_dot(sm.tab + 256 * 7, n1.w, hmask), part);
            part += __shfl_xor_sync(kFull, part, 16);
            const int r = r0 + rr;
            if (half == 0 && r < count) {
                const float est = qnorm * part;
                const float v = __fadd_rn(est, 0.0f);     // the score the key orders by
                vlo = fminf(vlo, v);
                vhi = fmaxf(vhi, v);
                keys[r] = make_key(est, (int32_t)(uint32_t)keys[r]);
                if (dest) dest[r] = est;
            }
        }
        __syncwarp();                                 // stage consumed before it is refilled
        issue(t + kRrStages - 1, (t + kRrStages - 1) % kRrStages);
    }
    cp_async_wait<0>();
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        vlo = fminf(vlo, __shfl_xor_sync(kFull, vlo, o));
        vhi = fmaxf(vhi, __shfl_xor_sync(kFull, vhi, o));
    }
    float *red = reinterpret_cast<float *>(&sm.red[0][0]);
    if (lane == 0) {
        red[warp] = vlo;
        red[NW + warp] = vhi;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < NW; w++) {
        vlo = fminf(vlo, red[w]);
        vhi = fmaxf(vhi, red[NW + w]);
    }

    // ---- Top-k set of the slice (unordered) and its smallest key
    const int have = min(count, k);
    if (count > k) {
        // the ring is free now: NW KB of it hold the per-warp histograms
        if (!block_topk_select_linear<NT>(sm, keys, count, k, reinterpret_cast<uint32_t *>(ring_all), vlo, vhi))
            block_topk_select<NT>(sm, keys, count, k);
    } else {
        for (int i = tid; i < count; i += NT) sm.tmp[i] = keys[i];
        __syncthreads();
    }
    // the slice's set, sorted descending (zeros pad a slice shorter than k)
    u64 *part = a.partial + ((size_t)bh * a.max_slices + sl) * a.topk_cap;
    rank_by_count<NT>(sm.tmp, have, [&](int r, u64 x) { part[r] = x; });
    for (int i = have + tid; i < k; i += NT) part[i] = 0ull;
    pdl_trigger();
}

// keys the merge's dynamic shared memory holds for a list capacity cap
__host__ __device__ inline int64_t merge_keys(int cap) { return (int64_t)cap + (cap + 1) / 2 + 64 + 1024; }

__global__ void __launch_bounds__(kRrThreads) k_topk_merge(MergeArgs a)
{
    extern __shared__ __align__(16) unsigned char s_dyn[];
    __shared__ RrShared sm;
    u64 *keys = reinterpret_cast<u64 *>(s_dyn);
    const int bh = blockIdx.x;
    const int tid = threadIdx.x;
    const int k = a.topk;
    const int cap = a.cap;                     // keys[] capacity (>= 2k)
    pdl_wait();                                   // per-slice lists come from the rerank
    const int64_t total = (int64_t)a.nslices * k;
    const u64 *plist = a.partial + (size_t)bh * a.max_slices * a.topk_cap;
    const int ns = a.nslices;
    if (k <= 128 && (ns == 1 || warp_tree_keys(ns) <= merge_keys(cap))) {
        // lists of at most 128 keys: warp merges in registers
        const u64 *res = ns == 1 ? plist : warp_merge_tree<kRrWarps>(plist, a.topk_cap, true, ns, k, keys);
        if (tid < 32) {                          // keys in the result: one warp counts
            int got = 0;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const int e = 32 * j + tid;
                got += __popc(__ballot_sync(kFull, e < k && (ns == 1 ? __ldcg(res + e) : res[e]) != 0ull));
            }
            if (tid == 0 && got < k) devchk(a.dev_err, nullptr, DEVCHK_CAND_COUNT, got);
        }
        for (int d = tid; d < k; d += kRrThreads)
            emit_topk(a.out_idx, a.out_score, bh, k, d, ns == 1 ? __ldcg(res + d) : res[d]);
        __syncthreads();                          // release the attention only once every output is written
        pdl_trigger();
        return;
    }
    if (total <= cap) {
        constexpr int kLd = 16;                   // loads in flight per thread
        for (int e0 = 0; e0 < (int)total; e0 += kLd * kRrThreads) {
            u64 v[kLd];
#pragma unroll
            for (int u = 0; u < kLd; u++) {
                const int e = e0 + u * kRrThreads + tid;
                v[u] = 0ull;
                if (e < (int)total) {
                    const int sl = e / k, r = e - sl * k;
                    v[u] = plist[(size_t)sl * a.topk_cap + r];
                }
            }
#pragma unroll
            for (int u = 0; u < kLd; u++) {
                const int e = e0 + u * kRrThreads + tid;
                if (e < (int)total) keys[e] = v[u];
            }
        }
        __syncthreads();
        const u64 *res = merge_tree<kRrThreads>(keys, keys + cap, a.nslices, k);
        if (tid == 0 && res[k - 1] == 0ull) {
            int got = 0;
            while (got < k && res[got] != 0ull) got++;
            devchk(a.dev_err, nullptr, DEVCHK_CAND_COUNT, got);
        }
        for (int d = tid; d < k; d += kRrThreads) emit_topk(a.out_idx, a.out_score, bh, k, d, res[d]);
        pdl_trigger();
        return;
    }
    int cnt = 0;
    u64 tau = 0ull;
    for (int64_t e0 = 0; e0 < total; e0 += cap - k) {
        const int64_t e1 = min(total, e0 + (cap - k));
        if (tid == 0) sm.cnt = (uint32_t)cnt;
        __syncthreads();
        constexpr int kB8 = 8;       // loads in flight per thread
        for (int64_t eb = e0; eb < e1; eb += (int64_t)kB8 * kRrThreads) {
            u64 x[kB8];
#pragma unroll
            for (int u = 0; u < kB8; u++) {
                const int64_t e = eb + (int64_t)u * kRrThreads + tid;
                x[u] = 0ull;
                if (e < e1) {
                    const int64_t j = e / k, r = e - j * k;
                    x[u] = plist[(size_t)j * a.topk_cap + r];
                }
            }
#pragma unroll
            for (int u = 0; u < kB8; u++) {
                const bool take = x[u] != 0ull && x[u] > tau;
                const uint32_t pos = warp_append(&sm.cnt, take);
                if (take) keys[pos] = x[u];
            }
        }
        __syncthreads();
        cnt = (int)sm.cnt;
        if (cnt > k) {
            tau = block_topk_select<kRrThreads>(sm, keys, cnt, k);
            for (int i = tid; i < k; i += kRrThreads) keys[i] = sm.tmp[i];
            cnt = k;
            __syncthreads();
        }
    }
    const int got = min(cnt, k);
    if (got != k && tid == 0) devchk(a.dev_err, nullptr, DEVCHK_CAND_COUNT, got);
    rank_by_count<kRrThreads>(keys, got, [&](int r, u64 x) { emit_topk(a.out_idx, a.out_score, bh, k, r, x); });
    for (int i = got + tid; i < k; i += kRrThreads) emit_topk(a.out_idx, a.out_score, bh, k, i, 0ull);
    pdl_trigger();
}

// dynamic shared memory of the merge: cap keys for the lists, (cap + 1) / 2 + k
// for the first level of the merge tree
size_t merge_smem(int cap) { return (size_t)merge_keys(cap) * sizeof(u64); }

cudaError_t launch_topk_merge(const MergeArgs &a, int bh, cudaStream_t s)
{
    static std::atomic<int> smem_set[kMaxDevices];
    const size_t smem = merge_smem(a.cap);
    const cudaError_t e = dyn_smem_limit(k_topk_merge, (int)merge_smem(kMergeCap), smem_set);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_topk_merge, dim3(bh), dim3(kRrThreads), smem, s, a);
}

size_t rerank_smem(int slice, int nt) { return rr_ring_bytes(nt) + (size_t)slice * sizeof(u64); }

template <int NT>
cudaError_t launch_rerank_nt(const RerankArgs &a, int bh, cudaStream_t s)
{
    static std::atomic<int> smem_set[kMaxDevices];
    const size_t smem = rerank_smem(a.slice, NT);
    const cudaError_t e = dyn_smem_limit(k_rerank_topk<NT>, (int)rerank_smem(kSelPer * NT, NT), smem_set);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_rerank_topk<NT>, dim3(a.nslices, bh), dim3(NT), smem, s, a);
}

cudaError_t launch_rerank_topk(const RerankArgs &a, int bh, cudaStream_t s)
{
    if (a.slice > kSelPer * a.nt) return cudaErrorInvalidValue;
    return a.nt == 128 ? launch_rerank_nt<128>(a, bh, s) : launch_rerank_nt<256>(a, bh, s);
}

}  // namespace pk
