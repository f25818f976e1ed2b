// k_query_prep.cu -- per (sequence, KV head) query preparation.
//
// (1) GQA aggregation q_agg = ((q_0 + q_1) + ..) + q_{G-1} in fp32, then the
//     canonical normalise + SRHT rotate (ParisKV slides, Eq. 5).
// (2) Stage I bucket tiers (slides, Sec. 4.2.2 / App. B.2.1 Eq. 15; README,
//     pipeline step 2: per subspace, the centroids nearest the query's
//     direction are the active ones): in block b every
//     sign-pattern centre c gets the score L_b(c) = sum_j +-q~_{b,j} (minus
//     where bit j of c is set; the 1/sqrt(m) factor does not change the order),
//     the 256 centres are ranked by (L desc, c asc), P(c) = number of keys in
//     better-ranked buckets (from the occupancy table), and a bucket inside
//     the top-rho fraction (P(c) < R = ceil(rho n)) gets bonus 6 - floor(6P/R).
//
// Grid (2, pairs): a CTA of 8 warps takes 8 blocks, one warp per block, so
// a block's ranking needs no block barrier.  Warp 0 aggregates and rotates
// the query once per CTA and shares it through shared memory.  Flipping all 8
// signs of a centre negates its score exactly (fp32 addition is symmetric
// under negation), so the 128 centres with bit 7 clear are sorted -- 4 keys
// per lane, in registers and shuffles -- and the other 128 are their mirror
// images in reverse order: the 256 keys then form an ascending run followed
// by a descending one, and one 8-stage bitonic merge ranks them all.  A warp
// scan turns bucket sizes in rank order into P(c), and the warp packs the
// bonus table 4 bits per centre in the layout the collision scan keeps in
// registers -- lane l's word holds the bonus of centre 32 t + l in the 4 bits
// starting at bit (4 t + r(l)) mod 32, r(l) = (l >> 3) & 3.  With few pairs
// the SMs have room for more parallelism per block, and k_query_prep_wide
// (4 warps per block) runs instead; the host chooses.  For per-query-head
// search each unit is one query head, and the prep also writes every bonus
// as byte g of the word (block, centre) of its pair's table, g = the head's
// index in its group, which the per-head scan copies whole into shared memory.
#include "pk_internal.cuh"

namespace pk {

constexpr int kQpWarps = 8;                   // blocks per CTA, one warp each
constexpr int kQpThreads = 32 * kQpWarps;

// the 4-warp layout (k_query_prep_wide)
constexpr int kQpHalf = 128;                  // threads per block of centres
constexpr int kQpBlocks = 2;                  // blocks per CTA
constexpr int kQwThreads = kQpHalf * kQpBlocks;
constexpr int kQwWarps = kQwThreads / 32;

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ void load_heads(float (&qv)[4][kMaxGroup], const T *qp, int G, int lane)
{
#pragma unroll
    for (int r = 0; r < 4; r++)
#pragma unroll
        for (int g = 0; g < kMaxGroup; g++) {
            const int gg = g < G ? g : G - 1;          // in bounds; unused when g >= G
            qv[r][g] = to_f32(qp[lane + 32 * r + gg * kD]);
        }
}

// The G query heads of a unit (rows of kD at q + base): qv[r][g] = q_g[lane + 32 r].
// When the rows start on a 16-byte boundary the warp reads them with 16-byte
// loads into `stage` ([kMaxGroup][kD] fp32, shared) and picks its elements
// from there: one request per 16 bytes, which matters when q sits in host
// memory.  Otherwise one element per load.  The values are the same either way.
__device__ __forceinline__ void load_query(float (&qv)[4][kMaxGroup], const PrepArgs &a, int64_t base, int lane,
                                           float *stage)
{
    const int G = a.G;
    const uintptr_t at = reinterpret_cast<uintptr_t>(a.q) + (uintptr_t)base * (a.is_bf16 ? 2u : 4u);
    if ((at & 15u) != 0) {
        if (a.is_bf16)
            load_heads(qv, reinterpret_cast<const __nv_bfloat16 *>(a.q) + base, G, lane);
        else
            load_heads(qv, reinterpret_cast<const float *>(a.q) + base, G, lane);
        return;
    }
    if (a.is_bf16) {
        const uint4 *src = reinterpret_cast<const uint4 *>(at);
        for (int v = lane; v < G * kD / 8; v += 32) {         // element 8 v of the rows
            const uint4 x = src[v];
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
            float4 lo, hi;
            float2 f;
            f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[0])); lo.x = f.x; lo.y = f.y;
            f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[1])); lo.z = f.x; lo.w = f.y;
            f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[2])); hi.x = f.x; hi.y = f.y;
            f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[3])); hi.z = f.x; hi.w = f.y;
            reinterpret_cast<float4 *>(stage)[2 * v] = lo;
            reinterpret_cast<float4 *>(stage)[2 * v + 1] = hi;
        }
    } else {
        const float4 *src = reinterpret_cast<const float4 *>(at);
        for (int v = lane; v < G * kD / 4; v += 32) reinterpret_cast<float4 *>(stage)[v] = src[v];
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 4; r++)
#pragma unroll
        for (int g = 0; g < kMaxGroup; g++) {
            const int gg = g < G ? g : G - 1;          // in bounds; unused when g >= G
            qv[r][g] = stage[gg * kD + lane + 32 * r];
        }
}

// per-query-head search: where unit bh's bonus of centre c of block b goes
// in its pair's packed table (byte g of the entry, g = bh % kvg)
__device__ __forceinline__ uint8_t *head_bonus_ptr(const PrepArgs &a, int bh, int b, int c)
{
    const int pair = bh / a.kvg, g = bh - pair * a.kvg;
    return a.bonus_heads + (((size_t)pair * kB + b) * kNC + c) * (4 * a.heads_np) + 4 * (g >> 2) + (g & 3);
}

__device__ __forceinline__ uint32_t tier_bonus(uint32_t P, unsigned long long R)
{
    // 6 - floor(6P/R) for P < R, else 0: floor(6P/R) = #{j = 1..5 : 6P >= jR},
    // exact in integers without a division
    if ((unsigned long long)P >= R) return 0u;
    const unsigned long long p6 = 6ull * P;
    return 6u - (uint32_t)(p6 >= R) - (uint32_t)(p6 >= 2 * R) - (uint32_t)(p6 >= 3 * R) -
           (uint32_t)(p6 >= 4 * R) - (uint32_t)(p6 >= 5 * R);
}

typedef unsigned long long u64;

// sort key of a centre: ascending key order = rank order (score desc, id asc)
__device__ __forceinline__ u64 centre_key(float L, uint32_t c)
{
    return ((u64)(~ord_f32(__fadd_rn(L, 0.0f))) << 8) | c;   // +0 folds -0: equal scores tie
}

// the key of the mirror centre c ^ 0xff, whose score is exactly -L
__device__ __forceinline__ u64 mirror_key(u64 key)
{
    const float L = unord_f32(~(uint32_t)(key >> 8));
    return centre_key(-L, (uint32_t)(key & 0xffu) ^ 0xffu);
}

__device__ __forceinline__ void cmp_swap(u64 &lo, u64 &hi, bool up)
{
    const u64 a = lo < hi ? lo : hi, b = lo < hi ? hi : lo;
    lo = up ? a : b;
    hi = up ? b : a;
}

__global__ void __launch_bounds__(kQpThreads) k_query_prep(PrepArgs a)
{
    const int bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = kQpWarps * blockIdx.x + warp;              // this warp's block
    const int b_seq = bh / a.H, h = bh - b_seq * a.H;
    __shared__ __align__(16) uint32_t s_occ[kQpWarps][kNC];
    __shared__ float s_x[kD];
    __shared__ uint8_t s_bonus[kQpWarps][kNC];
    __shared__ __align__(16) float s_qs[kMaxGroup * kD];

    if (blockIdx.x == 0) {   // reset the per-call counters of the collision scan and the rerank
        for (int i = tid; i < kBins; i += kQpThreads) a.head_hist[(size_t)bh * kBins + i] = 0u;
        if (tid < 2) a.tickets[(size_t)bh * 2 + tid] = 0u;
    }
    // global loads first: 8 bucket sizes per lane; warp 0 the G query heads
    const uint4 *occ = reinterpret_cast<const uint4 *>(a.occ + ((size_t)index_pair(bh, a.kvg) * kB + b) * kNC);
    const uint4 o0 = occ[2 * lane], o1 = occ[2 * lane + 1];
    if (warp == 0) {
        float qv[4][kMaxGroup];
        const int64_t base = ((int64_t)b_seq * a.H * a.G + (int64_t)h * a.G) * kD;
        load_query(qv, a, base, lane, s_qs);
        float x[4];
#pragma unroll
        for (int r = 0; r < 4; r++) {
            float acc = qv[r][0];
#pragma unroll
            for (int g = 1; g < kMaxGroup; g++)
                if (g < a.G) acc = __fadd_rn(acc, qv[r][g]);
            x[r] = acc;
        }
        const float nrm = warp_rotate128(x, a.rot, lane);
#pragma unroll
        for (int r = 0; r < 4; r++) s_x[lane + 32 * r] = x[r];
        if (blockIdx.x == 0) {
#pragma unroll
            for (int r = 0; r < 4; r++) {
                a.qt[(size_t)bh * kD + lane + 32 * r] = x[r];
                if (a.dbg_qt) a.dbg_qt[(size_t)bh * kD + lane + 32 * r] = x[r];
            }
            if (lane == 0) {
                a.qnorm[bh] = nrm;
                if (a.dbg_qnorm) a.dbg_qnorm[bh] = nrm;
            }
        }
    }
    reinterpret_cast<uint4 *>(s_occ[warp])[2 * lane] = o0;
    reinterpret_cast<uint4 *>(s_occ[warp])[2 * lane + 1] = o1;
    __syncthreads();
    float xq[kM];
#pragma unroll
    for (int j = 0; j < kM; j++) xq[j] = s_x[kM * b + j];

    // the 128 centres with bit 7 clear, element e = 4 lane + i holding centre e;
    // L(c) = sum_j +-q~_j (minus where bit j of c is set), summed in j order
    u64 v[8];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint32_t c = 4 * lane + i;
        float L = 0.0f;
#pragma unroll
        for (int j = 0; j < kM; j++) L = __fadd_rn(L, ((c >> j) & 1) ? -xq[j] : xq[j]);
        v[i] = centre_key(L, c);
    }
    // bitonic sort of the 128 keys, ascending: strides 1, 2 inside a lane,
    // 4 .. 64 across lanes (lane ^ stride / 4)
#pragma unroll
    for (int k = 2; k <= 128; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j < 4) {
#pragma unroll
                for (int i = 0; i < 4; i++)
                    if ((i & j) == 0) cmp_swap(v[i], v[i | j], ((4 * lane + i) & k) == 0);
            } else {
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const u64 o = __shfl_xor_sync(kFull, v[i], j >> 2);
                    const int e = 4 * lane + i;
                    const bool take_min = ((e & j) == 0) == ((e & k) == 0);
                    v[i] = take_min ? (o < v[i] ? o : v[i]) : (o > v[i] ? o : v[i]);
                }
            }
        }
    }
    // positions 128 + 4 lane + i: the mirror of position 4 lane + i, so the
    // second half descends; an 8-stage bitonic merge sorts all 256
#pragma unroll
    for (int i = 0; i < 4; i++) v[4 + i] = mirror_key(v[i]);
#pragma unroll
    for (int i = 0; i < 4; i++) cmp_swap(v[i], v[4 + i], true);           // stride 128
#pragma unroll
    for (int j = 64; j >= 4; j >>= 1) {                                       // across lanes
        const bool lower = ((4 * lane) & j) == 0;                             // keeps the smaller key
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const u64 o = __shfl_xor_sync(kFull, v[i], j >> 2);
            v[i] = lower ? (o < v[i] ? o : v[i]) : (o > v[i] ? o : v[i]);
        }
    }
#pragma unroll
    for (int hh = 0; hh < 8; hh += 4) {                                      // strides 2, 1
        cmp_swap(v[hh + 0], v[hh + 2], true);
        cmp_swap(v[hh + 1], v[hh + 3], true);
        cmp_swap(v[hh + 0], v[hh + 1], true);
        cmp_swap(v[hh + 2], v[hh + 3], true);
    }

    // P(c): bucket sizes of the better-ranked centres (rank p = 4 lane + i,
    // then 128 + 4 lane + i), by a lane prefix and a warp scan per half
    uint32_t n[8], pre[8];
#pragma unroll
    for (int i = 0; i < 8; i++) n[i] = s_occ[warp][v[i] & 0xffu];
    uint32_t half_base = 0;
#pragma unroll
    for (int hh = 0; hh < 8; hh += 4) {
        uint32_t run = 0;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            pre[hh + i] = run;
            run += n[hh + i];
        }
        uint32_t incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - run + half_base;
#pragma unroll
        for (int i = 0; i < 4; i++) pre[hh + i] += excl;
        half_base += __shfl_sync(kFull, incl, 31);
    }
    const unsigned long long R = (unsigned long long)a.R;
    uint8_t *db = a.dbg_bonus ? a.dbg_bonus + ((size_t)bh * kB + b) * kNC : nullptr;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const uint32_t c = (uint32_t)(v[i] & 0xffu);
        const uint8_t bon = (uint8_t)tier_bonus(pre[i], R);
        s_bonus[warp][c] = bon;
        if (db) db[c] = bon;
        if (a.bonus_heads) *head_bonus_ptr(a, bh, b, (int)c) = bon;
    }
    __syncwarp();
    uint32_t word = 0;
#pragma unroll
    for (int tt = 0; tt < 8; tt++) word |= (uint32_t)s_bonus[warp][32 * tt + lane] << (4 * tt);
    const uint32_t rl = (uint32_t)(lane >> 3) & 3u;
    a.bonus_packed[((size_t)bh * kB + b) * 32 + lane] = __funnelshift_l(word, word, rl);
}

// The same preparation with 4 warps per block (2 blocks per 256-thread CTA,
// grid (8, pairs)): each 128-thread half ranks its block's 256 centres by a
// bitonic sort holding 2 keys per thread (shuffles inside a warp, shared
// memory for the 3 stages that cross warps).  Shorter per block than the warp
// version, so it is taken when there are few pairs and the SMs have room.
__global__ void __launch_bounds__(kQwThreads) k_query_prep_wide(PrepArgs a)
{
    const int bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int half = tid / kQpHalf, t = tid % kQpHalf;      // t: thread within the half
    const int b = kQpBlocks * blockIdx.x + half;             // this half's block
    const int b_seq = bh / a.H, h = bh - b_seq * a.H;
    __shared__ uint32_t s_occ[kQpBlocks][kNC];
    __shared__ u64 s_key[2][kQpBlocks][kNC];
    __shared__ float s_x[kD];
    __shared__ uint32_t s_ws[kQwWarps];
    __shared__ uint8_t s_bonus[kQpBlocks][kNC];
    __shared__ __align__(16) float s_qs[kMaxGroup * kD];

    if (blockIdx.x == 0) {   // reset the per-call counters of the collision scan and the rerank
        for (int i = tid; i < kBins; i += kQwThreads) a.head_hist[(size_t)bh * kBins + i] = 0u;
        if (tid < 2) a.tickets[(size_t)bh * 2 + tid] = 0u;
    }
    // global loads: 2 bucket sizes per thread; warp 0 the G query heads
    const uint32_t *occ = a.occ + ((size_t)index_pair(bh, a.kvg) * kB + b) * kNC;
    const uint32_t o0 = occ[t], o1 = occ[t + kQpHalf];
    if (warp == 0) {
        float qv[4][kMaxGroup];
        const int64_t base = ((int64_t)b_seq * a.H * a.G + (int64_t)h * a.G) * kD;
        load_query(qv, a, base, lane, s_qs);
        float x[4];
#pragma unroll
        for (int r = 0; r < 4; r++) {
            float acc = qv[r][0];
#pragma unroll
            for (int g = 1; g < kMaxGroup; g++)
                if (g < a.G) acc = __fadd_rn(acc, qv[r][g]);
            x[r] = acc;
        }
        const float nrm = warp_rotate128(x, a.rot, lane);
#pragma unroll
        for (int r = 0; r < 4; r++) s_x[lane + 32 * r] = x[r];
        if (blockIdx.x == 0) {
#pragma unroll
            for (int r = 0; r < 4; r++) {
                a.qt[(size_t)bh * kD + lane + 32 * r] = x[r];
                if (a.dbg_qt) a.dbg_qt[(size_t)bh * kD + lane + 32 * r] = x[r];
            }
            if (lane == 0) {
                a.qnorm[bh] = nrm;
                if (a.dbg_qnorm) a.dbg_qnorm[bh] = nrm;
            }
        }
    }
    s_occ[half][t] = o0;
    s_occ[half][t + kQpHalf] = o1;
    __syncthreads();
    float xq[kM];
#pragma unroll
    for (int j = 0; j < kM; j++) xq[j] = s_x[kM * b + j];
    // element e = 2 t + i starts as centre c = e; sort key (ascending order =
    // rank order): high 32 bits = ~ord(L) (L desc), low 8 bits = c (c asc)
    u64 key[2];
#pragma unroll
    for (int i = 0; i < 2; i++) {
        const int c = 2 * t + i;
        float L = 0.0f;
#pragma unroll
        for (int j = 0; j < kM; j++) L = __fadd_rn(L, ((c >> j) & 1) ? -xq[j] : xq[j]);
        L = __fadd_rn(L, 0.0f);   // fold -0 into +0 so equal scores tie
        key[i] = ((u64)(~ord_f32(L)) << 8) | (unsigned)c;
    }
    // bitonic sort, ascending, 256 elements over the half
    int buf = 0;
#pragma unroll
    for (int k = 2; k <= kNC; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 1) {                      // both elements in this thread
                const bool up = ((2 * t) & k) == 0;
                const u64 lo = key[0] < key[1] ? key[0] : key[1];
                const u64 hi = key[0] < key[1] ? key[1] : key[0];
                key[0] = up ? lo : hi;
                key[1] = up ? hi : lo;
            } else {
                u64 o[2];
                if (j <= 32) {                 // partner thread t ^ (j/2), same warp
#pragma unroll
                    for (int i = 0; i < 2; i++) o[i] = __shfl_xor_sync(kFull, key[i], j >> 1);
                } else {                       // partner in another warp of the half
#pragma unroll
                    for (int i = 0; i < 2; i++) s_key[buf][half][2 * t + i] = key[i];
                    __syncthreads();
#pragma unroll
                    for (int i = 0; i < 2; i++) o[i] = s_key[buf][half][(2 * t + i) ^ j];
                    buf ^= 1;
                }
#pragma unroll
                for (int i = 0; i < 2; i++) {
                    const int e = 2 * t + i;
                    const bool take_min = ((e & j) == 0) == ((e & k) == 0);
                    key[i] = take_min ? (o[i] < key[i] ? o[i] : key[i]) : (o[i] > key[i] ? o[i] : key[i]);
                }
            }
        }
    }
    // exclusive prefix of bucket sizes in rank order (over the half) -> tier bonus
    const int c0 = (int)(key[0] & 0xffu), c1 = (int)(key[1] & 0xffu);
    const uint32_t n0 = s_occ[half][c0], n1 = s_occ[half][c1];   // visible: the sort passed barriers
    uint32_t incl = n0 + n1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_ws[warp] = incl;
    __syncthreads();
    uint32_t P0 = incl - (n0 + n1);
    for (int w = half * (kQpHalf / 32); w < warp; w++) P0 += s_ws[w];
    const unsigned long long R = (unsigned long long)a.R;
    const uint32_t bon0 = tier_bonus(P0, R), bon1 = tier_bonus(P0 + n0, R);
    s_bonus[half][c0] = (uint8_t)bon0;
    s_bonus[half][c1] = (uint8_t)bon1;
    if (a.dbg_bonus) {
        uint8_t *db = a.dbg_bonus + ((size_t)bh * kB + b) * kNC;
        db[c0] = (uint8_t)bon0;
        db[c1] = (uint8_t)bon1;
    }
    if (a.bonus_heads) {
        *head_bonus_ptr(a, bh, b, c0) = (uint8_t)bon0;
        *head_bonus_ptr(a, bh, b, c1) = (uint8_t)bon1;
    }
    __syncthreads();
    if (t < 32) {                              // first warp of each half
        uint32_t word = 0;
#pragma unroll
        for (int tt = 0; tt < 8; tt++) word |= (uint32_t)s_bonus[half][32 * tt + lane] << (4 * tt);
        const uint32_t rl = (uint32_t)(lane >> 3) & 3u;
        a.bonus_packed[((size_t)bh * kB + b) * 32 + lane] = __funnelshift_l(word, word, rl);
    }
}

cudaError_t launch_query_prep(const PrepArgs &a, cudaStream_t s)
{
    static_assert(kB % kQpWarps == 0 && kB % kQpBlocks == 0, "whole blocks per CTA");
    if (a.wide)
        k_query_prep_wide<<<dim3(kB / kQpBlocks, a.bh), kQwThreads, 0, s>>>(a);
    else
        k_query_prep<<<dim3(kB / kQpWarps, a.bh), kQpThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace pk
