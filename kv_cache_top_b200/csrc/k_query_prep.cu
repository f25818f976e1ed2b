// k_query_prep.cu -- per (sequence, KV head) query preparation.
//
// (1) GQA aggregation q_agg = ((q_0 + q_1) + ..) + q_{G-1} in fp32, then the
//     canonical normalise + SRHT rotate (ParisKV slides, Eq. 5).
// (2) Stage I bucket tiers (slides, "Stage I uses multi-tier collision votes
//     to prune keys", Sec. 4.2.2 / App. B.2.1 Eq. 15; README "activates the
//     nearest direction centroids in each subspace"): in block b every
//     sign-pattern centre c gets the score L_b(c) = sum_j +-q~_{b,j} (minus
//     where bit j of c is set; the 1/sqrt(m) factor does not change the order),
//     the 256 centres are ranked by (L desc, c asc), P(c) = number of keys in
//     better-ranked buckets (from the occupancy table), and a bucket inside
//     the top-rho fraction (P(c) < R = ceil(rho n)) gets bonus 6 - floor(6P/R).
//
// Grid (16 blocks, pairs), one warp per CTA: the warp rotates the query, ranks
// the 256 centres of its block with a register bitonic sort (8 keys per lane,
// shuffles only, no block barriers), scans the bucket sizes in rank order and
// packs the bonus table 4 bits per centre in the layout the collision scan
// keeps in registers -- lane l's word holds, in nibble t, the bonus of centre
// 32 t + l.
#include "pk_internal.cuh"

namespace pk {

__global__ void __launch_bounds__(32) k_query_prep(PrepArgs a)
{
    const int b = blockIdx.x, bh = blockIdx.y;
    const int lane = threadIdx.x;
    const int b_seq = bh / a.H, h = bh - b_seq * a.H;
    __shared__ uint8_t s_bonus[kNC];

    if (b == 0) {   // reset the per-call counters of the collision scan and the rerank
        for (int i = lane; i < kBins; i += 32) a.head_hist[(size_t)bh * kBins + i] = 0u;
        if (lane < 2) a.tickets[(size_t)bh * 2 + lane] = 0u;
    }
    float x[4];
    {
        const int64_t base = ((int64_t)b_seq * a.H * a.G + (int64_t)h * a.G) * kD;
#pragma unroll
        for (int r = 0; r < 4; r++) {
            const int64_t j = base + lane + 32 * r;
            float acc = ld_as_f32(a.q, j, a.is_bf16);
            for (int g = 1; g < a.G; g++) acc = __fadd_rn(acc, ld_as_f32(a.q, j + (int64_t)g * kD, a.is_bf16));
            x[r] = acc;
        }
    }
    const float nrm = warp_rotate128(x, a.rot, lane);
    if (b == 0) {
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
    // coordinates 8b..8b+7 live in register b/4 of lanes 8(b%4)..8(b%4)+7
    float xq[kM];
    {
        float src = x[0];
#pragma unroll
        for (int r = 1; r < 4; r++) src = (b / 4 == r) ? x[r] : src;
#pragma unroll
        for (int j = 0; j < kM; j++) xq[j] = __shfl_sync(kFull, src, 8 * (b % 4) + j);
    }
    // element e = 8 lane + i starts as centre c = e; sort key (ascending order =
    // rank order): high 32 bits = ~ord(L) (L desc), low 8 bits = c (c asc)
    unsigned long long key[8];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const int c = lane * 8 + i;
        float L = 0.0f;
#pragma unroll
        for (int j = 0; j < kM; j++) L = __fadd_rn(L, ((c >> j) & 1) ? -xq[j] : xq[j]);
        L = __fadd_rn(L, 0.0f);   // fold -0 into +0 so equal scores tie
        key[i] = ((unsigned long long)(~ord_f32(L)) << 8) | (unsigned)c;
    }
    // bitonic sort, ascending, 256 elements over the warp
#pragma unroll
    for (int k = 2; k <= 256; k <<= 1) {
#pragma unroll
        for (int jj = k >> 1; jj > 0; jj >>= 1) {
            if (jj >= 8) {
                const int lx = jj >> 3;
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const int e = lane * 8 + i;
                    const unsigned long long o = __shfl_xor_sync(kFull, key[i], lx);
                    const bool take_min = ((e & jj) == 0) == ((e & k) == 0);
                    key[i] = take_min ? (o < key[i] ? o : key[i]) : (o > key[i] ? o : key[i]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    if ((i & jj) == 0) {
                        const int e = lane * 8 + i;
                        const bool up = (e & k) == 0;
                        const unsigned long long x0 = key[i], x1 = key[i ^ jj];
                        const unsigned long long lo = x0 < x1 ? x0 : x1, hi = x0 < x1 ? x1 : x0;
                        key[i] = up ? lo : hi;
                        key[i ^ jj] = up ? hi : lo;
                    }
                }
            }
        }
    }
    // exclusive prefix of bucket sizes in rank order -> tier bonus
    const uint32_t *occ = a.occ + ((size_t)bh * kB + b) * kNC;
    uint32_t cnt[8], run = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        cnt[i] = occ[key[i] & 0xffu];
        run += cnt[i];
    }
    uint32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
    }
    uint32_t P = incl - run;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const int c = (int)(key[i] & 0xffu);
        uint32_t bon = 0;
        if ((int64_t)P < a.R) bon = 6u - (uint32_t)((6ull * P) / (unsigned long long)a.R);
        s_bonus[c] = (uint8_t)bon;
        if (a.dbg_bonus) a.dbg_bonus[((size_t)bh * kB + b) * kNC + c] = (uint8_t)bon;
        P += cnt[i];
    }
    __syncwarp();
    uint32_t word = 0;
#pragma unroll
    for (int t = 0; t < 8; t++) word |= (uint32_t)s_bonus[32 * t + lane] << (4 * t);
    a.bonus_packed[((size_t)bh * kB + b) * 32 + lane] = word;
}

cudaError_t launch_query_prep(const PrepArgs &a, cudaStream_t s)
{
    k_query_prep<<<dim3(kB, a.bh), 32, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace pk
