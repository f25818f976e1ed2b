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
// Grid (16 blocks, pairs): CTA (b, pair) ranks the 256 centres of block b with
// a shared-memory bitonic sort, one thread per centre.  Output: the bonus
// table packed 4 bits per centre in the layout the collision scan keeps in
// registers -- lane l's word holds, in nibble t, the bonus of centre 32 t + l.
#include "pk_internal.cuh"

namespace pk {

__global__ void __launch_bounds__(256) k_query_prep(PrepArgs a)
{
    const int b = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b_seq = bh / a.H, h = bh - b_seq * a.H;
    __shared__ float s_q[kD];
    __shared__ float s_qt[kD];
    __shared__ unsigned long long s_key[kNC];
    __shared__ uint8_t s_bonus[kNC];
    __shared__ uint32_t s_ws[9];

    if (b == 0) {   // reset the per-call counters of the collision scan and the rerank
        if (tid < kBins) a.head_hist[(size_t)bh * kBins + tid] = 0u;
        if (tid < 2) a.tickets[(size_t)bh * 2 + tid] = 0u;
    }
    if (tid < kD) {
        const int64_t base = ((int64_t)b_seq * a.H * a.G + (int64_t)h * a.G) * kD + tid;
        float acc = ld_as_f32(a.q, base, a.is_bf16);
        for (int g = 1; g < a.G; g++) acc = __fadd_rn(acc, ld_as_f32(a.q, base + (int64_t)g * kD, a.is_bf16));
        s_q[tid] = acc;
    }
    __syncthreads();
    if (warp == 0) {
        float x[4];
#pragma unroll
        for (int r = 0; r < 4; r++) x[r] = s_q[lane + 32 * r];
        const float nrm = warp_rotate128(x, a.rot, lane);
#pragma unroll
        for (int r = 0; r < 4; r++) s_qt[lane + 32 * r] = x[r];
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
    }
    __syncthreads();

    // centre c = tid: score L_b(c), summed over j = 0..7 in order
    const int c = tid;
    float L = 0.0f;
#pragma unroll
    for (int j = 0; j < kM; j++) {
        const float x = s_qt[b * kM + j];
        L = __fadd_rn(L, ((c >> j) & 1) ? -x : x);
    }
    L = __fadd_rn(L, 0.0f);   // fold -0 into +0 so equal scores tie
    // sort key, ascending = rank order: (L desc, c asc)
    s_key[c] = ((unsigned long long)(~ord_f32(L)) << 8) | (unsigned)c;
    __syncthreads();
    // bitonic sort of the 256 keys, one per thread
    for (int k = 2; k <= kNC; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            const int p = tid ^ j;
            if (p > tid) {
                const unsigned long long x = s_key[tid], y = s_key[p];
                const bool up = (tid & k) == 0;
                if (up ? (x > y) : (x < y)) {
                    s_key[tid] = y;
                    s_key[p] = x;
                }
            }
            __syncthreads();
        }
    }
    // thread r now owns the centre of rank r; P = keys in better-ranked buckets
    const int cr = (int)(s_key[tid] & 0xffu);
    const uint32_t cnt = a.occ[((size_t)bh * kB + b) * kNC + cr];
    uint32_t tot;
    const uint32_t P = block_excl_scan<256>(cnt, s_ws, &tot);
    uint32_t bon = 0;
    if ((int64_t)P < a.R) bon = 6u - (uint32_t)((6ull * P) / (unsigned long long)a.R);
    s_bonus[cr] = (uint8_t)bon;
    if (a.dbg_bonus) a.dbg_bonus[((size_t)bh * kB + b) * kNC + cr] = (uint8_t)bon;
    __syncthreads();
    if (tid < 32) {
        uint32_t word = 0;
#pragma unroll
        for (int t = 0; t < 8; t++) word |= (uint32_t)s_bonus[32 * t + tid] << (4 * t);
        a.bonus_packed[((size_t)bh * kB + b) * 32 + tid] = word;
    }
}

}  // namespace pk

namespace pk {
cudaError_t launch_query_prep(const PrepArgs &a, cudaStream_t s)
{
    k_query_prep<<<dim3(kB, a.bh), 256, 0, s>>>(a);
    return cudaGetLastError();
}
}  // namespace pk
