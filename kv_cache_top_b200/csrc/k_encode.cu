// k_encode.cu -- key encoding for pk_build_index / pk_append.
//
// Per key (ParisKV slides, Sec. 4.1.1-4.1.2 Eqs. 5-6: normalise and rotate so
// that one fixed codebook serves every key; Eqs. 7-10: the 4-bit summary that
// Stage II scores):
//   k~ = R k/||k||; per block b of m = 8 coordinates:
//   r_b = ||k~_b||, u_b = k~_b / r_b,
//   code_b = sign pattern of u_b (bit j set iff u_j < 0)    -> PolarANN centre id
//   t_j    = #{t : |u_j| > theta_t}                          -> 3-bit magnitude index
//   alpha_b = sum_j l_{t_j} |u_j|,  w_b = (||k|| r_b) / alpha_b
// in one fixed fp32 operation order (the oracle follows the same order), so
// codes, indices and weights are bit-exact across implementations.
//
// One warp per key: lane l holds coordinates l + 32 r (r = 0..3), so register
// r holds blocks 4r..4r+3, one block per aligned 8-lane group.
//
// Record layout (128 B per key, 16-byte aligned):
//   for g = 0..3:  [16 B: blocks 4g..4g+3, one u32 each, nibble j = coordinate
//                   j of the block: bit 3 = sign (1 = negative), bits 0-2 = t]
//                  [16 B: w_{4g} .. w_{4g+3} as fp32]
#include "pk_internal.cuh"

namespace pk {

__global__ void __launch_bounds__(256) k_encode(EncodeArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t total = (int64_t)a.bh * a.n_new;
    for (int64_t e = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); e < total;
         e += warps) {
        const int64_t bh = e / a.n_new;
        const int64_t i = e - bh * a.n_new;
        const int64_t pos = a.pos0 + i;
        float x[4];
#pragma unroll
        for (int r = 0; r < 4; r++) x[r] = ld_as_f32(a.K, e * kD + lane + 32 * r, a.is_bf16);
        const float nk = warp_rotate128(x, a.rot, lane);

        uint8_t *codes = a.codes + ((size_t)bh * a.n_cap + pos) * kB;
        uint8_t *rec = a.rec + ((size_t)bh * a.n_cap + pos) * kRecBytes;
        const int g = lane >> 3;       // block within the register group
        const int j = lane & 7;        // coordinate within the block
#pragma unroll
        for (int r = 0; r < 4; r++) {
            const float xv = x[r];
            float sq = __fmul_rn(xv, xv);
            sq = __fadd_rn(sq, __shfl_xor_sync(kFull, sq, 4));   // tree h = 4, 2, 1
            sq = __fadd_rn(sq, __shfl_xor_sync(kFull, sq, 2));
            sq = __fadd_rn(sq, __shfl_xor_sync(kFull, sq, 1));
            const float rb = __fsqrt_rn(sq);
            // rb is uniform over the 8-lane group; a zero block keeps u = 0,
            // t = 0, w = 0.  No branch around the shuffles below.
            const bool live = rb != 0.0f;
            const float u = live ? __fdiv_rn(xv, rb) : 0.0f;
            const bool neg = u < 0.0f;
            const float au = fabsf(u);
            int t = 0;
#pragma unroll
            for (int q = 0; q < kL - 1; q++) t += (au > a.lv.thr[q]) ? 1 : 0;
            float p = __fmul_rn(a.lv.lev[t], au);
            p = __fadd_rn(p, __shfl_xor_sync(kFull, p, 4));
            p = __fadd_rn(p, __shfl_xor_sync(kFull, p, 2));
            p = __fadd_rn(p, __shfl_xor_sync(kFull, p, 1));
            const float w = live ? __fdiv_rn(__fmul_rn(nk, rb), p) : 0.0f;
            const uint32_t bal = __ballot_sync(kFull, neg);
            uint32_t word = (uint32_t)(((neg ? 8 : 0) | t) << (4 * j));
            word |= __shfl_xor_sync(kFull, word, 4);
            word |= __shfl_xor_sync(kFull, word, 2);
            word |= __shfl_xor_sync(kFull, word, 1);
            if (j == 0) {
                const int b = 4 * r + g;
                const uint32_t code = (bal >> (8 * g)) & 0xffu;
                codes[b] = (uint8_t)code;
                reinterpret_cast<uint32_t *>(rec + 32 * r)[g] = word;
                reinterpret_cast<float *>(rec + 32 * r + 16)[g] = w;
                atomicAdd(&a.occ[((size_t)bh * kB + b) * kNC + code], 1u);
            }
        }
    }
}

}  // namespace pk

namespace pk {
cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t s)
{
    const int64_t keys = (int64_t)a.bh * a.n_new;
    if (keys <= 0) return cudaSuccess;
    const int64_t blocks = (keys + 7) / 8;                 // 8 warps per CTA, one key each
    const int grid = (int)(blocks < 65535 * 16 ? blocks : 65535 * 16);
    k_encode<<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}
}  // namespace pk
