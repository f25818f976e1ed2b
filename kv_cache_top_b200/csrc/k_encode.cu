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
// r holds blocks 4r..4r+3, one block per aligned 8-lane group.  Large batches
// (the prefill, a batched re-indexing) count their occupancy per CTA in
// shared memory; a few keys count straight into the table.
//
// Record layout (128 B per key, 16-byte aligned):
//   for g = 0..3:  [16 B: blocks 4g..4g+3, one u32 each, nibble j = coordinate
//                   j of the block: bit 3 = sign (1 = negative), bits 0-2 = t]
//                  [16 B: w_{4g} .. w_{4g+3} as fp32]
#include "pk_internal.cuh"

namespace pk {

constexpr int kEncWarps = 8;
constexpr int kEncKeysShared = 1024;   // keys per CTA when the occupancy counts go through shared memory

// Encode one key (a warp): writes its codes and record; each of the 16
// (block, code) counts goes to count(b, code).
template <typename Count>
__device__ __forceinline__ void encode_key(const EncodeArgs &a, int64_t bh, int64_t i, int lane, Count count)
{
    const int64_t pos = a.pos0 + i;
    float x[4];
#pragma unroll
    for (int r = 0; r < 4; r++) x[r] = ld_as_f32(a.K, (bh * a.k_stride + i) * kD + lane + 32 * r, a.is_bf16);
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
            count(b, code);
        }
    }
}

// Few keys: one warp per key over all pairs, counts straight to global memory.
__global__ void __launch_bounds__(32 * kEncWarps) k_encode(EncodeArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * kEncWarps;
    const int64_t total = (int64_t)a.bh * a.n_new;
    for (int64_t e = (int64_t)blockIdx.x * kEncWarps + (threadIdx.x >> 5); e < total; e += warps) {
        const int64_t bh = e / a.n_new;
        encode_key(a, bh, e - bh * a.n_new, lane, [&](int b, uint32_t code) {
            atomicAdd(&a.occ[((size_t)bh * kB + b) * kNC + code], 1u);
        });
    }
}

// Many keys: CTA (x, pair) encodes keys x kEncKeysShared .. of one pair and
// counts them in shared memory; the non-zero counts are added to the pair's
// table once per CTA (at most 4096 global atomics instead of 16 per key).
__global__ void __launch_bounds__(32 * kEncWarps) k_encode_shared(EncodeArgs a)
{
    __shared__ uint32_t s_occ[kB * kNC];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t bh = blockIdx.y;
    for (int i = threadIdx.x; i < kB * kNC; i += 32 * kEncWarps) s_occ[i] = 0u;
    __syncthreads();
    const int64_t k0 = (int64_t)blockIdx.x * kEncKeysShared;
    const int64_t k1 = min(a.n_new, k0 + kEncKeysShared);
    for (int64_t i = k0 + warp; i < k1; i += kEncWarps)
        encode_key(a, bh, i, lane, [&](int b, uint32_t code) { atomicAdd(&s_occ[b * kNC + code], 1u); });
    __syncthreads();
    uint32_t *occ = a.occ + (size_t)bh * kB * kNC;
    for (int i = threadIdx.x; i < kB * kNC; i += 32 * kEncWarps) {
        const uint32_t v = s_occ[i];
        if (v) atomicAdd(&occ[i], v);
    }
}

// K and V rows into the interleaved store: rows 0..n_new-1 of every pair of
// srcK / srcV ([BH][src_stride][D], row_bytes each, device or mapped host) go
// to positions pos0.. of the pair in the store, K at dstK, V at dstV, rows
// `pitch` bytes apart and pairs `pair_rows` rows apart.  Consecutive threads
// copy consecutive 16-byte pieces, so a row is one coalesced write (posted
// writes over the host link when the store is pinned host memory).
// CTA (x, p) copies rows x kStoreRows .. of pair p; a row is per_row =
// 2^lg 16-byte pieces (16 for bf16, 32 for fp32).
constexpr int kStoreRows = 64;
__global__ void __launch_bounds__(256) k_store_rows(StoreArgs a)
{
    const int lg = a.row_bytes == 512 ? 5 : 4;
    const int64_t p = blockIdx.y;
    const int64_t r0 = (int64_t)blockIdx.x * kStoreRows;
    const int rows = (int)min((int64_t)kStoreRows, a.n_new - r0);
    const unsigned char *sK = a.srcK + (size_t)(p * a.src_stride + r0) * a.row_bytes;
    const unsigned char *sV = a.srcV + (size_t)(p * a.src_stride + r0) * a.row_bytes;
    unsigned char *dK = a.dstK + (size_t)(p * a.pair_rows + a.pos0 + r0) * a.pitch;
    unsigned char *dV = a.dstV + (size_t)(p * a.pair_rows + a.pos0 + r0) * a.pitch;
    for (int e = threadIdx.x; e < (rows << lg); e += 256) {
        const int r = e >> lg, c = e & ((1 << lg) - 1);
        const uint4 k = *reinterpret_cast<const uint4 *>(sK + (size_t)r * a.row_bytes + 16 * c);
        const uint4 v = *reinterpret_cast<const uint4 *>(sV + (size_t)r * a.row_bytes + 16 * c);
        *reinterpret_cast<uint4 *>(dK + (size_t)r * a.pitch + 16 * c) = k;
        *reinterpret_cast<uint4 *>(dV + (size_t)r * a.pitch + 16 * c) = v;
    }
}

// Publishing staged keys: their counts join the table, and the side table is
// left at zero for the next staging.
__global__ void __launch_bounds__(256) k_occ_merge(uint32_t *occ, uint32_t *add, int64_t count)
{
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < count; i += (int64_t)gridDim.x * 256) {
        const uint32_t v = add[i];
        if (v) {
            occ[i] += v;
            add[i] = 0u;
        }
    }
}

}  // namespace pk

namespace pk {
cudaError_t launch_occ_merge(uint32_t *occ, uint32_t *add, int64_t count, cudaStream_t s)
{
    const int64_t blocks = (count + 255) / 256;
    k_occ_merge<<<(unsigned)(blocks < 1184 ? blocks : 1184), 256, 0, s>>>(occ, add, count);
    return cudaGetLastError();
}

cudaError_t launch_store_rows(const StoreArgs &a, cudaStream_t s)
{
    if (a.n_new <= 0 || a.bh <= 0) return cudaSuccess;
    if (a.bh > 65535) return cudaErrorInvalidValue;
    const int64_t gx = (a.n_new + kStoreRows - 1) / kStoreRows;
    k_store_rows<<<dim3((unsigned)gx, (unsigned)a.bh), 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t s)
{
    const int64_t keys = (int64_t)a.bh * a.n_new;
    if (keys <= 0) return cudaSuccess;
    // the shared-memory counts pay off from a few thousand keys per pair, and
    // their grid (one CTA per 1024 keys of a pair) must fill the GPU; other
    // batches (a decode-time re-indexing, few pairs) take one warp per key
    // across all pairs, so the whole batch encodes in parallel
    const int64_t gx = (a.n_new + kEncKeysShared - 1) / kEncKeysShared;
    if (a.n_new >= 4 * kEncKeysShared && a.bh <= 65535 && gx * a.bh >= 512) {
        k_encode_shared<<<dim3((unsigned)gx, (unsigned)a.bh), 32 * kEncWarps, 0, s>>>(a);
    } else {
        const int64_t blocks = (keys + kEncWarps - 1) / kEncWarps;   // one key per warp
        const int grid = (int)(blocks < 65535 * 16 ? blocks : 65535 * 16);
        k_encode<<<grid, 32 * kEncWarps, 0, s>>>(a);
    }
    return cudaGetLastError();
}
}  // namespace pk
