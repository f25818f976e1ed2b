// pk_internal.cuh -- shared device helpers and kernel argument blocks of the
// ParisKV retrieval library (sm_100a).  Not part of the public C-ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pariskv.h"

namespace pk {

constexpr int kD = 128;          // head_dim
constexpr int kM = 8;            // sub-space dimension m
constexpr int kB = kD / kM;      // blocks per key (16)
constexpr int kNC = 1 << kM;     // sign-pattern centres per block (256)
constexpr int kL = 8;            // magnitude levels (3 bits)
constexpr int kSMax = 6 * kB;    // largest collision score (96)
constexpr int kBins = kSMax + 1; // score histogram bins (97)
constexpr int kCum = kBins + 1;  // suffix-count entries per chunk (98, last = 0)
constexpr int kRecBytes = 128;   // 4-bit summary record per key
constexpr int kMaxTopk = 1024;
constexpr int kMaxGroup = 8;
constexpr int kSelPer = 16;      // candidates per rerank thread (upper bound): a slice has <= kSelPer x CTA size
constexpr int kMaxSlice = kSelPer * 256;  // candidates per rerank CTA (upper bound)
constexpr int kAtRows = 32;      // selected rows per attention CTA (upper bound)
constexpr int kMergeCap = 16384; // partial keys one merge CTA holds at once
constexpr unsigned kFull = 0xffffffffu;

// Device-check codes written to the index's error word (first one wins).
enum : int32_t { DEVCHK_NONE = 0, DEVCHK_BAD_INDEX = 1, DEVCHK_CAND_COUNT = 2 };

struct RotConst {
    uint32_t sign_mask[4];   // bit l of word r: coordinate l + 32 r has s = -1
    float c;                 // fp32(1/sqrt(D))
};

struct Levels {
    float lev[kL];
    float thr[kL - 1];
};

struct EncodeArgs {
    const void *K;           // [BH][k_stride][D] kv dtype: rows 0..n_new-1 of each pair
    int64_t k_stride;        // rows between pairs of the input (>= n_new)
    int64_t n_new;
    int64_t pos0;            // first position written
    int64_t n_cap;
    int32_t bh;
    int32_t is_bf16;
    uint8_t *codes;          // [BH][n_cap][16]
    uint8_t *rec;            // [BH][n_cap][128]
    uint32_t *occ;           // [BH][16][256]  counts are added here
    RotConst rot;
    Levels lv;
};

struct StoreArgs {
    const unsigned char *srcK, *srcV;   // [BH][src_stride][row_bytes]
    unsigned char *dstK, *dstV;         // first K / V row of the store
    int64_t src_stride, n_new, pos0, pair_rows, pitch;
    int32_t bh, row_bytes;
};

struct PrepArgs {
    const void *q;           // [batch][H*G][D]
    int32_t H, G, is_bf16, bh;
    int64_t R;               // collision budget ceil(rho n)
    int32_t kvg;             // query units per index pair (1, or G for per-head search)
    int32_t wide;            // 1: 4 warps per block (few pairs); 0: one warp per block
    const uint32_t *occ;
    RotConst rot;
    float *qt;               // [BH][D]
    float *qnorm;            // [BH]
    uint32_t *bonus_packed;  // [BH][16][32]  (4-bit bonus per centre)
    uint32_t *head_hist;     // [BH][kBins]   zeroed here
    uint32_t *tickets;       // [BH][2]       zeroed here
    uint8_t *dbg_bonus;      // [BH][16][256] or null
    // per-query-head search (kvg query units per pair): every unit's bonus
    // also goes to byte (g & 3) of word (g >> 2) of entry (pair, block,
    // centre) of a per-pair table [pairs][16][256][heads_np] u32, g = unit % kvg
    uint8_t *bonus_heads;
    int32_t heads_np;
    float *dbg_qt;
    float *dbg_qnorm;
};

struct ScanArgs {
    const uint8_t *codes;
    const uint32_t *bonus_packed;
    const uint8_t *bonus_bytes;   // [pairs][16][256][np] u32 packed bonuses of the kvg query heads of a pair
    int64_t n, n_cap, chunk, C;   // n_cap: row stride of the per-key arrays
    int32_t nchunks;
    int32_t kvg;             // query units per index pair
    uint8_t *S;              // [BH][n_cap]
    uint32_t *chunk_cum;     // [BH][max_chunks][kCum]
    uint32_t *head_hist;     // [BH][kBins]
    uint32_t *tickets;       // [BH][2]
    uint2 *chunk_info;       // [BH][max_chunks]  (first candidate slot, tie quota)
    int32_t *sstar;          // [BH]
    int32_t max_chunks;
    uint8_t *dbg_S;
    uint32_t *dbg_hist;
    int32_t *dbg_sstar;
};

struct CompactArgs {
    const uint8_t *S;
    const uint2 *chunk_info;
    const int32_t *sstar;
    int64_t n, stride, chunk, C;
    int32_t max_chunks;
    int32_t groups;          // 16-key groups per thread: ceil(chunk / 4096) <= 8
    int32_t *cand;           // [BH][stride]  candidate ids, ascending
    int32_t *dbg_cand;       // [BH][C] or null
    int32_t *dev_err;
};

struct RerankArgs {
    const int32_t *cand;     // [BH][stride]
    const uint8_t *rec;
    const float *qt;
    const float *qnorm;
    int64_t stride, C;
    int32_t kvg;             // query units per index pair
    int32_t slice, nslices, max_slices, topk, topk_cap;
    int32_t nt;              // threads per CTA: 256 or 128
    unsigned long long *partial;   // [BH][max_slices][topk_cap]  per-slice Top-k sets
    Levels lv;
    float *dbg_est;          // [BH][C] or null
};

struct AttendArgs {
    const void *q;           // [batch][H*G][D]
    const int32_t *idx;      // [BH][topk]
    const void *K;           // first K row of the store [BH][stride][2][D] (device or mapped host)
    const void *V;           // first V row
    int64_t kv_pitch;        // bytes from one key's rows to the next
    float *out;              // [batch][H*G][D]
    int64_t n, stride;
    int32_t H, G, topk, is_bf16;
    int32_t nsplit;          // CTAs (one cluster) per pair, 1..8
    int32_t kvg;             // query units per index pair (K/V and dense rows of pair unit / kvg)
    float scale;
    int32_t *dev_err;
    long long *dev_err_detail;
    // dense rows kept outside the index (sink and local tokens), attended
    // under the same softmax: [BH][dstride][D] kv_dtype, rows 0..dlen-1
    const void *dK, *dV;
    int64_t dstride;
    int32_t dlen;
    // per-query-head rows, gathered once per pair: idx is [BH][G][topk]
    // (each query head's own list), the CTA's rows are the union of the G
    // lists, and head g's softmax runs over its own rows only
    int32_t union_heads;
};
constexpr int kUnionMax = 1024;   // G x topk entries a union-gather attention accepts

struct MergeArgs {
    const unsigned long long *partial;
    int32_t nslices, max_slices, topk, topk_cap, cap;
    int32_t *out_idx;        // [BH][topk]
    float *out_score;        // [BH][topk] or null
    int32_t *dev_err;
};


// ---------------------------------------------------------------- helpers
// index pair of query unit u (the per-head search runs G units per pair)
__device__ __forceinline__ int index_pair(int u, int kvg) { return kvg > 1 ? u / kvg : u; }

__device__ __forceinline__ float ld_as_f32(const void *p, int64_t i, int is_bf16)
{
    if (is_bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

// 16-byte asynchronous global -> shared copy (L2 only, no register staging)
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src)
{
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Map an fp32 value to an unsigned key whose integer order is the float order.
// -0.0 must already be folded into +0.0 by the caller (x + 0.0f).
__device__ __forceinline__ uint32_t ord_f32(float x)
{
    uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float unord_f32(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while its predecessor finishes; it must wait here
// before touching the predecessor's outputs (a no-op for ordinary launches).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the dependent grid launch once every CTA of this grid has called this
// (or exited); called after a CTA's main work.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Record a device-check failure (first writer wins) without trapping.
__device__ __forceinline__ void devchk(int32_t *err, long long *detail, int32_t code, long long v)
{
    if (err && atomicCAS(err, 0, code) == 0 && detail) *detail = v;
}

// Canonical fp32 normalise + SRHT rotate of one 128-vector held by a warp:
// lane l holds x[r] = coordinate l + 32 r.  Every operation is one IEEE
// round-to-nearest step in the fixed order (i) sum of squares by the halving
// tree, sqrt; (ii) divide by the norm; (iii) sign diagonal; (iv) Walsh-Hadamard
// butterflies h = 1, 2, .., 64; (v) scale by c.  Returns the norm; a zero
// vector stays zero.
__device__ __forceinline__ float warp_rotate128(float x[4], const RotConst &rc, int lane)
{
    float s0 = __fmul_rn(x[0], x[0]), s1 = __fmul_rn(x[1], x[1]);
    float s2 = __fmul_rn(x[2], x[2]), s3 = __fmul_rn(x[3], x[3]);
    s0 = __fadd_rn(s0, s2);          // h = 64: s[j] += s[j+64]
    s1 = __fadd_rn(s1, s3);
    s0 = __fadd_rn(s0, s1);          // h = 32: s[j] += s[j+32]
#pragma unroll
    for (int h = 16; h >= 1; h >>= 1) s0 = __fadd_rn(s0, __shfl_xor_sync(kFull, s0, h));
    const float nrm = __fsqrt_rn(s0);
    if (nrm == 0.0f) {
#pragma unroll
        for (int r = 0; r < 4; r++) x[r] = 0.0f;
        return 0.0f;
    }
#pragma unroll
    for (int r = 0; r < 4; r++) {
        float y = __fdiv_rn(x[r], nrm);
        x[r] = ((rc.sign_mask[r] >> lane) & 1u) ? -y : y;
    }
#pragma unroll
    for (int h = 1; h <= 16; h <<= 1) {
        const bool hi = (lane & h) != 0;
#pragma unroll
        for (int r = 0; r < 4; r++) {
            float p = __shfl_xor_sync(kFull, x[r], h);
            x[r] = hi ? __fsub_rn(p, x[r]) : __fadd_rn(x[r], p);
        }
    }
    {   // h = 32: registers (0,1), (2,3)
        float a = x[0], b = x[1];
        x[0] = __fadd_rn(a, b); x[1] = __fsub_rn(a, b);
        a = x[2]; b = x[3];
        x[2] = __fadd_rn(a, b); x[3] = __fsub_rn(a, b);
    }
    {   // h = 64: registers (0,2), (1,3)
        float a = x[0], b = x[2];
        x[0] = __fadd_rn(a, b); x[2] = __fsub_rn(a, b);
        a = x[1]; b = x[3];
        x[1] = __fadd_rn(a, b); x[3] = __fsub_rn(a, b);
    }
#pragma unroll
    for (int r = 0; r < 4; r++) x[r] = __fmul_rn(x[r], rc.c);
    return nrm;
}

// Block-wide exclusive scan of one u32 per thread (blockDim.x == NT, NT a
// multiple of 32, NT <= 1024).  `ws` needs NT/32 + 1 words of shared memory.
// Returns the exclusive prefix; *total receives the block sum.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *ws, uint32_t *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) ws[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = (lane < NT / 32) ? ws[lane] : 0u;
        uint32_t t = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(kFull, t, o);
            if (lane >= o) t += y;
        }
        if (lane < NT / 32) ws[lane] = t - w;
        if (lane == 31) ws[NT / 32] = t;
    }
    __syncthreads();
    uint32_t r = ws[warp] + x - v;
    *total = ws[NT / 32];
    __syncthreads();
    return r;
}

}  // namespace pk

namespace pk {
// kernel launchers (one per kernel translation unit)
cudaError_t launch_encode(const EncodeArgs &a, cudaStream_t s);
cudaError_t launch_store_rows(const StoreArgs &a, cudaStream_t s);
// occ[i] += add[i], add[i] = 0 for i < count
cudaError_t launch_occ_merge(uint32_t *occ, uint32_t *add, int64_t count, cudaStream_t s);
cudaError_t launch_query_prep(const PrepArgs &a, cudaStream_t s);
cudaError_t launch_collision_scan(const ScanArgs &a, int bh, cudaStream_t s);
cudaError_t launch_collision_scan_heads(const ScanArgs &a, int pairs, cudaStream_t s);
cudaError_t launch_compact(const CompactArgs &a, int nchunks, int bh, cudaStream_t s);
cudaError_t launch_rerank_topk(const RerankArgs &a, int bh, cudaStream_t s);
cudaError_t launch_topk_merge(const MergeArgs &a, int bh, cudaStream_t s);
cudaError_t launch_gather_attend(const AttendArgs &a, int bh, cudaStream_t s);
size_t rerank_smem(int slice, int nt);

// Launch with programmatic stream serialisation (the kernel calls pdl_wait()
// before reading what earlier kernels of the stream wrote).
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}
// host-side Lloyd-Max levels of the magnitude prior (closed-form integrals)
int lloyd_max_levels(int m, int L, double *lev, double *thr);
}  // namespace pk
