// k_gather_attend.cu -- gather of the selected K/V rows and exact attention.
//
// o_g = sum_r softmax_r(scale <q_g, K[sel_r]>) V[sel_r] for every query head
// g of the KV head (ParisKV slides, "The target is high-score KV indices at
// each decode step", Sec. 3 Eqs. 1-3: "recompute softmax and value
// aggregation using the selected full-precision KV").  The K/V rows are read
// where the index keeps them: HBM, or pinned host memory through UVA (README,
// "Attention: fetch only selected KV pairs ... from pinned CPU memory via
// UVA").
//
// One CTA per pair.  Rows are staged 64 at a time into shared memory with
// every thread issuing 16-byte loads at once, so a tile costs one round trip
// over the host link; softmax is accumulated online across tiles in fp32.
// Selected ids outside [0, n) are skipped and recorded in the device-check
// word (no trap).
#include "pk_internal.cuh"

namespace pk {

constexpr int kAtThreads = 256;
constexpr int kAtWarps = kAtThreads / 32;
constexpr int kTileRows = 64;

__global__ void __launch_bounds__(kAtThreads) k_gather_attend(AttendArgs a)
{
    extern __shared__ __align__(16) unsigned char s_raw[];
    __shared__ int32_t s_idx[kTileRows];
    __shared__ float s_sc[kMaxGroup][kTileRows];
    __shared__ float s_m[kMaxGroup], s_l[kMaxGroup], s_alpha[kMaxGroup];
    __shared__ float s_q[kMaxGroup][kD];

    const int bh = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b_seq = bh / a.H, h = bh - b_seq * a.H;
    const int G = a.G;
    const int es = a.is_bf16 ? 2 : 4;
    const int row_bytes = kD * es;
    const int vec_per_row = row_bytes / 16;
    unsigned char *sK = s_raw;
    unsigned char *sV = s_raw + (size_t)kTileRows * row_bytes;

    const int64_t qbase = ((int64_t)b_seq * a.H * G + (int64_t)h * G) * kD;
    for (int i = tid; i < G * kD; i += kAtThreads) s_q[i / kD][i % kD] = ld_as_f32(a.q, qbase + i, a.is_bf16);
    if (tid < G) {
        s_m[tid] = -INFINITY;
        s_l[tid] = 0.0f;
    }
    // output ownership: thread -> dim d, heads g = gsel, gsel + 2, ...
    const int d = tid & (kD - 1);
    const int gsel = tid >> 7;
    float acc[kMaxGroup / 2];
#pragma unroll
    for (int i = 0; i < kMaxGroup / 2; i++) acc[i] = 0.0f;

    const unsigned char *Kb = reinterpret_cast<const unsigned char *>(a.K) + (size_t)bh * a.n_cap * row_bytes;
    const unsigned char *Vb = reinterpret_cast<const unsigned char *>(a.V) + (size_t)bh * a.n_cap * row_bytes;
    const int32_t *sel = a.idx + (size_t)bh * a.topk;
    __syncthreads();

    for (int t0 = 0; t0 < a.topk; t0 += kTileRows) {
        const int rows = min(kTileRows, a.topk - t0);
        if (tid < rows) {
            const int32_t id = sel[t0 + tid];
            const bool ok = id >= 0 && (int64_t)id < a.n;
            if (!ok) devchk(a.dev_err, a.dev_err_detail, DEVCHK_BAD_INDEX, id);
            s_idx[tid] = ok ? id : -1;
        }
        __syncthreads();
        // stage K and V rows of the tile (all loads in flight together)
        for (int i = tid; i < rows * vec_per_row; i += kAtThreads) {
            const int r = i / vec_per_row, c = i - r * vec_per_row;
            const int32_t id = s_idx[r];
            uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
            if (id >= 0) {
                kv = *reinterpret_cast<const uint4 *>(Kb + (size_t)id * row_bytes + 16 * c);
                vv = *reinterpret_cast<const uint4 *>(Vb + (size_t)id * row_bytes + 16 * c);
            }
            *reinterpret_cast<uint4 *>(sK + (size_t)r * row_bytes + 16 * c) = kv;
            *reinterpret_cast<uint4 *>(sV + (size_t)r * row_bytes + 16 * c) = vv;
        }
        __syncthreads();
        // scores: warp w takes rows w, w+8, ..; lane holds dims 4 lane .. 4 lane + 3
        for (int r = warp; r < rows; r += kAtWarps) {
            float kx[4];
            if (a.is_bf16) {
                const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(sK + (size_t)r * row_bytes) + 2 * lane;
                const float2 f0 = __bfloat1622float2(p[0]), f1 = __bfloat1622float2(p[1]);
                kx[0] = f0.x; kx[1] = f0.y; kx[2] = f1.x; kx[3] = f1.y;
            } else {
                const float4 f = reinterpret_cast<const float4 *>(sK + (size_t)r * row_bytes)[lane];
                kx[0] = f.x; kx[1] = f.y; kx[2] = f.z; kx[3] = f.w;
            }
            for (int g = 0; g < G; g++) {
                float s = kx[0] * s_q[g][4 * lane] + kx[1] * s_q[g][4 * lane + 1] +
                          kx[2] * s_q[g][4 * lane + 2] + kx[3] * s_q[g][4 * lane + 3];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
                if (lane == 0) s_sc[g][r] = (s_idx[r] >= 0) ? s * a.scale : -INFINITY;
            }
        }
        __syncthreads();
        // online softmax bookkeeping: warp g handles head g
        if (warp < G) {
            const int g = warp;
            float mx = -INFINITY;
            for (int r = lane; r < rows; r += 32) mx = fmaxf(mx, s_sc[g][r]);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
            const float m_old = s_m[g];
            const float m_new = fmaxf(m_old, mx);
            float sum = 0.0f;
            for (int r = lane; r < rows; r += 32) {
                const float p = (m_new == -INFINITY) ? 0.0f : expf(s_sc[g][r] - m_new);
                s_sc[g][r] = p;
                sum += p;
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
            if (lane == 0) {
                const float alpha = (m_old == -INFINITY) ? 0.0f : expf(m_old - m_new);
                s_alpha[g] = alpha;
                s_l[g] = s_l[g] * alpha + sum;
                s_m[g] = m_new;
            }
        }
        __syncthreads();
        // P V: thread owns dim d of heads gsel, gsel + 2, ...
#pragma unroll
        for (int i = 0; i < kMaxGroup / 2; i++) {
            const int g = gsel + 2 * i;
            if (g < G) {
                float v = acc[i] * s_alpha[g];
                for (int r = 0; r < rows; r++) {
                    const float vv = a.is_bf16
                        ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sV + (size_t)r * row_bytes)[d])
                        : reinterpret_cast<const float *>(sV + (size_t)r * row_bytes)[d];
                    v = fmaf(s_sc[g][r], vv, v);
                }
                acc[i] = v;
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < kMaxGroup / 2; i++) {
        const int g = gsel + 2 * i;
        if (g < G) {
            const float l = s_l[g];
            a.out[qbase + (int64_t)g * kD + d] = (l > 0.0f) ? acc[i] / l : 0.0f;
        }
    }
}

size_t gather_attend_smem(int is_bf16) { return (size_t)2 * kTileRows * kD * (is_bf16 ? 2 : 4); }

}  // namespace pk

namespace pk {
cudaError_t launch_gather_attend(const AttendArgs &a, int bh, cudaStream_t s)
{
    const size_t smem = gather_attend_smem(a.is_bf16);
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k_gather_attend, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)gather_attend_smem(0));
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    k_gather_attend<<<bh, kAtThreads, smem, s>>>(a);
    return cudaGetLastError();
}
}  // namespace pk
