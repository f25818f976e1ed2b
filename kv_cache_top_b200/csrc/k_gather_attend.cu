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
// Grid (splits, pairs): each CTA takes up to 32 of the pair's selected rows
// and issues every 16-byte load of its K and V rows before using any, so a
// CTA costs one round trip over the host link; several CTAs per pair keep
// many rows in flight.  Each CTA computes a partial softmax (max, sum,
// weighted V) in fp32; the last CTA of the pair (ticket counter) merges the
// partials with the log-sum-exp rule.  Ids outside [0, n) are skipped and
// recorded in the device-check word (no trap).
#include "pk_internal.cuh"

namespace pk {

constexpr int kAtThreads = 256;
constexpr int kAtWarps = kAtThreads / 32;

__global__ void __launch_bounds__(kAtThreads) k_gather_attend(AttendArgs a)
{
    __shared__ __align__(16) unsigned char sK[kAtRows * kD * 4];
    __shared__ __align__(16) unsigned char sV[kAtRows * kD * 4];
    __shared__ int32_t s_idx[kAtRows];
    __shared__ float s_q[kMaxGroup][kD];
    __shared__ float s_p[kMaxGroup][kAtRows];
    __shared__ float s_m[kMaxGroup], s_l[kMaxGroup];
    __shared__ int s_last;

    const int sp = blockIdx.x, bh = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b_seq = bh / a.H, h = bh - b_seq * a.H;
    const int G = a.G;
    const int es = a.is_bf16 ? 2 : 4;
    const int row_bytes = kD * es;
    const int vpr = row_bytes / 16;
    const int r0 = sp * a.rows_per;
    const int rows = min(a.rows_per, a.topk - r0);

    const int64_t qbase = ((int64_t)b_seq * a.H * G + (int64_t)h * G) * kD;
    for (int i = tid; i < G * kD; i += kAtThreads) s_q[i / kD][i % kD] = ld_as_f32(a.q, qbase + i, a.is_bf16);
    if (tid < rows) {
        const int32_t id = a.idx[(size_t)bh * a.topk + r0 + tid];
        const bool ok = id >= 0 && (int64_t)id < a.n;
        if (!ok) devchk(a.dev_err, a.dev_err_detail, DEVCHK_BAD_INDEX, id);
        s_idx[tid] = ok ? id : -1;
    }
    __syncthreads();

    // ---- gather: every load of the CTA in flight at once
    const unsigned char *Kb = reinterpret_cast<const unsigned char *>(a.K) + (size_t)bh * a.stride * row_bytes;
    const unsigned char *Vb = reinterpret_cast<const unsigned char *>(a.V) + (size_t)bh * a.stride * row_bytes;
    const int nvec = rows * vpr;
    {
        uint4 kr[kAtRows * 32 / kAtThreads], vr[kAtRows * 32 / kAtThreads];
#pragma unroll
        for (int u = 0; u < kAtRows * 32 / kAtThreads; u++) {
            const int i = tid + u * kAtThreads;
            kr[u] = vr[u] = make_uint4(0, 0, 0, 0);
            if (i < nvec) {
                const int r = i / vpr, c = i - r * vpr;
                const int32_t id = s_idx[r];
                if (id >= 0) {
                    kr[u] = *reinterpret_cast<const uint4 *>(Kb + (size_t)id * row_bytes + 16 * c);
                    vr[u] = *reinterpret_cast<const uint4 *>(Vb + (size_t)id * row_bytes + 16 * c);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kAtRows * 32 / kAtThreads; u++) {
            const int i = tid + u * kAtThreads;
            if (i < nvec) {
                reinterpret_cast<uint4 *>(sK)[i] = kr[u];
                reinterpret_cast<uint4 *>(sV)[i] = vr[u];
            }
        }
    }
    __syncthreads();

    // ---- scores: warp w takes rows w, w+8, ..; lane holds dims 4 lane .. 4 lane + 3
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
            if (lane == 0) s_p[g][r] = (s_idx[r] >= 0) ? s * a.scale : -INFINITY;
        }
    }
    __syncthreads();
    // ---- partial softmax of this CTA's rows: warp g handles head g
    if (warp < G) {
        const int g = warp;
        float mx = -INFINITY;
        for (int r = lane; r < rows; r += 32) mx = fmaxf(mx, s_p[g][r]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        float sum = 0.0f;
        for (int r = lane; r < rows; r += 32) {
            const float p = (mx == -INFINITY) ? 0.0f : expf(s_p[g][r] - mx);
            s_p[g][r] = p;
            sum += p;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
        if (lane == 0) {
            s_m[g] = mx;
            s_l[g] = sum;
        }
    }
    __syncthreads();
    // ---- P V: thread owns dim d of heads gsel, gsel + 2, ...
    const int d = tid & (kD - 1);
    const int gsel = tid >> 7;
    float acc[kMaxGroup / 2];
#pragma unroll
    for (int i = 0; i < kMaxGroup / 2; i++) {
        const int g = gsel + 2 * i;
        float v = 0.0f;
        if (g < G) {
            for (int r = 0; r < rows; r++) {
                const float vv = a.is_bf16
                    ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sV + (size_t)r * row_bytes)[d])
                    : reinterpret_cast<const float *>(sV + (size_t)r * row_bytes)[d];
                v = fmaf(s_p[g][r], vv, v);
            }
        }
        acc[i] = v;
    }
    if (a.nsplit == 1) {
#pragma unroll
        for (int i = 0; i < kMaxGroup / 2; i++) {
            const int g = gsel + 2 * i;
            if (g < G) a.out[qbase + (int64_t)g * kD + d] = (s_l[g] > 0.0f) ? acc[i] / s_l[g] : 0.0f;
        }
        return;
    }
    // ---- several CTAs per pair: publish the partial, the last one merges
    float *part = a.part + ((size_t)bh * a.max_splits + sp) * kMaxGroup * (kD + 2);
#pragma unroll
    for (int i = 0; i < kMaxGroup / 2; i++) {
        const int g = gsel + 2 * i;
        if (g < G) part[g * (kD + 2) + d] = acc[i];
    }
    if (tid < G) {
        part[tid * (kD + 2) + kD] = s_m[tid];
        part[tid * (kD + 2) + kD + 1] = s_l[tid];
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&a.tickets[bh], 1u) == (unsigned)(a.nsplit - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
#pragma unroll
    for (int i = 0; i < kMaxGroup / 2; i++) {
        const int g = gsel + 2 * i;
        if (g >= G) continue;
        float M = -INFINITY;
        for (int s = 0; s < a.nsplit; s++) {
            const float *ps = a.part + ((size_t)bh * a.max_splits + s) * kMaxGroup * (kD + 2) + g * (kD + 2);
            M = fmaxf(M, __ldcg(ps + kD));
        }
        float num = 0.0f, den = 0.0f;
        if (M != -INFINITY) {
            for (int s = 0; s < a.nsplit; s++) {
                const float *ps = a.part + ((size_t)bh * a.max_splits + s) * kMaxGroup * (kD + 2) + g * (kD + 2);
                const float ms = __ldcg(ps + kD);
                const float f = (ms == -INFINITY) ? 0.0f : expf(ms - M);
                num = fmaf(f, __ldcg(ps + d), num);
                den = fmaf(f, __ldcg(ps + kD + 1), den);
            }
        }
        a.out[qbase + (int64_t)g * kD + d] = (den > 0.0f) ? num / den : 0.0f;
    }
    if (tid == 0) a.tickets[bh] = 0u;
}

cudaError_t launch_gather_attend(const AttendArgs &a, int bh, cudaStream_t s)
{
    k_gather_attend<<<dim3(a.nsplit, bh), kAtThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace pk
