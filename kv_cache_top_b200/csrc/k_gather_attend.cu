// k_gather_attend.cu -- gather of the selected K/V rows and exact attention.
//
// o_g = sum_r softmax_r(scale <q_g, K[sel_r]>) V[sel_r] for every query head
// g of the KV head (ParisKV slides, "The target is high-score KV indices at
// each decode step", Sec. 3 Eqs. 1-3: "recompute softmax and value
// aggregation using the selected full-precision KV").  Optionally the rows
// kept densely on the GPU outside the index -- the sink and recent local
// tokens -- join the same softmax (README, step 3: attention "over sink
// tokens, local tokens, and retrieved tokens"; slides, Fig. 5 layout).  The K/V rows are read
// where the index keeps them: HBM, or pinned host memory through UVA (README,
// "Attention: fetch only selected KV pairs ... from pinned CPU memory via
// UVA").
//
// One thread-block cluster per pair (grid x = cluster x = splits <= 8): each
// CTA takes a contiguous share of the selected rows, 32 rows per tile, and
// issues every 16-byte load of a tile's K and V rows before using any, so a
// tile costs one round trip over the host link and several SMs pull rows at
// once.  Each CTA keeps an online softmax (max, sum, weighted V) in fp32, then
// pushes its partial into CTA rank 0's shared memory with distributed-shared-
// memory stores (no remote round trip), and rank 0 merges the partials with
// the log-sum-exp rule.  Ids outside [0, n) are skipped and recorded in the
// device-check word (no trap).
#include <cooperative_groups.h>

#include "pk_internal.cuh"

namespace cg = cooperative_groups;

namespace pk {

constexpr int kAtThreads = 256;
constexpr int kAtWarps = kAtThreads / 32;
constexpr int kAtLoads = kAtRows * 32 / kAtThreads;   // 16-byte loads per thread per tile

__global__ void __launch_bounds__(kAtThreads, 4) k_gather_attend(AttendArgs a)
{
    // the K and V tiles; after the row loop rank 0 reuses them for the
    // cluster's partial accumulators [8][kMaxGroup][kD] (32 KB)
    __shared__ __align__(16) unsigned char s_kv[2 * kAtRows * kD * 4];
    unsigned char *sK = s_kv;
    unsigned char *sV = s_kv + kAtRows * kD * 4;
    __shared__ int32_t s_idx[kAtRows];
    __shared__ float s_q[kMaxGroup][kD];
    __shared__ float s_p[kMaxGroup][kAtRows];
    __shared__ float s_m[kMaxGroup], s_l[kMaxGroup], s_alpha[kMaxGroup];
    // rank 0 only: every CTA's partial (running max, sum, accumulator), pushed
    // here with distributed-shared-memory stores before the cluster barrier
    __shared__ float s_pm[8][kMaxGroup], s_pl[8][kMaxGroup];
    static_assert(8 * kMaxGroup * kD * 4 <= 2 * kAtRows * kD * 4, "partials fit in the row tiles");
    float (*s_pacc)[kMaxGroup][kD] = reinterpret_cast<float (*)[kMaxGroup][kD]>(s_kv);

    cg::cluster_group cluster = cg::this_cluster();
    const int sp = (int)cluster.block_rank(), bh = blockIdx.y;
    const int nsp = a.nsplit;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b_seq = bh / a.H, h = bh - b_seq * a.H;
    const int G = a.G;
    const int es = a.is_bf16 ? 2 : 4;
    const int row_bytes = kD * es;
    const int vpr = row_bytes / 16;
    // the pair's rows: the topk selected ids, then the dlen dense rows
    const int nrows = a.topk + a.dlen;
    const int per = (nrows + nsp - 1) / nsp;
    const int r_beg = min(nrows, sp * per), r_end = min(nrows, r_beg + per);

    const int64_t qbase = ((int64_t)b_seq * a.H * G + (int64_t)h * G) * kD;
    for (int i = tid; i < G * kD; i += kAtThreads) s_q[i / kD][i % kD] = ld_as_f32(a.q, qbase + i, a.is_bf16);
    if (tid < G) {
        s_m[tid] = -INFINITY;
        s_l[tid] = 0.0f;
    }
    pdl_wait();                                   // the selected ids may come from the search
    const size_t kp = (size_t)index_pair(bh, a.kvg);     // the index pair holding this unit's rows
    const unsigned char *Kb = reinterpret_cast<const unsigned char *>(a.K) + kp * a.stride * row_bytes;
    const unsigned char *Vb = reinterpret_cast<const unsigned char *>(a.V) + kp * a.stride * row_bytes;
    const unsigned char *dKb = a.dlen ? reinterpret_cast<const unsigned char *>(a.dK) + kp * a.dstride * row_bytes : nullptr;
    const unsigned char *dVb = a.dlen ? reinterpret_cast<const unsigned char *>(a.dV) + kp * a.dstride * row_bytes : nullptr;
    const int d = tid & (kD - 1);
    const int gsel = tid >> 7;
    float acc[kMaxGroup / 2];
#pragma unroll
    for (int i = 0; i < kMaxGroup / 2; i++) acc[i] = 0.0f;

    for (int t0 = r_beg; t0 < r_end; t0 += kAtRows) {
        const int rows = min(kAtRows, r_end - t0);
        __syncthreads();                                  // previous tile fully consumed
        // row slot code: a selected id (>= 0), -1 (id out of range: skipped),
        // or -2 - j for dense row j
        if (tid < rows) {
            const int rr = t0 + tid;
            if (rr < a.topk) {
                const int32_t id = a.idx[(size_t)bh * a.topk + rr];
                const bool ok = id >= 0 && (int64_t)id < a.n;
                if (!ok) devchk(a.dev_err, a.dev_err_detail, DEVCHK_BAD_INDEX, id);
                s_idx[tid] = ok ? id : -1;
            } else {
                s_idx[tid] = -2 - (rr - a.topk);
            }
        }
        __syncthreads();
        // ---- gather: every load of the tile in flight at once
        const int nvec = rows * vpr;
        uint4 kr[kAtLoads], vr[kAtLoads];
#pragma unroll
        for (int u = 0; u < kAtLoads; u++) {
            const int i = tid + u * kAtThreads;
            kr[u] = vr[u] = make_uint4(0, 0, 0, 0);
            if (i < nvec) {
                const int r = i / vpr, c = i - r * vpr;
                const int32_t id = s_idx[r];
                if (id >= 0) {
                    kr[u] = *reinterpret_cast<const uint4 *>(Kb + (size_t)id * row_bytes + 16 * c);
                    vr[u] = *reinterpret_cast<const uint4 *>(Vb + (size_t)id * row_bytes + 16 * c);
                } else if (id <= -2) {
                    const size_t j = (size_t)(-2 - id);
                    kr[u] = *reinterpret_cast<const uint4 *>(dKb + j * row_bytes + 16 * c);
                    vr[u] = *reinterpret_cast<const uint4 *>(dVb + j * row_bytes + 16 * c);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kAtLoads; u++) {
            const int i = tid + u * kAtThreads;
            if (i < nvec) {
                reinterpret_cast<uint4 *>(sK)[i] = kr[u];
                reinterpret_cast<uint4 *>(sV)[i] = vr[u];
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
                if (lane == 0) s_p[g][r] = (s_idx[r] != -1) ? s * a.scale : -INFINITY;
            }
        }
        __syncthreads();
        // ---- online softmax bookkeeping: warp g handles head g
        if (warp < G) {
            const int g = warp;
            float mx = -INFINITY;
            for (int r = lane; r < rows; r += 32) mx = fmaxf(mx, s_p[g][r]);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
            const float m_old = s_m[g];
            const float m_new = fmaxf(m_old, mx);
            float sum = 0.0f;
            for (int r = lane; r < rows; r += 32) {
                const float p = (m_new == -INFINITY) ? 0.0f : expf(s_p[g][r] - m_new);
                s_p[g][r] = p;
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
        // ---- P V: thread owns dim d of heads gsel, gsel + 2, ...
#pragma unroll
        for (int i = 0; i < kMaxGroup / 2; i++) {
            const int g = gsel + 2 * i;
            if (g < G) {
                float v = acc[i] * s_alpha[g];
                for (int r = 0; r < rows; r++) {
                    const float vv = a.is_bf16
                        ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sV + (size_t)r * row_bytes)[d])
                        : reinterpret_cast<const float *>(sV + (size_t)r * row_bytes)[d];
                    v = fmaf(s_p[g][r], vv, v);
                }
                acc[i] = v;
            }
        }
    }
    // ---- push this CTA's partial into rank 0 (remote stores: no round trip)
    float *pm = cluster.map_shared_rank(&s_pm[0][0], 0);
    float *pl = cluster.map_shared_rank(&s_pl[0][0], 0);
    float *pacc = cluster.map_shared_rank(&s_pacc[0][0][0], 0);
    cluster.sync();                                   // every CTA is done with its rows (and s_m, s_l)
    if (tid < G) {
        pm[sp * kMaxGroup + tid] = s_m[tid];
        pl[sp * kMaxGroup + tid] = s_l[tid];
    }
#pragma unroll
    for (int i = 0; i < kMaxGroup / 2; i++) {
        const int g = gsel + 2 * i;
        if (g < G) pacc[((size_t)sp * kMaxGroup + g) * kD + d] = acc[i];
    }
    cluster.sync();                                   // every partial has landed in rank 0
    if (sp == 0) {
        // log-sum-exp merge of the nsp partials, from local shared memory
#pragma unroll
        for (int i = 0; i < kMaxGroup / 2; i++) {
            const int g = gsel + 2 * i;
            if (g >= G) continue;
            float M = -INFINITY;
            for (int r = 0; r < nsp; r++) M = fmaxf(M, s_pm[r][g]);
            float num = 0.0f, den = 0.0f;
            if (M != -INFINITY) {
                for (int r = 0; r < nsp; r++) {
                    const float mr = s_pm[r][g];
                    const float f = (mr == -INFINITY) ? 0.0f : expf(mr - M);
                    num = fmaf(f, s_pacc[r][g][d], num);
                    den = fmaf(f, s_pl[r][g], den);
                }
            }
            a.out[qbase + (int64_t)g * kD + d] = (den > 0.0f) ? num / den : 0.0f;
        }
    }
}

cudaError_t launch_gather_attend(const AttendArgs &a, int bh, cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.nsplit, bh, 1);
    cfg.blockDim = dim3(kAtThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.nsplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k_gather_attend, a);
}

}  // namespace pk
