// k_gather_attend.cu -- gather of the selected K/V rows and exact attention.
//
// o_g = sum_r softmax_r(scale <q_g, K[sel_r]>) V[sel_r] for every query head
// g of the KV head (ParisKV slides, Sec. 3 Eqs. 1-3: softmax and the value sum
// are computed again over the selected rows, in full precision).  Optionally
// the rows kept densely on the GPU outside the index -- the sink and recent
// local tokens -- join the same softmax (README, pipeline step 3; slides,
// Fig. 5 layout).  The K/V rows are read where the index keeps them: HBM, or
// pinned host memory through UVA (README, pipeline step 3: only the selected
// rows cross from host memory, read through UVA).
//
// One thread-block cluster per pair (grid x = cluster x = splits <= 8): each
// CTA takes a contiguous share of the selected rows, 32 rows per tile, and
// issues every 16-byte load of a tile's K and V rows before using any, so a
// tile costs one round trip over the host link and several SMs pull rows at
// once.  A tile's scores take 8 threads per row, each a partial dot over
// every 8th 16-byte piece of the row (conflict-free shared-memory reads), and
// 3 shuffles.  Each CTA keeps an online softmax (max, sum, weighted V) in
// fp32, then pushes its partial into a region of CTA rank 0's shared memory
// that nothing else uses, with distributed-shared-memory stores (no remote
// round trip), and arrives at the cluster barrier; rank 0 merges the
// partials with the log-sum-exp rule.  The only other cluster barrier phase
// is arrived at on entry, so the pushes know every CTA of the cluster runs.
// Ids outside [0, n) are skipped and recorded in the device-check word (no
// trap).
//
// Per-query-head rows (union_heads): each query head of the pair has its own
// list, and one cluster serves all G heads.  In the prologue every CTA puts
// the pair's G x topk ids into the same open-addressing table in shared
// memory (over the not yet used K/V tiles): key = id + 1, with the mask of
// heads whose list holds it and the smallest entry index e = g topk + r that
// holds it.  Entry e is a row iff it is that smallest index, so the rows are
// the union of the lists in order of first appearance: the same on every CTA,
// each id once, whatever order the inserts ran in.  Each row is fetched once; head g
// scores it only if its mask holds g (others see -inf, weight 0).
#include <cooperative_groups.h>

#include "pk_internal.cuh"
#include "pk_launch.cuh"

namespace cg = cooperative_groups;

namespace pk {

constexpr int kAtThreads = 256;
constexpr int kAtLoads = kAtRows * 32 / kAtThreads;   // 16-byte loads per thread per tile
constexpr int kQPad = kD + kD / 8;                    // padded query row (4 floats after every 32)

// query element d of a head in the padded row: the 8 threads of a score row
// read 16-byte pieces whose banks then never collide
__device__ __forceinline__ int qpad(int d) { return d + 4 * (d >> 5); }

// split cluster barrier (every thread of every CTA of the cluster takes part)
__device__ __forceinline__ void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// dynamic shared memory: the partials [nsplit][G][kD] fp32, then (union
// rows only) the row list [G x topk] of (head mask << 32 | id)
size_t attend_smem(int nsplit, int G, int union_entries)
{
    return (size_t)nsplit * G * kD * sizeof(float) + (size_t)union_entries * sizeof(unsigned long long);
}

// open-addressing slots for E union entries: a power of two >= 2E
__host__ __device__ inline int union_slots(int E)
{
    int h = 64;
    while (h < 2 * E) h <<= 1;
    return h;
}

__device__ __forceinline__ uint32_t union_hash(uint32_t key)
{
    return key * 0x9E3779B1u;     // Fibonacci hashing; the slot index takes the high bits
}

__global__ void __launch_bounds__(kAtThreads, 3) k_gather_attend(AttendArgs a)
{
    // the K and V tiles
    __shared__ __align__(16) unsigned char s_kv[2 * kAtRows * kD * 4];
    unsigned char *sK = s_kv;
    unsigned char *sV = s_kv + kAtRows * kD * 4;
    __shared__ int32_t s_idx[kAtRows];
    __shared__ uint32_t s_msk[kAtRows];            // heads that score the row (union rows)
    __shared__ uint32_t s_ws[kAtThreads / 32 + 1];
    __shared__ __align__(16) float s_q[kMaxGroup][kQPad];
    __shared__ float s_p[kMaxGroup][kAtRows];
    __shared__ float s_m[kMaxGroup], s_l[kMaxGroup], s_alpha[kMaxGroup];
    // rank 0 only: every CTA's partial (running max, sum, accumulator), pushed
    // here with distributed-shared-memory stores before the cluster barrier
    __shared__ float s_pm[8][kMaxGroup], s_pl[8][kMaxGroup];
    extern __shared__ __align__(16) float s_pacc[];            // [nsplit][G][kD]

    cluster_arrive_relaxed();                     // this CTA runs (waited for before the pushes)
    cg::cluster_group cluster = cg::this_cluster();
    const int sp = (int)cluster.block_rank(), bh = blockIdx.y;
    const int nsp = a.nsplit;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b_seq = bh / a.H, h = bh - b_seq * a.H;
    const int G = a.G;
    const int es = a.is_bf16 ? 2 : 4;
    const int row_bytes = kD * es;
    const int vpr = row_bytes / 16;
    const int64_t qbase = ((int64_t)b_seq * a.H * G + (int64_t)h * G) * kD;
    if (tid < G) {
        s_m[tid] = -INFINITY;
        s_l[tid] = 0.0f;
    }
    unsigned long long *s_rows = reinterpret_cast<unsigned long long *>(s_pacc + (size_t)nsp * G * kD);
    pdl_wait();                                   // the selected ids may come from the search
    // the pair's rows: the topk selected ids (or the union of the G heads'
    // lists), then the dlen dense rows
    int nsel = a.topk;
    if (a.union_heads) {
        const int E = G * a.topk, HS = union_slots(E);
        const int32_t *ids = a.idx + (size_t)bh * E;
        // keys, head masks, first entries: 12 HS bytes <= the K/V tiles (HS <= 2048)
        uint32_t *hk = reinterpret_cast<uint32_t *>(s_kv), *hm = hk + HS, *hf = hm + HS;
        for (int i = tid; i < HS; i += kAtThreads) {
            hk[i] = hm[i] = 0u;
            hf[i] = 0xffffffffu;
        }
        __syncthreads();
        const int sh = 32 - (31 - __clz(HS));         // slot = high log2(HS) bits of the hash
        // insert (e >= 0): claim or find the key's slot, add head e / topk and entry e;
        // look up (e < 0): the key's slot or -1.  At most HS probes; E < HS keys.
        auto slot_of = [&](uint32_t key, int e) -> int {
            uint32_t p = union_hash(key) >> sh;
            for (int t = 0; t < HS; t++, p = (p + 1) & (HS - 1)) {
                const uint32_t cur = e >= 0 ? atomicCAS(&hk[p], 0u, key) : hk[p];
                if (cur == key || (e >= 0 && cur == 0u)) {
                    if (e >= 0) {
                        atomicOr(&hm[p], 1u << (e / a.topk));
                        atomicMin(&hf[p], (uint32_t)e);
                    }
                    return (int)p;
                }
                if (cur == 0u) return -1;
            }
            return -1;
        };
        for (int e = tid; e < E; e += kAtThreads) {
            const int32_t id = ids[e];
            if (id >= 0 && (int64_t)id < a.n) slot_of((uint32_t)id + 1u, e);
            else devchk(a.dev_err, a.dev_err_detail, DEVCHK_BAD_INDEX, id);
        }
        __syncthreads();
        // rows in entry order: thread t takes entries [t * per_t, ...) so the scan keeps that order
        const int per_t = (E + kAtThreads - 1) / kAtThreads;
        const int e0 = tid * per_t, e1 = min(E, e0 + per_t);
        uint32_t cnt = 0;
        for (int e = e0; e < e1; e++) {
            const int32_t id = ids[e];
            if (id >= 0 && (int64_t)id < a.n) {
                const int p = slot_of((uint32_t)id + 1u, -1);
                cnt += (p >= 0 && hf[p] == (uint32_t)e);
            }
        }
        uint32_t tot;
        uint32_t pos = block_excl_scan<kAtThreads>(cnt, s_ws, &tot);
        for (int e = e0; e < e1; e++) {
            const int32_t id = ids[e];
            if (id >= 0 && (int64_t)id < a.n) {
                const int p = slot_of((uint32_t)id + 1u, -1);
                if (p >= 0 && hf[p] == (uint32_t)e)
                    s_rows[pos++] = ((unsigned long long)hm[p] << 32) | (uint32_t)id;
            }
        }
        nsel = (int)tot;
        __syncthreads();                          // rows written; the table's storage goes back to the tiles
    }
    const int nrows = nsel + a.dlen;
    const int per = (nrows + nsp - 1) / nsp;
    const int r_beg = min(nrows, sp * per), r_end = min(nrows, r_beg + per);
    // the first tile's selected ids and the query heads load together (one round trip)
    const int rr0 = r_beg + tid;
    const int32_t id0 = (tid < kAtRows && rr0 < r_end && rr0 < nsel && !a.union_heads)
        ? a.idx[(size_t)bh * a.topk + rr0] : 0;
    {   // the query heads: 16-byte loads when the rows start on a 16-byte boundary
        const uintptr_t at = reinterpret_cast<uintptr_t>(a.q) + (uintptr_t)qbase * (uintptr_t)es;
        if ((at & 15u) == 0 && a.is_bf16) {
            for (int v = tid; v < G * kD / 8; v += kAtThreads) {
                const uint4 x = reinterpret_cast<const uint4 *>(at)[v];
                const int g = v / (kD / 8), d0 = 8 * (v % (kD / 8));   // 8 elements in one 32-group
                const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.x));
                const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.y));
                const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.z));
                const float2 f3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.w));
                float4 *dst = reinterpret_cast<float4 *>(&s_q[g][qpad(d0)]);
                dst[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
                dst[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
            }
        } else if ((at & 15u) == 0) {
            for (int v = tid; v < G * kD / 4; v += kAtThreads) {
                const int g = v / (kD / 4), d0 = 4 * (v % (kD / 4));
                *reinterpret_cast<float4 *>(&s_q[g][qpad(d0)]) = reinterpret_cast<const float4 *>(at)[v];
            }
        } else {
            for (int i = tid; i < G * kD; i += kAtThreads) s_q[i / kD][qpad(i % kD)] = ld_as_f32(a.q, qbase + i, a.is_bf16);
        }
    }
    const size_t kp = (size_t)index_pair(bh, a.kvg);     // the index pair holding this unit's rows
    const unsigned char *Kb = reinterpret_cast<const unsigned char *>(a.K) + kp * a.stride * a.kv_pitch;
    const unsigned char *Vb = reinterpret_cast<const unsigned char *>(a.V) + kp * a.stride * a.kv_pitch;
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
            if (rr < nsel && a.union_heads) {     // checked and deduplicated in the prologue
                const unsigned long long rw = s_rows[rr];
                s_idx[tid] = (int32_t)(uint32_t)rw;
                s_msk[tid] = (uint32_t)(rw >> 32);
            } else if (rr < nsel) {
                const int32_t id = t0 == r_beg ? id0 : a.idx[(size_t)bh * a.topk + rr];
                const bool ok = id >= 0 && (int64_t)id < a.n;
                if (!ok) devchk(a.dev_err, a.dev_err_detail, DEVCHK_BAD_INDEX, id);
                s_idx[tid] = ok ? id : -1;
                s_msk[tid] = ~0u;
            } else {
                s_idx[tid] = -2 - (rr - nsel);
                s_msk[tid] = ~0u;
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
                    kr[u] = *reinterpret_cast<const uint4 *>(Kb + (size_t)id * a.kv_pitch + 16 * c);
                    vr[u] = *reinterpret_cast<const uint4 *>(Vb + (size_t)id * a.kv_pitch + 16 * c);
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
        // ---- scores: thread (row tid / 8, part j = tid % 8) dots 16-byte pieces
        // j, j + 8, .. of the row with the matching query elements
        {
            const int r = tid >> 3, j = tid & 7;
            float sc[kMaxGroup];
#pragma unroll
            for (int g = 0; g < kMaxGroup; g++) sc[g] = 0.0f;
            if (r < rows) {
                const uint4 *krow = reinterpret_cast<const uint4 *>(sK + (size_t)r * row_bytes);
                if (a.is_bf16) {
#pragma unroll
                    for (int c = j; c < kD / 8; c += 8) {            // 8 bf16 per piece
                        const uint4 kv = krow[c];
                        const float2 k0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kv.x));
                        const float2 k1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kv.y));
                        const float2 k2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kv.z));
                        const float2 k3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kv.w));
                        const int q0 = qpad(8 * c);
#pragma unroll
                        for (int g = 0; g < kMaxGroup; g++) {
                            if (g < G) {
                                const float4 qa = *reinterpret_cast<const float4 *>(&s_q[g][q0]);
                                const float4 qb = *reinterpret_cast<const float4 *>(&s_q[g][q0 + 4]);
                                float t = sc[g];
                                t = fmaf(k0.x, qa.x, t); t = fmaf(k0.y, qa.y, t);
                                t = fmaf(k1.x, qa.z, t); t = fmaf(k1.y, qa.w, t);
                                t = fmaf(k2.x, qb.x, t); t = fmaf(k2.y, qb.y, t);
                                t = fmaf(k3.x, qb.z, t); t = fmaf(k3.y, qb.w, t);
                                sc[g] = t;
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int c = j; c < kD / 4; c += 8) {            // 4 fp32 per piece
                        const float4 kv = reinterpret_cast<const float4 *>(krow)[c];
                        const int q0 = qpad(4 * c);
#pragma unroll
                        for (int g = 0; g < kMaxGroup; g++) {
                            if (g < G) {
                                const float4 qa = *reinterpret_cast<const float4 *>(&s_q[g][q0]);
                                float t = sc[g];
                                t = fmaf(kv.x, qa.x, t); t = fmaf(kv.y, qa.y, t);
                                t = fmaf(kv.z, qa.z, t); t = fmaf(kv.w, qa.w, t);
                                sc[g] = t;
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < kMaxGroup; g++) {
                if (g < G) {
                    sc[g] += __shfl_xor_sync(kFull, sc[g], 1);
                    sc[g] += __shfl_xor_sync(kFull, sc[g], 2);
                    sc[g] += __shfl_xor_sync(kFull, sc[g], 4);
                    if (j == 0 && r < rows)
                        s_p[g][r] = (s_idx[r] != -1 && ((s_msk[r] >> g) & 1u)) ? sc[g] * a.scale : -INFINITY;
                }
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
                const float p = (m_new == -INFINITY) ? 0.0f : __expf(s_p[g][r] - m_new);
                s_p[g][r] = p;
                sum += p;
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
            if (lane == 0) {
                const float alpha = (m_old == -INFINITY) ? 0.0f : __expf(m_old - m_new);
                s_alpha[g] = alpha;
                s_l[g] = s_l[g] * alpha + sum;
                s_m[g] = m_new;
            }
        }
        __syncthreads();
        // ---- P V: thread owns dim d of heads gsel, gsel + 2, ...
        // (one V element per row, used by every head this thread owns)
#pragma unroll
        for (int i = 0; i < kMaxGroup / 2; i++)
            if (gsel + 2 * i < G) acc[i] *= s_alpha[gsel + 2 * i];
#pragma unroll 4
        for (int r = 0; r < rows; r++) {
            const float vv = a.is_bf16
                ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sV + (size_t)r * row_bytes)[d])
                : reinterpret_cast<const float *>(sV + (size_t)r * row_bytes)[d];
#pragma unroll
            for (int i = 0; i < kMaxGroup / 2; i++)
                if (gsel + 2 * i < G) acc[i] = fmaf(s_p[gsel + 2 * i][r], vv, acc[i]);
        }
    }
    // ---- push this CTA's partial into rank 0 (remote stores: no round trip)
    float *pm = cluster.map_shared_rank(&s_pm[0][0], 0);
    float *pl = cluster.map_shared_rank(&s_pl[0][0], 0);
    float *pacc = cluster.map_shared_rank(s_pacc, 0);
    cluster_wait();                                   // every CTA of the cluster has started
    if (tid < G) {
        pm[sp * kMaxGroup + tid] = s_m[tid];
        pl[sp * kMaxGroup + tid] = s_l[tid];
    }
#pragma unroll
    for (int i = 0; i < kMaxGroup / 2; i++) {
        const int g = gsel + 2 * i;
        if (g < G) pacc[((size_t)sp * G + g) * kD + d] = acc[i];
    }
    cluster_arrive();
    cluster_wait();                                   // every partial has landed in rank 0
    if (sp == 0) {
        // log-sum-exp merge of the nsp partials, from local shared memory: the
        // weight e^(m_r - M) / sum_r' e^(m_r' - M) l_r' of partial r and head g
        // once per (r, g), then one weighted sum per output
        __shared__ float s_w[8][kMaxGroup];
        if (tid < G) {
            const int g = tid;
            float M = -INFINITY;
            for (int r = 0; r < nsp; r++) M = fmaxf(M, s_pm[r][g]);
            float den = 0.0f;
            for (int r = 0; r < nsp; r++) {
                const float mr = s_pm[r][g];
                const float f = (M == -INFINITY || mr == -INFINITY) ? 0.0f : __expf(mr - M);
                s_w[r][g] = f;
                den = fmaf(f, s_pl[r][g], den);
            }
            const float inv = den > 0.0f ? 1.0f / den : 0.0f;
            for (int r = 0; r < nsp; r++) s_w[r][g] *= inv;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kMaxGroup / 2; i++) {
            const int g = gsel + 2 * i;
            if (g >= G) continue;
            float num = 0.0f;
            for (int r = 0; r < nsp; r++) num = fmaf(s_w[r][g], s_pacc[((size_t)r * G + g) * kD + d], num);
            a.out[qbase + (int64_t)g * kD + d] = num;
        }
    }
}

cudaError_t launch_gather_attend(const AttendArgs &a, int bh, cudaStream_t s)
{
    static std::atomic<int> smem_set[kMaxDevices];   // the partials region may pass 48 KB in total
    const cudaError_t e = dyn_smem_limit(k_gather_attend, (int)attend_smem(8, kMaxGroup, kUnionMax), smem_set);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.nsplit, bh, 1);
    cfg.blockDim = dim3(kAtThreads, 1, 1);
    cfg.dynamicSmemBytes = attend_smem(a.nsplit, a.G, a.union_heads ? a.G * a.topk : 0);
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
