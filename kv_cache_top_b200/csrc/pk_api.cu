// pk_api.cu -- host side of the C-ABI declared in include/pariskv.h:
// argument checks, index storage, launch configuration and tracing.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "pk_internal.cuh"

using namespace pk;

struct TraceRec {
    int kind;
    cudaEvent_t a, b;
};

// Search workspace for `units` query units: one per pair for the aggregated
// query, G per pair for per-query-head search.
struct Work {
    int32_t units = 0;
    int32_t scan_units = 0;      // CTAs' worth of work units per chunk of the scan: units, or pairs
                                 // when one scan pass serves the G query heads of a pair
    uint8_t *bonus_bytes = nullptr;   // [pairs][16][256][np] u32: the kvg heads' bonuses packed per pair (per-head search)
    int32_t max_chunks = 1, max_slices = 1;
    float *qt = nullptr, *qnorm = nullptr;
    uint32_t *bonus_packed = nullptr;
    uint8_t *S = nullptr;
    uint32_t *chunk_cum = nullptr, *head_hist = nullptr, *tickets = nullptr;
    uint2 *chunk_info = nullptr;
    int32_t *sstar = nullptr;
    int32_t *cand = nullptr;
    unsigned long long *partial = nullptr;
};

struct pk_index {
    pk_params p;
    int32_t bh = 0;
    int64_t n = 0;
    int64_t stride = 0;          // rows per pair in every per-key array (n_cap rounded up to 16)
    int device = 0;
    int num_sms = 148;
    int32_t topk_cap = 100;
    int es = 2;
    float scale = 0.0f;
    RotConst rot{};
    Levels lv{};
    // index storage (device)
    uint8_t *codes = nullptr;
    uint8_t *rec = nullptr;
    uint32_t *occ = nullptr;
    // K/V store (device, or mapped pinned host): one allocation [BH][stride][2][D],
    // the K and V rows of a key adjacent (one translation covers both when the
    // attention gathers them); K and V point at the first K and V row
    void *KV = nullptr, *K = nullptr, *V = nullptr;
    bool kv_host = false;
    // staged appends: n_staged keys encoded at rows n .. n + n_staged - 1,
    // their occupancy counts in occ_stage [BH][16][256] (zero when nothing is
    // staged), not yet visible to search; stage_ev marks the staging work
    int64_t n_staged = 0;
    uint32_t *occ_stage = nullptr;
    cudaEvent_t stage_ev = nullptr;
    // search workspaces (device): w for the aggregated query, wh for
    // per-query-head search (made on first use)
    Work w, wh;

    int32_t *dev_err = nullptr;
    long long *dev_err_detail = nullptr;
    // tracing
    bool trace = false;
    std::vector<TraceRec> tr;
    std::vector<cudaEvent_t> ev_pool;
    size_t ev_used = 0;
};

namespace {

constexpr int64_t kMinChunk = 1024;
constexpr int64_t kMaxChunk = 32768;   // keys per chunk: the compaction kernel holds a chunk in registers

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

pk_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return PK_OK;
    if (e == cudaErrorMemoryAllocation) return PK_ERR_OOM;
    return PK_ERR_CUDA;
}

// A pointer the GPU can read: device memory of the current device, or
// page-locked / managed host memory.
bool device_accessible(const void *ptr)
{
    if (!ptr) return false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (at.type == cudaMemoryTypeDevice) {
        // device memory of another GPU is not read through here: the kernels
        // launch on the current device
        int dev = -1;
        return cudaGetDevice(&dev) == cudaSuccess && at.device == dev;
    }
    return at.type == cudaMemoryTypeHost || at.type == cudaMemoryTypeManaged;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

void ratio_table(int64_t n, double *beta, double *rho)
{
    // README adaptive ratio table; K = 1000, half-open ranges.
    if (n < 5000) { *beta = 0.50; *rho = 0.50; }
    else if (n < 10000) { *beta = 0.25; *rho = 0.30; }
    else if (n < 30000) { *beta = 0.20; *rho = 0.25; }
    else { *beta = 0.10; *rho = 0.20; }
}

void resolve(int64_t n, int64_t cand_budget, float collision_ratio, int32_t topk, int64_t *C,
             int64_t *R)
{
    double beta, rho;
    ratio_table(n, &beta, &rho);
    int64_t c = cand_budget > 0 ? cand_budget : (int64_t)std::ceil(beta * (double)n);
    if (c < topk) c = topk;
    if (c > n) c = n;
    const double r = collision_ratio > 0.0f ? (double)collision_ratio : rho;
    int64_t rr = (int64_t)std::ceil(r * (double)n);
    if (rr < 1) rr = 1;
    if (rr > n) rr = n;
    *C = c;
    *R = rr;
}

uint64_t splitmix64(uint64_t x)
{
    uint64_t z = x + 0x9e3779b97f4a7c15ULL;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

// Key chunks of the scan and the compaction: at most one wave (4 resident
// CTAs per SM) when the chunk-size cap allows, never fewer than
// ceil(n / kMaxChunk) chunks.
void chunking(const pk_index *ix, const Work &w, int64_t n, int32_t *nchunks, int64_t *chunk)
{
    int64_t nch = std::max<int64_t>(1, (4 * (int64_t)ix->num_sms) / w.scan_units);
    nch = std::min<int64_t>(nch, ceil_div(n, kMinChunk));
    nch = std::max<int64_t>(nch, ceil_div(n, kMaxChunk));
    nch = std::max<int64_t>(1, std::min<int64_t>(nch, w.max_chunks));
    int64_t ch = ceil_div(ceil_div(n, nch), 16) * 16;
    *chunk = ch;
    *nchunks = (int32_t)ceil_div(n, ch);
}

// rerank work split: slices of each unit's candidate list.  A CTA of nt
// threads holds at most kSelPer x nt candidates, and 512 / nt CTAs fit on an
// SM.  Per CTA size: at most one wave unless the slice cap forces more; then
// the size whose busiest SM gets fewer records (ties: 256, fewer lists to
// merge).
int32_t slice_lo(const pk_index *ix) { return std::max<int32_t>(256, 2 * ix->topk_cap); }

void slicing(const pk_index *ix, const Work &w, int64_t C, int32_t *slice, int32_t *nslices, int32_t *nt)
{
    int64_t best_load = -1;
    for (int t : {256, 128}) {
        const int64_t slots = (512 / t) * (int64_t)ix->num_sms, cap = (int64_t)kSelPer * t;
        int64_t ns = std::max<int64_t>(1, slots / w.units);
        ns = std::max<int64_t>(ns, ceil_div(C, cap));
        int64_t sl = ceil_div(ceil_div(C, ns), 16) * 16;
        sl = std::max<int64_t>(sl, slice_lo(ix));
        sl = std::min<int64_t>(sl, cap);
        const int64_t nsl = ceil_div(C, sl);
        const int64_t load = ceil_div(nsl * w.units, (int64_t)ix->num_sms) * sl;   // records on the busiest SM
        if (best_load < 0 || load < best_load) {
            best_load = load;
            *slice = (int32_t)sl;
            *nslices = (int32_t)nsl;
            *nt = t;
        }
    }
}

// attention work split: one cluster of up to 8 CTAs per pair, ~2 CTAs per SM
int32_t splitting(const pk_index *ix, int32_t units, int32_t topk)
{
    int64_t ns = ceil_div(2 * (int64_t)ix->num_sms, units);
    ns = std::max<int64_t>(1, std::min<int64_t>(ns, 8));
    ns = std::min<int64_t>(ns, topk);
    return (int32_t)ns;
}

void work_free(Work &w)
{
    cudaFree(w.qt);
    cudaFree(w.qnorm);
    cudaFree(w.bonus_packed);
    cudaFree(w.S);
    cudaFree(w.chunk_cum);
    cudaFree(w.head_hist);
    cudaFree(w.tickets);
    cudaFree(w.chunk_info);
    cudaFree(w.sstar);
    cudaFree(w.cand);
    cudaFree(w.partial);
    cudaFree(w.bonus_bytes);
    w = Work{};
}

template <typename T>
cudaError_t dalloc(T **p, size_t count);

// Workspace for `units` query units (kvg per index pair) of an index of
// capacity n_cap; the counters start at zero.  On failure nothing stays
// allocated.
cudaError_t work_alloc(pk_index *ix, Work &w, int32_t units, int32_t kvg, int64_t n_cap, cudaStream_t s)
{
    w.units = units;
    w.scan_units = units / kvg;
    w.max_chunks = (int32_t)std::max<int64_t>(std::max<int64_t>(1, (4 * (int64_t)ix->num_sms) / w.scan_units),
                                              ceil_div(n_cap, kMaxChunk) + 1);
    {   // largest slice count any C <= n_cap can need
        const int64_t lo = slice_lo(ix);
        const int64_t by_target = std::max<int64_t>(1, (4 * (int64_t)ix->num_sms) / units);
        w.max_slices = (int32_t)std::max<int64_t>(std::min<int64_t>(ceil_div(n_cap, lo), by_target),
                                                  ceil_div(n_cap, kSelPer * 128)) + 1;
    }
    const size_t U = units, NC = ix->stride, MC = w.max_chunks, MS = w.max_slices;
    cudaError_t e = cudaSuccess;
    auto chk = [&](cudaError_t x) { if (e == cudaSuccess) e = x; };
    chk(dalloc(&w.qt, U * kD));
    chk(dalloc(&w.qnorm, U));
    chk(dalloc(&w.bonus_packed, U * kB * 32));
    chk(dalloc(&w.S, U * NC));
    chk(dalloc(&w.chunk_cum, U * MC * kCum));
    chk(dalloc(&w.head_hist, U * kBins));
    chk(dalloc(&w.tickets, U * 2));
    chk(dalloc(&w.chunk_info, U * MC));
    chk(dalloc(&w.sstar, U));
    chk(dalloc(&w.cand, U * NC));
    chk(dalloc(&w.partial, U * MS * (size_t)ix->topk_cap));
    if (kvg > 1) {   // the per-pair packed bonus tables of per-head search, unused bytes zero
        const size_t bytes = (size_t)(U / kvg) * kB * kNC * 4 * ((kvg + 3) / 4);
        chk(dalloc(&w.bonus_bytes, bytes));
        chk(cudaMemsetAsync(w.bonus_bytes, 0, bytes, s));
    }
    chk(cudaMemsetAsync(w.head_hist, 0, U * kBins * sizeof(uint32_t), s));
    chk(cudaMemsetAsync(w.tickets, 0, U * 2 * sizeof(uint32_t), s));
    if (e != cudaSuccess) {
        cudaGetLastError();
        work_free(w);
    }
    return e;
}

void free_all(pk_index *ix)
{
    if (!ix) return;
    cudaFree(ix->codes);
    cudaFree(ix->rec);
    cudaFree(ix->occ);
    if (ix->kv_host) cudaFreeHost(ix->KV);
    else cudaFree(ix->KV);
    work_free(ix->w);
    work_free(ix->wh);

    cudaFree(ix->dev_err);
    cudaFree(ix->dev_err_detail);
    cudaFree(ix->occ_stage);
    if (ix->stage_ev) cudaEventDestroy(ix->stage_ev);
    for (cudaEvent_t e : ix->ev_pool) cudaEventDestroy(e);
}

template <class T>
cudaError_t dalloc(T **p, size_t count)
{
    return cudaMalloc((void **)p, count * sizeof(T) + 16);
}

// ---- tracing
void trace_begin(pk_index *ix, int kind, cudaStream_t s)
{
    if (!ix->trace) return;
    if (ix->ev_used + 2 > ix->ev_pool.size()) {
        for (int i = 0; i < 256; i++) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return;
            ix->ev_pool.push_back(e);
        }
    }
    TraceRec r{kind, ix->ev_pool[ix->ev_used], ix->ev_pool[ix->ev_used + 1]};
    ix->ev_used += 2;
    cudaEventRecord(r.a, s);
    ix->tr.push_back(r);
}

void trace_end(pk_index *ix, cudaStream_t s)
{
    if (!ix->trace || ix->tr.empty()) return;
    cudaEventRecord(ix->tr.back().b, s);
}

pk_status check_params(const pk_params *p)
{
    if (!p) return PK_ERR_INVALID_ARG;
    if (p->head_dim != kD || p->sub_dim != kM) return PK_ERR_UNSUPPORTED;
    if (p->batch < 1 || p->n_kv_heads < 1 || p->group < 1 || p->group > kMaxGroup)
        return PK_ERR_INVALID_ARG;
    if (p->topk < 1) return PK_ERR_INVALID_ARG;
    if (p->topk > kMaxTopk) return PK_ERR_UNSUPPORTED;
    // one grid row per query unit (pair x query head for per-head search)
    if ((int64_t)p->batch * p->n_kv_heads * p->group > 65535) return PK_ERR_UNSUPPORTED;
    if (p->kv_dtype != PK_F32 && p->kv_dtype != PK_BF16) return PK_ERR_INVALID_ARG;
    if (p->kv_location != PK_KV_DEVICE && p->kv_location != PK_KV_HOST_PINNED)
        return PK_ERR_INVALID_ARG;
    if (p->cand_budget < 0 || !(p->collision_ratio >= 0.0f) || p->collision_ratio > 1.0f ||
        !(p->attn_scale >= 0.0f))
        return PK_ERR_INVALID_ARG;
    return PK_OK;
}

// Encode rows 0..n_new-1 of every pair of Kin ([BH][k_stride][D]) at
// positions pos0.. and add their occupancy counts to occ.
pk_status encode_range(pk_index *ix, const void *Kin, int64_t k_stride, int64_t n_new, int64_t pos0,
                       uint32_t *occ, cudaStream_t s)
{
    EncodeArgs a{};
    a.K = Kin;
    a.k_stride = k_stride;
    a.n_new = n_new;
    a.pos0 = pos0;
    a.n_cap = ix->stride;
    a.bh = ix->bh;
    a.is_bf16 = ix->p.kv_dtype == PK_BF16;
    a.codes = ix->codes;
    a.rec = ix->rec;
    a.occ = occ;
    a.rot = ix->rot;
    a.lv = ix->lv;
    trace_begin(ix, PK_K_ENCODE, s);
    cudaError_t e = launch_encode(a, s);
    trace_end(ix, s);
    return cuda_status(e);
}

// copy rows 0..n_new-1 of every pair of k_src / v_src ([BH][src_stride][D])
// into the interleaved store at positions pos0.. of each pair: one kernel of
// 16-byte pieces when both sources are 16-byte aligned, else two 3-D copies
pk_status copy_rows(pk_index *ix, const void *k_src, const void *v_src, int64_t src_stride, int64_t n_new,
                    int64_t pos0, cudaStream_t s)
{
    if (!aligned(k_src, 16) || !aligned(v_src, 16)) {
        const size_t row = (size_t)kD * ix->es;
        cudaError_t e = cudaSuccess;
        for (int kv = 0; kv < 2 && e == cudaSuccess; kv++) {
            cudaMemcpy3DParms p = {};
            p.srcPtr = make_cudaPitchedPtr(const_cast<void *>(kv ? v_src : k_src), row, row, (size_t)src_stride);
            p.dstPtr = make_cudaPitchedPtr((char *)(kv ? ix->V : ix->K) + (size_t)pos0 * 2 * row, 2 * row, row,
                                           (size_t)ix->stride);
            p.extent = make_cudaExtent(row, (size_t)n_new, (size_t)ix->bh);
            p.kind = cudaMemcpyDefault;
            e = cudaMemcpy3DAsync(&p, s);
        }
        return cuda_status(e);
    }
    StoreArgs a{};
    a.srcK = reinterpret_cast<const unsigned char *>(k_src);
    a.srcV = reinterpret_cast<const unsigned char *>(v_src);
    a.dstK = reinterpret_cast<unsigned char *>(ix->K);
    a.dstV = reinterpret_cast<unsigned char *>(ix->V);
    a.src_stride = src_stride;
    a.n_new = n_new;
    a.pos0 = pos0;
    a.pair_rows = ix->stride;
    a.row_bytes = kD * ix->es;
    a.pitch = 2 * (int64_t)kD * ix->es;
    a.bh = ix->bh;
    return cuda_status(launch_store_rows(a, s));
}

// One search over work `w`: kvg query units per index pair (1: the
// aggregated query of each pair; G: every query head of the pair).
pk_status search_impl(pk_index *ix, Work &w, int32_t kvg, const void *q, int32_t topk, int32_t *out_idx,
                      float *out_score, const pk_debug_out *dbg, cudaStream_t s)
{
    if (!ix || !q || !out_idx) return PK_ERR_INVALID_ARG;
    if (topk < 1 || topk > ix->topk_cap) return PK_ERR_INVALID_ARG;
    if (ix->n < topk) return PK_ERR_CAPACITY;
    if (!device_accessible(q) || !device_accessible(out_idx) ||
        (out_score && !device_accessible(out_score)))
        return PK_ERR_INVALID_ARG;
    if (!aligned(q, ix->es) || !aligned(out_idx, 4) || (out_score && !aligned(out_score, 4)))
        return PK_ERR_INVALID_ARG;
    int64_t C, R;
    resolve(ix->n, ix->p.cand_budget, ix->p.collision_ratio, topk, &C, &R);
    int32_t nchunks;
    int64_t chunk;
    chunking(ix, w, ix->n, &nchunks, &chunk);

    PrepArgs pa{};
    pa.q = q;
    pa.H = ix->p.n_kv_heads * kvg;        // per-head units: H*G units of one query head each
    pa.G = ix->p.group / kvg;
    pa.kvg = kvg;
    pa.is_bf16 = ix->p.kv_dtype == PK_BF16;
    pa.bh = w.units;
    // one warp per block unless the 4-warp layout still fits about two CTAs per SM
    pa.wide = (int64_t)w.units * (kB / 2) <= 2 * (int64_t)ix->num_sms;
    pa.R = R;
    pa.occ = ix->occ;
    pa.rot = ix->rot;
    pa.qt = w.qt;
    pa.qnorm = w.qnorm;
    pa.bonus_packed = w.bonus_packed;
    pa.head_hist = w.head_hist;
    pa.tickets = w.tickets;
    if (dbg) {
        pa.dbg_bonus = dbg->bonus;
        pa.dbg_qt = dbg->qt;
        pa.dbg_qnorm = dbg->qnorm;
    }
    if (kvg > 1) {   // the per-head scan reads the pairs' packed bonus tables
        pa.bonus_heads = w.bonus_bytes;
        pa.heads_np = (kvg + 3) / 4;
    }
    trace_begin(ix, PK_K_QUERY_PREP, s);
    cudaError_t e = launch_query_prep(pa, s);
    trace_end(ix, s);
    if (e != cudaSuccess) return cuda_status(e);

    ScanArgs sa{};
    sa.codes = ix->codes;
    sa.bonus_packed = w.bonus_packed;
    sa.kvg = kvg;
    sa.n = ix->n;
    sa.n_cap = ix->stride;
    sa.chunk = chunk;
    sa.C = C;
    sa.nchunks = nchunks;
    sa.S = w.S;
    sa.chunk_cum = w.chunk_cum;
    sa.head_hist = w.head_hist;
    sa.tickets = w.tickets;
    sa.chunk_info = w.chunk_info;
    sa.sstar = w.sstar;
    sa.max_chunks = w.max_chunks;
    if (dbg) {
        sa.dbg_S = dbg->S;
        sa.dbg_hist = dbg->hist;
        sa.dbg_sstar = dbg->sstar;
    }
    trace_begin(ix, PK_K_COLLISION_SCAN, s);
    if (kvg > 1) {   // one pass over each pair's codes for its kvg query heads
        sa.bonus_bytes = w.bonus_bytes;
        e = launch_collision_scan_heads(sa, w.units / kvg, s);
    } else {
        e = launch_collision_scan(sa, w.units, s);
    }
    trace_end(ix, s);
    if (e != cudaSuccess) return cuda_status(e);

    CompactArgs ca{};
    ca.S = w.S;
    ca.chunk_info = w.chunk_info;
    ca.sstar = w.sstar;
    ca.n = ix->n;
    ca.stride = ix->stride;
    ca.chunk = chunk;
    ca.C = C;
    ca.max_chunks = w.max_chunks;
    ca.groups = (int32_t)ceil_div(chunk, 16 * 256);
    ca.cand = w.cand;
    ca.dbg_cand = dbg ? dbg->cand : nullptr;
    ca.dev_err = ix->dev_err;
    trace_begin(ix, PK_K_COMPACT, s);
    e = launch_compact(ca, nchunks, w.units, s);
    trace_end(ix, s);
    if (e != cudaSuccess) return cuda_status(e);

    RerankArgs ra{};
    ra.cand = w.cand;
    ra.kvg = kvg;
    ra.rec = ix->rec;
    ra.qt = w.qt;
    ra.qnorm = w.qnorm;
    ra.stride = ix->stride;
    ra.C = C;
    slicing(ix, w, C, &ra.slice, &ra.nslices, &ra.nt);
    if (ra.nslices > w.max_slices) return PK_ERR_CAPACITY;
    ra.max_slices = w.max_slices;
    ra.topk = topk;
    ra.topk_cap = ix->topk_cap;
    ra.partial = w.partial;
    ra.lv = ix->lv;
    ra.dbg_est = dbg ? dbg->cand_est : nullptr;
    trace_begin(ix, PK_K_RERANK_TOPK, s);
    e = launch_rerank_topk(ra, w.units, s);
    trace_end(ix, s);
    if (e != cudaSuccess) return cuda_status(e);

    MergeArgs ma{};
    ma.partial = w.partial;
    ma.nslices = ra.nslices;
    ma.max_slices = w.max_slices;
    ma.topk = topk;
    ma.topk_cap = ix->topk_cap;
    {
        const int64_t want = (int64_t)ra.nslices * topk;
        // room for every partial key at once (one select) when it fits
        ma.cap = (int32_t)std::max<int64_t>(2 * (int64_t)topk, std::min<int64_t>(want + topk, kMergeCap));
    }
    ma.out_idx = out_idx;
    ma.out_score = out_score;
    ma.dev_err = ix->dev_err;
    trace_begin(ix, PK_K_TOPK_MERGE, s);
    e = launch_topk_merge(ma, w.units, s);
    trace_end(ix, s);
    return cuda_status(e);
}

// Attention for kvg query units per index pair (1: each pair's G query heads
// over the pair's selected rows; G: each query head over its own rows).
// union_heads (kvg = 1): sel_idx holds each query head's own list, and one
// cluster per pair gathers the union of the pair's lists once.
pk_status attend_impl(pk_index *ix, int32_t kvg, const void *q, const int32_t *sel_idx, int32_t topk,
                      const void *dK, const void *dV, int64_t dstride, int32_t dlen, float *out, cudaStream_t s,
                      bool union_heads = false)
{
    if (!ix || !q || !out) return PK_ERR_INVALID_ARG;
    if (topk < 0 || topk > ix->topk_cap || dlen < 0 || topk + (int64_t)dlen < 1) return PK_ERR_INVALID_ARG;
    if (topk > 0 && (!sel_idx || !device_accessible(sel_idx) || !aligned(sel_idx, 4))) return PK_ERR_INVALID_ARG;
    if (!device_accessible(q) || !device_accessible(out)) return PK_ERR_INVALID_ARG;
    if (!aligned(q, ix->es) || !aligned(out, 4)) return PK_ERR_INVALID_ARG;
    if (dlen > 0) {   // dense rows are read 16 bytes at a time
        if (!dK || !dV || dstride < dlen || !device_accessible(dK) || !device_accessible(dV) ||
            !aligned(dK, 16) || !aligned(dV, 16))
            return PK_ERR_INVALID_ARG;
    }
    AttendArgs a{};
    a.dK = dK;
    a.dV = dV;
    a.dstride = dstride;
    a.dlen = dlen;
    a.q = q;
    a.idx = sel_idx;
    a.K = ix->K;
    a.V = ix->V;
    a.kv_pitch = 2 * (int64_t)kD * ix->es;
    a.out = out;
    a.n = ix->n;
    a.stride = ix->stride;
    a.H = ix->p.n_kv_heads * kvg;
    a.G = ix->p.group / kvg;
    a.kvg = kvg;
    a.topk = topk;
    a.is_bf16 = ix->p.kv_dtype == PK_BF16;
    a.scale = ix->scale;
    a.union_heads = union_heads ? 1 : 0;
    const int32_t units = ix->bh * kvg;
    a.nsplit = splitting(ix, units, (union_heads ? a.G * topk : topk) + dlen);
    a.dev_err = ix->dev_err;
    a.dev_err_detail = ix->dev_err_detail;
    trace_begin(ix, PK_K_GATHER_ATTEND, s);
    cudaError_t e = launch_gather_attend(a, units, s);
    trace_end(ix, s);
    return cuda_status(e);
}

}  // namespace

// ======================================================================
extern "C" {

void pk_default_params(pk_params *p)
{
    if (!p) return;
    std::memset(p, 0, sizeof(*p));
    p->batch = 1;
    p->n_kv_heads = 8;
    p->group = 4;
    p->head_dim = kD;
    p->sub_dim = kM;
    p->topk = 100;
    p->n_cap = 0;
    p->cand_budget = 0;
    p->collision_ratio = 0.0f;
    p->attn_scale = 0.0f;
    p->rot_seed = 0;
    p->kv_dtype = PK_BF16;
    p->kv_location = PK_KV_DEVICE;
}

const char *pk_status_str(pk_status s)
{
    switch (s) {
    case PK_OK: return "ok";
    case PK_ERR_INVALID_ARG: return "invalid argument";
    case PK_ERR_CAPACITY: return "capacity exceeded";
    case PK_ERR_OOM: return "out of memory";
    case PK_ERR_CUDA: return "CUDA error";
    case PK_ERR_TIMEOUT: return "device wait timed out";
    case PK_ERR_DEVICE_CHECK: return "device-side check failed";
    case PK_ERR_UNSUPPORTED: return "unsupported configuration";
    }
    return "unknown status";
}

pk_status pk_resolve(int64_t n, int64_t cand_budget, float collision_ratio, int32_t topk,
                     int64_t *C, int64_t *R)
{
    if (n < 1 || !C || !R || topk < 1 || cand_budget < 0 || !(collision_ratio >= 0.0f))
        return PK_ERR_INVALID_ARG;
    resolve(n, cand_budget, collision_ratio, topk, C, R);
    return PK_OK;
}

pk_status pk_magnitude_levels(int32_t m, int32_t L, float *levels, float *thresholds)
{
    if (m < 3 || L < 2 || L > 4096 || !levels || !thresholds) return PK_ERR_INVALID_ARG;
    std::vector<double> lev(L), thr(L - 1);
    if (lloyd_max_levels(m, L, lev.data(), thr.data()) < 0) return PK_ERR_CUDA;
    for (int t = 0; t < L; t++) levels[t] = (float)lev[t];
    for (int t = 0; t < L - 1; t++) thresholds[t] = (float)thr[t];
    return PK_OK;
}

pk_status pk_build_index(const void *K, const void *V, int64_t n, const pk_params *params,
                         void *stream, pk_index **out)
{
    if (!out) return PK_ERR_INVALID_ARG;
    *out = nullptr;
    pk_status st = check_params(params);
    if (st != PK_OK) return st;
    if (!K || !V || n < 1) return PK_ERR_INVALID_ARG;
    const int64_t n_cap = params->n_cap > 0 ? params->n_cap : n;
    if (n > n_cap || n_cap > (int64_t)0x7fffffff - 16) return PK_ERR_CAPACITY;
    if (!device_accessible(K) || !device_accessible(V)) return PK_ERR_INVALID_ARG;
    const int es = params->kv_dtype == PK_BF16 ? 2 : 4;
    if (!aligned(K, es) || !aligned(V, es)) return PK_ERR_INVALID_ARG;

    pk_index *ix = new (std::nothrow) pk_index();
    if (!ix) return PK_ERR_OOM;
    ix->p = *params;
    ix->p.n_cap = n_cap;
    ix->stride = ceil_div(n_cap, 16) * 16;    // keeps every per-pair row 16-byte aligned
    ix->bh = params->batch * params->n_kv_heads;
    ix->es = es;
    ix->topk_cap = params->topk;
    ix->scale = params->attn_scale > 0.0f ? params->attn_scale : (float)(1.0 / std::sqrt((double)kD));
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaGetDevice(&ix->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&ix->num_sms, cudaDevAttrMultiProcessorCount, ix->device);
    if (e != cudaSuccess) {
        delete ix;
        return cuda_status(e);
    }

    // SRHT sign diagonal and scale; Lloyd-Max levels
    for (int r = 0; r < 4; r++) ix->rot.sign_mask[r] = 0;
    for (int j = 0; j < kD; j++)
        if (splitmix64(params->rot_seed * (uint64_t)kD + (uint64_t)j) >> 63)
            ix->rot.sign_mask[j / 32] |= 1u << (j % 32);
    ix->rot.c = (float)(1.0 / std::sqrt((double)kD));
    {
        double lev[kL], thr[kL - 1];
        if (lloyd_max_levels(kM, kL, lev, thr) < 0) {
            delete ix;
            return PK_ERR_CUDA;
        }
        for (int t = 0; t < kL; t++) ix->lv.lev[t] = (float)lev[t];
        for (int t = 0; t < kL - 1; t++) ix->lv.thr[t] = (float)thr[t];
    }

    const size_t BH = ix->bh, NC = ix->stride;
    e = cudaSuccess;
    auto chk = [&](cudaError_t x) { if (e == cudaSuccess) e = x; };
    chk(dalloc(&ix->codes, BH * NC * kB));
    chk(dalloc(&ix->rec, BH * NC * kRecBytes));
    chk(dalloc(&ix->occ, BH * kB * kNC));
    chk(work_alloc(ix, ix->w, ix->bh, 1, n_cap, s));

    chk(dalloc(&ix->dev_err, 1));
    chk(dalloc(&ix->dev_err_detail, 1));
    const size_t kv_bytes = 2 * BH * NC * kD * (size_t)es;
    if (params->kv_location == PK_KV_HOST_PINNED) {
        ix->kv_host = true;
        chk(cudaHostAlloc(&ix->KV, kv_bytes, cudaHostAllocMapped | cudaHostAllocPortable));
    } else {
        chk(cudaMalloc(&ix->KV, kv_bytes));
    }
    if (ix->KV) {
        ix->K = ix->KV;
        ix->V = (char *)ix->KV + (size_t)kD * es;
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        free_all(ix);
        delete ix;
        return PK_ERR_OOM;
    }
    chk(cudaMemsetAsync(ix->occ, 0, BH * kB * kNC * sizeof(uint32_t), s));
    chk(cudaMemsetAsync(ix->dev_err, 0, sizeof(int32_t), s));
    chk(cudaMemsetAsync(ix->dev_err_detail, 0, sizeof(long long), s));
    if (e == cudaSuccess) st = copy_rows(ix, K, V, n, n, 0, s);
    if (e == cudaSuccess && st == PK_OK) st = encode_range(ix, K, n, n, 0, ix->occ, s);
    if (e != cudaSuccess || st != PK_OK) {
        cudaStreamSynchronize(s);
        free_all(ix);
        delete ix;
        return e != cudaSuccess ? cuda_status(e) : st;
    }
    ix->n = n;
    *out = ix;
    return PK_OK;
}

pk_status pk_append(pk_index *ix, const void *k_new, const void *v_new, int64_t n_new, void *stream)
{
    if (!ix || !k_new || !v_new || n_new < 1) return PK_ERR_INVALID_ARG;
    if (ix->n_staged) return PK_ERR_INVALID_ARG;       // publish staged keys first
    if (ix->n + n_new > ix->p.n_cap) return PK_ERR_CAPACITY;
    if (!device_accessible(k_new) || !device_accessible(v_new)) return PK_ERR_INVALID_ARG;
    if (!aligned(k_new, ix->es) || !aligned(v_new, ix->es)) return PK_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    pk_status st = copy_rows(ix, k_new, v_new, n_new, n_new, ix->n, s);
    if (st == PK_OK) st = encode_range(ix, k_new, n_new, n_new, ix->n, ix->occ, s);
    if (st == PK_OK) ix->n += n_new;
    return st;
}

pk_status pk_append_stage(pk_index *ix, const void *k_new, const void *v_new, int64_t n_new, int64_t src_stride,
                          void *stream)
{
    if (!ix || !k_new || !v_new || n_new < 1) return PK_ERR_INVALID_ARG;
    if (src_stride == 0) src_stride = n_new;
    if (src_stride < n_new) return PK_ERR_INVALID_ARG;
    if (ix->n + ix->n_staged + n_new > ix->p.n_cap) return PK_ERR_CAPACITY;
    if (!device_accessible(k_new) || !device_accessible(v_new)) return PK_ERR_INVALID_ARG;
    if (!aligned(k_new, ix->es) || !aligned(v_new, ix->es)) return PK_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t occ_words = (size_t)ix->bh * kB * kNC;
    if (!ix->occ_stage) {
        cudaError_t e = dalloc(&ix->occ_stage, occ_words);
        if (e == cudaSuccess) e = cudaMemsetAsync(ix->occ_stage, 0, occ_words * sizeof(uint32_t), s);
        if (e == cudaSuccess && !ix->stage_ev) e = cudaEventCreateWithFlags(&ix->stage_ev, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            cudaGetLastError();
            cudaFree(ix->occ_stage);
            ix->occ_stage = nullptr;
            return cuda_status(e);
        }
    }
    const int64_t pos0 = ix->n + ix->n_staged;
    pk_status st = copy_rows(ix, k_new, v_new, src_stride, n_new, pos0, s);
    if (st == PK_OK) st = encode_range(ix, k_new, src_stride, n_new, pos0, ix->occ_stage, s);
    if (st == PK_OK) st = cuda_status(cudaEventRecord(ix->stage_ev, s));
    if (st == PK_OK) ix->n_staged += n_new;
    return st;
}

pk_status pk_append_publish(pk_index *ix, void *stream)
{
    if (!ix) return PK_ERR_INVALID_ARG;
    if (!ix->n_staged) return PK_OK;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaStreamWaitEvent(s, ix->stage_ev, 0);
    if (e == cudaSuccess) e = launch_occ_merge(ix->occ, ix->occ_stage, (int64_t)ix->bh * kB * kNC, s);
    if (e != cudaSuccess) return cuda_status(e);
    ix->n += ix->n_staged;
    ix->n_staged = 0;
    return PK_OK;
}

pk_status pk_search(pk_index *ix, const void *q, int32_t topk, int32_t *out_idx, float *out_score,
                    void *stream)
{
    if (!ix) return PK_ERR_INVALID_ARG;
    return search_impl(ix, ix->w, 1, q, topk, out_idx, out_score, nullptr, (cudaStream_t)stream);
}

pk_status pk_search_debug(pk_index *ix, const void *q, int32_t topk, int32_t *out_idx,
                          float *out_score, const pk_debug_out *dbg, void *stream)
{
    if (!ix) return PK_ERR_INVALID_ARG;
    return search_impl(ix, ix->w, 1, q, topk, out_idx, out_score, dbg, (cudaStream_t)stream);
}

pk_status pk_attend(pk_index *ix, const void *q, const int32_t *sel_idx, int32_t topk, float *out,
                    void *stream)
{
    if (topk < 1) return PK_ERR_INVALID_ARG;
    return attend_impl(ix, 1, q, sel_idx, topk, nullptr, nullptr, 0, 0, out, (cudaStream_t)stream);
}

pk_status pk_attend_dense(pk_index *ix, const void *q, const int32_t *sel_idx, int32_t topk,
                          const void *dense_K, const void *dense_V, int64_t dense_stride,
                          int32_t dense_len, float *out, void *stream)
{
    return attend_impl(ix, 1, q, sel_idx, topk, dense_K, dense_V, dense_stride, dense_len, out,
                       (cudaStream_t)stream);
}

pk_status pk_search_heads(pk_index *ix, const void *q, int32_t topk, int32_t *out_idx, float *out_score,
                          void *stream)
{
    if (!ix) return PK_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (ix->wh.units == 0) {      // the per-head workspace, made on first use
        const cudaError_t e = work_alloc(ix, ix->wh, ix->bh * ix->p.group, ix->p.group, ix->p.n_cap, s);
        if (e != cudaSuccess) return e == cudaErrorMemoryAllocation ? PK_ERR_OOM : PK_ERR_CUDA;
    }
    return search_impl(ix, ix->wh, ix->p.group, q, topk, out_idx, out_score, nullptr, s);
}

pk_status pk_attend_heads(pk_index *ix, const void *q, const int32_t *sel_idx, int32_t topk, float *out,
                          void *stream)
{
    if (!ix) return PK_ERR_INVALID_ARG;
    if (topk < 1) return PK_ERR_INVALID_ARG;
    // K/V in host memory: every row of a pair crosses the host link once (the
    // union of its heads' lists) when the lists fit the kernel's table.  K/V in
    // HBM, or longer lists: one cluster per query head (more CTAs in flight).
    if (ix->p.kv_location == PK_KV_HOST_PINNED && (int64_t)ix->p.group * topk <= kUnionMax)
        return attend_impl(ix, 1, q, sel_idx, topk, nullptr, nullptr, 0, 0, out, (cudaStream_t)stream, true);
    return attend_impl(ix, ix->p.group, q, sel_idx, topk, nullptr, nullptr, 0, 0, out, (cudaStream_t)stream);
}

void pk_free(pk_index *ix)
{
    if (!ix) return;
    cudaDeviceSynchronize();
    free_all(ix);
    delete ix;
}

pk_status pk_last_device_error(pk_index *ix, int64_t *detail)
{
    if (!ix) return PK_ERR_INVALID_ARG;
    int32_t code = 0;
    long long det = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(&code, ix->dev_err, sizeof(code), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(&det, ix->dev_err_detail, sizeof(det), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(ix->dev_err, 0, sizeof(int32_t));
    if (e == cudaSuccess) e = cudaMemset(ix->dev_err_detail, 0, sizeof(long long));
    if (e != cudaSuccess) return cuda_status(e);
    if (detail) *detail = det;
    return code == 0 ? PK_OK : PK_ERR_DEVICE_CHECK;
}

pk_status pk_get_info(const pk_index *ix, pk_info *info)
{
    if (!ix || !info) return PK_ERR_INVALID_ARG;
    std::memset(info, 0, sizeof(*info));
    info->n = ix->n;
    info->n_staged = ix->n_staged;
    info->n_cap = ix->p.n_cap;
    info->bh = ix->bh;
    chunking(ix, ix->w, ix->n, &info->nchunks, &info->chunk);
    resolve(ix->n, ix->p.cand_budget, ix->p.collision_ratio, ix->p.topk, &info->cand, &info->coll);
    info->index_bytes = (int64_t)ix->bh * ix->stride * (kB + kRecBytes) + (int64_t)ix->bh * kB * kNC * 4;
    info->kv_bytes = 2 * (int64_t)ix->bh * ix->stride * kD * ix->es;   // K and V rows
    info->kv_location = ix->p.kv_location;
    info->num_sms = ix->num_sms;
    return PK_OK;
}

pk_status pk_export_index(const pk_index *ix, uint8_t *codes, uint8_t *records, uint32_t *occ,
                          void *stream)
{
    if (!ix) return PK_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    if (codes)
        e = cudaMemcpy2DAsync(codes, (size_t)ix->n * kB, ix->codes, (size_t)ix->stride * kB,
                              (size_t)ix->n * kB, ix->bh, cudaMemcpyDefault, s);
    if (e == cudaSuccess && records)
        e = cudaMemcpy2DAsync(records, (size_t)ix->n * kRecBytes, ix->rec, (size_t)ix->stride * kRecBytes,
                              (size_t)ix->n * kRecBytes, ix->bh, cudaMemcpyDefault, s);
    if (e == cudaSuccess && occ)
        e = cudaMemcpyAsync(occ, ix->occ, (size_t)ix->bh * kB * kNC * sizeof(uint32_t), cudaMemcpyDefault, s);
    return cuda_status(e);
}

pk_status pk_trace_enable(pk_index *ix, int32_t on)
{
    if (!ix) return PK_ERR_INVALID_ARG;
    ix->trace = on != 0;
    return PK_OK;
}

pk_status pk_trace_read(pk_index *ix, int64_t *launches, double *total_ms)
{
    if (!ix || !launches || !total_ms) return PK_ERR_INVALID_ARG;
    for (int k = 0; k < PK_K_COUNT; k++) {
        launches[k] = 0;
        total_ms[k] = 0.0;
    }
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e);
    for (const TraceRec &r : ix->tr) {
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
            launches[r.kind] += 1;
            total_ms[r.kind] += ms;
        } else {
            cudaGetLastError();
        }
    }
    ix->tr.clear();
    ix->ev_used = 0;
    return PK_OK;
}

}  // extern "C"
