// pk_noalloc.cu -- candidate selection that allocates nothing.
//
// Some callers cannot allocate device memory when they need a candidate set:
// code running inside a CUDA graph capture (cudaMalloc is not capturable), a
// serving runtime whose memory pool is fully reserved up front, or a host
// thread that must not take the allocator's locks on the decode path.  For
// them, pk_select_candidates_noalloc turns a row of collision scores into its
// Top-C candidate ids (the same set, in the same ascending order, as the
// candidate step inside pk_search) using only a fixed scratch area that this
// file declares as a static device array.
//
// The scratch array exists once per GPU that loads the library and lives
// until the process exits.  Every call shares it, and it keeps whatever the
// last call left there: the fields that must start at zero are cleared at the
// start of each call.  Two calls whose work overlaps on the GPU (different
// streams, or several host threads) race on it and give wrong results; calls
// on one stream are ordered and safe.
#include <mutex>

#include "pk_internal.cuh"

namespace pk {

constexpr int kNaThreads = 256;
constexpr int kNaBins = 256;                 // any byte value has a bin
constexpr int kNaMaxChunks = 256;
constexpr int64_t kNaChunk = 16384;          // keys per chunk
constexpr int64_t kNaMaxKeys = kNaMaxChunks * kNaChunk;   // 4,194,304 keys per call

struct NaScratch {
    uint32_t hist[kNaBins];                  // counts of the whole row (cleared per call)
    uint32_t ticket;                         // CTAs done with the histogram (cleared per call)
    int32_t sstar;                           // threshold s*
    uint32_t pad[62];
    uint32_t cum[kNaMaxChunks][kNaBins + 1]; // per chunk: #{S >= s}, s = 0..256
    uint2 info[kNaMaxChunks];                // per chunk: (first candidate slot, ties kept)
};

// The scratch area: 256-byte aligned, 266,496 bytes per GPU.
static_assert(sizeof(NaScratch) == 266496, "scratch size is part of the documented contract");
static __device__ __align__(256) NaScratch g_na_scratch;

// Per chunk: histogram of S, its suffix counts, and (last CTA to finish, by
// ticket -- no spin-wait) the threshold s* = max{s : #{S >= s} >= C} and each
// chunk's first output slot and tie quota, lower ids first.
__global__ void __launch_bounds__(kNaThreads) k_na_threshold(const uint8_t *S, int64_t n, int64_t C,
                                                             int32_t nchunks, NaScratch *sc)
{
    __shared__ uint32_t s_hist[kNaBins];
    __shared__ uint32_t s_ws[kNaThreads / 32 + 1];
    __shared__ int s_last;
    const int tid = threadIdx.x, chunk = blockIdx.x;
    for (int i = tid; i < kNaBins; i += kNaThreads) s_hist[i] = 0u;
    __syncthreads();
    const int64_t lo = (int64_t)chunk * kNaChunk;
    const int64_t hi = min(lo + kNaChunk, n);
    for (int64_t i = lo + tid; i < hi; i += kNaThreads) atomicAdd(&s_hist[S[i]], 1u);
    __syncthreads();
    // suffix counts: thread tid handles bin s = 255 - tid
    {
        const int s = kNaBins - 1 - tid;
        const uint32_t v = s_hist[s];
        uint32_t tot;
        const uint32_t ex = block_excl_scan<kNaThreads>(v, s_ws, &tot);
        sc->cum[chunk][s] = ex + v;
        if (tid == 0) sc->cum[chunk][kNaBins] = 0u;
        if (v) atomicAdd(&sc->hist[s], v);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&sc->ticket, 1u) == (unsigned)(nchunks - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    __shared__ uint32_t s_cum[kNaBins + 1];  // #{S >= s} over the whole row
    int sstar;
    {
        const int s = kNaBins - 1 - tid;
        const uint32_t v = __ldcg(&sc->hist[s]);
        uint32_t tot;
        const uint32_t ex = block_excl_scan<kNaThreads>(v, s_ws, &tot);
        s_cum[s] = ex + v;
        if (tid == 0) s_cum[kNaBins] = 0u;
        const int pred = ((int64_t)(ex + v) >= C);
        const int nsat = __syncthreads_count(pred);
        sstar = nsat - 1;                    // #{S >= 0} = n >= C, so nsat >= 1
        if (tid == 0) sc->sstar = sstar;
    }
    // ties to take = C - #{S > s*}
    const int64_t ties = C - (int64_t)s_cum[sstar + 1];
    uint32_t carry_eq = 0, carry_slot = 0;
    for (int j0 = 0; j0 < nchunks; j0 += kNaThreads) {
        const int j = j0 + tid;
        uint32_t gt = 0, eq = 0;
        if (j < nchunks) {
            const uint32_t c0 = __ldcg(&sc->cum[j][sstar]), c1 = __ldcg(&sc->cum[j][sstar + 1]);
            gt = c1;
            eq = c0 - c1;
        }
        uint32_t tot_eq;
        const uint32_t ex_eq = carry_eq + block_excl_scan<kNaThreads>(eq, s_ws, &tot_eq);
        const int64_t room = ties - (int64_t)ex_eq;
        const uint32_t quota = room <= 0 ? 0u : (room >= (int64_t)eq ? eq : (uint32_t)room);
        uint32_t tot_slot;
        const uint32_t ex_slot = carry_slot + block_excl_scan<kNaThreads>(gt + quota, s_ws, &tot_slot);
        if (j < nchunks) sc->info[j] = make_uint2(ex_slot, quota);
        carry_eq += tot_eq;
        carry_slot += tot_slot;
    }
}

// Per chunk: write the chunk's candidates (S > s*, then its quota of S = s*
// keys, lower ids first) at its first slot, in ascending id order.  Each
// thread owns 64 consecutive keys; one block-wide scan orders the threads.
__global__ void __launch_bounds__(kNaThreads) k_na_compact(const uint8_t *S, int64_t n, int64_t C,
                                                           const NaScratch *sc, int32_t *cand)
{
    __shared__ uint32_t s_ws[kNaThreads / 32 + 1];
    const int tid = threadIdx.x, chunk = blockIdx.x;
    const int64_t lo = (int64_t)chunk * kNaChunk;
    const int64_t hi = min(lo + kNaChunk, n);
    const uint2 info = sc->info[chunk];
    const uint32_t quota = info.y;
    const int sstar = sc->sstar;
    constexpr int kPer = kNaChunk / kNaThreads;   // 64 keys per thread
    const int64_t t0 = lo + (int64_t)kPer * tid;
    uint32_t ngt = 0, neq = 0;
    for (int u = 0; u < kPer; u++) {
        const int64_t i = t0 + u;
        if (i < hi) {
            const int s = S[i];
            ngt += s > sstar;
            neq += s == sstar;
        }
    }
    uint32_t tot;
    const uint32_t ex = block_excl_scan<kNaThreads>((ngt << 16) | neq, s_ws, &tot);
    uint32_t gtb = ex >> 16, eqb = ex & 0xffffu;
    uint32_t slot = info.x + gtb + min(eqb, quota);
    for (int u = 0; u < kPer; u++) {
        const int64_t i = t0 + u;
        if (i >= hi) break;
        const int s = S[i];
        const bool take = s > sstar || (s == sstar && eqb < quota);
        eqb += s == sstar;
        if (take) {
            if ((int64_t)slot < C) cand[slot] = (int32_t)i;
            slot++;
        }
    }
}

}  // namespace pk

using namespace pk;

namespace {

// Device address of g_na_scratch, looked up once per device with that device
// current (the host-side symbol is only a stand-in, never a device address).
constexpr int kMaxDevices = 64;
std::mutex g_na_mutex;
void *g_na_ptr[kMaxDevices] = {};

pk_status na_scratch(NaScratch **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return PK_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_na_mutex);
    if (!g_na_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_na_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return PK_ERR_CUDA;
        }
        g_na_ptr[dev] = p;
    }
    *out = reinterpret_cast<NaScratch *>(g_na_ptr[dev]);
    return PK_OK;
}

// Device memory of the current device, or page-locked / managed host memory.
bool na_device_accessible(const void *ptr)
{
    cudaPointerAttributes at;
    if (!ptr || cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
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

}  // namespace

extern "C" pk_status pk_select_candidates_noalloc(const uint8_t *S, int64_t n, int64_t C, int32_t *cand,
                                                  void *stream)
{
    if (!S || !cand || n < 1 || C < 1 || C > n) return PK_ERR_INVALID_ARG;
    if (n > kNaMaxKeys) return PK_ERR_CAPACITY;
    if (!na_device_accessible(S) || !na_device_accessible(cand) || ((uintptr_t)cand % 4) != 0)
        return PK_ERR_INVALID_ARG;
    NaScratch *sc = nullptr;
    pk_status st = na_scratch(&sc);
    if (st != PK_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const int32_t nchunks = (int32_t)((n + kNaChunk - 1) / kNaChunk);
    // the histogram and the ticket must start at zero; the rest is overwritten
    cudaError_t e = cudaMemsetAsync(sc, 0, offsetof(NaScratch, sstar), s);
    if (e == cudaSuccess) {
        k_na_threshold<<<nchunks, kNaThreads, 0, s>>>(S, n, C, nchunks, sc);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        k_na_compact<<<nchunks, kNaThreads, 0, s>>>(S, n, C, sc, cand);
        e = cudaGetLastError();
    }
    if (e == cudaErrorMemoryAllocation) return PK_ERR_OOM;
    return e == cudaSuccess ? PK_OK : PK_ERR_CUDA;
}
