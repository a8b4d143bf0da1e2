// route.cu -- route/bucket kernel: groups the T*k routes of a forward by
// expert.
//
// The layer sends each token to k experts ("MiMo-V2.6-Flash-RL GGUF for a
// single DGX Spark", "Architecture notes": 8 of 256 routed experts), and the
// expert matmuls want all of an expert's tokens together ("Speed": with a
// 512-token micro-batch the per-expert matmuls are too small to be efficient).
// This kernel produces, for one forward:
//   offsets[E+1]  exclusive scan of the per-expert route counts
//   perm[n_valid] route ids r = t*k + s, ordered by (expert, r) -- stable, so
//                 the order is fully determined by the input
//   active[E+1]   active[0] = number of experts with at least one route,
//                 active[1..] = those experts in ascending order
// Route ids of -1 are "no route"; any other id outside [0, E) is skipped and
// raises FLAG_ROUTE_RANGE in the status word.
//
// One CTA of 1024 threads does it all: a shared-memory histogram, a scan,
// then the routes in tiles of 1024 in index order, each route's rank among
// equal experts found with __match_any_sync inside a warp and per-warp
// counts across warps.
#include <mutex>

#include "internal.cuh"

namespace moeq {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

__global__ void __launch_bounds__(kThreads, 1)
route_bucket_kernel(const int32_t *__restrict__ ids, int32_t n_routes, int32_t E,
                    int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
                    int32_t *__restrict__ active, uint32_t *__restrict__ status) {
    extern __shared__ int32_t smem[];
    int32_t *cnt = smem;                 // [E]
    int32_t *base = smem + E;            // [E]
    int32_t *wcnt = smem + 2 * E;        // [kWarps][E]
    __shared__ int32_t s_total;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int i = tid; i < E * (2 + kWarps); i += kThreads) smem[i] = 0;
    __syncthreads();

    // 1. histogram
    bool bad = false;
    for (int r = tid; r < n_routes; r += kThreads) {
        int32_t e = ids[r];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        else if (e != -1) bad = true;
    }
    if (__syncthreads_or(bad) && tid == 0) atomicOr(status, FLAG_ROUTE_RANGE);

    // 2. exclusive scan of counts and compaction of active experts (warp 0)
    if (warp == 0) {
        int32_t run = 0, nact = 0;
        for (int c0 = 0; c0 < E; c0 += 32) {
            int e = c0 + lane;
            int32_t v = (e < E) ? cnt[e] : 0;
            int32_t incl = v;
            for (int o = 1; o < 32; o <<= 1) {
                int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            uint32_t act = __ballot_sync(0xffffffffu, v > 0);
            if (e < E) {
                offsets[e] = run + incl - v;
                base[e] = run + incl - v;
                if (v > 0) active[1 + nact + __popc(act & ((1u << lane) - 1u))] = e;
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
            nact += __popc(act);
        }
        if (lane == 0) {
            offsets[E] = run;
            active[0] = nact;
            s_total = run;
        }
    }
    __syncthreads();

    // 3. stable scatter, one tile of kThreads routes at a time
    for (int t0 = 0; t0 < n_routes; t0 += kThreads) {
        int r = t0 + tid;
        int32_t e = (r < n_routes) ? ids[r] : -1;
        bool valid = (e >= 0 && e < E);
        int32_t key = valid ? e : -1 - lane;  // invalid lanes match nobody
        uint32_t same = __match_any_sync(0xffffffffu, key);
        int rank = __popc(same & ((1u << lane) - 1u));
        bool leader = rank == 0;
        if (valid && leader) wcnt[warp * E + e] = __popc(same);
        __syncthreads();
        int pos = 0;
        if (valid) {
            pos = base[e] + rank;
            for (int w2 = 0; w2 < warp; ++w2) pos += wcnt[w2 * E + e];
            perm[pos] = r;
        }
        __syncthreads();
        if (valid && leader) {
            atomicAdd(&base[e], __popc(same));
            wcnt[warp * E + e] = 0;
        }
        __syncthreads();
    }
    (void)s_total;
}

constexpr int kMaxDevices = 64;
std::mutex g_route_mu;   // guards the per-device set-up of both entry points
bool g_route_attr[kMaxDevices] = {};

// The kernel's dynamic shared-memory limit on device `dev` (current), set
// once per device under g_route_mu.
cudaError_t route_smem_limit(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_route_mu);
    if (!g_route_attr[dev]) {
        cudaError_t e = cudaFuncSetAttribute(route_bucket_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(sizeof(int32_t) * kMaxExperts * (2 + kWarps)));
        if (e != cudaSuccess) return e;
        g_route_attr[dev] = true;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_route_bucket(const Layer &L, const int32_t *topk_ids, int32_t n_routes,
                                int32_t *offsets, int32_t *perm, int32_t *active, cudaStream_t s) {
    const int E = L.d.n_experts;
    size_t smem = sizeof(int32_t) * (size_t)E * (2 + kWarps);
    const cudaError_t err = route_smem_limit(L.d.device);
    if (err != cudaSuccess) return err;
    L.count_launches(1);
    route_bucket_kernel<<<1, kThreads, smem, s>>>(topk_ids, n_routes, E, offsets, perm, active,
                                                  L.status);
    return cudaGetLastError();
}

// ------------------------------------------------ allocation-free variant
//
// moeq_route_noalloc runs route_bucket_kernel with its scratch (the active
// list and the status word) in the fixed array below instead of a layer's
// workspace, for callers that cannot allocate device memory.
namespace {

constexpr int kNoAllocStatusWord = kMaxExperts + 1;   // after active[0 .. kMaxExperts]
constexpr int kNoAllocWords = kMaxExperts + 2;        // 4104 bytes

// One copy per device that loads the library.  In host code this name is a
// host-side stand-in for the array, not its device address: that comes
// from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) int32_t g_route_scratch[kNoAllocWords];

constexpr int kNoAllocMaxDevices = kMaxDevices;
std::mutex g_noalloc_mu;
int32_t *g_noalloc_scratch[kNoAllocMaxDevices] = {};

// Set-up for the current device `dev` (once): the scratch's device address
// and the kernel's dynamic shared-memory limit.
cudaError_t noalloc_scratch(int dev, int32_t **out) {
    cudaError_t e = route_smem_limit(dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_scratch[dev]) {
        int32_t *p = nullptr;
        e = cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_route_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_scratch[dev] = p;
    }
    *out = g_noalloc_scratch[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace moeq

extern "C" moeq_status moeq_route_noalloc(const int32_t *topk_ids, int32_t n_tokens, int32_t top_k,
                                          int32_t n_experts, int32_t *offsets_out, int32_t *perm_out,
                                          void *stream) {
    using namespace moeq;
    if (!topk_ids || !offsets_out || !perm_out || n_tokens < 1 || top_k < 1 || top_k > kMaxTopK ||
        n_experts < 1 || (long long)n_tokens * top_k > (1LL << 30))
        return MOEQ_ERR_INVALID_ARGUMENT;
    if (n_experts > kMaxExperts) return MOEQ_ERR_UNSUPPORTED;   // the scratch holds kMaxExperts + 1 entries
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return MOEQ_ERR_CUDA;
    int32_t *scratch = nullptr;
    if (noalloc_scratch(dev, &scratch) != cudaSuccess) return MOEQ_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t *status = reinterpret_cast<uint32_t *>(scratch + kNoAllocStatusWord);
    if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return MOEQ_ERR_CUDA;
    const size_t smem = sizeof(int32_t) * (size_t)n_experts * (2 + kWarps);
    route_bucket_kernel<<<1, kThreads, smem, s>>>(topk_ids, n_tokens * top_k, n_experts, offsets_out, perm_out,
                                                  scratch, status);
    return cudaGetLastError() == cudaSuccess ? MOEQ_OK : MOEQ_ERR_CUDA;
}
