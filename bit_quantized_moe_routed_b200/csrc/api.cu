// api.cu -- the extern "C" entry points of libmoeq (declared in moeq.h):
// argument validation, device memory ownership and kernel dispatch.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "internal.cuh"

using namespace moeq;

namespace moeq {

// Host-side fault injection for tests: MOEQ_TEST_FAIL_ALLOC=n makes the
// n-th device allocation of this process (1-based, counted over every
// allocation the library makes) report out-of-memory.
namespace {
std::atomic<long> g_alloc_count{0};
}
cudaError_t dev_alloc(void **p, size_t bytes) {
    static const long fail_at = [] {
        const char *s = std::getenv("MOEQ_TEST_FAIL_ALLOC");
        return s ? std::atol(s) : 0L;
    }();
    const long n = ++g_alloc_count;
    if (fail_at > 0 && n == fail_at) {
        *p = nullptr;
        return cudaErrorMemoryAllocation;
    }
    return cudaMalloc(p, bytes ? bytes : 16);
}

}  // namespace moeq

// The opaque handle of moeq.h is the library's layer object.
struct moeq_layer : moeq::Layer {};

namespace {

// Restores the caller's current device on scope exit.
struct DeviceGuard {
    int prev = -1;
    cudaError_t err = cudaSuccess;
    explicit DeviceGuard(int dev) {
        cudaGetDevice(&prev);
        if (prev != dev) err = cudaSetDevice(dev);
    }
    ~DeviceGuard() {
        int cur = -1;
        cudaGetDevice(&cur);
        if (prev >= 0 && cur != prev) cudaSetDevice(prev);
    }
};

moeq_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MOEQ_OK;
    if (e == cudaErrorMemoryAllocation) return MOEQ_ERR_OUT_OF_MEMORY;
    return MOEQ_ERR_CUDA;
}

size_t row_bytes(int fmt, int plane, int K) {
    // plane 0: codes / idx13; plane 1: scales / idx8
    if (fmt == MOEQ_FMT_MXFP4) return plane == 0 ? (size_t)K / 2 : (size_t)K / 32;
    return plane == 0 ? (size_t)K * 13 / 64 : (size_t)K / 8;
}

void free_layer(moeq_layer *L) {
    if (!L) return;
    for (int p = 0; p < 3; ++p) {
        cudaFree(L->w.codes[p]);
        cudaFree(L->w.scales[p]);
        cudaFree(L->w.idx13[p]);
        cudaFree(L->w.idx8[p]);
        cudaFree(L->w.gain[p]);
        cudaFree(L->w.code12[p]);
        cudaFree(L->w.hi1[p]);
    }
    cudaFree(L->w.gbook13);
    cudaFree(L->w.gbook8);
    cudaFree(L->w.book13);
    cudaFree(L->w.book8);
    cudaFree(L->b.offsets);
    cudaFree(L->b.perm);
    cudaFree(L->b.active);
    cudaFree(L->h);
    cudaFree(L->acc);
    cudaFree(L->dec_ybuf);
    cudaFree(L->dec_counters);
    cudaFree(L->vq_acc);
    cudaFree(L->vq_done);
    cudaFree(L->status);
    cudaFree(L->x_stage);
    cudaFree(L->out_stage);
    cudaFree(L->ids_stage);
    cudaFree(L->w_stage);
    prefill_mx_free(*L);
    prefill_vq_free(*L);
    router_free(*L);
    delete L;
}

bool desc_valid(const moeq_layer_desc *d) {
    if (d->hidden <= 0 || d->inter <= 0 || d->n_experts <= 0 || d->top_k <= 0 || d->max_tokens <= 0)
        return false;
    if (d->n_experts > kMaxExperts || d->top_k > d->n_experts || d->top_k > kMaxTopK) return false;
    if (d->act != MOEQ_ACT_F32 && d->act != MOEQ_ACT_BF16) return false;
    if (d->fmt == MOEQ_FMT_MXFP4) {
        // whole 128-weight groups per row; rows of 1024 or more in whole
        // 1024-weight chunks (the device layout, MxGeom)
        if (d->hidden % 128 || d->inter % 128) return false;
        if ((d->hidden > 1024 && d->hidden % 1024) || (d->inter > 1024 && d->inter % 1024)) return false;
    } else if (is_vq13(d->fmt) || is_gvq1(d->fmt)) {
        if (d->hidden % 64 || d->inter % 64) return false;
    } else {
        return false;
    }
    // sizes that must fit the kernels' 32-bit index arithmetic
    if ((long long)d->max_tokens * d->top_k > (1LL << 30)) return false;
    return true;
}

moeq_status launch_forward(moeq_layer *L, const void *x, const int32_t *ids, const float *w, int32_t T,
                           void *out, cudaStream_t s, const cudaEvent_t *ev = nullptr) {
    if (ev) record_phase(ev[0], s);
    // the decode kernels bulk-copy token rows of x: 16-byte aligned x only
    if (decode_mx_supported(*L, T) && ((uintptr_t)x & 15u) == 0) return from_cuda(launch_decode_mx(*L, x, ids, w, T, out, s, ev));
    // the prefill kernels read x rows as 16-byte vectors
    if (prefill_mx_supported(*L, T) && ((uintptr_t)x & 15u) == 0)
        return from_cuda(launch_prefill_mx(*L, x, ids, w, T, out, s, ev));
    // the VQ decode kernels also store out as 8-byte vectors
    if (decode_vq_supported(*L, T) && ((uintptr_t)x & 15u) == 0 && ((uintptr_t)out & 7u) == 0)
        return from_cuda(launch_decode_vq(*L, x, ids, w, T, out, s, ev));
    if (prefill_vq_supported(*L, T) && ((uintptr_t)x & 15u) == 0)
        return from_cuda(launch_prefill_vq(*L, x, ids, w, T, out, s, ev));
    cudaError_t e = launch_route_bucket(*L, ids, T * L->d.top_k, L->b.offsets, L->b.perm, L->b.active, s);
    if (e != cudaSuccess) return from_cuda(e);
    if (ev) record_phase(ev[1], s);
    e = launch_ffn_simt(*L, x, w, T, out, s, ev);
    return from_cuda(e);
}

}  // namespace

extern "C" {

const char *moeq_status_string(moeq_status s) {
    switch (s) {
        case MOEQ_OK: return "ok";
        case MOEQ_ERR_INVALID_ARGUMENT: return "invalid argument";
        case MOEQ_ERR_UNSUPPORTED: return "unsupported";
        case MOEQ_ERR_OUT_OF_MEMORY: return "out of device memory";
        case MOEQ_ERR_CUDA: return "CUDA error";
        case MOEQ_ERR_NOT_UPLOADED: return "weights not uploaded";
        case MOEQ_ERR_ROUTE_OUT_OF_RANGE: return "route id outside [-1, n_experts)";
        case MOEQ_ERR_TIMEOUT: return "a bounded device wait timed out";
    }
    return "unknown status";
}

moeq_status moeq_layer_create(const moeq_layer_desc *desc, moeq_layer_t *out) {
    if (!out) return MOEQ_ERR_INVALID_ARGUMENT;
    *out = nullptr;
    if (!desc || !desc_valid(desc)) return MOEQ_ERR_INVALID_ARGUMENT;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || desc->device < 0 || desc->device >= ndev)
        return MOEQ_ERR_CUDA;
    DeviceGuard g(desc->device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    moeq_layer *L = new (std::nothrow) moeq_layer();
    if (!L) return MOEQ_ERR_OUT_OF_MEMORY;
    L->d = *desc;
    cudaDeviceGetAttribute(&L->sm_count, cudaDevAttrMultiProcessorCount, desc->device);
    if (const char *wc = std::getenv("MOEQ_TEST_WAIT_CYCLES")) {
        const long long v = std::atoll(wc);
        if (v > 0) L->wait_cycles = v;
    }
    const int E = desc->n_experts, H = desc->hidden, I = desc->inter, k = desc->top_k;
    const size_t M = (size_t)desc->max_tokens;
    const int fmt = desc->fmt;
    cudaError_t e = cudaSuccess;
#define ALLOC(ptr, bytes)                                              \
    do {                                                               \
        if (e == cudaSuccess) e = dev_alloc((void **)&(ptr), (bytes)); \
    } while (0)
    for (int p = 0; p < 3; ++p) {
        const int N = (p == MOEQ_DOWN) ? H : I, K = (p == MOEQ_DOWN) ? I : H;
        const size_t rows = (size_t)E * N;
        if (fmt == MOEQ_FMT_MXFP4) {
            // codes and scales share one plane in the device layout (MxGeom)
            ALLOC(L->w.codes[p], (size_t)E * MxGeom(N, K).expert_bytes());
            (void)rows;
        } else if (is_gvq1(fmt)) {
            ALLOC(L->w.code12[p], rows * K * 3 / 16);
            ALLOC(L->w.hi1[p], rows * K / 64);
            if (has_r8(fmt)) ALLOC(L->w.idx8[p], rows * (K / 8));
            ALLOC(L->w.gain[p], rows * sizeof(uint16_t));
        } else {
            // 16 bytes of slack: the tensor-core path reads each row's 13-byte
            // index chunk of a 64-column slab as four aligned 32-bit words
            ALLOC(L->w.idx13[p], rows * row_bytes(fmt, 0, K) + 16);
            if (fmt == MOEQ_FMT_VQ13_R8) ALLOC(L->w.idx8[p], rows * row_bytes(fmt, 1, K));
            ALLOC(L->w.gain[p], rows * sizeof(uint16_t));
        }
    }
    if (is_vq13(fmt)) {
        ALLOC(L->w.book13, sizeof(uint16_t) * kBook13Rows * 8);
        if (fmt == MOEQ_FMT_VQ13_R8) ALLOC(L->w.book8, sizeof(uint16_t) * kBook8Rows * 8);
    }
    if (is_gvq1(fmt)) {
        ALLOC(L->w.gbook13, (size_t)kBook13Rows * 8);
        if (has_r8(fmt)) ALLOC(L->w.gbook8, (size_t)kBook8Rows * 8);
    }
    if (fmt != MOEQ_FMT_MXFP4) {
        ALLOC(L->vq_acc, sizeof(float) * kDecMaxTokens * H);
        ALLOC(L->vq_done, sizeof(int));
    }
    ALLOC(L->b.offsets, sizeof(int32_t) * (E + 1));
    ALLOC(L->b.active, sizeof(int32_t) * (E + 1));
    ALLOC(L->b.perm, sizeof(int32_t) * M * k);
    ALLOC(L->h, sizeof(float) * M * k * I);
    ALLOC(L->acc, sizeof(float) * M * H);
    ALLOC(L->dec_ybuf, sizeof(float) * kDecMaxRoutes * kDecMaxTokens * H);
    ALLOC(L->dec_counters, sizeof(int) * 2);
    ALLOC(L->status, sizeof(uint32_t));
    ALLOC(L->x_stage, (size_t)L->elem_bytes() * M * H);
    ALLOC(L->out_stage, (size_t)L->elem_bytes() * M * H);
    ALLOC(L->ids_stage, sizeof(int32_t) * M * k);
    ALLOC(L->w_stage, sizeof(float) * M * k);
#undef ALLOC
    if (e == cudaSuccess) e = prefill_mx_create(*L);
    if (e == cudaSuccess) e = prefill_vq_create(*L);
    if (e == cudaSuccess) e = cudaMemset(L->status, 0, sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemset(L->dec_counters, 0, sizeof(int) * 2);
    if (e == cudaSuccess && L->vq_acc) e = cudaMemset(L->vq_acc, 0, sizeof(float) * kDecMaxTokens * H);
    if (e == cudaSuccess && L->vq_done) e = cudaMemset(L->vq_done, 0, sizeof(int));
    if (e != cudaSuccess) {
        free_layer(L);
        cudaGetLastError();  // clear a sticky allocation error
        return from_cuda(e);
    }
    *out = L;
    return MOEQ_OK;
}

void moeq_layer_destroy(moeq_layer_t layer) {
    if (!layer) return;
    DeviceGuard g(layer->d.device);
    cudaDeviceSynchronize();
    free_layer(layer);
}

moeq_status moeq_upload_weights(moeq_layer_t L, const moeq_weights *w, void *stream) {
    if (!L || !w) return MOEQ_ERR_INVALID_ARGUMENT;
    const int fmt = L->d.fmt, E = L->d.n_experts, H = L->d.hidden, I = L->d.inter;
    const bool mx = fmt == MOEQ_FMT_MXFP4, vq = is_vq13(fmt), gq = is_gvq1(fmt), r8 = has_r8(fmt);
    // presence / absence of every plane
    int n_gain = 0;
    for (int p = 0; p < 3; ++p) {
        if (mx != (w->codes[p] != nullptr) || mx != (w->scales[p] != nullptr)) return MOEQ_ERR_INVALID_ARGUMENT;
        if (vq != (w->idx13[p] != nullptr)) return MOEQ_ERR_INVALID_ARGUMENT;
        if (gq != (w->code12[p] != nullptr) || gq != (w->hi1[p] != nullptr)) return MOEQ_ERR_INVALID_ARGUMENT;
        if (r8 != (w->idx8[p] != nullptr)) return MOEQ_ERR_INVALID_ARGUMENT;
        if (w->gain[p]) {
            if (mx) return MOEQ_ERR_INVALID_ARGUMENT;
            ++n_gain;
        }
    }
    if (n_gain != 0 && n_gain != 3) return MOEQ_ERR_INVALID_ARGUMENT;
    if (vq != (w->book13 != nullptr) || (vq && r8) != (w->book8 != nullptr)) return MOEQ_ERR_INVALID_ARGUMENT;
    if (gq != (w->gbook13 != nullptr) || (gq && r8) != (w->gbook8 != nullptr)) return MOEQ_ERR_INVALID_ARGUMENT;
    if (gq) {
        // E4M3 NaN entries and non-finite scales are not valid
        for (size_t i = 0; i < (size_t)kBook13Rows * 8; ++i)
            if ((w->gbook13[i] & 0x7F) == 0x7F) return MOEQ_ERR_INVALID_ARGUMENT;
        if (r8)
            for (size_t i = 0; i < (size_t)kBook8Rows * 8; ++i)
                if ((w->gbook8[i] & 0x7F) == 0x7F) return MOEQ_ERR_INVALID_ARGUMENT;
        if (!std::isfinite(w->gscale[0]) || (r8 && !std::isfinite(w->gscale[1]))) return MOEQ_ERR_INVALID_ARGUMENT;
    }
    // E8M0 255 is NaN and not a valid scale
    if (mx) {
        for (int p = 0; p < 3; ++p) {
            const int N = (p == MOEQ_DOWN) ? H : I, K = (p == MOEQ_DOWN) ? I : H;
            size_t n = (size_t)E * N * row_bytes(fmt, 1, K);
            if (std::memchr(w->scales[p], 0xFF, n)) return MOEQ_ERR_INVALID_ARGUMENT;
        }
    }
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    // MXFP4: copy the logical planes a batch of experts at a time into
    // temporary device buffers and pack them into the device layout (MxGeom)
    uint8_t *tmp_c = nullptr, *tmp_s = nullptr;
    int batch = 1;
    if (mx) {
        const size_t per_expert = (size_t)H * I / 2 + (size_t)H * I / 32;   // largest projection
        batch = (int)std::max<size_t>(1, ((size_t)64 << 20) / per_expert);
        batch = std::min(batch, E);
        e = dev_alloc((void **)&tmp_c, (size_t)batch * H * I / 2);
        if (e == cudaSuccess) e = dev_alloc((void **)&tmp_s, (size_t)batch * H * I / 32);
    }
    for (int p = 0; p < 3 && e == cudaSuccess; ++p) {
        const int N = (p == MOEQ_DOWN) ? H : I, K = (p == MOEQ_DOWN) ? I : H;
        const size_t rows = (size_t)E * N;
        if (mx) {
            const MxGeom geo(N, K);
            for (int e0 = 0; e0 < E && e == cudaSuccess; e0 += batch) {
                const int ne = std::min(batch, E - e0);
                e = cudaMemcpyAsync(tmp_c, w->codes[p] + (size_t)e0 * N * (K / 2), (size_t)ne * N * (K / 2),
                                    cudaMemcpyHostToDevice, s);
                if (e == cudaSuccess)
                    e = cudaMemcpyAsync(tmp_s, w->scales[p] + (size_t)e0 * N * (K / 32), (size_t)ne * N * (K / 32),
                                        cudaMemcpyHostToDevice, s);
                if (e == cudaSuccess)
                    e = launch_mx_pack(tmp_c, tmp_s, L->w.codes[p] + (size_t)e0 * geo.expert_bytes(), geo, ne, s);
                if (e == cudaSuccess) e = prefill_mx_upload(*L, p, tmp_c, tmp_s, e0, ne, s);
            }
        } else if (gq) {
            e = cudaMemcpyAsync(L->w.code12[p], w->code12[p], rows * K * 3 / 16, cudaMemcpyHostToDevice, s);
            if (e == cudaSuccess) e = cudaMemcpyAsync(L->w.hi1[p], w->hi1[p], rows * K / 64, cudaMemcpyHostToDevice, s);
            if (e == cudaSuccess && r8)
                e = cudaMemcpyAsync(L->w.idx8[p], w->idx8[p], rows * (K / 8), cudaMemcpyHostToDevice, s);
            if (e == cudaSuccess && n_gain)
                e = cudaMemcpyAsync(L->w.gain[p], w->gain[p], rows * sizeof(uint16_t), cudaMemcpyHostToDevice, s);
        } else {
            e = cudaMemcpyAsync(L->w.idx13[p], w->idx13[p], rows * row_bytes(fmt, 0, K), cudaMemcpyHostToDevice, s);
            if (e == cudaSuccess && r8)
                e = cudaMemcpyAsync(L->w.idx8[p], w->idx8[p], rows * row_bytes(fmt, 1, K), cudaMemcpyHostToDevice, s);
            if (e == cudaSuccess && n_gain)
                e = cudaMemcpyAsync(L->w.gain[p], w->gain[p], rows * sizeof(uint16_t), cudaMemcpyHostToDevice, s);
        }
    }
    if (e == cudaSuccess && vq)
        e = cudaMemcpyAsync(L->w.book13, w->book13, sizeof(uint16_t) * kBook13Rows * 8, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && vq && r8)
        e = cudaMemcpyAsync(L->w.book8, w->book8, sizeof(uint16_t) * kBook8Rows * 8, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && gq)
        e = cudaMemcpyAsync(L->w.gbook13, w->gbook13, (size_t)kBook13Rows * 8, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && gq && r8)
        e = cudaMemcpyAsync(L->w.gbook8, w->gbook8, (size_t)kBook8Rows * 8, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && mx) e = prefill_mx_finish_upload(*L);
    cudaFree(tmp_c);
    cudaFree(tmp_s);
    if (e != cudaSuccess) return from_cuda(e);
    L->w.has_gain = n_gain == 3;
    if (gq) {
        L->w.gscale[0] = w->gscale[0];
        L->w.gscale[1] = r8 ? w->gscale[1] : 0.f;
        // the books of the tensor-core path (layers created for more than 8 tokens)
        e = prefill_vq_upload_gvq1_books(*L, w->gbook13, r8 ? w->gbook8 : nullptr, L->w.gscale);
        if (e != cudaSuccess) return from_cuda(e);
    }
    L->uploaded = true;
    return MOEQ_OK;
}

moeq_status moeq_forward(moeq_layer_t L, const void *x, const int32_t *ids, const float *w, int32_t T,
                         void *out, void *stream) {
    if (!L) return MOEQ_ERR_INVALID_ARGUMENT;
    if (T < 0 || T > L->d.max_tokens) return MOEQ_ERR_INVALID_ARGUMENT;
    if (T == 0) return MOEQ_OK;
    if (!x || !ids || !w || !out) return MOEQ_ERR_INVALID_ARGUMENT;
    if (!L->uploaded) return MOEQ_ERR_NOT_UPLOADED;
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    return launch_forward(L, x, ids, w, T, out, (cudaStream_t)stream);
}

moeq_status moeq_forward_profiled(moeq_layer_t L, const void *x, const int32_t *ids, const float *w,
                                  int32_t T, void *out, void *stream, void *const *events) {
    if (!L || !events) return MOEQ_ERR_INVALID_ARGUMENT;
    for (int i = 0; i < 5; ++i)
        if (!events[i]) return MOEQ_ERR_INVALID_ARGUMENT;
    if (T < 0 || T > L->d.max_tokens) return MOEQ_ERR_INVALID_ARGUMENT;
    if (T == 0) return MOEQ_OK;
    if (!x || !ids || !w || !out) return MOEQ_ERR_INVALID_ARGUMENT;
    if (!L->uploaded) return MOEQ_ERR_NOT_UPLOADED;
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    cudaEvent_t ev[5];
    for (int i = 0; i < 5; ++i) ev[i] = (cudaEvent_t)events[i];
    return launch_forward(L, x, ids, w, T, out, (cudaStream_t)stream, ev);
}

moeq_status moeq_route(moeq_layer_t L, const int32_t *ids, int32_t T, int32_t *offsets_out,
                       int32_t *perm_out, void *stream) {
    if (!L || !ids || !offsets_out || !perm_out || T < 1 || T > L->d.max_tokens)
        return MOEQ_ERR_INVALID_ARGUMENT;
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    return from_cuda(launch_route_bucket(*L, ids, T * L->d.top_k, offsets_out, perm_out, L->b.active,
                                         (cudaStream_t)stream));
}

moeq_status moeq_forward_host(moeq_layer_t L, const void *x, const int32_t *ids, const float *w,
                              int32_t T, void *out, void *stream) {
    if (!L) return MOEQ_ERR_INVALID_ARGUMENT;
    if (T < 0 || T > L->d.max_tokens) return MOEQ_ERR_INVALID_ARGUMENT;
    if (T == 0) return MOEQ_OK;
    if (!x || !ids || !w || !out) return MOEQ_ERR_INVALID_ARGUMENT;
    if (!L->uploaded) return MOEQ_ERR_NOT_UPLOADED;
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t xb = (size_t)L->elem_bytes() * T * L->d.hidden;
    const size_t rb = (size_t)T * L->d.top_k;
    cudaError_t e = cudaMemcpyAsync(L->x_stage, x, xb, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(L->ids_stage, ids, rb * sizeof(int32_t), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(L->w_stage, w, rb * sizeof(float), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return from_cuda(e);
    moeq_status st = launch_forward(L, L->x_stage, L->ids_stage, L->w_stage, T, L->out_stage, s);
    if (st != MOEQ_OK) return st;
    e = cudaMemcpyAsync(out, L->out_stage, xb, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return from_cuda(e);
}

moeq_status moeq_router_upload(moeq_layer_t L, const float *wr, int32_t score, void *stream) {
    if (!L || !wr || (score != MOEQ_SCORE_SIGMOID && score != MOEQ_SCORE_SOFTMAX)) return MOEQ_ERR_INVALID_ARGUMENT;
    const size_t n = (size_t)L->d.n_experts * L->d.hidden;
    for (size_t i = 0; i < n; ++i)   // finite and within bf16's range (the terms of the bf16 path)
        if (!(std::fabs(wr[i]) <= 3.38e38f)) return MOEQ_ERR_INVALID_ARGUMENT;
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    return from_cuda(router_upload(*L, wr, score, (cudaStream_t)stream));
}

moeq_status moeq_router(moeq_layer_t L, const void *x, int32_t T, int32_t *topk_ids, float *topk_w, float *logits,
                        void *stream) {
    if (!L || !x || !topk_ids || !topk_w || T < 1 || T > L->d.max_tokens) return MOEQ_ERR_INVALID_ARGUMENT;
    if (((uintptr_t)x & 3u) != 0) return MOEQ_ERR_INVALID_ARGUMENT;
    if (!L->router || !L->router->ready) return MOEQ_ERR_NOT_UPLOADED;
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    return from_cuda(launch_router(*L, x, T, topk_ids, topk_w, logits, (cudaStream_t)stream));
}

moeq_status moeq_forward_routed(moeq_layer_t L, const void *x, int32_t T, int32_t *topk_ids, float *topk_w,
                                void *out, void *stream) {
    if (!L || T < 0 || T > L->d.max_tokens) return MOEQ_ERR_INVALID_ARGUMENT;
    if (T == 0) return MOEQ_OK;
    if (!x || !topk_ids || !topk_w || !out || ((uintptr_t)x & 3u) != 0) return MOEQ_ERR_INVALID_ARGUMENT;
    if (!L->uploaded) return MOEQ_ERR_NOT_UPLOADED;
    if (!L->router || !L->router->ready) return MOEQ_ERR_NOT_UPLOADED;
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = launch_router(*L, x, T, topk_ids, topk_w, nullptr, s);
    if (e != cudaSuccess) return from_cuda(e);
    return launch_forward(L, x, topk_ids, topk_w, T, out, s);
}

moeq_status moeq_dequant(moeq_layer_t L, int32_t expert, int32_t proj, float *out, void *stream) {
    if (!L || !out || expert < 0 || expert >= L->d.n_experts || proj < 0 || proj > 2)
        return MOEQ_ERR_INVALID_ARGUMENT;
    if (!L->uploaded) return MOEQ_ERR_NOT_UPLOADED;
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    return from_cuda(launch_dequant(*L, expert, proj, out, (cudaStream_t)stream));
}

int64_t moeq_kernel_launches(moeq_layer_t L) { return L ? (int64_t)L->launches : -1; }

moeq_status moeq_layer_status(moeq_layer_t L, int32_t clear) {
    if (!L) return MOEQ_ERR_INVALID_ARGUMENT;
    DeviceGuard g(L->d.device);
    if (g.err != cudaSuccess) return MOEQ_ERR_CUDA;
    uint32_t v = 0;
    cudaError_t e = cudaMemcpy(&v, L->status, sizeof(v), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && clear) e = cudaMemset(L->status, 0, sizeof(uint32_t));
    // a decode step that gave up on a wait may have left its grid barrier
    // part-way: clearing the status resets it
    if (e == cudaSuccess && clear && (v & FLAG_TIMEOUT))
        e = cudaMemset(L->dec_counters, 0, sizeof(int) * 2);
    if (e != cudaSuccess) return from_cuda(e);
    if (v & FLAG_ROUTE_RANGE) return MOEQ_ERR_ROUTE_OUT_OF_RANGE;
    if (v & FLAG_TIMEOUT) return MOEQ_ERR_TIMEOUT;
    return MOEQ_OK;
}

}  // extern "C"
