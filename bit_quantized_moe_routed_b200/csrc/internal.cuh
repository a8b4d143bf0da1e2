// internal.cuh -- shared declarations of the moeq CUDA library (not part of
// the public ABI; see include/moeq.h for that).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moeq.h"

namespace moeq {

// Device status-word flags (atomicOr'ed by kernels, read by moeq_layer_status).
enum : uint32_t { FLAG_ROUTE_RANGE = 1u, FLAG_TIMEOUT = 2u };

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 64;
constexpr int kBook13Rows = 8192;
constexpr int kBook8Rows = 256;
// decode fast path: most CTAs a decode kernel launches, routes it handles,
// tokens it handles
constexpr int kDecMaxGrid = 1024;
constexpr int kDecMaxRoutes = 64;
constexpr int kDecMaxTokens = 8;

// Device copies of the compressed weights.  Layout is the logical one of
// moeq_weights (row-major [E][N][...] per projection).
struct DevWeights {
    uint8_t *codes[3] = {nullptr, nullptr, nullptr};
    uint8_t *scales[3] = {nullptr, nullptr, nullptr};
    uint8_t *idx13[3] = {nullptr, nullptr, nullptr};
    uint8_t *idx8[3] = {nullptr, nullptr, nullptr};
    uint16_t *gain[3] = {nullptr, nullptr, nullptr};
    uint16_t *book13 = nullptr;
    uint16_t *book8 = nullptr;
    // GVQ1: 12-bit code streams, bit-12 planes, E4M3 books and their scales
    uint8_t *code12[3] = {nullptr, nullptr, nullptr};
    uint8_t *hi1[3] = {nullptr, nullptr, nullptr};
    uint8_t *gbook13 = nullptr;
    uint8_t *gbook8 = nullptr;
    float gscale[2] = {0.f, 0.f};
    bool has_gain = false;
};

// Routing tables produced by the route/bucket kernel for one forward.
struct Buckets {
    int32_t *offsets = nullptr;  // [E+1] exclusive scan of per-expert route counts
    int32_t *perm = nullptr;     // [T*k] route ids r = t*k+s, sorted by (expert, r)
    int32_t *active = nullptr;   // [E+1] active[0] = #experts with routes, then their ids ascending
};

// Everything one projection kernel needs to find and decode a matrix.
struct ProjView {
    const uint8_t *codes;   // MXFP4 nibbles          [E][N][K/2]
    const uint8_t *scales;  // MXFP4 E8M0 bytes       [E][N][K/32]
    const uint8_t *idx13;   // VQ 13-bit stream       [E][N][K*13/64]
    const uint8_t *idx8;    // VQ residual indices    [E][N][K/8] or null
    const uint16_t *gain;   // f16 row gains          [E][N] or null
    const uint16_t *book13; // bf16 [8192][8]
    const uint16_t *book8;  // bf16 [256][8] or null
    const uint8_t *code12;  // GVQ1 12-bit stream     [E][N][K*3/16]
    const uint8_t *hi1;     // GVQ1 bit-12 plane      [E][N][K/64]
    const uint8_t *gbook13; // E4M3 [8192][8]
    const uint8_t *gbook8;  // E4M3 [256][8] or null
    float gs13, gs8;        // their scales
    int32_t N, K;
};

inline bool is_gvq1(int fmt) { return fmt == MOEQ_FMT_GVQ1 || fmt == MOEQ_FMT_GVQ1_R8; }
inline bool is_vq13(int fmt) { return fmt == MOEQ_FMT_VQ13 || fmt == MOEQ_FMT_VQ13_R8; }
inline bool has_r8(int fmt) { return fmt == MOEQ_FMT_VQ13_R8 || fmt == MOEQ_FMT_GVQ1_R8; }

// Prefill path for MXFP4 (prefill_mx.cu): a second copy of the weights in the
// logical layout for tensor copies, scale atoms, activation workspaces and the
// tensor maps over them.
struct PrefillMx {
    CUtensorMap map_w[3];          // codes [E*N][K] as 4-bit elements
    CUtensorMap map_x[2];          // activation terms [route position][H]
    CUtensorMap map_h[2];          // intermediate terms [route position][I]
    uint8_t *codes[3] = {nullptr, nullptr, nullptr};      // [E*N][K/2], logical layout
    uint8_t *sf_atoms[3] = {nullptr, nullptr, nullptr};   // [E][N/128][K/128][512]
    int32_t *tile_base = nullptr;  // [E+1]
    uint8_t *xq[2] = {nullptr, nullptr};
    uint8_t *sfx = nullptr;
    uint8_t *hq[2] = {nullptr, nullptr};
    uint8_t *sfh = nullptr;
    bool maps_ready = false;
};

// Tensor-core path for VQ layers with bf16 activations (prefill_vq.cu):
// activations gathered by route, bf16 intermediates, tensor maps over them.
struct PrefillVq {
    CUtensorMap map_x;             // gathered activations [route position][H] bf16
    CUtensorMap map_h;             // intermediates [route position][I] bf16
    int32_t *tile_base = nullptr;  // [E+1]
    uint16_t *xg = nullptr;
    uint16_t *hg = nullptr;
    // GVQ1 layers: the books as the kernels read them, bf16 of the f32
    // products e4m3(entry) x book scale, filled at upload
    uint16_t *gbook13 = nullptr;   // [8192][8]
    uint16_t *gbook8 = nullptr;    // [256][8]
    bool ready = false;
    bool books_ready = false;
};

// Router of a layer (router.cu): the router matrix in the kernels' layout,
// the partial logits of the K slices and the token tiles' arrival counters.
struct RouterState {
    uint4 *wfrag = nullptr;    // bf16 activations: three bf16 terms of Wr in tensor-core fragment order
    float *wt = nullptr;       // f32 activations: Wr transposed, [H][E]
    float *wrow = nullptr;     // Wr as given, [E][H] f32 (the decode-size GEMV)
    float *part = nullptr;     // [K slices][T][E] partial logits
    int *counters = nullptr;   // [token tiles], zero between calls
    int score = 0;             // moeq_score
    bool ready = false;
};

struct Layer {
    moeq_layer_desc d{};
    RouterState *router = nullptr;
    PrefillMx *pf = nullptr;
    PrefillVq *pv = nullptr;
    DevWeights w;
    Buckets b;
    float *h = nullptr;        // [max_tokens*k][I] SwiGLU intermediates, route-sorted order
    float *acc = nullptr;      // [max_tokens][H] f32 combine accumulator
    // decode fast path scratch
    float *dec_ybuf = nullptr;     // [kDecMaxRoutes][kDecMaxTokens][H] per-expert partial outputs
    int *dec_counters = nullptr;   // [2] grid barrier of the one-launch MXFP4 decode (arrivals, generation)
    float *vq_acc = nullptr;       // VQ decode: [kDecMaxTokens][H] f32 combine accumulator, zero between calls
    int *vq_done = nullptr;        // VQ decode: CTA arrival counter of the down kernel, zero between calls
    uint32_t *status = nullptr;
    // staging for moeq_forward_host
    void *x_stage = nullptr;
    void *out_stage = nullptr;
    int32_t *ids_stage = nullptr;
    float *w_stage = nullptr;
    bool uploaded = false;
    int sm_count = 0;
    // limit, in SM clocks, of the kernels' waits on one another (mbarriers,
    // issue counters); on expiry a kernel raises FLAG_TIMEOUT and unwinds.
    // About a second at the default; a test may shorten it at create
    // (MOEQ_TEST_WAIT_CYCLES) to make a wait run out on purpose.
    long long wait_cycles = 2000000000LL;
    // kernels launched (or captured into a graph) by this layer so far
    mutable long long launches = 0;
    void count_launches(int n) const { launches += n; }

    ProjView view(int p) const {
        ProjView v{};
        v.codes = w.codes[p];
        v.scales = w.scales[p];
        v.idx13 = w.idx13[p];
        v.idx8 = has_r8(d.fmt) ? w.idx8[p] : nullptr;
        v.gain = w.has_gain ? w.gain[p] : nullptr;
        v.book13 = w.book13;
        v.book8 = (d.fmt == MOEQ_FMT_VQ13_R8) ? w.book8 : nullptr;
        v.code12 = w.code12[p];
        v.hi1 = w.hi1[p];
        v.gbook13 = w.gbook13;
        v.gbook8 = (d.fmt == MOEQ_FMT_GVQ1_R8) ? w.gbook8 : nullptr;
        v.gs13 = w.gscale[0];
        v.gs8 = w.gscale[1];
        v.N = (p == MOEQ_DOWN) ? d.hidden : d.inter;
        v.K = (p == MOEQ_DOWN) ? d.inter : d.hidden;
        return v;
    }
    int elem_bytes() const { return d.act == MOEQ_ACT_F32 ? 4 : 2; }
};

// Every device allocation of the library goes through here (cudaMalloc, plus
// the MOEQ_TEST_FAIL_ALLOC fault injection of the tests).
cudaError_t dev_alloc(void **p, size_t bytes);

// ---- launchers (each returns cudaGetLastError() of its launch) ----
cudaError_t launch_route_bucket(const Layer &L, const int32_t *topk_ids, int32_t n_routes,
                                int32_t *offsets, int32_t *perm, int32_t *active, cudaStream_t s);
cudaError_t launch_dequant(const Layer &L, int expert, int proj, float *out, cudaStream_t s);
// ev: null, or the 5 phase events of moeq_forward_profiled (ev[0] and ev[1]
// are recorded by the caller around routing).
bool decode_mx_supported(const Layer &L, int T);
cudaError_t launch_decode_mx(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T,
                             void *out, cudaStream_t s, const cudaEvent_t *ev);
bool prefill_mx_supported(const Layer &L, int T);
cudaError_t prefill_mx_create(Layer &L);
void prefill_mx_free(Layer &L);
// experts [e0, e0+ne) of projection p from logical planes already on the device
cudaError_t prefill_mx_upload(Layer &L, int p, const uint8_t *codes, const uint8_t *scales, int e0, int ne,
                              cudaStream_t s);
cudaError_t prefill_mx_finish_upload(Layer &L);
cudaError_t launch_prefill_mx(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                              cudaStream_t s, const cudaEvent_t *ev);
// tile_base[e] = sum over e' < e of ceil(n_e' / 64) (the route tiles of the tensor-core paths)
cudaError_t launch_route_tiles(const int32_t *offsets, int E, int32_t *tile_base, cudaStream_t s);
bool decode_vq_supported(const Layer &L, int T);
cudaError_t launch_decode_vq(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                             cudaStream_t s, const cudaEvent_t *ev);
bool prefill_vq_supported(const Layer &L, int T);
cudaError_t prefill_vq_create(Layer &L);
void prefill_vq_free(Layer &L);
cudaError_t prefill_vq_upload_gvq1_books(Layer &L, const uint8_t *book13, const uint8_t *book8, const float scale[2]);
cudaError_t launch_prefill_vq(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                              cudaStream_t s, const cudaEvent_t *ev);
cudaError_t router_upload(Layer &L, const float *wr, int score, cudaStream_t s);
void router_free(Layer &L);
cudaError_t launch_router(const Layer &L, const void *x, int T, int32_t *topk_ids, float *topk_w, float *logits,
                          cudaStream_t s);
cudaError_t launch_ffn_simt(const Layer &L, const void *x, const float *topk_w, int32_t n_tokens,
                            void *out, cudaStream_t s, const cudaEvent_t *ev);

// Record a phase event of moeq_forward_profiled.  External, so that under
// stream capture it becomes an event-record node of the graph (a plain
// record is only a dependency marker there) and can be timed on replay.
inline void record_phase(cudaEvent_t e, cudaStream_t s) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &st);
    if (st == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
    else cudaEventRecord(e, s);
}

// ---- small device helpers shared by the kernels ----
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ float f16_bits_to_f32(uint16_t b) {
    return __half2float(__ushort_as_half(b));
}

// E2M1 code (4 bits) -> f32.  Exponent field e (bias 1) and mantissa m:
// e > 0 gives 2^(e-1) (1 + m/2), whose f32 pattern is ((126+e)<<23)|(m<<22)
// = (code&7)<<22 + (126<<23); e == 0 gives 0 or 0.5.
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
    uint32_t mag = c & 7u;
    uint32_t bits = (mag >= 2u) ? ((mag << 22) + (126u << 23)) : (mag ? 0x3F000000u : 0u);
    return __uint_as_float(bits | ((c & 8u) << 28));
}

// E8M0 byte -> f32 2^(b-127): b<<23 for b >= 1, the subnormal 2^-127 for
// b == 0, NaN for 255 (rejected at upload).
__device__ __forceinline__ float e8m0_to_f32(uint32_t b) {
    return __uint_as_float(b == 0u ? 0x00400000u : (b == 255u ? 0x7FC00000u : (b << 23)));
}

// Device layout of one MXFP4 projection (codes and scales in one plane).
// Per expert, the N x K matrix is cut into tiles of 16 rows and chunks of
// KC = min(K, 1024) columns; the (tile, chunk) blocks follow each other
// tile by tile, chunk by chunk.  A block is 16 * (KC/2 + KC/32) bytes (8704
// for KC = 1024) and holds
//   [16 rows][KC/2 code bytes]            then
//   [KC/128 groups][16 rows][4 scale bytes]
// Inside a code row, each 64-byte group carries four 32-weight blocks with
// its 4x4 matrix of 32-bit words transposed (word t of block j at byte
// 16t + 4j), and in odd rows the 64-byte groups are swapped in pairs
// (group g stored at g ^ 1; only when a chunk row has an even number of
// groups).  With this layout a tensor-core fragment slice
// (bytes 4t..4t+3 of four consecutive blocks) is one 16-byte word, a whole
// block is one contiguous bulk copy, and the staged rows and scale words
// are read from shared memory without bank conflicts.
struct MxGeom {
    int N, K, KC, nchunk, block_bytes;
    __host__ __device__ MxGeom(int n, int k)
        : N(n), K(k), KC(k < 1024 ? k : 1024), nchunk(k / (k < 1024 ? k : 1024)),
          block_bytes(16 * ((k < 1024 ? k : 1024) / 2 + (k < 1024 ? k : 1024) / 32)) {}
    __host__ __device__ size_t expert_bytes() const { return (size_t)(N / 16) * nchunk * block_bytes; }
    __host__ __device__ size_t block_off(int tile, int chunk) const {
        return ((size_t)tile * nchunk + chunk) * block_bytes;
    }
    // byte offset, inside an expert, of code word t of 32-weight block blk of row n
    __host__ __device__ size_t code_word_off(int n, int blk, int t) const {
        const int kb = blk * 16;                     // logical byte of the block in the row
        const int chunk = kb / (KC / 2), within = kb % (KC / 2);
        const int r = n % 16, grp = (within / 64) ^ ((KC / 128) % 2 == 0 ? (r & 1) : 0), j = (within % 64) / 16;
        return block_off(n / 16, chunk) + (size_t)r * (KC / 2) + grp * 64 + 16 * t + 4 * j;
    }
    // byte offset, inside an expert, of the E8M0 scale of block blk of row n
    __host__ __device__ size_t scale_off(int n, int blk) const {
        const int chunk = blk / (KC / 32), within = blk % (KC / 32);
        return block_off(n / 16, chunk) + 16 * (KC / 2) + (size_t)(within / 4) * 64 + (n % 16) * 4 + (within % 4);
    }
};

// The 16 logical code bytes of 32-weight block blk of row n (word t =
// logical bytes 4t..4t+3), and its scale byte.  e = the expert's base.
__device__ __forceinline__ uint4 mx_block(const uint8_t *e, const MxGeom &g, int n, int blk) {
    return make_uint4(*reinterpret_cast<const uint32_t *>(e + g.code_word_off(n, blk, 0)),
                      *reinterpret_cast<const uint32_t *>(e + g.code_word_off(n, blk, 1)),
                      *reinterpret_cast<const uint32_t *>(e + g.code_word_off(n, blk, 2)),
                      *reinterpret_cast<const uint32_t *>(e + g.code_word_off(n, blk, 3)));
}
__device__ __forceinline__ uint32_t mx_scale(const uint8_t *e, const MxGeom &g, int n, int blk) {
    return e[g.scale_off(n, blk)];
}
// Rewrite experts [e0, e0+ne) of a projection from the logical planes (codes
// [ne][N][K/2], scales [ne][N][K/32], device memory) into the device layout.
cudaError_t launch_mx_pack(const uint8_t *codes, const uint8_t *scales, uint8_t *dst, const MxGeom &g, int ne,
                           cudaStream_t s);

// 13-bit index j of a row's little-endian index stream.  Reads the third
// byte only when the field reaches it, so the last index of the last row
// never reads past the array.
__device__ __forceinline__ uint32_t idx13_at(const uint8_t *row, int j) {
    uint32_t bit = 13u * (uint32_t)j;
    const uint8_t *p = row + (bit >> 3);
    uint32_t sh = bit & 7u;
    uint32_t win = (uint32_t)p[0] | ((uint32_t)p[1] << 8);
    if (sh > 3u) win |= (uint32_t)p[2] << 16;
    return (win >> sh) & 0x1FFFu;
}

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + expf(-g)); }

// E4M3 byte -> f32, exact (sign, 4 exponent bits with bias 7, 3 mantissa
// bits; exponent 0 is subnormal; 0x7F / 0xFF are NaN, rejected at upload):
// a normal value's f32 pattern is (e + 120) << 23 | m << 20.
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u, s = (b & 0x80u) << 24;
    const float mag = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;   // m * 2^-9
    return __uint_as_float(__float_as_uint(mag) | s);
}

// GVQ1 index j of a row: low 12 bits from the 12-bit stream, bit 12 from
// the plane.  Reads the second byte of a code only when the field reaches it.
__device__ __forceinline__ uint32_t gvq1_idx_at(const uint8_t *code_row, const uint8_t *hi_row, int j) {
    const uint32_t bit = 12u * (uint32_t)j;
    const uint8_t *p = code_row + (bit >> 3);
    const uint32_t lo = (((uint32_t)p[0] | ((uint32_t)p[1] << 8)) >> (bit & 7u)) & 0xFFFu;
    return lo | ((uint32_t)((hi_row[j >> 3] >> (j & 7)) & 1u) << 12);
}

}  // namespace moeq
