// vq_encode.cu -- VQ encoder: nearest-codeword assignment of a matrix's
// 8-weight vectors to the 13-bit base book, then of the remainder to the
// 8-bit residual book, packed as the format stores them.
//
// Source ("MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe"): each 8-weight
// vector of an expert row is replaced by the index of a codebook entry, the
// row scaled by an f16 gain; a second, 256-entry book encodes the remainder
// the first stage leaves, without changing the first stage's indices; the
// assignment minimises an error weighted per column by importance.  The codebooks, gains and column weights are inputs
// (their training is not part of this path).
//
// Error of a candidate for vector v (columns 8j..8j+7) of a row with gain g
// and column weights omega: sum_i omega_i (v_i - g b_i)^2.  Expanded, the
// terms that depend on the candidate are g^2 sum omega b^2 - 2 g sum
// (omega v) b: a dot product with the weighted vector plus a norm of the
// candidate, the same for every row -- the GEMM shape of a distance kernel.
// Both are f32 here; the base index is chosen first, on the base error
// alone, then the residual index for it.  Ties go to the lowest index
// (candidates are scanned in ascending order with a strict comparison).
//
// Work: one CTA per SM keeps both books in shared memory (132 KB) and walks
// items of 128 rows x 8 vectors (64 columns, i.e. 13 whole bytes of each
// row's stream).  Warp w takes vector 8 b + w of the item, lane l rows
// l, l+32, l+64, l+96, so every lane of a warp reads the same candidate at
// the same time (a broadcast) and computes its norm once for four vectors.
// The item's indices are packed into the 13-bit stream in shared memory
// and written as whole bytes: no device scratch.
#include <algorithm>
#include <mutex>

#include "async.cuh"
#include "internal.cuh"

namespace moeq {
namespace {

constexpr int kEThreads = 256;
constexpr int kERows = 128;
constexpr int kEV = kERows / 32;      // vectors per thread
constexpr int kEB13 = kBook13Rows * 16, kEB8 = kBook8Rows * 16;

struct EncArgs {
    const float *w;          // [N][K] f32
    const uint16_t *gain;    // f16 [N] or null
    const float *colw;       // [K] or null
    const uint16_t *book13, *book8;
    uint8_t *idx13;          // [N][K*13/64]
    uint8_t *idx8;           // [N][K/8] or null
    int N, K;
};

__device__ __forceinline__ void unpack8(const uint4 &q, float b[8]) {
    b[0] = __uint_as_float(q.x << 16); b[1] = __uint_as_float(q.x & 0xFFFF0000u);
    b[2] = __uint_as_float(q.y << 16); b[3] = __uint_as_float(q.y & 0xFFFF0000u);
    b[4] = __uint_as_float(q.z << 16); b[5] = __uint_as_float(q.z & 0xFFFF0000u);
    b[6] = __uint_as_float(q.w << 16); b[7] = __uint_as_float(q.w & 0xFFFF0000u);
}

__global__ void __launch_bounds__(kEThreads, 1) vq_encode_kernel(EncArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t *b13 = smem, *b8 = smem + kEB13;
    __shared__ uint16_t sel13[kERows][8];
    __shared__ uint8_t sel8[kERows][8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // both books, plain 16-byte loads (once per CTA)
    for (int i = threadIdx.x; i < (kEB13 + (a.book8 ? kEB8 : 0)) / 16; i += kEThreads) {
        const uint4 *src = i < kEB13 / 16 ? reinterpret_cast<const uint4 *>(a.book13) + i
                                          : reinterpret_cast<const uint4 *>(a.book8) + (i - kEB13 / 16);
        reinterpret_cast<uint4 *>(smem)[i] = __ldg(src);
    }
    __syncthreads();
    const int gblocks = a.K / 64, rblocks = (a.N + kERows - 1) / kERows;
    const int sb = a.K * 13 / 64;   // stream bytes per row
    for (int it = blockIdx.x; it < rblocks * gblocks; it += gridDim.x) {
        const int r0 = (it / gblocks) * kERows, gb = it % gblocks;
        const int j = gb * 8 + warp;             // this warp's vector (group of 8 columns)
        float om[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) om[i] = a.colw ? __ldg(a.colw + 8 * j + i) : 1.f;
        float u[kEV][8], g[kEV], best[kEV];
        int bi[kEV];
#pragma unroll
        for (int q = 0; q < kEV; ++q) {
            const int n = r0 + lane + 32 * q;
            const bool live = n < a.N;
            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (live) {
                const float4 v0 = __ldg(reinterpret_cast<const float4 *>(a.w + (size_t)n * a.K + 8 * j));
                const float4 v1 = __ldg(reinterpret_cast<const float4 *>(a.w + (size_t)n * a.K + 8 * j + 4));
                v[0] = v0.x; v[1] = v0.y; v[2] = v0.z; v[3] = v0.w;
                v[4] = v1.x; v[5] = v1.y; v[6] = v1.z; v[7] = v1.w;
            }
            g[q] = (live && a.gain) ? f16_bits_to_f32(__ldg(a.gain + n)) : 1.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) u[q][i] = om[i] * v[i];
            best[q] = INFINITY;
            bi[q] = 0;
        }
        // base stage: every candidate, in ascending order
        for (int c = 0; c < kBook13Rows; ++c) {
            float b[8];
            unpack8(lds128(b13 + 16 * c), b);
            float nb = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) nb = fmaf(om[i] * b[i], b[i], nb);
#pragma unroll
            for (int q = 0; q < kEV; ++q) {
                float dot = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) dot = fmaf(u[q][i], b[i], dot);
                const float d = fmaf(g[q] * g[q], nb, -2.f * g[q] * dot);
                if (d < best[q]) {
                    best[q] = d;
                    bi[q] = c;
                }
            }
        }
        // residual stage for the chosen base entry: the target is v - g b
        int br[kEV] = {0};
        if (a.book8) {
#pragma unroll
            for (int q = 0; q < kEV; ++q) {
                float b[8], t[8];
                unpack8(lds128(b13 + 16 * bi[q]), b);
                // u = omega v, so omega t = u - omega g b
#pragma unroll
                for (int i = 0; i < 8; ++i) t[i] = u[q][i] - om[i] * g[q] * b[i];
                float bst = INFINITY;
                for (int r = 0; r < kBook8Rows; ++r) {
                    float e[8];
                    unpack8(lds128(b8 + 16 * r), e);
                    float nr = 0.f, dot = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        nr = fmaf(om[i] * e[i], e[i], nr);
                        dot = fmaf(t[i], e[i], dot);
                    }
                    const float d = fmaf(g[q] * g[q], nr, -2.f * g[q] * dot);
                    if (d < bst) {
                        bst = d;
                        br[q] = r;
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kEV; ++q) {
            sel13[lane + 32 * q][warp] = (uint16_t)bi[q];
            sel8[lane + 32 * q][warp] = (uint8_t)br[q];
        }
        __syncthreads();
        // pack: thread t < 128 writes row r0 + t's 13 stream bytes (and 8 residual bytes)
        if (threadIdx.x < kERows && r0 + (int)threadIdx.x < a.N) {
            const int n = r0 + threadIdx.x;
            uint64_t lo = 0, hi = 0;   // 104 bits
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const uint64_t x = sel13[threadIdx.x][v];
                const int p = 13 * v;
                if (p + 13 <= 64) lo |= x << p;
                else if (p >= 64) hi |= x << (p - 64);
                else {
                    lo |= x << p;
                    hi |= x >> (64 - p);
                }
            }
            uint8_t *dst = a.idx13 + (size_t)n * sb + (size_t)gb * 13;
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = (uint8_t)(lo >> (8 * i));
#pragma unroll
            for (int i = 0; i < 5; ++i) dst[8 + i] = (uint8_t)(hi >> (8 * i));
            if (a.idx8) {
                uint2 pk;
                pk.x = sel8[threadIdx.x][0] | (sel8[threadIdx.x][1] << 8) | (sel8[threadIdx.x][2] << 16) |
                       ((uint32_t)sel8[threadIdx.x][3] << 24);
                pk.y = sel8[threadIdx.x][4] | (sel8[threadIdx.x][5] << 8) | (sel8[threadIdx.x][6] << 16) |
                       ((uint32_t)sel8[threadIdx.x][7] << 24);
                *reinterpret_cast<uint2 *>(a.idx8 + (size_t)n * (a.K / 8) + (size_t)gb * 8) = pk;
            }
        }
        __syncthreads();
    }
}

std::mutex g_enc_mu;
bool g_enc_attr[64] = {};

}  // namespace
}  // namespace moeq

extern "C" moeq_status moeq_vq_encode(const float *w, int32_t n_rows, int32_t n_cols, const uint16_t *gain,
                                      const float *col_weight, const uint16_t *book13, const uint16_t *book8,
                                      uint8_t *idx13_out, uint8_t *idx8_out, void *stream) {
    using namespace moeq;
    if (!w || !book13 || !idx13_out || n_rows < 1 || n_cols < 64 || n_cols % 64) return MOEQ_ERR_INVALID_ARGUMENT;
    if ((book8 == nullptr) != (idx8_out == nullptr)) return MOEQ_ERR_INVALID_ARGUMENT;
    if (((uintptr_t)w & 15u) || ((uintptr_t)book13 & 15u) || ((uintptr_t)book8 & 15u) || ((uintptr_t)idx8_out & 7u))
        return MOEQ_ERR_INVALID_ARGUMENT;
    if ((long long)n_rows * n_cols > (1LL << 40)) return MOEQ_ERR_INVALID_ARGUMENT;
    int dev = -1, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOEQ_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOEQ_ERR_CUDA;
    const size_t smem = kEB13 + kEB8;
    {
        std::lock_guard<std::mutex> lock(g_enc_mu);
        if (!g_enc_attr[dev]) {
            if (cudaFuncSetAttribute(vq_encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
                cudaSuccess)
                return MOEQ_ERR_CUDA;
            g_enc_attr[dev] = true;
        }
    }
    EncArgs a{w, gain, col_weight, book13, book8, idx13_out, idx8_out, n_rows, n_cols};
    const long long items = (long long)((n_rows + kERows - 1) / kERows) * (n_cols / 64);
    const int grid = (int)std::min<long long>(items, sms);
    vq_encode_kernel<<<grid, kEThreads, smem, (cudaStream_t)stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? MOEQ_OK : MOEQ_ERR_CUDA;
}
