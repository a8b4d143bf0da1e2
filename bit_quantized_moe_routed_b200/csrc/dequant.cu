// dequant.cu -- decode one expert projection to f32 [N][K], bit-exact.
//
// MXFP4 ("MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture
// notes"): w = e2m1(nibble) * 2^(scale-127); the product of an E2M1 value
// and a power of two is exact in f32 unless it overflows (then +-inf under
// round-to-nearest), so one f32 multiply gives the defined value.
// VQ ("MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe"): w[8j+i] =
// (B13[idx13_j][i] + R8[idx8_j][i]) * gain, each step one IEEE f32
// operation in that order (__fadd_rn / __fmul_rn, never contracted).
// The library is built without flush-to-zero, so f32 subnormals survive.
#include "internal.cuh"

namespace moeq {
namespace {

// One thread per 32 consecutive weights of a row.
__global__ void dequant_mxfp4_kernel(const uint8_t *__restrict__ codes,
                                     const uint8_t *__restrict__ scales, int N, int K,
                                     float *__restrict__ out) {
    const int units_per_row = K / 32;
    long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= (long long)N * units_per_row) return;
    int n = (int)(u / units_per_row), b = (int)(u % units_per_row);
    const uint8_t *row = codes + (size_t)n * (K / 2);
    float sc = e8m0_to_f32(scales[(size_t)n * units_per_row + b]);
    float *o = out + (size_t)n * K + (size_t)b * 32;
    uint4 raw = mx_block(row, b);
    uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t nib = (words[q] >> (4 * i)) & 0xFu;
            o[q * 8 + i] = __fmul_rn(e2m1_to_f32(nib), sc);
        }
    }
}

__global__ void dequant_vq_kernel(const uint8_t *__restrict__ idx13, const uint8_t *__restrict__ idx8,
                                  const uint16_t *__restrict__ book13,
                                  const uint16_t *__restrict__ book8,
                                  const uint16_t *__restrict__ gain, int N, int K,
                                  float *__restrict__ out) {
    const int groups = K / 8;
    long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= (long long)N * groups) return;
    int n = (int)(u / groups), j = (int)(u % groups);
    const uint8_t *row13 = idx13 + (size_t)n * (K / 8) * 13 / 8;
    uint32_t i13 = idx13_at(row13, j);
    const uint16_t *b = book13 + (size_t)i13 * 8;
    const uint16_t *r = idx8 ? book8 + (size_t)idx8[(size_t)n * groups + j] * 8 : nullptr;
    float g = gain ? f16_bits_to_f32(gain[n]) : 1.0f;
    float *o = out + (size_t)n * K + (size_t)j * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float v = bf16_bits_to_f32(b[i]);
        if (r) v = __fadd_rn(v, bf16_bits_to_f32(r[i]));
        if (gain) v = __fmul_rn(v, g);
        o[i] = v;
    }
}

// In-place 4x4 transpose of the 32-bit words of every 64-byte group (the
// device layout of MXFP4 codes; see mx_word).
__global__ void mx_repack_kernel(uint4 *__restrict__ codes, size_t n_groups) {
    size_t gi = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gi >= n_groups) return;
    uint4 *g = codes + 4 * gi;
    uint4 a = g[0], b = g[1], c = g[2], d = g[3];
    g[0] = make_uint4(a.x, b.x, c.x, d.x);
    g[1] = make_uint4(a.y, b.y, c.y, d.y);
    g[2] = make_uint4(a.z, b.z, c.z, d.z);
    g[3] = make_uint4(a.w, b.w, c.w, d.w);
}

}  // namespace

cudaError_t launch_mx_repack(uint8_t *codes, size_t bytes, cudaStream_t s) {
    size_t n_groups = bytes / 64;
    if (n_groups == 0) return cudaSuccess;
    mx_repack_kernel<<<(unsigned)((n_groups + 255) / 256), 256, 0, s>>>(reinterpret_cast<uint4 *>(codes), n_groups);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const Layer &L, int expert, int proj, float *out, cudaStream_t s) {
    ProjView v = L.view(proj);
    L.count_launches(1);
    const int threads = 256;
    if (L.d.fmt == MOEQ_FMT_MXFP4) {
        long long units = (long long)v.N * (v.K / 32);
        const uint8_t *c = v.codes + (size_t)expert * v.N * (v.K / 2);
        const uint8_t *sc = v.scales + (size_t)expert * v.N * (v.K / 32);
        dequant_mxfp4_kernel<<<(unsigned)((units + threads - 1) / threads), threads, 0, s>>>(
            c, sc, v.N, v.K, out);
    } else {
        long long units = (long long)v.N * (v.K / 8);
        const uint8_t *i13 = v.idx13 + (size_t)expert * v.N * (v.K / 8) * 13 / 8;
        const uint8_t *i8 = v.idx8 ? v.idx8 + (size_t)expert * v.N * (v.K / 8) : nullptr;
        const uint16_t *g = v.gain ? v.gain + (size_t)expert * v.N : nullptr;
        dequant_vq_kernel<<<(unsigned)((units + threads - 1) / threads), threads, 0, s>>>(
            i13, i8, v.book13, v.book8, g, v.N, v.K, out);
    }
    return cudaGetLastError();
}

}  // namespace moeq
