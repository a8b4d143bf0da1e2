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

// One thread per 32 consecutive weights of a row; e = the expert's base in
// the device layout.
__global__ void dequant_mxfp4_kernel(const uint8_t *__restrict__ e, MxGeom g, float *__restrict__ out) {
    const int N = g.N, K = g.K, units_per_row = K / 32;
    long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= (long long)N * units_per_row) return;
    int n = (int)(u / units_per_row), b = (int)(u % units_per_row);
    float sc = e8m0_to_f32(mx_scale(e, g, n, b));
    float *o = out + (size_t)n * K + (size_t)b * 32;
    uint4 raw = mx_block(e, g, n, b);
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

// GVQ1 ("MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe": 12-bit code
// stream plus a 1-bit plane): w[8j+i] = (e4m3(B13q[c][i]) * s13 +
// e4m3(B8q[r][i]) * s8) * gain, each step one f32 operation in that order.
__global__ void dequant_gvq1_kernel(const uint8_t *__restrict__ code12, const uint8_t *__restrict__ hi1,
                                    const uint8_t *__restrict__ idx8, const uint8_t *__restrict__ b13q,
                                    const uint8_t *__restrict__ b8q, float s13, float s8,
                                    const uint16_t *__restrict__ gain, int N, int K, float *__restrict__ out) {
    const int groups = K / 8;
    long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= (long long)N * groups) return;
    int n = (int)(u / groups), j = (int)(u % groups);
    const uint32_t c = gvq1_idx_at(code12 + (size_t)n * K * 3 / 16, hi1 + (size_t)n * K / 64, j);
    const uint8_t *b = b13q + (size_t)c * 8;
    const uint8_t *r = idx8 ? b8q + (size_t)idx8[(size_t)n * groups + j] * 8 : nullptr;
    float g = gain ? f16_bits_to_f32(gain[n]) : 1.0f;
    float *o = out + (size_t)n * K + (size_t)j * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float v = __fmul_rn(e4m3_to_f32(b[i]), s13);
        if (r) v = __fadd_rn(v, __fmul_rn(e4m3_to_f32(r[i]), s8));
        if (gain) v = __fmul_rn(v, g);
        o[i] = v;
    }
}

// Logical planes (codes [ne][N][K/2], scales [ne][N][K/32]) -> device
// layout (MxGeom).  One thread per 32-weight block of a row.
__global__ void mx_pack_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                               uint8_t *__restrict__ dst, MxGeom g, int ne) {
    const int bpr = g.K / 32;
    long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= (long long)ne * g.N * bpr) return;
    const int b = (int)(u % bpr);
    const long long rowg = u / bpr;          // expert * N + n
    const int n = (int)(rowg % g.N), e = (int)(rowg / g.N);
    const uint4 raw = *reinterpret_cast<const uint4 *>(codes + rowg * (g.K / 2) + (size_t)b * 16);
    uint8_t *de = dst + (size_t)e * g.expert_bytes();
    *reinterpret_cast<uint32_t *>(de + g.code_word_off(n, b, 0)) = raw.x;
    *reinterpret_cast<uint32_t *>(de + g.code_word_off(n, b, 1)) = raw.y;
    *reinterpret_cast<uint32_t *>(de + g.code_word_off(n, b, 2)) = raw.z;
    *reinterpret_cast<uint32_t *>(de + g.code_word_off(n, b, 3)) = raw.w;
    de[g.scale_off(n, b)] = scales[rowg * bpr + b];
}

}  // namespace

cudaError_t launch_mx_pack(const uint8_t *codes, const uint8_t *scales, uint8_t *dst, const MxGeom &g, int ne,
                           cudaStream_t s) {
    const long long n = (long long)ne * g.N * (g.K / 32);
    if (n == 0) return cudaSuccess;
    mx_pack_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(codes, scales, dst, g, ne);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const Layer &L, int expert, int proj, float *out, cudaStream_t s) {
    ProjView v = L.view(proj);
    L.count_launches(1);
    const int threads = 256;
    if (L.d.fmt == MOEQ_FMT_MXFP4) {
        const MxGeom g(v.N, v.K);
        long long units = (long long)v.N * (v.K / 32);
        dequant_mxfp4_kernel<<<(unsigned)((units + threads - 1) / threads), threads, 0, s>>>(
            v.codes + (size_t)expert * g.expert_bytes(), g, out);
    } else if (is_gvq1(L.d.fmt)) {
        long long units = (long long)v.N * (v.K / 8);
        const uint8_t *c12 = v.code12 + (size_t)expert * v.N * v.K * 3 / 16;
        const uint8_t *h1 = v.hi1 + (size_t)expert * v.N * v.K / 64;
        const uint8_t *i8 = v.idx8 ? v.idx8 + (size_t)expert * v.N * (v.K / 8) : nullptr;
        const uint16_t *g = v.gain ? v.gain + (size_t)expert * v.N : nullptr;
        dequant_gvq1_kernel<<<(unsigned)((units + threads - 1) / threads), threads, 0, s>>>(
            c12, h1, i8, v.gbook13, v.gbook8, v.gs13, v.gs8, g, v.N, v.K, out);
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
