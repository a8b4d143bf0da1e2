// ffn_simt.cu -- the general routed-FFN path on CUDA cores (any format, f32
// or bf16 activations, any token count).
//
//   gate/up: h[p][n] = silu(W_gate,e[n] . x[t]) * (W_up,e[n] . x[t])  for the
//            route p (route-sorted position) of token t on expert e
//   down:    acc[t][m] += topk_w[r] * (W_down,e[m] . h[p])            (atomic f32)
//   cast:    out = acc rounded once to the output dtype
// Structure from "MiMo-V2.6-Flash-RL GGUF for a single DGX Spark",
// "Architecture notes" (routed gate/up/down experts) and "Recipe"
// (intermediates kept in f32).  Weights are decoded to their exact f32
// values (the same values moeq_dequant returns) and every product and sum
// is an f32 FMA, so this path is the accurate one used for f32 activations.
// One warp computes one output row; lanes split K in units of 32 weights.
#include "internal.cuh"

namespace moeq {
namespace {

constexpr int kRowsPerCta = 8;          // one row per warp
constexpr int kTok = 4;                 // tokens per pass over a row

enum { FMT_MX = 0, FMT_VQ = 1, FMT_G = 2 };

// Exact f32 values of weights 32u .. 32u+31 of row n of expert e.
template <int FMT>
__device__ __forceinline__ void decode_unit(const ProjView &v, int e, int n, int u, float w[32]) {
    const size_t row = (size_t)e * v.N + n;
    if constexpr (FMT == FMT_MX) {
        const MxGeom mg(v.N, v.K);
        const uint8_t *eb = v.codes + (size_t)e * mg.expert_bytes();
        uint4 raw = mx_block(eb, mg, n, u);
        float sc = e8m0_to_f32(mx_scale(eb, mg, n, u));
        uint32_t q[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int i = 0; i < 8; ++i) w[a * 8 + i] = __fmul_rn(e2m1_to_f32((q[a] >> (4 * i)) & 0xFu), sc);
    } else if constexpr (FMT == FMT_G) {
        const uint8_t *c12 = v.code12 + row * (size_t)v.K * 3 / 16, *h1 = v.hi1 + row * (size_t)v.K / 64;
        float g = v.gain ? f16_bits_to_f32(__ldg(v.gain + row)) : 1.0f;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int j = 4 * u + a;
            const uint32_t c = gvq1_idx_at(c12, h1, j);
            const uint2 b = __ldg(reinterpret_cast<const uint2 *>(v.gbook13) + c);
            uint2 r = make_uint2(0u, 0u);
            if (v.idx8) r = __ldg(reinterpret_cast<const uint2 *>(v.gbook8) + __ldg(v.idx8 + row * (v.K / 8) + j));
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t bb = ((i < 4 ? b.x : b.y) >> (8 * (i & 3))) & 0xFFu;
                float val = __fmul_rn(e4m3_to_f32(bb), v.gs13);
                if (v.idx8) val = __fadd_rn(val, __fmul_rn(e4m3_to_f32(((i < 4 ? r.x : r.y) >> (8 * (i & 3))) & 0xFFu), v.gs8));
                if (v.gain) val = __fmul_rn(val, g);
                w[a * 8 + i] = val;
            }
        }
    } else {
        const uint8_t *row13 = v.idx13 + row * (size_t)(v.K / 8) * 13 / 8;
        float g = v.gain ? f16_bits_to_f32(__ldg(v.gain + row)) : 1.0f;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            int j = 4 * u + a;
            uint32_t i13 = idx13_at(row13, j);
            uint4 b = __ldg(reinterpret_cast<const uint4 *>(v.book13) + i13);
            uint32_t bw[4] = {b.x, b.y, b.z, b.w};
            uint32_t rw[4] = {0, 0, 0, 0};
            if (v.idx8) {
                uint4 r = __ldg(reinterpret_cast<const uint4 *>(v.book8) + __ldg(v.idx8 + row * (v.K / 8) + j));
                rw[0] = r.x; rw[1] = r.y; rw[2] = r.z; rw[3] = r.w;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t bb = (bw[i / 2] >> (16 * (i & 1))) & 0xFFFFu;
                float val = bf16_bits_to_f32(bb);
                if (v.idx8) val = __fadd_rn(val, bf16_bits_to_f32((rw[i / 2] >> (16 * (i & 1))) & 0xFFFFu));
                if (v.gain) val = __fmul_rn(val, g);
                w[a * 8 + i] = val;
            }
        }
    }
}

template <bool BF16>
__device__ __forceinline__ void load_x32(const void *x, size_t off, float xv[32]) {
    if constexpr (BF16) {
        const uint4 *p = reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(x) + off);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            uint4 r = __ldg(p + a);
            uint32_t q[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xv[a * 8 + 2 * i] = __uint_as_float(q[i] << 16);
                xv[a * 8 + 2 * i + 1] = __uint_as_float(q[i] & 0xFFFF0000u);
            }
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + off);
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            float4 r = __ldg(p + a);
            xv[4 * a] = r.x; xv[4 * a + 1] = r.y; xv[4 * a + 2] = r.z; xv[4 * a + 3] = r.w;
        }
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int FMT, bool BF16>
__global__ void __launch_bounds__(32 * kRowsPerCta)
gateup_simt_kernel(ProjView G, ProjView U, const void *__restrict__ x, int k,
                   const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm,
                   const int32_t *__restrict__ active, float *__restrict__ h) {
    if ((int)blockIdx.y >= active[0]) return;
    const int e = active[1 + blockIdx.y];
    const int beg = offsets[e], cnt = offsets[e + 1] - beg;
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
    const int H = G.K, I = G.N;
    if (n >= I) return;
    for (int t0 = 0; t0 < cnt; t0 += kTok) {
        float g[kTok], u[kTok];
        int tok[kTok];
#pragma unroll
        for (int j = 0; j < kTok; ++j) {
            g[j] = 0.f;
            u[j] = 0.f;
            tok[j] = (t0 + j < cnt) ? perm[beg + t0 + j] / k : -1;
        }
        for (int un = lane; un < H / 32; un += 32) {
            float wg[32], wu[32];
            decode_unit<FMT>(G, e, n, un, wg);
            decode_unit<FMT>(U, e, n, un, wu);
#pragma unroll
            for (int j = 0; j < kTok; ++j) {
                if (tok[j] < 0) continue;
                float xv[32];
                load_x32<BF16>(x, (size_t)tok[j] * H + (size_t)un * 32, xv);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    g[j] = fmaf(wg[i], xv[i], g[j]);
                    u[j] = fmaf(wu[i], xv[i], u[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kTok; ++j) {
            float gs = warp_sum(g[j]), us = warp_sum(u[j]);
            if (lane == 0 && tok[j] >= 0) h[(size_t)(beg + t0 + j) * I + n] = silu_f32(gs) * us;
        }
    }
}

template <int FMT>
__global__ void __launch_bounds__(32 * kRowsPerCta)
down_simt_kernel(ProjView D, const float *__restrict__ h, const float *__restrict__ topk_w, int k,
                 const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm,
                 const int32_t *__restrict__ active, float *__restrict__ acc) {
    if ((int)blockIdx.y >= active[0]) return;
    const int e = active[1 + blockIdx.y];
    const int beg = offsets[e], cnt = offsets[e + 1] - beg;
    const int lane = threadIdx.x & 31;
    const int m = blockIdx.x * kRowsPerCta + (threadIdx.x >> 5);
    const int H = D.N, I = D.K;
    if (m >= H) return;
    for (int t0 = 0; t0 < cnt; t0 += kTok) {
        float y[kTok];
#pragma unroll
        for (int j = 0; j < kTok; ++j) y[j] = 0.f;
        for (int un = lane; un < I / 32; un += 32) {
            float wd[32];
            decode_unit<FMT>(D, e, m, un, wd);
#pragma unroll
            for (int j = 0; j < kTok; ++j) {
                if (t0 + j >= cnt) continue;
                const float4 *hp = reinterpret_cast<const float4 *>(h + (size_t)(beg + t0 + j) * I + (size_t)un * 32);
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    float4 hv = hp[a];
                    y[j] = fmaf(wd[4 * a], hv.x, y[j]);
                    y[j] = fmaf(wd[4 * a + 1], hv.y, y[j]);
                    y[j] = fmaf(wd[4 * a + 2], hv.z, y[j]);
                    y[j] = fmaf(wd[4 * a + 3], hv.w, y[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kTok; ++j) {
            float ys = warp_sum(y[j]);
            if (lane == 0 && t0 + j < cnt) {
                int r = perm[beg + t0 + j];
                atomicAdd(acc + (size_t)(r / k) * H + m, topk_w[r] * ys);
            }
        }
    }
}

template <bool BF16>
__global__ void cast_out_kernel(const float *__restrict__ acc, void *__restrict__ out, long long n) {
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    if constexpr (BF16) reinterpret_cast<__nv_bfloat16 *>(out)[i] = __float2bfloat16_rn(acc[i]);
    else reinterpret_cast<float *>(out)[i] = acc[i];
}

template <int FMT, bool BF16>
cudaError_t run(const Layer &L, const void *x, const float *topk_w, int32_t T, void *out,
                cudaStream_t s, const cudaEvent_t *ev) {
    const int H = L.d.hidden, I = L.d.inter, k = L.d.top_k, E = L.d.n_experts;
    const int ny = (T * k < E) ? T * k : E;
    cudaError_t err = cudaMemsetAsync(L.acc, 0, sizeof(float) * (size_t)T * H, s);
    if (err != cudaSuccess) return err;
    dim3 blk(32 * kRowsPerCta);
    L.count_launches(3);
    gateup_simt_kernel<FMT, BF16><<<dim3((I + kRowsPerCta - 1) / kRowsPerCta, ny), blk, 0, s>>>(
        L.view(MOEQ_GATE), L.view(MOEQ_UP), x, k, L.b.offsets, L.b.perm, L.b.active, L.h);
    if (ev) record_phase(ev[2], s);
    down_simt_kernel<FMT><<<dim3((H + kRowsPerCta - 1) / kRowsPerCta, ny), blk, 0, s>>>(
        L.view(MOEQ_DOWN), L.h, topk_w, k, L.b.offsets, L.b.perm, L.b.active, L.acc);
    if (ev) record_phase(ev[3], s);
    long long n = (long long)T * H;
    cast_out_kernel<BF16><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(L.acc, out, n);
    if (ev) record_phase(ev[4], s);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_simt(const Layer &L, const void *x, const float *topk_w, int32_t n_tokens,
                            void *out, cudaStream_t s, const cudaEvent_t *ev) {
    const bool mx = L.d.fmt == MOEQ_FMT_MXFP4;
    const bool bf = L.d.act == MOEQ_ACT_BF16;
    if (mx) return bf ? run<FMT_MX, true>(L, x, topk_w, n_tokens, out, s, ev)
                      : run<FMT_MX, false>(L, x, topk_w, n_tokens, out, s, ev);
    if (is_gvq1(L.d.fmt))
        return bf ? run<FMT_G, true>(L, x, topk_w, n_tokens, out, s, ev)
                  : run<FMT_G, false>(L, x, topk_w, n_tokens, out, s, ev);
    return bf ? run<FMT_VQ, true>(L, x, topk_w, n_tokens, out, s, ev)
              : run<FMT_VQ, false>(L, x, topk_w, n_tokens, out, s, ev);
}

}  // namespace moeq
