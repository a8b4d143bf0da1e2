// decode_vq.cu -- VQ13 / VQ13+R8 routed-expert FFN at decode sizes (1..8
// tokens, bf16 activations): a grouped GEMV, one warp per output row.
//
// Format ("MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe"): an expert row is
// cut into 8-weight vectors, each stored as a 13-bit index into the layer's
// 8192 x 8 codebook (VQ13+R8: and an 8-bit index into a 256 x 8 residual
// book); the row is scaled by an f16 gain:
//     w[n][8j+i] = (B13[c_nj][i] + R8[r_nj][i]) * gain[n].
// "Why 13 bits plus an 8-bit residual": the kernels keep the layer's whole
// codebook in shared memory while they decode every selected expert -- here
// both books (132 KB of bf16 entries) stay resident for the kernel's life.
//
// Work: a row of a selected expert (gate and up together in the first
// kernel, so that the warp owns both halves of SwiGLU) is one warp item;
// each warp takes a contiguous range of items.  A row's 13-bit stream
// splits evenly over the 32 lanes (K = 4096: 26 bytes, 16 vectors per lane;
// K = 2048: 13 bytes, 8 vectors), so every lane loads its own stretch
// straight from HBM into registers -- no staging -- one item ahead of the
// one it computes.  Per vector a lane extracts the index with a funnel
// shift, gathers the 16-byte codewords from shared memory, adds base and
// residual as bf16 pairs, and accumulates the dot products with the
// staged activations of the expert's tokens in f32 (packed f32x2 FMAs).
// The activation rows are staged with a skew of 16 bytes per lane chunk so
// that the 8 lanes of a quarter warp read 8 different bank groups.
//
// The on-chip gather is what bounds this path on B200: two random 16-byte
// shared-memory reads per 8 weights (one without the residual stage).
//
// The down kernel stages, per (expert, token) column of its experts, the
// sum over the token's routes of w * h in bf16, and adds each row's result
// into an f32 accumulator with one atomic per (row, token); the CTA that
// finishes last casts the accumulator to bf16 and clears it for the next
// call.
#include <algorithm>
#include <cmath>
#include <mutex>
#include <type_traits>

#include "async.cuh"
#include "decode_common.cuh"
#include "internal.cuh"

namespace moeq {
namespace {

using dec::RouteTable;
using dec::build_route_table;

constexpr int kVThreads = 512;
constexpr int kVWarps = kVThreads / 32;
constexpr int kB13Bytes = kBook13Rows * 16;
constexpr int kB8Bytes = kBook8Rows * 16;
constexpr int kVMaxT = 8;
constexpr int kVMaxSmem = 232448 - 4096;   // dynamic; room for the static tables

struct VqdArgs {
    const uint8_t *idx13[3];   // [E][N][K*13/64] little-endian 13-bit streams
    const uint8_t *idx8[3];    // [E][N][K/8] residual indices (R8 only)
    const uint16_t *gain[3];   // f16 [E][N] or null
    const uint16_t *book13;    // bf16 [8192][8]
    const uint16_t *book8;     // bf16 [256][8] (R8 only)
    const uint16_t *x;         // bf16 [T][H]
    const int32_t *ids;        // [T][k]
    const float *topk_w;       // [T][k]
    float *h;                  // [T*k][I] f32 by route id
    float *acc;                // [kVMaxT][H] f32, zero between calls
    uint16_t *out;             // bf16 [T][H]
    int *done;                 // arrival counter of the down kernel's CTAs, zero between calls
    uint32_t *status;
    long long wait_cycles;
    // GVQ1 layers
    const uint8_t *code12[3];  // [E][N][K*3/16] 12-bit code streams
    const uint8_t *hi1[3];     // [E][N][K/64] bit-12 planes
    const uint8_t *gbook13;    // E4M3 [8192][8]
    const uint8_t *gbook8;     // E4M3 [256][8] (R8 only)
    float gs13;                // base book scale
    uint32_t rho2;             // (residual scale / base scale) as an f16 pair
    int T, k, E, H, I;
};

// Per expert slot of the route table: its distinct tokens (the B columns).
struct ColTable {
    int ncol[dec::kMaxR];
    uint8_t tok[dec::kMaxR][kVMaxT];
};

// Warp 0, after build_route_table.
__device__ void build_cols(ColTable &ct, const RouteTable &tb) {
    const int lane = threadIdx.x & 31;
    for (int d = lane; d < tb.D; d += 32) {
        unsigned mask = 0u;
        for (int c = tb.col_beg[d]; c < tb.col_beg[d + 1]; ++c) mask |= 1u << tb.tok[tb.route[c]];
        int n = 0;
        for (int t = 0; t < kVMaxT; ++t)
            if ((mask >> t) & 1u) ct.tok[d][n++] = (uint8_t)t;
        ct.ncol[d] = n;
    }
}

// Skewed staging of a row of K values split into 32 lane chunks of 8 VPL:
// element c at c + 8 (c / (8 VPL)), so chunk l starts at 8 l (VPL + 1).
template <int VPL>
__host__ __device__ inline int skew_stride(int K) { return K + K / VPL; }
template <int VPL>
__device__ __forceinline__ int skew_pos(int c) { return c + 8 * (c / (8 * VPL)); }

// The lane's stretch of one row's 13-bit stream (13 VPL / 8 bytes at byte
// 13 VPL l / 8), loaded as whole words and shifted so that bit 0 of w[0]
// is the lane's first index.
template <int VPL>
struct Idx13 {
    static constexpr int BPL = 13 * VPL / 8;                 // 26 or 13
    static constexpr int NW = (BPL + 3 + 3) / 4;             // 7 or 4
    uint32_t w[NW];
    __device__ __forceinline__ void load(const uint8_t *row, int lane) {
        const int byte = BPL * lane;
        const uint32_t *p = reinterpret_cast<const uint32_t *>(row + (byte & ~3));
#pragma unroll
        for (int q = 0; q < NW; ++q) w[q] = __ldcs(reinterpret_cast<const unsigned int *>(p + q));
        shift_ = (byte & 3) * 8;
    }
    __device__ __forceinline__ void align() {
#pragma unroll
        for (int q = 0; q + 1 < NW; ++q) w[q] = __funnelshift_r(w[q], w[q + 1], shift_);
        w[NW - 1] >>= shift_;
    }
    // index m of the lane (m a compile-time constant once the caller's loop
    // is unrolled, so that w stays in registers)
    __device__ __forceinline__ uint32_t get(int m) const {
        const int p = 13 * m, q = p >> 5, s = p & 31;
        const int q1 = q + 1 < NW ? q + 1 : NW - 1;
        return (s + 13 <= 32 ? (w[q] >> s) : __funnelshift_r(w[q], w[q1], s)) & 0x1FFFu;
    }
    uint32_t shift_;
};

// The lane's residual indices: VPL bytes at VPL l.
template <int VPL>
struct Idx8 {
    uint32_t w[VPL / 4];
    __device__ __forceinline__ void load(const uint8_t *row, int lane) {
        if constexpr (VPL == 16) {
            const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(row) + lane);
            w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
        } else {
            const uint2 v = __ldcs(reinterpret_cast<const uint2 *>(row) + lane);
            w[0] = v.x; w[1] = v.y;
        }
    }
    __device__ __forceinline__ uint32_t get(int m) const { return (w[m >> 2] >> (8 * (m & 3))) & 0xFFu; }
};

// GVQ1: the lane's stretch of one row's 12-bit code stream (12 VPL / 8
// bytes at byte 12 VPL l / 8: whole words) and its VPL bits of the bit-12
// plane.
template <int VPL>
struct Idx12 {
    static constexpr int NW = 12 * VPL / 32;                 // 6 or 3
    uint32_t w[NW];
    uint32_t hi;
    __device__ __forceinline__ void load(const uint8_t *code_row, const uint8_t *hi_row, int lane) {
        const uint32_t *p = reinterpret_cast<const uint32_t *>(code_row) + NW * lane;
#pragma unroll
        for (int q = 0; q < NW; ++q) w[q] = __ldcs(reinterpret_cast<const unsigned int *>(p + q));
        if constexpr (VPL == 16) hi = __ldcs(reinterpret_cast<const unsigned short *>(hi_row) + lane);
        else hi = __ldcs(reinterpret_cast<const unsigned char *>(hi_row) + lane);
    }
    __device__ __forceinline__ void align() {}
    __device__ __forceinline__ uint32_t get(int m) const {
        const int p = 12 * m, q = p >> 5, s = p & 31;
        const int q1 = q + 1 < NW ? q + 1 : NW - 1;
        const uint32_t lo = (s + 12 <= 32 ? (w[q] >> s) : __funnelshift_r(w[q], w[q1], s)) & 0xFFFu;
        return lo | (((hi >> m) & 1u) << 12);
    }
};
template <int VPL, bool G1>
using IdxT = typename std::conditional<G1, Idx12<VPL>, Idx13<VPL>>::type;

// Eight E4M3 bytes -> four f16 pairs, exact (byte i lands in element i).
__device__ __forceinline__ uint4 e4m3x8_to_f16x2(uint2 v) {
    uint4 r;
    asm("{\n\t.reg .b16 a0, a1, a2, a3;\n\t"
        "mov.b32 {a0, a1}, %4;\n\tmov.b32 {a2, a3}, %5;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a0;\n\tcvt.rn.f16x2.e4m3x2 %1, a1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %2, a2;\n\tcvt.rn.f16x2.e4m3x2 %3, a3;\n\t}"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "r"(v.x), "r"(v.y));
    return r;
}
__device__ __forceinline__ uint32_t hfma2_f16(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}
// (acc0, acc1) += (f32(w.lo), f32(w.hi)) * (x.lo, x.hi) for an f16 pair w and
// a bf16 pair x, in f32.
__device__ __forceinline__ void dot2h(float &acc0, float &acc1, uint32_t w, uint32_t x) {
    asm("{\n\t.reg .b16 h0, h1;\n\t.reg .f32 f0, f1;\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b32 {h0, h1}, %2;\n\tcvt.f32.f16 f0, h0;\n\tcvt.f32.f16 f1, h1;\n\t"
        "mov.b64 ra, {f0, f1};\n\tmov.b64 rb, {%3, %4};\n\tmov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(acc0), "+f"(acc1)
        : "r"(w), "r"(x << 16), "r"(x & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t hadd2_bf16(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// (acc0, acc1) += (a.lo, a.hi) * (b.lo, b.hi) for bf16 pairs a, b, in f32.
__device__ __forceinline__ void dot2(float &acc0, float &acc1, uint32_t a, uint32_t b) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(acc0), "+f"(acc1)
        : "r"(a << 16), "r"(a & 0xFFFF0000u), "r"(b << 16), "r"(b & 0xFFFF0000u));
}
// The dot product of a vector's 8 weights (bf16 pairs, or f16 pairs for
// GVQ1) with 8 bf16 activations, into two f32 partial sums.
template <bool G1 = false>
__device__ __forceinline__ void dot8(float acc[2], const uint4 &w, const uint4 &x) {
    if constexpr (G1) {
        dot2h(acc[0], acc[1], w.x, x.x);
        dot2h(acc[0], acc[1], w.y, x.y);
        dot2h(acc[0], acc[1], w.z, x.z);
        dot2h(acc[0], acc[1], w.w, x.w);
    } else {
        dot2(acc[0], acc[1], w.x, x.x);
        dot2(acc[0], acc[1], w.y, x.y);
        dot2(acc[0], acc[1], w.z, x.z);
        dot2(acc[0], acc[1], w.w, x.w);
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// This warp's contiguous share [i0, i1) of n items over the whole grid.
__device__ __forceinline__ void warp_range(int n, int &i0, int &i1) {
    const long long gw = (long long)blockIdx.x * kVWarps + (threadIdx.x >> 5), nw = (long long)gridDim.x * kVWarps;
    i0 = (int)(n * gw / nw);
    i1 = (int)(n * (gw + 1) / nw);
}

// ---------------------------------------------------------------- books

// Shared-memory bytes of the books; with RI the residual book is stored 8
// times, copy q in 16-byte bank group q only (entry r of copy q at
// (8 r + q) * 16), and lane l reads copy l % 8: the 8 lanes of a quarter
// warp then never share a bank group, however random their indices.  GVQ1
// entries are 8 bytes: the base book takes 64 KB, and the interleaved
// residual book 16 copies (8-byte slots, a half warp per phase).
constexpr int kG13Bytes = kBook13Rows * 8, kG8Bytes = kBook8Rows * 8;
template <bool R8, bool RI, bool G1 = false>
constexpr int books_bytes() {
    if constexpr (G1) return kG13Bytes + (R8 ? (RI ? 16 * kG8Bytes : kG8Bytes) : 0);
    else return kB13Bytes + (R8 ? (RI ? 8 * kB8Bytes : kB8Bytes) : 0);
}
// Staged-operand bytes of each kernel for K = 256 VPL.
constexpr int gu_stage_bytes(int TB, int VPL) { return TB * (256 * VPL + 256) * 2; }
constexpr int dn_stage_bytes(int TB, int VPL) { return 2 * TB * (256 * VPL + 256) * 2; }
// The residual book interleaved when it and the staged operands fit.
template <int VPL, bool R8, int TB, bool DOWN, bool G1 = false>
constexpr bool use_ri() {
    return R8 &&
           books_bytes<true, true, G1>() + (DOWN ? dn_stage_bytes(TB, VPL) : gu_stage_bytes(TB, VPL)) <= kVMaxSmem;
}

// Both books into shared memory (warp 0): the base book by bulk copies on
// `bar`; the residual book by the same copy, or, interleaved (RI), by the
// whole CTA with plain loads (call fill_ri after the barrier's init).
template <bool RI, bool G1 = false>
__device__ void load_books(uint8_t *b13, uint8_t *b8, const VqdArgs &a, uint64_t *bar) {
    const int lane = threadIdx.x & 31;
    const uint8_t *src13 = G1 ? a.gbook13 : reinterpret_cast<const uint8_t *>(a.book13);
    const uint8_t *src8 = G1 ? a.gbook8 : reinterpret_cast<const uint8_t *>(a.book8);
    constexpr int n13 = G1 ? kG13Bytes : kB13Bytes, n8 = G1 ? kG8Bytes : kB8Bytes;
    const bool copy8 = src8 && !RI;
    if (lane == 0) mbar_arrive_expect_tx(bar, n13 + (copy8 ? n8 : 0));
    __syncwarp();
    if (lane < 4) bulk_g2s(b13 + lane * (n13 / 4), src13 + lane * (n13 / 4), n13 / 4, bar);
    if (lane == 4 && copy8) bulk_g2s(b8, src8, n8, bar);
    __syncwarp();
}
template <bool G1 = false>
__device__ void fill_ri(uint8_t *b8, const VqdArgs &a) {
    if constexpr (G1) {
        for (int i = threadIdx.x; i < kBook8Rows * 16; i += kVThreads) {
            const int r = i >> 4, q = i & 15;
            reinterpret_cast<uint2 *>(b8)[16 * r + q] = __ldg(reinterpret_cast<const uint2 *>(a.gbook8) + r);
        }
    } else {
        for (int i = threadIdx.x; i < kBook8Rows * 8; i += kVThreads) {
            const int r = i >> 3, q = i & 7;
            reinterpret_cast<uint4 *>(b8)[8 * r + q] = __ldg(reinterpret_cast<const uint4 *>(a.book8) + r);
        }
    }
}

// The 8 weights of a vector: base (+ residual) as bf16 pairs; for GVQ1 as
// f16 pairs of base + rho * residual (both E4M3 values exact in f16; the
// base scale and the gain are applied to the row's sum).
template <bool R8, bool RI, bool G1 = false>
__device__ __forceinline__ uint4 codeword2(const uint8_t *b13, const uint8_t *b8, uint32_t c, uint32_t r, int lane,
                                           uint32_t rho2 = 0u) {
    if constexpr (G1) {
        uint4 v = e4m3x8_to_f16x2(*reinterpret_cast<const uint2 *>(b13 + 8u * c));
        if constexpr (R8) {
            const uint4 q = e4m3x8_to_f16x2(
                *reinterpret_cast<const uint2 *>(b8 + 8u * (RI ? 16u * r + (uint32_t)(lane & 15) : r)));
            v.x = hfma2_f16(q.x, rho2, v.x);
            v.y = hfma2_f16(q.y, rho2, v.y);
            v.z = hfma2_f16(q.z, rho2, v.z);
            v.w = hfma2_f16(q.w, rho2, v.w);
        }
        return v;
    }
    const int q8 = lane & 7;
    uint4 v = lds128(b13 + 16u * c);
    if constexpr (R8) {
        const uint4 q = lds128(b8 + 16u * (RI ? 8u * r + (uint32_t)q8 : r));
        v.x = hadd2_bf16(v.x, q.x);
        v.y = hadd2_bf16(v.y, q.y);
        v.z = hadd2_bf16(v.z, q.z);
        v.w = hadd2_bf16(v.w, q.w);
    }
    return v;
}

// ---------------------------------------------------------------- gate/up

template <int VPL, bool R8, bool G1>
struct GURow {
    IdxT<VPL, G1> g13, u13;
    Idx8<VPL> g8, u8;
};

// Shared state of a CTA that the per-row work reads.
struct VqdShared {
    RouteTable tb;
    ColTable ct;
};

// One gate/up row pair for an expert with NC token columns: the dot
// products over the lane's stretch, the warp sums, SwiGLU, h.
// Columns j0 .. j0 + NC - 1 (at most four per pass: more would not fit the
// registers; a fifth to eighth column takes a second pass over the row).
// The index words must be aligned (Idx13::align) before the first pass.
template <int VPL, bool R8, bool RI, int NC, bool G1>
__device__ __forceinline__ void gu_row(const VqdArgs &a, const VqdShared &s, const uint8_t *b13, const uint8_t *b8,
                                       const uint16_t *xs, int xstride, int chunk, int d, int n, int j0,
                                       const GURow<VPL, R8, G1> &r) {
    const int lane = threadIdx.x & 31, I = a.I;
    float ag[NC][2], au[NC][2];
    const uint16_t *xr[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        ag[j][0] = ag[j][1] = au[j][0] = au[j][1] = 0.f;
        xr[j] = xs + (size_t)s.ct.tok[d][j0 + j] * xstride + chunk;
    }
#pragma unroll
    for (int m = 0; m < VPL; ++m) {
        uint32_t rg = 0, ru = 0;
        if constexpr (R8) {
            rg = r.g8.get(m);
            ru = r.u8.get(m);
        }
        const uint4 wg = codeword2<R8, RI, G1>(b13, b8, r.g13.get(m), rg, lane, a.rho2);
        const uint4 wu = codeword2<R8, RI, G1>(b13, b8, r.u13.get(m), ru, lane, a.rho2);
#pragma unroll
        for (int j = 0; j < NC; ++j) {
            const uint4 xv = lds128(xr[j] + 8 * m);
            dot8<G1>(ag[j], wg, xv);
            dot8<G1>(au[j], wu, xv);
        }
    }
    const size_t row = (size_t)s.tb.expert[d] * I + n;
    const float bs = G1 ? a.gs13 : 1.f;   // the GVQ1 base scale
    const float gg = (a.gain[0] ? f16_bits_to_f32(__ldg(a.gain[0] + row)) : 1.f) * bs;
    const float gu = (a.gain[1] ? f16_bits_to_f32(__ldg(a.gain[1] + row)) : 1.f) * bs;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        const float g = warp_sum(ag[j][0] + ag[j][1]) * gg;
        const float u = warp_sum(au[j][0] + au[j][1]) * gu;
        const float hv = silu_f32(g) * u;
        // every route of (expert d, token of column j0 + j)
        const int tk = s.ct.tok[d][j0 + j];
        for (int c = s.tb.col_beg[d] + lane; c < s.tb.col_beg[d + 1]; c += 32) {
            const int rt = s.tb.route[c];
            if (s.tb.tok[rt] == tk) a.h[(size_t)rt * I + n] = hv;
        }
    }
}

template <int VPL, bool R8, int TB, bool G1>   // VPL = H / 256; TB >= tokens; G1: GVQ1 format
__global__ void __launch_bounds__(kVThreads, 1) vqd_gateup_kernel(VqdArgs a) {
    constexpr bool RI = use_ri<VPL, R8, TB, false, G1>();
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *b13 = smem, *b8 = smem + (G1 ? kG13Bytes : kB13Bytes);
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem + books_bytes<R8, RI, G1>());
    __shared__ VqdShared s;
    __shared__ __align__(8) uint64_t bar;
    const int H = a.H, I = a.I, T = a.T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int xstride = skew_stride<VPL>(H);
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    // the books are weights: fetch them before waiting for the previous kernel
    if (warp == 0) load_books<RI, G1>(b13, b8, a, &bar);
    if constexpr (RI) fill_ri<G1>(b8, a);
    pdl_wait_primary();
    if (warp == 0) {
        build_route_table(s.tb, a.ids, a.topk_w, T * a.k, a.k, a.E, a.status, blockIdx.x == 0);
        __syncwarp();
        build_cols(s.ct, s.tb);
    }
    // activations, bf16, skewed rows
    for (int i = threadIdx.x; i < T * (H / 8); i += kVThreads) {
        const int t = i / (H / 8), c = (i % (H / 8)) * 8;
        *reinterpret_cast<uint4 *>(xs + (size_t)t * xstride + skew_pos<VPL>(c)) =
            __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)t * H + c));
    }
    volatile int abort_flag = 0;
    // block-uniform: the warps' shuffles below need every lane
    const bool books_ok = __syncthreads_and(mbar_poll_abort(&bar, 0, &abort_flag, a.wait_cycles));
    pdl_launch_dependents();
    if (!books_ok) {
        if (threadIdx.x == 0) atomicOr(a.status, FLAG_TIMEOUT);
        return;
    }

    const int RB13 = H * 13 / 64, RB8 = H / 8;
    const int lI = 31 - __clz(I);
    int i0, i1;
    warp_range(s.tb.D * I, i0, i1);
    const int chunk = skew_pos<VPL>(lane * 8 * VPL);   // this lane's columns in a staged row
    auto load = [&](int i, GURow<VPL, R8, G1> &r) {
        const size_t row = (size_t)s.tb.expert[i >> lI] * I + (i & (I - 1));
        if constexpr (G1) {
            r.g13.load(a.code12[0] + row * (H * 3 / 16), a.hi1[0] + row * (H / 64), lane);
            r.u13.load(a.code12[1] + row * (H * 3 / 16), a.hi1[1] + row * (H / 64), lane);
        } else {
            r.g13.load(a.idx13[0] + row * RB13, lane);
            r.u13.load(a.idx13[1] + row * RB13, lane);
        }
        if constexpr (R8) {
            r.g8.load(a.idx8[0] + row * RB8, lane);
            r.u8.load(a.idx8[1] + row * RB8, lane);
        }
    };
    auto compute = [&](int i, GURow<VPL, R8, G1> &r) {
        const int d = i >> lI, n = i & (I - 1);
        r.g13.align();
        r.u13.align();
        // the expert's column count, a compile-time constant inside
        const int nc = s.ct.ncol[d];
        if (nc > 4) {
            if constexpr (TB >= 8) gu_row<VPL, R8, RI, 4, G1>(a, s, b13, b8, xs, xstride, chunk, d, n, 0, r);
        }
        const int j0 = nc > 4 ? 4 : 0;
        switch (nc - j0) {
            case 1: gu_row<VPL, R8, RI, 1, G1>(a, s, b13, b8, xs, xstride, chunk, d, n, j0, r); break;
            case 2: if constexpr (TB >= 2) gu_row<VPL, R8, RI, 2, G1>(a, s, b13, b8, xs, xstride, chunk, d, n, j0, r); break;
            case 3: if constexpr (TB >= 4) gu_row<VPL, R8, RI, 3, G1>(a, s, b13, b8, xs, xstride, chunk, d, n, j0, r); break;
            case 4: if constexpr (TB >= 4) gu_row<VPL, R8, RI, 4, G1>(a, s, b13, b8, xs, xstride, chunk, d, n, j0, r); break;
            default: break;
        }
    };
    GURow<VPL, R8, G1> ra, rb;
    if (i0 < i1) load(i0, ra);
    for (int i = i0; i < i1; i += 2) {
        if (i + 1 < i1) load(i + 1, rb);
        compute(i, ra);
        if (i + 1 >= i1) break;
        if (i + 2 < i1) load(i + 2, ra);
        compute(i + 1, rb);
    }
}

// ---------------------------------------------------------------- down

template <int VPL, bool R8, bool G1>
struct DNRow {
    IdxT<VPL, G1> c13;
    Idx8<VPL> c8;
};

// One output row m of expert slot d (staged columns at vr) for NC columns:
// the dot products, the warp sums, one atomic per (row, token).
template <int VPL, bool R8, bool RI, int NC, bool G1>
__device__ __forceinline__ void dn_row(const VqdArgs &a, const VqdShared &s, const uint8_t *b13, const uint8_t *b8,
                                       const uint16_t *vr, int vstride, int d, int m, int j0,
                                       const DNRow<VPL, R8, G1> &r) {
    const int lane = threadIdx.x & 31, H = a.H;
    vr += (size_t)j0 * vstride;
    float ay[NC][2];
#pragma unroll
    for (int j = 0; j < NC; ++j) ay[j][0] = ay[j][1] = 0.f;
#pragma unroll
    for (int mm = 0; mm < VPL; ++mm) {
        uint32_t rr = 0;
        if constexpr (R8) rr = r.c8.get(mm);
        const uint4 wv = codeword2<R8, RI, G1>(b13, b8, r.c13.get(mm), rr, lane, a.rho2);
#pragma unroll
        for (int j = 0; j < NC; ++j) dot8<G1>(ay[j], wv, lds128(vr + (size_t)j * vstride + 8 * mm));
    }
    const size_t row = (size_t)s.tb.expert[d] * H + m;
    const float gd = (a.gain[2] ? f16_bits_to_f32(__ldg(a.gain[2] + row)) : 1.f) * (G1 ? a.gs13 : 1.f);
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        const float y = warp_sum(ay[j][0] + ay[j][1]) * gd;
        if (lane == 0) atomicAdd(a.acc + (size_t)s.ct.tok[d][j0 + j] * H + m, y);
    }
}

template <int VPL, bool R8, int TB, bool G1>   // VPL = I / 256; G1: GVQ1 format
__global__ void __launch_bounds__(kVThreads, 1) vqd_down_kernel(VqdArgs a) {
    constexpr bool RI = use_ri<VPL, R8, TB, true, G1>();
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *b13 = smem, *b8 = smem + (G1 ? kG13Bytes : kB13Bytes);
    uint16_t *vs = reinterpret_cast<uint16_t *>(smem + books_bytes<R8, RI, G1>());   // [2][TB][skewed I] bf16
    __shared__ VqdShared s;
    __shared__ __align__(8) uint64_t bar;
    __shared__ int is_last;
    const int H = a.H, I = a.I, T = a.T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vstride = skew_stride<VPL>(I);
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (warp == 0) {
        load_books<RI, G1>(b13, b8, a, &bar);
        build_route_table(s.tb, a.ids, a.topk_w, T * a.k, a.k, a.E, nullptr, false);
        __syncwarp();
        build_cols(s.ct, s.tb);
    }
    if constexpr (RI) fill_ri<G1>(b8, a);
    __syncthreads();
    // this CTA's items (expert slot, output row) span at most two experts
    // (the grid has at least as many CTAs as there are experts)
    const int lH = 31 - __clz(H);
    const int n_items = s.tb.D * H;
    const int c0 = (int)((long long)n_items * blockIdx.x / gridDim.x);
    const int c1 = (int)((long long)n_items * (blockIdx.x + 1) / gridDim.x);
    const int d_lo = c0 >> lH;
    const int d_hi = c1 > c0 ? (c1 - 1) >> lH : d_lo - 1;
    // h comes from the gate/up kernel
    pdl_wait_primary();
    // B columns: for expert slot d in [d_lo, d_hi] and its column j (token
    // tk), v[k] = sum over the routes r of (d, tk) of w_r h_r[k], as bf16
    for (int dd = 0; dd < 2 && d_lo + dd <= d_hi; ++dd) {
        const int d = d_lo + dd;
        const int nc = s.ct.ncol[d];
        for (int idx = threadIdx.x; idx < nc * (I / 8); idx += kVThreads) {
            const int j = idx / (I / 8), k8 = (idx % (I / 8)) * 8, tk = s.ct.tok[d][j];
            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int c = s.tb.col_beg[d]; c < s.tb.col_beg[d + 1]; ++c) {
                const int rt = s.tb.route[c];
                if (s.tb.tok[rt] != tk) continue;
                const float w = s.tb.w[rt];
                const float4 h0 = __ldcg(reinterpret_cast<const float4 *>(a.h + (size_t)rt * I + k8));
                const float4 h1 = __ldcg(reinterpret_cast<const float4 *>(a.h + (size_t)rt * I + k8 + 4));
                v[0] = fmaf(w, h0.x, v[0]); v[1] = fmaf(w, h0.y, v[1]); v[2] = fmaf(w, h0.z, v[2]);
                v[3] = fmaf(w, h0.w, v[3]); v[4] = fmaf(w, h1.x, v[4]); v[5] = fmaf(w, h1.y, v[5]);
                v[6] = fmaf(w, h1.z, v[6]); v[7] = fmaf(w, h1.w, v[7]);
            }
            __nv_bfloat162 p0 = __floats2bfloat162_rn(v[0], v[1]), p1 = __floats2bfloat162_rn(v[2], v[3]);
            __nv_bfloat162 p2 = __floats2bfloat162_rn(v[4], v[5]), p3 = __floats2bfloat162_rn(v[6], v[7]);
            *reinterpret_cast<uint4 *>(vs + ((size_t)dd * TB + j) * vstride + skew_pos<VPL>(k8)) =
                make_uint4(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1),
                           *reinterpret_cast<uint32_t *>(&p2), *reinterpret_cast<uint32_t *>(&p3));
        }
    }
    volatile int abort_flag = 0;
    const bool books_ok = __syncthreads_and(mbar_poll_abort(&bar, 0, &abort_flag, a.wait_cycles));
    pdl_launch_dependents();

    if (books_ok) {
        const int RB13 = I * 13 / 64, RB8 = I / 8;
        // this warp's share of the CTA's items
        const int w0 = c0 + (int)((long long)(c1 - c0) * warp / kVWarps);
        const int w1 = c0 + (int)((long long)(c1 - c0) * (warp + 1) / kVWarps);
        const int chunk = skew_pos<VPL>(lane * 8 * VPL);
        auto load = [&](int i, DNRow<VPL, R8, G1> &r) {
            const size_t row = (size_t)s.tb.expert[i >> lH] * H + (i & (H - 1));
            if constexpr (G1) r.c13.load(a.code12[2] + row * (I * 3 / 16), a.hi1[2] + row * (I / 64), lane);
            else r.c13.load(a.idx13[2] + row * RB13, lane);
            if constexpr (R8) r.c8.load(a.idx8[2] + row * RB8, lane);
        };
        auto compute = [&](int i, DNRow<VPL, R8, G1> &r) {
            const int d = i >> lH, m = i & (H - 1);
            const uint16_t *vr = vs + (size_t)(d - d_lo) * TB * vstride + chunk;
            r.c13.align();
            const int nc = s.ct.ncol[d];
            if (nc > 4) {
                if constexpr (TB >= 8) dn_row<VPL, R8, RI, 4, G1>(a, s, b13, b8, vr, vstride, d, m, 0, r);
            }
            const int j0 = nc > 4 ? 4 : 0;
            switch (nc - j0) {
                case 1: dn_row<VPL, R8, RI, 1, G1>(a, s, b13, b8, vr, vstride, d, m, j0, r); break;
                case 2: if constexpr (TB >= 2) dn_row<VPL, R8, RI, 2, G1>(a, s, b13, b8, vr, vstride, d, m, j0, r); break;
                case 3: if constexpr (TB >= 4) dn_row<VPL, R8, RI, 3, G1>(a, s, b13, b8, vr, vstride, d, m, j0, r); break;
                case 4: if constexpr (TB >= 4) dn_row<VPL, R8, RI, 4, G1>(a, s, b13, b8, vr, vstride, d, m, j0, r); break;
                default: break;
            }
        };
        DNRow<VPL, R8, G1> ra, rb;
        if (w0 < w1) load(w0, ra);
        for (int i = w0; i < w1; i += 2) {
            if (i + 1 < w1) load(i + 1, rb);
            compute(i, ra);
            if (i + 1 >= w1) break;
            if (i + 2 < w1) load(i + 2, ra);
            compute(i + 1, rb);
        }
    } else if (threadIdx.x == 0) {
        atomicOr(a.status, FLAG_TIMEOUT);
    }
    // the last CTA to finish casts the accumulator and clears it
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int prev = atomicAdd(a.done, 1);
        is_last = prev == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    for (int i = threadIdx.x; i < T * H / 4; i += kVThreads) {
        float4 v = __ldcg(reinterpret_cast<const float4 *>(a.acc) + i);
        __nv_bfloat162 p0 = __floats2bfloat162_rn(v.x, v.y), p1 = __floats2bfloat162_rn(v.z, v.w);
        reinterpret_cast<uint2 *>(a.out)[i] =
            make_uint2(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1));
        __stcg(reinterpret_cast<float4 *>(a.acc) + i, make_float4(0.f, 0.f, 0.f, 0.f));
    }
    if (threadIdx.x == 0) *a.done = 0;
}

// ---------------------------------------------------------------- host

template <int VPL, bool R8, int TB, bool G1>
size_t gu_smem() { return books_bytes<R8, use_ri<VPL, R8, TB, false, G1>(), G1>() + gu_stage_bytes(TB, VPL); }
template <int VPL, bool R8, int TB, bool G1>
size_t dn_smem() { return books_bytes<R8, use_ri<VPL, R8, TB, true, G1>(), G1>() + dn_stage_bytes(TB, VPL); }

int tokens_bound(int T) { return T <= 1 ? 1 : (T <= 2 ? 2 : (T <= 4 ? 4 : 8)); }

template <typename K, typename A>
cudaError_t launch_pdl(K kernel, int grid, size_t smem, cudaStream_t s, bool pdl, A args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kVThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args);
}

template <int VPLG, int VPLD, bool R8, int TB, bool G1>
cudaError_t run(const Layer &L, const VqdArgs &a, cudaStream_t s, const cudaEvent_t *ev) {
    const int dev = L.d.device;
    static std::once_flag once[64];
    static cudaError_t err[64];
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
        cudaError_t e = cudaFuncSetAttribute(vqd_gateup_kernel<VPLG, R8, TB, G1>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kVMaxSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(vqd_down_kernel<VPLD, R8, TB, G1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kVMaxSmem);
        err[dev] = e;
    });
    if (err[dev] != cudaSuccess) return err[dev];
    L.count_launches(2);
    if (ev) record_phase(ev[1], s);
    cudaError_t e = launch_pdl(vqd_gateup_kernel<VPLG, R8, TB, G1>, L.sm_count, gu_smem<VPLG, R8, TB, G1>(), s,
                               ev == nullptr, a);
    if (e != cudaSuccess) return e;
    if (ev) record_phase(ev[2], s);
    e = launch_pdl(vqd_down_kernel<VPLD, R8, TB, G1>, L.sm_count, dn_smem<VPLD, R8, TB, G1>(), s, ev == nullptr, a);
    if (e != cudaSuccess) return e;
    if (ev) {
        record_phase(ev[3], s);
        record_phase(ev[4], s);
    }
    return cudaSuccess;
}

template <int VPLG, int VPLD, bool R8, bool G1>
cudaError_t run_tb(const Layer &L, const VqdArgs &a, cudaStream_t s, const cudaEvent_t *ev) {
    switch (tokens_bound(a.T)) {
        case 1: return run<VPLG, VPLD, R8, 1, G1>(L, a, s, ev);
        case 2: return run<VPLG, VPLD, R8, 2, G1>(L, a, s, ev);
        case 4: return run<VPLG, VPLD, R8, 4, G1>(L, a, s, ev);
        default: return run<VPLG, VPLD, R8, 8, G1>(L, a, s, ev);
    }
}

template <bool R8, bool G1>
cudaError_t run_shape(const Layer &L, const VqdArgs &a, cudaStream_t s, const cudaEvent_t *ev) {
    if (a.H == 4096 && a.I == 2048) return run_tb<16, 8, R8, G1>(L, a, s, ev);
    if (a.H == 2048 && a.I == 2048) return run_tb<8, 8, R8, G1>(L, a, s, ev);
    if (a.H == 4096 && a.I == 4096) return run_tb<16, 16, R8, G1>(L, a, s, ev);
    if (a.H == 2048 && a.I == 4096) return run_tb<8, 16, R8, G1>(L, a, s, ev);
    return cudaErrorInvalidValue;
}

// The GVQ1 residual term is folded into the base entries as an f16 pair
// multiple: the ratio of the book scales must be an f16 value (normal, or
// zero without a residual stage), and the base scale nonzero.
bool gvq1_ratio(const Layer &L, uint32_t *rho2) {
    const float s13 = L.w.gscale[0], s8 = has_r8(L.d.fmt) ? L.w.gscale[1] : 0.f;
    if (!(s13 != 0.f) || !std::isfinite(s13)) return false;
    const float rho = s8 / s13;
    if (!std::isfinite(rho) || (rho != 0.f && (std::fabs(rho) > 65504.f || std::fabs(rho) < 6.103515625e-05f)))
        return false;
    const uint16_t b = __half_as_ushort(__float2half_rn(rho));
    if (rho2) *rho2 = (uint32_t)b | ((uint32_t)b << 16);
    return true;
}

}  // namespace

bool decode_vq_supported(const Layer &L, int T) {
    const moeq_layer_desc &d = L.d;
    if (!(is_vq13(d.fmt) || is_gvq1(d.fmt)) || d.act != MOEQ_ACT_BF16) return false;
    if (is_gvq1(d.fmt) && !gvq1_ratio(L, nullptr)) return false;
    if (!L.vq_acc || !L.vq_done) return false;
    if (T < 1 || T > kVMaxT || T * d.top_k > dec::kMaxR) return false;
    if (!((d.hidden == 2048 || d.hidden == 4096) && (d.inter == 2048 || d.inter == 4096))) return false;
    // the staged operands fit beside the books (without the interleaved residual copies)
    const int TB = tokens_bound(T);
    const int books = is_gvq1(d.fmt) ? books_bytes<true, false, true>() : books_bytes<true, false>();
    if (books + gu_stage_bytes(TB, d.hidden / 256) > kVMaxSmem) return false;
    if (books + dn_stage_bytes(TB, d.inter / 256) > kVMaxSmem) return false;
    // a down CTA's items span at most two experts: at least one CTA per routed expert
    return L.sm_count >= std::min(dec::kMaxR, d.n_experts) && L.sm_count <= 4096;
}

cudaError_t launch_decode_vq(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                             cudaStream_t s, const cudaEvent_t *ev) {
    VqdArgs a{};
    for (int p = 0; p < 3; ++p) {
        const ProjView v = L.view(p);
        a.idx13[p] = v.idx13;
        a.idx8[p] = v.idx8;
        a.gain[p] = v.gain;
        a.code12[p] = v.code12;
        a.hi1[p] = v.hi1;
    }
    const bool g1 = is_gvq1(L.d.fmt), r8 = has_r8(L.d.fmt);
    a.book13 = L.w.book13;
    a.book8 = L.d.fmt == MOEQ_FMT_VQ13_R8 ? L.w.book8 : nullptr;
    a.gbook13 = L.w.gbook13;
    a.gbook8 = L.d.fmt == MOEQ_FMT_GVQ1_R8 ? L.w.gbook8 : nullptr;
    a.gs13 = L.w.gscale[0];
    if (g1 && !gvq1_ratio(L, &a.rho2)) return cudaErrorInvalidValue;
    a.x = reinterpret_cast<const uint16_t *>(x);
    a.ids = ids;
    a.topk_w = topk_w;
    a.h = L.h;
    a.acc = L.vq_acc;
    a.out = reinterpret_cast<uint16_t *>(out);
    a.done = L.vq_done;
    a.status = L.status;
    a.wait_cycles = L.wait_cycles;
    a.T = T;
    a.k = L.d.top_k;
    a.E = L.d.n_experts;
    a.H = L.d.hidden;
    a.I = L.d.inter;
    if (g1) return r8 ? run_shape<true, true>(L, a, s, ev) : run_shape<false, true>(L, a, s, ev);
    return r8 ? run_shape<true, false>(L, a, s, ev) : run_shape<false, false>(L, a, s, ev);
}

}  // namespace moeq
