// decode_mx.cu -- MXFP4 routed-expert FFN at decode sizes (1..8 tokens,
// bf16 activations): a grouped GEMV that streams each selected expert's
// packed codes from HBM once.
//
// Layer: out[t] = sum_s w[t,s] W_down,e (silu(W_gate,e x_t) * (W_up,e x_t))
// ("MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture notes":
// top-8 of 256 routed experts, MXFP4 experts with one E8M0 exponent per 32
// values; "Recipe": expert intermediates stay in a type with f32's range).
//
// Work: a unit is one expert's 16 gate + 16 up rows (gate/up kernel) or 32
// down rows (down kernel) over the full K; each CTA (one per SM) takes a
// contiguous, balanced range of units.  Its 16 warps stream the units
// directly from HBM into registers: when the CTA has fewer units than
// warps, each unit's K is split into S equal parts (S a power of two up to
// 8) so that nearly every warp streams; otherwise each warp takes whole
// units.  Per 128-column group a lane loads its A-fragment words of both
// halves (gate and up, or the two 16-row down tiles) -- four 16-byte
// words and four scale words -- two groups ahead of the one it computes, so
// that every warp keeps about 5 KB of weight reads in flight.  No stage
// ring, no producer warp, no waits between warps: one CTA barrier sums
// the parts of split units.  The loads carry an evict-first L2 policy:
// every weight byte is read once per call.
//
// Memory: the device layout (MxGeom) keeps each (16-row tile, 1024-column
// chunk) block contiguous, and inside a row each 64-byte group holds a
// lane's fragment words of four 32-weight blocks as one 16-byte word, so
// the fragment loads of a warp are 64-byte coalesced runs.  The gate/up
// kernel lets the down kernel launch as its CTAs finish (programmatic
// dependent launch); the down kernel pulls its own weight range into L2
// (bulk prefetch) before it waits for h, so the down weights stream while
// gate/up drains, and it lets the next gate/up launch early in turn (which
// waits for it before reading anything).
//
// Math: warp-level mma.sync.m16n8k16 (f16 in, f32 accumulate).  Each thread
// decodes its A-fragment slice of four 32-weight blocks with
// cvt.rn.f16x2.e2m1x2 (exact).  Per block the two MMAs accumulate into a
// fresh fragment that is folded into the running f32 sum times the block's
// E8M0 scale (one packed f32x2 FMA per row pair), so the scale is applied
// exactly.  The B operand is f16 after a power-of-two prescale that puts the
// largest magnitude in [2^14, 2^15): per token for the activations, per
// (expert, token) column of w * h for the down projection.  f16 cannot
// overflow, and the scale is undone in f32.
//
// Combine: the down kernel writes each expert's contribution, prescale
// undone, to its own slice of a scratch buffer; the last unit to finish a
// 32-row tile (per-tile arrival counter) sums the experts in a fixed order
// and writes bf16 out, so the result does not depend on timing.
#include <algorithm>
#include <mutex>

#include "async.cuh"
#include "decode_common.cuh"
#include "internal.cuh"

namespace moeq {
namespace {

using dec::RouteTable;
using dec::build_route_table;
using dec::exp2i;
using dec::prescale_exp;
constexpr int kMaxT = 8;
constexpr int kMaxR = dec::kMaxR;
constexpr int kXPad = 32;  // f16 elements of padding after each staged x row

// Four E2M1 pairs (the bytes of w) -> four f16x2, exact; byte i's low
// nibble (the even element) lands in the low half.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                                uint32_t &r3) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
        : "r"(w));
}

// d = A(16x16) * B(16x8), f16 inputs, f32 result (accumulator starts at 0).
__device__ __forceinline__ void mma_f16_zero(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}
__device__ __forceinline__ void mma_f16(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four E8M0 bytes (one scale word) -> four f32 scales, exact: two
// cvt.rn.bf16x2.ue8m0x2 (2^(b-127) is a bf16 value, the subnormal 2^-127
// for b = 0 included), then bf16 -> f32 by position.
__device__ __forceinline__ void e8m0x4(uint32_t w, float s[4]) {
    uint32_t lo, hi;
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.bf16x2.ue8m0x2 %0, a;\n\tcvt.rn.bf16x2.ue8m0x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
    s[0] = __uint_as_float(lo << 16);
    s[1] = __uint_as_float(lo & 0xFFFF0000u);
    s[2] = __uint_as_float(hi << 16);
    s[3] = __uint_as_float(hi & 0xFFFF0000u);
}

// (a0, a1) += s * (b0, b1) with one packed f32x2 FMA.
__device__ __forceinline__ void ffma2(float &a0, float &a1, float s, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %2};\n\tmov.b64 rb, {%3, %4};\n\t"
        "mov.b64 rc, {%0, %1};\n\tfma.rn.f32x2 rc, ra, rb, rc;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(s), "f"(b0), "f"(b1));
}

// One 32-weight block of a 16-row A tile: rows g (word wa) and g+8 (word wb),
// thread slice bytes 4t..4t+3, against B fragment {x01, x23, x45, x67}.
// acc += scale_g * blk (rows g) and scale_g8 * blk (rows g+8).
__device__ __forceinline__ void block_mma(float acc[4], uint32_t wa, uint32_t wb, uint4 xb, float sa, float sb) {
    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
    e2m1x8_to_f16x2(wa, a0, a1, a2, a3);
    e2m1x8_to_f16x2(wb, b0, b1, b2, b3);
    float c[4];
    mma_f16_zero(c, a0, b0, a1, b1, xb.x, xb.y);
    mma_f16(c, a2, b2, a3, b3, xb.z, xb.w);
    ffma2(acc[0], acc[1], sa, c[0], c[1]);
    ffma2(acc[2], acc[3], sb, c[2], c[3]);
}
__device__ __forceinline__ uint32_t u4get(const uint4 &v, int j) {
    return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}

constexpr int kDWarps = 16;                 // warps per CTA, all streaming
constexpr int kDThreads = 32 * kDWarps;
constexpr int kKC = 1024;                       // weights of K per chunk (the layout's chunk)
constexpr int kBlk = 16 * (kKC / 2 + kKC / 32); // one (16-row tile, chunk) block of the device layout
constexpr int kMaxSplit = 8;                    // K parts of one unit
constexpr int kMaxUnits = 128;                  // units of one CTA (checked on the host)
constexpr int kMaxDynSmem = 232448 - 8192;      // leave room for the static shared memory

// Address of this thread's fragment word (bytes 4t..4t+3 of the four blocks
// of K-group grp) of row r (0..15) of a block, and of the scale word.
__device__ __forceinline__ const uint8_t *frag_ptr(const uint8_t *blk, int r, int grp, int t) {
    return blk + (size_t)r * (kKC / 2) + ((grp ^ (r & 1)) * 64) + 16 * t;
}
__device__ __forceinline__ const uint8_t *scale_ptr(const uint8_t *blk, int r, int grp) {
    return blk + 16 * (kKC / 2) + grp * 64 + r * 4;
}

// This CTA's contiguous share [beg, end) of n units (n * gridDim.x < 2^32).
__device__ __forceinline__ void my_range(int n, int &beg, int &end) {
    beg = (int)(((unsigned)n * blockIdx.x) / gridDim.x);
    end = (int)(((unsigned)n * (blockIdx.x + 1)) / gridDim.x);
}

// Read-once global loads: not kept in L1, first out of L2.
__device__ __forceinline__ uint4 ldg_once128(const void *p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}
__device__ __forceinline__ uint32_t ldg_once32(const void *p, uint64_t pol) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.u32 %0, [%1], %2;" : "=r"(v) : "l"(p), "l"(pol));
    return v;
}

// A warp's share of one K-group of a unit: the fragment words of rows g and
// g+8 of both halves (half-0 block b0, half-1 block b1) and their scale words.
struct GroupFrags {
    uint4 a0, a8, b0, b8;
    uint32_t sa0, sa8, sb0, sb8;
};
__device__ __forceinline__ void load_group(const uint8_t *b0, const uint8_t *b1, int g, int t, int gp, uint64_t pol,
                                           GroupFrags &f) {
    f.a0 = ldg_once128(frag_ptr(b0, g, gp, t), pol);
    f.a8 = ldg_once128(frag_ptr(b0, g + 8, gp, t), pol);
    f.b0 = ldg_once128(frag_ptr(b1, g, gp, t), pol);
    f.b8 = ldg_once128(frag_ptr(b1, g + 8, gp, t), pol);
    f.sa0 = ldg_once32(scale_ptr(b0, g, gp), pol);
    f.sa8 = ldg_once32(scale_ptr(b0, g + 8, gp), pol);
    f.sb0 = ldg_once32(scale_ptr(b1, g, gp), pol);
    f.sb8 = ldg_once32(scale_ptr(b1, g + 8, gp), pol);
}
// The four 32-weight block pairs of a loaded group against the four B
// fragments xb[0..3] of that group.
__device__ __forceinline__ void compute_group(const GroupFrags &f, const uint4 xb[4], float acc0[4], float acc1[4]) {
    float sa0[4], sa8[4], sb0[4], sb8[4];
    e8m0x4(f.sa0, sa0);
    e8m0x4(f.sa8, sa8);
    e8m0x4(f.sb0, sb0);
    e8m0x4(f.sb8, sb8);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        block_mma(acc0, u4get(f.a0, jj), u4get(f.a8, jj), xb[jj], sa0[jj], sa8[jj]);
        block_mma(acc1, u4get(f.b0, jj), u4get(f.b8, jj), xb[jj], sb0[jj], sb8[jj]);
    }
}

// How a CTA's n units map onto its warps: S parts per unit (S > 1 when there
// are fewer units than warps), G groups of 128 columns per unit.
struct Split {
    int S, G;
    // this warp's units [j0, j1) and groups [q0, q1) of each
    __device__ void range(int n, int warp, int &j0, int &j1, int &q0, int &q1) const {
        if (S == 1) {
            j0 = n * warp / kDWarps;
            j1 = n * (warp + 1) / kDWarps;
            q0 = 0;
            q1 = G;
        } else if (warp < n * S) {
            j0 = warp / S;
            j1 = j0 + 1;
            q0 = (warp % S) * (G / S);
            q1 = q0 + G / S;
        } else {
            j0 = j1 = q0 = q1 = 0;
        }
    }
};
__device__ __forceinline__ Split make_split(int n, int G) {
    int S = 1;
    while (2 * S * n <= kDWarps && 2 * S <= kMaxSplit && G % (2 * S) == 0) S *= 2;
    return Split{S, G};
}

// Stream the groups of a warp's work: for unit j in [j0, j1), groups
// [q0, q1), two groups in flight ahead of the computed one.  blocks(j, c,
// b0, b1) gives the two half-blocks of unit j's chunk c; xfrag(j, q, xb)
// the B fragments of group q; done(j, acc0, acc1) takes a unit's partial
// sums.
template <typename Blocks, typename XFrag, typename Done>
__device__ __forceinline__ void stream_units(int j0, int j1, int q0, int q1, int g, int t, Blocks blocks, XFrag xfrag,
                                             Done done) {
    const int per = q1 - q0, ns = (j1 - j0) * per;
    if (ns <= 0) return;
    const uint64_t pol = l2_evict_first_policy();
    auto load = [&](int k, GroupFrags &f) {
        const int j = j0 + k / per, q = q0 + k % per;
        const uint8_t *b0, *b1;
        blocks(j, q >> 3, b0, b1);
        load_group(b0, b1, g, t, q & 7, pol, f);
    };
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
    auto step = [&](int k, const GroupFrags &f) {
        const int j = j0 + k / per, q = q0 + k % per;
        uint4 xb[4];
        xfrag(j, q, xb);
        compute_group(f, xb, acc0, acc1);
        if (k % per == per - 1) {
            done(j, acc0, acc1);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc0[i] = acc1[i] = 0.f;
        }
    };
    GroupFrags f0, f1, f2;
    load(0, f0);
    if (ns > 1) load(1, f1);
    for (int k = 0; k < ns; k += 3) {
        if (k + 2 < ns) load(k + 2, f2);
        step(k, f0);
        if (k + 1 >= ns) break;
        if (k + 3 < ns) load(k + 3, f0);
        step(k + 1, f1);
        if (k + 2 >= ns) break;
        if (k + 4 < ns) load(k + 4, f1);
        step(k + 2, f2);
    }
}

// Partial sums of split units, [unit * S + part][lane][8] (acc0 then acc1).
constexpr int kPartFloats = kDWarps * 32 * 8;
__device__ __forceinline__ void put_part(float *part, int slot, const float a0[4], const float a1[4]) {
    float4 *p = reinterpret_cast<float4 *>(part + ((size_t)slot * 32 + (threadIdx.x & 31)) * 8);
    p[0] = make_float4(a0[0], a0[1], a0[2], a0[3]);
    p[1] = make_float4(a1[0], a1[1], a1[2], a1[3]);
}
__device__ __forceinline__ void sum_parts(const float *part, int j, int S, float a0[4], float a1[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) a0[i] = a1[i] = 0.f;
    for (int p = 0; p < S; ++p) {
        const float4 *q = reinterpret_cast<const float4 *>(part + ((size_t)(j * S + p) * 32 + (threadIdx.x & 31)) * 8);
        const float4 u = q[0], v = q[1];
        a0[0] += u.x; a0[1] += u.y; a0[2] += u.z; a0[3] += u.w;
        a1[0] += v.x; a1[1] += v.y; a1[2] += v.z; a1[3] += v.w;
    }
}

// ---------------------------------------------------------------- gate/up

struct GateUpArgs {
    const uint8_t *codes_g, *codes_u;   // gate, up projections in the device layout (MxGeom)
    const uint16_t *x;                  // bf16 [T][H]
    const int32_t *ids;                 // [T][k]
    const float *topk_w;                // [T][k]
    float *h;                           // [T*k][I] f32, by route id
    uint32_t *status;
    int T, k, E, H, I;
};

__host__ __device__ inline size_t gu_part_off(int T, int H) {
    return (sizeof(uint16_t) * (size_t)T * (H + kXPad) + 15) & ~(size_t)15;
}
__host__ __device__ inline size_t gu_bytes(int T, int H) { return gu_part_off(T, H) + sizeof(float) * kPartFloats; }

// Unit i -> (expert slot d, column chunk, 16-row tile): an expert's routes
// are taken 8 columns per pass (the MMA's N; more routes than tokens only
// when a token lists an expert twice).  A CTA keeps its own range of units
// as packed words: d | tile << 6 | first column << 15 | columns << 22.
struct GUItems {
    int n;
    int beg[kMaxR + 1];
};
__device__ __forceinline__ int unit_d(uint32_t u) { return (int)(u & 63u); }
__device__ __forceinline__ int unit_tile(uint32_t u) { return (int)((u >> 6) & 511u); }
__device__ __forceinline__ int unit_cb(uint32_t u) { return (int)((u >> 15) & 127u); }
__device__ __forceinline__ int unit_ncol(uint32_t u) { return (int)(u >> 22); }

template <int NCH>   // K chunks per unit = H / kKC
__global__ void __launch_bounds__(kDThreads, 1) dec_gateup_mx_kernel(GateUpArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ GUItems items;
    __shared__ uint32_t units[kMaxUnits];
    __shared__ int n_units, unit0;
    __shared__ float xinv[kMaxT];
    const int H = a.H, I = a.I, T = a.T, k = a.k;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem_raw);
    float *part = reinterpret_cast<float *>(smem_raw + gu_part_off(T, H));
    const int xs_stride = H + kXPad;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tiles = I / 16;
    const MxGeom geo(I, H);

    // launched as a programmatic dependent of the previous kernel in the
    // stream: its outputs (these inputs, or h that kernel still reads) are
    // ready and free only after this wait
    pdl_wait_primary();
    if (warp == 0) {
        build_route_table(tb, a.ids, a.topk_w, T * k, k, a.E, a.status, blockIdx.x == 0);
        __syncwarp();
        if (lane == 0) {
            int n = 0;
            for (int d = 0; d < tb.D; ++d) {
                items.beg[d] = n;
                n += ((tb.col_beg[d + 1] - tb.col_beg[d] + kMaxT - 1) / kMaxT) * tiles;
            }
            items.beg[tb.D] = n;
            items.n = n;
            int i0, i1;
            my_range(n, i0, i1);
            unit0 = i0;
            n_units = min(i1 - i0, kMaxUnits);
        }
        __syncwarp();
        // this CTA's units, one per lane (tiles is a power of two; binary
        // search for the expert slot: beg[d] <= i < beg[d + 1])
        const int ltiles = 31 - __clz(tiles), D = tb.D;
        for (int j = lane; j < n_units; j += 32) {
            const int i = unit0 + j;
            int lo = 0, hi = D - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (items.beg[mid] <= i) lo = mid;
                else hi = mid - 1;
            }
            const int d = lo, rel = i - items.beg[d], pass = rel >> ltiles, tile = rel & (tiles - 1);
            const int cb = tb.col_beg[d] + pass * kMaxT, ncol = min(kMaxT, tb.col_beg[d + 1] - cb);
            units[j] = (uint32_t)d | ((uint32_t)tile << 6) | ((uint32_t)cb << 15) | ((uint32_t)ncol << 22);
        }
    } else {
        // the activations, bf16 as they are, into padded rows
        for (int i = threadIdx.x - 32; i < T * (H / 8); i += kDThreads - 32) {
            const int tk = i / (H / 8), c = (i % (H / 8)) * 8;
            *reinterpret_cast<uint4 *>(xs + (size_t)tk * xs_stride + c) =
                __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)tk * H + c));
        }
    }
    __syncthreads();
    // x -> f16 in place with a per-token power-of-two prescale (warp w <-> token w)
    if (warp < T) {
        uint4 *row = reinterpret_cast<uint4 *>(xs + (size_t)warp * xs_stride);
        float m = 0.f;
        for (int i = lane; i < H / 8; i += 32) {
            const uint4 v = row[i];
            const uint32_t qv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                m = fmaxf(m, fmaxf(fabsf(__uint_as_float(qv[j] << 16)), fabsf(__uint_as_float(qv[j] & 0xFFFF0000u))));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int s = prescale_exp(m);
        const float sc = exp2i(s);
        if (lane == 0) xinv[warp] = exp2i(-s);
        for (int i = lane; i < H / 8; i += 32) {
            const uint4 v = row[i];
            const uint32_t qv[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __half2 hv = __floats2half2_rn(__uint_as_float(qv[j] << 16) * sc,
                                               __uint_as_float(qv[j] & 0xFFFF0000u) * sc);
                o[j] = *reinterpret_cast<uint32_t *>(&hv);
            }
            row[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    __syncthreads();
    // the down kernel may take SMs as this grid's CTAs finish: it prefetches
    // its weights at once and reads h only after this grid completes
    pdl_launch_dependents();

    const int n = n_units;
    const Split sp = make_split(n, NCH * 8);
    // SwiGLU of a unit's complete sums: lane (g, t) holds rows g and g+8,
    // columns 2t and 2t+1 (routes cb + col)
    auto finish = [&](int j, const float gs[4], const float us[4]) {
        const uint32_t u = units[j];
        const int cb = unit_cb(u), ncol = unit_ncol(u), n0 = unit_tile(u) * 16;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int col = 2 * t + (i & 1), row = g + 8 * (i >> 1);
            if (col < ncol) {
                const int route = tb.route[cb + col];
                const float inv = xinv[tb.tok[route]];
                a.h[(size_t)route * I + n0 + row] = silu_f32(gs[i] * inv) * (us[i] * inv);
            }
        }
    };
    int j0, j1, q0, q1;
    sp.range(n, warp, j0, j1, q0, q1);
    stream_units(
        j0, j1, q0, q1, g, t,
        [&](int j, int c, const uint8_t *&b0, const uint8_t *&b1) {
            const uint32_t u = units[j];
            const size_t off = (size_t)tb.expert[unit_d(u)] * geo.expert_bytes() + geo.block_off(unit_tile(u), c);
            b0 = a.codes_g + off;
            b1 = a.codes_u + off;
        },
        [&](int j, int q, uint4 xb[4]) {
            const uint32_t u = units[j];
            const bool live = g < unit_ncol(u);
            const int tok = live ? tb.tok[tb.route[unit_cb(u) + g]] : 0;
            const uint16_t *xq = xs + (size_t)tok * xs_stride + 8 * t + (size_t)q * 128;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) xb[jj] = live ? lds128(xq + jj * 32) : make_uint4(0u, 0u, 0u, 0u);
        },
        [&](int j, const float a0[4], const float a1[4]) {
            if (sp.S == 1) finish(j, a0, a1);
            else put_part(part, j * sp.S + q0 / (sp.G / sp.S), a0, a1);
        });
    if (sp.S > 1) {
        __syncthreads();
        for (int j = warp; j < n; j += kDWarps) {
            float gs[4], us[4];
            sum_parts(part, j, sp.S, gs, us);
            finish(j, gs, us);
        }
    }
}

// ---------------------------------------------------------------- down

struct DownArgs {
    const uint8_t *codes;           // down projection in the device layout (MxGeom)
    const float *h;                 // [T*k][I]
    const int32_t *ids;
    const float *topk_w;
    float *ybuf;                    // [kMaxR expert slots][kMaxT][H]
    int *counters;                  // [H/32], zero between calls
    uint16_t *out;                  // bf16 [T][H]
    uint32_t *status;
    int T, k, E, H, I;
};

// Staged (expert, token) B columns per CTA.  A CTA's contiguous range of
// units is no longer than one expert's tiles when the grid has at least as
// many CTAs as there are routed experts, so it touches at most two experts:
// at most 2T columns.
constexpr int kMaxBSlots = 16;
constexpr int kMaxTiles = 128;   // H / 32 for H <= 4096
__host__ __device__ inline int dn_slots(int T) { return 2 * T < kMaxBSlots ? 2 * T : kMaxBSlots; }
__host__ __device__ inline size_t dn_part_off(int T, int I) {
    return (sizeof(uint16_t) * (size_t)dn_slots(T) * (I + kXPad) + 15) & ~(size_t)15;
}
__host__ __device__ inline size_t dn_bytes(int T, int I) { return dn_part_off(T, I) + sizeof(float) * kPartFloats; }

template <int NCH>   // K chunks per unit = I / kKC
__global__ void __launch_bounds__(kDThreads, 1) dec_down_mx_kernel(DownArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ int slot_of[2][kMaxT];    // (expert slot - d_lo, token) -> staged B column, -1 none
    __shared__ int slot_d[kMaxBSlots], slot_t[kMaxBSlots];
    __shared__ unsigned slot_max[kMaxBSlots];
    __shared__ float slot_scale[kMaxBSlots], slot_inv[kMaxBSlots];
    __shared__ int n_slots, n_last;
    __shared__ int last_tiles[kMaxTiles];
    const int H = a.H, I = a.I, T = a.T, k = a.k;
    uint16_t *bs = reinterpret_cast<uint16_t *>(smem_raw);   // [slot][I + pad] f16
    float *part = reinterpret_cast<float *>(smem_raw + dn_part_off(T, I));
    const int bs_stride = I + kXPad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tiles = H / 32;
    const MxGeom geo(H, I);

    if (tid == 0) n_last = 0;
    if (tid < kMaxBSlots) slot_max[tid] = 0u;
    // the routing is an input of the call: ready before the gate/up kernel started
    if (warp == 0) build_route_table(tb, a.ids, a.topk_w, T * k, k, a.E, nullptr, false);
    __syncthreads();
    const int n_units = tb.D * tiles;
    if (tb.D == 0) {   // no valid route at all: every output is zero
        pdl_wait_primary();
        for (int i = blockIdx.x * kDThreads + tid; i < T * H; i += gridDim.x * kDThreads) a.out[i] = 0;
        return;
    }
    int u0, u1;
    my_range(n_units, u0, u1);
    const int n_mine = u1 - u0;
    // unit u -> expert slot u / tiles, 32-row tile u % tiles (tiles is a power of two)
    const int ltiles = 31 - __clz(tiles);
    const int d_lo = n_mine > 0 ? u0 >> ltiles : 0;
    // the weights do not depend on the gate/up kernel: pull this CTA's range
    // into L2 now (a unit's two 16-row tiles are one contiguous run)
    if (warp == 0)
        for (int j = lane; j < n_mine; j += 32) {
            const int u = u0 + j, d = u >> ltiles, t32 = u & (tiles - 1);
            const uint8_t *p = a.codes + (size_t)tb.expert[d] * geo.expert_bytes() + geo.block_off(2 * t32, 0);
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"((uint32_t)(2 * NCH * kBlk))
                         : "memory");
        }
    // the (expert, token) columns of this CTA's experts
    if (tid == 0) {
        int ns = 0;
        const int d_hi = n_mine > 0 ? (u1 - 1) >> ltiles : -1;
        for (int dd = 0; dd < 2; ++dd)
            for (int tk = 0; tk < kMaxT; ++tk) slot_of[dd][tk] = -1;
        for (int d = d_lo; d <= d_hi && d < d_lo + 2; ++d)
            for (int cc = tb.col_beg[d]; cc < tb.col_beg[d + 1]; ++cc) {
                const int tk = tb.tok[tb.route[cc]];
                if (ns < kMaxBSlots && slot_of[d - d_lo][tk] < 0) {
                    slot_of[d - d_lo][tk] = ns;
                    slot_d[ns] = d;
                    slot_t[ns++] = tk;
                }
            }
        n_slots = ns;
    }
    // h comes from the gate/up kernel
    pdl_wait_primary();
    __syncthreads();
    // the next kernel may take SMs as this grid's CTAs finish (it waits for
    // this grid's completion before touching memory this kernel uses)
    pdl_launch_dependents();
    // B column sl = (sum of w_r h_r over the token's routes to the expert,
    // in f32) * 2^s_sl in f16, the power of two putting the column's largest
    // magnitude in [2^14, 2^15): f16 cannot overflow and the epilogue undoes
    // the scale exactly.  Pass 1 finds the maxima, pass 2 stores.
    const int n_idx = n_slots * (I / 8);
    auto col8 = [&](int idx, float *vv) {   // 8 values of B column idx / (I/8) from k = 8 (idx % (I/8))
        const int sl = idx / (I / 8), k8 = (idx % (I / 8)) * 8, d = slot_d[sl], tk = slot_t[sl];
#pragma unroll
        for (int i = 0; i < 8; ++i) vv[i] = 0.f;
        for (int cc = tb.col_beg[d]; cc < tb.col_beg[d + 1]; ++cc) {
            const int r = tb.route[cc];
            if (tb.tok[r] != tk) continue;
            const float w = tb.w[r];
            const float4 h0 = __ldcg(reinterpret_cast<const float4 *>(a.h + (size_t)r * I + k8));
            const float4 h1 = __ldcg(reinterpret_cast<const float4 *>(a.h + (size_t)r * I + k8 + 4));
            vv[0] = fmaf(w, h0.x, vv[0]); vv[1] = fmaf(w, h0.y, vv[1]); vv[2] = fmaf(w, h0.z, vv[2]);
            vv[3] = fmaf(w, h0.w, vv[3]); vv[4] = fmaf(w, h1.x, vv[4]); vv[5] = fmaf(w, h1.y, vv[5]);
            vv[6] = fmaf(w, h1.z, vv[6]); vv[7] = fmaf(w, h1.w, vv[7]);
        }
    };
    for (int idx = tid; idx < n_idx; idx += kDThreads) {
        float vv[8];
        col8(idx, vv);
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(vv[i]));
        if (m > 0.f) atomicMax(&slot_max[idx / (I / 8)], __float_as_uint(isfinite(m) ? m : 3.0e38f));
    }
    __syncthreads();
    if (tid < n_slots) {
        const int sc = prescale_exp(__uint_as_float(slot_max[tid]));
        slot_scale[tid] = exp2i(sc);
        slot_inv[tid] = exp2i(-sc);
    }
    __syncthreads();
    for (int idx = tid; idx < n_idx; idx += kDThreads) {
        float vv[8];
        col8(idx, vv);
        const int sl = idx / (I / 8), k8 = (idx % (I / 8)) * 8;
        const float rs = slot_scale[sl];
        __half2 p0 = __floats2half2_rn(rs * vv[0], rs * vv[1]), p1 = __floats2half2_rn(rs * vv[2], rs * vv[3]);
        __half2 p2 = __floats2half2_rn(rs * vv[4], rs * vv[5]), p3 = __floats2half2_rn(rs * vv[6], rs * vv[7]);
        *reinterpret_cast<uint4 *>(bs + (size_t)sl * bs_stride + k8) =
            make_uint4(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1),
                       *reinterpret_cast<uint32_t *>(&p2), *reinterpret_cast<uint32_t *>(&p3));
    }
    __syncthreads();

    // the expert's f32 slice of a unit, prescale undone: lane (g, t) holds
    // rows g, g+8 of both 16-row halves, columns (tokens) 2t and 2t+1
    auto finish = [&](int j, const float s0[4], const float s1[4]) {
        const int u = u0 + j, d = u >> ltiles, m0 = (u & (tiles - 1)) * 32;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int col = 2 * t + (i & 1), row = g + 8 * ((i >> 1) & 1) + 16 * (i >> 2);
            if (col < T) {
                const int sl = slot_of[d - d_lo][col];
                const float v = sl >= 0 ? (i < 4 ? s0[i] : s1[i - 4]) * slot_inv[sl] : 0.f;
                __stcg(a.ybuf + ((size_t)d * kMaxT + col) * H + m0 + row, v);
            }
        }
    };
    const Split sp = make_split(n_mine, NCH * 8);
    int j0, j1, q0, q1;
    sp.range(n_mine, warp, j0, j1, q0, q1);
    stream_units(
        j0, j1, q0, q1, g, t,
        [&](int j, int c, const uint8_t *&b0, const uint8_t *&b1) {
            const int u = u0 + j, d = u >> ltiles, t32 = u & (tiles - 1);
            const uint8_t *eb = a.codes + (size_t)tb.expert[d] * geo.expert_bytes();
            b0 = eb + geo.block_off(2 * t32, c);
            b1 = eb + geo.block_off(2 * t32 + 1, c);
        },
        [&](int j, int q, uint4 xb[4]) {
            const int d = (u0 + j) >> ltiles;
            const int my_slot = (g < T) ? slot_of[d - d_lo][g] : -1;   // B column g = token g
            const uint16_t *xq = bs + (size_t)(my_slot < 0 ? 0 : my_slot) * bs_stride + 8 * t + (size_t)q * 128;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) xb[jj] = my_slot >= 0 ? lds128(xq + jj * 32) : make_uint4(0u, 0u, 0u, 0u);
        },
        [&](int j, const float s0[4], const float s1[4]) {
            if (sp.S == 1) finish(j, s0, s1);
            else put_part(part, j * sp.S + q0 / (sp.G / sp.S), s0, s1);
        });
    if (sp.S > 1) {
        __syncthreads();
        for (int j = warp; j < n_mine; j += kDWarps) {
            float s0[4], s1[4];
            sum_parts(part, j, sp.S, s0, s1);
            finish(j, s0, s1);
        }
    }
    // Combine: once every expert's slice of a 32-row tile is in, the CTA
    // whose unit completed it sums the slices in expert order and writes
    // bf16; the order of the sum does not depend on timing.
    __threadfence();
    __syncthreads();
    for (int j = tid; j < n_mine; j += kDThreads) {
        const int tile = (u0 + j) & (tiles - 1);
        if (atomicAdd(a.counters + tile, 1) == tb.D - 1) last_tiles[atomicAdd(&n_last, 1)] = tile;
    }
    __syncthreads();
    if (n_last > 0) {
        __threadfence();
        for (int idx = tid; idx < n_last * 32 * T; idx += kDThreads) {
            const int row = idx & 31, col = (idx >> 5) % T, m0 = last_tiles[(idx >> 5) / T] * 32;
            float sum = 0.f;
            for (int dd = 0; dd < tb.D; ++dd) sum += __ldcg(a.ybuf + ((size_t)dd * kMaxT + col) * H + m0 + row);
            __nv_bfloat16 o = __float2bfloat16_rn(sum);
            a.out[(size_t)col * H + m0 + row] = *reinterpret_cast<uint16_t *>(&o);
        }
        for (int li = tid; li < n_last; li += kDThreads) a.counters[last_tiles[li]] = 0;
    }
}

template <typename K, typename A>
cudaError_t launch_ex(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, A args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args);
}

template <int NCU, int NCD>
cudaError_t run_decode(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                       cudaStream_t s, const cudaEvent_t *ev) {
    const int H = L.d.hidden, I = L.d.inter;
    const int grid = L.sm_count;
    // the kernels' shared-memory limit, once per device (the caller made the
    // layer's device current); concurrent first calls from several host
    // threads run it once
    static std::once_flag attr_once[64];
    static cudaError_t attr_err[64];
    const int dev = L.d.device;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(attr_once[dev], [&] {
        cudaError_t e = cudaFuncSetAttribute(dec_gateup_mx_kernel<NCU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kMaxDynSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(dec_down_mx_kernel<NCD>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
        attr_err[dev] = e;
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    GateUpArgs ga;
    ga.codes_g = L.w.codes[MOEQ_GATE];
    ga.codes_u = L.w.codes[MOEQ_UP];
    ga.x = reinterpret_cast<const uint16_t *>(x);
    ga.ids = ids;
    ga.topk_w = topk_w;
    ga.h = L.h;
    ga.status = L.status;
    ga.T = T;
    ga.k = L.d.top_k;
    ga.E = L.d.n_experts;
    ga.H = H;
    ga.I = I;
    L.count_launches(2);
    if (ev) record_phase(ev[1], s);   // routing is fused into both kernels' prologues
    cudaError_t e = launch_ex(dec_gateup_mx_kernel<NCU>, dim3(grid), dim3(kDThreads), gu_bytes(T, H), s,
                              ev == nullptr, ga);
    if (e != cudaSuccess) return e;
    if (ev) record_phase(ev[2], s);
    DownArgs da;
    da.codes = L.w.codes[MOEQ_DOWN];
    da.h = L.h;
    da.ids = ids;
    da.topk_w = topk_w;
    da.ybuf = L.dec_ybuf;
    da.counters = L.dec_counters;
    da.out = reinterpret_cast<uint16_t *>(out);
    da.status = L.status;
    da.T = T;
    da.k = L.d.top_k;
    da.E = L.d.n_experts;
    da.H = H;
    da.I = I;
    // programmatic dependent launch: the down kernel prefetches its weights
    // while the gate/up kernel drains, and waits for that grid before
    // reading h.  Not with phase events between the launches.
    e = launch_ex(dec_down_mx_kernel<NCD>, dim3(grid), dim3(kDThreads), dn_bytes(T, I), s, ev == nullptr, da);
    if (e != cudaSuccess) return e;
    if (ev) {
        record_phase(ev[3], s);
        record_phase(ev[4], s);
    }
    return cudaSuccess;
}

}  // namespace

bool decode_mx_supported(const Layer &L, int T) {
    const moeq_layer_desc &d = L.d;
    if (d.fmt != MOEQ_FMT_MXFP4 || d.act != MOEQ_ACT_BF16) return false;
    if (T < 1 || T > kMaxT || T * d.top_k > kMaxR) return false;
    if (!((d.hidden == 2048 || d.hidden == 4096) && (d.inter == 2048 || d.inter == 4096))) return false;
    if (gu_bytes(kMaxT, d.hidden) > (size_t)kMaxDynSmem || dn_bytes(kMaxT, d.inter) > (size_t)kMaxDynSmem) return false;
    // a CTA's gate/up units fit its unit table
    const long long max_units = (long long)kMaxR * (d.inter / 16);   // passes <= routes
    if (L.sm_count <= 0 || (max_units + L.sm_count - 1) / L.sm_count > kMaxUnits) return false;
    // a down CTA's units span at most two experts: one CTA per routed expert at least
    if (L.sm_count < std::min(kMaxR, d.n_experts)) return false;
    if (d.hidden / 32 > kMaxTiles) return false;
    return L.sm_count > 0 && L.sm_count <= kDecMaxGrid;
}

cudaError_t launch_decode_mx(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T,
                             void *out, cudaStream_t s, const cudaEvent_t *ev) {
    const int H = L.d.hidden, I = L.d.inter;
    if (H == 2048 && I == 2048) return run_decode<2, 2>(L, x, ids, topk_w, T, out, s, ev);
    if (H == 2048 && I == 4096) return run_decode<2, 4>(L, x, ids, topk_w, T, out, s, ev);
    if (H == 4096 && I == 2048) return run_decode<4, 2>(L, x, ids, topk_w, T, out, s, ev);
    if (H == 4096 && I == 4096) return run_decode<4, 4>(L, x, ids, topk_w, T, out, s, ev);
    return cudaErrorInvalidValue;
}

}  // namespace moeq
