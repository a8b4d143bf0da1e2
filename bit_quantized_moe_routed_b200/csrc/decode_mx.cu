// decode_mx.cu -- MXFP4 routed-expert FFN at decode sizes (1..8 tokens,
// bf16 activations): a grouped GEMV that streams each selected expert's
// packed codes from HBM once.
//
// Layer: out[t] = sum_s w[t,s] W_down,e (silu(W_gate,e x_t) * (W_up,e x_t))
// ("MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture notes":
// top-8 of 256 routed experts, MXFP4 experts with one E8M0 exponent per 32
// values; "Recipe": expert intermediates stay in a type with f32's range).
//
// Memory: a unit is one expert's 16 gate + 16 up rows (gate/up kernel) or 32
// down rows (down kernel) over the full K.  Its rows are contiguous in HBM,
// so one warp moves a whole unit into shared memory with 1-D bulk copies
// (TMA, one per row, rows padded so that the A-fragment reads below hit
// distinct banks) and signals an mbarrier; a ring of stages keeps the next
// unit(s) in flight while the current one is computed.  One CTA per SM.
//
// Math: warp-level mma.sync.m16n8k16 (f16 in, f32 accumulate).  Each thread
// reads its A-fragment slice of four 32-weight blocks (bytes 4t..4t+3 of
// each block; the upload transposes the words of each 64-byte group so the
// slice is one 16-byte word) and decodes it with cvt.rn.f16x2.e2m1x2
// (exact).  Per block the two MMAs accumulate into a fresh fragment that is
// folded into the running f32 sum times the block's E8M0 scale, so the scale
// is applied exactly.  The B operand (activations, or w * h for the down
// projection) is f16 after a per-token power-of-two prescale that puts the
// largest magnitude in [2^14, 2^15): f16 cannot overflow, and the scale is
// undone in f32.  The 16 warps split K; their fragments are summed through
// shared memory.
//
// Combine: the down kernel writes each expert's contribution to its own
// slice of a scratch buffer; the last unit to finish a 32-row tile
// (per-tile arrival counter) sums the experts in a fixed order, undoes the
// prescale and writes bf16 out, so the result does not depend on timing.
#include "async.cuh"
#include "internal.cuh"

namespace moeq {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxT = 8;
constexpr int kMaxR = 64;
constexpr int kXPad = 32;  // f16 elements of padding after each staged x row

struct RouteTable {
    int D;                   // experts with at least one valid route
    int n_valid;
    int expert[kMaxR];       // those experts, ascending
    int col_beg[kMaxR + 1];  // routes of expert slot d: route[col_beg[d] .. col_beg[d+1])
    int route[kMaxR];        // valid route ids sorted by (expert, route id)
    int sid[kMaxR];          // copy of topk_ids
};

// Warp 0 builds the table (R = T*k <= 64 routes).
__device__ void build_route_table(RouteTable &tb, const int32_t *__restrict__ ids, int R, int E,
                                  uint32_t *status, bool report) {
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    const int r0 = lane, r1 = lane + 32;
    const int id0 = r0 < R ? ids[r0] : -1, id1 = r1 < R ? ids[r1] : -1;
    if (r0 < R) tb.sid[r0] = id0;
    if (r1 < R) tb.sid[r1] = id1;
    const bool v0 = id0 >= 0 && id0 < E, v1 = id1 >= 0 && id1 < E;
    const bool bad = (r0 < R && !v0 && id0 != -1) || (r1 < R && !v1 && id1 != -1);
    if (report && __any_sync(full, bad) && lane == 0) atomicOr(status, FLAG_ROUTE_RANGE);
    int rank0 = 0, rank1 = 0;
    for (int q = 0; q < R; ++q) {
        const int idq = __shfl_sync(full, q < 32 ? id0 : id1, q & 31);
        if (idq >= 0 && idq < E) {
            rank0 += (idq < id0 || (idq == id0 && q < r0));
            rank1 += (idq < id1 || (idq == id1 && q < r1));
        }
    }
    if (v0) tb.route[rank0] = r0;
    if (v1) tb.route[rank1] = r1;
    const int n_valid = __popc(__ballot_sync(full, v0)) + __popc(__ballot_sync(full, v1));
    __syncwarp();
    int base = 0;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int p = lane + 32 * hh;
        const int ep = p < n_valid ? tb.sid[tb.route[p]] : -1;
        const int prev = (p > 0 && p < n_valid) ? tb.sid[tb.route[p - 1]] : -2;
        const bool first = p < n_valid && ep != prev;
        const unsigned m = __ballot_sync(full, first);
        if (first) {
            const int slot = base + __popc(m & ((1u << lane) - 1u));
            tb.expert[slot] = ep;
            tb.col_beg[slot] = p;
        }
        base += __popc(m);
    }
    if (lane == 0) {
        tb.D = base;
        tb.n_valid = n_valid;
        tb.col_beg[base] = n_valid;
    }
}

// 2^s for s in [-126, 127]
__device__ __forceinline__ float exp2i(int s) { return __uint_as_float((uint32_t)(s + 127) << 23); }

// Prescale exponent for a set whose largest magnitude is m: m * 2^s in [2^14, 2^15).
__device__ __forceinline__ int prescale_exp(float m) {
    if (!(m > 0.f)) return 0;
    int eb = (int)((__float_as_uint(m) >> 23) & 0xFFu);
    int e = eb ? eb - 127 : -127;
    int s = 14 - e;
    return s < -126 ? -126 : (s > 126 ? 126 : s);
}

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

// E8M0 byte j of `word` -> 2^(b-127) as f32 (b = 0 gives the subnormal 2^-127).
__device__ __forceinline__ float e8m0_byte(uint32_t word, int j) {
    uint32_t b = (word >> (8 * j)) & 0xFFu;
    return __uint_as_float(max(b << 23, 0x00400000u));
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
    acc[0] = fmaf(sa, c[0], acc[0]);
    acc[1] = fmaf(sa, c[1], acc[1]);
    acc[2] = fmaf(sb, c[2], acc[2]);
    acc[3] = fmaf(sb, c[3], acc[3]);
}

__device__ __forceinline__ uint32_t u4get(const uint4 &v, int j) {
    return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}

// After a timed-out wait: wait (bounded again) for the copies of the units
// after it that were already issued, so none lands in shared memory after
// the CTA has gone.
__device__ void drain_stages(uint64_t *full, int n_stages, int j0, int n_units) {
    for (int j = j0; j < j0 + n_stages - 1; ++j) {
        if ((int)blockIdx.x + j * (int)gridDim.x >= n_units) break;
        mbar_wait_bounded(&full[j % n_stages], (uint32_t)((j / n_stages) & 1), 200000000LL);
    }
}

// ---------------------------------------------------------------- gate/up

struct GateUpArgs {
    const uint8_t *codes_g, *codes_u, *scales_g, *scales_u;
    const uint16_t *x;      // bf16 [T][H]
    const int32_t *ids;     // [T][k]
    const float *topk_w;    // [T][k]
    float *h;               // [T*k][I] f32, by route id
    float *gmax;            // [gridDim.x][kMaxT]: per-CTA max |w h| per token
    uint32_t *status;
    int T, k, E, H, I;
};

constexpr int kGUStages = 2;
constexpr int kRowPad = 64;    // bytes after each staged code row
constexpr int kScalePad = 16;  // bytes after each staged scale row

struct GULayout {
    int row_stride, sc_stride, stage_bytes, xs_stride;
    __host__ __device__ GULayout(int H) {
        row_stride = H / 2 + kRowPad;
        sc_stride = H / 32 + kScalePad;
        stage_bytes = 32 * row_stride + 32 * sc_stride;
        xs_stride = H + kXPad;
    }
    // [stages][stage] [x16: T rows] [red: 16 warps x 32 lanes x 8]
    __host__ __device__ size_t xs_off() const { return (size_t)kGUStages * stage_bytes; }
    __host__ __device__ size_t red_off(int T) const { return xs_off() + sizeof(uint16_t) * (size_t)T * xs_stride; }
    __host__ __device__ size_t bytes(int T) const { return red_off(T) + sizeof(float) * kWarps * 32 * 8; }
};

// Warp 0: put unit j's 16 gate + 16 up rows and their scale rows in stage j % kGUStages.
__device__ __forceinline__ void gu_issue(const GateUpArgs &a, const RouteTable &tb, const GULayout &ly,
                                         uint8_t *stages, uint64_t *full, int j, int n_units) {
    const int u = blockIdx.x + j * gridDim.x;
    if (u >= n_units) return;
    const int lane = threadIdx.x & 31;
    const int tiles = a.I / 16;
    const int d = u / tiles, n0 = (u % tiles) * 16;
    const size_t row0 = (size_t)tb.expert[d] * a.I + n0;
    uint8_t *st = stages + (size_t)(j % kGUStages) * ly.stage_bytes;
    uint64_t *bar = full + (j % kGUStages);
    const uint32_t code_b = a.H / 2, sc_b = a.H / 32;
    if (lane == 0) mbar_arrive_expect_tx(bar, 32u * (code_b + sc_b));
    __syncwarp();
    const int mat = lane >> 4, r = lane & 15;   // lane -> (gate|up, row)
    const uint8_t *codes = mat ? a.codes_u : a.codes_g;
    const uint8_t *scales = mat ? a.scales_u : a.scales_g;
    bulk_g2s(st + (size_t)(mat * 16 + r) * ly.row_stride, codes + (row0 + r) * code_b, code_b, bar);
    bulk_g2s(st + (size_t)32 * ly.row_stride + (size_t)(mat * 16 + r) * ly.sc_stride, scales + (row0 + r) * sc_b,
             sc_b, bar);
}

// NG = groups of four 32-weight blocks per warp's K slice = H / 2048.
template <int NG>
__global__ void __launch_bounds__(kThreads, 1) dec_gateup_mx_kernel(GateUpArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ __align__(8) uint64_t full[kGUStages];
    __shared__ float xinv[kMaxT];
    __shared__ unsigned cta_max[kMaxT];
    const int H = a.H, I = a.I, T = a.T, k = a.k;
    const GULayout ly(H);
    uint8_t *stages = smem_raw;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem_raw + ly.xs_off());
    float *red = reinterpret_cast<float *>(smem_raw + ly.red_off(T));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;

    if (tid == 0) {
        for (int s = 0; s < kGUStages; ++s) mbar_init(&full[s], 1);
        mbar_fence_init();
    }
    if (tid < kMaxT) cta_max[tid] = 0u;
    if (warp == 0) build_route_table(tb, a.ids, T * k, a.E, a.status, blockIdx.x == 0);
    __syncthreads();
    const int tiles = I / 16;
    const int n_units = tb.D * tiles;
    if (warp == 0)
        for (int j = 0; j < kGUStages; ++j) gu_issue(a, tb, ly, stages, full, j, n_units);
    // let the down kernel's CTAs launch as SMs free up (they wait for this
    // grid before reading h)
    pdl_launch_dependents();
    // stage x as f16 with a per-token power-of-two prescale (warp w+1 <-> token w)
    if (warp >= 1 && warp <= T) {
        const int tk = warp - 1;
        const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + (size_t)tk * H);
        float m = 0.f;
        for (int i = lane; i < H / 8; i += 32) {
            uint4 v = xr[i];
            uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                m = fmaxf(m, fmaxf(fabsf(__uint_as_float(q[j] << 16)), fabsf(__uint_as_float(q[j] & 0xFFFF0000u))));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int s = prescale_exp(m);
        const float sc = exp2i(s);
        if (lane == 0) xinv[tk] = exp2i(-s);
        uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)tk * ly.xs_stride);
        for (int i = lane; i < H / 8; i += 32) {
            uint4 v = xr[i];
            uint32_t q[4] = {v.x, v.y, v.z, v.w}, o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __half2 hv = __floats2half2_rn(__uint_as_float(q[j] << 16) * sc,
                                               __uint_as_float(q[j] & 0xFFFF0000u) * sc);
                o[j] = *reinterpret_cast<uint32_t *>(&hv);
            }
            dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    __syncthreads();

    for (int j = 0;; ++j) {
        const int u = blockIdx.x + j * gridDim.x;
        if (u >= n_units) break;
        const uint32_t parity = (uint32_t)((j / kGUStages) & 1);
        const bool ok = mbar_wait_bounded(&full[j % kGUStages], parity);
        // also keeps red[] from being rewritten before the last unit's readers finish
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(a.status, FLAG_TIMEOUT);
                drain_stages(full, kGUStages, j + 1, n_units);
            }
            break;
        }
        const int d = u / tiles, n0 = (u % tiles) * 16;
        const uint8_t *st = stages + (size_t)(j % kGUStages) * ly.stage_bytes;
        for (int cb = tb.col_beg[d]; cb < tb.col_beg[d + 1]; cb += 8) {
            if (cb > tb.col_beg[d]) __syncthreads();   // red[] reuse within a unit
            const int ncol = min(8, tb.col_beg[d + 1] - cb);
            const bool live = g < ncol;
            const int tok = live ? tb.route[cb + g] / k : 0;
            const uint16_t *xrow = xs + (size_t)tok * ly.xs_stride + 8 * t;
            float aG[4] = {0.f, 0.f, 0.f, 0.f}, aU[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int G = 0; G < NG; ++G) {
                const int gg = warp * NG + G;   // group index within the row
                const uint8_t *cp = st + (size_t)g * ly.row_stride + gg * 64 + 16 * t;
                const uint4 ag0 = lds128(cp), ag8 = lds128(cp + 8 * ly.row_stride);
                const uint4 au0 = lds128(cp + 16 * ly.row_stride), au8 = lds128(cp + 24 * ly.row_stride);
                const uint8_t *sp = st + (size_t)32 * ly.row_stride + (size_t)g * ly.sc_stride + gg * 4;
                const uint32_t sg0 = lds32(sp), sg8 = lds32(sp + 8 * ly.sc_stride);
                const uint32_t su0 = lds32(sp + 16 * ly.sc_stride), su8 = lds32(sp + 24 * ly.sc_stride);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint4 xb = live ? lds128(xrow + (gg * 4 + jj) * 32) : make_uint4(0u, 0u, 0u, 0u);
                    block_mma(aG, u4get(ag0, jj), u4get(ag8, jj), xb, e8m0_byte(sg0, jj), e8m0_byte(sg8, jj));
                    block_mma(aU, u4get(au0, jj), u4get(au8, jj), xb, e8m0_byte(su0, jj), e8m0_byte(su8, jj));
                }
            }
            float4 *mine = reinterpret_cast<float4 *>(red + ((size_t)warp * 32 + lane) * 8);
            mine[0] = make_float4(aG[0], aG[1], aG[2], aG[3]);
            mine[1] = make_float4(aU[0], aU[1], aU[2], aU[3]);
            __syncthreads();
            // every warp is done reading this stage: refill it with unit j + kGUStages
            if (warp == 0 && cb + 8 >= tb.col_beg[d + 1]) gu_issue(a, tb, ly, stages, full, j + kGUStages, n_units);
            if (tid < 128) {
                const int row = tid >> 3, col = tid & 7;   // 16 rows x 8 columns
                if (col < ncol) {
                    const int gl = row & 7, hi = row >> 3, tl = col >> 1, cbit = col & 1;
                    const int src_lane = gl * 4 + tl, slot = hi * 2 + cbit;
                    float gs = 0.f, us = 0.f;
#pragma unroll
                    for (int ww = 0; ww < kWarps; ++ww) {
                        gs += red[((size_t)ww * 32 + src_lane) * 8 + slot];
                        us += red[((size_t)ww * 32 + src_lane) * 8 + 4 + slot];
                    }
                    const int route = tb.route[cb + col];
                    const float inv = xinv[route / k];
                    const float hv = silu_f32(gs * inv) * (us * inv);
                    a.h[(size_t)route * I + n0 + row] = hv;
                    const float wh = fabsf(a.topk_w[route] * hv);
                    if (wh > 0.f) atomicMax(&cta_max[route / k], __float_as_uint(isfinite(wh) ? wh : 3.0e38f));
                }
            }
        }
    }
    __syncthreads();
    if (tid < kMaxT) a.gmax[(size_t)blockIdx.x * kMaxT + tid] = __uint_as_float(cta_max[tid]);
}

// ---------------------------------------------------------------- down

struct DownArgs {
    const uint8_t *codes, *scales;  // down projection [E][H][I/2] (device layout), [E][H][I/32]
    const float *h;                 // [T*k][I]
    const float *gmax;              // [n_gmax][kMaxT]
    int n_gmax;
    const int32_t *ids;
    const float *topk_w;
    float *ybuf;                    // [kMaxR expert slots][kMaxT][H]
    int *counters;                  // [H/32], zero between calls
    uint16_t *out;                  // bf16 [T][H]
    uint32_t *status;
    int T, k, E, H, I;
};

constexpr int kDNStages = 4;

struct DNLayout {
    int row_stride, sc_stride, stage_bytes;
    __host__ __device__ DNLayout(int I) {
        row_stride = I / 2 + kRowPad;
        sc_stride = I / 32 + kScalePad;
        stage_bytes = 32 * row_stride + 32 * sc_stride;
    }
    __host__ __device__ size_t red_off() const { return (size_t)kDNStages * stage_bytes; }
    __host__ __device__ size_t bytes() const { return red_off() + sizeof(float) * kWarps * 32 * 8; }
};

__device__ __forceinline__ void dn_issue(const DownArgs &a, const RouteTable &tb, const DNLayout &ly,
                                         uint8_t *stages, uint64_t *full, int j, int n_units) {
    const int u = blockIdx.x + j * gridDim.x;
    if (u >= n_units) return;
    const int lane = threadIdx.x & 31;
    const int tiles = a.H / 32;
    const int d = u / tiles, m0 = (u % tiles) * 32;
    const size_t row = (size_t)tb.expert[d] * a.H + m0 + lane;
    uint8_t *st = stages + (size_t)(j % kDNStages) * ly.stage_bytes;
    uint64_t *bar = full + (j % kDNStages);
    const uint32_t code_b = a.I / 2, sc_b = a.I / 32;
    if (lane == 0) mbar_arrive_expect_tx(bar, 32u * (code_b + sc_b));
    __syncwarp();
    bulk_g2s(st + (size_t)lane * ly.row_stride, a.codes + row * code_b, code_b, bar);
    bulk_g2s(st + (size_t)32 * ly.row_stride + (size_t)lane * ly.sc_stride, a.scales + row * sc_b, sc_b, bar);
}

// NG = groups of four 32-weight blocks per warp's K slice = I / 2048.
template <int NG>
__global__ void __launch_bounds__(kThreads, 1) dec_down_mx_kernel(DownArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ __align__(8) uint64_t full[kDNStages];
    __shared__ float tok_scale[kMaxT], tok_inv[kMaxT];
    __shared__ float rscale[kMaxR];
    __shared__ int last_flag;
    const int H = a.H, I = a.I, T = a.T, k = a.k;
    const DNLayout ly(I);
    uint8_t *stages = smem_raw;
    float *red = reinterpret_cast<float *>(smem_raw + ly.red_off());
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;

    if (tid == 0) {
        for (int s = 0; s < kDNStages; ++s) mbar_init(&full[s], 1);
        mbar_fence_init();
    }
    if (warp == 0) build_route_table(tb, a.ids, T * k, a.E, nullptr, false);
    __syncthreads();
    const int tiles = H / 32;
    const int n_units = tb.D * tiles;
    if (tb.D == 0) {   // no valid route at all: every output is zero
        for (int i = blockIdx.x * kThreads + tid; i < T * H; i += gridDim.x * kThreads) a.out[i] = 0;
        return;
    }
    // the weights do not depend on the gate/up kernel: start streaming them now
    if (warp == 0)
        for (int j = 0; j < kDNStages; ++j) dn_issue(a, tb, ly, stages, full, j, n_units);
    // h and gmax come from the gate/up kernel
    pdl_wait_primary();
    if (warp >= 1 && warp <= kMaxT) {
        const int tk = warp - 1;
        float m = 0.f;
        for (int i = lane; i < a.n_gmax; i += 32) m = fmaxf(m, __ldcg(a.gmax + (size_t)i * kMaxT + tk));
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) {
            const int s = prescale_exp(m);
            tok_scale[tk] = exp2i(s);
            tok_inv[tk] = exp2i(-s);
        }
    }
    __syncthreads();
    if (tid < T * k) rscale[tid] = a.topk_w[tid] * tok_scale[tid / k];
    __syncthreads();

    for (int j = 0;; ++j) {
        const int u = blockIdx.x + j * gridDim.x;
        if (u >= n_units) break;
        const int d = u / tiles, tile = u % tiles, m0 = tile * 32;
        // B column g = token g: sum over the token's routes to this expert of
        // w * prescale * h, this warp's K slice (loads issued before the wait)
        const bool live = g < T;
        float bsum[NG][4][8];
#pragma unroll
        for (int G = 0; G < NG; ++G)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                for (int i = 0; i < 8; ++i) bsum[G][jj][i] = 0.f;
        if (live) {
            for (int cc = tb.col_beg[d]; cc < tb.col_beg[d + 1]; ++cc) {
                const int r = tb.route[cc];
                if (r / k != g) continue;
                const float rs = rscale[r];
                const float *hp = a.h + (size_t)r * I + (size_t)warp * NG * 128 + 8 * t;
#pragma unroll
                for (int G = 0; G < NG; ++G)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const float4 v0 = __ldcg(reinterpret_cast<const float4 *>(hp + (4 * G + jj) * 32));
                        const float4 v1 = __ldcg(reinterpret_cast<const float4 *>(hp + (4 * G + jj) * 32 + 4));
                        float *bb = bsum[G][jj];
                        bb[0] = fmaf(rs, v0.x, bb[0]);
                        bb[1] = fmaf(rs, v0.y, bb[1]);
                        bb[2] = fmaf(rs, v0.z, bb[2]);
                        bb[3] = fmaf(rs, v0.w, bb[3]);
                        bb[4] = fmaf(rs, v1.x, bb[4]);
                        bb[5] = fmaf(rs, v1.y, bb[5]);
                        bb[6] = fmaf(rs, v1.z, bb[6]);
                        bb[7] = fmaf(rs, v1.w, bb[7]);
                    }
            }
        }
        const uint32_t parity = (uint32_t)((j / kDNStages) & 1);
        const bool ok = mbar_wait_bounded(&full[j % kDNStages], parity);
        if (__syncthreads_or(!ok)) {
            if (tid == 0) {
                atomicOr(a.status, FLAG_TIMEOUT);
                drain_stages(full, kDNStages, j + 1, n_units);
            }
            break;
        }
        const uint8_t *st = stages + (size_t)(j % kDNStages) * ly.stage_bytes;
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int G = 0; G < NG; ++G) {
            const int gg = warp * NG + G;
            const uint8_t *cp = st + (size_t)g * ly.row_stride + gg * 64 + 16 * t;
            const uint4 c0 = lds128(cp), c1 = lds128(cp + 8 * ly.row_stride);
            const uint4 c2 = lds128(cp + 16 * ly.row_stride), c3 = lds128(cp + 24 * ly.row_stride);
            const uint8_t *sp = st + (size_t)32 * ly.row_stride + (size_t)g * ly.sc_stride + gg * 4;
            const uint32_t q0 = lds32(sp), q1 = lds32(sp + 8 * ly.sc_stride);
            const uint32_t q2 = lds32(sp + 16 * ly.sc_stride), q3 = lds32(sp + 24 * ly.sc_stride);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                uint4 xb;
                __half2 h01 = __floats2half2_rn(bsum[G][jj][0], bsum[G][jj][1]);
                __half2 h23 = __floats2half2_rn(bsum[G][jj][2], bsum[G][jj][3]);
                __half2 h45 = __floats2half2_rn(bsum[G][jj][4], bsum[G][jj][5]);
                __half2 h67 = __floats2half2_rn(bsum[G][jj][6], bsum[G][jj][7]);
                xb.x = *reinterpret_cast<uint32_t *>(&h01);
                xb.y = *reinterpret_cast<uint32_t *>(&h23);
                xb.z = *reinterpret_cast<uint32_t *>(&h45);
                xb.w = *reinterpret_cast<uint32_t *>(&h67);
                block_mma(acc0, u4get(c0, jj), u4get(c1, jj), xb, e8m0_byte(q0, jj), e8m0_byte(q1, jj));
                block_mma(acc1, u4get(c2, jj), u4get(c3, jj), xb, e8m0_byte(q2, jj), e8m0_byte(q3, jj));
            }
        }
        float4 *mine = reinterpret_cast<float4 *>(red + ((size_t)warp * 32 + lane) * 8);
        mine[0] = make_float4(acc0[0], acc0[1], acc0[2], acc0[3]);
        mine[1] = make_float4(acc1[0], acc1[1], acc1[2], acc1[3]);
        __syncthreads();
        if (warp == 0) dn_issue(a, tb, ly, stages, full, j + kDNStages, n_units);
        if (tid < 256) {
            const int row = tid >> 3, col = tid & 7;   // 32 rows x 8 tokens
            if (col < T) {
                const int sub = row >> 4, rl = row & 15;
                const int gl = rl & 7, hi = rl >> 3, tl = col >> 1, cbit = col & 1;
                const int src_lane = gl * 4 + tl, slot = sub * 4 + hi * 2 + cbit;
                float s = 0.f;
#pragma unroll
                for (int ww = 0; ww < kWarps; ++ww) s += red[((size_t)ww * 32 + src_lane) * 8 + slot];
                __stcg(a.ybuf + ((size_t)d * kMaxT + col) * H + m0 + row, s);
            }
            __threadfence();
        }
        __syncthreads();
        if (tid == 0) {
            const int old = atomicAdd(a.counters + tile, 1);
            last_flag = (old == tb.D - 1);
        }
        __syncthreads();
        if (last_flag && tid < 256) {
            __threadfence();
            const int row = tid >> 3, col = tid & 7;
            if (col < T) {
                float s = 0.f;
                for (int dd = 0; dd < tb.D; ++dd) s += __ldcg(a.ybuf + ((size_t)dd * kMaxT + col) * H + m0 + row);
                __nv_bfloat16 o = __float2bfloat16_rn(s * tok_inv[col]);
                a.out[(size_t)col * H + m0 + row] = *reinterpret_cast<uint16_t *>(&o);
            }
            if (tid == 0) a.counters[tile] = 0;
        }
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

constexpr size_t kMaxDynSmem = 232448 - 4096;   // leave room for the static shared memory

template <int NGU, int NGD>
cudaError_t run_decode(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                       cudaStream_t s, const cudaEvent_t *ev) {
    const int H = L.d.hidden, I = L.d.inter;
    const int grid = L.sm_count;
    const GULayout gl(H);
    const DNLayout dl(I);
    static bool attr_done[64] = {};
    const int dev = L.d.device;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(dec_gateup_mx_kernel<NGU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)gl.bytes(kMaxT));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(dec_down_mx_kernel<NGD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)dl.bytes());
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    GateUpArgs ga;
    ga.codes_g = L.w.codes[MOEQ_GATE];
    ga.codes_u = L.w.codes[MOEQ_UP];
    ga.scales_g = L.w.scales[MOEQ_GATE];
    ga.scales_u = L.w.scales[MOEQ_UP];
    ga.x = reinterpret_cast<const uint16_t *>(x);
    ga.ids = ids;
    ga.topk_w = topk_w;
    ga.h = L.h;
    ga.gmax = L.dec_gmax;
    ga.status = L.status;
    ga.T = T;
    ga.k = L.d.top_k;
    ga.E = L.d.n_experts;
    ga.H = H;
    ga.I = I;
    L.count_launches(2);
    if (ev) record_phase(ev[1], s);   // routing is fused into both kernels' prologues
    cudaError_t e = launch_ex(dec_gateup_mx_kernel<NGU>, dim3(grid), dim3(kThreads), gl.bytes(T), s, false, ga);
    if (e != cudaSuccess) return e;
    if (ev) record_phase(ev[2], s);
    DownArgs da;
    da.codes = L.w.codes[MOEQ_DOWN];
    da.scales = L.w.scales[MOEQ_DOWN];
    da.h = L.h;
    da.gmax = L.dec_gmax;
    da.n_gmax = grid;
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
    // programmatic dependent launch: the down kernel's CTAs start streaming
    // weights while the gate/up kernel drains and wait for it before reading
    // h.  Not with phase events between the two launches.
    e = launch_ex(dec_down_mx_kernel<NGD>, dim3(grid), dim3(kThreads), dl.bytes(), s, ev == nullptr, da);
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
    if (GULayout(d.hidden).bytes(kMaxT) > kMaxDynSmem || DNLayout(d.inter).bytes() > kMaxDynSmem) return false;
    return L.sm_count > 0 && L.sm_count <= kDecMaxGrid;
}

cudaError_t launch_decode_mx(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T,
                             void *out, cudaStream_t s, const cudaEvent_t *ev) {
    const int H = L.d.hidden, I = L.d.inter;
    if (H == 2048 && I == 2048) return run_decode<1, 1>(L, x, ids, topk_w, T, out, s, ev);
    if (H == 2048 && I == 4096) return run_decode<1, 2>(L, x, ids, topk_w, T, out, s, ev);
    if (H == 4096 && I == 2048) return run_decode<2, 1>(L, x, ids, topk_w, T, out, s, ev);
    if (H == 4096 && I == 4096) return run_decode<2, 2>(L, x, ids, topk_w, T, out, s, ev);
    return cudaErrorInvalidValue;
}

}  // namespace moeq
