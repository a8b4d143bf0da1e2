// decode_mx.cu -- MXFP4 routed-expert FFN at decode sizes (1..8 tokens,
// bf16 activations): a grouped GEMV that streams each selected expert's
// packed codes from HBM once.
//
// Layer: out[t] = sum_s w[t,s] W_down,e (silu(W_gate,e x_t) * (W_up,e x_t))
// ("MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture notes":
// top-8 of 256 routed experts, MXFP4 experts with one E8M0 exponent per 32
// values; "Recipe": expert intermediates stay in a type with f32's range).
//
// The products run on the tensor cores through warp-level
// mma.sync.m16n8k16 (f16 in, f32 accumulate): a decode step is bound by HBM,
// and the warp MMA lets each thread turn the bytes it loaded straight into
// A-fragment registers (cvt.rn.f16x2.e2m1x2, exact) without a shared-memory
// round trip for the weights.  Per 32-weight block the two MMAs accumulate
// into a fresh fragment that is then folded into the running f32 sum times
// the block's E8M0 scale, so the scale is applied exactly.  The B operand
// (activations, or w * h for the down projection) is f16 after a per-token
// power-of-two prescale that puts the largest magnitude in [2^14, 2^15):
// f16 cannot overflow, and the scale is undone in f32 afterwards.
//
// Work split: one CTA per SM with two teams of 8 warps.  A unit is one
// expert's 16 gate+up rows (gate/up kernel) or 32 down rows (down kernel)
// over the full K; the 8 warps of a team each take K/8 and their partial
// fragments are summed through shared memory.  The two teams take alternate
// units so that one team's loads are in flight while the other reduces.
// The down kernel writes each expert's contribution to its own slice of a
// scratch buffer; the last unit to finish a 32-row tile (per-tile arrival
// counter) sums the experts in a fixed order, applies 1/prescale and writes
// bf16 out, so the result does not depend on unit timing.
#include "internal.cuh"

namespace moeq {
namespace {

constexpr int kTeamWarps = 8;
constexpr int kTeams = 2;
constexpr int kThreads = 32 * kTeamWarps * kTeams;
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

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ldg_nc_u32(const void *p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

// Named barrier for one team (ids 1, 2; 0 is __syncthreads).
__device__ __forceinline__ void team_sync(int team) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(32 * kTeamWarps));
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

// NG = groups of 4 blocks per warp slice = H / 1024.
template <int NG>
__global__ void __launch_bounds__(kThreads, 1) dec_gateup_mx_kernel(GateUpArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ float xinv[kMaxT];
    __shared__ unsigned cta_max[kMaxT];
    const int H = a.H, I = a.I, T = a.T, k = a.k;
    const int xs_stride = H + kXPad;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem_raw);                               // [T][H+pad] f16
    float *red = reinterpret_cast<float *>(smem_raw + sizeof(uint16_t) * T * xs_stride);  // [2 teams][2][8 warps][32][8]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int team = warp / kTeamWarps, w = warp % kTeamWarps;
    const int g = lane >> 2, t = lane & 3;

    if (warp == 0) build_route_table(tb, a.ids, T * k, a.E, a.status, blockIdx.x == 0);
    if (tid < kMaxT) cta_max[tid] = 0u;
    // stage x as f16 with a per-token power-of-two prescale (warp w <-> token w)
    if (warp < T) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + (size_t)warp * H);
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
        if (lane == 0) xinv[warp] = exp2i(-s);
        uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)warp * xs_stride);
        for (int i = lane; i < H / 8; i += 32) {
            uint4 v = xr[i];
            uint32_t q[4] = {v.x, v.y, v.z, v.w}, o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __half2 hv = __floats2half2_rn(__uint_as_float(q[j] << 16) * sc, __uint_as_float(q[j] & 0xFFFF0000u) * sc);
                o[j] = *reinterpret_cast<uint32_t *>(&hv);
            }
            dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    __syncthreads();

    const int tiles = I / 16;
    const int n_units = tb.D * tiles;
    const int slice_blocks = 4 * NG;                 // blocks of 32 per warp slice
    const size_t rowb = (size_t)H / 2, rows = (size_t)H / 32;
    // let the down kernel's CTAs launch as SMs free up (they wait for this
    // grid before reading h)
    asm volatile("griddepcontrol.launch_dependents;");
    int rc = 0;  // reductions done by this team: picks the red buffer
    for (int u = blockIdx.x + team * gridDim.x; u < n_units; u += kTeams * gridDim.x) {
        const int d = u / tiles, tile = u % tiles;
        const int e = tb.expert[d];
        const int n0 = tile * 16;
        const size_t r0 = (size_t)e * I + n0 + g;
        const uint8_t *pg0 = a.codes_g + r0 * rowb + (size_t)w * slice_blocks * 16 + 16 * t;
        const uint8_t *pu0 = a.codes_u + r0 * rowb + (size_t)w * slice_blocks * 16 + 16 * t;
        const uint8_t *sg0 = a.scales_g + r0 * rows + (size_t)w * slice_blocks;
        const uint8_t *su0 = a.scales_u + r0 * rows + (size_t)w * slice_blocks;
        for (int cb = tb.col_beg[d]; cb < tb.col_beg[d + 1]; cb += 8) {
            const int ncol = min(8, tb.col_beg[d + 1] - cb);
            // this thread's B column: column g of the chunk
            const bool live = g < ncol;
            const int tok = live ? tb.route[cb + g] / k : 0;
            const uint16_t *xrow = xs + (size_t)tok * xs_stride + (size_t)w * slice_blocks * 32 + 8 * t;
            uint4 cg0[NG], cg8[NG], cu0[NG], cu8[NG];
            uint32_t qg0[NG], qg8[NG], qu0[NG], qu8[NG];
#pragma unroll
            for (int G = 0; G < NG; ++G) {
                cg0[G] = ldg_nc_v4(pg0 + 64 * G);
                cg8[G] = ldg_nc_v4(pg0 + 8 * rowb + 64 * G);
                cu0[G] = ldg_nc_v4(pu0 + 64 * G);
                cu8[G] = ldg_nc_v4(pu0 + 8 * rowb + 64 * G);
                qg0[G] = ldg_nc_u32(sg0 + 4 * G);
                qg8[G] = ldg_nc_u32(sg0 + 8 * rows + 4 * G);
                qu0[G] = ldg_nc_u32(su0 + 4 * G);
                qu8[G] = ldg_nc_u32(su0 + 8 * rows + 4 * G);
            }
            float aG[4] = {0.f, 0.f, 0.f, 0.f}, aU[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int G = 0; G < NG; ++G) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 xb = live ? *reinterpret_cast<const uint4 *>(xrow + (4 * G + j) * 32)
                                          : make_uint4(0u, 0u, 0u, 0u);
                    block_mma(aG, u4get(cg0[G], j), u4get(cg8[G], j), xb, e8m0_byte(qg0[G], j), e8m0_byte(qg8[G], j));
                    block_mma(aU, u4get(cu0[G], j), u4get(cu8[G], j), xb, e8m0_byte(qu0[G], j), e8m0_byte(qu8[G], j));
                }
            }
            // team reduction over the 8 K-slices
            // (red[rc&1] is rewritten two reductions later, after a team_sync
            // that every reader of this one has passed)
            float *rb = red + ((size_t)(team * 2 + (rc & 1)) * kTeamWarps) * 32 * 8;
            ++rc;
            float4 *mine = reinterpret_cast<float4 *>(rb + ((size_t)w * 32 + lane) * 8);
            mine[0] = make_float4(aG[0], aG[1], aG[2], aG[3]);
            mine[1] = make_float4(aU[0], aU[1], aU[2], aU[3]);
            team_sync(team);
            const int ttid = tid - team * 32 * kTeamWarps;
            if (ttid < 128) {
                const int row = ttid >> 3, col = ttid & 7;   // 16 rows x 8 columns
                if (col < ncol) {
                    const int gl = row & 7, hi = row >> 3, tl = col >> 1, cbit = col & 1;
                    const int src_lane = gl * 4 + tl, slot = hi * 2 + cbit;
                    float gs = 0.f, us = 0.f;
#pragma unroll
                    for (int ww = 0; ww < kTeamWarps; ++ww) {
                        gs += rb[((size_t)ww * 32 + src_lane) * 8 + slot];
                        us += rb[((size_t)ww * 32 + src_lane) * 8 + 4 + slot];
                    }
                    const int route = tb.route[cb + col];
                    const float inv = xinv[route / k];
                    const float gv = gs * inv, uv = us * inv;
                    const float hv = silu_f32(gv) * uv;
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
    const uint8_t *codes, *scales;  // down projection [E][H][I/2], [E][H][I/32]
    const float *h;                 // [T*k][I]
    const float *gmax;              // [n_gmax][kMaxT]
    int n_gmax;
    const int32_t *ids;
    const float *topk_w;
    float *ybuf;                    // [kMaxR expert slots][kMaxT][H]
    int *counters;                  // [H/32], zero between calls
    uint16_t *out;                  // bf16 [T][H]
    int T, k, E, H, I;
};

template <int NG>
__global__ void __launch_bounds__(kThreads, 1) dec_down_mx_kernel(DownArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ float tok_scale[kMaxT], tok_inv[kMaxT];
    __shared__ float rscale[kMaxR];
    __shared__ int last_flag[kTeams];
    const int H = a.H, I = a.I, T = a.T, k = a.k;
    float *red = reinterpret_cast<float *>(smem_raw);  // [2 teams][2][8 warps][32][8]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int team = warp / kTeamWarps, w = warp % kTeamWarps;
    const int g = lane >> 2, t = lane & 3;

    if (warp == 0) build_route_table(tb, a.ids, T * k, a.E, nullptr, false);
    // h and gmax come from the gate/up kernel (a no-op without PDL)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp >= 1 && warp - 1 < kMaxT) {
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

    const int tiles = H / 32;
    const int n_units = tb.D * tiles;
    const int slice_blocks = 4 * NG;
    const size_t rowb = (size_t)I / 2, rows = (size_t)I / 32;
    int it = 0;  // units done by this team: picks the red buffer
    for (int u = blockIdx.x + team * gridDim.x; u < n_units; u += kTeams * gridDim.x, ++it) {
        const int d = u / tiles, tile = u % tiles;
        const int e = tb.expert[d];
        const int m0 = tile * 32;
        const size_t r0 = (size_t)e * H + m0 + g;
        const uint8_t *p0 = a.codes + r0 * rowb + (size_t)w * slice_blocks * 16 + 16 * t;
        const uint8_t *s0 = a.scales + r0 * rows + (size_t)w * slice_blocks;
        uint4 c[4][NG];
        uint32_t q[4][NG];
#pragma unroll
        for (int G = 0; G < NG; ++G)
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                c[rr][G] = ldg_nc_v4(p0 + (size_t)(8 * rr) * rowb + 64 * G);
                q[rr][G] = ldg_nc_u32(s0 + (size_t)(8 * rr) * rows + 4 * G);
            }
        // B column g = token g: sum of w * prescale * h over the token's routes to e
        const bool live = g < T;
        float bsum[NG][4][8];
#pragma unroll
        for (int G = 0; G < NG; ++G)
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int i = 0; i < 8; ++i) bsum[G][j][i] = 0.f;
        if (live) {
            for (int cc = tb.col_beg[d]; cc < tb.col_beg[d + 1]; ++cc) {
                const int r = tb.route[cc];
                if (r / k != g) continue;
                const float rs = rscale[r];
                const float *hp = a.h + (size_t)r * I + (size_t)w * slice_blocks * 32 + 8 * t;
#pragma unroll
                for (int G = 0; G < NG; ++G)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float4 v0 = __ldcg(reinterpret_cast<const float4 *>(hp + (4 * G + j) * 32));
                        const float4 v1 = __ldcg(reinterpret_cast<const float4 *>(hp + (4 * G + j) * 32 + 4));
                        bsum[G][j][0] = fmaf(rs, v0.x, bsum[G][j][0]);
                        bsum[G][j][1] = fmaf(rs, v0.y, bsum[G][j][1]);
                        bsum[G][j][2] = fmaf(rs, v0.z, bsum[G][j][2]);
                        bsum[G][j][3] = fmaf(rs, v0.w, bsum[G][j][3]);
                        bsum[G][j][4] = fmaf(rs, v1.x, bsum[G][j][4]);
                        bsum[G][j][5] = fmaf(rs, v1.y, bsum[G][j][5]);
                        bsum[G][j][6] = fmaf(rs, v1.z, bsum[G][j][6]);
                        bsum[G][j][7] = fmaf(rs, v1.w, bsum[G][j][7]);
                    }
            }
        }
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int G = 0; G < NG; ++G)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 xb;
                __half2 h01 = __floats2half2_rn(bsum[G][j][0], bsum[G][j][1]);
                __half2 h23 = __floats2half2_rn(bsum[G][j][2], bsum[G][j][3]);
                __half2 h45 = __floats2half2_rn(bsum[G][j][4], bsum[G][j][5]);
                __half2 h67 = __floats2half2_rn(bsum[G][j][6], bsum[G][j][7]);
                xb.x = *reinterpret_cast<uint32_t *>(&h01);
                xb.y = *reinterpret_cast<uint32_t *>(&h23);
                xb.z = *reinterpret_cast<uint32_t *>(&h45);
                xb.w = *reinterpret_cast<uint32_t *>(&h67);
                block_mma(acc0, u4get(c[0][G], j), u4get(c[1][G], j), xb, e8m0_byte(q[0][G], j), e8m0_byte(q[1][G], j));
                block_mma(acc1, u4get(c[2][G], j), u4get(c[3][G], j), xb, e8m0_byte(q[2][G], j), e8m0_byte(q[3][G], j));
            }
        float *rb = red + ((size_t)(team * 2 + (it & 1)) * kTeamWarps) * 32 * 8;
        float4 *mine = reinterpret_cast<float4 *>(rb + ((size_t)w * 32 + lane) * 8);
        mine[0] = make_float4(acc0[0], acc0[1], acc0[2], acc0[3]);
        mine[1] = make_float4(acc1[0], acc1[1], acc1[2], acc1[3]);
        team_sync(team);
        const int ttid = tid - team * 32 * kTeamWarps;   // 0..255: 32 rows x 8 tokens
        {
            const int row = ttid >> 3, col = ttid & 7;
            if (col < T) {
                const int sub = row >> 4, rl = row & 15;
                const int gl = rl & 7, hi = rl >> 3, tl = col >> 1, cbit = col & 1;
                const int src_lane = gl * 4 + tl, slot = sub * 4 + hi * 2 + cbit;
                float s = 0.f;
#pragma unroll
                for (int ww = 0; ww < kTeamWarps; ++ww) s += rb[((size_t)ww * 32 + src_lane) * 8 + slot];
                __stcg(a.ybuf + ((size_t)d * kMaxT + col) * H + m0 + row, s);
            }
        }
        __threadfence();
        team_sync(team);
        if (ttid == 0) {
            const int old = atomicAdd(a.counters + tile, 1);
            last_flag[team] = (old == tb.D - 1);
        }
        team_sync(team);
        if (last_flag[team]) {
            __threadfence();
            const int row = ttid >> 3, col = ttid & 7;
            if (col < T) {
                float s = 0.f;
                for (int dd = 0; dd < tb.D; ++dd) s += __ldcg(a.ybuf + ((size_t)dd * kMaxT + col) * H + m0 + row);
                __nv_bfloat16 o = __float2bfloat16_rn(s * tok_inv[col]);
                a.out[(size_t)col * H + m0 + row] = *reinterpret_cast<uint16_t *>(&o);
            }
            if (ttid == 0) a.counters[tile] = 0;
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

template <int NGU, int NGD>
cudaError_t run_decode(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                       cudaStream_t s, const cudaEvent_t *ev) {
    const int H = L.d.hidden, I = L.d.inter;
    const int grid = L.sm_count;
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
    const size_t red_bytes = sizeof(float) * kTeams * 2 * kTeamWarps * 32 * 8;
    const size_t smem_gu = sizeof(uint16_t) * T * (H + kXPad) + red_bytes;
    static bool attr_done[64] = {};
    const int dev = L.d.device;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(dec_gateup_mx_kernel<NGU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(sizeof(uint16_t) * kMaxT * (H + kXPad) + red_bytes));
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(dec_down_mx_kernel<NGD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)red_bytes);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    L.count_launches(2);
    if (ev) {
        cudaEventRecord(ev[1], s);   // routing is fused into both kernels' prologues
    }
    cudaError_t e = launch_ex(dec_gateup_mx_kernel<NGU>, dim3(grid), dim3(kThreads), smem_gu, s, false, ga);
    if (e != cudaSuccess) return e;
    if (ev) cudaEventRecord(ev[2], s);
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
    da.T = T;
    da.k = L.d.top_k;
    da.E = L.d.n_experts;
    da.H = H;
    da.I = I;
    // programmatic dependent launch: the down kernel's CTAs may start while
    // the gate/up kernel drains; they wait (cudaGridDependencySynchronize)
    // before reading h.  Not with phase events between the two launches.
    e = launch_ex(dec_down_mx_kernel<NGD>, dim3(grid), dim3(kThreads), red_bytes, s, ev == nullptr, da);
    if (e != cudaSuccess) return e;
    if (ev) {
        cudaEventRecord(ev[3], s);
        cudaEventRecord(ev[4], s);
    }
    return cudaSuccess;
}

}  // namespace

bool decode_mx_supported(const Layer &L, int T) {
    const moeq_layer_desc &d = L.d;
    if (d.fmt != MOEQ_FMT_MXFP4 || d.act != MOEQ_ACT_BF16) return false;
    if (T < 1 || T > kMaxT || T * d.top_k > kMaxR) return false;
    const bool hk = d.hidden == 1024 || d.hidden == 2048 || d.hidden == 4096 || d.hidden == 8192;
    const bool ik = d.inter == 1024 || d.inter == 2048 || d.inter == 4096 || d.inter == 8192;
    return hk && ik && d.inter % 16 == 0 && d.hidden % 32 == 0 && L.sm_count > 0 && L.sm_count <= kDecMaxGrid;
}

cudaError_t launch_decode_mx(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T,
                             void *out, cudaStream_t s, const cudaEvent_t *ev) {
    const int H = L.d.hidden, I = L.d.inter;
#define MOEQ_DEC(HV, IV)                                                                          \
    if (H == HV * 1024 && I == IV * 1024) return run_decode<HV, IV>(L, x, ids, topk_w, T, out, s, ev);
    MOEQ_DEC(1, 1) MOEQ_DEC(1, 2) MOEQ_DEC(1, 4) MOEQ_DEC(1, 8)
    MOEQ_DEC(2, 1) MOEQ_DEC(2, 2) MOEQ_DEC(2, 4) MOEQ_DEC(2, 8)
    MOEQ_DEC(4, 1) MOEQ_DEC(4, 2) MOEQ_DEC(4, 4) MOEQ_DEC(4, 8)
    MOEQ_DEC(8, 1) MOEQ_DEC(8, 2) MOEQ_DEC(8, 4) MOEQ_DEC(8, 8)
#undef MOEQ_DEC
    return cudaErrorInvalidValue;
}

}  // namespace moeq
