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
// contiguous, balanced range of units, and each of its 16 consumer warps
// owns whole units, so no reduction or barrier sits in the main loop.
//
// Memory: the device layout (MxGeom) keeps each (16-row tile, 1024-column
// chunk) block contiguous, so a producer warp streams a chunk of a unit as
// two 8.7 KB bulk copies (TMA) into a ring of 8 shared-memory stages with
// full/empty mbarriers, in the order the consumers take them (units in waves
// of 16, chunk by chunk).  Bulk copies of several KB are what keep HBM busy;
// the layout also makes the fragment and scale reads bank-conflict free.
//
// Math: warp-level mma.sync.m16n8k16 (f16 in, f32 accumulate).  Each thread
// reads its A-fragment slice of four 32-weight blocks (bytes 4t..4t+3 of
// each block: one 16-byte word in the layout) and decodes it with
// cvt.rn.f16x2.e2m1x2 (exact).  Per block the two MMAs accumulate into a
// fresh fragment that is folded into the running f32 sum times the block's
// E8M0 scale (one packed f32x2 FMA per row pair), so the scale is applied
// exactly.  The B operand (activations, or w * h for the down projection) is
// f16 after a per-token power-of-two prescale that puts the largest
// magnitude in [2^14, 2^15): f16 cannot overflow, and the scale is undone in
// f32.
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

constexpr int kCW = 16;   // consumer warps per CTA

// Barrier among the kCW consumer warps (id 1; the producer warp does not join).
__device__ __forceinline__ void named_sync_consumers() {
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kCW) : "memory");
}

// ---------------------------------------------------------------- staging

// Warp roles: kCW consumer warps, each owning whole units, plus one producer
// warp that streams (tile, chunk) blocks into a ring of shared-memory stages.
constexpr int kWSThreads = 32 * (kCW + 1);
constexpr int kProducerWarp = kCW;
constexpr int kKC = 1024;                       // weights of K per chunk (the layout's chunk)
constexpr int kBlk = 16 * (kKC / 2 + kKC / 32); // one (16-row tile, chunk) block of the device layout
constexpr int kStageBytes = 2 * kBlk;           // two blocks: gate + up tile, or two down tiles
constexpr int kMaxStages = 8;
constexpr int kMaxDynSmem = 232448 - 4096;      // leave room for static shared memory

// Producer (one thread): two contiguous blocks of the device layout into
// stage `st`, completing `bar`.
__device__ __forceinline__ void issue_chunk(uint8_t *st, uint64_t *bar, const uint8_t *blk0, const uint8_t *blk1) {
    mbar_arrive_expect_tx(bar, 2u * kBlk);
    bulk_g2s(st, blk0, kBlk, bar);
    bulk_g2s(st + kBlk, blk1, kBlk, bar);
}

// Shared-memory address of this thread's fragment word (bytes 4t..4t+3 of
// the four blocks of K-group grp) of staged row r (0..15) of a block.
__device__ __forceinline__ const uint8_t *frag_ptr(const uint8_t *blk, int r, int grp, int t) {
    return blk + (size_t)r * (kKC / 2) + ((grp ^ (r & 1)) * 64) + 16 * t;
}
// ... and of the scale word (four blocks) of row r, K-group grp.
__device__ __forceinline__ const uint8_t *scale_ptr(const uint8_t *blk, int r, int grp) {
    return blk + 16 * (kKC / 2) + grp * 64 + r * 4;
}

// This CTA's contiguous share [beg, end) of n units.
__device__ __forceinline__ void my_range(int n, int &beg, int &end) {
    beg = (int)(((long long)n * blockIdx.x) / gridDim.x);
    end = (int)(((long long)n * (blockIdx.x + 1)) / gridDim.x);
}

// Chunk order shared by producer and consumers: units go in waves of kCW
// (warp w takes unit w of each wave); within a wave, chunk q of every unit
// comes before chunk q+1.  Returns the global chunk index of (unit j of this
// CTA's range, chunk q).
__device__ __forceinline__ int chunk_index(int j, int q, int n_mine, int nch) {
    const int wave = j / kCW, wbeg = wave * kCW;
    const int wn = min(kCW, n_mine - wbeg);
    return wbeg * nch + q * wn + (j - wbeg);
}

// Producer loop: chunk c of this CTA, in the order above.  After issuing
// chunk c it publishes issued = c + 1.  Chunk c reuses the stage of chunk
// c - S only after that chunk's consumer released it, so a consumer that has
// seen issued > c knows the stage's barrier is in the phase of chunk c; this
// keeps a warp that runs ahead of the others (it waits on a stage whose
// previous chunk, another warp's, is still in flight) from matching the
// parity of a phase two rounds old.
template <typename BlockOf>
__device__ __forceinline__ void produce(uint8_t *stages, uint64_t *full, uint64_t *empty, int S, int n_mine, int nch,
                                        uint32_t *status, volatile int *issued, BlockOf block_of) {
    const int lane = threadIdx.x & 31;
    int c = 0;
    for (int wbeg = 0; wbeg < n_mine; wbeg += kCW) {
        const int wn = min(kCW, n_mine - wbeg);
        for (int q = 0; q < nch; ++q)
            for (int jj = 0; jj < wn; ++jj, ++c) {
                const int s = c % S, kk = c / S;
                if (lane == 0) {
                    if (kk >= 1 && !mbar_wait_bounded(&empty[s], (uint32_t)((kk - 1) & 1)))
                        atomicOr(status, FLAG_TIMEOUT);
                    const uint8_t *b0, *b1;
                    block_of(wbeg + jj, q, b0, b1);
                    issue_chunk(stages + (size_t)s * kStageBytes, &full[s], b0, b1);
                    __threadfence_block();
                    *issued = c + 1;
                }
                __syncwarp();
            }
    }
}

// Consumer: wait until chunk c is issued, then for its data.  False on timeout.
__device__ __forceinline__ bool wait_chunk(uint64_t *full, int S, int c, volatile int *issued) {
    if (*issued <= c) {
        const long long t0 = clock64();
        while (*issued <= c) {
            if (clock64() - t0 > 2000000000LL) return false;
            __nanosleep(32);
        }
    }
    __threadfence_block();
    return mbar_wait_bounded(&full[c % S], (uint32_t)((c / S) & 1));
}

// ---------------------------------------------------------------- gate/up

struct GateUpArgs {
    const uint8_t *codes_g, *codes_u;   // gate, up projections in the device layout (MxGeom)
    const uint16_t *x;                  // bf16 [T][H]
    const int32_t *ids;                 // [T][k]
    const float *topk_w;                // [T][k]
    float *h;                           // [T*k][I] f32, by route id
    float *gmax;                        // [gridDim.x][kMaxT]: per-CTA max |w h| per token
    uint32_t *status;
    int T, k, E, H, I, n_stages;
};

__host__ __device__ inline size_t gu_xs_off(int n_stages) { return (size_t)n_stages * kStageBytes; }
__host__ __device__ inline size_t gu_bytes(int n_stages, int T, int H) {
    return gu_xs_off(n_stages) + sizeof(uint16_t) * (size_t)T * (H + kXPad);
}

// Unit i -> (expert slot d, column chunk, 16-row tile): experts with more
// than 8 routes take one pass per 8 columns.
struct GUItems {
    int n;
    int beg[kMaxR + 1];
};

template <int NCH>   // K chunks per unit = H / kKC
__global__ void __launch_bounds__(kWSThreads, 1) dec_gateup_mx_kernel(GateUpArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ GUItems items;
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
    __shared__ int issued;   // chunks issued by the producer (see produce)
    __shared__ float xinv[kMaxT];
    __shared__ unsigned cta_max[kMaxT];
    const int H = a.H, I = a.I, T = a.T, k = a.k, S = a.n_stages;
    uint8_t *stages = smem_raw;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem_raw + gu_xs_off(S));
    const int xs_stride = H + kXPad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tiles = I / 16;
    const MxGeom geo(I, H);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_fence_init();
        issued = 0;
    }
    if (tid < kMaxT) cta_max[tid] = 0u;
    if (warp == 0) {
        build_route_table(tb, a.ids, T * k, a.E, a.status, blockIdx.x == 0);
        __syncwarp();
        if (lane == 0) {
            int n = 0;
            for (int d = 0; d < tb.D; ++d) {
                items.beg[d] = n;
                n += ((tb.col_beg[d + 1] - tb.col_beg[d] + 7) / 8) * tiles;
            }
            items.beg[tb.D] = n;
            items.n = n;
        }
    }
    __syncthreads();
    int i0, i1;
    my_range(items.n, i0, i1);
    const int n_mine = i1 - i0;
    auto decode_item = [&](int i, int &d, int &rel) {
        d = 0;
        while (items.beg[d + 1] <= i) ++d;
        rel = i - items.beg[d];
    };

    if (warp == kProducerWarp) {
        produce(stages, full, empty, S, n_mine, NCH, a.status, &issued, [&](int j, int q, const uint8_t *&b0, const uint8_t *&b1) {
            int d, rel;
            decode_item(i0 + j, d, rel);
            const size_t off = (size_t)tb.expert[d] * geo.expert_bytes() + geo.block_off(rel % tiles, q);
            b0 = a.codes_g + off;
            b1 = a.codes_u + off;
        });
        return;
    }

    // ---- consumers: stage x as f16 with a per-token power-of-two prescale
    // (warp w <-> token w)
    if (warp < T) {
        const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + (size_t)warp * H);
        float m = 0.f;
        for (int i = lane; i < H / 8; i += 32) {
            uint4 v = xr[i];
            uint32_t qv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                m = fmaxf(m, fmaxf(fabsf(__uint_as_float(qv[j] << 16)), fabsf(__uint_as_float(qv[j] & 0xFFFF0000u))));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int s = prescale_exp(m);
        const float sc = exp2i(s);
        if (lane == 0) xinv[warp] = exp2i(-s);
        uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)warp * xs_stride);
        for (int i = lane; i < H / 8; i += 32) {
            uint4 v = xr[i];
            uint32_t qv[4] = {v.x, v.y, v.z, v.w}, o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __half2 hv = __floats2half2_rn(__uint_as_float(qv[j] << 16) * sc,
                                               __uint_as_float(qv[j] & 0xFFFF0000u) * sc);
                o[j] = *reinterpret_cast<uint32_t *>(&hv);
            }
            dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    named_sync_consumers();

    bool timed_out = false;
    for (int j = warp; j < n_mine; j += kCW) {
        int d, rel;
        decode_item(i0 + j, d, rel);
        const int cb = tb.col_beg[d] + (rel / tiles) * 8, n0 = (rel % tiles) * 16;
        const int ncol = min(8, tb.col_beg[d + 1] - cb);
        const bool live = g < ncol;
        const int tok = live ? tb.route[cb + g] / k : 0;
        const uint16_t *xrow = xs + (size_t)tok * xs_stride + 8 * t;
        float aG[4] = {0.f, 0.f, 0.f, 0.f}, aU[4] = {0.f, 0.f, 0.f, 0.f};
        for (int q = 0; q < NCH; ++q) {
            const int c = chunk_index(j, q, n_mine, NCH), s = c % S;
            if (!wait_chunk(full, S, c, &issued)) timed_out = true;
            const uint8_t *st = stages + (size_t)s * kStageBytes;
#pragma unroll 2
            for (int gp = 0; gp < kKC / 128; ++gp) {   // K-groups of four 32-weight blocks
                // stage = [gate block][up block]; rows g and g+8 of each
                const uint4 ag0 = lds128(frag_ptr(st, g, gp, t)), ag8 = lds128(frag_ptr(st, g + 8, gp, t));
                const uint4 au0 = lds128(frag_ptr(st + kBlk, g, gp, t));
                const uint4 au8 = lds128(frag_ptr(st + kBlk, g + 8, gp, t));
                float sg0[4], sg8[4], su0[4], su8[4];
                e8m0x4(lds32(scale_ptr(st, g, gp)), sg0);
                e8m0x4(lds32(scale_ptr(st, g + 8, gp)), sg8);
                e8m0x4(lds32(scale_ptr(st + kBlk, g, gp)), su0);
                e8m0x4(lds32(scale_ptr(st + kBlk, g + 8, gp)), su8);
                const uint16_t *xq = xrow + (size_t)(q * (kKC / 32) + gp * 4) * 32;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint4 xb = live ? lds128(xq + jj * 32) : make_uint4(0u, 0u, 0u, 0u);
                    block_mma(aG, u4get(ag0, jj), u4get(ag8, jj), xb, sg0[jj], sg8[jj]);
                    block_mma(aU, u4get(au0, jj), u4get(au8, jj), xb, su0[jj], su8[jj]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);   // this warp is done with the stage
        }
        // epilogue: rows (g, g+8) x columns (2t, 2t+1)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int row = g + 8 * (e >> 1), col = 2 * t + (e & 1);
            if (col < ncol) {
                const int route = tb.route[cb + col];
                const float inv = xinv[route / k];
                const float hv = silu_f32(aG[e] * inv) * (aU[e] * inv);
                a.h[(size_t)route * I + n0 + row] = hv;
                const float wh = fabsf(a.topk_w[route] * hv);
                if (wh > 0.f) atomicMax(&cta_max[route / k], __float_as_uint(isfinite(wh) ? wh : 3.0e38f));
            }
        }
    }
    if (timed_out && lane == 0) atomicOr(a.status, FLAG_TIMEOUT);
    named_sync_consumers();
    if (tid < kMaxT) a.gmax[(size_t)blockIdx.x * kMaxT + tid] = __uint_as_float(cta_max[tid]);
}

// ---------------------------------------------------------------- down

struct DownArgs {
    const uint8_t *codes;           // down projection in the device layout (MxGeom)
    const float *h;                 // [T*k][I]
    const float *gmax;              // [n_gmax][kMaxT]
    int n_gmax;
    const int32_t *ids;
    const float *topk_w;
    float *ybuf;                    // [kMaxR expert slots][kMaxT][H]
    int *counters;                  // [H/32], zero between calls
    uint16_t *out;                  // bf16 [T][H]
    uint32_t *status;
    int T, k, E, H, I, n_stages;
};

constexpr int kMaxBSlots = 16;   // staged (expert, token) B columns per CTA

__host__ __device__ inline size_t dn_bytes(int n_stages, int I) {
    return (size_t)n_stages * kStageBytes + sizeof(uint16_t) * (size_t)kMaxBSlots * (I + kXPad);
}

template <int NCH>   // K chunks per unit = I / kKC
__global__ void __launch_bounds__(kWSThreads, 1) dec_down_mx_kernel(DownArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
    __shared__ int issued;   // chunks issued by the producer (see produce)
    __shared__ float tok_scale[kMaxT], tok_inv[kMaxT];
    __shared__ int slot_of[kMaxR][kMaxT];   // (expert slot - d_lo, token) -> staged B column, -1 none
    __shared__ int slot_d[kMaxBSlots], slot_t[kMaxBSlots];
    __shared__ int n_slots;
    const int H = a.H, I = a.I, T = a.T, k = a.k, S = a.n_stages;
    uint8_t *stages = smem_raw;
    uint16_t *bs = reinterpret_cast<uint16_t *>(smem_raw + (size_t)S * kStageBytes);   // [slot][I+pad] f16
    const int bs_stride = I + kXPad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tiles = H / 32;
    const MxGeom geo(H, I);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_fence_init();
        issued = 0;
    }
    if (warp == 0) build_route_table(tb, a.ids, T * k, a.E, nullptr, false);
    __syncthreads();
    const int n_units = tb.D * tiles;
    if (tb.D == 0) {   // no valid route at all: every output is zero
        for (int i = blockIdx.x * kWSThreads + tid; i < T * H; i += gridDim.x * kWSThreads) a.out[i] = 0;
        return;
    }
    int u0, u1;
    my_range(n_units, u0, u1);
    const int n_mine = u1 - u0;

    if (warp == kProducerWarp) {
        // the weights do not depend on the gate/up kernel: stream them at once
        produce(stages, full, empty, S, n_mine, NCH, a.status, &issued, [&](int j, int q, const uint8_t *&b0, const uint8_t *&b1) {
            const int u = u0 + j, d = u / tiles, t32 = u % tiles;
            const uint8_t *eb = a.codes + (size_t)tb.expert[d] * geo.expert_bytes();
            b0 = eb + geo.block_off(2 * t32, q);
            b1 = eb + geo.block_off(2 * t32 + 1, q);
        });
        return;
    }

    // the experts this CTA's units touch, and their (expert, token) columns
    const int d_lo = n_mine > 0 ? u0 / tiles : 0, d_hi = n_mine > 0 ? (u1 - 1) / tiles : -1;
    if (tid == 0) {
        int ns = 0;
        for (int d = d_lo; d <= d_hi; ++d)
            for (int tk = 0; tk < T; ++tk) {
                bool used = false;
                for (int cc = tb.col_beg[d]; cc < tb.col_beg[d + 1]; ++cc) used |= (tb.route[cc] / k == tk);
                int sl = -1;
                if (used) {
                    if (ns < kMaxBSlots) {
                        slot_d[ns] = d;
                        slot_t[ns] = tk;
                    }
                    sl = ns++;
                }
                slot_of[d - d_lo][tk] = sl;
            }
        n_slots = ns;
    }
    // h and gmax come from the gate/up kernel
    pdl_wait_primary();
    if (warp < kMaxT) {
        float m = 0.f;
        for (int i = lane; i < a.n_gmax; i += 32) m = fmaxf(m, __ldcg(a.gmax + (size_t)i * kMaxT + warp));
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) {
            const int s = prescale_exp(m);
            tok_scale[warp] = exp2i(s);
            tok_inv[warp] = exp2i(-s);
        }
    }
    named_sync_consumers();
    const bool staged = n_slots <= kMaxBSlots;
    if (staged) {
        // B column (d, token) = sum over the token's routes to expert d of
        // w * prescale * h, as f16 (summed in f32 first)
        for (int idx = tid; idx < n_slots * (I / 8); idx += 32 * kCW) {
            const int sl = idx / (I / 8), k8 = (idx % (I / 8)) * 8;
            const int d = slot_d[sl], tk = slot_t[sl];
            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int cc = tb.col_beg[d]; cc < tb.col_beg[d + 1]; ++cc) {
                const int r = tb.route[cc];
                if (r / k != tk) continue;
                const float rs = a.topk_w[r] * tok_scale[tk];
                const float4 h0 = __ldcg(reinterpret_cast<const float4 *>(a.h + (size_t)r * I + k8));
                const float4 h1 = __ldcg(reinterpret_cast<const float4 *>(a.h + (size_t)r * I + k8 + 4));
                v[0] = fmaf(rs, h0.x, v[0]); v[1] = fmaf(rs, h0.y, v[1]); v[2] = fmaf(rs, h0.z, v[2]);
                v[3] = fmaf(rs, h0.w, v[3]); v[4] = fmaf(rs, h1.x, v[4]); v[5] = fmaf(rs, h1.y, v[5]);
                v[6] = fmaf(rs, h1.z, v[6]); v[7] = fmaf(rs, h1.w, v[7]);
            }
            __half2 p0 = __floats2half2_rn(v[0], v[1]), p1 = __floats2half2_rn(v[2], v[3]);
            __half2 p2 = __floats2half2_rn(v[4], v[5]), p3 = __floats2half2_rn(v[6], v[7]);
            *reinterpret_cast<uint4 *>(bs + (size_t)sl * bs_stride + k8) =
                make_uint4(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1),
                           *reinterpret_cast<uint32_t *>(&p2), *reinterpret_cast<uint32_t *>(&p3));
        }
        named_sync_consumers();
    }

    bool timed_out = false;
    for (int j = warp; j < n_mine; j += kCW) {
        const int u = u0 + j;
        const int d = u / tiles, tile = u % tiles, m0 = tile * 32;
        const int my_slot = (g < T) ? slot_of[d - d_lo][g] : -1;   // B column g = token g
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        for (int q = 0; q < NCH; ++q) {
            const int c = chunk_index(j, q, n_mine, NCH), s = c % S;
            if (!wait_chunk(full, S, c, &issued)) timed_out = true;
            const uint8_t *st = stages + (size_t)s * kStageBytes;
#pragma unroll 2
            for (int gp = 0; gp < kKC / 128; ++gp) {
                const int kbase = q * kKC + gp * 128 + 8 * t;   // this thread's first K of block 0
                uint4 xb[4];
                if (staged) {
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        xb[jj] = my_slot >= 0 ? lds128(bs + (size_t)my_slot * bs_stride + kbase + jj * 32)
                                              : make_uint4(0u, 0u, 0u, 0u);
                } else {
                    // more columns than staged slots: build B from h in L2
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        if (g < T)
                            for (int cc = tb.col_beg[d]; cc < tb.col_beg[d + 1]; ++cc) {
                                const int r = tb.route[cc];
                                if (r / k != g) continue;
                                const float rs = a.topk_w[r] * tok_scale[g];
                                const float *hp = a.h + (size_t)r * I + kbase + jj * 32;
                                const float4 h0 = __ldcg(reinterpret_cast<const float4 *>(hp));
                                const float4 h1 = __ldcg(reinterpret_cast<const float4 *>(hp + 4));
                                v[0] = fmaf(rs, h0.x, v[0]); v[1] = fmaf(rs, h0.y, v[1]);
                                v[2] = fmaf(rs, h0.z, v[2]); v[3] = fmaf(rs, h0.w, v[3]);
                                v[4] = fmaf(rs, h1.x, v[4]); v[5] = fmaf(rs, h1.y, v[5]);
                                v[6] = fmaf(rs, h1.z, v[6]); v[7] = fmaf(rs, h1.w, v[7]);
                            }
                        __half2 p0 = __floats2half2_rn(v[0], v[1]), p1 = __floats2half2_rn(v[2], v[3]);
                        __half2 p2 = __floats2half2_rn(v[4], v[5]), p3 = __floats2half2_rn(v[6], v[7]);
                        xb[jj] = make_uint4(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1),
                                            *reinterpret_cast<uint32_t *>(&p2), *reinterpret_cast<uint32_t *>(&p3));
                    }
                }
                // stage = [rows m0..m0+15 block][rows m0+16..m0+31 block]
                const uint4 c0 = lds128(frag_ptr(st, g, gp, t)), c1 = lds128(frag_ptr(st, g + 8, gp, t));
                const uint4 c2 = lds128(frag_ptr(st + kBlk, g, gp, t)), c3 = lds128(frag_ptr(st + kBlk, g + 8, gp, t));
                float s0[4], s1[4], s2[4], s3[4];
                e8m0x4(lds32(scale_ptr(st, g, gp)), s0);
                e8m0x4(lds32(scale_ptr(st, g + 8, gp)), s1);
                e8m0x4(lds32(scale_ptr(st + kBlk, g, gp)), s2);
                e8m0x4(lds32(scale_ptr(st + kBlk, g + 8, gp)), s3);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    block_mma(acc0, u4get(c0, jj), u4get(c1, jj), xb[jj], s0[jj], s1[jj]);
                    block_mma(acc1, u4get(c2, jj), u4get(c3, jj), xb[jj], s2[jj], s3[jj]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        // this expert's contribution to rows m0..m0+31, tokens 0..T-1
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            // e < 4: first tile (rows g, g+8), else second tile (rows 16+g, 24+g)
            const int row = g + 8 * ((e >> 1) & 1) + (e < 4 ? 0 : 16), col = 2 * t + (e & 1);
            const float v = e < 4 ? acc0[e] : acc1[e - 4];
            if (col < T) __stcg(a.ybuf + ((size_t)d * kMaxT + col) * H + m0 + row, v);
        }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = (atomicAdd(a.counters + tile, 1) == tb.D - 1);
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {   // every expert of this tile is in: sum in expert order, write bf16
            __threadfence();
            for (int col = 0; col < T; ++col) {
                float sum = 0.f;
                for (int dd = 0; dd < tb.D; ++dd) sum += __ldcg(a.ybuf + ((size_t)dd * kMaxT + col) * H + m0 + lane);
                __nv_bfloat16 o = __float2bfloat16_rn(sum * tok_inv[col]);
                a.out[(size_t)col * H + m0 + lane] = *reinterpret_cast<uint16_t *>(&o);
            }
            if (lane == 0) a.counters[tile] = 0;
        }
    }
    if (timed_out && lane == 0) atomicOr(a.status, FLAG_TIMEOUT);
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

int gu_stages(int T, int H) {
    int s = (int)((kMaxDynSmem - gu_bytes(0, T, H)) / kStageBytes);
    return s > kMaxStages ? kMaxStages : s;
}
int dn_stages(int I) {
    int s = (int)((kMaxDynSmem - dn_bytes(0, I)) / kStageBytes);
    return s > kMaxStages ? kMaxStages : s;
}

template <int NCU, int NCD>
cudaError_t run_decode(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                       cudaStream_t s, const cudaEvent_t *ev) {
    const int H = L.d.hidden, I = L.d.inter;
    const int grid = L.sm_count;
    static bool attr_done[64] = {};
    const int dev = L.d.device;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(dec_gateup_mx_kernel<NCU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kMaxDynSmem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(dec_down_mx_kernel<NCD>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    GateUpArgs ga;
    ga.codes_g = L.w.codes[MOEQ_GATE];
    ga.codes_u = L.w.codes[MOEQ_UP];
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
    ga.n_stages = gu_stages(T, H);
    L.count_launches(2);
    if (ev) record_phase(ev[1], s);   // routing is fused into both kernels' prologues
    cudaError_t e = launch_ex(dec_gateup_mx_kernel<NCU>, dim3(grid), dim3(kWSThreads),
                              gu_bytes(ga.n_stages, T, H), s, false, ga);
    if (e != cudaSuccess) return e;
    if (ev) record_phase(ev[2], s);
    DownArgs da;
    da.codes = L.w.codes[MOEQ_DOWN];
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
    da.n_stages = dn_stages(I);
    // programmatic dependent launch: the down kernel's producer streams
    // weights while the gate/up kernel drains; its consumers wait for that
    // grid before reading h.  Not with phase events between the launches.
    e = launch_ex(dec_down_mx_kernel<NCD>, dim3(grid), dim3(kWSThreads), dn_bytes(da.n_stages, I), s, ev == nullptr,
                  da);
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
    if (gu_stages(kMaxT, d.hidden) < 2 || dn_stages(d.inter) < 2) return false;
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
