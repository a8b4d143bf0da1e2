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
// contiguous, balanced range of units.  The 16 consumer warps form one group
// per 1024-column chunk of K, so every chunk of a unit is in compute at
// once; inside a group each warp takes a share of the chunk's 32-weight
// block columns for both halves (gate and up, or the two 16-row down tiles),
// i.e. two independent accumulator chains.  Once per unit, after one
// barrier, threads spread over all warps sum the partial fragments.
//
// Memory: the device layout (MxGeom) keeps each (16-row tile, 1024-column
// chunk) block contiguous, so a producer warp streams a chunk of a unit as
// two 8.7 KB bulk copies (TMA) into a ring of shared-memory stages with
// full/empty mbarriers, unit by unit and chunk by chunk; the activations
// arrive first, one bulk copy per token.  Bulk copies of several KB are what
// keep HBM busy; the layout also makes the fragment and scale reads
// bank-conflict free.
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

// Warp roles: kCW consumer warps plus one producer warp that streams
// (tile, chunk) blocks into a ring of shared-memory stages.
constexpr int kWSThreads = 32 * (kCW + 1);
constexpr int kProducerWarp = kCW;
constexpr int kKC = 1024;                       // weights of K per chunk (the layout's chunk)
constexpr int kBlk = 16 * (kKC / 2 + kKC / 32); // one (16-row tile, chunk) block of the device layout
// A stage holds one piece: cps consecutive chunks of a unit, both halves
// (gate and up tile, or the two down tiles): [half 0: cps blocks][half 1:
// cps blocks], each half one contiguous run of the device layout.
__host__ __device__ inline size_t piece_bytes(int cps) { return 2 * (size_t)cps * kBlk; }
constexpr int kMaxStages = 12;
constexpr int kMaxDynSmem = 232448 - 4096;      // leave room for static shared memory

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

// Chunk c of this CTA is chunk c % nch of unit c / nch (units in order),
// and piece p holds chunks [p cps, (p+1) cps).  The producer warp refills G
// pieces per step: lanes 2i and 2i+1 wait for the stage of piece p0 + i to
// be released, then each issues the bulk copy of one half of it, so one
// instruction starts 2G copies of cps blocks each (fewer, larger copies keep
// more of HBM busy than many small ones).  After a step it publishes issued
// = p0 + G.  Piece p reuses the stage of piece p - S only after every
// consumer released that piece, so a consumer that has seen issued > p knows
// the stage's barrier is in the phase of piece p; this keeps a warp that
// runs ahead of the others from matching the parity of a phase two rounds
// old.
template <typename BlockOf>
__device__ __forceinline__ void produce(uint8_t *stages, uint64_t *full, uint64_t *empty, int S, int cps,
                                        int n_pieces, uint32_t *status, volatile int *issued, BlockOf block_of) {
    const int lane = threadIdx.x & 31, i = lane >> 1, half = lane & 1;
    const int G = min(S, max(1, 4 / cps));
    const uint32_t half_bytes = (uint32_t)cps * kBlk;
    for (int p0 = 0; p0 < n_pieces; p0 += G) {
        const int p = p0 + i;
        const bool mine = i < G && p < n_pieces;
        const int s = mine ? p % S : 0;
        if (mine && half == 0 && p >= S && !mbar_wait_bounded(&empty[s], (uint32_t)((p / S - 1) & 1)))
            atomicOr(status, FLAG_TIMEOUT);
        __syncwarp();
        if (mine && half == 0) mbar_arrive_expect_tx(&full[s], 2u * half_bytes);
        __syncwarp();
        if (mine) {
            const uint8_t *b0, *b1;
            block_of(p, b0, b1);
            bulk_g2s(stages + (size_t)s * piece_bytes(cps) + half * half_bytes, half ? b1 : b0, half_bytes, &full[s]);
        }
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            *issued = min(p0 + G, n_pieces);
        }
    }
}

// Consumer: wait until piece p is issued, then for its data.  False on timeout.
__device__ __forceinline__ bool wait_piece(uint64_t *full, int S, int p, volatile int *issued) {
    if (*issued <= p) {
        const long long t0 = clock64();
        while (*issued <= p) {
            if (clock64() - t0 > 2000000000LL) return false;
            __nanosleep(32);
        }
    }
    return mbar_wait_bounded(&full[p % S], (uint32_t)((p / S) & 1));
}

// Chunk q of every unit is computed by the 16/NCH warps [q*16/NCH, ...): a
// chunk is 16 pieces (8 K-groups x 2 halves: gate/up blocks, or the two
// down tiles) and each of those warps takes NCH of them, K-groups
// (i*NCH/2 ...) of both halves, so NCH chunks are in compute at once and
// each warp runs two independent accumulator chains.  The partial
// fragments go to red[unit parity][warp][half][row][column] and are summed
// in warp order after one barrier per unit.  A unit has at most Tc = min(T,
// 8) columns, so only those are kept.
__host__ __device__ inline int red_cols(int T) { return T < kMaxT ? T : kMaxT; }
__host__ __device__ inline size_t red_bytes(int T) {
    return 2 * (size_t)kCW * 2 * 16 * red_cols(T) * sizeof(float);
}

__device__ __forceinline__ void put_partials(float *rb, int Tc, int warp, int g, int t, const float a0[4],
                                             const float a1[4]) {
    float *h0 = rb + (size_t)warp * 2 * 16 * Tc, *h1 = h0 + 16 * Tc;
    const int c0 = 2 * t, c1 = 2 * t + 1;
    if (c0 < Tc) {
        h0[g * Tc + c0] = a0[0];
        h0[(g + 8) * Tc + c0] = a0[2];
        h1[g * Tc + c0] = a1[0];
        h1[(g + 8) * Tc + c0] = a1[2];
    }
    if (c1 < Tc) {
        h0[g * Tc + c1] = a0[1];
        h0[(g + 8) * Tc + c1] = a0[3];
        h1[g * Tc + c1] = a1[1];
        h1[(g + 8) * Tc + c1] = a1[3];
    }
}
__device__ __forceinline__ float sum_partials(const float *rb, int Tc, int half, int row, int col) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kCW; ++w) s += rb[((size_t)(w * 2 + half) * 16 + row) * Tc + col];
    return s;
}

// A warp's share of one K-group of a staged chunk, read into registers so
// that the stage can be released before the math: the fragment words of
// rows g and g+8 of both halves (half-0 block st0, half-1 block st1) and
// their scale words.
struct GroupFrags {
    uint4 a0, a8, b0, b8;
    uint32_t sa0, sa8, sb0, sb8;
};
__device__ __forceinline__ void load_group(const uint8_t *st0, const uint8_t *st1, int g, int t, int gp,
                                           GroupFrags &f) {
    f.a0 = lds128(frag_ptr(st0, g, gp, t));
    f.a8 = lds128(frag_ptr(st0, g + 8, gp, t));
    f.b0 = lds128(frag_ptr(st1, g, gp, t));
    f.b8 = lds128(frag_ptr(st1, g + 8, gp, t));
    f.sa0 = lds32(scale_ptr(st0, g, gp));
    f.sa8 = lds32(scale_ptr(st0, g + 8, gp));
    f.sb0 = lds32(scale_ptr(st1, g, gp));
    f.sb8 = lds32(scale_ptr(st1, g + 8, gp));
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

// ---------------------------------------------------------------- gate/up

struct GateUpArgs {
    const uint8_t *codes_g, *codes_u;   // gate, up projections in the device layout (MxGeom)
    const uint16_t *x;                  // bf16 [T][H]
    const int32_t *ids;                 // [T][k]
    const float *topk_w;                // [T][k]
    float *h;                           // [T*k][I] f32, by route id
    float *gmax;                        // [gridDim.x][kMaxT]: per-CTA max |w h| per token
    uint32_t *status;
    int T, k, E, H, I, n_stages, cps;
};

__host__ __device__ inline size_t gu_xs_off(int n_stages, int cps) { return (size_t)n_stages * piece_bytes(cps); }
__host__ __device__ inline size_t gu_red_off(int n_stages, int cps, int T, int H) {
    return gu_xs_off(n_stages, cps) + sizeof(uint16_t) * (size_t)T * (H + kXPad);
}
__host__ __device__ inline size_t gu_bytes(int n_stages, int cps, int T, int H) {
    return gu_red_off(n_stages, cps, T, H) + red_bytes(T);
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
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages], xbar;
    __shared__ int issued;   // chunks issued by the producer (see produce)
    __shared__ float xinv[kMaxT];
    __shared__ unsigned cta_max[kMaxT];
    const int H = a.H, I = a.I, T = a.T, k = a.k, S = a.n_stages, cps = a.cps, Tc = red_cols(a.T);
    uint8_t *stages = smem_raw;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem_raw + gu_xs_off(S, cps));
    float *red = reinterpret_cast<float *>(smem_raw + gu_red_off(S, cps, T, H));
    const int xs_stride = H + kXPad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tiles = I / 16;
    const MxGeom geo(I, H);
    constexpr int WPC = kCW / NCH;   // warps per chunk

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], WPC * cps);
        }
        mbar_init(&xbar, 1);
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
        // the activations first (one bulk copy per token row, into padded rows)
        if (lane == 0) mbar_arrive_expect_tx(&xbar, (uint32_t)(T * H * 2));
        __syncwarp();
        if (lane < T) bulk_g2s(xs + (size_t)lane * xs_stride, a.x + (size_t)lane * H, H * 2, &xbar);
        produce(stages, full, empty, S, cps, n_mine * NCH / cps, a.status, &issued,
                [&](int p, const uint8_t *&b0, const uint8_t *&b1) {
                    const int c = p * cps;
                    int d, rel;
                    decode_item(i0 + c / NCH, d, rel);
                    const size_t off = (size_t)tb.expert[d] * geo.expert_bytes() + geo.block_off(rel % tiles, c % NCH);
                    b0 = a.codes_g + off;
                    b1 = a.codes_u + off;
                });
        return;
    }

    // ---- consumers: x -> f16 in place, with a per-token power-of-two
    // prescale (warp w <-> token w)
    bool timed_out = !mbar_wait_bounded(&xbar, 0);
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
    named_sync_consumers();

    const int q = warp / WPC, wi = warp % WPC;   // this warp's chunk of every unit and its place in it
    for (int j = 0; j < n_mine; ++j) {
        int d, rel;
        decode_item(i0 + j, d, rel);
        const int cb = tb.col_beg[d] + (rel / tiles) * 8, n0 = (rel % tiles) * 16;
        const int ncol = min(8, tb.col_beg[d + 1] - cb);
        const bool live = g < ncol;
        const int tok = live ? tb.route[cb + g] / k : 0;
        const uint16_t *xrow = xs + (size_t)tok * xs_stride + 8 * t;
        float aG[4] = {0.f, 0.f, 0.f, 0.f}, aU[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int c = j * NCH + q, pc = c / cps, s = pc % S;
            if (!wait_piece(full, S, pc, &issued)) timed_out = true;
            // [gate blocks of the piece][up blocks of the piece]
            const uint8_t *st0 = stages + (size_t)s * piece_bytes(cps) + (size_t)(c % cps) * kBlk;
            const uint8_t *st1 = st0 + (size_t)cps * kBlk;
            GroupFrags fr[NCH / 2];
#pragma unroll
            for (int p = 0; p < NCH / 2; ++p) load_group(st0, st1, g, t, wi * (NCH / 2) + p, fr[p]);
            // the stage is free again once every warp holds its share
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
            for (int p = 0; p < NCH / 2; ++p) {
                const int gp = wi * (NCH / 2) + p;
                const uint16_t *xq = xrow + (size_t)(q * (kKC / 32) + gp * 4) * 32;
                uint4 xb[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) xb[jj] = live ? lds128(xq + jj * 32) : make_uint4(0u, 0u, 0u, 0u);
                compute_group(fr[p], xb, aG, aU);
            }
        }
        float *rb = red + (size_t)(j & 1) * kCW * 2 * 16 * Tc;
        put_partials(rb, Tc, warp, g, t, aG, aU);
        named_sync_consumers();
        if ((lane & 3) == 0) {   // readers spread over the warps: (row, column) = r % 16, r / 16
            const int r = warp + kCW * (lane >> 2), row = r & 15, col = r >> 4;
            if (col < ncol) {
                const float gs = sum_partials(rb, Tc, 0, row, col), us = sum_partials(rb, Tc, 1, row, col);
                const int route = tb.route[cb + col];
                const float inv = xinv[route / k];
                const float hv = silu_f32(gs * inv) * (us * inv);
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
    int T, k, E, H, I, n_stages, cps;
};

// Staged (expert, token) B columns per CTA.  A CTA's contiguous range of
// units is shorter than one expert's tiles, so it touches at most two
// experts: 2T columns (capped; beyond the cap B is built from h in L2).
constexpr int kMaxBSlots = 16;
constexpr int kMaxTiles = 128;   // H / 32 for H <= 4096
__host__ __device__ inline int dn_slots(int T) { return 2 * T < kMaxBSlots ? 2 * T : kMaxBSlots; }
__host__ __device__ inline size_t dn_red_off(int n_stages, int cps, int T, int I) {
    return (size_t)n_stages * piece_bytes(cps) + sizeof(uint16_t) * (size_t)dn_slots(T) * (I + kXPad);
}
__host__ __device__ inline size_t dn_bytes(int n_stages, int cps, int T, int I) {
    return dn_red_off(n_stages, cps, T, I) + red_bytes(T);
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
    __shared__ int n_slots, n_last;
    __shared__ int last_tiles[kMaxTiles];
    const int H = a.H, I = a.I, T = a.T, k = a.k, S = a.n_stages, cps = a.cps, Tc = red_cols(a.T);
    const int cap = dn_slots(T);
    uint8_t *stages = smem_raw;
    uint16_t *bs = reinterpret_cast<uint16_t *>(smem_raw + (size_t)S * piece_bytes(cps));   // [slot][I+pad] f16
    float *red = reinterpret_cast<float *>(smem_raw + dn_red_off(S, cps, T, I));
    const int bs_stride = I + kXPad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tiles = H / 32;
    const MxGeom geo(H, I);
    constexpr int WPC = kCW / NCH;   // warps per chunk

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], WPC * cps);
        }
        mbar_fence_init();
        issued = 0;
        n_last = 0;
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
        produce(stages, full, empty, S, cps, n_mine * NCH / cps, a.status, &issued,
                [&](int p, const uint8_t *&b0, const uint8_t *&b1) {
                    const int c = p * cps;
                    const int u = u0 + c / NCH, d = u / tiles, t32 = u % tiles, q = c % NCH;
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
                    if (ns < cap) {
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
        // eight independent loads per lane cover 256 CTAs in one round trip
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int i = lane + 32 * q;
            v[q] = i < a.n_gmax ? __ldcg(a.gmax + (size_t)i * kMaxT + warp) : 0.f;
        }
        float m = fmaxf(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])), fmaxf(fmaxf(v[4], v[5]), fmaxf(v[6], v[7])));
        for (int i = lane + 256; i < a.n_gmax; i += 32) m = fmaxf(m, __ldcg(a.gmax + (size_t)i * kMaxT + warp));
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) {
            const int s = prescale_exp(m);
            tok_scale[warp] = exp2i(s);
            tok_inv[warp] = exp2i(-s);
        }
    }
    named_sync_consumers();
    const bool staged = n_slots <= cap;
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

    const int q = warp / WPC, wi = warp % WPC;   // this warp's chunk of every unit and its place in it
    bool timed_out = false;
    for (int j = 0; j < n_mine; ++j) {
        const int u = u0 + j;
        const int d = u / tiles, tile = u % tiles, m0 = tile * 32;
        const int my_slot = (g < T) ? slot_of[d - d_lo][g] : -1;   // B column g = token g
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        {
            uint4 xb[NCH / 2][4];
#pragma unroll
            for (int p = 0; p < NCH / 2; ++p) {
                const int gp = wi * (NCH / 2) + p;
                const int kbase = q * kKC + gp * 128 + 8 * t;   // this thread's first K of the group's block 0
                if (staged) {
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        xb[p][jj] = my_slot >= 0 ? lds128(bs + (size_t)my_slot * bs_stride + kbase + jj * 32)
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
                        xb[p][jj] = make_uint4(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1),
                                               *reinterpret_cast<uint32_t *>(&p2), *reinterpret_cast<uint32_t *>(&p3));
                    }
                }
            }
            const int c = j * NCH + q, pc = c / cps, s = pc % S;
            if (!wait_piece(full, S, pc, &issued)) timed_out = true;
            // [rows m0..+15: blocks of the piece][rows m0+16..+31: blocks of the piece]
            const uint8_t *st0 = stages + (size_t)s * piece_bytes(cps) + (size_t)(c % cps) * kBlk;
            const uint8_t *st1 = st0 + (size_t)cps * kBlk;
            GroupFrags fr[NCH / 2];
#pragma unroll
            for (int p = 0; p < NCH / 2; ++p) load_group(st0, st1, g, t, wi * (NCH / 2) + p, fr[p]);
            // the stage is free again once every warp holds its share
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
            for (int p = 0; p < NCH / 2; ++p) compute_group(fr[p], xb[p], acc0, acc1);
        }
        float *rb = red + (size_t)(j & 1) * kCW * 2 * 16 * Tc;
        put_partials(rb, Tc, warp, g, t, acc0, acc1);
        named_sync_consumers();
        if ((lane & 1) == 0) {   // readers spread over the warps: (row, token) = r % 32, r / 32
            const int r = warp + kCW * (lane >> 1), row = r & 31, col = r >> 5;
            if (col < T)
                __stcg(a.ybuf + ((size_t)d * kMaxT + col) * H + m0 + row,
                       sum_partials(rb, Tc, row >> 4, row & 15, col));
        }
    }
    // Combine: once every expert's slice of a 32-row tile is in, the CTA
    // whose unit completed it sums the slices in expert order, undoes the
    // prescale and writes bf16; the order of the sum does not depend on
    // timing.
    __threadfence();
    named_sync_consumers();
    for (int j = tid; j < n_mine; j += 32 * kCW) {
        const int tile = (u0 + j) % tiles;
        if (atomicAdd(a.counters + tile, 1) == tb.D - 1) last_tiles[atomicAdd(&n_last, 1)] = tile;
    }
    named_sync_consumers();
    if (n_last > 0) {
        __threadfence();
        for (int idx = tid; idx < n_last * 32 * T; idx += 32 * kCW) {
            const int row = idx & 31, col = (idx >> 5) % T, m0 = last_tiles[(idx >> 5) / T] * 32;
            float sum = 0.f;
            for (int dd = 0; dd < tb.D; ++dd) sum += __ldcg(a.ybuf + ((size_t)dd * kMaxT + col) * H + m0 + row);
            __nv_bfloat16 o = __float2bfloat16_rn(sum * tok_inv[col]);
            a.out[(size_t)col * H + m0 + row] = *reinterpret_cast<uint16_t *>(&o);
        }
        for (int li = tid; li < n_last; li += 32 * kCW) a.counters[last_tiles[li]] = 0;
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

// Stages and chunks per stage (cps, a divisor of the unit's nch chunks) for
// a kernel whose other shared memory takes `fixed` bytes: the largest pieces
// that still leave three stages, else one chunk per stage.
struct StagePlan {
    int S, cps;
};
StagePlan plan_stages(int nch, size_t fixed) {
    for (int cps = nch; cps >= 1; cps /= 2) {
        long long s = ((long long)kMaxDynSmem - (long long)fixed) / (long long)piece_bytes(cps);
        if (s > kMaxStages) s = kMaxStages;
        if (s >= 3 || cps == 1) return {(int)(s < 0 ? 0 : s), cps};
    }
    return {0, 1};
}
StagePlan gu_plan(int T, int H) { return plan_stages(H / kKC, gu_bytes(0, 1, T, H)); }
StagePlan dn_plan(int T, int I) { return plan_stages(I / kKC, dn_bytes(0, 1, T, I)); }

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
    const StagePlan gp = gu_plan(T, H);
    ga.n_stages = gp.S;
    ga.cps = gp.cps;
    L.count_launches(2);
    if (ev) record_phase(ev[1], s);   // routing is fused into both kernels' prologues
    cudaError_t e = launch_ex(dec_gateup_mx_kernel<NCU>, dim3(grid), dim3(kWSThreads),
                              gu_bytes(ga.n_stages, ga.cps, T, H), s, false, ga);
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
    const StagePlan dp = dn_plan(T, I);
    da.n_stages = dp.S;
    da.cps = dp.cps;
    // programmatic dependent launch: the down kernel's producer streams
    // weights while the gate/up kernel drains; its consumers wait for that
    // grid before reading h.  Not with phase events between the launches.
    e = launch_ex(dec_down_mx_kernel<NCD>, dim3(grid), dim3(kWSThreads), dn_bytes(da.n_stages, da.cps, T, I), s, ev == nullptr,
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
    for (int tt = 1; tt <= kMaxT; ++tt)
        if (gu_plan(tt, d.hidden).S < 2 || dn_plan(tt, d.inter).S < 2) return false;
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
