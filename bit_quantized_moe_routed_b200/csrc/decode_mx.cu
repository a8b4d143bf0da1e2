// decode_mx.cu -- MXFP4 routed-expert FFN at decode sizes (1..8 tokens,
// bf16 activations): a grouped GEMV that streams each selected expert's
// packed codes from HBM once, the whole step in one kernel launch.
//
// Layer: out[t] = sum_s w[t,s] W_down,e (silu(W_gate,e x_t) * (W_up,e x_t))
// ("MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture notes":
// top-8 of 256 routed experts, MXFP4 experts with one E8M0 exponent per 32
// values; "Recipe": expert intermediates stay in a type with f32's range).
//
// One cooperative launch, one CTA per SM, all co-resident: phase 1 computes
// h for the gate/up units, phase 2 the down units, phase 3 the combine; two
// grid barriers (bounded waits) separate them.  The route table is built
// once per CTA.  A gate/up unit is one expert's 16 gate + 16 up rows over
// the full K, a down unit 32 down rows; each CTA takes a contiguous,
// balanced range of units in each phase.  The 8 consumer warps form one
// group per 1024-column chunk of K, so every chunk of a unit is in compute
// at once; inside a group each warp takes a share of the chunk's 32-weight
// block columns for both halves (gate and up, or the two 16-row down
// tiles), i.e. two independent accumulator chains.  A warp reads the
// fragments of its next group while it computes the current one.  Per unit
// the warps hand their partial fragments to two epilogue warps through a
// two-slot ring (full/empty mbarriers), which sum them (SwiGLU and h in
// phase 1, the expert's f32 output slice in phase 2), so the consumers
// never wait for one another.  Eight consumer warps keep every register a
// warp needs (up to 161, no spills).
//
// Memory: the device layout (MxGeom) keeps each (16-row tile, 1024-column
// chunk) block contiguous, so a producer warp streams a chunk of a unit as
// two 8.7 KB bulk copies (TMA) into a ring of shared-memory stages with
// full/empty mbarriers.  The ring serves both weight phases (a piece is the
// same pair of blocks in both), and the producer runs on from the last
// gate/up piece into the down pieces: the down weights stream in while
// phase 1 drains and while the CTA waits at the barrier.  The activations
// arrive first, one bulk copy per token, issued before the routing is read.
// Bulk copies of several KB are what keep HBM busy; the layout also makes
// the fragment and scale reads bank-conflict free.
//
// Math: warp-level mma.sync.m16n8k16 (f16 in, f32 accumulate).  Each thread
// reads its A-fragment slice of four 32-weight blocks (bytes 4t..4t+3 of
// each block: one 16-byte word in the layout) and decodes it with
// cvt.rn.f16x2.e2m1x2 (exact).  Per block the two MMAs accumulate into a
// fresh fragment that is folded into the running f32 sum times the block's
// E8M0 scale (one packed f32x2 FMA per row pair), so the scale is applied
// exactly.  The B operand is f16 after a power-of-two prescale that puts the
// largest magnitude in [2^14, 2^15): per token for the activations, per
// (expert, token) column of w * h for the down projection.  f16 cannot
// overflow, and the scale is undone in f32.
//
// Combine: phase 2 writes each expert's contribution, prescale undone, to
// its own slice of a scratch buffer; after the second barrier every CTA sums
// the slices of its share of the outputs in expert order and writes bf16,
// so the result does not depend on timing.
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

constexpr int kCW = 8;    // consumer warps per CTA (at up to 153 registers: no spills)

// Barrier among the kCW consumer warps (id 1; the producer warp does not join).
__device__ __forceinline__ void named_sync_consumers() {
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kCW) : "memory");
}

// ---------------------------------------------------------------- staging

// Warp roles: kCW consumer warps, one producer warp that streams (tile,
// chunk) blocks into a ring of shared-memory stages, and epilogue warps
// that reduce the consumers' partial sums.
constexpr int kProducerWarp = kCW;
constexpr int kKC = 1024;                       // weights of K per chunk (the layout's chunk)
constexpr int kBlk = 16 * (kKC / 2 + kKC / 32); // one (16-row tile, chunk) block of the device layout
// A stage holds one piece: cps consecutive chunks of a unit, both halves
// (gate and up tile, or the two down tiles): [half 0: cps blocks][half 1:
// cps blocks], each half one contiguous run of the device layout.
__host__ __device__ inline size_t piece_bytes(int cps) { return 2 * (size_t)cps * kBlk; }
constexpr int kMaxStages = 12;
constexpr int kMaxDynSmem = 232448 - 5120;      // leave room for static shared memory (4.3 KB in the down kernel)

// Shared-memory address of this thread's fragment word (bytes 4t..4t+3 of
// the four blocks of K-group grp) of staged row r (0..15) of a block.
__device__ __forceinline__ const uint8_t *frag_ptr(const uint8_t *blk, int r, int grp, int t) {
    return blk + (size_t)r * (kKC / 2) + ((grp ^ (r & 1)) * 64) + 16 * t;
}
// ... and of the scale word (four blocks) of row r, K-group grp.
__device__ __forceinline__ const uint8_t *scale_ptr(const uint8_t *blk, int r, int grp) {
    return blk + 16 * (kKC / 2) + grp * 64 + r * 4;
}

// This CTA's contiguous share [beg, end) of n units (n * gridDim.x < 2^32).
__device__ __forceinline__ void my_range(int n, int &beg, int &end) {
    beg = (int)(((unsigned)n * blockIdx.x) / gridDim.x);
    end = (int)(((unsigned)n * (blockIdx.x + 1)) / gridDim.x);
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
// n / d and n % d for 0 <= n < 2^16 and 2 <= d < 2^16 with one
// multiply-high, m = ceil(2^32 / d) (the error n (m d - 2^32) / 2^32 stays
// below one part in d): integer division by a runtime value would take
// the conversion pipe, which the weight decode keeps busy.
struct FastDiv {
    uint32_t d, m;
    __device__ __forceinline__ uint32_t div(uint32_t n) const { return __umulhi(n, m); }
};
inline FastDiv make_fastdiv(uint32_t d) { return {d, (uint32_t)((0x100000000ull + d - 1) / d)}; }

template <typename BlockOf>
__device__ __forceinline__ void produce(uint8_t *stages, uint64_t *full, uint64_t *empty, FastDiv S, int cps,
                                        int n_pieces, volatile int *abort, long long limit, volatile int *issued,
                                        BlockOf block_of) {
    const int lane = threadIdx.x & 31, i = lane >> 1, half = lane & 1;
    const int G = min((int)S.d, max(1, 4 / cps));
    const uint32_t half_bytes = (uint32_t)cps * kBlk;
    // every weight byte is read once per call
    const uint64_t policy = l2_evict_first_policy();
    int n_issued = 0;
    for (int p0 = 0; p0 < n_pieces; p0 += G) {
        const int p = p0 + i;
        const bool mine = i < G && p < n_pieces;
        const uint32_t rnd = S.div((uint32_t)p);
        const int s = mine ? p - (int)(rnd * S.d) : 0;
        bool ok = true;
        if (mine && half == 0 && rnd > 0) ok = mbar_wait_abort(&empty[s], (rnd - 1) & 1u, abort, limit);
        // once any role of the CTA has given up, issue nothing more
        if (__any_sync(0xffffffffu, !ok || *abort)) break;
        if (mine && half == 0) mbar_arrive_expect_tx(&full[s], 2u * half_bytes);
        __syncwarp();
        if (mine) {
            const uint8_t *b0, *b1;
            block_of(p, b0, b1);
            bulk_g2s_hint(stages + (size_t)s * piece_bytes(cps) + half * half_bytes, half ? b1 : b0, half_bytes, &full[s],
                          policy);
        }
        __syncwarp();
        n_issued = min(p0 + G, n_pieces);
        if (lane == 0) {
            __threadfence_block();
            *issued = n_issued;
        }
    }
    // Before the CTA exits, wait for the copies this warp issued and that may
    // still be in flight: the last S pieces (piece p - S was consumed, so
    // landed, before piece p reused its stage).  The limit is the fixed drain
    // limit, whatever happened to the other waits.
    if (lane == 0)
        for (int p = max(0, n_issued - (int)S.d); p < n_issued; ++p) {
            const uint32_t rnd = S.div((uint32_t)p);
            if (!mbar_wait_bounded(&full[p - (int)(rnd * S.d)], rnd & 1u, kDrainCycles)) *abort = 1;
        }
    __syncwarp();
}

// Consumer: wait until piece p is issued, then for its data.  False when it
// gave up (limit reached, or another role gave up first).
__device__ __forceinline__ bool wait_piece(uint64_t *full, FastDiv S, int p, volatile int *issued,
                                           volatile int *abort, long long limit) {
    if (*issued <= p) {
        const long long t0 = clock64();
        while (*issued <= p) {
            if (*abort) return false;
            if (clock64() - t0 > limit) {
                *abort = 1;
                return false;
            }
            __nanosleep(32);
        }
    }
    const uint32_t rnd = S.div((uint32_t)p);
    return mbar_wait_abort(&full[p - (int)(rnd * S.d)], rnd & 1u, abort, limit);
}

// Chunk q of every unit is computed by the 16/NCH warps [q*16/NCH, ...): a
// chunk is 16 pieces (8 K-groups x 2 halves: gate/up blocks, or the two
// down tiles) and each of those warps takes NCH of them, K-groups
// (i*NCH/2 ...) of both halves, so NCH chunks are in compute at once and
// each warp runs two independent accumulator chains.  The partial
// fragments go to red[slot][warp][half][row][column] (two slots, handed to
// the epilogue warps) and are summed in warp order.  A unit has at most
// Tc = min(T, 8) columns, so only those are kept.
__host__ __device__ inline int red_cols(int T) { return T < kMaxT ? T : kMaxT; }
// Partial-sum slots between the consumer warps and the epilogue warps.
constexpr int kRedSlots = 2;
constexpr int kEpiWarps = 2;
// red: [slot][consumer warp][half][16 rows][Tc columns] f32
__host__ __device__ inline size_t red_bytes(int T) {
    return (size_t)kRedSlots * kCW * 2 * 16 * red_cols(T) * sizeof(float);
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

// ---------------------------------------------------------------- units

constexpr int kGUThreads = 32 * (kCW + 1 + kEpiWarps);
constexpr int kEpiWarp0 = kCW + 1;

// Unit i -> (expert slot d, column chunk, 16-row tile): an expert's routes
// are taken Tc = min(T, 8) columns per pass (the width of the partial-sum
// slots; more routes than tokens only when a token lists an expert twice).  A CTA keeps its own range of
// units as packed words: d | tile << 6 | first column << 15 | columns << 22.
struct GUItems {
    int n;
    int beg[kMaxR + 1];
};
constexpr int kMaxUnits = 128;   // units of one CTA (checked on the host)
__device__ __forceinline__ int unit_d(uint32_t u) { return (int)(u & 63u); }
__device__ __forceinline__ int unit_tile(uint32_t u) { return (int)((u >> 6) & 511u); }
__device__ __forceinline__ int unit_cb(uint32_t u) { return (int)((u >> 15) & 127u); }
__device__ __forceinline__ int unit_ncol(uint32_t u) { return (int)(u >> 22); }

// Staged (expert, token) B columns per CTA.  A CTA's contiguous range of
// units is no longer than one expert's tiles when the grid has at least as
// many CTAs as there are routed experts, so it touches at most two experts:
// at most 2T columns.
constexpr int kMaxBSlots = 16;
constexpr int kMaxTiles = 128;   // H / 32 for H <= 4096
__host__ __device__ inline int dn_slots(int T) { return 2 * T < kMaxBSlots ? 2 * T : kMaxBSlots; }

// ---------------------------------------------------------------- one launch

// The whole decode step as one cooperative launch (one CTA per SM, all
// co-resident): phase 1 the gate/up units, phase 2 the down units, phase 3
// the combine, separated by two grid barriers.  One ring of stages serves
// both weight phases (a piece is the same pair of blocks of a chunk in
// both), and the producer runs on from the last gate/up piece into the down
// pieces, so the down weights stream in while gate/up drains and while the
// CTA waits at the barrier; the route table is built once.  The region of
// the staged activations holds the down B columns once phase 1 is over.

// Grid barrier: bar[0] counts arrivals, bar[1] is a generation number that
// the last arrival advances after it resets the count.  A CTA reads the
// generation once before its first arrival (gen0) and has passed barrier b
// (1 or 2) once the generation is gen0 + b.  Each CTA arrives once per
// barrier, and at barrier 2 only after it passed barrier 1, so an arrival
// is never counted at the wrong barrier.
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ int atom_add_acq_rel_gpu(int *p, int v) {
    int old;
    asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void red_add_release_gpu(int *p, int v) {
    asm volatile("red.add.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// The arrival releases what this thread (and, through the CTA barrier before
// it, its CTA) wrote; the last arrival acquires every other arrival's
// release, resets the count and releases the new generation.
__device__ __forceinline__ void grid_arrive(int *bar) {
    if (atom_add_acq_rel_gpu(bar, 1) == (int)gridDim.x - 1) {
        // every CTA has arrived and none touches the count again before the
        // generation moves on: a plain store resets it, the release orders it
        asm volatile("st.relaxed.gpu.global.s32 [%0], 0;" ::"l"(bar) : "memory");
        red_add_release_gpu(bar + 1, 1);
    }
}
__device__ __forceinline__ bool grid_wait(const int *bar, int gen0, int b, volatile int *abort, long long limit) {
    const long long t0 = clock64();
    while (ld_acquire_gpu(bar + 1) - gen0 < b) {
        if (*abort) return false;
        if (clock64() - t0 > limit) {
            *abort = 1;
            return false;
        }
        __nanosleep(20);
    }
    return true;
}

// Barrier among the epilogue warps (id 2).
__device__ __forceinline__ void named_sync_epilogue() {
    asm volatile("bar.sync 2, %0;" ::"r"(32 * kEpiWarps) : "memory");
}

// The consumer warps' side of one weight phase: n units of NCH chunks each,
// the phase's pieces numbered from p0 in the ring and its partial-sum
// hand-offs from r0.  brow(j, live) is this lane's B row for unit j (f16,
// offset by 8t).  Each warp releases a stage with NCH arrivals, so a piece
// takes kCW * cps arrivals in either phase.  False if a wait gave up.
template <int NCH, typename BRow>
__device__ __forceinline__ bool consume_phase(const uint8_t *stages, uint64_t *full, uint64_t *empty,
                                              uint64_t *red_full, uint64_t *red_empty, float *red, int Tc,
                                              FastDiv S, int cps, int n, int p0, int r0, volatile int *issued,
                                              volatile int *abort, long long lim, BRow brow) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    constexpr int WPC = kCW / NCH;   // warps per chunk
    constexpr int NG = 8 / WPC;      // K-groups of this warp per unit
    const int q = warp / WPC, wi = warp % WPC;
    const int lcps = cps == 4 ? 2 : (cps == 2 ? 1 : 0);
    bool ok = true;
    const uint8_t *st0 = stages, *st1 = stages;
    int s_cur = 0;
    auto open_unit = [&](int j, const uint8_t *&b0, const uint8_t *&b1, int &s) {
        const int c = j * NCH + q, pc = p0 + (c >> lcps);
        if (!wait_piece(full, S, pc, issued, abort, lim)) ok = false;
        s = pc - (int)(S.div((uint32_t)pc) * S.d);
        b0 = stages + (size_t)s * piece_bytes(cps) + (size_t)(c & (cps - 1)) * kBlk;
        b1 = b0 + (size_t)cps * kBlk;
    };
    GroupFrags cur;
    if (n > 0) {
        open_unit(0, st0, st1, s_cur);
        load_group(st0, st1, g, t, wi * NG, cur);
    }
    for (int j = 0; j < n && ok; ++j) {
        bool live;
        const uint16_t *row = brow(j, live);
        float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < NG; ++p) {
            const int gp = wi * NG + p;
            const uint8_t *n0 = st0, *n1 = st1;
            int ns = s_cur;
            GroupFrags nxt;
            if (p + 1 < NG) {
                load_group(st0, st1, g, t, gp + 1, nxt);
            } else {
                // the unit's groups are all in registers: release its stage
                // before waiting for the next unit's piece
                __syncwarp();
                if (lane == 0) mbar_arrive_cnt(&empty[s_cur], NCH);
                if (j + 1 < n) {
                    open_unit(j + 1, n0, n1, ns);
                    load_group(n0, n1, g, t, wi * NG, nxt);
                }
            }
            const uint16_t *xq = row + q * kKC + gp * 128;
            uint4 xb[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) xb[jj] = live ? lds128(xq + jj * 32) : make_uint4(0u, 0u, 0u, 0u);
            compute_group(cur, xb, a0, a1);
            cur = nxt;
            st0 = n0;
            st1 = n1;
            s_cur = ns;
        }
        const int jj = r0 + j, slot = jj % kRedSlots;
        if (jj >= kRedSlots && !mbar_wait_abort(&red_empty[slot], (uint32_t)((jj / kRedSlots - 1) & 1), abort, lim))
            ok = false;
        put_partials(red + (size_t)slot * kCW * 2 * 16 * Tc, Tc, warp, g, t, a0, a1);
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_full[slot]);
    }
    return ok;
}

struct FusedArgs {
    const uint8_t *codes_g, *codes_u, *codes_d;   // the three projections in the device layout (MxGeom)
    const uint16_t *x;                            // bf16 [T][H]
    const int32_t *ids;                           // [T][k]
    const float *topk_w;                          // [T][k]
    float *h;                                     // [T*k][I] f32, by route id
    float *ybuf;                                  // [kMaxR expert slots][kMaxT][H]
    int *gbar;                                    // grid barrier words (count, generation)
    uint16_t *out;                                // bf16 [T][H]
    uint32_t *status;
    long long wait_cycles;                        // limit of every wait but the final drains
    FastDiv S;                                    // stages
    int T, k, E, H, I, cps;
};

// Shared memory: [stages][activations | down B columns][partial sums].
__host__ __device__ inline size_t fu_xb_bytes(int T, int H, int I) {
    const size_t xr = sizeof(uint16_t) * (size_t)T * (H + kXPad);
    const size_t br = sizeof(uint16_t) * (size_t)dn_slots(T) * (I + kXPad);
    return xr > br ? xr : br;
}
__host__ __device__ inline size_t fu_red_off(int n_stages, int cps, int T, int H, int I) {
    return (size_t)n_stages * piece_bytes(cps) + fu_xb_bytes(T, H, I);
}
__host__ __device__ inline size_t fu_bytes(int n_stages, int cps, int T, int H, int I) {
    return fu_red_off(n_stages, cps, T, H, I) + red_bytes(T);
}

template <int NCU, int NCD>   // K chunks of a gate/up unit (H / kKC) and of a down unit (I / kKC)
__global__ void __launch_bounds__(kGUThreads, 1) dec_fused_mx_kernel(FusedArgs a) {
    static_assert(kCW % NCU == 0 && 8 % (kCW / NCU) == 0 && kCW % NCD == 0 && 8 % (kCW / NCD) == 0,
                  "warps per chunk must divide the 8 K-groups of a chunk");
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ GUItems items;
    __shared__ uint32_t units[kMaxUnits];
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages], xbar, red_full[kRedSlots],
        red_empty[kRedSlots];
    __shared__ int issued;                 // pieces issued by the producer (see produce)
    __shared__ volatile int abort_flag;    // set by the first role that gives up on a wait
    __shared__ int n_gu, unit0, gen0;
    __shared__ float xinv[kMaxT];
    __shared__ int slot_of[2][kMaxT];      // (expert slot - d_lo, token) -> staged B column, -1 none
    __shared__ int slot_d[kMaxBSlots], slot_t[kMaxBSlots];
    __shared__ unsigned slot_max[kMaxBSlots];
    __shared__ float slot_scale[kMaxBSlots], slot_inv[kMaxBSlots];
    __shared__ int n_slots;
    const int H = a.H, I = a.I, T = a.T, k = a.k, S = (int)a.S.d, cps = a.cps, Tc = red_cols(a.T);
    uint8_t *stages = smem_raw;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem_raw + (size_t)S * piece_bytes(cps));   // phase 1
    uint16_t *bs = xs;                                                                       // phase 2
    float *red = reinterpret_cast<float *>(smem_raw + fu_red_off(S, cps, T, H, I));
    const int xs_stride = H + kXPad, bs_stride = I + kXPad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int gu_tiles = I / 16, dn_tiles = H / 32;
    const MxGeom ggeo(I, H), dgeo(H, I);

    // the activations do not depend on the routing: the producer warp
    // starts their copies first thing (one bulk copy per token row)
    if (warp == kProducerWarp) {
        if (lane == 0) {
            mbar_init(&xbar, 1);
            mbar_fence_init();
            mbar_arrive_expect_tx(&xbar, (uint32_t)(T * H * 2));
        }
        __syncwarp();
        if (lane < T) bulk_g2s(xs + (size_t)lane * xs_stride, a.x + (size_t)lane * H, H * 2, &xbar);
    }
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCW * cps);
        }
        for (int r = 0; r < kRedSlots; ++r) {
            mbar_init(&red_full[r], kCW);
            mbar_init(&red_empty[r], kEpiWarps);
        }
        mbar_fence_init();
        issued = 0;
        abort_flag = 0;
    }
    if (warp == kEpiWarp0 && lane == 0) gen0 = ld_acquire_gpu(a.gbar + 1);   // before this CTA's first arrival
    if (tid < kMaxBSlots) slot_max[tid] = 0u;
    const long long lim = a.wait_cycles;
    if (warp == 0) {
        build_route_table(tb, a.ids, a.topk_w, T * k, k, a.E, a.status, blockIdx.x == 0);
        __syncwarp();
        // units per expert slot (lane d and d + 32), exclusive prefix sum over the warp
        const int D = tb.D;
        int c0 = 0, c1 = 0;
        if (lane < D) c0 = ((tb.col_beg[lane + 1] - tb.col_beg[lane] + Tc - 1) / Tc) * gu_tiles;
        if (lane + 32 < D) c1 = ((tb.col_beg[lane + 33] - tb.col_beg[lane + 32] + Tc - 1) / Tc) * gu_tiles;
        int s0 = c0, s1 = c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v0 = __shfl_up_sync(0xffffffffu, s0, o), v1 = __shfl_up_sync(0xffffffffu, s1, o);
            if (lane >= o) {
                s0 += v0;
                s1 += v1;
            }
        }
        const int tot0 = __shfl_sync(0xffffffffu, s0, 31);
        if (lane < D) items.beg[lane] = s0 - c0;
        if (lane + 32 < D) items.beg[lane + 32] = tot0 + s1 - c1;
        const int n = tot0 + __shfl_sync(0xffffffffu, s1, 31);
        if (lane == 0) {
            items.beg[D] = n;
            items.n = n;
            int i0, i1;
            my_range(n, i0, i1);
            unit0 = i0;
            n_gu = min(i1 - i0, kMaxUnits);
        }
        __syncwarp();
        // this CTA's gate/up units, one per lane (binary search for the
        // expert slot: beg[d] <= i < beg[d + 1])
        const int ltiles = 31 - __clz(gu_tiles);
        for (int j = lane; j < n_gu; j += 32) {
            const int i = unit0 + j;
            int lo = 0, hi = D - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (items.beg[mid] <= i) lo = mid;
                else hi = mid - 1;
            }
            const int d = lo, rel = i - items.beg[d], pass = rel >> ltiles, tile = rel & (gu_tiles - 1);
            const int cb = tb.col_beg[d] + pass * Tc, ncol = min(Tc, tb.col_beg[d + 1] - cb);
            units[j] = (uint32_t)d | ((uint32_t)tile << 6) | ((uint32_t)cb << 15) | ((uint32_t)ncol << 22);
        }
    }
    __syncthreads();
    // down units: unit u -> expert slot u / dn_tiles, 32-row tile u % dn_tiles
    const int n_gu_units = n_gu;
    const int ldt = 31 - __clz(dn_tiles);
    int u0, u1;
    my_range(tb.D * dn_tiles, u0, u1);
    const int n_dn = u1 - u0;
    const int d_lo = n_dn > 0 ? u0 >> ldt : 0;
    const int n_gu_p = n_gu_units * NCU / cps;   // pieces of phase 1

    if (warp == kProducerWarp) {
        produce(stages, full, empty, a.S, cps, n_gu_p + n_dn * NCD / cps, &abort_flag, lim, &issued,
                [&](int p, const uint8_t *&b0, const uint8_t *&b1) {
                    if (p < n_gu_p) {
                        const int c = p * cps;
                        const uint32_t u = units[c / NCU];
                        const size_t off = (size_t)tb.expert[unit_d(u)] * ggeo.expert_bytes() +
                                           ggeo.block_off(unit_tile(u), c % NCU);
                        b0 = a.codes_g + off;
                        b1 = a.codes_u + off;
                    } else {
                        const int c = (p - n_gu_p) * cps;
                        const int u = u0 + c / NCD, d = u >> ldt, t32 = u & (dn_tiles - 1), qq = c % NCD;
                        const uint8_t *eb = a.codes_d + (size_t)tb.expert[d] * dgeo.expert_bytes();
                        b0 = eb + dgeo.block_off(2 * t32, qq);
                        b1 = eb + dgeo.block_off(2 * t32 + 1, qq);
                    }
                });
        return;
    }

    if (warp >= kEpiWarp0) {
        const int e = warp - kEpiWarp0;
        bool ok = true;
        // phase 1: sum the consumers' partial fragments of a unit, SwiGLU, h
        for (int j = 0; j < n_gu_units && ok; ++j) {
            const int slot = j % kRedSlots;
            if (!mbar_wait_abort(&red_full[slot], (uint32_t)((j / kRedSlots) & 1), &abort_flag, lim)) {
                ok = false;
                break;
            }
            const uint32_t u = units[j];
            const int cb = unit_cb(u), ncol = unit_ncol(u), n0 = unit_tile(u) * 16;
            const float *rb = red + (size_t)slot * kCW * 2 * 16 * Tc;
            for (int idx = lane + 32 * e; idx < 16 * ncol; idx += 32 * kEpiWarps) {
                const int row = idx & 15, col = idx >> 4;
                const float gs = sum_partials(rb, Tc, 0, row, col), us = sum_partials(rb, Tc, 1, row, col);
                const int route = tb.route[cb + col];
                const float inv = xinv[tb.tok[route]];
                a.h[(size_t)route * I + n0 + row] = silu_f32(gs * inv) * (us * inv);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_empty[slot]);
        }
        // this CTA's share of h is written: one arrival at barrier 1
        named_sync_epilogue();
        if (e == 0 && lane == 0 && ok && !abort_flag) grid_arrive(a.gbar);
        // phase 2: undo the column prescale and store the expert's f32 slice
        for (int j = 0; j < n_dn && ok; ++j) {
            const int jj = n_gu_units + j, slot = jj % kRedSlots;
            if (!mbar_wait_abort(&red_full[slot], (uint32_t)((jj / kRedSlots) & 1), &abort_flag, lim)) {
                ok = false;
                break;
            }
            const int u = u0 + j, d = u >> ldt, m0 = (u & (dn_tiles - 1)) * 32;
            const float *rb = red + (size_t)slot * kCW * 2 * 16 * Tc;
            for (int idx = lane + 32 * e; idx < 32 * T; idx += 32 * kEpiWarps) {
                const int row = idx & 31, col = idx >> 5;
                const int sl = slot_of[d - d_lo][col];
                const float v = sl >= 0 ? sum_partials(rb, Tc, row >> 4, row & 15, col) * slot_inv[sl] : 0.f;
                __stcg(a.ybuf + ((size_t)d * kMaxT + col) * H + m0 + row, v);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_empty[slot]);
        }
        // the slices are written: one arrival at barrier 2, after barrier 1
        // (which a CTA with down units has passed before its first one)
        named_sync_epilogue();
        if (e == 0 && lane == 0 && ok && !abort_flag && (n_dn > 0 || grid_wait(a.gbar, gen0, 1, &abort_flag, lim)))
            grid_arrive(a.gbar);
        __syncwarp();
        if (abort_flag && lane == 0) atomicOr(a.status, FLAG_TIMEOUT);
        return;
    }

    // ---- consumers.  The B columns of this CTA's down experts (the
    // (expert, token) pairs with routes), while the weights stream in
    if (tid == 0) {
        int ns = 0;
        const int d_hi = n_dn > 0 ? (u1 - 1) >> ldt : -1;
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
    // x -> f16 in place, with a per-token power-of-two prescale (warp w <-> token w)
    bool ok = mbar_wait_abort(&xbar, 0, &abort_flag, lim);
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

    // phase 1
    if (ok)
        ok = consume_phase<NCU>(stages, full, empty, red_full, red_empty, red, Tc, a.S, cps, n_gu_units, 0, 0,
                                &issued, &abort_flag, lim, [&](int j, bool &live) {
                                    const uint32_t u = units[j];
                                    live = g < unit_ncol(u);
                                    const int tok = live ? tb.tok[tb.route[unit_cb(u) + g]] : 0;
                                    return xs + (size_t)tok * xs_stride + 8 * t;
                                });
    // every consumer is done with the activations (their region takes the B
    // columns next), and every CTA's h is written
    named_sync_consumers();
    if (tid == 0 && ok && !abort_flag) grid_wait(a.gbar, gen0, 1, &abort_flag, lim);
    named_sync_consumers();
    ok = ok && !abort_flag;

    // B column sl = (sum of w_r h_r over the token's routes to the expert,
    // in f32) * 2^s_sl in f16, the power of two putting the column's largest
    // magnitude in [2^14, 2^15): f16 cannot overflow and the epilogue undoes
    // the scale exactly.  Pass 1 finds the maxima with the values kept in
    // registers (two 8-value pieces per thread; larger layers build them
    // again in pass 2).
    const int n_idx = ok ? n_slots * (I / 8) : 0;
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
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(vv[i]));
        if (m > 0.f) atomicMax(&slot_max[sl], __float_as_uint(isfinite(m) ? m : 3.0e38f));
    };
    float v[2][8];
#pragma unroll
    for (int it = 0; it < 2; ++it)
        if (tid + it * 32 * kCW < n_idx) col8(tid + it * 32 * kCW, v[it]);
    for (int idx = tid + 2 * 32 * kCW; idx < n_idx; idx += 32 * kCW) {
        float vv[8];
        col8(idx, vv);
    }
    named_sync_consumers();
    if (tid < n_slots) {
        const int sc = prescale_exp(__uint_as_float(slot_max[tid]));
        slot_scale[tid] = exp2i(sc);
        slot_inv[tid] = exp2i(-sc);
    }
    named_sync_consumers();
    auto put_b = [&](int idx, const float *vv) {
        const int sl = idx / (I / 8), k8 = (idx % (I / 8)) * 8;
        const float rs = slot_scale[sl];
        __half2 p0 = __floats2half2_rn(rs * vv[0], rs * vv[1]), p1 = __floats2half2_rn(rs * vv[2], rs * vv[3]);
        __half2 p2 = __floats2half2_rn(rs * vv[4], rs * vv[5]), p3 = __floats2half2_rn(rs * vv[6], rs * vv[7]);
        *reinterpret_cast<uint4 *>(bs + (size_t)sl * bs_stride + k8) =
            make_uint4(*reinterpret_cast<uint32_t *>(&p0), *reinterpret_cast<uint32_t *>(&p1),
                       *reinterpret_cast<uint32_t *>(&p2), *reinterpret_cast<uint32_t *>(&p3));
    };
#pragma unroll
    for (int it = 0; it < 2; ++it)
        if (tid + it * 32 * kCW < n_idx) put_b(tid + it * 32 * kCW, v[it]);
    for (int idx = tid + 2 * 32 * kCW; idx < n_idx; idx += 32 * kCW) {
        float vv[8];
        col8(idx, vv);
        put_b(idx, vv);
    }
    named_sync_consumers();

    // phase 2
    if (ok)
        ok = consume_phase<NCD>(stages, full, empty, red_full, red_empty, red, Tc, a.S, cps, n_dn, n_gu_p,
                                n_gu_units, &issued, &abort_flag, lim, [&](int j, bool &live) {
                                    const int d = (u0 + j) >> ldt;
                                    const int sl = g < T ? slot_of[d - d_lo][g] : -1;   // column g = token g
                                    live = sl >= 0;
                                    return bs + (size_t)(live ? sl : 0) * bs_stride + 8 * t;
                                });

    // phase 3, after every CTA's slices are written: this CTA's share of
    // the outputs, the experts' slices summed in expert order (16 loads in
    // flight at a time), one bf16 rounding
    named_sync_consumers();
    if (tid == 0 && ok && !abort_flag) grid_wait(a.gbar, gen0, 2, &abort_flag, lim);
    named_sync_consumers();
    if (ok && !abort_flag) {
        const int D = tb.D;
        int o0, o1;
        my_range(T * H, o0, o1);
        for (int i = o0 + tid; i < o1; i += 32 * kCW) {
            const float *yb = a.ybuf + i;   // element i = col * H + m of slice d at d * kMaxT * H
            float sum = 0.f;
            for (int d0 = 0; d0 < D; d0 += 16) {
                float vv[16];
#pragma unroll
                for (int qq = 0; qq < 16; ++qq) vv[qq] = d0 + qq < D ? __ldcg(yb + (size_t)(d0 + qq) * kMaxT * H) : 0.f;
#pragma unroll
                for (int qq = 0; qq < 16; ++qq)
                    if (d0 + qq < D) sum += vv[qq];
            }
            __nv_bfloat16 o = __float2bfloat16_rn(sum);
            a.out[i] = *reinterpret_cast<uint16_t *>(&o);
        }
    } else {
        ok = false;
    }
    if ((!ok || abort_flag) && lane == 0) atomicOr(a.status, FLAG_TIMEOUT);
}

// Stages and chunks per stage (cps, a divisor of the unit's nch chunks) for
// a kernel whose other shared memory takes `fixed` bytes: of the choices
// with at least three stages, the one with the most bytes in flight
// (smaller pieces on a tie: the warps of a chunk start on it as soon as it
// has landed), else one chunk per stage.
struct StagePlan {
    int S, cps;
};
StagePlan plan_stages(int nch, size_t fixed) {
    StagePlan best{0, 1};
    long long best_bytes = -1;
    for (int cps = 1; cps <= nch; cps *= 2) {
        long long s = ((long long)kMaxDynSmem - (long long)fixed) / (long long)piece_bytes(cps);
        if (s > kMaxStages) s = kMaxStages;
        if (s < 3 && cps != 1) continue;
        const long long bytes = s * (long long)piece_bytes(cps);
        if (bytes > best_bytes) {
            best = {(int)(s < 0 ? 0 : s), cps};
            best_bytes = bytes;
        }
    }
    return best;
}
StagePlan fu_plan(int T, int H, int I) {
    return plan_stages(std::min(H, I) / kKC, fu_bytes(0, 1, T, H, I));
}

// The one-launch decode step: a cooperative launch (all CTAs co-resident,
// which the grid barriers need; the launch fails rather than hangs when they
// cannot be).
template <int NCU, int NCD>
cudaError_t run_fused(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                      cudaStream_t s, const cudaEvent_t *ev) {
    const int H = L.d.hidden, I = L.d.inter;
    static std::once_flag attr_once[64];
    static cudaError_t attr_err[64];
    const int dev = L.d.device;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(attr_once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(dec_fused_mx_kernel<NCU, NCD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kMaxDynSmem);
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
    FusedArgs fa;
    fa.codes_g = L.w.codes[MOEQ_GATE];
    fa.codes_u = L.w.codes[MOEQ_UP];
    fa.codes_d = L.w.codes[MOEQ_DOWN];
    fa.x = reinterpret_cast<const uint16_t *>(x);
    fa.ids = ids;
    fa.topk_w = topk_w;
    fa.h = L.h;
    fa.ybuf = L.dec_ybuf;
    fa.gbar = L.dec_counters;
    fa.out = reinterpret_cast<uint16_t *>(out);
    fa.status = L.status;
    fa.wait_cycles = L.wait_cycles;
    fa.T = T;
    fa.k = L.d.top_k;
    fa.E = L.d.n_experts;
    fa.H = H;
    fa.I = I;
    const StagePlan pl = fu_plan(T, H, I);
    fa.S = make_fastdiv((uint32_t)pl.S);
    fa.cps = pl.cps;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(L.sm_count);
    cfg.blockDim = dim3(kGUThreads);
    cfg.dynamicSmemBytes = fu_bytes(pl.S, pl.cps, T, H, I);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    L.count_launches(1);
    // routing, gate/up, down and the combine are one kernel: their phase
    // events are recorded back to back around it
    if (ev) record_phase(ev[1], s);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, dec_fused_mx_kernel<NCU, NCD>, fa);
    if (e != cudaSuccess) return e;
    if (ev) {
        record_phase(ev[2], s);
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
        if (fu_plan(tt, d.hidden, d.inter).S < 3) return false;
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
    if (H == 2048 && I == 2048) return run_fused<2, 2>(L, x, ids, topk_w, T, out, s, ev);
    if (H == 2048 && I == 4096) return run_fused<2, 4>(L, x, ids, topk_w, T, out, s, ev);
    if (H == 4096 && I == 2048) return run_fused<4, 2>(L, x, ids, topk_w, T, out, s, ev);
    if (H == 4096 && I == 4096) return run_fused<4, 4>(L, x, ids, topk_w, T, out, s, ev);
    return cudaErrorInvalidValue;
}

}  // namespace moeq
