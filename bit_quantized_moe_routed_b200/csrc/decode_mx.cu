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
// contiguous, balanced range of units.  The 8 consumer warps form one group
// per 1024-column chunk of K, so every chunk of a unit is in compute at
// once; inside a group each warp takes a share of the chunk's 32-weight
// block columns for both halves (gate and up, or the two 16-row down tiles),
// i.e. two independent accumulator chains.  A warp reads the fragments of
// its next group while it computes the current one.  Per unit the warps
// hand their partial fragments to two epilogue warps through a two-slot
// ring (full/empty mbarriers), which sum them (SwiGLU and h for gate/up),
// so the consumers never wait for one another.  (Four slots took shared
// memory from the stage ring and measured slower at T = 8.)  Eight consumer warps keep every register a warp
// needs (up to 153, no spills); sixteen did not fit without spilling.
//
// Memory: the device layout (MxGeom) keeps each (16-row tile, 1024-column
// chunk) block contiguous, so a producer warp streams a chunk of a unit as
// two 8.7 KB bulk copies (TMA) into a ring of shared-memory stages with
// full/empty mbarriers, unit by unit and chunk by chunk (one chunk per stage
// where the stage count allows it, so a chunk's warps start as soon as it
// lands); the activations
// arrive first, one bulk copy per token.  Bulk copies of several KB are what
// keep HBM busy; the layout also makes the fragment and scale reads
// bank-conflict free.  The gate/up kernel lets the down kernel launch as its
// CTAs finish (programmatic dependent launch): the down weights stream in
// while gate/up drains, and only the down consumers wait for h.  The down
// kernel does the same for the next gate/up launch, which waits for it
// before reading anything.
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
// Combine: the down kernel writes each expert's contribution, prescale
// undone, to its own slice of a scratch buffer; a third, small kernel (one
// output element per thread, launched as a programmatic dependent) sums the
// slices in expert order and writes bf16 out, so the result does not depend
// on timing and the sum is spread over the whole GPU.
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

// ---------------------------------------------------------------- gate/up

struct GateUpArgs {
    const uint8_t *codes_g, *codes_u;   // gate, up projections in the device layout (MxGeom)
    const uint16_t *x;                  // bf16 [T][H]
    const int32_t *ids;                 // [T][k]
    const float *topk_w;                // [T][k]
    float *h;                           // [T*k][I] f32, by route id
    uint32_t *status;
    long long wait_cycles;              // limit of every wait but the final drains
    FastDiv S;                          // stages
    int T, k, E, H, I, cps;
};

constexpr int kGUThreads = 32 * (kCW + 1 + kEpiWarps);
constexpr int kEpiWarp0 = kCW + 1;

__host__ __device__ inline size_t gu_xs_off(int n_stages, int cps) { return (size_t)n_stages * piece_bytes(cps); }
__host__ __device__ inline size_t gu_red_off(int n_stages, int cps, int T, int H) {
    return gu_xs_off(n_stages, cps) + sizeof(uint16_t) * (size_t)T * (H + kXPad);
}
__host__ __device__ inline size_t gu_bytes(int n_stages, int cps, int T, int H) {
    return gu_red_off(n_stages, cps, T, H) + red_bytes(T);
}

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

template <int NCH>   // K chunks per unit = H / kKC
__global__ void __launch_bounds__(kGUThreads, 1) dec_gateup_mx_kernel(GateUpArgs a) {
    static_assert(kCW % NCH == 0 && 8 % (kCW / NCH) == 0, "warps per chunk must divide the 8 K-groups of a chunk");
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ GUItems items;
    __shared__ uint32_t units[kMaxUnits];
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages], xbar, red_full[kRedSlots],
        red_empty[kRedSlots];
    __shared__ int issued;   // chunks issued by the producer (see produce)
    __shared__ volatile int abort_flag;   // set by the first role that gives up on a wait
    __shared__ int n_units, unit0;
    __shared__ float xinv[kMaxT];
    const int H = a.H, I = a.I, T = a.T, k = a.k, S = (int)a.S.d, cps = a.cps, Tc = red_cols(a.T);
    uint8_t *stages = smem_raw;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem_raw + gu_xs_off(S, cps));
    float *red = reinterpret_cast<float *>(smem_raw + gu_red_off(S, cps, T, H));
    const int xs_stride = H + kXPad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tiles = I / 16;
    const MxGeom geo(I, H);
    constexpr int WPC = kCW / NCH;   // warps per chunk
    const int lcps = cps == 4 ? 2 : (cps == 2 ? 1 : 0);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], WPC * cps);
        }
        mbar_init(&xbar, 1);
        for (int r = 0; r < kRedSlots; ++r) {
            mbar_init(&red_full[r], kCW);
            mbar_init(&red_empty[r], kEpiWarps);
        }
        mbar_fence_init();
        issued = 0;
        abort_flag = 0;
    }
    const long long lim = a.wait_cycles;
    // launched as a programmatic dependent of the previous kernel in the
    // stream: its outputs (these inputs, or h that kernel still reads) are
    // ready and free only after this wait; the dependents this kernel lets
    // launch below therefore see finished inputs as well
    pdl_wait_primary();
    if (warp == 0) {
        build_route_table(tb, a.ids, a.topk_w, T * k, k, a.E, a.status, blockIdx.x == 0);
        __syncwarp();
        if (lane == 0) {
            int n = 0;
            for (int d = 0; d < tb.D; ++d) {
                items.beg[d] = n;
                n += ((tb.col_beg[d + 1] - tb.col_beg[d] + Tc - 1) / Tc) * tiles;
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
            const int cb = tb.col_beg[d] + pass * Tc, ncol = min(Tc, tb.col_beg[d + 1] - cb);
            units[j] = (uint32_t)d | ((uint32_t)tile << 6) | ((uint32_t)cb << 15) | ((uint32_t)ncol << 22);
        }
    }
    __syncthreads();
    // the down kernel may take SMs as this grid's CTAs finish: it streams
    // its weights at once and reads h only after this grid completes
    pdl_launch_dependents();
    const int n_mine = n_units;

    if (warp == kProducerWarp) {
        // the activations first (one bulk copy per token row, into padded rows)
        if (lane == 0) mbar_arrive_expect_tx(&xbar, (uint32_t)(T * H * 2));
        __syncwarp();
        if (lane < T) bulk_g2s(xs + (size_t)lane * xs_stride, a.x + (size_t)lane * H, H * 2, &xbar);
        produce(stages, full, empty, a.S, cps, n_mine * NCH / cps, &abort_flag, lim, &issued,
                [&](int p, const uint8_t *&b0, const uint8_t *&b1) {
                    const int c = p * cps;
                    const uint32_t u = units[c / NCH];
                    const size_t off = (size_t)tb.expert[unit_d(u)] * geo.expert_bytes() +
                                       geo.block_off(unit_tile(u), c % NCH);
                    b0 = a.codes_g + off;
                    b1 = a.codes_u + off;
                });
        return;
    }

    if (warp >= kEpiWarp0) {
        // epilogue: sum the 16 warps' partial fragments of a unit, SwiGLU, h
        const int e = warp - kEpiWarp0;
        for (int j = 0; j < n_mine; ++j) {
            const int slot = j % kRedSlots;
            if (!mbar_wait_abort(&red_full[slot], (uint32_t)((j / kRedSlots) & 1), &abort_flag, lim)) break;
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
        __syncwarp();
        if (abort_flag && lane == 0) atomicOr(a.status, FLAG_TIMEOUT);
        return;
    }

    // ---- consumers: x -> f16 in place, with a per-token power-of-two
    // prescale (warp w <-> token w)
    bool timed_out = !mbar_wait_abort(&xbar, 0, &abort_flag, lim);
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

    // Each warp walks its groups of every unit one ahead: the fragments of
    // the next group (the next unit's first group at the end of a unit) are
    // read from shared memory while the current group is computed.  A unit's
    // stage is released once its last group is in registers, before the
    // warp waits for the next unit's piece.
    const int q = warp / WPC, wi = warp % WPC;   // this warp's chunk of every unit and its place in it
    constexpr int NG = 8 / WPC;                  // groups of this warp per unit (8 per chunk)
    const uint8_t *st0 = stages, *st1 = stages;
    int s_cur = 0;
    auto open_unit = [&](int j, const uint8_t *&b0, const uint8_t *&b1, int &s) {
        const int c = j * NCH + q, pc = c >> lcps;
        if (!wait_piece(full, a.S, pc, &issued, &abort_flag, lim)) timed_out = true;
        s = pc - (int)(a.S.div((uint32_t)pc) * a.S.d);
        // [gate blocks of the piece][up blocks of the piece]
        b0 = stages + (size_t)s * piece_bytes(cps) + (size_t)(c & (cps - 1)) * kBlk;
        b1 = b0 + (size_t)cps * kBlk;
    };
    GroupFrags cur;
    if (n_mine > 0) {
        open_unit(0, st0, st1, s_cur);
        load_group(st0, st1, g, t, wi * NG, cur);
    }
    for (int j = 0; j < n_mine && !timed_out; ++j) {
        const uint32_t u = units[j];
        const int cb = unit_cb(u), ncol = unit_ncol(u);
        const bool live = g < ncol;
        const int tok = live ? tb.tok[tb.route[cb + g]] : 0;
        const uint16_t *xrow = xs + (size_t)tok * xs_stride + 8 * t;
        float aG[4] = {0.f, 0.f, 0.f, 0.f}, aU[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < NG; ++p) {
            const int gp = wi * NG + p;
            const uint8_t *n0 = st0, *n1 = st1;
            int ns = s_cur;
            GroupFrags nxt;
            if (p + 1 < NG) {
                load_group(st0, st1, g, t, gp + 1, nxt);
            } else {
                // every group of this unit was read before the compute that
                // precedes this step: release the stage before waiting for
                // the next unit's piece (holding it could wait on itself)
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s_cur]);
                if (j + 1 < n_mine) {
                    open_unit(j + 1, n0, n1, ns);
                    load_group(n0, n1, g, t, wi * NG, nxt);
                }
            }
            const uint16_t *xq = xrow + (size_t)(q * (kKC / 32) + gp * 4) * 32;
            uint4 xb[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) xb[jj] = live ? lds128(xq + jj * 32) : make_uint4(0u, 0u, 0u, 0u);
            compute_group(cur, xb, aG, aU);
            cur = nxt;
            st0 = n0;
            st1 = n1;
            s_cur = ns;
        }
        // hand the partial fragments to the epilogue warps
        const int slot = j % kRedSlots;
        if (j >= kRedSlots && !mbar_wait_abort(&red_empty[slot], (uint32_t)((j / kRedSlots - 1) & 1), &abort_flag, lim))
            timed_out = true;
        put_partials(red + (size_t)slot * kCW * 2 * 16 * Tc, Tc, warp, g, t, aG, aU);
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_full[slot]);
    }
    if ((timed_out || abort_flag) && lane == 0) atomicOr(a.status, FLAG_TIMEOUT);
}

// ---------------------------------------------------------------- down

struct DownArgs {
    const uint8_t *codes;           // down projection in the device layout (MxGeom)
    const float *h;                 // [T*k][I]
    const int32_t *ids;
    const float *topk_w;
    float *ybuf;                    // [kMaxR expert slots][kMaxT][H]
    int *n_routed;                  // out: number of experts with routes in this call (for the combine)
    uint16_t *out;                  // bf16 [T][H]
    uint32_t *status;
    long long wait_cycles;          // limit of every wait but the final drains
    FastDiv S;                      // stages
    int T, k, E, H, I, cps;
};

// Staged (expert, token) B columns per CTA.  A CTA's contiguous range of
// units is no longer than one expert's tiles when the grid has at least as
// many CTAs as there are routed experts, so it touches at most two experts:
// at most 2T columns.
constexpr int kMaxBSlots = 16;
constexpr int kMaxTiles = 128;   // H / 32 for H <= 4096
constexpr int kDNThreads = kGUThreads;
__host__ __device__ inline int dn_slots(int T) { return 2 * T < kMaxBSlots ? 2 * T : kMaxBSlots; }
__host__ __device__ inline size_t dn_red_off(int n_stages, int cps, int T, int I) {
    return (size_t)n_stages * piece_bytes(cps) + sizeof(uint16_t) * (size_t)dn_slots(T) * (I + kXPad);
}
__host__ __device__ inline size_t dn_bytes(int n_stages, int cps, int T, int I) {
    return dn_red_off(n_stages, cps, T, I) + red_bytes(T);
}

template <int NCH>   // K chunks per unit = I / kKC
__global__ void __launch_bounds__(kDNThreads, 1) dec_down_mx_kernel(DownArgs a) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ RouteTable tb;
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages], red_full[kRedSlots], red_empty[kRedSlots];
    __shared__ int issued;   // chunks issued by the producer (see produce)
    __shared__ volatile int abort_flag;   // set by the first role that gives up on a wait
    __shared__ int slot_of[2][kMaxT];    // (expert slot - d_lo, token) -> staged B column, -1 none
    __shared__ int slot_d[kMaxBSlots], slot_t[kMaxBSlots];
    __shared__ unsigned slot_max[kMaxBSlots];
    __shared__ float slot_scale[kMaxBSlots], slot_inv[kMaxBSlots];
    __shared__ int n_slots;
    const int H = a.H, I = a.I, T = a.T, k = a.k, S = (int)a.S.d, cps = a.cps, Tc = red_cols(a.T);
    uint8_t *stages = smem_raw;
    uint16_t *bs = reinterpret_cast<uint16_t *>(smem_raw + (size_t)S * piece_bytes(cps));   // [slot][I+pad] f16
    float *red = reinterpret_cast<float *>(smem_raw + dn_red_off(S, cps, T, I));
    const int bs_stride = I + kXPad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tiles = H / 32;
    const MxGeom geo(H, I);
    constexpr int WPC = kCW / NCH;   // warps per chunk
    const int lcps = cps == 4 ? 2 : (cps == 2 ? 1 : 0);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], WPC * cps);
        }
        for (int r = 0; r < kRedSlots; ++r) {
            mbar_init(&red_full[r], kCW);
            mbar_init(&red_empty[r], kEpiWarps);
        }
        mbar_fence_init();
        issued = 0;
        abort_flag = 0;
    }
    const long long lim = a.wait_cycles;
    if (tid < kMaxBSlots) slot_max[tid] = 0u;
    if (warp == 0) build_route_table(tb, a.ids, a.topk_w, T * k, k, a.E, nullptr, false);
    __syncthreads();
    // the next kernel may take SMs as this grid's CTAs finish (it waits for
    // this grid's completion before touching memory this kernel uses)
    pdl_launch_dependents();
    const int n_units = tb.D * tiles;
    // the combine kernel sums this many slices (it runs after this grid completes)
    if (blockIdx.x == 0 && tid == 0) *a.n_routed = tb.D;
    if (tb.D == 0) return;   // no valid route at all: the combine writes zeros
    int u0, u1;
    my_range(n_units, u0, u1);
    const int n_mine = u1 - u0;
    // unit u -> expert slot u / tiles, 32-row tile u % tiles (tiles is a power of two)
    const int ltiles = 31 - __clz(tiles);
    const int d_lo = n_mine > 0 ? u0 >> ltiles : 0;

    if (warp == kProducerWarp) {
        // the weights do not depend on the gate/up kernel: stream them at once
        produce(stages, full, empty, a.S, cps, n_mine * NCH / cps, &abort_flag, lim, &issued,
                [&](int p, const uint8_t *&b0, const uint8_t *&b1) {
                    const int c = p * cps;
                    const int u = u0 + c / NCH, d = u >> ltiles, t32 = u & (tiles - 1), q = c % NCH;
                    const uint8_t *eb = a.codes + (size_t)tb.expert[d] * geo.expert_bytes();
                    b0 = eb + geo.block_off(2 * t32, q);
                    b1 = eb + geo.block_off(2 * t32 + 1, q);
                });
        return;
    }

    if (warp >= kEpiWarp0) {
        // epilogue: sum the 16 warps' partial fragments of a unit, undo the
        // column's prescale and store the expert's f32 slice for the combine
        const int e = warp - kEpiWarp0;
        for (int j = 0; j < n_mine; ++j) {
            const int slot = j % kRedSlots;
            if (!mbar_wait_abort(&red_full[slot], (uint32_t)((j / kRedSlots) & 1), &abort_flag, lim)) break;
            const int u = u0 + j, d = u >> ltiles, m0 = (u & (tiles - 1)) * 32;
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
        __syncwarp();
        if (abort_flag && lane == 0) atomicOr(a.status, FLAG_TIMEOUT);
        // the slices reach the combine kernel through this grid's completion
        return;
    }

    // ---- consumers.  The (expert, token) columns of this CTA's experts
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
    named_sync_consumers();
    // B column sl = (sum of w_r h_r over the token's routes to the expert,
    // in f32) * 2^s_sl in f16, the power of two putting the column's largest
    // magnitude in [2^14, 2^15): f16 cannot overflow and the epilogue undoes
    // the scale exactly.  Pass 1 finds the maxima with the values kept in
    // registers (two 8-value pieces per thread; larger layers build them
    // again in pass 2).
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

    // the units, one group ahead as in the gate/up kernel
    const int q = warp / WPC, wi = warp % WPC;   // this warp's chunk of every unit and its place in it
    constexpr int NG = 8 / WPC;
    bool timed_out = false;
    const uint8_t *st0 = stages, *st1 = stages;
    int s_cur = 0;
    auto open_unit = [&](int j, const uint8_t *&b0, const uint8_t *&b1, int &s) {
        const int c = j * NCH + q, pc = c >> lcps;
        if (!wait_piece(full, a.S, pc, &issued, &abort_flag, lim)) timed_out = true;
        s = pc - (int)(a.S.div((uint32_t)pc) * a.S.d);
        // [rows m0..+15: blocks of the piece][rows m0+16..+31: blocks of the piece]
        b0 = stages + (size_t)s * piece_bytes(cps) + (size_t)(c & (cps - 1)) * kBlk;
        b1 = b0 + (size_t)cps * kBlk;
    };
    GroupFrags cur;
    if (n_mine > 0) {
        open_unit(0, st0, st1, s_cur);
        load_group(st0, st1, g, t, wi * NG, cur);
    }
    for (int j = 0; j < n_mine && !timed_out; ++j) {
        const int d = (u0 + j) >> ltiles;
        const int my_slot = (g < T) ? slot_of[d - d_lo][g] : -1;   // B column g = token g
        const uint16_t *brow = bs + (size_t)(my_slot < 0 ? 0 : my_slot) * bs_stride + 8 * t;
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int p = 0; p < NG; ++p) {
            const int gp = wi * NG + p;
            const uint8_t *n0 = st0, *n1 = st1;
            int ns = s_cur;
            GroupFrags nxt;
            if (p + 1 < NG) {
                load_group(st0, st1, g, t, gp + 1, nxt);
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s_cur]);
                if (j + 1 < n_mine) {
                    open_unit(j + 1, n0, n1, ns);
                    load_group(n0, n1, g, t, wi * NG, nxt);
                }
            }
            const uint16_t *xq = brow + q * kKC + gp * 128;
            uint4 xb[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) xb[jj] = my_slot >= 0 ? lds128(xq + jj * 32) : make_uint4(0u, 0u, 0u, 0u);
            compute_group(cur, xb, acc0, acc1);
            cur = nxt;
            st0 = n0;
            st1 = n1;
            s_cur = ns;
        }
        const int slot = j % kRedSlots;
        if (j >= kRedSlots && !mbar_wait_abort(&red_empty[slot], (uint32_t)((j / kRedSlots - 1) & 1), &abort_flag, lim))
            timed_out = true;
        put_partials(red + (size_t)slot * kCW * 2 * 16 * Tc, Tc, warp, g, t, acc0, acc1);
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_full[slot]);
    }
    if ((timed_out || abort_flag) && lane == 0) atomicOr(a.status, FLAG_TIMEOUT);
}

// Combine (one output element per thread): the experts' f32 slices of the
// down kernel summed in expert order, rounded once to bf16.  Launched as a
// programmatic dependent of the down kernel, whose completion it waits for;
// the order of the sum does not depend on timing.
constexpr int kCombineThreads = 256;
__global__ void __launch_bounds__(kCombineThreads) dec_combine_kernel(const float *ybuf, const int *n_routed,
                                                                       uint16_t *out, int T, int H) {
    pdl_wait_primary();
    pdl_launch_dependents();
    const int D = __ldcg(n_routed);
    const int i = blockIdx.x * kCombineThreads + threadIdx.x;
    if (i >= T * H) return;
    const float *yb = ybuf + i;   // [d][col][m]: element i = col * H + m of slice d at d * kMaxT * H
    // the slices 16 loads at a time (independent, so they overlap), added in expert order
    float sum = 0.f;
    for (int d0 = 0; d0 < D; d0 += 16) {
        float v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] = d0 + q < D ? __ldcg(yb + (size_t)(d0 + q) * kMaxT * H) : 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q)
            if (d0 + q < D) sum += v[q];
    }
    __nv_bfloat16 o = __float2bfloat16_rn(sum);
    out[i] = *reinterpret_cast<uint16_t *>(&o);
}

template <typename K, typename... A>
cudaError_t launch_ex(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, A... args) {
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
    return cudaLaunchKernelEx(&cfg, kernel, args...);
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
StagePlan gu_plan(int T, int H) { return plan_stages(H / kKC, gu_bytes(0, 1, T, H)); }
StagePlan dn_plan(int T, int I) { return plan_stages(I / kKC, dn_bytes(0, 1, T, I)); }

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
    ga.wait_cycles = L.wait_cycles;
    ga.T = T;
    ga.k = L.d.top_k;
    ga.E = L.d.n_experts;
    ga.H = H;
    ga.I = I;
    const StagePlan gp = gu_plan(T, H);
    ga.S = make_fastdiv((uint32_t)gp.S);
    ga.cps = gp.cps;
    L.count_launches(3);
    if (ev) record_phase(ev[1], s);   // routing is fused into both kernels' prologues
    cudaError_t e = launch_ex(dec_gateup_mx_kernel<NCU>, dim3(grid), dim3(kGUThreads),
                              gu_bytes(gp.S, ga.cps, T, H), s, ev == nullptr, ga);
    if (e != cudaSuccess) return e;
    if (ev) record_phase(ev[2], s);
    DownArgs da;
    da.codes = L.w.codes[MOEQ_DOWN];
    da.h = L.h;
    da.ids = ids;
    da.topk_w = topk_w;
    da.ybuf = L.dec_ybuf;
    da.n_routed = L.dec_counters;
    da.out = reinterpret_cast<uint16_t *>(out);
    da.status = L.status;
    da.wait_cycles = L.wait_cycles;
    da.T = T;
    da.k = L.d.top_k;
    da.E = L.d.n_experts;
    da.H = H;
    da.I = I;
    const StagePlan dp = dn_plan(T, I);
    da.S = make_fastdiv((uint32_t)dp.S);
    da.cps = dp.cps;
    // programmatic dependent launch: the down kernel's producer streams
    // weights while the gate/up kernel drains; its consumers wait for that
    // grid before reading h.  Not with phase events between the launches.
    e = launch_ex(dec_down_mx_kernel<NCD>, dim3(grid), dim3(kDNThreads), dn_bytes(dp.S, da.cps, T, I), s, ev == nullptr,
                  da);
    if (e != cudaSuccess) return e;
    if (ev) record_phase(ev[3], s);
    const int n_out = T * H;
    e = launch_ex(dec_combine_kernel, dim3((n_out + kCombineThreads - 1) / kCombineThreads), dim3(kCombineThreads), 0,
                  s, ev == nullptr, (const float *)L.dec_ybuf, (const int *)L.dec_counters, (uint16_t *)out, T, H);
    if (e != cudaSuccess) return e;
    if (ev) record_phase(ev[4], s);
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
