// prefill_vq.cu -- VQ13(+R8) and GVQ1(+R8) routed-expert FFN on the
// 5th-generation tensor cores (bf16 activations, any token count).
//
// Format ("MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe"): an expert row is
// cut into 8-weight vectors, each stored as a 13-bit index into the layer's
// 8192 x 8 codebook (optionally with an 8-bit index into a 256 x 8 residual
// book), the row scaled by an f16 gain; one codebook pair serves every expert and
// gate/up/down ("Why 13 bits": the books stay in shared memory while every
// selected expert is decoded).  Weight = (base + residual) * gain, in bf16
// for the tensor cores; activations are bf16 already,
// so the MMAs are tcgen05.mma kind::f16 (bf16 x bf16 -> f32).  The expansion
// adds base and residual codewords and applies the gain in bf16 pairs.
// The GVQ1 container (same page, "Recipe": a 12-bit code stream with a
// separate plane of one-bit flags, books of 1-byte entries) runs the same
// kernels, instantiated for
// its index layout, on bf16 images of its books made at upload (entry =
// bf16(f32(e4m3(byte) x book scale))).
//
// Steps of one forward:
//   route/bucket, route tiles (as for MXFP4: tiles of up to 64 routes)
//   vq_gather_x_kernel  -> x rows in route order (bf16)
//   vq_gateup_kernel    -> per (route tile, 128 rows of I): decoder warps
//                          expand gate and up codes into bf16 tiles in shared
//                          memory, the MMA thread multiplies them with the
//                          route tile, the epilogue writes h = silu(g) u (bf16)
//   vq_down_kernel      -> per (route tile, 128 rows of H): y, weighted and
//                          added into acc[T][H] (f32 atomics)
//   cast                -> out = bf16(acc)
//
// CTA roles (one CTA per SM): warp 0 loads the codebooks once, then the
// activation tiles by TMA; warp 1 issues the MMAs; warps 2..9 decode weight
// tiles (16-byte codeword gathers from shared memory: the step that bounds
// this path); warps 10..13 run the epilogue.  Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "async.cuh"
#include "internal.cuh"
#include "umma.cuh"

namespace moeq {
namespace {

using namespace umma;

constexpr int kDecWarps = 8;
constexpr int kVqThreads = 32 * (2 + kDecWarps + 4);
constexpr int kKS = 64;                        // K per slab: 64 bf16 = one 128-byte row
constexpr int kTileA = kT * kKS * 2;           // 16 KB
constexpr int kTileB = kRT * kKS * 2;          // 8 KB
constexpr int kBook13 = 8192 * 16, kBook8 = 256 * 16;
constexpr int kGUStage = 2 * kTileA + kTileB;  // [A gate][A up][B]
constexpr int kGUStages = 2;
constexpr int kDNStage = kTileA + kTileB;      // [A down][B]
constexpr int kDNStages = 3;
constexpr int kPrefetch = 6;                   // slabs ahead the activation boxes are pulled into L2

// kind::f16 instruction descriptor: bf16 A and B (K-major), f32 accumulate, M 128
__device__ __forceinline__ uint32_t idesc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kT >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

struct VqProj {
    const uint8_t *idx13;   // [E*N][K*13/64] (VQ13), or null
    const uint8_t *idx8;    // [E*N][K/8] or null
    const uint16_t *gain;   // [E*N] f16 or null
    const uint8_t *code12;  // GVQ1: [E*N][K*3/16], the low 12 bits of the indices; null for VQ13
    const uint8_t *hi1;     // GVQ1: [E*N][K/64], bit 12 of index j as bit j % 8 of byte j / 8
};

// The index data of one row for one 64-column slab, fetched ahead of its
// decode so that the global loads overlap the gathers of earlier slabs: the
// 13-byte chunk of 13-bit indices as four aligned words (the allocation has
// slack for the last row), the eight residual indices and the row gain.
struct RowRaw {
    uint32_t w[4];    // the chunk (VQ13: 13 bytes in four aligned words; GVQ1: 12 bytes in w[0..2])
    uint32_t shift;   // bit offset of the chunk inside w (VQ13)
    uint32_t hi;      // GVQ1: the slab's byte of bit-12 flags
    uint32_t i8lo, i8hi;
    uint32_t gain;    // f16 bits, 0x3C00 (1.0) when the layer has no gains
};
template <bool G1>   // GVQ1 container (else VQ13)
__device__ __forceinline__ RowRaw fetch_row(const VqProj &pj, int K, size_t grow, int sl) {
    RowRaw v;
    if constexpr (G1) {
        // 8 vectors x 12 bits = 12 bytes, 4-byte aligned (K * 3/16 and 12 are multiples of 4)
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(pj.code12 + grow * (size_t)(K * 3 / 16) +
                                                                (size_t)sl * (kKS / 8 * 12 / 8));
#pragma unroll
        for (int i = 0; i < 3; ++i) v.w[i] = __ldg(wp + i);
        v.w[3] = 0u;
        v.shift = 0u;
        v.hi = __ldg(pj.hi1 + grow * (size_t)(K / 64) + (size_t)sl);
    } else {
        const uint8_t *chunk = pj.idx13 + grow * (size_t)(K * 13 / 64) + (size_t)sl * (kKS / 8 * 13 / 8);
        const uintptr_t ad = reinterpret_cast<uintptr_t>(chunk);
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(ad & ~uintptr_t(3));
#pragma unroll
        for (int i = 0; i < 4; ++i) v.w[i] = __ldg(wp + i);
        v.shift = (uint32_t)(ad & 3) * 8;
        v.hi = 0u;
    }
    if (pj.idx8) {
        const uint2 q = __ldg(reinterpret_cast<const uint2 *>(pj.idx8 + grow * (size_t)(K / 8) + (size_t)sl * (kKS / 8)));
        v.i8lo = q.x;
        v.i8hi = q.y;
    } else {
        v.i8lo = v.i8hi = 0;
    }
    v.gain = pj.gain ? (uint32_t)__ldg(pj.gain + grow) : 0x3C00u;
    return v;
}
// The eight 13-bit indices of a fetched row chunk: VQ13 index j at bits
// 13j..13j+12 of the chunk; GVQ1 index j = bits 12j..12j+11 of the chunk,
// plus bit j of the slab's flag byte as bit 12.
template <bool G1>
__device__ __forceinline__ void row_indices(const RowRaw &v, uint32_t idx[8]) {
    if constexpr (G1) {
        const uint32_t w0 = v.w[0], w1 = v.w[1], w2 = v.w[2];
        idx[0] = w0 & 0xFFFu;
        idx[1] = (w0 >> 12) & 0xFFFu;
        idx[2] = __funnelshift_r(w0, w1, 24) & 0xFFFu;
        idx[3] = (w1 >> 4) & 0xFFFu;
        idx[4] = (w1 >> 16) & 0xFFFu;
        idx[5] = __funnelshift_r(w1, w2, 28) & 0xFFFu;
        idx[6] = (w2 >> 8) & 0xFFFu;
        idx[7] = (w2 >> 20) & 0xFFFu;
#pragma unroll
        for (int j = 0; j < 8; ++j) idx[j] |= ((v.hi >> j) & 1u) << 12;
        return;
    }
    const uint32_t x0 = __funnelshift_r(v.w[0], v.w[1], v.shift), x1 = __funnelshift_r(v.w[1], v.w[2], v.shift);
    const uint32_t x2 = __funnelshift_r(v.w[2], v.w[3], v.shift), x3 = v.w[3] >> v.shift;
    idx[0] = x0 & 0x1FFFu;
    idx[1] = (x0 >> 13) & 0x1FFFu;
    idx[2] = __funnelshift_r(x0, x1, 26) & 0x1FFFu;
    idx[3] = (x1 >> 7) & 0x1FFFu;
    idx[4] = __funnelshift_r(x1, x2, 20) & 0x1FFFu;
    idx[5] = (x2 >> 1) & 0x1FFFu;
    idx[6] = (x2 >> 14) & 0x1FFFu;
    idx[7] = __funnelshift_r(x2, x3, 27) & 0x1FFFu;
}

__device__ __forceinline__ uint32_t bf16x2_add(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Expand vector j of a row (13-bit index idx, residual index i8, gain bits)
// into 8 bf16 weights at the 128B-swizzled K-major position (tile row r,
// 16-byte chunk j) of a shared-memory A tile.  The base and residual
// codewords are added as bf16 pairs (one rounding of the exact sum) and
// scaled by the row gain as bf16 pairs: the tensor cores take bf16 operands,
// and two roundings to bf16 stay far inside the output tolerance
// (moeq_dequant keeps the exact f32 weights).
__device__ __forceinline__ void expand_vec(uint32_t idx, uint32_t i8, uint32_t gain, bool r8, int j,
                                           const uint8_t *book13, const uint8_t *book8, uint8_t *tile, int r) {
    uint4 o = lds128(book13 + (size_t)idx * 16);
    if (r8) {
        const uint4 rr = lds128(book8 + (size_t)i8 * 16);
        o = make_uint4(bf16x2_add(o.x, rr.x), bf16x2_add(o.y, rr.y), bf16x2_add(o.z, rr.z), bf16x2_add(o.w, rr.w));
    }
    if (gain != 0x3C00u) {
        const __nv_bfloat16 gb = __float2bfloat16_rn(__half2float(__ushort_as_half((unsigned short)gain)));
        const uint32_t g2 = (uint32_t)*reinterpret_cast<const uint16_t *>(&gb) * 0x10001u;
        o = make_uint4(bf16x2_mul(o.x, g2), bf16x2_mul(o.y, g2), bf16x2_mul(o.z, g2), bf16x2_mul(o.w, g2));
    }
    *reinterpret_cast<uint4 *>(tile + (r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4)) = o;
}

// Decode vectors [J0, J0 + NV) of one fetched row into tile row r.
template <bool G1, int J0, int NV>
__device__ __forceinline__ void expand_row(const RowRaw &v, bool r8, const uint8_t *book13, const uint8_t *book8,
                                           uint8_t *tile, int r) {
    uint32_t idx[8];
    row_indices<G1>(v, idx);
#pragma unroll
    for (int jj = 0; jj < NV; ++jj) {
        const int j = J0 + jj;
        const uint32_t i8 = ((j < 4 ? v.i8lo : v.i8hi) >> (8 * (j & 3))) & 0xFFu;
        expand_vec(idx[j], i8, v.gain, r8, j, book13, book8, tile, r);
    }
}

// One warp per route position: its token's x row, in route order.
__global__ void __launch_bounds__(256) vq_gather_x_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ perm,
                                                          const int32_t *__restrict__ offsets, int E, int k, int H,
                                                          uint16_t *__restrict__ xg) {
    const int n_valid = __ldg(offsets + E);
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int n_warps = (gridDim.x * blockDim.x) >> 5;
    for (int p = warp; p < n_valid; p += n_warps) {
        const int t = __ldg(perm + p) / k;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
        uint4 *dst = reinterpret_cast<uint4 *>(xg + (size_t)p * H);
        for (int i = lane; i < H / 8; i += 32) dst[i] = __ldg(src + i);
    }
}

struct VqArgs {
    const int32_t *offsets, *tile_base, *perm;
    const float *topk_w;
    VqProj w0, w1;            // gate/up: gate, up; down: down in w0
    const uint8_t *book13, *book8;
    uint16_t *hg;             // gate/up output [route position][I] bf16
    float *acc;               // down output [T][H]
    uint32_t *status;
    long long wait_cycles;        // limit of every wait but the final drains
    int E, H, I, k;
};

// Shared pieces of both kernels: the codebooks into shared memory (warp 0,
// before its TMA loop), on `bar`.
__device__ __forceinline__ void load_books(uint8_t *b13, uint8_t *b8, const VqArgs &a, uint64_t *bar, int lane) {
    const uint32_t bytes = kBook13 + (a.book8 ? kBook8 : 0);
    if (lane == 0) mbar_arrive_expect_tx(bar, bytes);
    __syncwarp();
    if (lane < 8) bulk_g2s(b13 + lane * (kBook13 / 8), a.book13 + lane * (kBook13 / 8), kBook13 / 8, bar);
    if (lane == 8 && a.book8) bulk_g2s(b8, a.book8, kBook8, bar);
    __syncwarp();
}

// ---------------------------------------------------------------- gate/up

template <bool G1>   // GVQ1 container (else VQ13)
__global__ void __launch_bounds__(kVqThreads, 1) vq_gateup_kernel(const __grid_constant__ CUtensorMap tX, VqArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *b13 = smem + kGUStages * kGUStage, *b8 = b13 + kBook13;
    __shared__ __align__(8) uint64_t a_full[kGUStages], b_full[kGUStages], empty[kGUStages], tmem_full[2],
        tmem_empty[2], tmem_done, book_bar;
    __shared__ uint32_t tslot;
    __shared__ volatile int abort_flag;
    __shared__ RouteTables rt;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, I = a.I, E = a.E;
    const int subs = I / kT, slabs = H / kKS;

    if (tid == 0) {
        for (int s = 0; s < kGUStages; ++s) {
            mbar_init(&a_full[s], kDecWarps);
            mbar_init(&b_full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 1);
            mbar_init(&tmem_empty[b], 4);
        }
        mbar_init(&tmem_done, 1);
        mbar_init(&book_bar, 1);
        mbar_fence_init();
        abort_flag = 0;
    }
    load_route_tables(rt, a.offsets, a.tile_base, a.E);
    if (warp == 1) tc_alloc(&tslot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;   // buffer b: gate at 128 b, up at 128 b + 64
    const int n_items = rt.tb[E] * subs;
    const int my_items = n_items > (int)blockIdx.x ? (n_items - (int)blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    const int total = my_items * slabs;

    if (warp == 0) {
        load_books(b13, b8, a, &book_bar, lane);
        if (lane == 0) {
            int c = 0;
            for (; c < total; ++c) {
                const int s = c % kGUStages;
                if (c >= kGUStages && !wait_or_abort(&empty[s], (uint32_t)((c / kGUStages - 1) & 1), &abort_flag, a.wait_cycles)) break;
                const Item m = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + (c / slabs) * gridDim.x);
                mbar_arrive_expect_tx(&b_full[s], kTileB);
                tma_load_2d(smem + (size_t)s * kGUStage + 2 * kTileA, &tX, (c % slabs) * kKS, m.row0, &b_full[s]);
                // the ring is short: start the activation box of a later slab towards L2
                if (c + kPrefetch < total) {
                    const Item mp = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + ((c + kPrefetch) / slabs) * gridDim.x);
                    tma_prefetch_2d(&tX, ((c + kPrefetch) % slabs) * kKS, mp.row0);
                }
            }
            drain_stages(b_full, kGUStages, c);
            mbar_wait_bounded(&book_bar, 0, kDrainCycles);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int c = 0;
            for (int q = 0; q < my_items && !abort_flag; ++q) {
                const Item m = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + q * gridDim.x);
                const int n = (m.cnt + 15) & ~15, b = q & 1;
                const uint32_t id = idesc_bf16(n);
                if (q >= 2 && !wait_or_abort(&tmem_empty[b], (uint32_t)(((q >> 1) - 1) & 1), &abort_flag, a.wait_cycles)) break;
                tc_fence_after();
                const uint32_t t_g = tmem + b * 2 * kRT, t_u = t_g + kRT;
                for (int sl = 0; sl < slabs; ++sl, ++c) {
                    const int s = c % kGUStages;
                    const uint32_t par = (uint32_t)((c / kGUStages) & 1);
                    if (!wait_or_abort(&a_full[s], par, &abort_flag, a.wait_cycles) || !wait_or_abort(&b_full[s], par, &abort_flag, a.wait_cycles)) break;
                    tc_fence_after();
                    const uint8_t *st = smem + (size_t)s * kGUStage;
#pragma unroll
                    for (int kk = 0; kk < kKS / 16; ++kk) {
                        const uint64_t ag = desc_sw128(st + kk * 32), au = desc_sw128(st + kTileA + kk * 32);
                        const uint64_t bx = desc_sw128(st + 2 * kTileA + kk * 32);
                        const uint32_t acc = (sl > 0 || kk > 0) ? 1u : 0u;
                        mma_bf16(t_g, ag, bx, id, acc);
                        mma_bf16(t_u, au, bx, id, acc);
                    }
                    tc_commit(&empty[s]);
                }
                tc_commit(&tmem_full[b]);
            }
            drain_mma(&tmem_done);
        }
    } else if (warp < 2 + kDecWarps) {
        // decoders: per slab 2 matrices x 128 rows x 8 vectors; thread t
        // takes all 8 vectors of row t % 128 of matrix t / 128.  Its index
        // data comes from HBM four slabs ahead, into a ring of four register
        // sets indexed at compile time (moving a register whose load is still
        // in flight would wait for it)
        const int dt = tid - 64, mat = dt >> 7, r = dt & 127;
        const bool r8 = a.book8 != nullptr;
        const VqProj &pj = mat ? a.w1 : a.w0;
        auto fetch = [&](int c, RowRaw &dst) {
            if (c >= total) return;
            const Item m = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + (c / slabs) * gridDim.x);
            dst = fetch_row<G1>(pj, H, (size_t)m.e * I + m.sub * kT + r, c % slabs);
        };
        RowRaw q0, q1, q2, q3;
        fetch(0, q0);
        fetch(1, q1);
        fetch(2, q2);
        fetch(3, q3);
        bool ok = wait_or_abort(&book_bar, 0, &abort_flag, a.wait_cycles);
        auto step = [&](int c, RowRaw &q) {
            if (c >= total || !ok) return;
            const int s = c % kGUStages;
            if (c >= kGUStages) ok = wait_or_abort(&empty[s], (uint32_t)((c / kGUStages - 1) & 1), &abort_flag, a.wait_cycles);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) return;
            expand_row<G1, 0, 8>(q, r8, b13, b8, smem + (size_t)s * kGUStage + mat * kTileA, r);
            fetch(c + 4, q);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[s]);
        };
        for (int c = 0; c < total && ok; c += 4) {
            step(c, q0);
            step(c + 1, q1);
            step(c + 2, q2);
            step(c + 3, q3);
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 = rows of I
        const int qd = warp & 3;
        for (int q = 0; q < my_items && !abort_flag; ++q) {
            const Item m = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + q * gridDim.x);
            const int b = q & 1;
            if (!wait_or_abort(&tmem_full[b], (uint32_t)((q >> 1) & 1), &abort_flag, a.wait_cycles)) break;
            tc_fence_after();
            const int i_row = m.sub * kT + 32 * qd + lane;
            const uint32_t t_g = tmem + b * 2 * kRT + ((uint32_t)(32 * qd) << 16), t_u = t_g + kRT;
            for (int n0 = 0; n0 < m.cnt; n0 += 16) {
                float g[16], u[16];
                tc_ld16(t_g + n0, g);
                tc_ld16(t_u + n0, u);
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const int n = n0 + jj;
                    if (n >= m.cnt) break;
                    const __nv_bfloat16 h = __float2bfloat16_rn(silu_f32(g[jj]) * u[jj]);
                    a.hg[(size_t)(m.row0 + n) * I + i_row] = *reinterpret_cast<const uint16_t *>(&h);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (abort_flag && tid == 0) atomicOr(a.status, FLAG_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        tc_dealloc(tmem, 256);
    }
}

// ---------------------------------------------------------------- down

template <bool G1>
__global__ void __launch_bounds__(kVqThreads, 1) vq_down_kernel(const __grid_constant__ CUtensorMap tH, VqArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *b13 = smem + kDNStages * kDNStage, *b8 = b13 + kBook13;
    __shared__ __align__(8) uint64_t a_full[kDNStages], b_full[kDNStages], empty[kDNStages], tmem_full[2],
        tmem_empty[2], tmem_done, book_bar;
    __shared__ uint32_t tslot;
    __shared__ volatile int abort_flag;
    __shared__ RouteTables rt;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, I = a.I, E = a.E, k = a.k;
    const int subs = H / kT, slabs = I / kKS;

    if (tid == 0) {
        for (int s = 0; s < kDNStages; ++s) {
            mbar_init(&a_full[s], kDecWarps);
            mbar_init(&b_full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 1);
            mbar_init(&tmem_empty[b], 4);
        }
        mbar_init(&tmem_done, 1);
        mbar_init(&book_bar, 1);
        mbar_fence_init();
        abort_flag = 0;
    }
    load_route_tables(rt, a.offsets, a.tile_base, a.E);
    if (warp == 1) tc_alloc(&tslot, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;   // buffer b at 64 b
    const int n_items = rt.tb[E] * subs;
    const int my_items = n_items > (int)blockIdx.x ? (n_items - (int)blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    const int total = my_items * slabs;

    if (warp == 0) {
        load_books(b13, b8, a, &book_bar, lane);
        if (lane == 0) {
            int c = 0;
            for (; c < total; ++c) {
                const int s = c % kDNStages;
                if (c >= kDNStages && !wait_or_abort(&empty[s], (uint32_t)((c / kDNStages - 1) & 1), &abort_flag, a.wait_cycles)) break;
                const Item m = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + (c / slabs) * gridDim.x);
                mbar_arrive_expect_tx(&b_full[s], kTileB);
                tma_load_2d(smem + (size_t)s * kDNStage + kTileA, &tH, (c % slabs) * kKS, m.row0, &b_full[s]);
                if (c + kPrefetch < total) {
                    const Item mp = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + ((c + kPrefetch) / slabs) * gridDim.x);
                    tma_prefetch_2d(&tH, ((c + kPrefetch) % slabs) * kKS, mp.row0);
                }
            }
            drain_stages(b_full, kDNStages, c);
            mbar_wait_bounded(&book_bar, 0, kDrainCycles);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int c = 0;
            for (int q = 0; q < my_items && !abort_flag; ++q) {
                const Item m = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + q * gridDim.x);
                const int n = (m.cnt + 15) & ~15, b = q & 1;
                const uint32_t id = idesc_bf16(n);
                if (q >= 2 && !wait_or_abort(&tmem_empty[b], (uint32_t)(((q >> 1) - 1) & 1), &abort_flag, a.wait_cycles)) break;
                tc_fence_after();
                const uint32_t t_y = tmem + b * kRT;
                for (int sl = 0; sl < slabs; ++sl, ++c) {
                    const int s = c % kDNStages;
                    const uint32_t par = (uint32_t)((c / kDNStages) & 1);
                    if (!wait_or_abort(&a_full[s], par, &abort_flag, a.wait_cycles) || !wait_or_abort(&b_full[s], par, &abort_flag, a.wait_cycles)) break;
                    tc_fence_after();
                    const uint8_t *st = smem + (size_t)s * kDNStage;
#pragma unroll
                    for (int kk = 0; kk < kKS / 16; ++kk)
                        mma_bf16(t_y, desc_sw128(st + kk * 32), desc_sw128(st + kTileA + kk * 32), id,
                                 (sl > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&empty[s]);
                }
                tc_commit(&tmem_full[b]);
            }
            drain_mma(&tmem_done);
        }
    } else if (warp < 2 + kDecWarps) {
        // decoders: per slab 128 rows x 8 vectors; thread t takes vectors
        // 4 (t % 2) .. + 3 of row t / 2, index data fetched two slabs ahead
        const int dt = tid - 64, r = dt >> 1, j0 = (dt & 1) * 4;
        const bool r8 = a.book8 != nullptr;
        auto fetch = [&](int c, RowRaw &dst) {
            if (c >= total) return;
            const Item m = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + (c / slabs) * gridDim.x);
            dst = fetch_row<G1>(a.w0, I, (size_t)m.e * H + m.sub * kT + r, c % slabs);
        };
        RowRaw q0, q1, q2, q3;   // four slabs ahead, as in the gate/up kernel
        fetch(0, q0);
        fetch(1, q1);
        fetch(2, q2);
        fetch(3, q3);
        bool ok = wait_or_abort(&book_bar, 0, &abort_flag, a.wait_cycles);
        auto step = [&](int c, RowRaw &q) {
            if (c >= total || !ok) return;
            const int s = c % kDNStages;
            if (c >= kDNStages) ok = wait_or_abort(&empty[s], (uint32_t)((c / kDNStages - 1) & 1), &abort_flag, a.wait_cycles);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) return;
            uint8_t *tile = smem + (size_t)s * kDNStage;
            if (j0 == 0) expand_row<G1, 0, 4>(q, r8, b13, b8, tile, r);
            else expand_row<G1, 4, 4>(q, r8, b13, b8, tile, r);
            fetch(c + 4, q);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[s]);
        };
        for (int c = 0; c < total && ok; c += 4) {
            step(c, q0);
            step(c + 1, q1);
            step(c + 2, q2);
            step(c + 3, q3);
        }
    } else {
        const int qd = warp & 3;
        for (int q = 0; q < my_items && !abort_flag; ++q) {
            const Item m = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + q * gridDim.x);
            const int b = q & 1;
            int tk0 = 0, tk1 = 0;
            float w0 = 0.f, w1 = 0.f;
            if (lane < m.cnt) {
                const int r = __ldg(a.perm + m.row0 + lane);
                tk0 = r / k;
                w0 = __ldg(a.topk_w + r);
            }
            if (lane + 32 < m.cnt) {
                const int r = __ldg(a.perm + m.row0 + 32 + lane);
                tk1 = r / k;
                w1 = __ldg(a.topk_w + r);
            }
            if (!wait_or_abort(&tmem_full[b], (uint32_t)((q >> 1) & 1), &abort_flag, a.wait_cycles)) break;
            tc_fence_after();
            const int h_row = m.sub * kT + 32 * qd + lane;
            const uint32_t t_y = tmem + b * kRT + ((uint32_t)(32 * qd) << 16);
            for (int n0 = 0; n0 < m.cnt; n0 += 16) {
                float y[16];
                tc_ld16(t_y + n0, y);
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const int n = n0 + jj;
                    if (n >= m.cnt) break;
                    const int tk = __shfl_sync(0xffffffffu, n < 32 ? tk0 : tk1, n & 31);
                    const float w = __shfl_sync(0xffffffffu, n < 32 ? w0 : w1, n & 31);
                    atomicAdd(a.acc + (size_t)tk * H + h_row, w * y[jj]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (abort_flag && tid == 0) atomicOr(a.status, FLAG_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        tc_dealloc(tmem, 128);
    }
}

__global__ void vq_cast_kernel(const float *__restrict__ acc, __nv_bfloat16 *__restrict__ out, long long n) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = __float2bfloat16_rn(acc[i]);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// bf16 [rows][cols] with 64 x 64 boxes, 128B swizzle
cudaError_t make_bf16_map(CUtensorMap *map, void *base, long long cols, long long rows) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
        return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kKS, (cuuint32_t)kRT};
    const cuuint32_t es[2] = {1, 1};
    const CUresult r = reinterpret_cast<EncodeTiledFn>(p)(
        map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

size_t gu_smem() { return (size_t)kGUStages * kGUStage + kBook13 + kBook8 + 1024; }
size_t dn_smem() { return (size_t)kDNStages * kDNStage + kBook13 + kBook8 + 1024; }

}  // namespace

bool prefill_vq_supported(const Layer &L, int T) {
    return L.pv != nullptr && L.pv->ready && T >= 1 && L.d.act == MOEQ_ACT_BF16 &&
           (is_vq13(L.d.fmt) || (is_gvq1(L.d.fmt) && L.pv->books_ready));
}

cudaError_t prefill_vq_create(Layer &L) {
    const moeq_layer_desc &d = L.d;
    if (!(is_vq13(d.fmt) || is_gvq1(d.fmt)) || d.act != MOEQ_ACT_BF16) return cudaSuccess;
    if (d.hidden % kT || d.inter % kT) return cudaSuccess;
    PrefillVq *pv = new (std::nothrow) PrefillVq();
    if (!pv) return cudaErrorMemoryAllocation;
    L.pv = pv;
    const size_t R = (size_t)d.max_tokens * d.top_k;
    cudaError_t e = dev_alloc((void **)&pv->tile_base, sizeof(int32_t) * (d.n_experts + 1));
    if (e == cudaSuccess) e = dev_alloc((void **)&pv->xg, R * d.hidden * 2);
    if (e == cudaSuccess) e = dev_alloc((void **)&pv->hg, R * d.inter * 2);
    if (e == cudaSuccess && is_gvq1(d.fmt)) e = dev_alloc((void **)&pv->gbook13, sizeof(uint16_t) * kBook13Rows * 8);
    if (e == cudaSuccess && is_gvq1(d.fmt) && has_r8(d.fmt))
        e = dev_alloc((void **)&pv->gbook8, sizeof(uint16_t) * kBook8Rows * 8);
    // route positions past a tile's routes feed discarded MMA columns: keep them finite
    if (e == cudaSuccess) e = cudaMemset(pv->xg, 0, R * d.hidden * 2);
    if (e == cudaSuccess) e = cudaMemset(pv->hg, 0, R * d.inter * 2);
    if (e != cudaSuccess) return e;
    e = make_bf16_map(&pv->map_x, pv->xg, d.hidden, (long long)R);
    if (e == cudaSuccess) e = make_bf16_map(&pv->map_h, pv->hg, d.inter, (long long)R);
    const bool g1 = is_gvq1(d.fmt);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(g1 ? vq_gateup_kernel<true> : vq_gateup_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gu_smem());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(g1 ? vq_down_kernel<true> : vq_down_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dn_smem());
    if (e == cudaSuccess) pv->ready = true;
    return e == cudaErrorNotSupported ? cudaSuccess : e;
}

void prefill_vq_free(Layer &L) {
    PrefillVq *pv = L.pv;
    if (!pv) return;
    cudaFree(pv->tile_base);
    cudaFree(pv->xg);
    cudaFree(pv->hg);
    cudaFree(pv->gbook13);
    cudaFree(pv->gbook8);
    delete pv;
    L.pv = nullptr;
}

// GVQ1 books for the tensor-core path: entry value e4m3(b) (the OCP 8-bit
// float without infinities: sign, 4 exponent bits with bias 7, 3 mantissa
// bits, subnormal below exponent 1) times the book's scale as an f32
// product, rounded to nearest even bf16 -- the f32 weight formula's product,
// one bf16 rounding.  NaN bytes were rejected at upload.
namespace {
float e4m3_value(uint8_t b) {
    const int sgn = b >> 7, ex = (b >> 3) & 15, man = b & 7;
    const float mag = ex ? std::ldexp(1.0f + man / 8.0f, ex - 7) : std::ldexp(man / 8.0f, -6);
    return sgn ? -mag : mag;
}
uint16_t bf16_rne(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)(u >> 16);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}
}  // namespace

cudaError_t prefill_vq_upload_gvq1_books(Layer &L, const uint8_t *book13, const uint8_t *book8, const float scale[2]) {
    PrefillVq *pv = L.pv;
    if (!pv || !pv->ready || !pv->gbook13) return cudaSuccess;
    std::vector<uint16_t> h13((size_t)kBook13Rows * 8), h8;
    for (size_t i = 0; i < h13.size(); ++i) h13[i] = bf16_rne(e4m3_value(book13[i]) * scale[0]);
    cudaError_t e = cudaMemcpy(pv->gbook13, h13.data(), h13.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && pv->gbook8 && book8) {
        h8.resize((size_t)kBook8Rows * 8);
        for (size_t i = 0; i < h8.size(); ++i) h8[i] = bf16_rne(e4m3_value(book8[i]) * scale[1]);
        e = cudaMemcpy(pv->gbook8, h8.data(), h8.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
    }
    pv->books_ready = e == cudaSuccess;
    return e;
}

cudaError_t launch_prefill_vq(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                              cudaStream_t s, const cudaEvent_t *ev) {
    const PrefillVq *pv = L.pv;
    const int E = L.d.n_experts, H = L.d.hidden, I = L.d.inter, k = L.d.top_k;
    cudaError_t e = launch_route_bucket(L, ids, T * k, L.b.offsets, L.b.perm, L.b.active, s);
    if (e != cudaSuccess) return e;
    if (ev) record_phase(ev[1], s);
    L.count_launches(5);
    if ((e = launch_route_tiles(L.b.offsets, E, pv->tile_base, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(L.acc, 0, sizeof(float) * (size_t)T * H, s)) != cudaSuccess) return e;
    {
        const int warps = T * k < 148 * 16 ? T * k : 148 * 16;
        vq_gather_x_kernel<<<(warps + 7) / 8, 256, 0, s>>>(reinterpret_cast<const uint16_t *>(x), L.b.perm, L.b.offsets,
                                                            E, k, H, pv->xg);
    }
    VqArgs a{};
    a.offsets = L.b.offsets;
    a.tile_base = pv->tile_base;
    a.perm = L.b.perm;
    a.topk_w = topk_w;
    const bool g1 = is_gvq1(L.d.fmt);
    a.book13 = reinterpret_cast<const uint8_t *>(g1 ? pv->gbook13 : L.w.book13);
    a.book8 = has_r8(L.d.fmt) ? reinterpret_cast<const uint8_t *>(g1 ? pv->gbook8 : L.w.book8) : nullptr;
    a.hg = pv->hg;
    a.acc = L.acc;
    a.status = L.status;
    a.wait_cycles = L.wait_cycles;
    a.E = E;
    a.H = H;
    a.I = I;
    a.k = k;
    auto proj = [&](int p) {
        const ProjView v = L.view(p);
        return g1 ? VqProj{nullptr, v.idx8, v.gain, v.code12, v.hi1} : VqProj{v.idx13, v.idx8, v.gain, nullptr, nullptr};
    };
    a.w0 = proj(MOEQ_GATE);
    a.w1 = proj(MOEQ_UP);
    if (g1) vq_gateup_kernel<true><<<L.sm_count, kVqThreads, gu_smem(), s>>>(pv->map_x, a);
    else vq_gateup_kernel<false><<<L.sm_count, kVqThreads, gu_smem(), s>>>(pv->map_x, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev) record_phase(ev[2], s);
    VqArgs b = a;
    b.w0 = proj(MOEQ_DOWN);
    b.w1 = VqProj{nullptr, nullptr, nullptr, nullptr, nullptr};
    if (g1) vq_down_kernel<true><<<L.sm_count, kVqThreads, dn_smem(), s>>>(pv->map_h, b);
    else vq_down_kernel<false><<<L.sm_count, kVqThreads, dn_smem(), s>>>(pv->map_h, b);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev) record_phase(ev[3], s);
    const long long n = (long long)T * H;
    vq_cast_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(L.acc, reinterpret_cast<__nv_bfloat16 *>(out), n);
    if (ev) record_phase(ev[4], s);
    return cudaGetLastError();
}

}  // namespace moeq
