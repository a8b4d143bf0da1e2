// umma.cuh -- tcgen05 (5th-generation tensor core) and TMA helpers shared by
// the prefill kernels, plus the route-tile work decomposition.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "async.cuh"
#include "internal.cuh"

namespace moeq {
namespace umma {

constexpr int kT = 128;           // MMA M (weight rows per tile)
constexpr int kRT = 64;           // routes per route tile: the largest MMA N used


__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Pull a future box of a tensor map into L2 (no shared memory involved).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}

// Shared-memory matrix descriptor, K-major.  128B swizzle: rows of 128 bytes,
// 8-row groups 1024 bytes apart.  None: 8 x 16-byte core matrices, groups of
// 8 rows `sbo` bytes apart, 16-byte columns `lbo` bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(const void *p) {
    return (uint64_t)((smem_u32(p) >> 4) & 0x3FFF) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}
__device__ __forceinline__ uint64_t desc_plain(const void *p, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((smem_u32(p) >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46);
}
// Instruction descriptor: kind::mxf8f6f4 block-scaled, A E2M1, B E4M3, f32
// accumulate, E8M0 scales, M 128, both operands K-major, K 32 per MMA;
// a_sf / b_sf pick the byte (the 32-block) of each scale-factor column.
__device__ __forceinline__ uint32_t idesc_mx(int n, int a_sf, int b_sf) {
    return ((uint32_t)(b_sf & 3) << 4) | (5u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) |
           ((uint32_t)(kT >> 4) << 24) | ((uint32_t)(a_sf & 3) << 29);
}
__device__ __forceinline__ void mma_mx(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc, uint32_t sfa,
                                       uint32_t sfb) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
}
__device__ __forceinline__ void tc_cp_atom(uint32_t taddr, const void *atom) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc_plain(atom, 128, 128))
                 : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_alloc(uint32_t *slot, int cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, int cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
// 16 consecutive f32 columns of this warp's 32 lanes
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float v[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Bounded wait that also gives up once another role has given up.  It polls
// with test_wait: a thread suspended in try_wait can resume well after the
// phase completed, and every hand-off between the roles is on the critical
// path.  `limit` is the layer's wait limit in SM clocks.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                              long long limit) {
    if (mbar_test_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_test_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// Before the CTA releases its shared and tensor memory: wait (bounded,
// whatever happened) for the copies of the last stages issued, and for every
// MMA this thread issued.
__device__ __forceinline__ void drain_stages(uint64_t *full, int S, int issued) {
    for (int c = issued > S ? issued - S : 0; c < issued; ++c)
        mbar_wait_bounded(&full[c % S], (uint32_t)((c / S) & 1), kDrainCycles);
}
__device__ __forceinline__ void drain_mma(uint64_t *done) {
    tc_commit(done);
    mbar_wait_bounded(done, 0, kDrainCycles);
}

// Scale-factor atom byte of (row r of a 128-row tile, 32-block kb of a 4-block group)
__device__ __forceinline__ int atom_byte(int r, int kb) { return (r & 31) * 16 + (r >> 5) * 4 + kb; }

// Expert of global route tile tau: the last e with tile_base[e] <= tau.
__device__ __forceinline__ int expert_of_tile(const int32_t *tile_base, int E, int tau) {
    int lo = 0, hi = E;   // tile_base[lo] <= tau < tile_base[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tile_base[mid] <= tau) lo = mid;
        else hi = mid;
    }
    return lo;
}

struct Item {
    int e, j, sub;     // expert, route tile of the expert, 128-row tile of the output
    int row0;          // first route position of the tile
    int cnt;           // routes in the tile (1..128)
    int tau;           // global route tile
};
// Shared-memory copies of the route offsets and route-tile bases (E <= 1024).
struct RouteTables {
    int32_t off[kMaxExperts + 1];
    int32_t tb[kMaxExperts + 1];
};
__device__ __forceinline__ void load_route_tables(RouteTables &rt, const int32_t *offsets, const int32_t *tile_base,
                                                  int E) {
    for (int i = threadIdx.x; i <= E; i += blockDim.x) {
        rt.off[i] = __ldg(offsets + i);
        rt.tb[i] = __ldg(tile_base + i);
    }
}

// offsets and tile_base are the kernel's shared-memory copies (see
// load_route_tables): the search runs once per work item and stage.
__device__ __forceinline__ Item decode_item(const int32_t *offsets, const int32_t *tile_base, int E, int subs,
                                            int it) {
    Item m;
    m.tau = it / subs;
    m.sub = it % subs;
    m.e = expert_of_tile(tile_base, E, m.tau);
    m.j = m.tau - tile_base[m.e];
    const int beg = offsets[m.e], n_e = offsets[m.e + 1] - beg;
    m.row0 = beg + kRT * m.j;
    m.cnt = min(kRT, n_e - kRT * m.j);
    return m;
}


}  // namespace umma
}  // namespace moeq
