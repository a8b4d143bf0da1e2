// prefill_mx.cu -- MXFP4 routed-expert FFN at prefill sizes (more than 8
// tokens, bf16 activations) on the 5th-generation tensor cores.
//
// Layer: out[t] = sum_s w[t,s] W_down,e (silu(W_gate,e x_t) * (W_up,e x_t))
// ("MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture notes":
// 8 of 256 routed experts per token, MXFP4 experts with one E8M0 exponent per
// 32 values; "Speed": prefill runs in micro-batches of 2048 tokens and each
// expert's tokens are gathered into one matmul; "Recipe": intermediates keep
// f32's range).
//
// The weights never pass through the SM's arithmetic: tcgen05.mma
// kind::mxf8f6f4.block_scale multiplies the E2M1 codes as stored, with their
// E8M0 block scales in tensor memory.  The other operand must be an 8-bit
// (or narrower) float with its own E8M0 scale per 32 values, so every
// activation block is written as x = 2^s (q1 + q2), q1 = RN_E4M3(x 2^-s),
// q2 = RN_E4M3(x 2^-s - q1), s chosen so that max|x| 2^-s lies in [128,
// 256).  For bf16 x (8 significant bits) q1 + q2 is exact (q1 keeps 4 bits,
// the remainder has at most 4); for the f32 intermediates h it keeps about
// 8 bits.  Two MMAs (one per term) accumulate into the same f32 tensor-
// memory tile, so the products are exact and the sums are f32.
//
// Steps of one forward (all on the stream, no host synchronisation):
//   route/bucket (route.cu)  -> offsets[E+1], perm (route ids by expert)
//   pf_tiles_kernel          -> tile_base[E+1]: expert e's routes form
//                               ceil(n_e/64) tiles of up to 64 routes
//   pf_quant_x_kernel        -> q1, q2 [route position][H] and their scale
//                               atoms, one row per route (a gather of x)
//   pf_gateup_kernel         -> per (route tile, 128 rows of I): gate and up
//                               tiles in tensor memory, SwiGLU in f32, h
//                               quantised the same way for the down matmul
//   pf_down_kernel           -> per (route tile, 128 rows of H): y tile,
//                               weighted by w[t,s] and added into acc[T][H]
//   pf_cast_kernel           -> out = bf16(acc)
//
// Data in HBM: each projection's codes in their logical layout [E*N][K/2]
// (read by TMA tensor copies that widen each 16-value packet to 16 bytes in
// shared memory, as the MMA wants E2M1 operands), and its scales re-laid
// into 512-byte atoms [E][N/128][K/128][32 rows][4 row groups][4 blocks]:
// the shared-memory image that tcgen05.cp copies into tensor memory.
//
// CTA roles (one CTA per SM, persistent over work items): warp 0 issues TMA
// copies into a ring of stages, warp 1 issues the MMAs (one thread) and owns
// the tensor memory (two accumulator buffers, so that the epilogue of one
// work item overlaps the MMAs of the next), warps 2..5 run the epilogue.
// Every wait is bounded;
// on expiry the kernel sets MOEQ_ERR_TIMEOUT, every role stops, and the
// tensor memory is released.
#include <cuda.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <mutex>

#include "async.cuh"
#include "internal.cuh"
#include "umma.cuh"

namespace moeq {
namespace {

using namespace umma;
constexpr int kPfThreads = 192;   // producer, MMA, 4 epilogue warps
constexpr int kBoxA = 8192;       // bytes one A box moves from HBM (128 rows x 128 E2M1 codes)
constexpr int kTileA = 16384;     // shared-memory bytes of one 128 x 128 A tile (codes widened)
constexpr int kTileB = 8192;      // shared-memory bytes of one 64-route x 128 B tile (E4M3)
constexpr int kAtom = 512;        // one scale-factor atom: 128 rows x 4 blocks of 32

// gate/up stage: [A gate][A up][B q1][B q2][SF gate][SF up][SF x], padded to 1 KB
constexpr int kGUStage = 2 * kTileA + 2 * kTileB + 3 * kAtom + 512;
constexpr int kGUStages = 4;
// down stage: [A down][B q1][B q2][SF down][SF h]
constexpr int kDNStage = kTileA + 2 * kTileB + 2 * kAtom;
constexpr int kDNStages = 6;
constexpr int kDNFill = 3;        // stages the producer fills per step

// tensor memory: two accumulator buffers (the epilogue of one item overlaps
// the MMAs of the next), then a scale-factor ring (4 columns per atom)
constexpr int kGUTmemCols = 512;   // 2 x (gate 64 + up 64), SF ring 4 stages x 12
constexpr int kDNTmemCols = 256;   // 2 x y 64, SF ring 6 stages x 8


// 2^s for s in [-126, 127]
__device__ __forceinline__ float pow2i(int s) { return __uint_as_float((uint32_t)(s + 127) << 23); }

// Split v (|v| < 256 after scaling) into two E4M3 terms, v = q1 + q2 (to the
// precision E4M3 keeps of the remainder).  Round to nearest even.
__device__ __forceinline__ void split_e4m3(float v, uint8_t &q1, uint8_t &q2) {
    const __nv_fp8_storage_t a = __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
    const float av = __half2float(__half(__nv_cvt_fp8_to_halfraw(a, __NV_E4M3)));
    const __nv_fp8_storage_t b = __nv_cvt_float_to_fp8(v - av, __NV_SATFINITE, __NV_E4M3);
    q1 = a;
    q2 = b;
}

// Block scale exponent for a block whose largest magnitude is m: m 2^-s in
// [128, 256); 0 for an all-zero block.  Kept inside E8M0's range.
__device__ __forceinline__ int block_exp(float m) {
    if (!(m > 0.f)) return 0;
    const int eb = (int)((__float_as_uint(m) >> 23) & 0xFF);
    int s = (eb ? eb - 127 : -127) - 7;
    return s < -127 ? -127 : (s > 127 ? 127 : s);
}
// v * 2^-s without leaving f32's range in the intermediate factor
__device__ __forceinline__ float scale_down(float v, int s) {
    const int a = -s / 2, b = -s - a;
    return v * pow2i(a) * pow2i(b);
}

// ---------------------------------------------------------------- small kernels

// tile_base[e] = sum over e' < e of ceil(n_e' / 64); tile_base[E] = all tiles.
__global__ void __launch_bounds__(1024) pf_tiles_kernel(const int32_t *__restrict__ offsets, int E,
                                                        int32_t *__restrict__ tile_base) {
    __shared__ int32_t warp_off[32];
    __shared__ int32_t chunk_total;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 1024) {
        const int e = e0 + tid;
        const int v = e < E ? (offsets[e + 1] - offsets[e] + kRT - 1) / kRT : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_off[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int ws = warp_off[lane];
            int wi = ws;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += y;
            }
            warp_off[lane] = wi - ws;
            if (lane == 31) chunk_total = wi;
        }
        __syncthreads();
        if (e < E) tile_base[e] = carry + warp_off[warp] + incl - v;
        carry += chunk_total;
        __syncthreads();
    }
    if (tid == 0) tile_base[E] = carry;
}

// One warp per route position p: x of its token, split into two E4M3 rows
// and a scale per 32 values, stored at row p (the gather by expert).
__global__ void __launch_bounds__(256) pf_quant_x_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ perm,
                                                         const int32_t *__restrict__ ids, const int32_t *__restrict__ offsets,
                                                         const int32_t *__restrict__ tile_base, int E, int k, int H,
                                                         uint8_t *__restrict__ q1, uint8_t *__restrict__ q2,
                                                         uint8_t *__restrict__ sfx) {
    const int n_valid = __ldg(offsets + E);
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int n_warps = (gridDim.x * blockDim.x) >> 5;
    for (int p = warp; p < n_valid; p += n_warps) {
        const int r = __ldg(perm + p), t = r / k, e = __ldg(ids + r);
        const int l = p - __ldg(offsets + e), tau = __ldg(tile_base + e) + l / kRT, row = l % kRT;
        const uint16_t *xr = x + (size_t)t * H;
        // lane handles 32-blocks lane, lane+32, ...
        for (int b = lane; b < H / 32; b += 32) {
            float v[32];
            const uint4 *src = reinterpret_cast<const uint4 *>(xr + b * 32);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 w = __ldg(src + c);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[c * 8 + 2 * j] = __uint_as_float(ww[j] << 16);
                    v[c * 8 + 2 * j + 1] = __uint_as_float(ww[j] & 0xFFFF0000u);
                }
            }
            float m = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
            const int s = block_exp(m);
            uint32_t o1[8], o2[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t a = 0, bb = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint8_t u1, u2;
                    split_e4m3(scale_down(v[4 * i + j], s), u1, u2);
                    a |= (uint32_t)u1 << (8 * j);
                    bb |= (uint32_t)u2 << (8 * j);
                }
                o1[i] = a;
                o2[i] = bb;
            }
            uint4 *d1 = reinterpret_cast<uint4 *>(q1 + (size_t)p * H + b * 32);
            uint4 *d2 = reinterpret_cast<uint4 *>(q2 + (size_t)p * H + b * 32);
            d1[0] = make_uint4(o1[0], o1[1], o1[2], o1[3]);
            d1[1] = make_uint4(o1[4], o1[5], o1[6], o1[7]);
            d2[0] = make_uint4(o2[0], o2[1], o2[2], o2[3]);
            d2[1] = make_uint4(o2[4], o2[5], o2[6], o2[7]);
            sfx[((size_t)tau * (H / kT) + b / 4) * kAtom + atom_byte(row, b % 4)] = (uint8_t)(s + 127);
        }
    }
}

// Weight scales [ne][N][K/32] -> atoms [ne][N/128][K/128][512].
__global__ void pf_sf_atoms_kernel(const uint8_t *__restrict__ sc, int ne, int N, int K, uint8_t *__restrict__ atoms) {
    const long long n = (long long)ne * N * (K / 32);
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int kb = (int)(i % (K / 32));
    const long long rowg = i / (K / 32);
    const int row = (int)(rowg % N);
    const long long e = rowg / N;
    const size_t atom = ((size_t)(e * (N / kT) + row / kT) * (K / kT) + kb / 4);
    atoms[atom * kAtom + atom_byte(row % kT, kb % 4)] = sc[i];
}

__global__ void pf_cast_kernel(const float *__restrict__ acc, __nv_bfloat16 *__restrict__ out, long long n) {
    const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (i + 3 < n) {
        const float4 v = *reinterpret_cast<const float4 *>(acc + i);
        out[i] = __float2bfloat16_rn(v.x);
        out[i + 1] = __float2bfloat16_rn(v.y);
        out[i + 2] = __float2bfloat16_rn(v.z);
        out[i + 3] = __float2bfloat16_rn(v.w);
    } else {
        for (long long j = i; j < n; ++j) out[j] = __float2bfloat16_rn(acc[j]);
    }
}

// ---------------------------------------------------------------- gate/up

struct PfArgs {
    const int32_t *offsets, *tile_base, *perm, *ids;
    const float *topk_w;
    const uint8_t *sfa0, *sfa1;   // weight scale atoms: gate, up (or down in sfa0)
    const uint8_t *sfb;           // activation scale atoms [tiles][K/128][512]
    uint8_t *hq1, *hq2, *sfh;     // gate/up: quantised h and its scale atoms
    float *acc;                   // down: f32 output accumulator [T][H]
    uint32_t *status;
    long long wait_cycles;        // limit of every wait but the final drains
    int E, H, I, k;
};

__global__ void __launch_bounds__(kPfThreads, 1)
    pf_gateup_kernel(const __grid_constant__ CUtensorMap tWg, const __grid_constant__ CUtensorMap tWu,
                     const __grid_constant__ CUtensorMap tX1, const __grid_constant__ CUtensorMap tX2, PfArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[kGUStages], empty[kGUStages], tmem_full[2], tmem_empty[2], tmem_done;
    __shared__ uint32_t tslot;
    __shared__ volatile int abort_flag;
    __shared__ RouteTables rt;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, I = a.I, E = a.E;
    const int subs = I / kT, slabs = H / kT;

    if (tid == 0) {
        for (int s = 0; s < kGUStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 1);
            mbar_init(&tmem_empty[b], 4);
        }
        mbar_init(&tmem_done, 1);
        mbar_fence_init();
        abort_flag = 0;
    }
    load_route_tables(rt, a.offsets, a.tile_base, a.E);
    if (warp == 1) tc_alloc(&tslot, kGUTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    const uint32_t t_sf = tmem + 4 * kRT;   // buffer b: gate at b*128, up at b*128 + 64
    const int n_items = rt.tb[E] * subs;

    if (warp == 0) {
        // Each work item's tile coordinates are decoded once; its slabs are
        // then streamed stage by stage: lane 0 waits for the stage to be
        // released and arms it, lanes 0..6 issue its seven copies at once.
        int c = 0, s = 0;
        uint32_t rp = 0;   // parity of the current round of the stage ring
        bool ok = true;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            const Item m = decode_item(rt.off, rt.tb, E, subs, it);
            const int wrow = m.e * I + m.sub * kT;
            const size_t wsf = (size_t)(m.e * subs + m.sub) * slabs * kAtom, xsf = (size_t)m.tau * slabs * kAtom;
            for (int sl = 0; sl < slabs; ++sl, ++c) {
                if (lane == 0 && c >= kGUStages) ok = wait_or_abort(&empty[s], rp ^ 1u, &abort_flag, a.wait_cycles);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) mbar_arrive_expect_tx(&full[s], 2 * kBoxA + 2 * kTileB + 3 * kAtom);
                __syncwarp();
                uint8_t *st = smem + (size_t)s * kGUStage;
                uint8_t *sf = st + 2 * kTileA + 2 * kTileB;
                switch (lane) {
                    case 0: tma_load_2d(st, &tWg, sl * kT, wrow, &full[s]); break;
                    case 1: tma_load_2d(st + kTileA, &tWu, sl * kT, wrow, &full[s]); break;
                    case 2: tma_load_2d(st + 2 * kTileA, &tX1, sl * kT, m.row0, &full[s]); break;
                    case 3: tma_load_2d(st + 2 * kTileA + kTileB, &tX2, sl * kT, m.row0, &full[s]); break;
                    case 4: bulk_g2s(sf, a.sfa0 + wsf + (size_t)sl * kAtom, kAtom, &full[s]); break;
                    case 5: bulk_g2s(sf + kAtom, a.sfa1 + wsf + (size_t)sl * kAtom, kAtom, &full[s]); break;
                    case 6: bulk_g2s(sf + 2 * kAtom, a.sfb + xsf + (size_t)sl * kAtom, kAtom, &full[s]); break;
                    default: break;
                }
                __syncwarp();
                if (++s == kGUStages) {
                    s = 0;
                    rp ^= 1u;
                }
            }
        }
        if (lane == 0) drain_stages(full, kGUStages, c);
    } else if (warp == 1) {
        if (lane == 0) {
            int c = 0, q = 0;
            for (int it = blockIdx.x; it < n_items && !abort_flag; it += gridDim.x, ++q) {
                const Item m = decode_item(rt.off, rt.tb, E, subs, it);
                const int n = (m.cnt + 15) & ~15, b = q & 1;
                if (q >= 2 && !wait_or_abort(&tmem_empty[b], (uint32_t)(((q >> 1) - 1) & 1), &abort_flag, a.wait_cycles)) break;
                tc_fence_after();
                const uint32_t t_g = tmem + b * 2 * kRT, t_u = t_g + kRT;
                for (int sl = 0; sl < slabs; ++sl, ++c) {
                    const int s = c % kGUStages;
                    if (!wait_or_abort(&full[s], (uint32_t)((c / kGUStages) & 1), &abort_flag, a.wait_cycles)) break;
                    tc_fence_after();
                    const uint8_t *st = smem + (size_t)s * kGUStage;
                    const uint8_t *sf = st + 2 * kTileA + 2 * kTileB;
                    const uint32_t sfg = t_sf + 12 * s, sfu = sfg + 4, sfx = sfg + 8;
                    tc_cp_atom(sfg, sf);
                    tc_cp_atom(sfu, sf + kAtom);
                    tc_cp_atom(sfx, sf + 2 * kAtom);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t id = idesc_mx(n, kk, kk);
                        const uint64_t ag = desc_sw128(st + kk * 32), au = desc_sw128(st + kTileA + kk * 32);
                        const uint64_t b1 = desc_sw128(st + 2 * kTileA + kk * 32);
                        const uint64_t b2 = desc_sw128(st + 2 * kTileA + kTileB + kk * 32);
                        const uint32_t acc = (sl > 0 || kk > 0) ? 1u : 0u;
                        mma_mx(t_g, ag, b1, id, acc, sfg, sfx);
                        mma_mx(t_g, ag, b2, id, 1u, sfg, sfx);
                        mma_mx(t_u, au, b1, id, acc, sfu, sfx);
                        mma_mx(t_u, au, b2, id, 1u, sfu, sfx);
                    }
                    tc_commit(&empty[s]);
                }
                tc_commit(&tmem_full[b]);
            }
            drain_mma(&tmem_done);
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 = rows of I
        const int qd = warp & 3;
        int q = 0;
        for (int it = blockIdx.x; it < n_items && !abort_flag; it += gridDim.x, ++q) {
            const Item m = decode_item(rt.off, rt.tb, E, subs, it);
            const int b = q & 1;
            if (!wait_or_abort(&tmem_full[b], (uint32_t)((q >> 1) & 1), &abort_flag, a.wait_cycles)) break;
            tc_fence_after();
            const int i_row = m.sub * kT + 32 * qd + lane;   // this lane's row of I
            const uint32_t t_g = tmem + b * 2 * kRT + ((uint32_t)(32 * qd) << 16), t_u = t_g + kRT;
            uint8_t *sfh = a.sfh + ((size_t)m.tau * subs + m.sub) * kAtom;
            for (int n0 = 0; n0 < m.cnt; n0 += 16) {
                float g[16], u[16];
                tc_ld16(t_g + n0, g);
                tc_ld16(t_u + n0, u);
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const int n = n0 + jj;
                    if (n >= m.cnt) break;
                    const float h = silu_f32(g[jj]) * u[jj];
                    // the 32 rows of this warp are one 32-block of the down matmul's K
                    const float ah = fabsf(h);
                    const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(isfinite(ah) ? ah : 3.0e38f));
                    const int s = block_exp(__uint_as_float(mb));
                    uint8_t b1, b2;
                    split_e4m3(scale_down(h, s), b1, b2);
                    const size_t p = (size_t)(m.row0 + n);
                    a.hq1[p * I + i_row] = b1;
                    a.hq2[p * I + i_row] = b2;
                    if (lane == 0) sfh[atom_byte(n, qd)] = (uint8_t)(s + 127);
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
        tc_dealloc(tmem, kGUTmemCols);
    }
}

// ---------------------------------------------------------------- down

__global__ void __launch_bounds__(kPfThreads, 1)
    pf_down_kernel(const __grid_constant__ CUtensorMap tWd, const __grid_constant__ CUtensorMap tH1,
                   const __grid_constant__ CUtensorMap tH2, PfArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[kDNStages], empty[kDNStages], tmem_full[2], tmem_empty[2], tmem_done;
    __shared__ uint32_t tslot;
    __shared__ volatile int abort_flag;
    __shared__ RouteTables rt;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H, I = a.I, E = a.E, k = a.k;
    const int subs = H / kT, slabs = I / kT;

    if (tid == 0) {
        for (int s = 0; s < kDNStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full[b], 1);
            mbar_init(&tmem_empty[b], 4);
        }
        mbar_init(&tmem_done, 1);
        mbar_fence_init();
        abort_flag = 0;
    }
    load_route_tables(rt, a.offsets, a.tile_base, a.E);
    if (warp == 1) tc_alloc(&tslot, kDNTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tslot;
    const uint32_t t_sf = tmem + 2 * kRT;   // buffer b at b*64
    const int n_items = rt.tb[E] * subs;

    if (warp == 0) {
        // kDNFill stages per step: lanes g < kDNFill wait for and arm stage
        // c0 + g, then lanes 5g + j issue copy j of it.  A down stage carries
        // half the MMAs of a gate/up stage, and refilling three stages per
        // step measured faster here than one at a time.
        const int my_items = n_items > (int)blockIdx.x ? (n_items - (int)blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
        const int total = my_items * slabs;
        const int g = lane / 5, j = lane % 5;
        int c0 = 0;
        for (; c0 < total; c0 += kDNFill) {
            const int c = c0 + (lane < kDNFill ? lane : 0), s = c % kDNStages;
            bool ok = true;
            if (lane < kDNFill && c < total && c >= kDNStages)
                ok = wait_or_abort(&empty[s], (uint32_t)((c / kDNStages - 1) & 1), &abort_flag, a.wait_cycles);
            if (__any_sync(0xffffffffu, !ok)) break;
            if (lane < kDNFill && c < total) mbar_arrive_expect_tx(&full[s], kBoxA + 2 * kTileB + 2 * kAtom);
            __syncwarp();
            const int cc = c0 + g;
            if (g < kDNFill && cc < total) {
                const int sc = cc % kDNStages, sl = cc % slabs;
                const Item m = decode_item(rt.off, rt.tb, E, subs, blockIdx.x + (cc / slabs) * gridDim.x);
                uint8_t *st = smem + (size_t)sc * kDNStage;
                uint8_t *sf = st + kTileA + 2 * kTileB;
                switch (j) {
                    case 0: tma_load_2d(st, &tWd, sl * kT, m.e * H + m.sub * kT, &full[sc]); break;
                    case 1: tma_load_2d(st + kTileA, &tH1, sl * kT, m.row0, &full[sc]); break;
                    case 2: tma_load_2d(st + kTileA + kTileB, &tH2, sl * kT, m.row0, &full[sc]); break;
                    case 3: bulk_g2s(sf, a.sfa0 + ((size_t)(m.e * subs + m.sub) * slabs + sl) * kAtom, kAtom, &full[sc]); break;
                    default: bulk_g2s(sf + kAtom, a.sfb + ((size_t)m.tau * slabs + sl) * kAtom, kAtom, &full[sc]); break;
                }
            }
            __syncwarp();
        }
        if (lane == 0) drain_stages(full, kDNStages, c0 < total ? c0 : total);
    } else if (warp == 1) {
        if (lane == 0) {
            int c = 0, q = 0;
            for (int it = blockIdx.x; it < n_items && !abort_flag; it += gridDim.x, ++q) {
                const Item m = decode_item(rt.off, rt.tb, E, subs, it);
                const int n = (m.cnt + 15) & ~15, b = q & 1;
                if (q >= 2 && !wait_or_abort(&tmem_empty[b], (uint32_t)(((q >> 1) - 1) & 1), &abort_flag, a.wait_cycles)) break;
                tc_fence_after();
                const uint32_t t_y = tmem + b * kRT;
                for (int sl = 0; sl < slabs; ++sl, ++c) {
                    const int s = c % kDNStages;
                    if (!wait_or_abort(&full[s], (uint32_t)((c / kDNStages) & 1), &abort_flag, a.wait_cycles)) break;
                    tc_fence_after();
                    const uint8_t *st = smem + (size_t)s * kDNStage;
                    const uint8_t *sf = st + kTileA + 2 * kTileB;
                    const uint32_t sfw = t_sf + 8 * s, sfh = sfw + 4;
                    tc_cp_atom(sfw, sf);
                    tc_cp_atom(sfh, sf + kAtom);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t id = idesc_mx(n, kk, kk);
                        const uint64_t aw = desc_sw128(st + kk * 32);
                        const uint64_t b1 = desc_sw128(st + kTileA + kk * 32);
                        const uint64_t b2 = desc_sw128(st + kTileA + kTileB + kk * 32);
                        const uint32_t acc = (sl > 0 || kk > 0) ? 1u : 0u;
                        mma_mx(t_y, aw, b1, id, acc, sfw, sfh);
                        mma_mx(t_y, aw, b2, id, 1u, sfw, sfh);
                    }
                    tc_commit(&empty[s]);
                }
                tc_commit(&tmem_full[b]);
            }
            drain_mma(&tmem_done);
        }
    } else {
        const int qd = warp & 3;
        int q = 0;
        for (int it = blockIdx.x; it < n_items && !abort_flag; it += gridDim.x, ++q) {
            const Item m = decode_item(rt.off, rt.tb, E, subs, it);
            const int b = q & 1;
            // the tile's routes: token and weight, two per lane, shared by shuffles
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
            const int h_row = m.sub * kT + 32 * qd + lane;   // this lane's output feature
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
        tc_dealloc(tmem, kDNTmemCols);
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D tensor map over `rows` rows of `cols` elements, boxes of 128 elements x
// `box_rows` rows, 128B swizzle.
cudaError_t make_map(CUtensorMap *map, bool e2m1, void *base, long long cols, long long rows, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(e2m1 ? cols / 2 : cols)};
    const cuuint32_t box[2] = {(cuuint32_t)kT, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    const CUresult r = fn(map, e2m1 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base,
                          dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

size_t gu_smem() { return (size_t)kGUStages * kGUStage + 1024; }
size_t dn_smem() { return (size_t)kDNStages * kDNStage + 1024; }

}  // namespace

cudaError_t launch_route_tiles(const int32_t *offsets, int E, int32_t *tile_base, cudaStream_t s) {
    pf_tiles_kernel<<<1, 1024, 0, s>>>(offsets, E, tile_base);
    return cudaGetLastError();
}

bool prefill_mx_supported(const Layer &L, int T) {
    return L.pf != nullptr && L.pf->maps_ready && T > kDecMaxTokens && L.d.fmt == MOEQ_FMT_MXFP4 &&
           L.d.act == MOEQ_ACT_BF16;
}

cudaError_t prefill_mx_create(Layer &L) {
    const moeq_layer_desc &d = L.d;
    if (d.fmt != MOEQ_FMT_MXFP4 || d.act != MOEQ_ACT_BF16 || d.max_tokens <= kDecMaxTokens) return cudaSuccess;
    if (d.hidden % kT || d.inter % kT) return cudaSuccess;
    PrefillMx *pf = new (std::nothrow) PrefillMx();
    if (!pf) return cudaErrorMemoryAllocation;
    L.pf = pf;
    const int E = d.n_experts, H = d.hidden, I = d.inter;
    const size_t R = (size_t)d.max_tokens * d.top_k;          // route positions
    const size_t tiles = R / kRT + (size_t)E;                  // upper bound on route tiles
    cudaError_t e = cudaSuccess;
    auto al = [&](void **p, size_t n) {
        if (e == cudaSuccess) e = dev_alloc(p, n);
    };
    for (int p = 0; p < 3; ++p) {
        const size_t N = p == MOEQ_DOWN ? H : I, K = p == MOEQ_DOWN ? I : H;
        al((void **)&pf->codes[p], (size_t)E * N * K / 2);
        al((void **)&pf->sf_atoms[p], (size_t)E * N * K / 32);
    }
    al((void **)&pf->tile_base, sizeof(int32_t) * (E + 1));
    al((void **)&pf->xq[0], R * H);
    al((void **)&pf->xq[1], R * H);
    al((void **)&pf->sfx, tiles * (H / kT) * kAtom);
    al((void **)&pf->hq[0], R * I);
    al((void **)&pf->hq[1], R * I);
    al((void **)&pf->sfh, tiles * (I / kT) * kAtom);
    // rows and scale atoms of route positions beyond a tile's routes are read
    // by the MMAs (their columns are discarded): keep them finite
    if (e == cudaSuccess) e = cudaMemset(pf->xq[0], 0, R * H);
    if (e == cudaSuccess) e = cudaMemset(pf->xq[1], 0, R * H);
    if (e == cudaSuccess) e = cudaMemset(pf->hq[0], 0, R * I);
    if (e == cudaSuccess) e = cudaMemset(pf->hq[1], 0, R * I);
    if (e == cudaSuccess) e = cudaMemset(pf->sfx, 127, tiles * (H / kT) * kAtom);
    if (e == cudaSuccess) e = cudaMemset(pf->sfh, 127, tiles * (I / kT) * kAtom);
    if (e != cudaSuccess) return e;
    // activation operand maps; rows past the last route position read as zeros
    e = make_map(&pf->map_x[0], false, pf->xq[0], H, (long long)R, kRT);
    if (e == cudaSuccess) e = make_map(&pf->map_x[1], false, pf->xq[1], H, (long long)R, kRT);
    if (e == cudaSuccess) e = make_map(&pf->map_h[0], false, pf->hq[0], I, (long long)R, kRT);
    if (e == cudaSuccess) e = make_map(&pf->map_h[1], false, pf->hq[1], I, (long long)R, kRT);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(pf_gateup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gu_smem());
    if (e == cudaSuccess) e = cudaFuncSetAttribute(pf_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dn_smem());
    // without the driver's tensor-map encoder this path stays off
    if (e == cudaErrorNotSupported) e = cudaSuccess;
    return e;
}

void prefill_mx_free(Layer &L) {
    PrefillMx *pf = L.pf;
    if (!pf) return;
    for (int p = 0; p < 3; ++p) {
        cudaFree(pf->codes[p]);
        cudaFree(pf->sf_atoms[p]);
    }
    cudaFree(pf->tile_base);
    cudaFree(pf->xq[0]);
    cudaFree(pf->xq[1]);
    cudaFree(pf->sfx);
    cudaFree(pf->hq[0]);
    cudaFree(pf->hq[1]);
    cudaFree(pf->sfh);
    delete pf;
    L.pf = nullptr;
}

cudaError_t prefill_mx_upload(Layer &L, int p, const uint8_t *codes, const uint8_t *scales, int e0, int ne,
                              cudaStream_t s) {
    PrefillMx *pf = L.pf;
    if (!pf) return cudaSuccess;
    const int H = L.d.hidden, I = L.d.inter;
    const int N = p == MOEQ_DOWN ? H : I, K = p == MOEQ_DOWN ? I : H;
    cudaError_t e = cudaMemcpyAsync(pf->codes[p] + (size_t)e0 * N * (K / 2), codes, (size_t)ne * N * (K / 2),
                                    cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return e;
    const long long n = (long long)ne * N * (K / 32);
    pf_sf_atoms_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(scales, ne, N, K,
                                                                   pf->sf_atoms[p] + (size_t)e0 * N * (K / 32));
    return cudaGetLastError();
}

cudaError_t prefill_mx_finish_upload(Layer &L) {
    PrefillMx *pf = L.pf;
    if (!pf) return cudaSuccess;
    const int E = L.d.n_experts, H = L.d.hidden, I = L.d.inter;
    cudaError_t e = make_map(&pf->map_w[MOEQ_GATE], true, pf->codes[MOEQ_GATE], H, (long long)E * I, kT);
    if (e == cudaSuccess) e = make_map(&pf->map_w[MOEQ_UP], true, pf->codes[MOEQ_UP], H, (long long)E * I, kT);
    if (e == cudaSuccess) e = make_map(&pf->map_w[MOEQ_DOWN], true, pf->codes[MOEQ_DOWN], I, (long long)E * H, kT);
    pf->maps_ready = e == cudaSuccess;
    return e == cudaErrorNotSupported ? cudaSuccess : e;
}

cudaError_t launch_prefill_mx(const Layer &L, const void *x, const int32_t *ids, const float *topk_w, int T, void *out,
                              cudaStream_t s, const cudaEvent_t *ev) {
    const PrefillMx *pf = L.pf;
    const int E = L.d.n_experts, H = L.d.hidden, I = L.d.inter, k = L.d.top_k;
    cudaError_t e = launch_route_bucket(L, ids, T * k, L.b.offsets, L.b.perm, L.b.active, s);
    if (e != cudaSuccess) return e;
    if (ev) record_phase(ev[1], s);
    L.count_launches(5);
    pf_tiles_kernel<<<1, 1024, 0, s>>>(L.b.offsets, E, pf->tile_base);
    e = cudaMemsetAsync(L.acc, 0, sizeof(float) * (size_t)T * H, s);
    if (e != cudaSuccess) return e;
    {
        const int warps = T * k < 148 * 16 ? T * k : 148 * 16;
        pf_quant_x_kernel<<<(warps + 7) / 8, 256, 0, s>>>(reinterpret_cast<const uint16_t *>(x), L.b.perm, ids,
                                                          L.b.offsets, pf->tile_base, E, k, H, pf->xq[0], pf->xq[1],
                                                          pf->sfx);
    }
    PfArgs a{};
    a.offsets = L.b.offsets;
    a.tile_base = pf->tile_base;
    a.perm = L.b.perm;
    a.ids = ids;
    a.topk_w = topk_w;
    a.status = L.status;
    a.wait_cycles = L.wait_cycles;
    a.E = E;
    a.H = H;
    a.I = I;
    a.k = k;
    a.sfa0 = pf->sf_atoms[MOEQ_GATE];
    a.sfa1 = pf->sf_atoms[MOEQ_UP];
    a.sfb = pf->sfx;
    a.hq1 = pf->hq[0];
    a.hq2 = pf->hq[1];
    a.sfh = pf->sfh;
    pf_gateup_kernel<<<L.sm_count, kPfThreads, gu_smem(), s>>>(pf->map_w[MOEQ_GATE], pf->map_w[MOEQ_UP], pf->map_x[0],
                                                               pf->map_x[1], a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev) record_phase(ev[2], s);
    PfArgs b = a;
    b.sfa0 = pf->sf_atoms[MOEQ_DOWN];
    b.sfa1 = nullptr;
    b.sfb = pf->sfh;
    b.acc = L.acc;
    pf_down_kernel<<<L.sm_count, kPfThreads, dn_smem(), s>>>(pf->map_w[MOEQ_DOWN], pf->map_h[0], pf->map_h[1], b);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (ev) record_phase(ev[3], s);
    const long long n = (long long)T * H;
    pf_cast_kernel<<<(unsigned)((n / 4 + 255) / 256), 256, 0, s>>>(L.acc, reinterpret_cast<__nv_bfloat16 *>(out), n);
    if (ev) record_phase(ev[4], s);
    return cudaGetLastError();
}

}  // namespace moeq
