// decode_common.cuh -- pieces shared by the decode-size kernels (1..8
// tokens): the per-CTA route table built from topk_ids / topk_w, and the
// power-of-two prescale of an f16 operand.
#pragma once

#include "internal.cuh"

namespace moeq {
namespace dec {

constexpr int kMaxR = kDecMaxRoutes;   // routes of one decode call (T * k)

struct RouteTable {
    int D;                   // experts with at least one valid route
    int n_valid;
    int expert[kMaxR];       // those experts, ascending
    int col_beg[kMaxR + 1];  // routes of expert slot d: route[col_beg[d] .. col_beg[d+1])
    int route[kMaxR];        // valid route ids sorted by (expert, route id)
    int sid[kMaxR];          // copy of topk_ids
    float w[kMaxR];          // copy of topk_w (kept on chip: a global load per unit stalls the warps)
    uint8_t tok[kMaxR];      // token of route id r (r / k)
};

// Warp 0 builds the table (R = T*k <= 64 routes).
__device__ inline void build_route_table(RouteTable &tb, const int32_t *__restrict__ ids, const float *__restrict__ topk_w,
                                  int R, int k, int E, uint32_t *status, bool report) {
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    const int r0 = lane, r1 = lane + 32;
    // all four loads in flight before the first use: one memory round trip
    const int id0 = r0 < R ? __ldg(ids + r0) : -1, id1 = r1 < R ? __ldg(ids + r1) : -1;
    const float w0 = r0 < R ? __ldg(topk_w + r0) : 0.f, w1 = r1 < R ? __ldg(topk_w + r1) : 0.f;
    if (r0 < R) {
        tb.sid[r0] = id0;
        tb.w[r0] = w0;
        tb.tok[r0] = (uint8_t)(r0 / k);
    }
    if (r1 < R) {
        tb.sid[r1] = id1;
        tb.w[r1] = w1;
        tb.tok[r1] = (uint8_t)(r1 / k);
    }
    const bool v0 = id0 >= 0 && id0 < E, v1 = id1 >= 0 && id1 < E;
    const bool bad = (r0 < R && !v0 && id0 != -1) || (r1 < R && !v1 && id1 != -1);
    if (report && __any_sync(full, bad) && lane == 0) atomicOr(status, FLAG_ROUTE_RANGE);
    int rank0 = 0, rank1 = 0;
#pragma unroll 8
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


}  // namespace dec
}  // namespace moeq
