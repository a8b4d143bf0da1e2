// router.cu -- the router that produces a forward's routing: logits
// z = Wr x (Wr [E][H] f32), the k largest per token (descending z, equal z
// to the lower expert id), and their weights: the sigmoid scores
// s = 1 / (1 + e^-z) of the selected experts divided by their sum, or a
// softmax over the selected logits.
//
// Source: "MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture
// notes": 256 routed experts, 8 active per token, no shared expert, sigmoid
// routing.  The router matrix's shape, the selection on the logits and the
// normalisation over the selected experts are readings (the page gives no
// more); the softmax weighting is the one the expert path's synthetic
// workloads use.
//
// bf16 activations: the logits run on the warp-level tensor cores
// (mma.sync m16n8k16, bf16 in, f32 accumulate) with the experts as the M
// dimension and the tokens as N, so a decode step of up to 8 tokens is one
// N tile.  Wr is stored at upload as three bf16 terms w1 + w2 + w3 (w1 =
// bf16(w), w2 = bf16(w - w1), w3 = bf16(w - w1 - w2), all differences exact
// in f32), so that every product with a bf16 activation is exact in f32 and
// the logit carries f32 accuracy, not bf16's.  The terms are laid out in the
// tensor-core A-fragment order: one 16-byte load per lane gives a warp its
// whole fragment of 16 experts x 16 K for one term, straight from global
// memory (the router matrix is read once per token tile; nothing is staged
// in shared memory).
// f32 activations: the same work split with f32 CUDA-core dot products
// (Wr stored transposed, [H][E], so a CTA's threads read rows coalesced).
//
// Work split: CTA (token tile of 32, K slice); each writes its partial
// logits [K slice][token][E], and the last CTA of a token tile to finish
// (arrival counter) sums the slices in slice order -- so the logits do not
// depend on timing -- selects and weights.
// Decode sizes (up to 8 tokens, either activation type): a GEMV on the CUDA
// cores instead, one CTA per expert row reading Wr as given ([E][H] f32,
// coalesced 16-byte loads, each byte once per call) with f32 FMAs (each
// product exact inside its FMA), the row's partial sums added in a fixed
// order; the last CTA to finish selects.  The tensor-core path would spend
// most of its work on the padding of a 32-token tile and read 1.5x the bytes.
#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "internal.cuh"

namespace moeq {
namespace {

constexpr int kRThreads = 256;            // 8 warps
constexpr int kRWarps = kRThreads / 32;
constexpr int kTileTok = 32;              // tokens per CTA (4 tensor-core N tiles)
constexpr int kMaxPerLane = kMaxExperts / 32;

// ------------------------------------------------------------ top-k + weights

// Warp-wide selection of the k largest of z[0..E) for one token: lane l
// holds z[l + 32 i] in v[i].  Writes ids/w (k entries).  score 0: sigmoid
// scores normalised over the selection; 1: softmax over the selection.
__device__ void select_topk(float (&v)[kMaxPerLane], int E, int k, int score, int32_t *ids, float *w,
                            float *sel_z) {
    const int lane = threadIdx.x & 31;
    const int per = (E + 31) / 32;
    uint32_t taken = 0u;
    for (int j = 0; j < k; ++j) {
        // this lane's best untaken candidate: largest z, then lowest id
        float bz = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            if (i >= per) break;
            const int e = lane + 32 * i;
            if (e >= E || ((taken >> i) & 1u)) continue;
            if (v[i] > bz || (v[i] == bz && e < be)) {
                bz = v[i];
                be = e;
            }
        }
        // warp arg-max with the same order
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (oz > bz || (oz == bz && oe < be)) {
                bz = oz;
                be = oe;
            }
        }
        if (be != 0x7fffffff && (be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == 0) {
            ids[j] = be;
            sel_z[j] = bz;
        }
    }
    __syncwarp();
    if (lane == 0) {
        // k <= 64 selected values; the first is the largest
        const float zmax = sel_z[0];
        float sum = 0.f;
        for (int j = 0; j < k; ++j) {
            const float s = score == 0 ? 1.0f / (1.0f + expf(-sel_z[j])) : expf(sel_z[j] - zmax);
            sel_z[j] = s;
            sum += s;
        }
        for (int j = 0; j < k; ++j) w[j] = sel_z[j] / sum;
    }
    __syncwarp();
}

// The last CTA of a token tile: the K slices of every logit of the tile
// summed in slice order, then one warp per token selects.  part:
// [nsplit][T][E].  With many slices (few token tiles) the whole CTA sums
// them first, in place of slice 0; with a few, each warp sums its token's.
__device__ void finish_tile(float *part, int nsplit, int T, int E, int k, int score, int t0, int32_t *topk_ids,
                            float *topk_w, float *logits, float (*sel)[kMaxTopK]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = min(kTileTok, T - t0);
    const bool presum = nsplit > 4;
    if (presum) {
        const size_t slice = (size_t)T * E;
        for (int i = threadIdx.x; i < nt * E; i += kRThreads) {
            float *p = part + (size_t)t0 * E + i;    // slice 0 of token t0 + i / E, expert i % E
            float s = __ldcg(p);
#pragma unroll 8
            for (int q = 1; q < nsplit; ++q) s += __ldcg(p + q * slice);
            __stcg(p, s);
        }
        __syncthreads();
    }
    const int per = (E + 31) / 32;
    for (int tt = warp; tt < nt; tt += kRWarps) {
        const int t = t0 + tt;
        float v[kMaxPerLane];
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            v[i] = 0.f;
            if (i >= per) continue;
            const int e = lane + 32 * i;
            if (e >= E) continue;
            float z = __ldcg(part + (size_t)t * E + e);
            if (!presum)
                for (int q = 1; q < nsplit; ++q) z += __ldcg(part + ((size_t)q * T + t) * E + e);
            v[i] = z;
            if (logits) logits[(size_t)t * E + e] = z;
        }
        select_topk(v, E, k, score, topk_ids + (size_t)t * k, topk_w + (size_t)t * k, sel[warp]);
    }
}

// Arrival on the tile's counter; true in the CTA that arrived last (the
// counter is reset for the next call).
__device__ bool last_of_tile(int *counter, int nsplit) {
    __shared__ int is_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int prev = atomicAdd(counter, 1);
        is_last = prev == nsplit - 1;
        if (is_last) *counter = 0;
    }
    __syncthreads();
    if (is_last) __threadfence();
    return is_last != 0;
}

struct RouterArgs {
    const void *x;            // [T][H] bf16 or f32
    const uint4 *wfrag;       // bf16 terms in fragment order (bf16 activations)
    const float *wt;          // [H][E] f32 (f32 activations)
    const float *wrow;        // [E][H] f32 (the GEMV)
    float *part;              // [nsplit][T][E]
    int *counters;            // [token tiles], zero between calls
    int32_t *topk_ids;
    float *topk_w;
    float *logits;            // [T][E] or null
    int T, H, E, k, score, nsplit, kslice;
};

// ------------------------------------------------------------ bf16 path

__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint4 &a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

// Fragment-order index of (16-expert tile mt, 16-K step ks, term q): 32
// lanes x 16 bytes.
__host__ __device__ inline size_t frag_index(int mt, int ks, int q, int n_ks) {
    return (((size_t)mt * n_ks + ks) * 3 + q) * 32;
}

// CTA (token tile blockIdx.x, K slice blockIdx.y): warp w computes experts
// [16 MT w, 16 MT (w + 1)) for the tile's 32 tokens over the slice, in f32
// accumulators, and stores them as the slice's partial logits.
template <int MT>
__global__ void __launch_bounds__(kRThreads, 2) router_bf16_kernel(RouterArgs a) {
    __shared__ float sel[kRWarps][kMaxTopK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
    const int t0 = blockIdx.x * kTileTok;
    const int n_ks = a.H / 16;
    const int ks0 = blockIdx.y * (a.kslice / 16), ks1 = ks0 + a.kslice / 16;
    const uint16_t *x = reinterpret_cast<const uint16_t *>(a.x);
    const int mtiles = (a.E + 15) / 16;
    for (int mt0 = warp * MT; mt0 < mtiles; mt0 += kRWarps * MT) {
        float acc[MT][4][4];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[m][n][i] = 0.f;
        // token rows of this lane's B fragments (zero past T)
        const uint16_t *xr[4];
        bool live[4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int t = t0 + 8 * n + g;
            live[n] = t < a.T;
            xr[n] = x + (size_t)(live[n] ? t : 0) * a.H + 2 * t4;
        }
#pragma unroll 2
        for (int ks = ks0; ks < ks1; ++ks) {
            uint32_t b[4][2];
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                b[n][0] = live[n] ? __ldg(reinterpret_cast<const uint32_t *>(xr[n] + 16 * ks)) : 0u;
                b[n][1] = live[n] ? __ldg(reinterpret_cast<const uint32_t *>(xr[n] + 16 * ks + 8)) : 0u;
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const int mt = mt0 + m;
                if (mt >= mtiles) break;
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                    const uint4 af = __ldg(a.wfrag + frag_index(mt, ks, q, n_ks) + lane);
#pragma unroll
                    for (int n = 0; n < 4; ++n) mma_bf16_16816(acc[m][n], af, b[n][0], b[n][1]);
                }
            }
        }
        // D fragment: (row g, cols 2t4, 2t4+1), (row g+8, same cols); row =
        // expert, col = token
        float *part = a.part + (size_t)blockIdx.y * a.T * a.E;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const int e0 = (mt0 + m) * 16 + g;
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int tc = t0 + 8 * n + 2 * t4;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int e = e0 + (i >> 1) * 8, t = tc + (i & 1);
                    if (e < a.E && t < a.T) __stcg(part + (size_t)t * a.E + e, acc[m][n][i]);
                }
            }
        }
    }
    if (last_of_tile(a.counters + blockIdx.x, a.nsplit))
        finish_tile(a.part, a.nsplit, a.T, a.E, a.k, a.score, t0, a.topk_ids, a.topk_w, a.logits, sel);
}

// ------------------------------------------------------------ decode sizes

constexpr int kGemvMaxT = 8;              // tokens per call served by the GEMV

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// CTA e computes logit row e for the call's T <= 8 tokens: warp w takes the
// w-th eighth of the row's 16-byte groups, lane l every 32nd group from its
// l-th, and accumulates one f32 FMA chain per token; the lanes' sums are
// added by a butterfly, the warps' in warp order.  The last CTA to finish
// selects, one warp per token.
template <bool BF>
__global__ void __launch_bounds__(kRThreads) router_gemv_kernel(RouterArgs a) {
    __shared__ float red[kRWarps][kGemvMaxT];
    __shared__ float sel[kRWarps][kMaxTopK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x, T = a.T, H = a.H, n4 = H >> 2;
    const int j0 = warp * n4 / kRWarps, j1 = (warp + 1) * n4 / kRWarps;
    const float4 *wr = reinterpret_cast<const float4 *>(a.wrow + (size_t)e * H);
    float acc[kGemvMaxT];
#pragma unroll
    for (int t = 0; t < kGemvMaxT; ++t) acc[t] = 0.f;
    for (int jb = j0 + lane; jb < j1; jb += 4 * 32) {
        float4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = jb + 32 * u;
            w[u] = j < j1 ? __ldcs(wr + j) : make_float4(0.f, 0.f, 0.f, 0.f);   // read once: evict first
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = jb + 32 * u;
            if (j >= j1) break;
#pragma unroll
            for (int t = 0; t < kGemvMaxT; ++t) {
                if (t >= T) break;
                float x0, x1, x2, x3;
                if constexpr (BF) {
                    // four bf16 at element 4j: two 4-byte words (x is 4-byte aligned)
                    const uint32_t *xp =
                        reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint16_t *>(a.x) + (size_t)t * H) +
                        2 * j;
                    const uint32_t p0 = __ldg(xp), p1 = __ldg(xp + 1);
                    x0 = __uint_as_float(p0 << 16);
                    x1 = __uint_as_float(p0 & 0xffff0000u);
                    x2 = __uint_as_float(p1 << 16);
                    x3 = __uint_as_float(p1 & 0xffff0000u);
                } else {
                    const float *xp = reinterpret_cast<const float *>(a.x) + (size_t)t * H + 4 * j;
                    x0 = __ldg(xp);
                    x1 = __ldg(xp + 1);
                    x2 = __ldg(xp + 2);
                    x3 = __ldg(xp + 3);
                }
                acc[t] = fmaf(x0, w[u].x, acc[t]);
                acc[t] = fmaf(x1, w[u].y, acc[t]);
                acc[t] = fmaf(x2, w[u].z, acc[t]);
                acc[t] = fmaf(x3, w[u].w, acc[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kGemvMaxT; ++t) {
        if (t >= T) break;
        const float v = warp_sum(acc[t]);
        if (lane == 0) red[warp][t] = v;
    }
    __syncthreads();
    if (threadIdx.x < T) {
        const int t = threadIdx.x;
        float z = 0.f;
#pragma unroll
        for (int w = 0; w < kRWarps; ++w) z += red[w][t];
        __stcg(a.part + (size_t)t * a.E + e, z);
        if (a.logits) a.logits[(size_t)t * a.E + e] = z;
    }
    if (last_of_tile(a.counters, gridDim.x) && warp < T) {
        const int t = warp, per = (a.E + 31) / 32;
        float v[kMaxPerLane];
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int ex = lane + 32 * i;
            v[i] = (i < per && ex < a.E) ? __ldcg(a.part + (size_t)t * a.E + ex) : 0.f;
        }
        select_topk(v, a.E, a.k, a.score, a.topk_ids + (size_t)t * a.k, a.topk_w + (size_t)t * a.k, sel[warp]);
    }
}

// ------------------------------------------------------------ f32 path

__global__ void __launch_bounds__(kRThreads) router_f32_kernel(RouterArgs a) {
    __shared__ float sel[kRWarps][kMaxTopK];
    __shared__ float xs[kTileTok][64];
    const int t0 = blockIdx.x * kTileTok;
    const int k0 = blockIdx.y * a.kslice, k1 = k0 + a.kslice;
    const float *x = reinterpret_cast<const float *>(a.x);
    float *part = a.part + (size_t)blockIdx.y * a.T * a.E;
    for (int e = threadIdx.x; e < ((a.E + kRThreads - 1) / kRThreads) * kRThreads; e += kRThreads) {
        float acc[kTileTok];
#pragma unroll
        for (int i = 0; i < kTileTok; ++i) acc[i] = 0.f;
        for (int kb = k0; kb < k1; kb += 64) {
            __syncthreads();
            for (int i = threadIdx.x; i < kTileTok * 64; i += kRThreads) {
                const int tt = i / 64, kk = i % 64, t = t0 + tt;
                xs[tt][kk] = (t < a.T && kb + kk < k1) ? x[(size_t)t * a.H + kb + kk] : 0.f;
            }
            __syncthreads();
            if (e < a.E) {
                for (int kk = 0; kk < 64 && kb + kk < k1; ++kk) {
                    const float wv = a.wt[(size_t)(kb + kk) * a.E + e];
#pragma unroll
                    for (int i = 0; i < kTileTok; ++i) acc[i] = fmaf(xs[i][kk], wv, acc[i]);
                }
            }
        }
        if (e < a.E)
            for (int i = 0; i < kTileTok; ++i)
                if (t0 + i < a.T) __stcg(part + (size_t)(t0 + i) * a.E + e, acc[i]);
    }
    if (last_of_tile(a.counters + blockIdx.x, a.nsplit))
        finish_tile(a.part, a.nsplit, a.T, a.E, a.k, a.score, t0, a.topk_ids, a.topk_w, a.logits, sel);
}

// K slices per token tile: enough CTAs for the 148 SMs twice over at
// prefill sizes, slices of at least 128 K at decode sizes (so a slice's
// fragment loads are few and all in flight at once).
int router_nsplit(int T, int H) {
    const int tiles = (T + kTileTok - 1) / kTileTok;
    int ns = 1;
    while (ns * 2 * tiles <= 296 && H % (ns * 2 * 64) == 0 && H / (ns * 2) >= 128) ns *= 2;
    return ns;
}

}  // namespace

// bf16 terms of Wr (host f32 [E][H]) in fragment order, or Wr transposed.
cudaError_t router_upload(Layer &L, const float *wr, int score, cudaStream_t s) {
    const int E = L.d.n_experts, H = L.d.hidden;
    RouterState *r = L.router;
    const bool bf = L.d.act == MOEQ_ACT_BF16;
    if (!r) {
        r = new (std::nothrow) RouterState();
        if (!r) return cudaErrorMemoryAllocation;
        L.router = r;
        const int tiles = (L.d.max_tokens + kTileTok - 1) / kTileTok;
        // partial logits: the most K slices x tokens any token count needs
        // (the slice count falls as the token tiles grow)
        size_t max_rows = 0;
        for (int T = 1; T <= L.d.max_tokens; ++T)
            max_rows = std::max(max_rows, (size_t)router_nsplit(T, H) * (size_t)T);
        const size_t mtiles = (size_t)(E + 15) / 16;
        cudaError_t e = cudaSuccess;
        if (bf) e = dev_alloc((void **)&r->wfrag, mtiles * (H / 16) * 3 * 32 * sizeof(uint4));
        else e = dev_alloc((void **)&r->wt, sizeof(float) * (size_t)E * H);
        if (e == cudaSuccess) e = dev_alloc((void **)&r->wrow, sizeof(float) * (size_t)E * H);
        if (e == cudaSuccess) e = dev_alloc((void **)&r->part, sizeof(float) * max_rows * E);
        if (e == cudaSuccess) e = dev_alloc((void **)&r->counters, sizeof(int) * (size_t)tiles);
        if (e == cudaSuccess) e = cudaMemset(r->counters, 0, sizeof(int) * (size_t)tiles);
        if (e != cudaSuccess) return e;
    }
    r->score = score;
    {
        cudaError_t e = cudaMemcpyAsync(r->wrow, wr, sizeof(float) * (size_t)E * H, cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return e;
    }
    // the host image: terms in fragment order, or the transpose
    if (bf) {
        const int n_ks = H / 16, mtiles = (E + 15) / 16;
        std::vector<uint16_t> img((size_t)mtiles * n_ks * 3 * 32 * 8, 0);
        auto bf16_rn = [](float f) -> uint16_t {
            uint32_t u;
            std::memcpy(&u, &f, 4);
            if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)(u >> 16);   // inf / nan kept
            u += 0x7fffu + ((u >> 16) & 1u);
            return (uint16_t)(u >> 16);
        };
        auto bf16_f = [](uint16_t b) {
            const uint32_t u = (uint32_t)b << 16;
            float f;
            std::memcpy(&f, &u, 4);
            return f;
        };
        for (int mt = 0; mt < mtiles; ++mt)
            for (int ks = 0; ks < n_ks; ++ks)
                for (int lane = 0; lane < 32; ++lane) {
                    const int g = lane >> 2, t4 = lane & 3;
                    // a0: (g, 2t4..+1), a1: (g+8, 2t4..), a2: (g, 2t4+8..), a3: (g+8, 2t4+8..)
                    for (int reg = 0; reg < 4; ++reg)
                        for (int hlf = 0; hlf < 2; ++hlf) {
                            const int row = g + 8 * (reg & 1), col = 2 * t4 + 8 * (reg >> 1) + hlf;
                            const int ex = mt * 16 + row, kk = ks * 16 + col;
                            float w = ex < E ? wr[(size_t)ex * H + kk] : 0.f;
                            uint16_t term[3];
                            for (int q = 0; q < 3; ++q) {
                                term[q] = bf16_rn(w);
                                w = w - bf16_f(term[q]);   // exact: w and its bf16 rounding share an exponent range
                            }
                            for (int q = 0; q < 3; ++q)
                                img[(frag_index(mt, ks, q, n_ks) + lane) * 8 + reg * 2 + hlf] = term[q];
                        }
                }
        cudaError_t e = cudaMemcpyAsync(r->wfrag, img.data(), img.size() * sizeof(uint16_t), cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return e;
    } else {
        std::vector<float> t((size_t)E * H);
        for (int ex = 0; ex < E; ++ex)
            for (int kk = 0; kk < H; ++kk) t[(size_t)kk * E + ex] = wr[(size_t)ex * H + kk];
        cudaError_t e = cudaMemcpyAsync(r->wt, t.data(), t.size() * sizeof(float), cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return e;
    }
    r->ready = true;
    return cudaSuccess;
}

void router_free(Layer &L) {
    RouterState *r = L.router;
    if (!r) return;
    cudaFree(r->wfrag);
    cudaFree(r->wt);
    cudaFree(r->wrow);
    cudaFree(r->part);
    cudaFree(r->counters);
    delete r;
    L.router = nullptr;
}

cudaError_t launch_router(const Layer &L, const void *x, int T, int32_t *topk_ids, float *topk_w, float *logits,
                          cudaStream_t s) {
    const RouterState *r = L.router;
    RouterArgs a{};
    a.x = x;
    a.wfrag = r->wfrag;
    a.wt = r->wt;
    a.wrow = r->wrow;
    a.part = r->part;
    a.counters = r->counters;
    a.topk_ids = topk_ids;
    a.topk_w = topk_w;
    a.logits = logits;
    a.T = T;
    a.H = L.d.hidden;
    a.E = L.d.n_experts;
    a.k = L.d.top_k;
    a.score = r->score;
    a.nsplit = router_nsplit(T, a.H);
    a.kslice = a.H / a.nsplit;
    L.count_launches(1);
    if (T <= kGemvMaxT) {
        if (L.d.act == MOEQ_ACT_BF16) router_gemv_kernel<true><<<a.E, kRThreads, 0, s>>>(a);
        else router_gemv_kernel<false><<<a.E, kRThreads, 0, s>>>(a);
        return cudaGetLastError();
    }
    const dim3 grid((T + kTileTok - 1) / kTileTok, a.nsplit);
    if (L.d.act == MOEQ_ACT_BF16) {
        // two 16-expert tiles per warp: 8 warps cover 256 experts per pass
        router_bf16_kernel<2><<<grid, kRThreads, 0, s>>>(a);
    } else {
        router_f32_kernel<<<grid, kRThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace moeq
