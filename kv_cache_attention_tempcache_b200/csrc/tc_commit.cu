// TempCache commit path: staging (copy + hash + bucketed top-1 search with the merge
// decision), then, when the next chunk arrives, the commit (append in token order and
// the deterministic list merge).
//
// FAST-AR technical summary, section 2.A "TempCache": each key of the current
// chunk is hashed with locality-sensitive hashing, its top-1 neighbour among the
// earlier cache entries is found, and near-duplicates above a similarity threshold
// are merged with their values averaged; the rest extend the cache.
//
// When the decisions are taken. A chunk is committed one call after it was staged,
// and nothing changes the cache in between, so the cache a staged token must be
// matched against (the entries committed before its commit) is already final when
// it is staged. The staging kernel therefore also hashes the keys and searches their
// buckets while the keys are on chip; the commit kernel only applies the decisions:
// it appends the unmatched tokens and merges the matched ones. Per chunk that is two
// launches (plus the in-chunk dedupe of the intra_chunk option, and two re-bucketing
// launches with running-mean keys).
//
// Exactness of the integer results. Every decision here (a hash bit, the best
// candidate, merge or not) is defined on fp64 dot products summed in index order
// 0..d-1 (products of bf16/fp32 values are exact in fp64). Hash bits are first
// computed in fp32 and kept only outside a rigorous bound of their rounding error,
// else recomputed in fp64 in index order. Similarities are computed in fp64 with the
// value of the index-order sum: exactly in any order when the exponent-span rule
// below holds, else as the index-order chain itself. Codes, matches and the append
// order are therefore bit-identical to the definition.
#include "tc_internal.h"
#include "tc_device.cuh"

#include <math.h>

namespace tc {

namespace {

// ------------------------------------------------------------------ lane groups
//
// The dedupe, append and merge kernels give each row to a group of 8 lanes: lane g
// of group q (lanes 8q .. 8q+7) holds elements [g*EPG, g*EPG + EPG) of the row, so
// one warp works on four rows at once and every lane moves 16-byte words.
template <typename E, int D>
struct GSlice {
    static constexpr int EPG = D / 8;
    static constexpr int NW = EPG * (int)sizeof(E) / 16;
    uint4 w[NW];
    __device__ __forceinline__ void load(const E* row, int gl) {
        const uint4* p = reinterpret_cast<const uint4*>(row) + gl * NW;
#pragma unroll
        for (int k = 0; k < NW; ++k) w[k] = p[k];
    }
    __device__ __forceinline__ void store(E* row, int gl) const {
        uint4* p = reinterpret_cast<uint4*>(row) + gl * NW;
#pragma unroll
        for (int k = 0; k < NW; ++k) p[k] = w[k];
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int k = 0; k < NW; ++k) w[k] = make_uint4(0u, 0u, 0u, 0u);
    }
    __device__ __forceinline__ uint32_t word(int i) const {
        const uint4& q = w[i >> 2];
        return (i & 3) == 0 ? q.x : (i & 3) == 1 ? q.y : (i & 3) == 2 ? q.z : q.w;
    }
    __device__ __forceinline__ void set_word(int i, uint32_t u) {
        uint4& q = w[i >> 2];
        if ((i & 3) == 0) q.x = u; else if ((i & 3) == 1) q.y = u; else if ((i & 3) == 2) q.z = u; else q.w = u;
    }
    __device__ __forceinline__ float at(int i) const {
        if constexpr (sizeof(E) == 2) {
            const uint32_t u = word(i >> 1);
            return (i & 1) ? __uint_as_float(u & 0xffff0000u) : __uint_as_float(u << 16);
        } else {
            return __uint_as_float(word(i));
        }
    }
    // Round EPG floats to the storage type (bf16: nearest even) and keep them.
    __device__ __forceinline__ void from_floats(const float (&v)[EPG]) {
        if constexpr (sizeof(E) == 2) {
#pragma unroll
            for (int i = 0; i < EPG / 2; ++i) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
                set_word(i, *reinterpret_cast<const uint32_t*>(&b));
            }
        } else {
#pragma unroll
            for (int i = 0; i < EPG; ++i) set_word(i, __float_as_uint(v[i]));
        }
    }
};

__device__ __forceinline__ double gsum64(double v, unsigned gmask) {
    v += __shfl_xor_sync(gmask, v, 4);
    v += __shfl_xor_sync(gmask, v, 2);
    v += __shfl_xor_sync(gmask, v, 1);
    return v;
}

// sum_i a_i b_i in fp64 in index order 0..d-1, handed from lane to lane of the
// group (each lane continues the previous lane's sum); every lane gets the result.
template <typename E, int D>
__device__ __forceinline__ double gchain_dot(const GSlice<E, D>& a, const GSlice<E, D>& b, int gl, int grp,
                                             unsigned gmask) {
    double acc = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (gl == k) {
#pragma unroll
            for (int i = 0; i < GSlice<E, D>::EPG; ++i) acc = fma((double)a.at(i), (double)b.at(i), acc);
        }
        acc = __shfl_sync(gmask, acc, 8 * grp + k);
    }
    return acc;
}

// This lane's part of sum_i a_i b_i in fp64 (its elements in index order).
template <typename E, int D>
__device__ __forceinline__ double lane_dot64(const GSlice<E, D>& a, const GSlice<E, D>& b) {
    double acc = 0.0;
#pragma unroll
    for (int i = 0; i < GSlice<E, D>::EPG; ++i) acc = fma((double)a.at(i), (double)b.at(i), acc);
    return acc;
}

// Exact fp64 sums of bf16 products. A nonzero bf16 value with exponent field f
// (f = 0, a subnormal, taken as 1) lies below 2^(f-126) and is a multiple of
// 2^(f-134). Let span(x) = max f - min f + 7 over the nonzero elements of a row
// (0 for a zero row). Every product x_i y_i, and so every partial sum in any
// order, is then a multiple of 2^(minf_x + minf_y - 268), while each partial sum
// is below d 2^(maxf_x + maxf_y - 252) in magnitude. When
//   span(x) + span(y) <= 51 - log2(d)
// every partial sum is an integer below 2^53 times that unit, so fp64 represents
// all of them exactly: the sum has no rounding at all and any summation order
// (lane sums, then the group butterfly) yields the bits of the index-order sum.
// Otherwise the kernels fall back to the index-order chain.
template <int D>
constexpr int kSpanLimit = 51 - (D == 128 ? 7 : 6);

template <int D>
__device__ __forceinline__ int gspan_bf16(const GSlice<__nv_bfloat16, D>& x, unsigned gmask) {
    int emax = 0, emin = 255;
#pragma unroll
    for (int i = 0; i < GSlice<__nv_bfloat16, D>::EPG / 2; ++i) {
        const uint32_t u = x.word(i);
        const uint32_t lo = u & 0xffffu, hi = u >> 16;
        if (lo & 0x7fffu) {
            const int f = max((int)((lo >> 7) & 0xffu), 1);
            emax = max(emax, f);
            emin = min(emin, f);
        }
        if (hi & 0x7fffu) {
            const int f = max((int)((hi >> 7) & 0xffu), 1);
            emax = max(emax, f);
            emin = min(emin, f);
        }
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
        emax = max(emax, __shfl_xor_sync(gmask, emax, o));
        emin = min(emin, __shfl_xor_sync(gmask, emin, o));
    }
    return emax >= emin ? emax - emin + 7 : 0;
}

// The last block of the grid to finish sums the per-window counts of new entries
// into the new cache sizes and raises the abort flag if a head would exceed its
// capacity. Every thread of the grid calls it once, after its last update.
__device__ void publish_sizes(const CacheView& c, const StageView& s, int32_t* ctr) {
    const int H = c.H;
    const int lane = threadIdx.x & 31;
    __shared__ bool last;
    __threadfence();   // this thread's list and count updates before the ticket
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&ctr[2 * H + 1], 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int nwin = (int)((s.T + 31) >> 5);
    const int warp = threadIdx.x >> 5;
    for (int h = warp; h < H; h += blockDim.x >> 5) {
        int u = 0;
        for (int w = lane; w < nwin; w += 32) u += __ldcg(&s.wcnt[(int64_t)h * (s.TmaxP >> 5) + w]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
        if (lane == 0) {
            const int nm = c.M[h] + u;
            ctr[H + h] = nm;
            if ((int64_t)nm > c.capacity) atomicExch(&ctr[2 * H], 1);
        }
    }
}
// ------------------------------------------------------------------ staging: copy, hash, search
//
// One warp per window of 32 consecutive tokens t0 .. t0+31 of one head h (the unit
// of the append order). The warp
//  1. copies the window's K rows into shared memory and, with its V rows, into the
//     head-major staging buffer (16-byte words, eight in flight per lane);
//  2. hashes: lane l takes token t0 + l and forms the nbits projections <R_b, k> in
//     fp32, the normals broadcast from a copy in shared memory;
//     bit b keeps the fp32 sign when
//       |<R_b,k>| > 2 (d+2) u |R_b| |k|   (u = 2^-24; any summation order errs by at
//                                          most (d+2) u sum|R_bi k_i| <= (d+2) u |R_b||k|,
//                                          doubled for margin)
//     and otherwise the lane redoes the sum in fp64 in index order;
//  3. searches: each lane walks its token's bucket list (the entries committed before
//     this chunk's commit with the same code) and forms every cosine
//     dot / sqrt(|k|^2 |e|^2) in fp64 with the value of the index-order sums; the best
//     candidate (ties to the lowest entry index) merges when its cosine is >= tau;
//  4. publishes: a matched token joins its target's merge list, the window's count of
//     unmatched tokens is stored for the append order. The last block to finish turns
//     the window counts into the new cache sizes and raises the abort flag when a head
//     would exceed its capacity.
// With the intra_chunk option step 4 keeps the best committed candidate and its
// similarity instead, and groups the chunk's tokens by bucket for the dedupe kernel.
//
// Exact similarities of bf16 rows. A product of two bf16 values has at most 16
// significant bits, so it is exact in fp32. When span(x) + span(y) <= kSpanLimit every
// partial sum of the products is exact in fp64 (see gspan_bf16), so four fp64 partial
// sums in any order give the bits of the index-order sum; otherwise the lane runs the
// index-order chain. With running-mean keys an entry whose key is not a bf16 value
// has span 255 and always takes the chain, over its fp32 key.
template <int D, int NBP>
struct StagePlanes {
    float v[NBP * D];   // normals (bf16 values), rows past nbits zero
    float rn[NBP];      // |R_b|, rounded up
};

constexpr int kStageWarps = 4;   // warps per block of the staging kernel
constexpr int kCandKeep = 8;     // candidates whose fp32 cosine a lane keeps for the exact recheck

template <typename E, int D>
struct StageSmem {
    static constexpr int RB = D * (int)sizeof(E) + 16;   // row pitch: consecutive rows start 4 banks apart
    static constexpr int WARP = 32 * RB;
    static constexpr int BYTES = kStageWarps * WARP;
};

// Element i of a row in shared memory, as a float.
template <typename E>
__device__ __forceinline__ float srow_at(const uint8_t* row, int i) {
    if constexpr (sizeof(E) == 2)
        return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(row)[i] << 16);
    else
        return reinterpret_cast<const float*>(row)[i];
}

// The floats packed in a 16-byte word of a row (8 bf16 values or 4 fp32 values).
template <typename E>
__device__ __forceinline__ void unpack16(const uint4& v, float (&x)[16 / sizeof(E)]) {
    if constexpr (sizeof(E) == 2) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            x[2 * k] = __uint_as_float(w[k] << 16);
            x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
    } else {
        x[0] = __uint_as_float(v.x);
        x[1] = __uint_as_float(v.y);
        x[2] = __uint_as_float(v.z);
        x[3] = __uint_as_float(v.w);
    }
}

// Index-order fp64 sum of x_i y_i over a shared-memory row x and a global row y.
template <typename E, typename F, int D>
__device__ __noinline__ double chain_dot(const uint8_t* x, const F* __restrict__ y) {
    double acc = 0.0;
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
        float yi;
        if constexpr (sizeof(F) == 2)
            yi = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(y)[i] << 16);
        else
            yi = y[i];
        acc = fma((double)srow_at<E>(x, i), (double)yi, acc);
    }
    return acc;
}

// Index-order fp64 sum of y_i^2 over an fp32 row in global memory.
template <int D>
__device__ __noinline__ double chain_dot_ff(const float* __restrict__ y) {
    double acc = 0.0;
#pragma unroll 8
    for (int i = 0; i < D; ++i) acc = fma((double)y[i], (double)y[i], acc);
    return acc;
}

// Exact sum of x_i y_i of two bf16 rows (x in shared memory, y from global memory) when
// the span rule holds: exact fp32 products, four fp64 partial sums.
template <int D>
__device__ __noinline__ double span_dot(const uint8_t* x, const uint4* __restrict__ y) {
    constexpr int W = D / 8;
    uint4 yw[W];
#pragma unroll
    for (int c = 0; c < W; ++c) yw[c] = y[c];
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
#pragma unroll
    for (int c = 0; c < W; ++c) {
        float xv[8], yv[8];
        unpack16<__nv_bfloat16>(*reinterpret_cast<const uint4*>(x + 16 * c), xv);
        unpack16<__nv_bfloat16>(yw[c], yv);
        a0 += (double)(xv[0] * yv[0]) + (double)(xv[4] * yv[4]);
        a1 += (double)(xv[1] * yv[1]) + (double)(xv[5] * yv[5]);
        a2 += (double)(xv[2] * yv[2]) + (double)(xv[6] * yv[6]);
        a3 += (double)(xv[3] * yv[3]) + (double)(xv[7] * yv[7]);
    }
    return (a0 + a1) + (a2 + a3);
}

// fp32 sum of x_i y_i of a bf16 row in shared memory and a bf16 row from global memory
// (exact products, rounded sums in four chains: within (d+2) u |x||y| of the exact sum).
template <int D>
__device__ __forceinline__ float dot32_bf16(const uint8_t* x, const uint4* __restrict__ y) {
    constexpr int W = D / 8;
    uint4 yw[W];
#pragma unroll
    for (int c = 0; c < W; ++c) yw[c] = y[c];
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int c = 0; c < W; ++c) {
        float xv[8], yv[8];
        unpack16<__nv_bfloat16>(*reinterpret_cast<const uint4*>(x + 16 * c), xv);
        unpack16<__nv_bfloat16>(yw[c], yv);
        a0 = fmaf(xv[0], yv[0], fmaf(xv[4], yv[4], a0));
        a1 = fmaf(xv[1], yv[1], fmaf(xv[5], yv[5], a1));
        a2 = fmaf(xv[2], yv[2], fmaf(xv[6], yv[6], a2));
        a3 = fmaf(xv[3], yv[3], fmaf(xv[7], yv[7], a3));
    }
    return (a0 + a1) + (a2 + a3);
}

// The same with an fp32 row y (running-mean keys that are not bf16 values).
template <typename E, int D>
__device__ __forceinline__ float dot32_f32(const uint8_t* x, const float* __restrict__ y) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
    for (int i = 0; i < D; i += 4) {
        const float4 yv = *reinterpret_cast<const float4*>(y + i);
        a0 = fmaf(srow_at<E>(x, i), yv.x, a0);
        a1 = fmaf(srow_at<E>(x, i + 1), yv.y, a1);
        a2 = fmaf(srow_at<E>(x, i + 2), yv.z, a2);
        a3 = fmaf(srow_at<E>(x, i + 3), yv.w, a3);
    }
    return (a0 + a1) + (a2 + a3);
}

template <typename E, int D, int NBP, bool INTRA, bool MEAN>
__global__ void __launch_bounds__(kStageWarps * 32, 4)
stage_search_kernel(const E* __restrict__ K, const E* __restrict__ V, CacheView c, StageView s,
                    const __grid_constant__ StagePlanes<D, NBP> pl, float tau,
                    int32_t* ctr, Stats* stats) {
    using S = StageSmem<E, D>;
    const double tau64 = (double)tau;
    // delta bounds |sim32 - sim| of the fp32 cosines: 2 x (2 (d+2) u + 3 u)
    const float delta = 2.f * (2.f * (float)(D + 2) * kU32 + 3.f * kU32);
    constexpr int W = D * (int)sizeof(E) / 16;   // 16-byte words per row
    constexpr int EPW = 16 / (int)sizeof(E);     // elements per word
    extern __shared__ __align__(16) uint8_t ss_smem[];
    __shared__ float sKmax[kStageWarps];
    __shared__ unsigned sRe[kStageWarps][2];
    __shared__ __align__(16) float sR[NBP * D];   // the normals (rows past nbits zero)
    __shared__ int sCj[kStageWarps][kCandKeep][32];     // per lane: its first candidates ...
    __shared__ float sCs[kStageWarps][kCandKeep][32];   // ... and their fp32 cosines
    for (int i = threadIdx.x; i < NBP * D; i += blockDim.x) sR[i] = pl.v[i];
    __syncthreads();
    grid_dependency_wait();   // the previous commit (and anything else before us in the stream)
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    uint8_t* rows = ss_smem + wib * S::WARP;
    const int H = c.H, nbits = c.nbits;
    const int64_t T = s.T;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < s.TmaxP;
         i += (int64_t)gridDim.x * blockDim.x)
        s.sbias[i] = (i < T) ? 0.f : -INFINITY;
    const int nwin = (int)((T + 31) >> 5);
    const float gam2 = 2.f * (float)(D + 2) * kU32;
    const E* Kc = reinterpret_cast<const E*>(c.Kc);
    float kmax = 0.f;                 // largest fp32 |k|^2 this lane staged
    unsigned hre = 0, mre = 0;        // hash bits and similarity sums that took the fp64 chain
    for (int64_t item = (int64_t)blockIdx.x * kStageWarps + wib; item < (int64_t)H * nwin;
         item += (int64_t)gridDim.x * kStageWarps) {   // warp-uniform
        const int h = (int)(item / nwin);
        const int w = (int)(item - (int64_t)h * nwin);
        const int t0 = w * 32;
        const int n = (T - t0 < 32) ? (int)(T - t0) : 32;
        const int64_t sbase = (int64_t)h * s.TmaxP + t0;
        // ---- 1. copy
        {
            uint4* ks = reinterpret_cast<uint4*>(reinterpret_cast<E*>(s.Ks) + sbase * D);
            uint4* vs = reinterpret_cast<uint4*>(reinterpret_cast<E*>(s.Vs) + sbase * D);
            const int nw = n * W;
#pragma unroll 1
            for (int q0 = 0; q0 < 32 * W; q0 += 4 * 32) {
                uint4 kb[4], vb[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int q = q0 + u * 32 + lane;
                    if (q < nw) {
                        const int row = q / W, col = q - row * W;
                        const int64_t src = ((int64_t)(t0 + row) * H + h) * D;
                        kb[u] = reinterpret_cast<const uint4*>(K + src)[col];
                        vb[u] = reinterpret_cast<const uint4*>(V + src)[col];
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int q = q0 + u * 32 + lane;
                    if (q < nw) {
                        const int row = q / W, col = q - row * W;
                        *reinterpret_cast<uint4*>(rows + row * S::RB + col * 16) = kb[u];
                        ks[q] = kb[u];
                        vs[q] = vb[u];
                    }
                }
            }
        }
        __syncwarp();
        // ---- 2. hash
        const bool valid = lane < n;
        const uint8_t* my = rows + lane * S::RB;
        uint32_t code = 0;
        int spx = 255;
        float n2 = 0.f;
        if (valid && sizeof(E) == 4) {   // fp32 storage (small workloads): plain loops
            for (int i = 0; i < D; ++i) n2 = fmaf(srow_at<E>(my, i), srow_at<E>(my, i), n2);
            const float nx = sqrtf(n2);
            for (int b = 0; b < nbits; ++b) {
                float a = 0.f;
                for (int i = 0; i < D; ++i) a = fmaf(sR[b * D + i], srow_at<E>(my, i), a);
                bool bit = a >= 0.f;
                if (!(fabsf(a) > gam2 * pl.rn[b] * nx + 1e-30f)) {
                    double s64 = 0.0;
                    for (int i = 0; i < D; ++i) s64 = fma((double)sR[b * D + i], (double)srow_at<E>(my, i), s64);
                    bit = s64 >= 0.0;
                    ++hre;
                }
                code |= (uint32_t)bit << b;
            }
            s.scode[sbase + lane] = code;
            kmax = fmaxf(kmax, n2);
        } else if (valid) {
            float acc[NBP];
#pragma unroll
            for (int b = 0; b < NBP; ++b) acc[b] = 0.f;
            uint32_t emax2 = 0u, emin2 = 0x7f807f80u;   // exponent fields of both bf16 halves
#pragma unroll 1
            for (int cw = 0; cw < W; ++cw) {
                const uint4 v4 = *reinterpret_cast<const uint4*>(my + cw * 16);
                float x[EPW];
                unpack16<E>(v4, x);
                if constexpr (sizeof(E) == 2) {
                    const uint32_t wd[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t f = wd[k] & 0x7f807f80u;
                        emax2 = __vmaxu2(emax2, f);
                        emin2 = __vminu2(emin2, f);
                    }
                }
#pragma unroll
                for (int k = 0; k < EPW; ++k) n2 = fmaf(x[k], x[k], n2);
#pragma unroll
                for (int b = 0; b < NBP; ++b) {
                    const float* rb = sR + b * D + cw * EPW;   // same address on every lane: broadcast
                    float t = acc[b];
#pragma unroll
                    for (int k = 0; k < EPW; k += 4) {
                        const float4 r4 = *reinterpret_cast<const float4*>(rb + k);
                        t = fmaf(r4.x, x[k], t);
                        t = fmaf(r4.y, x[k + 1], t);
                        t = fmaf(r4.z, x[k + 2], t);
                        t = fmaf(r4.w, x[k + 3], t);
                    }
                    acc[b] = t;
                }
            }
            const float nx = sqrtf(n2);
#pragma unroll
            for (int b = 0; b < NBP; ++b) {
                if (b >= nbits) break;
                bool bit = acc[b] >= 0.f;
                if (!(fabsf(acc[b]) > gam2 * pl.rn[b] * nx + 1e-30f)) {   // inside the band (or not finite)
                    // (the shared copy holds the bf16 normals exactly; products are exact in fp64)
                    double s64 = 0.0;
#pragma unroll 8
                    for (int i = 0; i < D; ++i) s64 = fma((double)sR[b * D + i], (double)srow_at<E>(my, i), s64);
                    bit = s64 >= 0.0;
                    ++hre;
                }
                code |= (uint32_t)bit << b;
            }
            if constexpr (sizeof(E) == 2) {
                // span from the exponent fields; a zero element counts as field 0, which only
                // widens the span (the exact-sum rule then sends the row to the chain)
                const int emax = (int)max(emax2 >> 23, (emax2 >> 7) & 0xffu);
                const int emin = max((int)min(emin2 >> 23, (emin2 >> 7) & 0xffu), 0);
                spx = emax >= 1 ? emax - emin + 7 + (emin == 0 ? 1 : 0) : 0;
            }
            s.scode[sbase + lane] = code;
            kmax = fmaxf(kmax, n2);
        }
        // ---- 3. search the bucket
        const int64_t hrow = (int64_t)h * c.capP;
        const int Mh = c.M[h];
        const int head = valid ? c.bhead[((int64_t)h << nbits) + code] : -1;
        double n1 = -1.0;   // exact |x|^2, formed when first needed
        // exact fp64 cosine of the lane's token with entry j (the value of the definition)
        auto exact_sim = [&](int j) -> double {
            if (n1 < 0.0) {
                if constexpr (sizeof(E) == 2) {
                    if (2 * spx <= kSpanLimit<D>) {
                        n1 = span_dot<D>(my, reinterpret_cast<const uint4*>(my));
                    } else {
                        n1 = chain_dot<E, __nv_bfloat16, D>(my, reinterpret_cast<const __nv_bfloat16*>(my));
                        ++mre;
                    }
                } else {
                    n1 = chain_dot<E, float, D>(my, reinterpret_cast<const float*>(my));
                }
            }
            double n2e = c.knorm64[hrow + j];
            double dot;
            if constexpr (sizeof(E) == 2) {
                const int spy = c.kspan[hrow + j];
                if constexpr (MEAN) {   // a merged key outside the exact-sum rule stores only an fp32 |k|^2
                    if (spy == 255) n2e = chain_dot_ff<D>(c.K32 + (hrow + j) * D);
                }
                if (spx + spy <= kSpanLimit<D>) {
                    dot = span_dot<D>(my, reinterpret_cast<const uint4*>(Kc + (hrow + j) * D));
                } else {
                    if constexpr (MEAN) dot = chain_dot<E, float, D>(my, c.K32 + (hrow + j) * D);
                    else dot = chain_dot<E, __nv_bfloat16, D>(my, reinterpret_cast<const __nv_bfloat16*>(Kc) + (hrow + j) * D);
                    ++mre;
                }
            } else {
                dot = chain_dot<E, float, D>(my, reinterpret_cast<const float*>(Kc) + (hrow + j) * D);
                ++mre;
            }
            return (n1 > 0.0 && n2e > 0.0) ? dot / sqrt(n1 * n2e) : 0.0;
        };
        double best = -INFINITY;   // exact best similarity (intra_chunk and exact paths)
        int bestj = -1, m = -1;
        if constexpr (INTRA || sizeof(E) != 2) {
            // every candidate exactly: the in-chunk dedupe needs the exact best similarity,
            // and fp32 rows have no certified shortcut here
            int ncand = 0;
            for (int j = head; j >= 0;) {   // per lane
                const int nxt = c.bnext[hrow + j];
                const double sim = exact_sim(j);
                if (sim > best || (sim == best && j < bestj)) {
                    best = sim;
                    bestj = j;
                }
                if (++ncand > Mh) {   // a bucket list can never be longer than the cache
                    atomicOr(&stats->error_bits, kErrBucketList);
                    break;
                }
                j = nxt;
            }
            m = (bestj >= 0 && best >= tau64) ? bestj : -1;
        } else {
            // fp32 cosines first. With delta a rigorous bound on |sim32 - sim|, the fp32
            // result decides when its best is below tau - delta (no merge), or above
            // tau + delta and ahead of every other candidate by more than 2 delta (merge into
            // it). Otherwise the candidates within 2 delta of the fp32 best (the only ones
            // that can be the exact best) are recomputed exactly.
            float b32 = -INFINITY, s32 = -INFINITY;
            int bj = -1, ncand = 0;
            bool weird = !(n2 > 1e-30f && n2 < 1e30f);
            for (int j = head; j >= 0;) {   // per lane
                const int nxt = c.bnext[hrow + j];
                const float ne = (float)c.knorm64[hrow + j];
                float dt;
                if constexpr (MEAN) {
                    if (c.kspan[hrow + j] == 255) dt = dot32_f32<E, D>(my, c.K32 + (hrow + j) * D);
                    else dt = dot32_bf16<D>(my, reinterpret_cast<const uint4*>(Kc + (hrow + j) * D));
                } else {
                    dt = dot32_bf16<D>(my, reinterpret_cast<const uint4*>(Kc + (hrow + j) * D));
                }
                if (nxt >= 0) {   // the next candidate's row (two 128-byte lines for d = 128)
                    const E* nr = Kc + (hrow + nxt) * D;
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(nr));
                    if (D * sizeof(E) > 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(nr + 128 / sizeof(E)));
                }
                weird = weird || !(ne > 1e-30f && ne < 1e30f && fabsf(dt) < 1e30f);
                const float sim = dt / sqrtf(n2 * ne);
                if (ncand < kCandKeep) {
                    sCj[wib][ncand][lane] = j;
                    sCs[wib][ncand][lane] = sim;
                }
                if (sim > b32 || (sim == b32 && j < bj)) {
                    s32 = b32;
                    b32 = sim;
                    bj = j;
                } else if (sim > s32) {
                    s32 = sim;
                }
                if (++ncand > Mh) {
                    atomicOr(&stats->error_bits, kErrBucketList);
                    break;
                }
                j = nxt;
            }
            if (ncand == 0) {
                m = -1;
            } else if (!weird && b32 < tau - delta) {
                m = -1;
            } else if (!weird && b32 > tau + delta && (ncand == 1 || b32 - s32 > 2.f * delta)) {
                m = bj;
            } else if (!weird && ncand <= kCandKeep) {   // exact recheck of the kept candidates near the best
                for (int q = 0; q < ncand; ++q) {
                    if (sCs[wib][q][lane] >= b32 - 2.f * delta) {
                        const int j = sCj[wib][q][lane];
                        const double sim = exact_sim(j);
                        if (sim > best || (sim == best && j < bestj)) {
                            best = sim;
                            bestj = j;
                        }
                    }
                }
                m = (bestj >= 0 && best >= tau64) ? bestj : -1;
            } else {   // exact recheck of the candidates that can still be the best
                int guard = 0;
                for (int j = head; j >= 0;) {
                    const int nxt = c.bnext[hrow + j];
                    bool near = weird;
                    if (!weird) {
                        const float ne = (float)c.knorm64[hrow + j];
                        float dt;
                        if constexpr (MEAN) {
                            if (c.kspan[hrow + j] == 255) dt = dot32_f32<E, D>(my, c.K32 + (hrow + j) * D);
                            else dt = dot32_bf16<D>(my, reinterpret_cast<const uint4*>(Kc + (hrow + j) * D));
                        } else {
                            dt = dot32_bf16<D>(my, reinterpret_cast<const uint4*>(Kc + (hrow + j) * D));
                        }
                        near = dt / sqrtf(n2 * ne) >= b32 - 2.f * delta;
                    }
                    if (near) {
                        const double sim = exact_sim(j);
                        if (sim > best || (sim == best && j < bestj)) {
                            best = sim;
                            bestj = j;
                        }
                    }
                    if (++guard > ncand) break;
                    j = nxt;
                }
                m = (bestj >= 0 && best >= tau64) ? bestj : -1;
            }
        }
        // ---- 4. publish
        const int64_t sidx = sbase + lane;
        const int t = t0 + lane;
        if constexpr (INTRA) {
            if (valid) {
                s.match[sidx] = bestj;
                s.bsim[sidx] = best;
                s.cbnext[sidx] = atomicExch(&c.cbhead[((int64_t)h << nbits) + code], t);
            }
            if (lane == 0) s.wcnt[(int64_t)h * (s.TmaxP >> 5) + w] = 0;   // counted by the dedupe kernel
        } else {
            bool first = false;   // this token starts its target's merge list: a new touched entry
            if (valid) {
                s.match[sidx] = m;
                if (m >= 0) {
                    const int old = atomicExch(&c.lhead[hrow + m], t);
                    s.lnext[sidx] = old;
                    first = old < 0;
                }
            }
            // one atomic per window for the new touched entries (a counter shared by the head)
            const unsigned fb = __ballot_sync(0xffffffffu, first);
            if (fb) {
                int base = 0;
                if (lane == __ffs(fb) - 1) base = atomicAdd(&ctr[h], __popc(fb));
                base = __shfl_sync(0xffffffffu, base, __ffs(fb) - 1);
                if (first) s.touched[(int64_t)h * s.TmaxP + base + __popc(fb & ((1u << lane) - 1u))] = m;
            }
            const unsigned un = __ballot_sync(0xffffffffu, valid && m < 0);
            if (lane == 0) s.wcnt[(int64_t)h * (s.TmaxP >> 5) + w] = __popc(un);
        }
        __syncwarp();   // the rows buffer is refilled by the warp's next window
    }
    // one bound per block: |k|^2 of the staged keys, rounded up past the fp32 sums' error
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        hre += __shfl_xor_sync(0xffffffffu, hre, o);
        mre += __shfl_xor_sync(0xffffffffu, mre, o);
    }
    if (lane == 0) {
        sKmax[wib] = kmax * (1.f + 1.f / 1024.f);
        sRe[wib][0] = hre;
        sRe[wib][1] = mre;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        unsigned a = 0, b = 0;
        for (int q = 0; q < kStageWarps; ++q) {
            m = fmaxf(m, sKmax[q]);
            a += sRe[q][0];
            b += sRe[q][1];
        }
        atomicMax(reinterpret_cast<int*>(c.kmax2s), __float_as_int(m));
        if (a) atomicAdd(&stats->hash_rechecks, (unsigned long long)a);
        if (b) atomicAdd(&stats->match_rechecks, (unsigned long long)b);
    }
    grid_dependents_launch();
    if (!INTRA) publish_sizes(c, s, ctr);
}

template <typename E, int D>
__device__ __forceinline__ double gexact_dot(const GSlice<E, D>& a, int spa, const GSlice<E, D>& b, int spb, int gl,
                                             int grp, unsigned gmask) {
    if constexpr (sizeof(E) == 2) {
        if (spa + spb <= kSpanLimit<D>) return gsum64(lane_dot64(a, b), gmask);
    }
    return gchain_dot(a, b, gl, grp, gmask);
}

template <typename E, int D>
__device__ __forceinline__ int grow_span(const GSlice<E, D>& x, unsigned gmask) {
    if constexpr (sizeof(E) == 2) return gspan_bf16<D>(x, gmask);
    return 255;
}

// ------------------------------------------------------------------ dedupe (matching inside the chunk)
constexpr int kDedupSmem = 48;   // bucket members ordered in shared memory (more: scan the codes)
//
// Used when a commit also matches tokens against entries created earlier in the same
// commit. The search left, per token, the exact best committed candidate (index and
// similarity) and grouped the chunk's tokens by (head, code): tokens can only meet
// tokens of their own bucket, so each bucket is an independent sequence. One lane
// group per bucket (started by its newest token, the list head) takes the bucket's
// tokens in ascending t. A token compares the exact cosine against every entry
// created earlier in the bucket, in creation order; with strict > the committed best
// (lower entry indices) and earlier creators keep exact ties. It then merges (into a
// committed entry: the entry's merge list; into a new entry: that entry's member
// chain, in ascending t) or creates an entry (counted in its 32-token window).
// Buckets of up to 8 tokens are ordered in the group's lanes, up to kDedupSmem in
// shared memory; larger ones visit their members by scanning the head's codes in
// token order. The last block publishes the new sizes.
template <typename E, int D>
__global__ void __launch_bounds__(kWarps * 32, 2)
dedupe_kernel(CacheView c, StageView s, double tau64, int32_t* ctr, Stats* stats) {
    grid_dependency_wait();
    __shared__ int sMem[kWarps * 4][kDedupSmem];   // one buffer per lane group
    __shared__ int sSrt[kWarps * 4][kDedupSmem];
    using G = GSlice<E, D>;
    const int lane = threadIdx.x & 31, gl = lane & 7, grp = lane >> 3;
    const unsigned gmask = 0xFFu << (8 * grp);
    const int H = c.H;
    const int64_t T = s.T;
    const int64_t rows = T * H;
    const E* Ks = reinterpret_cast<const E*>(s.Ks);
    int32_t* ntouched = ctr;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r4 = gw * 4; r4 < rows; r4 += nw * 4) {   // warp-uniform loop
        const int64_t r = r4 + grp;
        bool head = false;
        int h = 0;
        int64_t t = 0, bucket = 0;
        uint32_t code = 0;
        if (r < rows) {
            h = (int)((uint32_t)r / (uint32_t)T);
            t = r - (int64_t)h * T;
            code = s.scode[(int64_t)h * s.TmaxP + t];
            bucket = ((int64_t)h << c.nbits) + code;
            head = c.cbhead[bucket] == (int)t;
        }
        if (!head) continue;   // group-uniform; the loop has no warp-wide operations below
        const int64_t sbase = (int64_t)h * s.TmaxP;
        const int64_t hrow = (int64_t)h * c.capP;
        int cr_head = -1, cr_tail = -1;   // this bucket's new entries, in creation order
        auto process = [&](int tm) {
            const int64_t sm = sbase + tm;
            G x;
            x.load(Ks + sm * D, gl);
            const int spx = grow_span<E, D>(x, gmask);
            const double n1 = gexact_dot(x, spx, x, spx, gl, grp, gmask);
            int bj = s.match[sm];
            double bs = s.bsim[sm];
            int guard = 0;
            for (int u = cr_head; u >= 0; u = s.crnext[sbase + u]) {
                if (++guard > (int)T) break;
                G y;
                y.load(Ks + (sbase + u) * D, gl);
                const int spy = grow_span<E, D>(y, gmask);
                const double n2 = gexact_dot(y, spy, y, spy, gl, grp, gmask);
                const double dot = gexact_dot(x, spx, y, spy, gl, grp, gmask);
                const double sim = (n1 > 0.0 && n2 > 0.0) ? dot / sqrt(n1 * n2) : 0.0;
                if (sim > bs) {
                    bs = sim;
                    bj = -2 - u;
                }
            }
            const bool merge = bj != -1 && bs >= tau64;
            if (gl == 0) {
                if (merge && bj >= 0) {          // into a committed entry
                    s.match[sm] = bj;
                    const int old = atomicExch(&c.lhead[hrow + bj], tm);
                    s.lnext[sm] = old;
                    if (old < 0) s.touched[sbase + atomicAdd(&ntouched[h], 1)] = bj;
                } else if (merge) {              // into an entry created by token u
                    const int u = -2 - bj;
                    s.match[sm] = bj;
                    s.icnext[sm] = -1;
                    if (s.ichead[sbase + u] < 0) s.ichead[sbase + u] = tm;
                    else s.icnext[sbase + s.ictail[sbase + u]] = tm;
                    s.ictail[sbase + u] = tm;
                } else {                         // creates an entry
                    s.match[sm] = -1;
                    s.crnext[sm] = -1;
                    if (cr_tail >= 0) s.crnext[sbase + cr_tail] = tm;
                    atomicAdd(&s.wcnt[(int64_t)h * (s.TmaxP >> 5) + (tm >> 5)], 1);
                }
            }
            __syncwarp(gmask);
            if (!merge) {
                if (cr_head < 0) cr_head = tm;
                cr_tail = tm;
            }
        };
        // members: walk the bucket's token list (newest first) into the lanes, and up
        // to kDedupSmem of them into this group's shared buffer
        int* buf = sMem[threadIdx.x >> 3];
        int L = 0, id = 0x7fffffff;
        for (int u = (int)t; u >= 0; u = s.cbnext[sbase + u]) {
            if (gl == L) id = u;
            if (gl == 0 && L < kDedupSmem) buf[L] = u;
            if (++L > kDedupSmem) break;
        }
        __syncwarp(gmask);
        if (L <= 8) {
            int rank = 0;
            for (int k = 0; k < L; ++k) rank += (__shfl_sync(gmask, id, 8 * grp + k) < id);
            for (int q = 0; q < L; ++q) {
                const int src = __ffs((__ballot_sync(gmask, rank == q && gl < L) >> (8 * grp)) & 0xFFu) - 1;
                process(__shfl_sync(gmask, id, 8 * grp + src));
            }
        } else if (L <= kDedupSmem) {
            // order the ids in shared memory: each lane places its ids at their ranks
            int* srt = sSrt[threadIdx.x >> 3];
            for (int a = gl; a < L; a += 8) {
                const int mine = buf[a];
                int rank = 0;
                for (int b2 = 0; b2 < L; ++b2) rank += (buf[b2] < mine);
                srt[rank] = mine;
            }
            __syncwarp(gmask);
            for (int q = 0; q < L; ++q) process(srt[q]);
        } else {
            for (int64_t t0 = 0; t0 < T; t0 += 8) {
                const bool hit = t0 + gl < T && s.scode[sbase + t0 + gl] == code;
                unsigned b = (__ballot_sync(gmask, hit) >> (8 * grp)) & 0xFFu;
                while (b) {
                    const int k = __ffs(b) - 1;
                    b &= b - 1;
                    process((int)t0 + k);
                }
            }
        }
        if (gl == 0) c.cbhead[bucket] = -1;
        __syncwarp(gmask);
    }
    grid_dependents_launch();
    publish_sizes(c, s, ctr);
}

// |k|^2 of a row held by a lane group, in fp64 with the value of the index-order
// sum (exact by the span rule for bf16 rows that satisfy it, else the chain).
template <typename E, int D>
__device__ __forceinline__ double gnorm64(const GSlice<E, D>& x, int span, int gl, int grp, unsigned gmask) {
    if constexpr (sizeof(E) == 2) {
        if (2 * span <= kSpanLimit<D>) return gsum64(lane_dot64(x, x), gmask);
    }
    return gchain_dot(x, x, gl, grp, gmask);
}

// ------------------------------------------------------------------ commit: append + merge
//
// One kernel applies the decisions the staging of the chunk took. Its warps take work
// items in order: first the 32-token windows of every head (append), then groups of
// four slots of the per-head lists of touched entries (merge). The two kinds write
// disjoint entries (new ones at M_h and beyond, merged ones below M_h). The last block
// to finish publishes the new sizes and clears the per-commit counters.
//
// Append: unmatched tokens of a window take consecutive entries in token order:
// dest = M_h + (unmatched tokens of earlier windows) + (unmatched lanes below). Each
// becomes an entry (key, value mean, n = 1, log2 n = 0, code, |k|^2 with the value of
// the fp64 index-order sum) and is pushed on its bucket's list; lane groups copy two
// rows each per pass. With the intra_chunk option an entry created in the commit also
// averages the later tokens of the chunk that merged into it.
//
// Merge: one lane group per touched entry. The matched tokens' values are summed in
// fp32 in ascending token order (whatever order the atomics built the list in), then
// v <- (n v + sum) / (n + m), n <- n + m (Lemma 5.1: the merged entry carries the mean
// of its group and the group size). Lists of up to 8 tokens are ordered inside the
// group; longer ones go to the whole warp, which orders up to kListSmem tokens in
// shared memory and otherwise gathers them by scanning the head's match targets in
// token order. With running-mean keys every merge goes to the whole warp, which also
// averages the keys the same way in fp32, re-hashes the new key and records the entry
// when its code changed (the re-bucketing kernels then move it).
constexpr int kListSmem = 256;

constexpr int kHeadSlots = 64;   // heads whose bounds a commit block gathers in shared memory

// max into a per-block slot of head h when it has one, else straight into the global bound
__device__ __forceinline__ void bound_max(float* slots, float* global_h, int h, float v) {
    if (h < kHeadSlots) atomicMax(reinterpret_cast<int*>(slots + h), __float_as_int(v));   // floats >= 0
    else atomicMax(reinterpret_cast<int*>(global_h), __float_as_int(v));
}

template <typename E, int D, bool MEAN>
struct CommitArgs {
    CacheView c;
    StageView s;
    const float* R;       // device normals (fp64 re-checks of the new keys' codes)
    const float* Rnorm;   // |R_b|, rounded up
    int32_t* ctr;
    Stats* stats;
};

template <typename E, int D>
__device__ __forceinline__ void append_window(const CacheView& c, const StageView& s, int h, int w, int* sSrc,
                                              int lane) {
    using G = GSlice<E, D>;
    constexpr int EPG = G::EPG;
    const int gl = lane & 7, grp = lane >> 3;
    const unsigned gmask = 0xFFu << (8 * grp);
    const int64_t T = s.T;
    const E* Ks = reinterpret_cast<const E*>(s.Ks);
    const E* Vs = reinterpret_cast<const E*>(s.Vs);
    const int32_t* wc = s.wcnt + (int64_t)h * (s.TmaxP >> 5);
    int prefix = 0;
#pragma unroll 4
    for (int q = lane; q < w; q += 32) prefix += wc[q];   // independent loads, unrolled
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) prefix += __shfl_xor_sync(0xffffffffu, prefix, o);
    const int64_t t = (int64_t)w * 32 + lane;
    const bool valid = t < T;
    const int64_t sidx = (int64_t)h * s.TmaxP + t;
    const int m = valid ? s.match[sidx] : 0;
    const bool un = valid && m == -1;   // -2 - u: joins the entry token u creates
    const unsigned bal = __ballot_sync(0xffffffffu, un);
    const int rank = __popc(bal & ((1u << lane) - 1u));
    const int base = c.M[h] + prefix;
    if (valid) {
        if (m >= -1) {
            s.dest[sidx] = un ? base + rank : m;
            s.lmatch[sidx] = m;
        }
        s.lcode[sidx] = s.scode[sidx];
    }
    if (un) sSrc[rank] = lane;
    __syncwarp();
    const int nun = __popc(bal);
    const int64_t hrow = (int64_t)h * c.capP;
    const int64_t wrow = (int64_t)h * s.TmaxP + (int64_t)w * 32;
    float kmax = 0.f;   // largest |k|^2 of the entries this warp creates
    for (int k0 = 0; k0 < nun; k0 += 8) {   // warp-uniform
        G kr[2], vr[2];
        int64_t st[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int k = k0 + 4 * u + grp;
            st[u] = k < nun ? wrow + sSrc[k] : -1;
            if (st[u] >= 0) {
                kr[u].load(Ks + st[u] * D, gl);
                vr[u].load(Vs + st[u] * D, gl);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (st[u] < 0) continue;   // group-uniform
            const int k = k0 + 4 * u + grp;
            const int64_t e = hrow + base + k;
            kr[u].store(reinterpret_cast<E*>(c.Kc) + e * D, gl);
            if (c.K32 && (void*)c.K32 != c.Kc) {   // running-mean keys, bf16 storage: the fp32 key
                float4* k32 = reinterpret_cast<float4*>(c.K32 + e * D + gl * EPG);
#pragma unroll
                for (int q = 0; q < EPG / 4; ++q)
                    k32[q] = make_float4(kr[u].at(4 * q), kr[u].at(4 * q + 1), kr[u].at(4 * q + 2), kr[u].at(4 * q + 3));
            }
            float4* v32 = reinterpret_cast<float4*>(c.V32 + e * D + gl * EPG);
            int members = 0;   // later tokens of this chunk that joined this new entry
            const int64_t sbase = (int64_t)h * s.TmaxP;
            int tm = s.ichead[st[u]];
            if (tm < 0) {
                vr[u].store(reinterpret_cast<E*>(c.Vc) + e * D, gl);
#pragma unroll
                for (int q = 0; q < EPG / 4; ++q)
                    v32[q] = make_float4(vr[u].at(4 * q), vr[u].at(4 * q + 1), vr[u].at(4 * q + 2),
                                         vr[u].at(4 * q + 3));
            } else {   // group-uniform: mean of the creating token and its members, in t order
                float acc[EPG];
#pragma unroll
                for (int i = 0; i < EPG; ++i) acc[i] = 0.f;
                for (; tm >= 0; tm = s.icnext[sbase + tm]) {
                    G vm;
                    vm.load(Vs + (sbase + tm) * D, gl);
#pragma unroll
                    for (int i = 0; i < EPG; ++i) acc[i] = __fadd_rn(acc[i], vm.at(i));
                    if (gl == 0) {
                        s.lmatch[sbase + tm] = base + k;
                        s.dest[sbase + tm] = base + k;
                    }
                    if (++members > (int)T) break;
                }
                const float ft = (float)(1 + members);
                float nv[EPG];
#pragma unroll
                for (int i = 0; i < EPG; ++i) nv[i] = __fdiv_rn(__fadd_rn(vr[u].at(i), acc[i]), ft);
#pragma unroll
                for (int q = 0; q < EPG / 4; ++q)
                    v32[q] = make_float4(nv[4 * q], nv[4 * q + 1], nv[4 * q + 2], nv[4 * q + 3]);
                G out;
                out.from_floats(nv);
                out.store(reinterpret_cast<E*>(c.Vc) + e * D, gl);
                if (gl == 0) s.ichead[st[u]] = -1;
            }
            int span = 255;
            if constexpr (sizeof(E) == 2) span = min(gspan_bf16<D>(kr[u], gmask), 255);
            const double nk = gnorm64(kr[u], span, gl, grp, gmask);
            kmax = fmaxf(kmax, __double2float_ru(nk));
            if (gl == 0) {
                const uint32_t code = s.scode[st[u]];
                c.knorm64[e] = nk;
                c.kspan[e] = (uint8_t)span;
                c.cnt[e] = 1 + members;
                c.bias2[e] = log2f((float)(1 + members));
                if (members) atomicMax(reinterpret_cast<int*>(&c.bmax[h]), __float_as_int(log2f((float)(1 + members))));
                c.code[e] = code;
                c.bnext[e] = atomicExch(&c.bhead[((int64_t)h << c.nbits) + code], base + k);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    if (lane == 0 && nun > 0) atomicMax(reinterpret_cast<int*>(&c.kmax2[h]), __float_as_int(kmax));
    __syncwarp();
}

// One touched entry j of head h, merged by the whole warp (lane l: elements
// [l EPL, l EPL + EPL)). MEAN: the key is averaged too, then re-hashed.
template <typename E, int D, bool MEAN>
__device__ void merge_entry_warp(const CommitArgs<E, D, MEAN>& a, int h, int j, int32_t* sIds, int32_t* sSorted,
                                 float* sRow, float* sBm, float* sKm, int lane) {
    const CacheView& c = a.c;
    const StageView& s = a.s;
    constexpr int EPL = D / 32;
    using IO = RowIO<E, EPL>;
    const int64_t T = s.T;
    const int64_t sbase = (int64_t)h * s.TmaxP;
    const int64_t e = (int64_t)h * c.capP + j;
    const E* Vs = reinterpret_cast<const E*>(s.Vs);
    const E* Ks = reinterpret_cast<const E*>(s.Ks);
    int L = 0, id = 0x7fffffff;
    for (int tt = c.lhead[e]; tt >= 0; tt = s.lnext[sbase + tt]) {
        if (L < 32 && lane == L) id = tt;
        if (L < kListSmem && lane == 0) sIds[L] = tt;
        ++L;
        if (L > (int)T) break;   // a list is never longer than the chunk
    }
    __syncwarp();
    float acc[EPL], kacc[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) acc[q] = kacc[q] = 0.f;
    auto add_row = [&](int tt) {
        float v[EPL];
        IO::to_float(IO::load(Vs + (sbase + tt) * D, lane), v);
#pragma unroll
        for (int q = 0; q < EPL; ++q) acc[q] = __fadd_rn(acc[q], v[q]);
        if constexpr (MEAN) {
            float k[EPL];
            IO::to_float(IO::load(Ks + (sbase + tt) * D, lane), k);
#pragma unroll
            for (int q = 0; q < EPL; ++q) kacc[q] = __fadd_rn(kacc[q], k[q]);
        }
    };
    if (L <= 32) {
        int rank = 0;
        for (int k = 0; k < L; ++k) rank += (__shfl_sync(0xffffffffu, id, k) < id);
        for (int q2 = 0; q2 < L; ++q2) {
            const int src = __ffs(__ballot_sync(0xffffffffu, rank == q2 && lane < L)) - 1;
            add_row(__shfl_sync(0xffffffffu, id, src));
        }
    } else if (L <= kListSmem) {
        for (int p = lane; p < L; p += 32) {
            const int mine = sIds[p];
            int rank = 0;
            for (int b = 0; b < L; ++b) rank += (sIds[b] < mine);
            sSorted[rank] = mine;
        }
        __syncwarp();
        for (int q2 = 0; q2 < L; ++q2) add_row(sSorted[q2]);
    } else {
        for (int64_t t0 = 0; t0 < T; t0 += 32) {
            const bool hit = t0 + lane < T && s.match[sbase + t0 + lane] == j;
            unsigned b = __ballot_sync(0xffffffffu, hit);
            while (b) {
                const int src = __ffs(b) - 1;
                b &= b - 1;
                add_row((int)t0 + src);
            }
        }
    }
    const int nold = c.cnt[e];
    const int ntot = nold + L;
    const float fn = (float)nold, ft = (float)ntot;
    float nv[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
        const float old = c.V32[e * D + lane * EPL + q];
        nv[q] = __fdiv_rn(__fadd_rn(__fmul_rn(fn, old), acc[q]), ft);
        c.V32[e * D + lane * EPL + q] = nv[q];
    }
    IO::store(reinterpret_cast<E*>(c.Vc) + e * D, lane, IO::from_float(nv));
    if constexpr (MEAN) {
        // k <- (n k + sum k_t) / (n + m) in fp32, the same operations as the values
        float nk[EPL];
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const float old = c.K32[e * D + lane * EPL + q];
            nk[q] = __fdiv_rn(__fadd_rn(__fmul_rn(fn, old), kacc[q]), ft);
            c.K32[e * D + lane * EPL + q] = nk[q];
        }
        const typename IO::V kst = IO::from_float(nk);
        IO::store(reinterpret_cast<E*>(c.Kc) + e * D, lane, kst);
        // the storage copy's |k|^2 bounds the attention logits
        float ks[EPL];
        IO::to_float(kst, ks);
        float ks2 = 0.f;
#pragma unroll
        for (int q = 0; q < EPL; ++q) ks2 = fmaf(ks[q], ks[q], ks2);
        ks2 = warp_sum(ks2);
        // span of the new key when every element is a bf16 value (else 255: the search
        // then takes the chain over the fp32 key)
        bool exact16 = true;
        int emax = 0, emin = 255;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            const uint32_t u = __float_as_uint(nk[q]);
            exact16 = exact16 && (u & 0xffffu) == 0u;
            const uint32_t hb = u >> 16;
            if (hb & 0x7fffu) {
                const int f = max((int)((hb >> 7) & 0xffu), 1);
                emax = max(emax, f);
                emin = min(emin, f);
            }
        }
        exact16 = __all_sync(0xffffffffu, exact16) && sizeof(E) == 2;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
            emin = min(emin, __shfl_xor_sync(0xffffffffu, emin, o));
        }
        int span = exact16 ? min(emax >= emin ? emax - emin + 7 : 0, 255) : 255;
        // |k|^2: exact (any order) when the key is a bf16 row within the exponent-span rule;
        // otherwise the fp32 sum is stored and the span set to 255, which makes the search
        // form the exact value (the index-order chain over the fp32 key) whenever it needs it.
        float n2 = 0.f;
        double n64 = 0.0;
#pragma unroll
        for (int q = 0; q < EPL; ++q) {
            n2 = fmaf(nk[q], nk[q], n2);
            n64 += (double)(nk[q] * nk[q]);   // exact products when nk holds bf16 values
        }
        n2 = warp_sum(n2);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) n64 += __shfl_xor_sync(0xffffffffu, n64, o);
        if (!(exact16 && 2 * span <= kSpanLimit<D>)) {
            span = 255;
            if constexpr (sizeof(E) == 2) {
                n64 = (double)n2;
            } else {   // fp32 storage (the search takes the exact path for every candidate): the chain here
#pragma unroll
                for (int q = 0; q < EPL; ++q) sRow[lane * EPL + q] = nk[q];
                __syncwarp();
                double acc = 0.0;
                if (lane == 0)
                    for (int i = 0; i < D; ++i) acc = fma((double)sRow[i], (double)sRow[i], acc);
                n64 = __shfl_sync(0xffffffffu, acc, 0);
                __syncwarp();
            }
        }
        // the code of the new key: partial projections of the lane's elements, a
        // reduce-scatter leaves <R_b, k> (fp32) on lane b, kept outside the rounding bound
        // and otherwise redone in fp64 in index order over the key staged in shared memory
        float v[32];
#pragma unroll
        for (int b = 0; b < 32; ++b) {
            float t = 0.f;
            if (b < c.nbits) {
#pragma unroll
                for (int q = 0; q < EPL; ++q) t = fmaf(a.R[b * D + lane * EPL + q], nk[q], t);
            }
            v[b] = t;
        }
        const float p = reduce_scatter<32>(v, lane);
        const float nx = sqrtf(n2);
        const float gam2 = 2.f * (float)(D + 2) * kU32;
        bool bit = p >= 0.f;
        const bool need = lane < c.nbits && !(fabsf(p) > gam2 * a.Rnorm[lane] * nx + 1e-30f);
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
            for (int q = 0; q < EPL; ++q) sRow[lane * EPL + q] = nk[q];
            __syncwarp();
            if (need) {
                double acc = 0.0;
                for (int i = 0; i < D; ++i) acc = fma((double)a.R[lane * D + i], (double)sRow[i], acc);
                bit = acc >= 0.0;
            }
            __syncwarp();   // sRow is reused by the warp's next entry
        }
        const uint32_t code = __ballot_sync(0xffffffffu, lane < c.nbits && bit);
        const unsigned nre = __popc(__ballot_sync(0xffffffffu, need));
        if (lane == 0) {
            c.knorm64[e] = n64;
            c.kspan[e] = (uint8_t)span;
            bound_max(sKm, &c.kmax2[h], h, ks2 * (1.f + 1.f / 1024.f));
            if (nre) atomicAdd(&a.stats->hash_rechecks, (unsigned long long)nre);
            const uint32_t oc = c.code[e];
            if (code != oc) {   // the entry leaves its bucket after this commit
                c.code[e] = code;
                const int slot = atomicAdd(&a.ctr[2 * c.H + 4 + h], 1);
                s.moved[sbase + slot] = j;
                s.movedold[sbase + slot] = oc;
            }
        }
    }
    __syncwarp();
    if (lane == 0) {
        c.cnt[e] = ntot;
        c.bias2[e] = log2f(ft);
        c.lhead[e] = -1;
        bound_max(sBm, &c.bmax[h], h, log2f(ft));   // log2 n >= 0
    }
    __syncwarp();
}

// Four touched-list slots q4 .. q4+3 (slot q = h T + i is the i-th touched entry of
// head h, when i < ctr[h]), one lane group each; lists longer than 8 tokens (every
// list with running-mean keys) go to the whole warp afterwards.
template <typename E, int D, bool MEAN>
__device__ __forceinline__ void merge_quad(const CommitArgs<E, D, MEAN>& a, int64_t q4, int32_t* sIds,
                                           int32_t* sSorted, float* sRow, float* sBm, float* sKm, int lane) {
    const CacheView& c = a.c;
    const StageView& s = a.s;
    using G = GSlice<E, D>;
    constexpr int EPG = G::EPG;
    const int gl = lane & 7, grp = lane >> 3;
    const unsigned gmask = 0xFFu << (8 * grp);
    const int64_t T = s.T;
    const int H = c.H;
    const E* Vs = reinterpret_cast<const E*>(s.Vs);
    const int64_t q = q4 + grp;
    int h = 0, j = -1;
    bool act = false, big = false;
    if (q < (int64_t)H * T) {
        h = (int)((uint32_t)q / (uint32_t)T);
        const int slot = (int)(q - (int64_t)h * T);
        act = slot < a.ctr[h];
        if (act) j = s.touched[(int64_t)h * s.TmaxP + slot];
    }
    if (act && MEAN) {
        big = true;
    } else if (act) {   // group-uniform
        const int64_t sbase = (int64_t)h * s.TmaxP;
        const int64_t e = (int64_t)h * c.capP + j;
        const float4* v32p = reinterpret_cast<const float4*>(c.V32 + e * D + gl * EPG);
        float4 old[EPG / 4];
#pragma unroll
        for (int k = 0; k < EPG / 4; ++k) old[k] = v32p[k];
        const int nold = c.cnt[e];
        int L = 0, id = 0x7fffffff;
        for (int tt = c.lhead[e]; tt >= 0; tt = s.lnext[sbase + tt]) {
            if (gl == L) id = tt;
            if (++L > 8) break;
        }
        if (L > 8) {
            big = true;
        } else {
            int rank = 0;
            for (int k = 0; k < L; ++k) rank += (__shfl_sync(gmask, id, 8 * grp + k) < id);
            int srt = 0;   // lane gl gets the gl-th smallest token
            for (int k = 0; k < L; ++k) {
                const int idk = __shfl_sync(gmask, id, 8 * grp + k);
                const int rk = __shfl_sync(gmask, rank, 8 * grp + k);
                if (rk == gl) srt = idk;
            }
            float acc[EPG];
#pragma unroll
            for (int i = 0; i < EPG; ++i) acc[i] = 0.f;
            G cur;
            cur.load(Vs + (sbase + __shfl_sync(gmask, srt, 8 * grp)) * D, gl);
            for (int k = 0; k < L; ++k) {
                G nxt;
                const int tn = __shfl_sync(gmask, srt, 8 * grp + ((k + 1) & 7));
                if (k + 1 < L) nxt.load(Vs + (sbase + tn) * D, gl);
#pragma unroll
                for (int i = 0; i < EPG; ++i) acc[i] = __fadd_rn(acc[i], cur.at(i));
                cur = nxt;
            }
            const int ntot = nold + L;
            const float fn = (float)nold, ft = (float)ntot;
            float nv[EPG];
#pragma unroll
            for (int k = 0; k < EPG / 4; ++k) {
                nv[4 * k] = __fdiv_rn(__fadd_rn(__fmul_rn(fn, old[k].x), acc[4 * k]), ft);
                nv[4 * k + 1] = __fdiv_rn(__fadd_rn(__fmul_rn(fn, old[k].y), acc[4 * k + 1]), ft);
                nv[4 * k + 2] = __fdiv_rn(__fadd_rn(__fmul_rn(fn, old[k].z), acc[4 * k + 2]), ft);
                nv[4 * k + 3] = __fdiv_rn(__fadd_rn(__fmul_rn(fn, old[k].w), acc[4 * k + 3]), ft);
            }
            float4* v32w = reinterpret_cast<float4*>(c.V32 + e * D + gl * EPG);
#pragma unroll
            for (int k = 0; k < EPG / 4; ++k)
                v32w[k] = make_float4(nv[4 * k], nv[4 * k + 1], nv[4 * k + 2], nv[4 * k + 3]);
            G out;
            out.from_floats(nv);
            out.store(reinterpret_cast<E*>(c.Vc) + e * D, gl);
            if (gl == 0) {
                c.cnt[e] = ntot;
                c.bias2[e] = log2f(ft);
                c.lhead[e] = -1;
                bound_max(sBm, &c.bmax[h], h, log2f(ft));   // log2 n >= 0
            }
        }
    }
    __syncwarp();
    unsigned bigm = __ballot_sync(0xffffffffu, big && gl == 0);
    while (bigm) {
        const int src = __ffs(bigm) - 1;
        bigm &= bigm - 1;
        const int bh = __shfl_sync(0xffffffffu, h, src);
        const int bj = __shfl_sync(0xffffffffu, j, src);
        merge_entry_warp<E, D, MEAN>(a, bh, bj, sIds, sSorted, sRow, sBm, sKm, lane);
    }
}

// The last block of a grid to finish (every thread calls this once, after its last
// update). With `sizes`, it publishes the new cache sizes. With `clear_lo` it clears
// the counters [0, 2H+4) (touched lists, sizes, abort flag and tickets); with
// `clear_moved`, the moved-entry counters [2H+4, 3H+4); its own ticket always.
__device__ void commit_done(const CacheView& c, int32_t* ctr, int ticket, bool sizes, bool clear_lo,
                            bool clear_moved) {
    const int H = c.H;
    __shared__ bool last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&ctr[ticket], 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    if (sizes)
        for (int h = threadIdx.x; h < H; h += blockDim.x) c.M[h] = __ldcg(&ctr[H + h]);
    __syncthreads();
    if (clear_lo)
        for (int i = threadIdx.x; i < 2 * H + 4; i += blockDim.x) ctr[i] = 0;
    if (clear_moved)
        for (int i = 2 * H + 4 + threadIdx.x; i < 3 * H + 4; i += blockDim.x) ctr[i] = 0;
    if (threadIdx.x == 0) ctr[ticket] = 0;
}

template <typename E, int D, bool MEAN>
__global__ void __launch_bounds__(kWarps * 32, 2) commit_kernel(const CommitArgs<E, D, MEAN> a) {
    grid_dependency_wait();
    __shared__ int sSrc[kWarps][32];
    __shared__ int32_t sIds[kWarps][kListSmem];
    __shared__ int32_t sSorted[kWarps][kListSmem];
    __shared__ float sRow[kWarps][MEAN ? D : 1];   // running-mean keys: the new key, for the re-hash
    __shared__ float sBm[kHeadSlots], sKm[kHeadSlots];   // this block's bounds of log2 n and |k|^2 per head
    const CacheView& c = a.c;
    const StageView& s = a.s;
    const int H = c.H;
    if (__ldcg(&a.ctr[2 * H])) return;   // refused: nothing changes, the decisions stay for a retry
    for (int i = threadIdx.x; i < kHeadSlots; i += blockDim.x) sBm[i] = sKm[i] = 0.f;
    __syncthreads();
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t T = s.T;
    const int64_t nA = (int64_t)H * ((T + 31) >> 5);
    const int64_t nM = ((int64_t)H * T + 3) / 4;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t it = gw; it < nA + nM; it += nw) {   // warp-uniform
        if (it < nA) {
            const int64_t nwin = (T + 31) >> 5;
            append_window<E, D>(c, s, (int)(it / nwin), (int)(it % nwin), sSrc[wib], lane);
        } else {
            merge_quad<E, D, MEAN>(a, (it - nA) * 4, sIds[wib], sSorted[wib], sRow[wib], sBm, sKm, lane);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < H && i < kHeadSlots; i += blockDim.x) {
        if (sBm[i] > 0.f) atomicMax(reinterpret_cast<int*>(&c.bmax[i]), __float_as_int(sBm[i]));
        if (sKm[i] > 0.f) atomicMax(reinterpret_cast<int*>(&c.kmax2[i]), __float_as_int(sKm[i]));
    }
    grid_dependents_launch();
    commit_done(c, a.ctr, 2 * H + 2, true, true, !MEAN);
}

// ------------------------------------------------------------------ re-bucketing (running-mean keys)
//
// An entry whose merged key changed code leaves its old bucket and joins the new one.
// Unlink: for every moved entry, the first thread to claim the old bucket rebuilds that
// bucket's list without the entries whose code is no longer the bucket's (so one thread
// owns each list). Push: every moved entry is pushed on its new bucket's list and the
// claims are released; the last block clears the moved-entry counters.
__global__ void rebucket_unlink_kernel(CacheView c, StageView s, const int32_t* ctr, int32_t* claim, Stats* stats) {
    grid_dependency_wait();
    const int H = c.H;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < (int64_t)H * s.TmaxP;
         q += (int64_t)gridDim.x * blockDim.x) {
        const int h = (int)(q / s.TmaxP);
        const int idx = (int)(q - (int64_t)h * s.TmaxP);
        if (idx >= __ldcg(&ctr[2 * H + 4 + h])) continue;
        const uint32_t oc = s.movedold[q];
        const int64_t b = ((int64_t)h << c.nbits) + oc;
        if (atomicExch(&claim[b], 1) != 0) continue;
        const int64_t hrow = (int64_t)h * c.capP;
        const int Mh = c.M[h];
        int head = -1, tail = -1, guard = 0;
        for (int e = c.bhead[b]; e >= 0;) {
            const int nx = c.bnext[hrow + e];
            if (c.code[hrow + e] == oc) {
                if (tail < 0) head = e;
                else c.bnext[hrow + tail] = e;
                tail = e;
            }
            if (++guard > Mh) {
                atomicOr(&stats->error_bits, kErrBucketList);
                break;
            }
            e = nx;
        }
        if (tail >= 0) c.bnext[hrow + tail] = -1;
        c.bhead[b] = head;
    }
    grid_dependents_launch();
}

__global__ void rebucket_push_kernel(CacheView c, StageView s, int32_t* ctr, int32_t* claim) {
    grid_dependency_wait();
    const int H = c.H;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < (int64_t)H * s.TmaxP;
         q += (int64_t)gridDim.x * blockDim.x) {
        const int h = (int)(q / s.TmaxP);
        const int idx = (int)(q - (int64_t)h * s.TmaxP);
        if (idx >= __ldcg(&ctr[2 * H + 4 + h])) continue;
        const int j = s.moved[q];
        const int64_t e = (int64_t)h * c.capP + j;
        c.bnext[e] = atomicExch(&c.bhead[((int64_t)h << c.nbits) + c.code[e]], j);
        claim[((int64_t)h << c.nbits) + s.movedold[q]] = 0;
    }
    grid_dependents_launch();
    commit_done(c, ctr, 2 * H + 3, false, false, true);
}

template <typename E, int D, int NBP, bool INTRA, bool MEAN>
cudaError_t stage_n(const CacheView& c, const StageView& s, const void* K, const void* V, const float* R,
                    const float* Rhost, const float* Rnorm_host, float tau, int32_t* ctr, Stats* stats,
                    int* launches, cudaStream_t st) {
    auto kern = stage_search_kernel<E, D, NBP, INTRA, MEAN>;
    constexpr int smem = StageSmem<E, D>::BYTES;
    cudaError_t e = smem_attr_once(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    StagePlanes<D, NBP> pl;
    for (int b = 0; b < NBP; ++b) {
        for (int i = 0; i < D; ++i) pl.v[b * D + i] = b < c.nbits ? Rhost[b * D + i] : 0.f;
        pl.rn[b] = b < c.nbits ? Rnorm_host[b] : 0.f;
    }
    const int64_t items = (int64_t)c.H * ((s.T + 31) / 32);
    const int grid = grid_for_rows(items, kStageWarps, 148 * 4);
    e = launch_pdl_smem(kern, grid, kStageWarps * 32, smem, st, reinterpret_cast<const E*>(K),
                        reinterpret_cast<const E*>(V), c, s, pl, tau, ctr, stats);
    *launches += 1;
    if (e == cudaSuccess && INTRA) {
        const int dgrid = grid_for_rows(s.T * c.H, 4 * kWarps, 148 * 2);
        e = launch_pdl(dedupe_kernel<E, D>, dgrid, kWarps * 32, st, c, s, (double)tau, ctr, stats);
        *launches += 1;
    }
    return e;
}

template <typename E, int D, bool INTRA, bool MEAN>
cudaError_t stage_t(const CacheView& c, const StageView& s, const void* K, const void* V, const float* R,
                    const float* Rhost, const float* Rnorm_host, float tau, int32_t* ctr, Stats* stats,
                    int* launches, cudaStream_t st) {
    if constexpr (sizeof(E) == 4)   // fp32 storage hashes with plain loops: one width of normals
        return stage_n<E, D, 32, INTRA, MEAN>(c, s, K, V, R, Rhost, Rnorm_host, tau, ctr, stats, launches, st);
    if (c.nbits <= 8)
        return stage_n<E, D, 8, INTRA, MEAN>(c, s, K, V, R, Rhost, Rnorm_host, tau, ctr, stats, launches, st);
    if (c.nbits <= 16)
        return stage_n<E, D, 16, INTRA, MEAN>(c, s, K, V, R, Rhost, Rnorm_host, tau, ctr, stats, launches, st);
    return stage_n<E, D, 32, INTRA, MEAN>(c, s, K, V, R, Rhost, Rnorm_host, tau, ctr, stats, launches, st);
}

template <typename E, int D>
cudaError_t stage_mode(const CacheView& c, const StageView& s, bool intra, bool mean, const void* K, const void* V,
                       const float* R, const float* Rhost, const float* Rnorm_host, float tau, int32_t* ctr,
                       Stats* stats, int* launches, cudaStream_t st) {
    if (intra) return stage_t<E, D, true, false>(c, s, K, V, R, Rhost, Rnorm_host, tau, ctr, stats, launches, st);
    if (mean) return stage_t<E, D, false, true>(c, s, K, V, R, Rhost, Rnorm_host, tau, ctr, stats, launches, st);
    return stage_t<E, D, false, false>(c, s, K, V, R, Rhost, Rnorm_host, tau, ctr, stats, launches, st);
}

template <typename E, int D, bool MEAN>
cudaError_t commit_t(const CacheView& c, const StageView& s, const float* R, const float* Rnorm, int32_t* ctr,
                     int32_t* claim, Stats* stats, int* launches, cudaStream_t st) {
    const int64_t items = (int64_t)c.H * ((s.T + 31) / 32) + ((int64_t)c.H * s.T + 3) / 4;
    const int grid = grid_for_rows(items, kWarps, 148 * 2);
    CommitArgs<E, D, MEAN> a{c, s, R, Rnorm, ctr, stats};
    cudaError_t e = launch_pdl(commit_kernel<E, D, MEAN>, grid, kWarps * 32, st, a);
    *launches += 1;
    if (MEAN && e == cudaSuccess) {
        const int rgrid = grid_for_rows((int64_t)c.H * s.TmaxP, 256, 148 * 2);
        e = launch_pdl(rebucket_unlink_kernel, rgrid, 256, st, c, s, (const int32_t*)ctr, claim, stats);
        if (e == cudaSuccess) e = launch_pdl(rebucket_push_kernel, rgrid, 256, st, c, s, ctr, claim);
        *launches += 2;
    }
    return e;
}

}  // namespace

cudaError_t launch_stage(const CacheView& c, const StageView& s, int dtype, bool intra, bool mean, const void* K,
                         const void* V, const float* R, const float* Rhost, const float* Rnorm_host, float tau,
                         int32_t* ctr, Stats* stats, int* launches, cudaStream_t st) {
    if (dtype == 0)
        return c.d == 128 ? stage_mode<__nv_bfloat16, 128>(c, s, intra, mean, K, V, R, Rhost, Rnorm_host, tau, ctr,
                                                           stats, launches, st)
                          : stage_mode<__nv_bfloat16, 64>(c, s, intra, mean, K, V, R, Rhost, Rnorm_host, tau, ctr,
                                                          stats, launches, st);
    return c.d == 128 ? stage_mode<float, 128>(c, s, intra, mean, K, V, R, Rhost, Rnorm_host, tau, ctr, stats,
                                               launches, st)
                      : stage_mode<float, 64>(c, s, intra, mean, K, V, R, Rhost, Rnorm_host, tau, ctr, stats,
                                              launches, st);
}

cudaError_t launch_commit(const CacheView& c, const StageView& s, int dtype, bool mean, const float* R,
                          const float* Rnorm, int32_t* ctr, int32_t* claim, Stats* stats, int* launches,
                          cudaStream_t st) {
    if (dtype == 0) {
        if (c.d == 128)
            return mean ? commit_t<__nv_bfloat16, 128, true>(c, s, R, Rnorm, ctr, claim, stats, launches, st)
                        : commit_t<__nv_bfloat16, 128, false>(c, s, R, Rnorm, ctr, claim, stats, launches, st);
        return mean ? commit_t<__nv_bfloat16, 64, true>(c, s, R, Rnorm, ctr, claim, stats, launches, st)
                    : commit_t<__nv_bfloat16, 64, false>(c, s, R, Rnorm, ctr, claim, stats, launches, st);
    }
    if (c.d == 128)
        return mean ? commit_t<float, 128, true>(c, s, R, Rnorm, ctr, claim, stats, launches, st)
                    : commit_t<float, 128, false>(c, s, R, Rnorm, ctr, claim, stats, launches, st);
    return mean ? commit_t<float, 64, true>(c, s, R, Rnorm, ctr, claim, stats, launches, st)
                : commit_t<float, 64, false>(c, s, R, Rnorm, ctr, claim, stats, launches, st);
}

}  // namespace tc
