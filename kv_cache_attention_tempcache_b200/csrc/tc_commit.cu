// TempCache commit path: stage + hash, bucketed top-1 search with the merge
// decision, append in token order, and the deterministic list merge.
//
// FAST-AR technical summary, section 2.A "TempCache": each key of the current
// chunk is hashed with locality-sensitive hashing, its top-1 neighbour among the
// earlier cache entries is found, and near-duplicates above a similarity threshold
// are merged with their values averaged; the rest extend the cache.
//
// Exactness of the integer results. Every decision here (a hash bit, the best
// candidate, merge or not) is defined on fp64 dot products summed in index order
// 0..d-1 (products of bf16/fp32 values are exact in fp64). The kernels first
// compute the same dots in fp32 and keep the fp32 decision only when it is
// certified: when the fp32 value is farther from the decision boundary than a
// rigorous bound on its rounding error. Otherwise they recompute the fp64 sums in
// index order, the same sequence of IEEE operations as the definition, so codes,
// matches and the append order are bit-identical to it.
#include "tc_internal.h"
#include "tc_device.cuh"

#include <math.h>

namespace tc {

namespace {

// ------------------------------------------------------------------ stage + hash
//
// One warp per input row r = t*H + h of the token-major chunk, four rows in flight.
// The row is copied to the head-major staging buffer. Lane l keeps columns
// [l*EPL, l*EPL + EPL) of every hyperplane in registers (as bf16 pairs: the normals
// are bf16 values) and forms the partial dot products of its columns; a
// reduce-scatter butterfly then leaves the full <R_b, k> (fp32) on lane b. Bit b
// keeps the fp32 sign when
//   |<R_b,k>| > 2 (d+2) u |R_b| |k|   (u = 2^-24; any summation order errs by at
//                                      most (d+2) u sum|R_bi k_i| <= (d+2) u |R_b||k|,
//                                      doubled for margin)
// and otherwise lane b redoes the sum in fp64 in index order. Bit b = [<R_b,k> >= 0].

template <typename E, int D, int NBP>
__global__ void __launch_bounds__(kWarps * 32, NBP <= 8 ? 3 : (NBP <= 16 ? 2 : 1))
stage_hash_kernel(const E* __restrict__ K, const E* __restrict__ V, CacheView c, StageView s,
                  const float* __restrict__ R, const float* __restrict__ Rnorm, int32_t* ctr, Stats* stats) {
    grid_dependency_wait();
    constexpr int EPL = D / 32;
    constexpr int ROWS = 2;
    using IO = RowIO<E, EPL>;
    __shared__ float sKey[kWarps][D];
    const int nbits = c.nbits, H = c.H;
    const int64_t T = s.T;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < s.TmaxP;
         i += (int64_t)gridDim.x * blockDim.x)
        s.sbias[i] = (i < T) ? 0.f : -INFINITY;
    // The commit of this chunk starts from zeroed counters (every commit follows the
    // staging of the chunk it commits; a refused commit is cleared by the host).
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < kCtrInts(H); i += blockDim.x) ctr[i] = 0;
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    uint32_t Rp[NBP][EPL / 2];   // hyperplane slices, bf16 pairs
#pragma unroll
    for (int b = 0; b < NBP; ++b)
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e)
            Rp[b][e] = (b < nbits) ? pack_bf16_exact(R[b * D + lane * EPL + 2 * e], R[b * D + lane * EPL + 2 * e + 1])
                                   : 0u;
    const bool mine = lane < nbits;   // lane b reports bit b
    const float gam2 = 2.f * (float)(D + 2) * kU32;
    const float rn = mine ? Rnorm[lane] : 0.f;
    const unsigned mask = (nbits >= 32) ? 0xffffffffu : ((1u << nbits) - 1u);
    const int64_t rows = T * H;
    const int64_t stride = (int64_t)gridDim.x * kWarps;
    int nq = 0;                    // rows queued for the bucket-head lookup
    int64_t q_sidx = 0, q_bucket = 0;
    float kmax = 0.f;              // largest |k|^2 this warp staged
    for (int64_t r0 = (int64_t)blockIdx.x * kWarps + wib; r0 < rows; r0 += ROWS * stride) {
        typename IO::V kv[ROWS], vv[ROWS];
#pragma unroll
        for (int q = 0; q < ROWS; ++q) {
            const int64_t r = r0 + q * stride;
            if (r < rows) {
                kv[q] = IO::load(K + r * D, lane);
                vv[q] = IO::load(V + r * D, lane);
            }
        }
#pragma unroll
        for (int q = 0; q < ROWS; ++q) {
            const int64_t r = r0 + q * stride;
            if (r >= rows) break;   // warp-uniform
            const int64_t t = (uint32_t)r / (uint32_t)H;   // rows < 2^31 (host check): 32-bit division
            const int h = (int)(r - t * H);
            const int64_t sidx = (int64_t)h * s.TmaxP + t;
            IO::store(reinterpret_cast<E*>(s.Ks) + sidx * D, lane, kv[q]);
            IO::store(reinterpret_cast<E*>(s.Vs) + sidx * D, lane, vv[q]);
            float x[EPL];
            IO::to_float(kv[q], x);
            float nk = 0.f;
            float v[NBP];
#pragma unroll
            for (int e = 0; e < EPL; ++e) nk = fmaf(x[e], x[e], nk);
#pragma unroll
            for (int b = 0; b < NBP; ++b) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < EPL / 2; ++e) {
                    a = fmaf(__uint_as_float(Rp[b][e] << 16), x[2 * e], a);
                    a = fmaf(__uint_as_float(Rp[b][e] & 0xffff0000u), x[2 * e + 1], a);
                }
                v[b] = a;
            }
            nk = warp_sum(nk);
            kmax = fmaxf(kmax, nk);
            const float p = reduce_scatter<NBP>(v, lane);
            const float err = gam2 * rn * sqrtf(nk) + 1e-30f;
            const bool need = mine && !(fabsf(p) > err);   // inside the band (or not finite)
            bool bit = p >= 0.f;
            if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                for (int e = 0; e < EPL; ++e) sKey[wib][lane * EPL + e] = x[e];
                __syncwarp();
                if (need) {   // exact: fp64, index order
                    double acc = 0.0;
                    const float* rb = R + lane * D;
                    for (int i = 0; i < D; ++i) acc = fma((double)rb[i], (double)sKey[wib][i], acc);
                    bit = (acc >= 0.0);
                }
                __syncwarp();
            }
            const unsigned code = __ballot_sync(0xffffffffu, mine && bit) & mask;
            const unsigned nre = __popc(__ballot_sync(0xffffffffu, need));
            if (lane == 0) {
                s.scode[sidx] = code;
                if (nre) atomicAdd(&stats->hash_rechecks, (unsigned long long)nre);
            }
            // The bucket-head lookups of up to 32 rows are batched, one row per lane, so
            // their latencies overlap instead of stalling the warp once per row.
            if (lane == nq) {
                q_sidx = sidx;
                q_bucket = ((int64_t)h << c.nbits) + code;
            }
            if (++nq == 32) {
                s.sfirst[q_sidx] = c.bhead[q_bucket];
                nq = 0;
            }
        }
    }
    if (lane < nq) s.sfirst[q_sidx] = c.bhead[q_bucket];
    // one bound per block: |k|^2 of the staged keys, rounded up past the fp32 sums' error
    __shared__ float sKmax[kWarps];
    if (lane == 0) sKmax[wib] = kmax * (1.f + 1.f / 1024.f);
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        for (int w = 0; w < kWarps; ++w) m = fmaxf(m, sKmax[w]);
        atomicMax(reinterpret_cast<int*>(c.kmax2s), __float_as_int(m));
    }
    grid_dependents_launch();
}

// ------------------------------------------------------------------ lane groups
//
// The search, append and merge kernels give each row to a group of 8 lanes: lane g
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

__device__ __forceinline__ float gsum(float v, unsigned gmask) {
    v += __shfl_xor_sync(gmask, v, 4);
    v += __shfl_xor_sync(gmask, v, 2);
    v += __shfl_xor_sync(gmask, v, 1);
    return v;
}
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

// ------------------------------------------------------------------ search + decide
//
// One 8-lane group per staged token (h, t). Candidates are the committed entries of
// the token's bucket: the list bhead/bnext holds exactly the entries committed
// before this commit, and its head was read when the token was staged (nothing
// changes the cache between staging and commit). The four groups of a warp walk
// their lists in lockstep, so each step has four independent row loads in flight.
// The grid is persistent (two blocks per SM).
//
// bf16 storage: every cosine is formed in fp64 exactly as the definition does
// (dot / sqrt(|k|^2 |e|^2), each sum in index order): the sums are exact by the
// span rule above (else the index-order chain), |e|^2 was stored the same way when
// the entry was appended, and the division and square root are IEEE-rounded on
// both sides. The best candidate (ties to the lowest entry index) merges when its
// cosine is >= tau.
//
// fp32 storage: fp32 cosines first; with delta a rigorous bound on |sim32 - sim|
// the fp32 result decides when best < tau - delta (no merge) or best > tau + delta
// and best - second > 2 delta (merge into the unique best). Any other case
// recomputes every candidate with the index-order chain.
//
// A matched token joins its target's merge list; unmatched tokens are counted per
// 32-token window. The last block to finish turns the window counts into the new
// cache sizes and raises the abort flag if some head would exceed its capacity.
template <typename E, int D>
__global__ void __launch_bounds__(kWarps * 32, 2)
search_kernel(CacheView c, StageView s, float tau, double tau64, float delta, bool intra, int32_t* ctr,
              Stats* stats) {
    grid_dependency_wait();
    using G = GSlice<E, D>;
    constexpr int EPG = G::EPG;
    const int lane = threadIdx.x & 31, gl = lane & 7, grp = lane >> 3;
    const unsigned gmask = 0xFFu << (8 * grp);
    const int H = c.H;
    const int64_t T = s.T;
    const int64_t rows = T * H;
    const E* Kc = reinterpret_cast<const E*>(c.Kc);
    const E* Ks = reinterpret_cast<const E*>(s.Ks);
    int32_t* ntouched = ctr;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;   // global warp
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    // The next token's key row and list head are loaded while the current token's
    // decision is published (its atomics wait for their old values).
    G xn;
    int first_n = -1;
    auto fetch = [&](int64_t r4n) {
        const int64_t rn = r4n + grp;
        if (rn < rows) {
            const int hn = (int)((uint32_t)rn / (uint32_t)T);
            const int64_t sn = (int64_t)hn * s.TmaxP + (rn - (int64_t)hn * T);
            xn.load(Ks + sn * D, gl);
            first_n = s.sfirst[sn];
        } else {
            xn.zero();
            first_n = -1;
        }
    };
    fetch(gw * 4);
    for (int64_t r4 = gw * 4; r4 < rows; r4 += nw * 4) {   // warp-uniform loop
        const int64_t r = r4 + grp;
        const bool valid = r < rows;
        const int h = valid ? (int)((uint32_t)r / (uint32_t)T) : 0;
        const int64_t t = valid ? r - (int64_t)h * T : 0;
        const int64_t sidx = (int64_t)h * s.TmaxP + t;
        const int64_t hrow = (int64_t)h * c.capP;
        const G x = xn;
        const int first = first_n;
        const int Mh = valid ? c.M[h] : 0;
        int m = -1, nslow = 0;
        double best64 = -INFINITY;   // exact best committed similarity and its entry
        int bj64 = -1;
        if constexpr (sizeof(E) == 2) {
            const int spx = gspan_bf16<D>(x, gmask);
            double n1 = gsum64(lane_dot64(x, x), gmask);
            if (2 * spx > kSpanLimit<D>) {
                n1 = gchain_dot(x, x, gl, grp, gmask);
                ++nslow;
            }
            double best = -INFINITY;
            int bestj = -1, ncand = 0;
            int j = first;
            while (__any_sync(0xffffffffu, j >= 0)) {
                const bool act = j >= 0;
                G y;
                int nxt = -1, spy = 0;
                double n2 = 0.0;
                if (act) {
                    y.load(Kc + (hrow + j) * D, gl);
                    nxt = c.bnext[hrow + j];
                    n2 = c.knorm64[hrow + j];
                    spy = c.kspan[hrow + j];   // stored at append
                } else {
                    y.zero();
                }
                double dot = gsum64(lane_dot64(x, y), gmask);
                if (act) {
                    if (spx + spy > kSpanLimit<D>) {
                        dot = gchain_dot(x, y, gl, grp, gmask);
                        ++nslow;
                    }
                    const double sim = (n1 > 0.0 && n2 > 0.0) ? dot / sqrt(n1 * n2) : 0.0;
                    if (sim > best || (sim == best && j < bestj)) {
                        best = sim;
                        bestj = j;
                    }
                    if (++ncand > Mh) {   // a bucket list can never be longer than the cache
                        if (gl == 0) atomicOr(&stats->error_bits, kErrBucketList);
                        nxt = -1;
                    }
                }
                j = nxt;
            }
            m = (bestj >= 0 && best >= tau64) ? bestj : -1;
            best64 = best;
            bj64 = bestj;
        } else {
            float nk = 0.f;
#pragma unroll
            for (int i = 0; i < EPG; ++i) nk = fmaf(x.at(i), x.at(i), nk);
            nk = gsum(nk, gmask);
            float best = -INFINITY, second = -INFINITY;
            int bestj = -1, ncand = 0;
            bool weird = false;
            int j = first;
            while (__any_sync(0xffffffffu, j >= 0)) {
                const bool act = j >= 0;
                G y;
                int nxt = -1;
                if (act) {
                    y.load(Kc + (hrow + j) * D, gl);
                    nxt = c.bnext[hrow + j];
                } else {
                    y.zero();
                }
                float dt = 0.f, ne = 0.f;
#pragma unroll
                for (int i = 0; i < EPG; ++i) {
                    dt = fmaf(x.at(i), y.at(i), dt);
                    ne = fmaf(y.at(i), y.at(i), ne);
                }
                dt = gsum(dt, gmask);
                ne = gsum(ne, gmask);
                if (act) {
                    const float den = nk * ne;
                    float sim = 0.f;
                    if (nk > 1e-30f && ne > 1e-30f && den < 1e38f && fabsf(dt) < 1e38f)
                        sim = dt / sqrtf(den);
                    else
                        weird = true;
                    if (sim > best) {
                        second = best;
                        best = sim;
                        bestj = j;
                    } else if (sim > second) {
                        second = sim;
                    }
                    if (++ncand > Mh) {
                        if (gl == 0) atomicOr(&stats->error_bits, kErrBucketList);
                        nxt = -1;
                    }
                }
                j = nxt;
            }
            bool exact = false;
            if (ncand > 0) {
                if (intra) exact = true;   // the exact best similarity is needed
                else if (!weird && best < tau - delta) m = -1;
                else if (!weird && best > tau + delta && (ncand == 1 || best - second > 2.f * delta)) m = bestj;
                else exact = true;
            }
            if (exact) {   // uniform inside the group
                nslow = 1;
                const double n1 = gchain_dot(x, x, gl, grp, gmask);
                double bsim = -INFINITY;
                int bj = -1, guard = 0;
                for (int jj = first; jj >= 0; jj = c.bnext[hrow + jj]) {
                    if (++guard > ncand) break;
                    G y;
                    y.load(Kc + (hrow + jj) * D, gl);
                    const double dot = gchain_dot(x, y, gl, grp, gmask);
                    const double n2 = c.knorm64[hrow + jj];
                    const double sim = (n1 > 0.0 && n2 > 0.0) ? dot / sqrt(n1 * n2) : 0.0;
                    if (sim > bsim || (sim == bsim && jj < bj)) {
                        bsim = sim;
                        bj = jj;
                    }
                }
                m = (bj >= 0 && bsim >= tau64) ? bj : -1;
                best64 = bsim;
                bj64 = bj;
            }
        }
        fetch(r4 + nw * 4);
        if (intra) {
            // Matching inside the chunk: keep the committed best for the dedupe kernel
            // and group the chunk's tokens by bucket.
            if (valid && gl == 0) {
                s.match[sidx] = bj64;
                s.bsim[sidx] = best64;
                if (nslow) atomicAdd(&stats->match_rechecks, (unsigned long long)nslow);
                const int old = atomicExch(&c.cbhead[((int64_t)h << c.nbits) + s.scode[sidx]], (int)t);
                s.cbnext[sidx] = old;
            }
            __syncwarp();
            continue;
        }
        if (valid && gl == 0) {
            s.match[sidx] = m;
            if (nslow) atomicAdd(&stats->match_rechecks, (unsigned long long)nslow);
            if (m >= 0) {
                const int old = atomicExch(&c.lhead[hrow + m], (int)t);
                s.lnext[sidx] = old;
                if (old < 0) s.touched[(int64_t)h * s.TmaxP + atomicAdd(&ntouched[h], 1)] = m;
            } else {
                atomicAdd(&s.wcnt[(int64_t)h * (s.TmaxP >> 5) + (t >> 5)], 1);
            }
        }
        __syncwarp();
    }
    grid_dependents_launch();
    if (!intra) publish_sizes(c, s, ctr);
}

// Exact fp64 cosine of two rows held by a lane group (the similarity of the
// definition; bf16 rows use the exact-sum rule, other rows the index-order chain).
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

// ------------------------------------------------------------------ append
//
// One warp per 32-token window of one head. Unmatched tokens of the window take
// consecutive entries in token order: dest = M_h + (unmatched tokens of earlier
// windows) + (unmatched lanes below). Each becomes an entry (key, value mean, n = 1,
// log2 n = 0, code, |k|^2 with the value of the fp64 index-order sum) and is pushed
// on its bucket's list; lane groups copy two rows each per pass.
template <typename E, int D>
__global__ void __launch_bounds__(kWarps * 32, 3) append_kernel(CacheView c, StageView s, const int32_t* ctr) {
    grid_dependency_wait();
    grid_dependents_launch();   // the merge only needs this kernel's completion
    using G = GSlice<E, D>;
    constexpr int EPG = G::EPG;
    __shared__ int sSrc[kWarps][32];
    const int H = c.H;
    if (ctr[2 * H]) return;  // commit aborted: nothing changes
    const int lane = threadIdx.x & 31, gl = lane & 7, grp = lane >> 3, wib = threadIdx.x >> 5;
    const unsigned gmask = 0xFFu << (8 * grp);
    const int64_t T = s.T;
    const int nwin = (int)((T + 31) >> 5);
    const E* Ks = reinterpret_cast<const E*>(s.Ks);
    const E* Vs = reinterpret_cast<const E*>(s.Vs);
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t wg = gw; wg < (int64_t)H * nwin; wg += nw) {
        const int h = (int)(wg / nwin);
        const int w = (int)(wg - (int64_t)h * nwin);
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
            if (m >= -1) s.dest[sidx] = un ? base + rank : m;
            s.lcode[sidx] = s.scode[sidx];
        }
        if (un) sSrc[wib][rank] = lane;
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
                st[u] = k < nun ? wrow + sSrc[wib][k] : -1;
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
                            s.match[sbase + tm] = base + k;
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
}

// ------------------------------------------------------------------ merge
//
// One lane group per entry touched by merges. The matched tokens' values are
// summed in fp32 in ascending token order (whatever order the atomics built the
// list in), then v <- (n v + sum) / (n + m), n <- n + m (Lemma 5.1: the merged
// entry carries the mean of its group and the group size). Lists of up to 8 tokens
// are ordered inside the group; longer ones go to the whole warp, which orders up
// to kListSmem tokens in shared memory and otherwise gathers them by scanning the
// head's match targets in token order. The kernel also leaves the per-commit state
// ready for the next commit (lists emptied, window counts zeroed, sizes published).
constexpr int kListSmem = 256;

template <typename E, int D>
__device__ void merge_long_list(const CacheView& c, const StageView& s, int h, int j, int32_t* sIds,
                                int32_t* sSorted, int lane) {
    constexpr int EPL = D / 32;
    using IO = RowIO<E, EPL>;
    const int64_t T = s.T;
    const int64_t sbase = (int64_t)h * s.TmaxP;
    const int64_t e = (int64_t)h * c.capP + j;
    const E* Vs = reinterpret_cast<const E*>(s.Vs);
    int L = 0, id = 0x7fffffff;
    for (int tt = c.lhead[e]; tt >= 0; tt = s.lnext[sbase + tt]) {
        if (L < 32 && lane == L) id = tt;
        if (L < kListSmem && lane == 0) sIds[L] = tt;
        ++L;
        if (L > (int)T) break;   // a list is never longer than the chunk
    }
    __syncwarp();
    float acc[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) acc[q] = 0.f;
    auto add_row = [&](int tt) {
        float v[EPL];
        IO::to_float(IO::load(Vs + (sbase + tt) * D, lane), v);
#pragma unroll
        for (int q = 0; q < EPL; ++q) acc[q] = __fadd_rn(acc[q], v[q]);
    };
    if (L <= 32) {
        int rank = 0;
        for (int k = 0; k < L; ++k) rank += (__shfl_sync(0xffffffffu, id, k) < id);
        for (int q2 = 0; q2 < L; ++q2) {
            const int src = __ffs(__ballot_sync(0xffffffffu, rank == q2 && lane < L)) - 1;
            add_row(__shfl_sync(0xffffffffu, id, src));
        }
    } else if (L <= kListSmem) {
        for (int a = lane; a < L; a += 32) {
            const int mine = sIds[a];
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
    __syncwarp();
    if (lane == 0) {
        c.cnt[e] = ntot;
        c.bias2[e] = log2f(ft);
        c.lhead[e] = -1;
        atomicMax(reinterpret_cast<int*>(&c.bmax[h]), __float_as_int(log2f(ft)));   // log2 n >= 0
    }
    __syncwarp();
}

template <typename E, int D>
__global__ void __launch_bounds__(kWarps * 32, 3) merge_kernel(CacheView c, StageView s, int32_t* ctr) {
    grid_dependency_wait();
    using G = GSlice<E, D>;
    constexpr int EPG = G::EPG;
    __shared__ int32_t sIds[kWarps][kListSmem];
    __shared__ int32_t sSorted[kWarps][kListSmem];
    const int H = c.H;
    const bool aborted = ctr[2 * H] != 0;
    const int lane = threadIdx.x & 31, gl = lane & 7, grp = lane >> 3, wib = threadIdx.x >> 5;
    const unsigned gmask = 0xFFu << (8 * grp);
    const int64_t T = s.T;
    const E* Vs = reinterpret_cast<const E*>(s.Vs);
    if (aborted)   // a refused commit leaves no member chains behind (matching inside the chunk)
        for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < (int64_t)H * T;
             q += (int64_t)gridDim.x * blockDim.x)
            s.ichead[(q / T) * s.TmaxP + (q % T)] = -1;
    if (!aborted && blockIdx.x == 0)
        for (int hh = threadIdx.x; hh < H; hh += blockDim.x) c.M[hh] = ctr[H + hh];
    const int nwin = (int)((T + 31) >> 5);
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < (int64_t)H * nwin;
         q += (int64_t)gridDim.x * blockDim.x)
        s.wcnt[(q / nwin) * (s.TmaxP >> 5) + (q % nwin)] = 0;
    const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t q4 = gw * 4; q4 < (int64_t)H * T; q4 += nw * 4) {   // warp-uniform
        const int64_t q = q4 + grp;
        int h = 0, j = -1;
        bool act = false, big = false;
        if (q < (int64_t)H * T) {
            h = (int)((uint32_t)q / (uint32_t)T);
            const int slot = (int)(q - (int64_t)h * T);
            act = slot < ctr[h];
            if (act) j = s.touched[(int64_t)h * s.TmaxP + slot];
        }
        if (act) {   // group-uniform
            const int64_t sbase = (int64_t)h * s.TmaxP;
            const int64_t e = (int64_t)h * c.capP + j;
            if (!aborted) {
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
                        atomicMax(reinterpret_cast<int*>(&c.bmax[h]), __float_as_int(log2f(ft)));   // log2 n >= 0
                    }
                }
            }
            __syncwarp(gmask);
            if (!big && gl == 0) c.lhead[e] = -1;
        }
        // lists longer than 8 tokens: the whole warp, one list at a time
        unsigned bigm = __ballot_sync(0xffffffffu, big && gl == 0);
        while (bigm) {
            const int src = __ffs(bigm) - 1;
            bigm &= bigm - 1;
            const int bh = __shfl_sync(0xffffffffu, h, src);
            const int bj = __shfl_sync(0xffffffffu, j, src);
            merge_long_list<E, D>(c, s, bh, bj, sIds[wib], sSorted[wib], lane);
        }
    }
    grid_dependents_launch();
}

template <typename E, int D, int NBP>
cudaError_t stage_hash_n(const CacheView& c, const StageView& s, const void* K, const void* V, const float* R,
                         const float* Rnorm, int32_t* ctr, Stats* stats, cudaStream_t st) {
    const int64_t rows = s.T * c.H;
    const int grid = grid_for_rows(rows > s.TmaxP ? rows : s.TmaxP, 4 * kWarps, 148 * 8);
    return launch_pdl(stage_hash_kernel<E, D, NBP>, grid, kWarps * 32, st, reinterpret_cast<const E*>(K),
                      reinterpret_cast<const E*>(V), c, s, R, Rnorm, ctr, stats);
}

template <typename E, int D>
cudaError_t stage_hash_t(const CacheView& c, const StageView& s, const void* K, const void* V,
                         const float* R, const float* Rnorm, int32_t* ctr, Stats* stats, cudaStream_t st) {
    if (c.nbits <= 8) return stage_hash_n<E, D, 8>(c, s, K, V, R, Rnorm, ctr, stats, st);
    if (c.nbits <= 16) return stage_hash_n<E, D, 16>(c, s, K, V, R, Rnorm, ctr, stats, st);
    return stage_hash_n<E, D, 32>(c, s, K, V, R, Rnorm, ctr, stats, st);
}

// The counters start at zero: the staging kernel of the chunk cleared them.
template <typename E, int D>
cudaError_t commit_t(const CacheView& c, const StageView& s, float tau, bool intra, int32_t* ctr, Stats* stats,
                     int* launches, cudaStream_t st) {
    const int H = c.H;
    const int64_t rows = s.T * H;
    // delta bounds |sim32 - sim| (see the search kernel): 2 x (2 (d+2) u + 3 u).
    const float delta = 2.f * (2.f * (float)(D + 2) * kU32 + 3.f * kU32);
    const int sgrid = grid_for_rows(rows, 4 * kWarps, 148 * 2);
    cudaError_t e = launch_pdl(search_kernel<E, D>, sgrid, kWarps * 32, st, c, s, tau, (double)tau, delta, intra,
                               ctr, stats);
    if (e == cudaSuccess && intra) {
        e = launch_pdl(dedupe_kernel<E, D>, sgrid, kWarps * 32, st, c, s, (double)tau, ctr, stats);
        *launches += 1;
    }
    const int64_t wins = (int64_t)H * ((s.T + 31) / 32);
    if (e == cudaSuccess)
        e = launch_pdl(append_kernel<E, D>, grid_for_rows(wins, kWarps, 148 * 16), kWarps * 32, st, c, s,
                       (const int32_t*)ctr);
    if (e == cudaSuccess)
        e = launch_pdl(merge_kernel<E, D>, grid_for_rows(rows, kWarps, 148 * 8), kWarps * 32, st, c, s, ctr);
    *launches += 3;
    return e;
}

}  // namespace

cudaError_t launch_stage_hash(const CacheView& c, const StageView& s, int dtype, const void* K,
                              const void* V, const float* R, const float* Rnorm, int32_t* ctr, Stats* stats,
                              cudaStream_t st) {
    if (dtype == 0) {
        return c.d == 128 ? stage_hash_t<__nv_bfloat16, 128>(c, s, K, V, R, Rnorm, ctr, stats, st)
                          : stage_hash_t<__nv_bfloat16, 64>(c, s, K, V, R, Rnorm, ctr, stats, st);
    }
    return c.d == 128 ? stage_hash_t<float, 128>(c, s, K, V, R, Rnorm, ctr, stats, st)
                      : stage_hash_t<float, 64>(c, s, K, V, R, Rnorm, ctr, stats, st);
}

cudaError_t launch_commit(const CacheView& c, const StageView& s, int dtype, float tau, bool intra, int32_t* ctr,
                          Stats* stats, int* launches, cudaStream_t st) {
    if (dtype == 0) {
        return c.d == 128 ? commit_t<__nv_bfloat16, 128>(c, s, tau, intra, ctr, stats, launches, st)
                          : commit_t<__nv_bfloat16, 64>(c, s, tau, intra, ctr, stats, launches, st);
    }
    return c.d == 128 ? commit_t<float, 128>(c, s, tau, intra, ctr, stats, launches, st)
                      : commit_t<float, 64>(c, s, tau, intra, ctr, stats, launches, st);
}

}  // namespace tc
