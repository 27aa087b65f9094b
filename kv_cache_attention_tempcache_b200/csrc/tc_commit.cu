// TempCache commit path: stage + hash, bucketed top-1 search with the merge
// decision, compaction scan, append, and the deterministic segmented merge.
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

#include <math.h>

namespace tc {

namespace {

constexpr float kU32 = 5.9604644775390625e-8f;  // 2^-24, fp32 unit roundoff

template <typename T, int EPL>
struct RowIO;

template <>
struct RowIO<__nv_bfloat16, 4> {
    using V = uint2;
    __device__ static V load(const __nv_bfloat16* row, int lane) {
        return reinterpret_cast<const V*>(row)[lane];
    }
    __device__ static void store(__nv_bfloat16* row, int lane, V v) {
        reinterpret_cast<V*>(row)[lane] = v;
    }
    __device__ static void to_float(V v, float (&x)[4]) {
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&v.x);
        __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&v.y);
        x[0] = __low2float(a); x[1] = __high2float(a);
        x[2] = __low2float(b); x[3] = __high2float(b);
    }
    __device__ static V from_float(const float (&x)[4]) {
        __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
        V v;
        v.x = *reinterpret_cast<uint32_t*>(&a);
        v.y = *reinterpret_cast<uint32_t*>(&b);
        return v;
    }
};

template <>
struct RowIO<__nv_bfloat16, 2> {
    using V = uint32_t;
    __device__ static V load(const __nv_bfloat16* row, int lane) {
        return reinterpret_cast<const V*>(row)[lane];
    }
    __device__ static void store(__nv_bfloat16* row, int lane, V v) {
        reinterpret_cast<V*>(row)[lane] = v;
    }
    __device__ static void to_float(V v, float (&x)[2]) {
        __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&v);
        x[0] = __low2float(a); x[1] = __high2float(a);
    }
    __device__ static V from_float(const float (&x)[2]) {
        __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
        return *reinterpret_cast<uint32_t*>(&a);
    }
};

template <>
struct RowIO<float, 4> {
    using V = float4;
    __device__ static V load(const float* row, int lane) { return reinterpret_cast<const V*>(row)[lane]; }
    __device__ static void store(float* row, int lane, V v) { reinterpret_cast<V*>(row)[lane] = v; }
    __device__ static void to_float(V v, float (&x)[4]) { x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w; }
    __device__ static V from_float(const float (&x)[4]) { return make_float4(x[0], x[1], x[2], x[3]); }
};

template <>
struct RowIO<float, 2> {
    using V = float2;
    __device__ static V load(const float* row, int lane) { return reinterpret_cast<const V*>(row)[lane]; }
    __device__ static void store(float* row, int lane, V v) { reinterpret_cast<V*>(row)[lane] = v; }
    __device__ static void to_float(V v, float (&x)[2]) { x[0] = v.x; x[1] = v.y; }
    __device__ static V from_float(const float (&x)[2]) { return make_float2(x[0], x[1]); }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ int warp_min(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

constexpr int kWarps = 8;  // warps per block of the warp-per-row kernels

inline int grid_for_rows(int64_t rows, int per_block, int max_blocks) {
    int64_t b = (rows + per_block - 1) / per_block;
    if (b < 1) b = 1;
    if (b > max_blocks) b = max_blocks;
    return (int)b;
}

// ------------------------------------------------------------------ stage + hash
//
// One warp per input row r = t*H + h of the token-major chunk. The row is copied
// to the head-major staging buffer; lane b < nbits then forms <R_b, k> in fp32,
// keeps its sign when |<R_b,k>| exceeds the certified bound
//   2 (d+2) u |R_b| |k|   (u = 2^-24; any summation order has error <= (d+2) u
//                         sum|R_bi k_i| <= (d+2) u |R_b||k|, doubled for margin)
// and otherwise redoes the sum in fp64 in index order. Bit b = [<R_b,k> >= 0].
template <typename E, int D>
__global__ void __launch_bounds__(kWarps * 32)
stage_hash_kernel(const E* __restrict__ K, const E* __restrict__ V, CacheView c, StageView s,
                  const float* __restrict__ R, const float* __restrict__ Rnorm, Stats* stats) {
    constexpr int EPL = D / 32;
    using IO = RowIO<E, EPL>;
    extern __shared__ float sm[];
    const int nbits = c.nbits, H = c.H;
    const int64_t T = s.T;
    float* sR = sm;                        // [nbits][D+1], padded: conflict-free column reads
    float* sKey = sm + nbits * (D + 1);    // [kWarps][D]
    for (int i = threadIdx.x; i < nbits * D; i += blockDim.x) sR[(i / D) * (D + 1) + (i % D)] = R[i];
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < s.TmaxP;
         i += (int64_t)gridDim.x * blockDim.x)
        s.sbias[i] = (i < T) ? 0.f : -INFINITY;
    __syncthreads();

    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    float* krow = sKey + wib * D;
    const float gam2 = 2.f * (float)(D + 2) * kU32;
    const float rn = (lane < nbits) ? Rnorm[lane] : 0.f;
    const unsigned mask = (nbits >= 32) ? 0xffffffffu : ((1u << nbits) - 1u);
    const int64_t rows = T * H;
    for (int64_t r = (int64_t)blockIdx.x * kWarps + wib; r < rows; r += (int64_t)gridDim.x * kWarps) {
        const int64_t t = r / H;
        const int h = (int)(r - t * H);
        const int64_t srow = ((int64_t)h * s.TmaxP + t) * D;
        auto kv = IO::load(K + r * D, lane);
        auto vv = IO::load(V + r * D, lane);
        IO::store(reinterpret_cast<E*>(s.Ks) + srow, lane, kv);
        IO::store(reinterpret_cast<E*>(s.Vs) + srow, lane, vv);
        float x[EPL];
        IO::to_float(kv, x);
        float nk = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            nk = fmaf(x[e], x[e], nk);
            krow[lane * EPL + e] = x[e];
        }
        nk = warp_sum(nk);
        __syncwarp();
        bool bit = false, rechk = false;
        if (lane < nbits) {
            const float* rb = sR + lane * (D + 1);
            float p = 0.f;
#pragma unroll 16
            for (int i = 0; i < D; ++i) p = fmaf(rb[i], krow[i], p);
            const float err = gam2 * rn * sqrtf(nk) + 1e-30f;
            if (!(fabsf(p) > err)) {  // inside the band (or not finite): exact fp64, index order
                rechk = true;
                double q = 0.0;
                for (int i = 0; i < D; ++i) q = fma((double)rb[i], (double)krow[i], q);
                bit = (q >= 0.0);
            } else {
                bit = (p >= 0.f);
            }
        }
        const unsigned code = __ballot_sync(0xffffffffu, bit) & mask;
        const unsigned nre = __popc(__ballot_sync(0xffffffffu, rechk));
        if (lane == 0) {
            s.scode[(int64_t)h * s.TmaxP + t] = code;
            if (nre) atomicAdd(&stats->hash_rechecks, (unsigned long long)nre);
        }
        __syncwarp();
    }
}

// ------------------------------------------------------------------ search + decide
//
// One warp per staged token (h, t). Candidates are the committed entries of the
// token's bucket (the linked list bhead/bnext holds exactly the entries committed
// before this commit). fp32 cosine per candidate; with delta a rigorous bound on
// |sim32 - sim|, the fp32 result decides when
//   best < tau - delta                         (no merge), or
//   best > tau + delta and best - second > 2 delta   (merge into the unique best).
// Any other case recomputes every candidate's cosine exactly as the definition
// does (fp64, index order) and takes the maximum, lowest entry index on ties.
template <typename E, int D>
__global__ void __launch_bounds__(kWarps * 32)
search_kernel(CacheView c, StageView s, float tau, double tau64, float delta, int32_t* ntouched,
              Stats* stats) {
    constexpr int EPL = D / 32;
    using IO = RowIO<E, EPL>;
    __shared__ float sTok[kWarps][D];
    __shared__ float sCand[kWarps][D];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t T = s.T;
    const int64_t rows = T * c.H;
    const E* Kc = reinterpret_cast<const E*>(c.Kc);
    const E* Ks = reinterpret_cast<const E*>(s.Ks);
    for (int64_t r = (int64_t)blockIdx.x * kWarps + wib; r < rows; r += (int64_t)gridDim.x * kWarps) {
        const int h = (int)(r / T);
        const int64_t t = r - (int64_t)h * T;
        const int64_t sidx = (int64_t)h * s.TmaxP + t;
        float x[EPL];
        IO::to_float(IO::load(Ks + sidx * D, lane), x);
        float nk = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) nk = fmaf(x[e], x[e], nk);
        nk = warp_sum(nk);
        const uint32_t code = s.scode[sidx];
        const int64_t hrow = (int64_t)h * c.capP;
        const int first = c.bhead[((int64_t)h << c.nbits) + code];
        float best = -INFINITY, second = -INFINITY;
        int bestj = -1, ncand = 0;
        bool weird = false;
        for (int j = first; j >= 0; j = c.bnext[hrow + j]) {
            if (ncand > c.M[h]) {  // a bucket list can never be longer than the cache
                if (lane == 0) atomicOr(&stats->error_bits, kErrBucketList);
                break;
            }
            float y[EPL];
            IO::to_float(IO::load(Kc + (hrow + j) * D, lane), y);
            float dt = 0.f, ne = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                dt = fmaf(x[e], y[e], dt);
                ne = fmaf(y[e], y[e], ne);
            }
            dt = warp_sum(dt);
            ne = warp_sum(ne);
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
            ++ncand;
        }
        int m = -1;
        bool exact = false;
        if (ncand > 0) {
            if (!weird && best < tau - delta) m = -1;
            else if (!weird && best > tau + delta && (ncand == 1 || best - second > 2.f * delta)) m = bestj;
            else exact = true;
        }
        if (exact) {
#pragma unroll
            for (int e = 0; e < EPL; ++e) sTok[wib][lane * EPL + e] = x[e];
            double bsim = -INFINITY;
            int bj = -1, guard = 0;
            for (int j = first; j >= 0; j = c.bnext[hrow + j]) {
                if (++guard > ncand) break;
                float y[EPL];
                IO::to_float(IO::load(Kc + (hrow + j) * D, lane), y);
                __syncwarp();
#pragma unroll
                for (int e = 0; e < EPL; ++e) sCand[wib][lane * EPL + e] = y[e];
                __syncwarp();
                double acc = 0.0;
                if (lane < 3) {
                    const float* a = (lane == 2) ? sCand[wib] : sTok[wib];
                    const float* b = (lane == 1) ? sTok[wib] : sCand[wib];
                    for (int i = 0; i < D; ++i) acc = fma((double)a[i], (double)b[i], acc);
                }
                const double dot = __shfl_sync(0xffffffffu, acc, 0);
                const double n1 = __shfl_sync(0xffffffffu, acc, 1);
                const double n2 = __shfl_sync(0xffffffffu, acc, 2);
                const double sim = (n1 > 0.0 && n2 > 0.0) ? dot / sqrt(n1 * n2) : 0.0;
                if (sim > bsim || (sim == bsim && j < bj)) {
                    bsim = sim;
                    bj = j;
                }
            }
            m = (bj >= 0 && bsim >= tau64) ? bj : -1;
        }
        if (lane == 0) {
            s.match[sidx] = m;
            if (exact) atomicAdd(&stats->match_rechecks, 1ull);
            if (m >= 0) {
                const int old = atomicAdd(&c.mcount[hrow + m], 1);
                if (old == 0) {
                    const int slot = atomicAdd(&ntouched[h], 1);
                    s.touched[(int64_t)h * s.TmaxP + slot] = m;
                }
            }
        }
        __syncwarp();
    }
}

// ------------------------------------------------------------------ scan
//
// One block per head. (a) dest[t] = M_h + (number of unmatched tokens before t)
// for unmatched tokens, match[t] otherwise; the new size is M_h + (unmatched
// count), and any head past capacity raises the abort flag for the whole commit.
// (b) Merge segments: the entries touched by merges get consecutive ranges of
// seg[] sized by their merge counts.
__device__ int block_exclusive_scan(int v, int* total) {
    __shared__ int wsum[32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) wsum[w] = inc;
    __syncthreads();
    if (w == 0) {
        int x = (lane < nw) ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += n;
        }
        wsum[lane] = x;  // inclusive prefix over warps
    }
    __syncthreads();
    const int before = (w > 0) ? wsum[w - 1] : 0;
    *total = wsum[nw - 1];
    __syncthreads();
    return before + inc - v;
}

__global__ void __launch_bounds__(1024) scan_kernel(CacheView c, StageView s, int32_t* ctr) {
    const int h = blockIdx.x, H = c.H;
    int32_t* ntouched = ctr;
    int32_t* newM = ctr + H;
    int32_t* abort_flag = ctr + 2 * H;
    const int64_t T = s.T;
    const int64_t base = (int64_t)h * s.TmaxP;
    const int nt = blockDim.x;
    const int64_t per = (T + nt - 1) / nt;
    const int64_t t0 = min(T, (int64_t)threadIdx.x * per), t1 = min(T, t0 + per);
    int u = 0;
    for (int64_t t = t0; t < t1; ++t) u += (s.match[base + t] < 0);
    int total = 0;
    const int ex = block_exclusive_scan(u, &total);
    const int Mh = c.M[h];
    int pos = Mh + ex;
    for (int64_t t = t0; t < t1; ++t) {
        const int m = s.match[base + t];
        s.dest[base + t] = (m < 0) ? pos++ : m;
        s.lcode[base + t] = s.scode[base + t];
    }
    if (threadIdx.x == 0) {
        newM[h] = Mh + total;
        if ((int64_t)Mh + total > c.capacity) atomicExch(abort_flag, 1);
    }
    const int ns = ntouched[h];
    const int per2 = (ns + nt - 1) / nt;
    const int s0 = min(ns, (int)threadIdx.x * per2), s1 = min(ns, s0 + per2);
    const int64_t hrow = (int64_t)h * c.capP;
    int cs = 0;
    for (int q = s0; q < s1; ++q) cs += c.mcount[hrow + s.touched[base + q]];
    int tot2 = 0;
    int off = block_exclusive_scan(cs, &tot2);
    for (int q = s0; q < s1; ++q) {
        const int j = s.touched[base + q];
        c.moff[hrow + j] = off;
        off += c.mcount[hrow + j];
    }
}

// ------------------------------------------------------------------ append
//
// One warp per staged token. Unmatched tokens become entries at dest (key, value
// mean, n = 1, log2 n = 0, code) and are pushed on their bucket's list; matched
// tokens claim a slot in their target's merge segment.
template <typename E, int D>
__global__ void __launch_bounds__(kWarps * 32) append_kernel(CacheView c, StageView s, const int32_t* ctr) {
    constexpr int EPL = D / 32;
    using IO = RowIO<E, EPL>;
    const int H = c.H;
    if (ctr[2 * H]) return;  // commit aborted: nothing changes
    if (blockIdx.x == 0)
        for (int hh = threadIdx.x; hh < H; hh += blockDim.x) c.M[hh] = ctr[H + hh];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t T = s.T;
    const int64_t rows = T * H;
    for (int64_t r = (int64_t)blockIdx.x * kWarps + wib; r < rows; r += (int64_t)gridDim.x * kWarps) {
        const int h = (int)(r / T);
        const int64_t t = r - (int64_t)h * T;
        const int64_t sidx = (int64_t)h * s.TmaxP + t;
        const int64_t hrow = (int64_t)h * c.capP;
        const int m = s.match[sidx];
        if (m < 0) {
            const int j = s.dest[sidx];
            const int64_t e = hrow + j;
            const auto kv = IO::load(reinterpret_cast<const E*>(s.Ks) + sidx * D, lane);
            const auto vv = IO::load(reinterpret_cast<const E*>(s.Vs) + sidx * D, lane);
            IO::store(reinterpret_cast<E*>(c.Kc) + e * D, lane, kv);
            IO::store(reinterpret_cast<E*>(c.Vc) + e * D, lane, vv);
            float v[EPL];
            IO::to_float(vv, v);
#pragma unroll
            for (int q = 0; q < EPL; ++q) c.V32[e * D + lane * EPL + q] = v[q];
            if (lane == 0) {
                const uint32_t code = s.scode[sidx];
                c.cnt[e] = 1;
                c.bias2[e] = 0.f;
                c.code[e] = code;
                c.bnext[e] = atomicExch(&c.bhead[((int64_t)h << c.nbits) + code], j);
            }
        } else if (lane == 0) {
            const int pos = c.moff[hrow + m] + atomicAdd(&c.mfill[hrow + m], 1);
            s.seg[(int64_t)h * s.TmaxP + pos] = (int)t;
        }
    }
}

// ------------------------------------------------------------------ merge
//
// One warp per entry touched by merges. The matched tokens' values are summed in
// fp32 in ascending token order (deterministic whatever order the atomics filled
// the segment in), then v <- (n v + sum) / (n + m), n <- n + m (Lemma 5.1: the
// merged entry carries the mean of its group and the group size).
template <typename E, int D>
__global__ void __launch_bounds__(kWarps * 32) merge_kernel(CacheView c, StageView s, int32_t* ctr) {
    constexpr int EPL = D / 32;
    using IO = RowIO<E, EPL>;
    const int H = c.H;
    const bool aborted = ctr[2 * H] != 0;
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t T = s.T;
    const int64_t rows = T * H;
    const E* Vs = reinterpret_cast<const E*>(s.Vs);
    for (int64_t r = (int64_t)blockIdx.x * kWarps + wib; r < rows; r += (int64_t)gridDim.x * kWarps) {
        const int h = (int)(r / T);
        const int slot = (int)(r - (int64_t)h * T);
        if (slot >= ctr[h]) continue;
        const int64_t sbase = (int64_t)h * s.TmaxP;
        const int64_t hrow = (int64_t)h * c.capP;
        const int j = s.touched[sbase + slot];
        const int64_t e = hrow + j;
        const int cntj = c.mcount[e];
        if (!aborted) {
            const int off = c.moff[e];
            float acc[EPL];
#pragma unroll
            for (int q = 0; q < EPL; ++q) acc[q] = 0.f;
            if (cntj <= 32) {
                const int id = (lane < cntj) ? s.seg[sbase + off + lane] : 0x7fffffff;
                int rank = 0;
                for (int k = 0; k < 32; ++k) rank += (__shfl_sync(0xffffffffu, id, k) < id);
                for (int q = 0; q < cntj; ++q) {
                    const int src = __ffs(__ballot_sync(0xffffffffu, rank == q)) - 1;
                    const int tt = __shfl_sync(0xffffffffu, id, src);
                    float v[EPL];
                    IO::to_float(IO::load(Vs + (sbase + tt) * D, lane), v);
#pragma unroll
                    for (int qq = 0; qq < EPL; ++qq) acc[qq] = __fadd_rn(acc[qq], v[qq]);
                }
            } else {
                int last = -1;
                for (int q = 0; q < cntj; ++q) {
                    int mn = 0x7fffffff;
                    for (int p = lane; p < cntj; p += 32) {
                        const int id = s.seg[sbase + off + p];
                        if (id > last && id < mn) mn = id;
                    }
                    mn = warp_min(mn);
                    float v[EPL];
                    IO::to_float(IO::load(Vs + (sbase + mn) * D, lane), v);
#pragma unroll
                    for (int qq = 0; qq < EPL; ++qq) acc[qq] = __fadd_rn(acc[qq], v[qq]);
                    last = mn;
                }
            }
            const int nold = c.cnt[e];
            const int ntot = nold + cntj;
            const float fn = (float)nold, ft = (float)ntot;
            float nv[EPL];
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
                const float old = c.V32[e * D + lane * EPL + q];
                nv[q] = __fdiv_rn(__fadd_rn(__fmul_rn(fn, old), acc[q]), ft);
                c.V32[e * D + lane * EPL + q] = nv[q];
            }
            IO::store(reinterpret_cast<E*>(c.Vc) + e * D, lane, IO::from_float(nv));
            if (lane == 0) {
                c.cnt[e] = ntot;
                c.bias2[e] = log2f(ft);
            }
        }
        if (lane == 0) {
            c.mcount[e] = 0;
            c.mfill[e] = 0;
        }
    }
}

template <typename E, int D>
cudaError_t stage_hash_t(const CacheView& c, const StageView& s, const void* K, const void* V,
                         const float* R, const float* Rnorm, Stats* stats, cudaStream_t st) {
    const int64_t rows = s.T * c.H;
    const int grid = grid_for_rows(rows > s.TmaxP ? rows : s.TmaxP, kWarps, 148 * 16);
    const size_t smem = sizeof(float) * ((size_t)c.nbits * (D + 1) + kWarps * D);
    stage_hash_kernel<E, D><<<grid, kWarps * 32, smem, st>>>(
        reinterpret_cast<const E*>(K), reinterpret_cast<const E*>(V), c, s, R, Rnorm, stats);
    return cudaGetLastError();
}

template <typename E, int D>
cudaError_t commit_t(const CacheView& c, const StageView& s, float tau, int32_t* ctr, Stats* stats,
                     int* launches, cudaStream_t st) {
    const int H = c.H;
    cudaError_t e = cudaMemsetAsync(ctr, 0, sizeof(int32_t) * kCtrInts(H), st);
    if (e != cudaSuccess) return e;
    const int64_t rows = s.T * H;
    const int grid = grid_for_rows(rows, kWarps, 148 * 16);
    // delta bounds |sim32 - sim| (see the kernel comment): 2 x (2 (d+2) u + 3 u).
    const float delta = 2.f * (2.f * (float)(D + 2) * kU32 + 3.f * kU32);
    search_kernel<E, D><<<grid, kWarps * 32, 0, st>>>(c, s, tau, (double)tau, delta, ctr, stats);
    scan_kernel<<<H, 1024, 0, st>>>(c, s, ctr);
    append_kernel<E, D><<<grid, kWarps * 32, 0, st>>>(c, s, ctr);
    merge_kernel<E, D><<<grid, kWarps * 32, 0, st>>>(c, s, ctr);
    *launches += 4;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stage_hash(const CacheView& c, const StageView& s, int dtype, const void* K,
                              const void* V, const float* R, const float* Rnorm, Stats* stats,
                              cudaStream_t st) {
    if (dtype == 0) {
        return c.d == 128 ? stage_hash_t<__nv_bfloat16, 128>(c, s, K, V, R, Rnorm, stats, st)
                          : stage_hash_t<__nv_bfloat16, 64>(c, s, K, V, R, Rnorm, stats, st);
    }
    return c.d == 128 ? stage_hash_t<float, 128>(c, s, K, V, R, Rnorm, stats, st)
                      : stage_hash_t<float, 64>(c, s, K, V, R, Rnorm, stats, st);
}

cudaError_t launch_commit(const CacheView& c, const StageView& s, int dtype, float tau, int32_t* ctr,
                          Stats* stats, int* launches, cudaStream_t st) {
    if (dtype == 0) {
        return c.d == 128 ? commit_t<__nv_bfloat16, 128>(c, s, tau, ctr, stats, launches, st)
                          : commit_t<__nv_bfloat16, 64>(c, s, tau, ctr, stats, launches, st);
    }
    return c.d == 128 ? commit_t<float, 128>(c, s, tau, ctr, stats, launches, st)
                      : commit_t<float, 64>(c, s, tau, ctr, stats, launches, st);
}

}  // namespace tc
