// AnnCA cross-attention: keep, per frame and head, the prompt tokens whose hash
// bucket holds at least one of the frame's queries, then attend over those only.
//
// FAST-AR technical summary, section 2.B "AnnCA": latent queries and prompt keys are
// projected into one hashed space, prompt tokens without a bucket shared with the
// current frame's queries are pruned for that frame, and cross-attention skips them.
//
// Kernels:
//   annca_prompt_kernel   once per prompt: copy Kp, Vp head-major, hash every key,
//                         bound |k|^2 per head.
//   annca_sort_kernel     once per prompt: sort each head's (code, token) pairs; every
//                         prompt token learns where its code's run starts.
//   annca_mark_kernel     per call: two lanes per query row hash it, then look its code
//                         up (a table of the head's codes for nbits <= 16, else a binary
//                         search of its sorted codes) and, if the prompt has that code,
//                         stamp the bucket with the call's number for the query's frame
//                         (written only while the stamp differs, so the many queries of
//                         one bucket rarely store).
//   annca_pack_kernel     per call: a few blocks per (head, frame) list the prompt tokens
//                         whose bucket carries this call's stamp, in ascending order, and
//                         pack their keys and values into 128-row tiles for the attention
//                         kernel (zero rows and a -inf logit shift past the last kept
//                         token). Stamps are never cleared: the next call has a new number.
//   attention             the tcgen05 flash-attention kernel of tc_attn_bf16.cu in its
//                         cross mode: the keys of a CTA are the packed tokens of its slot.
// Hash bits are exact as in the TempCache staging kernel: the fp32 sign is kept only
// outside its rounding bound, else the bit is recomputed as an fp64 sum in index order.
#include "../../include/tempcache.h"
#include "tc_internal.h"
#include "tc_device.cuh"

#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

namespace tc {

namespace {

constexpr int kMaxPrompt = 4096;   // prompt tokens (the sort runs in one block's shared memory)

// Code of the bf16 row x held by the warp (lane l: elements [l EPL, l EPL + EPL)),
// with the normals' bf16 pairs in Rp and |R_b| (rounded up) in rn on lane b. Returns
// the code on every lane; nk receives the fp32 |x|^2 and nre the re-checked bits.
template <int D, int NBP>
__device__ __forceinline__ unsigned hash_row(const float (&x)[D / 32], const uint32_t (&Rp)[NBP][D / 64],
                                             const float* __restrict__ R, float rn, int nbits, float* sRow,
                                             int lane, float& nk, unsigned& nre) {
    constexpr int EPL = D / 32;
    float n2 = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) n2 = fmaf(x[e], x[e], n2);
    float v[NBP];
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
    n2 = warp_sum(n2);
    const float p = reduce_scatter<NBP>(v, lane);
    const bool mine = lane < nbits;
    // |<R_b,x>| > 2 (d+2) u |R_b||x| certifies the fp32 sign (any summation order errs
    // by at most (d+2) u |R_b||x|; doubled for margin)
    const float err = 2.f * (float)(D + 2) * kU32 * rn * sqrtf(n2) + 1e-30f;
    const bool need = mine && !(fabsf(p) > err);
    bool bit = p >= 0.f;
    if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) sRow[lane * EPL + e] = x[e];
        __syncwarp();
        if (need) {
            double acc = 0.0;
            const float* rb = R + lane * D;
            for (int i = 0; i < D; ++i) acc = fma((double)rb[i], (double)sRow[i], acc);
            bit = acc >= 0.0;
        }
        __syncwarp();
    }
    nk = n2;
    nre = __popc(__ballot_sync(0xffffffffu, need));
    const unsigned mask = (nbits >= 32) ? 0xffffffffu : ((1u << nbits) - 1u);
    return __ballot_sync(0xffffffffu, mine && bit) & mask;
}

template <int D, int NBP>
__device__ __forceinline__ void load_planes(const float* __restrict__ R, int nbits, int lane,
                                            uint32_t (&Rp)[NBP][D / 64]) {
    constexpr int EPL = D / 32;
#pragma unroll
    for (int b = 0; b < NBP; ++b)
#pragma unroll
        for (int e = 0; e < EPL / 2; ++e)
            Rp[b][e] = (b < nbits) ? pack_bf16_exact(R[b * D + lane * EPL + 2 * e], R[b * D + lane * EPL + 2 * e + 1])
                                   : 0u;
}

// One warp per prompt row r = l H + h.
template <int D, int NBP>
__global__ void __launch_bounds__(kWarps * 32) annca_prompt_kernel(const __nv_bfloat16* __restrict__ Kp,
                                                                   const __nv_bfloat16* __restrict__ Vp, AnnView a,
                                                                   const float* __restrict__ R,
                                                                   const float* __restrict__ Rnorm, Stats* stats) {
    constexpr int EPL = D / 32;
    using IO = RowIO<__nv_bfloat16, EPL>;
    __shared__ float sRow[kWarps][D];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    uint32_t Rp[NBP][D / 64];
    load_planes<D, NBP>(R, a.nbits, lane, Rp);
    const float rn = lane < a.nbits ? Rnorm[lane] : 0.f;
    const int64_t rows = (int64_t)a.L * a.H;
    for (int64_t r = (int64_t)blockIdx.x * kWarps + wib; r < rows; r += (int64_t)gridDim.x * kWarps) {
        const int l = (int)((uint32_t)r / (uint32_t)a.H), h = (int)(r - (int64_t)l * a.H);
        const typename IO::V kv = IO::load(Kp + r * D, lane);
        const typename IO::V vv = IO::load(Vp + r * D, lane);
        const int64_t dst = (int64_t)h * a.Lp + l;
        IO::store(a.Kh + dst * D, lane, kv);
        IO::store(a.Vh + dst * D, lane, vv);
        float x[EPL];
        IO::to_float(kv, x);
        float nk;
        unsigned nre;
        const unsigned code = hash_row<D, NBP>(x, Rp, R, rn, a.nbits, sRow[wib], lane, nk, nre);
        if (lane == 0) {
            a.pcode[dst] = code;
            // |k|^2 rounded up past the fp32 sum's error; floats >= 0 order like their bits
            atomicMax(reinterpret_cast<int*>(a.kmax2 + h), __float_as_int(nk * (1.f + 1.f / 1024.f)));
            if (nre) atomicAdd(&stats->hash_rechecks, (unsigned long long)nre);
        }
    }
}

// One block per head: bitonic sort of the (code, token) pairs in shared memory.
__global__ void __launch_bounds__(1024) annca_sort_kernel(AnnView a) {
    __shared__ unsigned long long key[kMaxPrompt];
    const int h = blockIdx.x;
    int n = 1;
    while (n < a.L) n <<= 1;
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        key[i] = (i < a.L) ? ((unsigned long long)a.pcode[(int64_t)h * a.Lp + i] << 32) | (unsigned)i : ~0ull;
    __syncthreads();
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                const int p = i ^ j;
                if (p > i) {
                    const unsigned long long u = key[i], w = key[p];
                    if ((u > w) == ((i & k) == 0)) {
                        key[i] = w;
                        key[p] = u;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = threadIdx.x; i < a.L; i += blockDim.x) {
        const uint32_t c = (uint32_t)(key[i] >> 32);
        const int32_t l = (int32_t)(key[i] & 0xffffffffu);
        int lo = 0, hi = i;   // first sorted position of code c
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if ((uint32_t)(key[mid] >> 32) < c) lo = mid + 1;
            else hi = mid;
        }
        a.pcs[(int64_t)h * a.Lp + i] = c;
        a.pix[(int64_t)h * a.Lp + i] = l;
        a.prun[(int64_t)h * a.Lp + l] = lo;
        if (a.ptab && lo == i) a.ptab[((int64_t)h << a.nbits) + c] = i;   // (cleared to -1 by the host)
    }
}

// Stamps the prompt bucket `code` of head h for slot z, if the prompt has that code.
// Many queries of a frame share a code: the stamp is only written while it reads
// different (a stale read just repeats the store).
__device__ __forceinline__ void flag_bucket(const AnnView& a, int h, int64_t z, uint32_t code) {
    int lo;
    if (a.ptab) {
        lo = a.ptab[((int64_t)h << a.nbits) + code];
    } else {
        const uint32_t* cs = a.pcs + (int64_t)h * a.Lp;
        int hi = a.L;   // first sorted position with code >= `code`
        lo = 0;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (cs[mid] < code) lo = mid + 1;
            else hi = mid;
        }
        if (lo >= a.L || cs[lo] != code) lo = -1;
    }
    if (lo >= 0) {
        uint32_t* f = a.keep + z * a.Lp + lo;
        if (*f != a.gen) *f = a.gen;
    }
}

// Shared memory of the mark kernel: per warp 16 staged rows (row stride padded by 16
// bytes so that lanes reading their own rows hit distinct banks).
template <int D>
struct MarkSmem {
    static constexpr int RB = D * 2 + 16;
    static constexpr int BYTES = kWarps * 16 * RB;
};

// The normals as fp32 [NBP][D] (zero rows past nbits) and their rounded-up norms, passed
// by value; the mark kernel copies the normals into shared memory once per block.
template <int D, int NBP>
struct Planes {
    float v[NBP * D];
    float rn[NBP];
};

// Two lanes per query row, 16 consecutive rows r = t H + h per warp: the warp copies its
// rows (one contiguous block of the token-major input) into shared memory with coalesced
// loads, then lane 2 i + u forms projections u NBP/2 ... u NBP/2 + NBP/2 - 1 of row i in
// fp32 (normals broadcast from shared memory; the second half of the normals sits 16 bytes
// further so that the two lanes' loads fall in different banks), keeps the sign of each bit
// outside its rounding bound and recomputes the rest in fp64 in index order. The code is
// stored token-major, and the row's even lane stamps its code's prompt bucket for its frame.
template <int D, int NBP>
__global__ void __launch_bounds__(kWarps * 32)
annca_mark_kernel(const __nv_bfloat16* __restrict__ Q, int rows, int P, int F, AnnView a,
                  const __grid_constant__ Planes<D, NBP> pl, Stats* stats) {
    using S = MarkSmem<D>;
    constexpr int W = D / 8;        // 16-byte words per row
    constexpr int HB = NBP / 2;     // projections per lane
    static_assert(NBP % 2 == 0, "two lanes per row");
    extern __shared__ __align__(16) uint8_t mk_smem[];
    uint8_t* sRows = mk_smem;
    __shared__ __align__(16) float sR[NBP * D + 4];   // the normals; bits >= HB start 4 floats later
    for (int i = threadIdx.x; i < NBP * D; i += blockDim.x) sR[i + (i >= HB * D ? 4 : 0)] = pl.v[i];
    __syncthreads();
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int half = lane & 1, ri = lane >> 1;
    const float* myR = sR + half * (HB * D + 4);
    const int nbits = a.nbits;
    grid_dependency_wait();
    uint8_t* mine = sRows + wib * 16 * S::RB;
    const float gam2 = 2.f * (float)(D + 2) * kU32;
    unsigned rechecks = 0;
    for (int base = (blockIdx.x * kWarps + wib) * 16; base < rows; base += gridDim.x * kWarps * 16) {
        const int n = min(16, rows - base);
        const uint4* src = reinterpret_cast<const uint4*>(Q + (int64_t)base * D);
#pragma unroll 8
        for (int w = lane; w < n * W; w += 32) {
            const int row = w / W, col = w - row * W;
            *reinterpret_cast<uint4*>(mine + row * S::RB + col * 16) = src[w];
        }
        __syncwarp();
        uint32_t code = 0;
        if (ri < n) {
            const uint8_t* rowp = mine + ri * S::RB;
            float acc[HB];
#pragma unroll
            for (int b = 0; b < HB; ++b) acc[b] = 0.f;
            float n2 = 0.f;
#pragma unroll 1
            for (int c = 0; c < W; ++c) {
                const uint4 v = *reinterpret_cast<const uint4*>(rowp + c * 16);
                const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
                float x[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    x[2 * k] = __uint_as_float(wd[k] << 16);
                    x[2 * k + 1] = __uint_as_float(wd[k] & 0xffff0000u);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) n2 = fmaf(x[k], x[k], n2);
#pragma unroll
                for (int b = 0; b < HB; ++b) {
                    const float4 r0 = *reinterpret_cast<const float4*>(myR + b * D + c * 8);
                    const float4 r1 = *reinterpret_cast<const float4*>(myR + b * D + c * 8 + 4);
                    float t = acc[b];
                    t = fmaf(r0.x, x[0], t);
                    t = fmaf(r0.y, x[1], t);
                    t = fmaf(r0.z, x[2], t);
                    t = fmaf(r0.w, x[3], t);
                    t = fmaf(r1.x, x[4], t);
                    t = fmaf(r1.y, x[5], t);
                    t = fmaf(r1.z, x[6], t);
                    t = fmaf(r1.w, x[7], t);
                    acc[b] = t;
                }
            }
            // |<R_b,x>| > 2 (d+2) u |R_b||x| certifies the fp32 sign (any summation order
            // errs by at most (d+2) u |R_b||x|; doubled for margin); else fp64, index order
            const float nx = sqrtf(n2);
#pragma unroll
            for (int k = 0; k < HB; ++k) {
                const int b = half * HB + k;
                if (b >= nbits) break;
                bool bit = acc[k] >= 0.f;
                if (!(fabsf(acc[k]) > gam2 * pl.rn[b] * nx + 1e-30f)) {
                    // (the shared copy holds the bf16 normals exactly; products are exact in fp64)
                    const float* Rb = myR + k * D;
                    double s64 = 0.0;
#pragma unroll 8
                    for (int i = 0; i < D; ++i) {
                        const uint16_t u = *reinterpret_cast<const uint16_t*>(rowp + 2 * i);
                        s64 = fma((double)Rb[i], (double)__uint_as_float((uint32_t)u << 16), s64);
                    }
                    bit = s64 >= 0.0;
                    ++rechecks;
                }
                code |= (uint32_t)bit << b;
            }
        }
        code |= __shfl_xor_sync(0xffffffffu, code, 1);   // the two halves' bits
        if (ri < n && half == 0) {
            const int r = base + ri;
            a.qcode[r] = code;
            const int t = (int)((uint32_t)r / (uint32_t)a.H);
            const int h = r - t * a.H;
            flag_bucket(a, h, (int64_t)h * F + (int)((uint32_t)t / (uint32_t)P), code);
        }
        __syncwarp();
    }
    if (rechecks) atomicAdd(&stats->hash_rechecks, (unsigned long long)rechecks);
    grid_dependents_launch();
}

// Exclusive scan of one value per thread over the block (blockDim.x <= 1024).
__device__ int block_exclusive_scan(int v, int* total) {
    __shared__ int wsum[32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[w] = inc;
    __syncthreads();
    if (w == 0) {
        int y = (lane < nw) ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int s = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y += s;
        }
        wsum[lane] = y;
    }
    __syncthreads();
    const int before = (w > 0) ? wsum[w - 1] : 0;
    *total = wsum[nw - 1];
    __syncthreads();
    return before + inc - v;
}

// Blocks (z, part) for slot z = h F + f: every part lists the kept tokens (the list is
// short), part 0 publishes it with the count and the logit shifts, and each part packs
// its share of the rows.
constexpr int kPackParts = 4;

template <int D>
__global__ void __launch_bounds__(256) annca_pack_kernel(int F, AnnView a) {
    grid_dependency_wait();
    constexpr int W = D / 8;   // 16-byte words per row
    __shared__ int32_t sList[kMaxPrompt];
    const int64_t z = blockIdx.x;
    const int part = blockIdx.y;
    const int h = (int)(z / F);
    const uint32_t* stamp = a.keep + z * a.Lp;
    const int32_t* run = a.prun + (int64_t)h * a.Lp;
    const int per = (a.L + blockDim.x - 1) / blockDim.x;
    const int l0 = min(a.L, (int)threadIdx.x * per), l1 = min(a.L, l0 + per);
    int c = 0;
    for (int l = l0; l < l1; ++l) c += stamp[run[l]] == a.gen;
    int n = 0;
    int pos = block_exclusive_scan(c, &n);
    for (int l = l0; l < l1; ++l)
        if (stamp[run[l]] == a.gen) sList[pos++] = l;
    __syncthreads();
    const int nt = (n + 127) & ~127;
    if (part == 0) {
        for (int j = threadIdx.x; j < n; j += blockDim.x) a.sidx[z * a.Lp + j] = sList[j];
        for (int j = threadIdx.x; j < nt; j += blockDim.x) a.sbias[z * a.Lp + j] = (j < n) ? 0.f : -INFINITY;
        if (threadIdx.x == 0) a.nsel[z] = n;
    }
    const int share = (nt / 32 + gridDim.y - 1) / gridDim.y * 32;   // rows per part, whole warps of rows
    const int j0 = min(nt, part * share), j1 = min(nt, j0 + share);
    const uint4* Kh = reinterpret_cast<const uint4*>(a.Kh + (int64_t)h * a.Lp * D);
    const uint4* Vh = reinterpret_cast<const uint4*>(a.Vh + (int64_t)h * a.Lp * D);
    uint4* Ks = reinterpret_cast<uint4*>(a.Ks + z * a.Lp * D);
    uint4* Vs = reinterpret_cast<uint4*>(a.Vs + z * a.Lp * D);
    for (int i = j0 * W + threadIdx.x; i < j1 * W; i += blockDim.x) {
        const int j = i / W, w = i - j * W;
        uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = kv;
        if (j < n) {
            const int64_t l = sList[j];
            kv = Kh[l * W + w];
            vv = Vh[l * W + w];
        }
        Ks[(int64_t)j * W + w] = kv;
        Vs[(int64_t)j * W + w] = vv;
    }
    grid_dependents_launch();
}

template <int D>
cudaError_t prompt_t(const AnnView& a, const void* Kp, const void* Vp, const float* R, const float* Rnorm,
                     Stats* stats, cudaStream_t st) {
    const int grid = grid_for_rows((int64_t)a.L * a.H, kWarps, 148 * 8);
    const auto* K = reinterpret_cast<const __nv_bfloat16*>(Kp);
    const auto* V = reinterpret_cast<const __nv_bfloat16*>(Vp);
    if (a.nbits <= 8) annca_prompt_kernel<D, 8><<<grid, kWarps * 32, 0, st>>>(K, V, a, R, Rnorm, stats);
    else if (a.nbits <= 16) annca_prompt_kernel<D, 16><<<grid, kWarps * 32, 0, st>>>(K, V, a, R, Rnorm, stats);
    else annca_prompt_kernel<D, 32><<<grid, kWarps * 32, 0, st>>>(K, V, a, R, Rnorm, stats);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    annca_sort_kernel<<<a.H, 1024, 0, st>>>(a);
    return cudaGetLastError();
}

template <int D, int NBP>
cudaError_t mark_t(const __nv_bfloat16* Q, int rows, int P, int F, const AnnView& a, const float* R,
                   const float* Rhost, const float* Rnorm_host, Stats* stats, cudaStream_t st) {
    cudaError_t e = smem_attr_once(reinterpret_cast<const void*>(annca_mark_kernel<D, NBP>), MarkSmem<D>::BYTES);
    if (e != cudaSuccess) return e;
    Planes<D, NBP> pl;
    for (int b = 0; b < NBP; ++b) {
        for (int i = 0; i < D; ++i) pl.v[b * D + i] = (b < a.nbits) ? Rhost[b * D + i] : 0.f;
        pl.rn[b] = (b < a.nbits) ? Rnorm_host[b] : 0.f;
    }
    const int grid = (rows + kWarps * 16 - 1) / (kWarps * 16);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = MarkSmem<D>::BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, annca_mark_kernel<D, NBP>, Q, rows, P, F, a, pl, stats);
}

template <int D>
cudaError_t select_t(const AnnView& a, const void* Qv, int64_t Tq, int P, int F, const float* R,
                     const float* Rhost, const float* Rnorm_host, Stats* stats, cudaStream_t st) {
    const auto* Q = reinterpret_cast<const __nv_bfloat16*>(Qv);
    const int rows = (int)(Tq * a.H);   // < 2^31 (host check)
    cudaError_t e;
    if (a.nbits <= 8) e = mark_t<D, 8>(Q, rows, P, F, a, R, Rhost, Rnorm_host, stats, st);
    else if (a.nbits <= 12) e = mark_t<D, 12>(Q, rows, P, F, a, R, Rhost, Rnorm_host, stats, st);
    else if (a.nbits <= 16) e = mark_t<D, 16>(Q, rows, P, F, a, R, Rhost, Rnorm_host, stats, st);
    else e = mark_t<D, 24>(Q, rows, P, F, a, R, Rhost, Rnorm_host, stats, st);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.H * F), (unsigned)kPackParts);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, annca_pack_kernel<D>, F, a);
}

// ------------------------------------------------------------------ AnnSA
//
// FAST-AR technical summary, section 2.C "AnnSA": the buckets found while pruning the
// cross-attention are reused and every token's self-attention query only sees the keys
// of its own bucket. Here a token's bucket is its AnnCA query code in the same head; the
// tokens of the block are put in bucket order per head, packed, and the attention
// kernel's sparse mode runs every 128-row query tile against the key tiles spanning its
// buckets, masked per element to the same bucket.

constexpr int kMaxSparseT = 16384;   // tokens per block (the ordering sorts in shared memory)

// Start of every ordering kernel (one block per head h, launched as a programmatic
// dependent of the previous kernel in the stream, which may be the previous call's
// attention reading the arrays rewritten here): wait for it, clear the head's key bound
// for the packing kernel, and let the packing kernel be scheduled.
__device__ __forceinline__ void order_prologue(const SparseBufs& b, int h) {
    grid_dependency_wait();
    if (threadIdx.x == 0) b.kmax2[h] = 0.f;
    grid_dependents_launch();
}

// One block per head: bitonic sort of (code, token); per packed row its token and code;
// per query tile the key tiles from the start of its first row's bucket to the end of its
// last row's bucket.
__global__ void __launch_bounds__(1024) annsa_order_kernel(SparseBufs b) {
    extern __shared__ unsigned long long okey[];
    const int h = blockIdx.x;
    const int T = (int)b.T;
    order_prologue(b, h);
    int n = 1;
    while (n < T) n <<= 1;
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        okey[i] = (i < T) ? ((unsigned long long)b.codes[(int64_t)i * b.H + h] << 32) | (unsigned)i : ~0ull;
    __syncthreads();
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                const int p = i ^ j;
                if (p > i) {
                    const unsigned long long u = okey[i], w = okey[p];
                    if ((u > w) == ((i & k) == 0)) {
                        okey[i] = w;
                        okey[p] = u;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int64_t i = threadIdx.x; i < b.Tp; i += blockDim.x) {
        const int64_t o = (int64_t)h * b.Tp + i;
        b.perm[o] = (i < T) ? (int32_t)(okey[i] & 0xffffffffu) : -1;
        b.grp[o] = (i < T) ? (uint32_t)(okey[i] >> 32) : 0xffffffffu;
    }
    const int nqt = (int)(b.Tp / 128);   // row stride of tiles
    for (int k = threadIdx.x; k < (T + 127) / 128; k += blockDim.x) {
        const int f = 128 * k, l = min(f + 127, T - 1);
        const uint32_t cf = (uint32_t)(okey[f] >> 32), cl = (uint32_t)(okey[l] >> 32);
        int lo = 0, hi = f;   // first row of cf's bucket
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if ((uint32_t)(okey[mid] >> 32) < cf) lo = mid + 1;
            else hi = mid;
        }
        int lo2 = l, hi2 = T;   // one past the last row of cl's bucket
        while (lo2 < hi2) {
            const int mid = (lo2 + hi2) >> 1;
            if ((uint32_t)(okey[mid] >> 32) <= cl) lo2 = mid + 1;
            else hi2 = mid;
        }
        b.tiles[(int64_t)h * nqt + k] = make_int2(lo / 128, (lo2 + 127) / 128);
    }
}

// The same order by counting, for codes below 2^kCountBits (one block per head, 1024
// threads): bucket sizes by shared-memory atomics, bucket starts by a scan, then the
// tokens are placed chunk by chunk in token order: inside a warp, lanes with the same
// code rank themselves with a match mask, and the warps of a chunk take their places in
// order, one warp per step, from a running cursor per code. The result equals the sort
// of (code, token) above.
constexpr int kCountBits = 13;

__global__ void __launch_bounds__(1024) annsa_count_kernel(SparseBufs b, int nbits) {
    extern __shared__ int32_t cs_smem[];
    const int ncodes = 1 << nbits;
    int32_t* cnt = cs_smem;              // [ncodes]
    int32_t* cur = cs_smem + ncodes;     // [ncodes] running cursor, finally the bucket end
    int32_t* sBase = cur + ncodes;       // [32][32] base position of each (warp, lane) group
    __shared__ int wsum[32];
    const int h = blockIdx.x, T = (int)b.T;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    order_prologue(b, h);
    for (int c = threadIdx.x; c < ncodes; c += blockDim.x) cnt[c] = 0;
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x) atomicAdd(&cnt[b.codes[(int64_t)t * b.H + h]], 1);
    __syncthreads();
    {   // exclusive scan of cnt into cur: each thread a contiguous run of codes
        const int per = (ncodes + blockDim.x - 1) / blockDim.x;
        const int c0 = min(ncodes, (int)threadIdx.x * per), c1 = min(ncodes, c0 + per);
        int run = 0;
        for (int c = c0; c < c1; ++c) run += cnt[c];
        int inc = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane == 31) wsum[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            int y = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int z = __shfl_up_sync(0xffffffffu, y, o);
                if (lane >= o) y += z;
            }
            wsum[lane] = y;
        }
        __syncthreads();
        int pos = (warp > 0 ? wsum[warp - 1] : 0) + inc - run;
        for (int c = c0; c < c1; ++c) {
            cur[c] = pos;
            pos += cnt[c];
        }
    }
    __syncthreads();
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < T; base += blockDim.x) {
        const int t = base + threadIdx.x;
        const bool valid = t < T;
        const uint32_t c = valid ? b.codes[(int64_t)t * b.H + h] : 0xffffffffu;
        const unsigned same = __match_any_sync(0xffffffffu, c);
        const int rank = __popc(same & lt), lead = __ffs(same) - 1;
        for (int w = 0; w < 32; ++w) {
            if (warp == w && valid && lane == lead) {
                sBase[w * 32 + lane] = cur[c];
                cur[c] += __popc(same);
            }
            __syncthreads();
        }
        if (valid) {
            const int64_t o = (int64_t)h * b.Tp + sBase[warp * 32 + lead] + rank;
            b.perm[o] = t;
            b.grp[o] = c;
        }
        __syncthreads();
    }
    for (int64_t i = T + threadIdx.x; i < b.Tp; i += blockDim.x) {
        b.perm[(int64_t)h * b.Tp + i] = -1;
        b.grp[(int64_t)h * b.Tp + i] = 0xffffffffu;
    }
    __syncthreads();   // (this block's own global writes, read back below)
    const int nqt = (int)(b.Tp / 128);
    for (int k = threadIdx.x; k < (T + 127) / 128; k += blockDim.x) {
        const int f = 128 * k, l = min(f + 127, T - 1);
        const uint32_t cf = b.grp[(int64_t)h * b.Tp + f], cl = b.grp[(int64_t)h * b.Tp + l];
        b.tiles[(int64_t)h * nqt + k] = make_int2((cur[cf] - cnt[cf]) / 128, (cur[cl] + 127) / 128);
    }
}

// The same order for codes of at most kSegBits bits, spread over kOrdBlocks blocks per head
// in two kernels. Block (h, j) owns the contiguous token range [j S, j S + S), S =
// ceil(T / kOrdBlocks). The first kernel counts each code over every block's range; the
// second sums, per code, all blocks' counts (the bucket size) and the earlier blocks' ones
// (this block's offset inside the bucket), scans the bucket sizes into bucket starts, counts
// its range again per warp (each warp a contiguous sub-range, one 16-byte row of eight
// counts per code) and places its tokens in order, ranking equal codes inside each 32-token
// step with a match mask. Positions fit 16 bits (T <= kMaxSparseT).
constexpr int kSegBits = 10;
constexpr int kOrdBlocks = 8;
constexpr int kOrdSteps = kMaxSparseT / kOrdBlocks / 8 / 32;   // 32-token steps of one warp's sub-range, at most

__device__ __forceinline__ void ord_range(int T, int j, int& a, int& e) {
    const int S = (T + kOrdBlocks - 1) / kOrdBlocks;
    a = min(T, j * S);
    e = min(T, a + S);
}

__device__ __forceinline__ int ord_code_at(const int32_t* cstart, int ncodes, int f) {
    int lo = 0, hi = ncodes;   // the last code whose bucket starts at or before packed row f
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (cstart[mid] <= f) lo = mid + 1;
        else hi = mid;
    }
    return lo - 1;
}

__global__ void __launch_bounds__(256) annsa_bcount_kernel(SparseBufs b, int nbits) {
    extern __shared__ int32_t bc_smem[];   // [ncodes]
    const int ncodes = 1 << nbits, h = blockIdx.x / kOrdBlocks, j = blockIdx.x % kOrdBlocks;
    order_prologue(b, h);
    for (int c = threadIdx.x; c < ncodes; c += blockDim.x) bc_smem[c] = 0;
    __syncthreads();
    int a, e;
    ord_range((int)b.T, j, a, e);
    for (int t = a + threadIdx.x; t < e; t += blockDim.x) atomicAdd(&bc_smem[b.codes[(int64_t)t * b.H + h]], 1);
    __syncthreads();
    int32_t* dst = b.bcnt + ((int64_t)h * kOrdBlocks + j) * ncodes;
    for (int c = threadIdx.x; c < ncodes; c += blockDim.x) dst[c] = bc_smem[c];
}

__global__ void __launch_bounds__(256) annsa_bplace_kernel(SparseBufs b, int nbits) {
    extern __shared__ __align__(16) int32_t bp_smem[];
    const int ncodes = 1 << nbits, h = blockIdx.x / kOrdBlocks, j = blockIdx.x % kOrdBlocks;
    int32_t* cstart = bp_smem;                                       // [ncodes] bucket start
    int32_t* ctot = cstart + ncodes;                                 // [ncodes] bucket size
    uint16_t* wh = reinterpret_cast<uint16_t*>(ctot + ncodes);       // [ncodes][8] per-warp counts
    __shared__ int wsum[8];
    const int T = (int)b.T, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt = (1u << lane) - 1u;
    grid_dependency_wait();   // the counts of every block
    grid_dependents_launch();
    int a, e;
    ord_range(T, j, a, e);
    const int sub = (e - a + 7) / 8, w0 = min(e, a + warp * sub), w1 = min(e, w0 + sub);
    uint32_t cc[kOrdSteps];
#pragma unroll
    for (int k = 0; k < kOrdSteps; ++k) {
        const int t = w0 + 32 * k + lane;
        cc[k] = (t < w1) ? b.codes[(int64_t)t * b.H + h] : 0xffffffffu;
    }
    for (int i = threadIdx.x; i < ncodes; i += blockDim.x) reinterpret_cast<uint4*>(wh)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kOrdSteps; ++k) {
        if (w0 + 32 * k >= w1) break;   // warp-uniform
        const uint32_t c = cc[k];
        const bool valid = w0 + 32 * k + lane < w1;
        const unsigned same = __match_any_sync(0xffffffffu, c);
        if (valid && lane == __ffs(same) - 1) wh[c * 8 + warp] += (uint16_t)__popc(same);
        __syncwarp();
    }
    // per code: bucket size and this block's offset in it from the blocks' counts; the bucket
    // starts by a block scan (consecutive codes per thread)
    const int per = (ncodes + blockDim.x - 1) / blockDim.x;
    const int c0 = min(ncodes, (int)threadIdx.x * per), c1 = min(ncodes, c0 + per);
    const int32_t* cnt = b.bcnt + (int64_t)h * kOrdBlocks * ncodes;
    int run = 0;
    for (int c = c0; c < c1; ++c) {
        int tot = 0, off = 0;
#pragma unroll
        for (int jj = 0; jj < kOrdBlocks; ++jj) {
            const int n = cnt[jj * ncodes + c];
            tot += n;
            off += (jj < j) ? n : 0;
        }
        ctot[c] = tot;
        cstart[c] = off;   // (for now: this block's offset inside the bucket)
        run += tot;
    }
    int inc = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();   // (also: every warp's counts)
    int pos = inc - run;
    for (int w = 0; w < warp; ++w) pos += wsum[w];
    for (int c = c0; c < c1; ++c) {
        const int off = cstart[c];
        cstart[c] = pos;
        uint4* row = reinterpret_cast<uint4*>(wh + c * 8);
        uint4 v = *row;
        uint32_t wd[4] = {v.x, v.y, v.z, v.w};
        uint32_t cur = (uint32_t)(pos + off);
#pragma unroll
        for (int q = 0; q < 4; ++q) {   // warps 2 q and 2 q + 1: their first positions for code c
            const uint32_t f0 = cur, f1 = f0 + (wd[q] & 0xffffu);
            cur = f1 + (wd[q] >> 16);
            wd[q] = f0 | (f1 << 16);
        }
        *row = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        pos += ctot[c];
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kOrdSteps; ++k) {
        if (w0 + 32 * k >= w1) break;   // warp-uniform
        const int t = w0 + 32 * k + lane;
        const bool valid = t < w1;
        const uint32_t c = cc[k];
        const unsigned same = __match_any_sync(0xffffffffu, c);
        const int lead = __ffs(same) - 1;
        int first = 0;
        if (valid && lane == lead) {
            first = wh[c * 8 + warp];
            wh[c * 8 + warp] = (uint16_t)(first + __popc(same));
        }
        first = __shfl_sync(0xffffffffu, first, lead);
        if (valid) {
            const int64_t o = (int64_t)h * b.Tp + first + __popc(same & lt);
            b.perm[o] = t;
            b.grp[o] = c;
        }
        __syncwarp();
    }
    for (int64_t i = T + (int64_t)j * blockDim.x + threadIdx.x; i < b.Tp; i += (int64_t)kOrdBlocks * blockDim.x) {
        b.perm[(int64_t)h * b.Tp + i] = -1;
        b.grp[(int64_t)h * b.Tp + i] = 0xffffffffu;
    }
    // per query tile the key tiles from its first row's bucket start to its last row's
    // bucket end (the rows' codes found from the bucket starts); block j takes tiles j, j + 8, ...
    const int nqt = (int)(b.Tp / 128);
    for (int k = j + kOrdBlocks * (int)threadIdx.x; k < (T + 127) / 128; k += kOrdBlocks * blockDim.x) {
        const int f = 128 * k, l = min(f + 127, T - 1);
        const int cf = ord_code_at(cstart, ncodes, f), cl = ord_code_at(cstart, ncodes, l);
        b.tiles[(int64_t)h * nqt + k] = make_int2(cstart[cf] / 128, (cstart[cl] + ctot[cl] + 127) / 128);
    }
}

// One warp per packed row r = h Tp + i: copy the token's q, k, v rows (zeros past T),
// its own logit scale log2(e) <q, k> (the first softmax reference when the kernel cannot
// use a fixed one) and the head's bound of |k|^2.
template <int D>
__global__ void __launch_bounds__(kWarps * 32) annsa_pack_kernel(SparseBufs b, const __nv_bfloat16* __restrict__ Q,
                                                                 const __nv_bfloat16* __restrict__ K,
                                                                 const __nv_bfloat16* __restrict__ V,
                                                                 float scale_log2) {
    grid_dependency_wait();
    constexpr int W = D / 8;        // 16-byte words per row: W lanes per row
    constexpr int RPW = 32 / W;     // rows per warp and step
    const int lane = threadIdx.x & 31, sub = lane / W, w = lane % W;
    const int64_t Tr = (b.T + 127) / 128 * 128;   // packed rows per head the attention reads
    const int64_t rows = (int64_t)b.H * Tr;
    const uint4* Q4 = reinterpret_cast<const uint4*>(Q);
    const uint4* K4 = reinterpret_cast<const uint4*>(K);
    const uint4* V4 = reinterpret_cast<const uint4*>(V);
    uint4* Qs4 = reinterpret_cast<uint4*>(b.Qs);
    uint4* Ks4 = reinterpret_cast<uint4*>(b.Ks);
    uint4* Vs4 = reinterpret_cast<uint4*>(b.Vs);
    // each block packs one contiguous range of rows (one or two heads), and gathers the
    // heads' |k|^2 bounds in shared memory: one atomic per head and block, not per row
    constexpr int kSlots = 4;
    __shared__ float sK[kSlots];
    if (threadIdx.x < kSlots) sK[threadIdx.x] = 0.f;
    __syncthreads();
    const int64_t per = ((rows + gridDim.x - 1) / gridDim.x + RPW - 1) / RPW * RPW;
    const int64_t rb0 = (int64_t)blockIdx.x * per, rb1 = min(rows, rb0 + per);
    const int hlo = (int)(min(rb0, rows - 1) / Tr);
    const int wib = threadIdx.x >> 5;
    for (int64_t rr0 = rb0 + (int64_t)wib * RPW; rr0 < rb1; rr0 += (int64_t)kWarps * RPW) {
        const int64_t rr = rr0 + sub;
        const bool live = rr < rb1;
        const int h = live ? (int)(rr / Tr) : 0;
        const int64_t r = (int64_t)h * b.Tp + (rr - (int64_t)h * Tr);
        const int32_t t = live ? b.perm[r] : -1;
        uint4 q4 = make_uint4(0u, 0u, 0u, 0u), k4 = q4, v4 = q4;
        if (t >= 0) {
            const int64_t src = ((int64_t)t * b.H + h) * W + w;
            q4 = Q4[src];
            k4 = K4[src];
            v4 = V4[src];
        }
        if (live) {
            Qs4[r * W + w] = q4;
            Ks4[r * W + w] = k4;
            Vs4[r * W + w] = v4;
        }
        const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w}, kw[4] = {k4.x, k4.y, k4.z, k4.w};
        float qk = 0.f, kk = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float ql = __uint_as_float(qw[e] << 16), qh = __uint_as_float(qw[e] & 0xffff0000u);
            const float kl = __uint_as_float(kw[e] << 16), kh = __uint_as_float(kw[e] & 0xffff0000u);
            qk = fmaf(ql, kl, fmaf(qh, kh, qk));
            kk = fmaf(kl, kl, fmaf(kh, kh, kk));
        }
#pragma unroll
        for (int o = 1; o < W; o <<= 1) {   // sums over the W lanes of this row
            qk += __shfl_xor_sync(0xffffffffu, qk, o);
            kk += __shfl_xor_sync(0xffffffffu, kk, o);
        }
        if (live && w == 0) {
            b.xself[r] = qk * scale_log2;
            const float kb = kk * (1.f + 1.f / 1024.f);   // floats >= 0 order like their bits
            if (h - hlo < kSlots) atomicMax(reinterpret_cast<int*>(sK + (h - hlo)), __float_as_int(kb));
            else atomicMax(reinterpret_cast<int*>(b.kmax2 + h), __float_as_int(kb));
        }
    }
    __syncthreads();
    if (threadIdx.x < kSlots && hlo + (int)threadIdx.x < b.H && sK[threadIdx.x] > 0.f)
        atomicMax(reinterpret_cast<int*>(b.kmax2 + hlo + threadIdx.x), __float_as_int(sK[threadIdx.x]));
    grid_dependents_launch();
}

}  // namespace

cudaError_t launch_annsa_pack(const SparseBufs& b, int nbits, const void* Q, const void* K, const void* V,
                              float scale_log2, cudaStream_t st) {
cudaError_t e = smem_attr_once(reinterpret_cast<const void*>(annsa_order_kernel), kMaxSparseT * 8);
    if (e == cudaSuccess)
        e = smem_attr_once(reinterpret_cast<const void*>(annsa_count_kernel), (2 << kCountBits) * 4 + 32 * 32 * 4);
    if (e != cudaSuccess) return e;
    if (nbits <= kSegBits) {
        const int ncodes = 1 << nbits;   // shared memory: counts; starts, sizes and [ncodes][8] uint16
        e = launch_pdl_smem(annsa_bcount_kernel, b.H * kOrdBlocks, 256, ncodes * 4, st, b, nbits);
        if (e == cudaSuccess)
            e = launch_pdl_smem(annsa_bplace_kernel, b.H * kOrdBlocks, 256, ncodes * 24, st, b, nbits);
    } else if (nbits <= kCountBits) {
        e = launch_pdl_smem(annsa_count_kernel, b.H, 1024, (2 << nbits) * 4 + 32 * 32 * 4, st, b, nbits);
    } else {
        int n = 1;
        while (n < b.T) n <<= 1;
        e = launch_pdl_smem(annsa_order_kernel, b.H, 1024, n * 8, st, b);
    }
    if (e != cudaSuccess) return e;
    const int grid = grid_for_rows((int64_t)b.H * ((b.T + 127) / 128 * 128), kWarps * (32 / (b.d / 8)), 148 * 8);
    const auto* q = reinterpret_cast<const __nv_bfloat16*>(Q);
    const auto* k = reinterpret_cast<const __nv_bfloat16*>(K);
    const auto* v = reinterpret_cast<const __nv_bfloat16*>(V);
    return b.d == 128 ? launch_pdl(annsa_pack_kernel<128>, grid, kWarps * 32, st, b, q, k, v, scale_log2)
                      : launch_pdl(annsa_pack_kernel<64>, grid, kWarps * 32, st, b, q, k, v, scale_log2);
}

cudaError_t launch_annca_prompt(const AnnView& a, const void* Kp, const void* Vp, const float* R,
                                const float* Rnorm, Stats* stats, cudaStream_t st) {
    return a.d == 128 ? prompt_t<128>(a, Kp, Vp, R, Rnorm, stats, st) : prompt_t<64>(a, Kp, Vp, R, Rnorm, stats, st);
}

cudaError_t launch_annca_select(const AnnView& a, const void* Q, int64_t Tq, int P, int F, const float* R,
                                const float* Rhost, const float* Rnorm_host, Stats* stats, cudaStream_t st) {
    return a.d == 128 ? select_t<128>(a, Q, Tq, P, F, R, Rhost, Rnorm_host, stats, st)
                      : select_t<64>(a, Q, Tq, P, F, R, Rhost, Rnorm_host, stats, st);
}

}  // namespace tc

// ------------------------------------------------------------------ C ABI

using namespace tc;

namespace {

constexpr uint32_t kAnnMagic = 0x7c7ca2c3u;

int64_t up128(int64_t x) { return (x + 127) / 128 * 128; }

}  // namespace

struct tc_annca_ctx {
    uint32_t magic = kAnnMagic;
    int H = 0, d = 0, nbits = 0;
    float scale = 0.f;
    int device = 0;
    AnnView a{};
    int64_t Lcap = 0;       // padded prompt rows allocated (a.Lp is this prompt's)
    bool prompt_set = false;
    int64_t last_T = 0, last_F = 0;
    float* R = nullptr;
    float* Rnorm = nullptr;
    Stats* stats = nullptr;
    std::vector<float> Rhost;
    std::vector<float> Rnorm_host;
    AttnMaps maps{};
    int64_t maps_Lp = -1;   // row stride the key/value maps were encoded with
    // AnnSA buffers, sized for sp_Tp packed rows per head
    SparseBufs sb{};
    int64_t sp_Tp = 0;
    float* sp_kmax2 = nullptr;
    AttnMaps sp_maps{};
    cudaStream_t last_stream = nullptr;
    tc_status sticky = TC_OK;

    void release(void*& p) {
        if (p) cudaFree(p);
        p = nullptr;
    }
    template <typename T>
    tc_status grab(T*& p, size_t bytes) {
        void* q = nullptr;
        if (dev_alloc(&q, bytes) != cudaSuccess) {
            cudaGetLastError();
            return TC_ENOMEM;
        }
        p = static_cast<T*>(q);
        return TC_OK;
    }
    void free_prompt() {
        void* ps[] = {a.Kh, a.Vh, a.pcode, a.pcs, a.pix, a.prun};
        for (void* p : ps) if (p) cudaFree(p);
        a.Kh = a.Vh = nullptr;
        a.pcode = a.pcs = nullptr;
        a.pix = a.prun = nullptr;
        // (ptab depends only on H and nbits: kept until the handle goes)
        Lcap = 0;
    }
    void free_queries() {
        if (a.qcode) cudaFree(a.qcode);
        a.qcode = nullptr;
        a.Tmax = 0;
    }
    void free_slots() {
        void* ps[] = {a.keep, a.nsel, a.sidx, a.Ks, a.Vs, a.sbias};
        for (void* p : ps) if (p) cudaFree(p);
        a.keep = nullptr;
        a.nsel = a.sidx = nullptr;
        a.Ks = a.Vs = nullptr;
        a.sbias = nullptr;
        a.Zmax = 0;
    }
    void free_sparse() {
        void* ps[] = {sb.perm, sb.grp, sb.tiles, sb.xself, sb.Qs, sb.Ks, sb.Vs, sb.bcnt};
        for (void* p : ps) if (p) cudaFree(p);
        sb = SparseBufs{};
        sp_Tp = 0;
    }
    ~tc_annca_ctx() {
        free_prompt();
        free_queries();
        free_slots();
        free_sparse();
        if (sp_kmax2) cudaFree(sp_kmax2);
        void* ps[] = {R, Rnorm, stats, a.kmax2, a.zeros, a.ptab};
        for (void* p : ps) if (p) cudaFree(p);
        magic = 0;
    }
};

namespace {

bool valid(tc_annca_handle h) { return h != nullptr && h->magic == kAnnMagic; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tc_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return TC_OK;
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? TC_ENOMEM : TC_ECUDA;
}

tc_status check_call(tc_annca_ctx* x) {
    if (!valid(x)) return TC_EINVAL;
    if (x->sticky != TC_OK) return x->sticky;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != x->device) {
        cudaGetLastError();
        return TC_EDEVICE;
    }
    return TC_OK;
}

// Per-slot arrays for Z = H F slots of the current prompt length; re-encodes the
// key and value tensor maps.
tc_status ensure_slots(tc_annca_ctx* x, int64_t Z) {
    AnnView& a = x->a;
    if (a.keep && Z <= a.Zmax && x->maps_Lp == a.Lp) return TC_OK;
    if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
    const int64_t Zn = std::max<int64_t>(Z, a.Zmax);
    x->free_slots();
    const size_t rows = (size_t)Zn * x->Lcap;
    tc_status st;
    if ((st = x->grab(a.keep, rows * 4)) || (st = x->grab(a.nsel, (size_t)Zn * 4)) || (st = x->grab(a.sidx, rows * 4)) ||
        (st = x->grab(a.Ks, rows * x->d * 2)) || (st = x->grab(a.Vs, rows * x->d * 2)) ||
        (st = x->grab(a.sbias, rows * 4))) {
        x->free_slots();
        return st;
    }
    if (cudaMemset(a.keep, 0, rows * 4) != cudaSuccess || cudaMemset(a.nsel, 0, (size_t)Zn * 4) != cudaSuccess) {
        x->free_slots();
        return cuda_status(cudaGetLastError());
    }
    a.Zmax = Zn;
    const uint64_t d = x->d;
    if (!encode3d(&x->maps.kc, a.Ks, d, a.Lp, Zn, d * 2, a.Lp * d * 2, 64, 128, 1) ||
        !encode3d(&x->maps.vc, a.Vs, d, a.Lp, Zn, d * 2, a.Lp * d * 2, 64, 128, 1)) {
        x->free_slots();
        return TC_ECUDA;
    }
    x->maps_Lp = a.Lp;
    return TC_OK;
}

}  // namespace

extern "C" {

tc_status tc_annca_create(int32_t H, int32_t d, int32_t nbits, const tc_options* opt, tc_annca_handle* out) {
    if (!out) return TC_EINVAL;
    *out = nullptr;
    tc_options o{TC_BF16, 0, 0.f, nullptr, 0};
    if (opt) o = *opt;
    if (H < 1 || H > 4096 || (d != 64 && d != 128) || nbits < 1 || nbits > 24 || !(o.softmax_scale >= 0.f) ||
        !std::isfinite(o.softmax_scale) || o.intra_chunk != 0 || (o.dtype != TC_BF16 && o.dtype != TC_F32))
        return TC_EINVAL;
    if (o.dtype != TC_BF16) return TC_ENOTIMPL;
    if (o.hyperplanes) {
        for (int i = 0; i < nbits * d; ++i)
            if (!std::isfinite(o.hyperplanes[i]) || !is_bf16_value(o.hyperplanes[i])) return TC_EINVAL;
    }
    int dev = 0;
    cudaDeviceProp prop;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
        cudaGetLastError();
        return TC_EDEVICE;
    }
    if (prop.major != 10) return TC_EDEVICE;
    if (!get_encoder()) return TC_ECUDA;
    tc_annca_ctx* x = new (std::nothrow) tc_annca_ctx;
    if (!x) return TC_ENOMEM;
    x->H = H;
    x->d = d;
    x->nbits = nbits;
    x->device = dev;
    x->scale = (o.softmax_scale > 0.f) ? o.softmax_scale : (float)(1.0 / std::sqrt((double)d));
    if (o.hyperplanes)
        x->Rhost.assign(o.hyperplanes, o.hyperplanes + (size_t)nbits * d);
    else
        default_hyperplanes(o.seed, nbits * d, x->Rhost);
    std::vector<float> rnorm(nbits);
    for (int b = 0; b < nbits; ++b) {
        double s2 = 0.0;
        for (int i = 0; i < d; ++i) s2 += (double)x->Rhost[(size_t)b * d + i] * x->Rhost[(size_t)b * d + i];
        rnorm[b] = std::nextafter((float)std::sqrt(s2), INFINITY);
    }
    x->Rnorm_host = rnorm;
    AnnView& a = x->a;
    a.H = H;
    a.d = d;
    a.nbits = nbits;
    tc_status st;
    cudaError_t e;
    if ((st = x->grab(x->R, (size_t)nbits * d * 4)) || (st = x->grab(x->Rnorm, (size_t)nbits * 4)) ||
        (st = x->grab(x->stats, sizeof(Stats))) || (st = x->grab(a.kmax2, (size_t)H * 4)) ||
        (st = x->grab(a.zeros, (size_t)H * 4)) ||
        (nbits <= 16 && (st = x->grab(a.ptab, ((size_t)H << nbits) * 4)))) {
        delete x;
        return st;
    }
    if ((e = cudaMemcpy(x->R, x->Rhost.data(), (size_t)nbits * d * 4, cudaMemcpyHostToDevice)) ||
        (e = cudaMemcpy(x->Rnorm, rnorm.data(), (size_t)nbits * 4, cudaMemcpyHostToDevice)) ||
        (e = cudaMemset(x->stats, 0, sizeof(Stats))) || (e = cudaMemset(a.kmax2, 0, (size_t)H * 4)) ||
        (e = cudaMemset(a.zeros, 0, (size_t)H * 4))) {
        delete x;
        return cuda_status(e);
    }
    *out = x;
    return TC_OK;
}

tc_status tc_annca_set_prompt(tc_annca_handle x, const void* Kp, const void* Vp, int32_t L, tc_stream stream) {
    tc_status st = check_call(x);
    if (st) return st;
    if (!Kp || !Vp || !aligned16(Kp) || !aligned16(Vp) || L < 1 || L > kMaxPrompt) return TC_EINVAL;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    AnnView& a = x->a;
    const int64_t Lp = up128(L);
    if (Lp > x->Lcap) {
        if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
        x->free_prompt();
        x->free_slots();   // their row stride follows the prompt's
        const size_t rows = (size_t)x->H * Lp;
        if ((st = x->grab(a.Kh, rows * x->d * 2)) || (st = x->grab(a.Vh, rows * x->d * 2)) ||
            (st = x->grab(a.pcode, rows * 4)) || (st = x->grab(a.pcs, rows * 4)) || (st = x->grab(a.pix, rows * 4)) ||
            (st = x->grab(a.prun, rows * 4))) {
            x->free_prompt();
            x->prompt_set = false;
            return st;
        }
        x->Lcap = Lp;
    }
    a.L = L;
    a.Lp = x->Lcap;   // one row stride for every prompt this allocation holds
    x->last_stream = cs;
    cudaError_t e = cudaMemsetAsync(a.kmax2, 0, (size_t)x->H * 4, cs);
    if (e == cudaSuccess && a.ptab) e = cudaMemsetAsync(a.ptab, 0xff, ((size_t)x->H << x->nbits) * 4, cs);
    if (e == cudaSuccess) e = launch_annca_prompt(a, Kp, Vp, x->R, x->Rnorm, x->stats, cs);
    if (e != cudaSuccess) {
        x->prompt_set = false;
        return cuda_status(e);
    }
    x->prompt_set = true;
    return TC_OK;
}

tc_status tc_annca_attend(tc_annca_handle x, const void* Q, int64_t Tq, int32_t P, void* out, tc_stream stream) {
    tc_status st = check_call(x);
    if (st) return st;
    if (!Q || !out || !aligned16(Q) || !aligned16(out) || P < 1 || Tq < 1 || Tq > ((int64_t)1 << 26) || Tq % P ||
        Tq * x->H >= ((int64_t)1 << 31))   // the kernels index rows t H + h in 32 bits
        return TC_EINVAL;
    const size_t bytes = (size_t)Tq * x->H * x->d * 2;
    const char* q = static_cast<const char*>(Q);
    const char* o = static_cast<const char*>(out);
    if (q < o + bytes && o < q + bytes) return TC_EINVAL;
    if (!x->prompt_set) return TC_ESTATE;
    const int64_t F = Tq / P;
    if ((int64_t)x->H * F > (1 << 30) || F * ((P + 127) / 128) > (1 << 30)) return TC_EINVAL;
    AnnView& a = x->a;
    if (!a.qcode || Tq > a.Tmax) {
        if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
        x->free_queries();
        if ((st = x->grab(a.qcode, (size_t)x->H * Tq * 4))) return st;
        a.Tmax = Tq;
    }
    if ((st = ensure_slots(x, (int64_t)x->H * F))) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    x->last_stream = cs;
    AttnMaps m = x->maps;
    if (!encode3d(&m.q, Q, x->d, x->H, Tq, (uint64_t)x->d * 2, (uint64_t)x->H * x->d * 2, 64, 1, 128))
        return TC_EINVAL;
    cudaError_t e = cudaSuccess;
    if (++a.gen == 0) {   // the stamps wrapped: start them over
        e = cudaMemsetAsync(a.keep, 0, (size_t)a.Zmax * a.Lp * 4, cs);
        a.gen = 1;
    }
    if (e == cudaSuccess)
        e = launch_annca_select(a, Q, Tq, P, (int)F, x->R, x->Rhost.data(), x->Rnorm_host.data(), x->stats, cs);
    if (e == cudaSuccess)
        e = launch_attend_cross_bf16(a, m, Tq, P, (int)F, static_cast<__nv_bfloat16*>(out),
                                     (float)((double)x->scale * 1.4426950408889634), x->stats, cs);
    if (e != cudaSuccess) return cuda_status(e);
    x->last_T = Tq;
    x->last_F = F;
    return TC_OK;
}

tc_status tc_annca_sync(tc_annca_handle x) {
    if (!valid(x)) return TC_EINVAL;
    if (x->sticky != TC_OK) return x->sticky;
    if (cudaStreamSynchronize(x->last_stream) != cudaSuccess) {
        cudaGetLastError();
        x->sticky = TC_ECUDA;
        return x->sticky;
    }
    Stats s{};
    if (cudaMemcpy(&s, x->stats, sizeof(Stats), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        x->sticky = TC_ECUDA;
    } else if (s.error_bits & kErrTimeout) {
        x->sticky = TC_ETIMEOUT;
    }
    return x->sticky;
}

tc_status tc_annca_kept(tc_annca_handle x, int64_t* T_out, int64_t* F_out, int32_t* L_out, int32_t* counts,
                        int32_t* index, uint32_t* qcodes, uint32_t* pcodes) {
    tc_status st = tc_annca_sync(x);
    if (st) return st;
    const AnnView& a = x->a;
    const int64_t F = x->last_F, Z = (int64_t)x->H * F;
    if (T_out) *T_out = x->last_T;
    if (F_out) *F_out = F;
    if (L_out) *L_out = x->prompt_set ? a.L : 0;
    cudaError_t e = cudaSuccess;
    if (counts && Z) e = cudaMemcpy(counts, a.nsel, (size_t)Z * 4, cudaMemcpyDeviceToHost);
    for (int64_t z = 0; index && e == cudaSuccess && z < Z; ++z)
        e = cudaMemcpy(index + z * a.L, a.sidx + z * a.Lp, (size_t)a.L * 4, cudaMemcpyDeviceToHost);
    if (qcodes && e == cudaSuccess && x->last_T) {   // stored token-major, returned head-major
        std::vector<uint32_t> tm((size_t)x->last_T * x->H);
        e = cudaMemcpy(tm.data(), a.qcode, tm.size() * 4, cudaMemcpyDeviceToHost);
        for (int64_t t = 0; e == cudaSuccess && t < x->last_T; ++t)
            for (int h = 0; h < x->H; ++h) qcodes[(int64_t)h * x->last_T + t] = tm[(size_t)t * x->H + h];
    }
    for (int h = 0; pcodes && e == cudaSuccess && h < x->H && x->prompt_set; ++h)
        e = cudaMemcpy(pcodes + (int64_t)h * a.L, a.pcode + (int64_t)h * a.Lp, (size_t)a.L * 4,
                       cudaMemcpyDeviceToHost);
    return cuda_status(e);
}

tc_status tc_annsa_attend(tc_annca_handle x, const void* Q, const void* K, const void* V, int64_t T, void* out,
                          tc_stream stream) {
    tc_status st = check_call(x);
    if (st) return st;
    if (!Q || !K || !V || !out || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || T < 1 ||
        T > kMaxSparseT)
        return TC_EINVAL;
    const size_t bytes = (size_t)T * x->H * x->d * 2;
    const char* o = static_cast<const char*>(out);
    for (const void* in : {Q, K, V}) {
        const char* p = static_cast<const char*>(in);
        if (p < o + bytes && o < p + bytes) return TC_EINVAL;
    }
    if (!x->prompt_set || x->last_T != T) return TC_ESTATE;   // the buckets of this block come from AnnCA
    if (up128(T) > x->sp_Tp) {
        const int64_t Tp = up128(T);
        if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
        x->free_sparse();
        SparseBufs& b = x->sb;
        const size_t rows = (size_t)x->H * Tp;
        if ((st = x->grab(b.perm, rows * 4)) || (st = x->grab(b.grp, rows * 4)) ||
            (st = x->grab(b.tiles, rows / 128 * sizeof(int2))) || (st = x->grab(b.xself, rows * 4)) ||
            (st = x->grab(b.Qs, rows * x->d * 2)) || (st = x->grab(b.Ks, rows * x->d * 2)) ||
            (st = x->grab(b.Vs, rows * x->d * 2)) ||
            (x->nbits <= kSegBits && (st = x->grab(b.bcnt, (size_t)x->H * kOrdBlocks * ((size_t)1 << x->nbits) * 4))) ||
            (!x->sp_kmax2 && (st = x->grab(x->sp_kmax2, (size_t)x->H * 4)))) {
            x->free_sparse();
            return st;
        }
        const uint64_t d = x->d;
        if (!encode3d(&x->sp_maps.q, b.Qs, d, Tp, x->H, d * 2, Tp * d * 2, 64, 128, 1) ||
            !encode3d(&x->sp_maps.kc, b.Ks, d, Tp, x->H, d * 2, Tp * d * 2, 64, 128, 1) ||
            !encode3d(&x->sp_maps.vc, b.Vs, d, Tp, x->H, d * 2, Tp * d * 2, 64, 128, 1)) {
            x->free_sparse();
            return TC_ECUDA;
        }
        x->sp_Tp = Tp;
    }
    const int64_t Tp = x->sp_Tp;   // row stride of the packed arrays (their allocation)
    SparseBufs b = x->sb;
    b.H = x->H;
    b.d = x->d;
    b.T = T;
    b.Tp = Tp;
    b.codes = x->a.qcode;
    b.kmax2 = x->sp_kmax2;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    x->last_stream = cs;
    const float scale_log2 = (float)((double)x->scale * 1.4426950408889634);
    cudaError_t e = launch_annsa_pack(b, x->nbits, Q, K, V, scale_log2, cs);   // (clears the key bounds first)
    if (e == cudaSuccess) {
        SparseArgs sp{b.tiles, b.grp, b.perm, b.xself, Tp, (int)(Tp / 128)};
        e = launch_attend_sparse_bf16(x->H, x->d, sp, x->sp_maps, T, x->sp_kmax2, x->a.zeros,
                                      static_cast<__nv_bfloat16*>(out), scale_log2, x->stats, cs);
    }
    return cuda_status(e);
}

tc_status tc_annca_get_hyperplanes(tc_annca_handle x, float* R) {
    if (!valid(x) || !R) return TC_EINVAL;
    std::memcpy(R, x->Rhost.data(), x->Rhost.size() * sizeof(float));
    return TC_OK;
}

void tc_annca_destroy(tc_annca_handle x) {
    if (!valid(x)) return;
    cudaDeviceSynchronize();
    cudaGetLastError();
    delete x;
}

}  // extern "C"
