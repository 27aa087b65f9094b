// tc_merge_means_noalloc: the merge step of the library (average matched rows into
// running means, add their counts) as a standalone call that allocates nothing.
//
// Who needs it: callers that may not call cudaMalloc after start-up, such as
// inference runtimes that reserve one fixed device arena and forbid later
// allocations, or plugins running inside a framework whose allocator owns all
// device memory. They pass their own input and output buffers; the only other
// memory used is the scratch array below, which is part of the library image.
//
// Scratch: one file-scope device array, kScratchWords 32-bit words (about 3.4 MB)
// on every GPU that loads the library, held until the process exits. Host code
// cannot pass the array's name to a kernel (on the host it is only a stand-in),
// so the first call in each CUDA context looks up the array's device address with
// cudaGetSymbolAddress while that context is current and caches it together with the
// context's unique id; a later call in another context (after cudaDeviceReset, or a
// context the caller made current) looks the address up again. Make the first call
// of a context before any stream capture. Every call shares the array and it keeps
// the last call's contents, so each call first clears the parts that must start at
// zero. Two calls whose work overlaps on the GPU (different streams, or different
// host threads on one device) race on the array and give wrong results.
#include "../../include/tempcache.h"
#include "tc_internal.h"

#include <mutex>

namespace {

constexpr int kMaxSrc = 65536;    // source rows per call
constexpr int kMaxDst = 262144;   // destination rows per call
constexpr int kMaxDevices = 64;
// layout: per-destination merge counts, fill cursors and segment offsets, then the
// touched-destination list and the source-id segments, then one counter
constexpr size_t kScratchWords = 3 * (size_t)kMaxDst + 2 * (size_t)kMaxSrc + 64;

static __device__ __align__(256) int32_t g_merge_scratch[kScratchWords];

struct Scratch {
    int32_t* cnt;      // [n_dst]
    int32_t* fill;     // [n_dst]
    int32_t* off;      // [n_dst]
    int32_t* touched;  // [n_src]
    int32_t* seg;      // [n_src]
    int32_t* ntouched; // [1]
};

Scratch carve(int32_t* base) {
    Scratch s;
    s.cnt = base;
    s.fill = base + kMaxDst;
    s.off = base + 2 * (size_t)kMaxDst;
    s.touched = base + 3 * (size_t)kMaxDst;
    s.seg = s.touched + kMaxSrc;
    s.ntouched = s.seg + kMaxSrc;
    return s;
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

std::mutex g_mu;
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
struct CachedAddr {
    unsigned long long ctx_id;   // unique id of the context the address belongs to (0: none yet)
    int32_t* addr;
};
CachedAddr g_addr[kMaxDevices] = {};

// Device address of the scratch array in the current context of device `dev`, looked
// up once per context: a context id that differs from the cached one (the device was
// reset, or the caller made another context current) triggers a new lookup.
cudaError_t scratch_address(int dev, int32_t** out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ctx_current || !g_ctx_id) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || !f1 ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess || !f2)
            return cudaErrorNotSupported;
        g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        g_ctx_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    // The context the runtime works in is the thread's current one (the caller's own,
    // or the device's primary context); with none current yet, the runtime makes the
    // primary context current on its first call, here cudaGetSymbolAddress.
    CUcontext ctx = nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    void* fresh = nullptr;
    if (!ctx) {
        cudaError_t e = cudaGetSymbolAddress(&fresh, g_merge_scratch);
        if (e != cudaSuccess) return e;
        if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
    }
    unsigned long long id = 0;
    if (g_ctx_id(ctx, &id) != CUDA_SUCCESS || id == 0) return cudaErrorDeviceUninitialized;
    if (g_addr[dev].ctx_id != id || !g_addr[dev].addr) {
        if (!fresh) {
            cudaError_t e = cudaGetSymbolAddress(&fresh, g_merge_scratch);
            if (e != cudaSuccess) return e;
        }
        g_addr[dev] = CachedAddr{id, static_cast<int32_t*>(fresh)};
    }
    *out = g_addr[dev].addr;
    return cudaSuccess;
}

__global__ void na_count(const int32_t* __restrict__ target, int n_src, int n_dst, Scratch s) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_src; i += gridDim.x * blockDim.x) {
        const int j = target[i];
        if (j < 0 || j >= n_dst) continue;
        if (atomicAdd(&s.cnt[j], 1) == 0) s.touched[atomicAdd(s.ntouched, 1)] = j;
    }
}

__device__ int na_block_exclusive_scan(int v, int* total) {
    __shared__ int wsum[32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    int inc = v;
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) wsum[w] = inc;
    __syncthreads();
    if (w == 0) {
        int x = (lane < nw) ? wsum[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += n;
        }
        wsum[lane] = x;
    }
    __syncthreads();
    const int before = (w > 0) ? wsum[w - 1] : 0;
    *total = wsum[nw - 1];
    __syncthreads();
    return before + inc - v;
}

// One block: each touched destination gets a contiguous range of seg[].
__global__ void __launch_bounds__(1024) na_offsets(Scratch s) {
    const int ns = *s.ntouched, nt = blockDim.x;
    const int per = (ns + nt - 1) / nt;
    const int q0 = min(ns, (int)threadIdx.x * per), q1 = min(ns, q0 + per);
    int c = 0;
    for (int q = q0; q < q1; ++q) c += s.cnt[s.touched[q]];
    int total = 0;
    int off = na_block_exclusive_scan(c, &total);
    for (int q = q0; q < q1; ++q) {
        const int j = s.touched[q];
        s.off[j] = off;
        off += s.cnt[j];
    }
}

__global__ void na_scatter(const int32_t* __restrict__ target, int n_src, int n_dst, Scratch s) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_src; i += gridDim.x * blockDim.x) {
        const int j = target[i];
        if (j < 0 || j >= n_dst) continue;
        s.seg[s.off[j] + atomicAdd(&s.fill[j], 1)] = i;
    }
}

template <typename E, int D>
__device__ __forceinline__ void na_load_row(const E* row, int lane, float (&x)[D / 32]) {
#pragma unroll
    for (int e = 0; e < D / 32; ++e) {
        if constexpr (sizeof(E) == 2)
            x[e] = __bfloat162float(row[lane * (D / 32) + e]);
        else
            x[e] = row[lane * (D / 32) + e];
    }
}

// One warp per touched destination: sum its sources in ascending source index in
// fp32, then mean <- (n mean + sum) / (n + m), count <- n + m (mean <- sum / m when
// n = 0, so a row that was never written does not matter). The warp puts the sources
// of its destination in ascending order: up to 32 in its lanes, up to kSortSmem in its
// own shared-memory buffer (each id placed at its rank), and beyond that it visits
// them by scanning target[] in source order, one 32-source window per ballot.
constexpr int kMergeWarps = 8;
constexpr int kSortSmem = 256;

template <typename E, int D>
__global__ void __launch_bounds__(kMergeWarps * 32) na_merge(const E* __restrict__ src,
                                                            const int32_t* __restrict__ target, int n_src,
                                                            float* __restrict__ mean, int32_t* __restrict__ count,
                                                            Scratch s) {
    constexpr int EPL = D / 32;
    __shared__ int32_t sIds[kMergeWarps][kSortSmem];
    __shared__ int32_t sSorted[kMergeWarps][kSortSmem];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int ns = *s.ntouched;
    for (int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < ns; w += (gridDim.x * blockDim.x) >> 5) {
        const int j = s.touched[w];
        const int m = s.cnt[j], off = s.off[j];
        float acc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        auto add_row = [&](int i) {
            float v[EPL];
            na_load_row<E, D>(src + (size_t)i * D, lane, v);
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = __fadd_rn(acc[e], v[e]);
        };
        if (m <= 32) {
            const int id = (lane < m) ? s.seg[off + lane] : 0x7fffffff;
            int rank = 0;
            for (int k = 0; k < 32; ++k) rank += (__shfl_sync(0xffffffffu, id, k) < id);
            for (int q = 0; q < m; ++q) {
                const int srcl = __ffs(__ballot_sync(0xffffffffu, rank == q)) - 1;
                add_row(__shfl_sync(0xffffffffu, id, srcl));
            }
        } else if (m <= kSortSmem) {
            for (int p = lane; p < m; p += 32) sIds[wib][p] = s.seg[off + p];
            __syncwarp();
            for (int p = lane; p < m; p += 32) {
                const int mine = sIds[wib][p];
                int rank = 0;
                for (int k = 0; k < m; ++k) rank += (sIds[wib][k] < mine);
                sSorted[wib][rank] = mine;   // ids are distinct: ranks are a permutation
            }
            __syncwarp();
            for (int q = 0; q < m; ++q) add_row(sSorted[wib][q]);
            __syncwarp();   // the buffers are reused by this warp's next destination
        } else {
            for (int i0 = 0; i0 < n_src; i0 += 32) {
                const bool hit = i0 + lane < n_src && target[i0 + lane] == j;
                unsigned b = __ballot_sync(0xffffffffu, hit);
                while (b) {
                    const int k = __ffs(b) - 1;
                    b &= b - 1;
                    add_row(i0 + k);
                }
            }
        }
        const int nold = count[j];
        const float fn = (float)nold, ft = (float)(nold + m);
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            float* p = mean + (size_t)j * D + lane * EPL + e;
            *p = nold == 0 ? __fdiv_rn(acc[e], ft) : __fdiv_rn(__fadd_rn(__fmul_rn(fn, *p), acc[e]), ft);
        }
        if (lane == 0) count[j] = nold + m;
    }
}

template <typename E, int D>
cudaError_t run(const void* src, const int32_t* target, int n_src, float* mean, int32_t* count, int n_dst,
                const Scratch& s, cudaStream_t st) {
    const int gs = (n_src + 255) / 256 > 1184 ? 1184 : (n_src + 255) / 256;
    na_count<<<gs, 256, 0, st>>>(target, n_src, n_dst, s);
    na_offsets<<<1, 1024, 0, st>>>(s);
    na_scatter<<<gs, 256, 0, st>>>(target, n_src, n_dst, s);
    const int gm = (n_src + kMergeWarps - 1) / kMergeWarps > 1184 ? 1184 : (n_src + kMergeWarps - 1) / kMergeWarps;
    na_merge<E, D><<<gm, kMergeWarps * 32, 0, st>>>(reinterpret_cast<const E*>(src), target, n_src, mean, count, s);
    return cudaGetLastError();
}

}  // namespace

extern "C" tc_status tc_merge_means_noalloc(const void* src, tc_dtype src_dtype, const int32_t* target,
                                            int32_t n_src, int32_t d, float* mean, int32_t* count, int32_t n_dst,
                                            tc_stream stream) {
    if (!src || !target || !mean || !count || (d != 64 && d != 128) ||
        (src_dtype != TC_BF16 && src_dtype != TC_F32) || n_src < 1 || n_dst < 1)
        return TC_EINVAL;
    if (n_src > kMaxSrc || n_dst > kMaxDst) return TC_EINVAL;  // beyond the fixed scratch
    // The inputs must not overlap the rows the call writes.
    const size_t esz = src_dtype == TC_BF16 ? 2 : 4;
    auto overlap = [](const void* a, size_t na, const void* b, size_t nb) {
        const char* x = static_cast<const char*>(a);
        const char* y = static_cast<const char*>(b);
        return x < y + nb && y < x + na;
    };
    const size_t src_b = (size_t)n_src * d * esz, tgt_b = (size_t)n_src * 4;
    const size_t mean_b = (size_t)n_dst * d * 4, cnt_b = (size_t)n_dst * 4;
    if (overlap(src, src_b, mean, mean_b) || overlap(src, src_b, count, cnt_b) || overlap(target, tgt_b, mean, mean_b) ||
        overlap(target, tgt_b, count, cnt_b) || overlap(mean, mean_b, count, cnt_b))
        return TC_EINVAL;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return TC_EDEVICE;
    }
    int32_t* base = nullptr;
    if (scratch_address(dev, &base) != cudaSuccess) {
        cudaGetLastError();
        return TC_ECUDA;
    }
    const Scratch s = carve(base);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: clear the counts, cursors and
    // the touched counter this call relies on starting at zero.
    cudaError_t e = cudaMemsetAsync(s.cnt, 0, sizeof(int32_t) * (size_t)n_dst, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(s.fill, 0, sizeof(int32_t) * (size_t)n_dst, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(s.ntouched, 0, sizeof(int32_t), st);
    if (e == cudaSuccess) {
        if (src_dtype == TC_BF16)
            e = d == 128 ? run<__nv_bfloat16, 128>(src, target, n_src, mean, count, n_dst, s, st)
                         : run<__nv_bfloat16, 64>(src, target, n_src, mean, count, n_dst, s, st);
        else
            e = d == 128 ? run<float, 128>(src, target, n_src, mean, count, n_dst, s, st)
                         : run<float, 64>(src, target, n_src, mean, count, n_dst, s, st);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return TC_ECUDA;
    }
    return TC_OK;
}
