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
// so the first call on each device looks up its device address with
// cudaGetSymbolAddress while that device is current and caches it; make that first
// call before any stream capture. Every call shares the array and it keeps the last
// call's contents, so each call first clears the parts that must start at zero.
// Two calls whose work overlaps on the GPU (different streams, or different host
// threads on one device) race on the array and give wrong results.
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

std::mutex g_mu;
int32_t* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t scratch_address(int dev, int32_t** out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_merge_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = static_cast<int32_t*>(p);
    }
    *out = g_addr[dev];
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
// fp32, then mean <- (n mean + sum) / (n + m), count <- n + m.
template <typename E, int D>
__global__ void __launch_bounds__(256) na_merge(const E* __restrict__ src, float* __restrict__ mean,
                                                int32_t* __restrict__ count, Scratch s) {
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const int ns = *s.ntouched;
    for (int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < ns; w += (gridDim.x * blockDim.x) >> 5) {
        const int j = s.touched[w];
        const int m = s.cnt[j], off = s.off[j];
        float acc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        if (m <= 32) {
            const int id = (lane < m) ? s.seg[off + lane] : 0x7fffffff;
            int rank = 0;
            for (int k = 0; k < 32; ++k) rank += (__shfl_sync(0xffffffffu, id, k) < id);
            for (int q = 0; q < m; ++q) {
                const int srcl = __ffs(__ballot_sync(0xffffffffu, rank == q)) - 1;
                const int i = __shfl_sync(0xffffffffu, id, srcl);
                float v[EPL];
                na_load_row<E, D>(src + (size_t)i * D, lane, v);
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[e] = __fadd_rn(acc[e], v[e]);
            }
        } else {
            int last = -1;
            for (int q = 0; q < m; ++q) {
                int mn = 0x7fffffff;
                for (int p = lane; p < m; p += 32) {
                    const int id = s.seg[off + p];
                    if (id > last && id < mn) mn = id;
                }
                for (int o = 16; o > 0; o >>= 1) mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                float v[EPL];
                na_load_row<E, D>(src + (size_t)mn * D, lane, v);
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[e] = __fadd_rn(acc[e], v[e]);
                last = mn;
            }
        }
        const int nold = count[j];
        const float fn = (float)nold, ft = (float)(nold + m);
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            float* p = mean + (size_t)j * D + lane * EPL + e;
            *p = __fdiv_rn(__fadd_rn(__fmul_rn(fn, *p), acc[e]), ft);
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
    const int gm = (n_src + 7) / 8 > 1184 ? 1184 : (n_src + 7) / 8;
    na_merge<E, D><<<gm, 256, 0, st>>>(reinterpret_cast<const E*>(src), mean, count, s);
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
