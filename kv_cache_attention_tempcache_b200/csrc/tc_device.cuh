// Device helpers shared by the kernels of the library: row loads of bf16/fp32
// rows spread over a warp, warp reductions, and programmatic dependent launch.
#pragma once

#include "tc_internal.h"

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

constexpr int kWarps = 8;  // warps per block of the warp-per-row kernels

// Programmatic dependent launch: each commit kernel may be scheduled while its
// predecessor in the stream finishes; it waits here for the predecessor's memory, and
// lets its own successor be scheduled once every block has passed its main loop.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_smem(void (*kern)(KArgs...), int grid, int block, int smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)block);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int block, cudaStream_t st, Args... args) {
    return launch_pdl_smem(kern, grid, block, 0, st, args...);
}

inline int grid_for_rows(int64_t rows, int per_block, int max_blocks) {
    int64_t b = (rows + per_block - 1) / per_block;
    if (b < 1) b = 1;
    if (b > max_blocks) b = max_blocks;
    return (int)b;
}

// v[0..NBP) summed over the warp's 32 lanes; lane l ends with the total of slot
// l mod NBP in v[0]. The first NBP-1 shuffles halve the vector (slot bit s-1 decided
// by lane bit s-1, and so on down), the remaining lane bits are plain sums.
template <int NBP>
__device__ __forceinline__ float reduce_scatter(float (&v)[NBP], int lane) {
#pragma unroll
    for (int o = NBP / 2, L = NBP; o >= 1; o >>= 1, L >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int k = 0; k < L / 2; ++k) {
            const float send = up ? v[k] : v[k + L / 2];
            const float keep = up ? v[k + L / 2] : v[k];
            v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
#pragma unroll
    for (int o = NBP; o < 32; o <<= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    return v[0];
}

__device__ __forceinline__ uint32_t pack_bf16_exact(float lo, float hi) {
    return (__float_as_uint(lo) >> 16) | (__float_as_uint(hi) & 0xffff0000u);
}

}  // namespace

}  // namespace tc
