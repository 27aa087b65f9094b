// Biased attention in fp32 (handles with fp32 storage).
//
// Same result as the tensor-core kernel: out_t = softmax_j(scale <q_t,k_j> + b_j) v
// over the committed entries (b_j = ln n_j, FAST-AR technical summary section 2.A,
// Lemma 5.1) and the staged chunk (b_j = 0), evaluated in base 2 in fp32.
//
// A block holds 8 warps = 8 query rows of one head. Keys and values stream through
// shared memory 32 at a time; lane k of a warp scores key k of the tile against its
// row, then the warp folds the tile into its online softmax and accumulates P V.
#include "tc_internal.h"

#include <math.h>

namespace tc {

namespace {

constexpr int kRows = 8;
constexpr int kTK = 32;

__device__ __forceinline__ float wmax(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float wsum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int D>
__global__ void __launch_bounds__(kRows * 32)
attend_f32_kernel(CacheView c, StageView s, const float* __restrict__ Q, int64_t Tq, float* __restrict__ out,
                  float scale_log2) {
    constexpr int EPL = D / 32;
    __shared__ float sK[kTK][D + 1];
    __shared__ float sV[kTK][D];
    __shared__ float sB[kTK];
    __shared__ float sQ[kRows][D];
    const int h = blockIdx.y;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * kRows + w;
    const bool active = row < Tq;
    const int H = c.H;
    for (int i = lane; i < D; i += 32) sQ[w][i] = active ? Q[(row * H + h) * D + i] : 0.f;
    const int Mh = c.M[h];
    const int64_t L = (int64_t)Mh + s.T;
    const float* Kc = reinterpret_cast<const float*>(c.Kc) + (int64_t)h * c.capP * D;
    const float* Vc = reinterpret_cast<const float*>(c.Vc) + (int64_t)h * c.capP * D;
    const float* Ks = reinterpret_cast<const float*>(s.Ks) + (int64_t)h * s.TmaxP * D;
    const float* Vs = reinterpret_cast<const float*>(s.Vs) + (int64_t)h * s.TmaxP * D;
    const float* b2 = c.bias2 + (int64_t)h * c.capP;
    float m = -INFINITY, l = 0.f, o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    for (int64_t j0 = 0; j0 < L; j0 += kTK) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kTK * D; idx += blockDim.x) {
            const int k = idx / D, i = idx % D;
            const int64_t j = j0 + k;
            float kv = 0.f, vv = 0.f;
            if (j < Mh) {
                kv = Kc[j * D + i];
                vv = Vc[j * D + i];
            } else if (j < L) {
                kv = Ks[(j - Mh) * D + i];
                vv = Vs[(j - Mh) * D + i];
            }
            sK[k][i] = kv;
            sV[k][i] = vv;
        }
        if (threadIdx.x < kTK) {
            const int64_t j = j0 + threadIdx.x;
            sB[threadIdx.x] = (j < Mh) ? b2[j] : ((j < L) ? 0.f : -INFINITY);
        }
        __syncthreads();
        float dot = 0.f;
#pragma unroll 8
        for (int i = 0; i < D; ++i) dot = fmaf(sQ[w][i], sK[lane][i], dot);
        const float x = fmaf(dot, scale_log2, sB[lane]);
        const float mt = wmax(x);
        const float mn = fmaxf(m, mt);
        const float corr = (m == -INFINITY) ? 0.f : exp2f(m - mn);
        const float p = exp2f(x - mn);
        l = l * corr + wsum(p);
        m = mn;
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[e] *= corr;
        for (int k = 0; k < kTK; ++k) {
            const float pk = __shfl_sync(0xffffffffu, p, k);
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[e] = fmaf(pk, sV[k][lane * EPL + e], o[e]);
        }
    }
    if (active) {
        const float inv = 1.f / l;
#pragma unroll
        for (int e = 0; e < EPL; ++e) out[(row * H + h) * D + lane * EPL + e] = o[e] * inv;
    }
}

}  // namespace

cudaError_t launch_attend_f32(const CacheView& c, const StageView& s, const float* Q, int64_t Tq, float* out,
                              float scale_log2, cudaStream_t st) {
    dim3 grid((unsigned)((Tq + kRows - 1) / kRows), (unsigned)c.H);
    if (c.d == 128)
        attend_f32_kernel<128><<<grid, kRows * 32, 0, st>>>(c, s, Q, Tq, out, scale_log2);
    else
        attend_f32_kernel<64><<<grid, kRows * 32, 0, st>>>(c, s, Q, Tq, out, scale_log2);
    return cudaGetLastError();
}

}  // namespace tc
