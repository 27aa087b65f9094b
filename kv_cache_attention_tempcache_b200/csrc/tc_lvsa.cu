// LVSA frame mask: query frame t attends only to the frames A(t) = G u W(t), with G the
// rotating global frames of the denoising step and W(t) a local window around t that is
// extended over the global frames it overlaps until t attends to C frames.
//
// LVSA technical summary, section 2 "Metodologia: Long Video Sparse Attention",
// "Mecanismo Central": G is a periodic set of global frames shifted by s mod T_per at
// step s (over T_per consecutive steps every frame is a global frame exactly once); the
// local window is extended when it overlaps global frames so that |A(t)| stays near the
// budget C. Here G_s = { g : g = s (mod T_per) }, and W(t) grows from {t} one frame at a
// time, on the side with fewer frames added so far (right first on a tie; the other side
// at the video's edge), until |G_s u W(t)| >= C or it covers every frame.
//
// Kernels: lvsa_tiles_kernel (one thread per query frame) builds A(t) and the list of
// token-major key tiles covering it (each run of consecutive frames tiled from its first
// row); lvsa_kbound_kernel bounds |k|^2 per head over the call's keys; the attention
// kernel of tc_attn_bf16.cu in its frame mode then runs each query frame's rows against its
// tiles, rows past a run's end shifted by -inf, with the fixed softmax reference whenever
// the rows' logit bounds allow it.
#include "../../include/tempcache.h"
#include "tc_internal.h"

#include <algorithm>
#include <cmath>
#include <new>

namespace tc {

namespace {

__global__ void lvsa_masktab_kernel(float* tab) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < 129 * 128; i += gridDim.x * blockDim.x)
        tab[i] = ((i & 127) < (i >> 7)) ? 0.f : -INFINITY;
}

// One thread per query frame t.
__global__ void lvsa_tiles_kernel(int T, int P, int T_per, int C, int s, int maxt, int2* tiles, int32_t* count,
                                  int32_t* nframes, int32_t* frames) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const int sm = s % T_per;
    auto anchor = [&](int f) { return f % T_per == sm; };
    const int nG = sm < T ? (T - 1 - sm) / T_per + 1 : 0;
    int size = nG + (anchor(t) ? 0 : 1);   // |G u W| with W = {t}
    int lo = t, hi = t, left = 0, right = 0;
    while (size < C && (lo > 0 || hi < T - 1)) {
        if (hi < T - 1 && (right <= left || lo == 0)) {
            ++hi;
            ++right;
            if (!anchor(hi)) ++size;
        } else {
            --lo;
            ++left;
            if (!anchor(lo)) ++size;
        }
    }
    int n = 0, nt = 0, run = -1;
    for (int f = 0; f <= T; ++f) {
        const bool in = f < T && (anchor(f) || (lo <= f && f <= hi));
        if (in) {
            frames[(int64_t)t * T + n++] = f;
            if (run < 0) run = f;
        } else if (run >= 0) {   // frames [run, f) : token rows [run P, f P)
            const int64_t end = (int64_t)f * P;
            for (int64_t r0 = (int64_t)run * P; r0 < end && nt < maxt; r0 += 128)
                tiles[(int64_t)t * maxt + nt++] = make_int2((int)r0, (int)(end - r0 < 128 ? end - r0 : 128));
            run = -1;
        }
    }
    count[t] = nt;
    nframes[t] = n;
}

// Upper bound of |k|^2 per head over the keys K [N, H, d] (bf16), rounded up past the fp32
// sums' error: the attention kernel's fixed softmax reference needs it. Each block takes one
// contiguous range of rows r = n H + h (W = d / 8 lanes per row) and gathers its heads'
// maxima in shared memory, one atomic per head and block.
template <int D>
__global__ void __launch_bounds__(256) lvsa_kbound_kernel(const __nv_bfloat16* __restrict__ K, int64_t rows, int H,
                                                          float* kmax2) {
    constexpr int W = D / 8, RPW = 32 / W, kSlots = 64;
    __shared__ float sK[kSlots];
    for (int i = threadIdx.x; i < kSlots; i += blockDim.x) sK[i] = 0.f;
    __syncthreads();
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5, sub = lane / W, w = lane % W;
    const int64_t per = ((rows + gridDim.x - 1) / gridDim.x + RPW - 1) / RPW * RPW;
    const int64_t r0 = (int64_t)blockIdx.x * per, r1 = min(rows, r0 + per);
    const uint4* K4 = reinterpret_cast<const uint4*>(K);
    for (int64_t rr = r0 + (int64_t)wib * RPW; rr < r1; rr += (int64_t)(blockDim.x >> 5) * RPW) {   // warp-uniform
        const int64_t r = rr + sub;
        float kk = 0.f;
        if (r < r1) {
            const uint4 v = K4[r * W + w];
            const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(wd[e] << 16), hi = __uint_as_float(wd[e] & 0xffff0000u);
                kk = fmaf(lo, lo, fmaf(hi, hi, kk));
            }
        }
#pragma unroll
        for (int o = 1; o < W; o <<= 1) kk += __shfl_xor_sync(0xffffffffu, kk, o);
        if (r < r1 && w == 0) {
            const int h = (int)(r % H);
            const float kb = kk * (1.f + 1.f / 1024.f);   // floats >= 0 order like their bits
            if (h < kSlots) atomicMax(reinterpret_cast<int*>(sK + h), __float_as_int(kb));
            else atomicMax(reinterpret_cast<int*>(kmax2 + h), __float_as_int(kb));
        }
    }
    __syncthreads();
    for (int h = threadIdx.x; h < H && h < kSlots; h += blockDim.x)
        if (sK[h] > 0.f) atomicMax(reinterpret_cast<int*>(kmax2 + h), __float_as_int(sK[h]));
}

}  // namespace

}  // namespace tc

using namespace tc;

namespace {

constexpr uint32_t kLvsaMagic = 0x7c7cf5a1u;

}  // namespace

struct tc_lvsa_ctx {
    uint32_t magic = kLvsaMagic;
    int H = 0, d = 0, P = 0, T_per = 0, C = 0;
    float scale = 0.f;
    int device = 0;
    float* masktab = nullptr;   // [129][128]
    float* consts = nullptr;    // [0, H) = 0
    float* kmax2 = nullptr;     // [H] bound of |k|^2 per head of the last call's keys
    Stats* stats = nullptr;
    int Tcap = 0, maxt = 0;     // frames the tables hold, tiles per frame
    int2* tiles = nullptr;
    int32_t* count = nullptr;
    int32_t* nframes = nullptr;
    int32_t* frames = nullptr;
    int last_T = 0;
    cudaStream_t last_stream = nullptr;
    tc_status sticky = TC_OK;

    void free_tables() {
        void* ps[] = {tiles, count, nframes, frames};
        for (void* p : ps) if (p) cudaFree(p);
        tiles = nullptr;
        count = nframes = frames = nullptr;
        Tcap = maxt = 0;
    }
    ~tc_lvsa_ctx() {
        free_tables();
        void* ps[] = {masktab, consts, kmax2, stats};
        for (void* p : ps) if (p) cudaFree(p);
        magic = 0;
    }
};

namespace {

bool valid(tc_lvsa_handle h) { return h != nullptr && h->magic == kLvsaMagic; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tc_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return TC_OK;
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? TC_ENOMEM : TC_ECUDA;
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

}  // namespace

extern "C" {

tc_status tc_lvsa_create(int32_t H, int32_t d, int32_t P, int32_t T_per, int32_t C, float softmax_scale,
                         tc_lvsa_handle* out) {
    if (!out) return TC_EINVAL;
    *out = nullptr;
    if (H < 1 || H > 4096 || (d != 64 && d != 128) || P < 1 || T_per < 1 || C < 1 || !(softmax_scale >= 0.f) ||
        !std::isfinite(softmax_scale))
        return TC_EINVAL;
    int dev = 0;
    cudaDeviceProp prop;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
        cudaGetLastError();
        return TC_EDEVICE;
    }
    if (prop.major != 10) return TC_EDEVICE;
    if (!get_encoder()) return TC_ECUDA;
    tc_lvsa_ctx* x = new (std::nothrow) tc_lvsa_ctx;
    if (!x) return TC_ENOMEM;
    x->H = H;
    x->d = d;
    x->P = P;
    x->T_per = T_per;
    x->C = C;
    x->device = dev;
    x->scale = softmax_scale > 0.f ? softmax_scale : (float)(1.0 / std::sqrt((double)d));
    tc_status st;
    if ((st = grab(x->masktab, 129 * 128 * 4)) || (st = grab(x->consts, (size_t)H * 4)) ||
        (st = grab(x->kmax2, (size_t)H * 4)) ||
        (st = grab(x->stats, sizeof(Stats)))) {
        delete x;
        return st;
    }
    std::vector<float> c((size_t)H, 0.f);
    cudaError_t e;
    if ((e = cudaMemcpy(x->consts, c.data(), c.size() * 4, cudaMemcpyHostToDevice)) ||
        (e = cudaMemset(x->stats, 0, sizeof(Stats)))) {
        delete x;
        return cuda_status(e);
    }
    lvsa_masktab_kernel<<<16, 256>>>(x->masktab);
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) {
        delete x;
        return cuda_status(e);
    }
    *out = x;
    return TC_OK;
}

tc_status tc_lvsa_attend(tc_lvsa_handle x, const void* Q, const void* K, const void* V, int32_t T, int32_t step,
                         void* out, tc_stream stream) {
    if (!valid(x)) return TC_EINVAL;
    if (x->sticky != TC_OK) return x->sticky;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != x->device) {
        cudaGetLastError();
        return TC_EDEVICE;
    }
    if (!Q || !K || !V || !out || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || T < 1 ||
        step < 0)
        return TC_EINVAL;
    const int64_t N = (int64_t)T * x->P;
    if (N * x->H >= ((int64_t)1 << 31) || (int64_t)T * ((x->P + 127) / 128) >= ((int64_t)1 << 31)) return TC_EINVAL;
    const size_t bytes = (size_t)N * x->H * x->d * 2;
    const char* o = static_cast<const char*>(out);
    for (const void* in : {Q, K, V}) {
        const char* p = static_cast<const char*>(in);
        if (p < o + bytes && o < p + bytes) return TC_EINVAL;
    }
    tc_status st;
    if (T > x->Tcap) {
        if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
        x->free_tables();
        const int maxt = (int)((N + 127) / 128) + T;
        if ((st = grab(x->tiles, (size_t)T * maxt * sizeof(int2))) || (st = grab(x->count, (size_t)T * 4)) ||
            (st = grab(x->nframes, (size_t)T * 4)) || (st = grab(x->frames, (size_t)T * T * 4))) {
            x->free_tables();
            return st;
        }
        x->Tcap = T;
        x->maxt = maxt;
    }
    // (a smaller T reuses the tables: maxt only needs to cover this call's tiles)
    AttnMaps m{};
    const uint64_t d = x->d, H = x->H;
    if (!encode3d(&m.q, Q, d, H, N, d * 2, H * d * 2, 64, 1, 128) ||
        !encode3d(&m.kc, K, d, H, N, d * 2, H * d * 2, 64, 1, 128) ||
        !encode3d(&m.vc, V, d, H, N, d * 2, H * d * 2, 64, 1, 128))
        return TC_EINVAL;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    x->last_stream = cs;
    lvsa_tiles_kernel<<<(T + 127) / 128, 128, 0, cs>>>(T, x->P, x->T_per, x->C, step, x->maxt, x->tiles, x->count,
                                                       x->nframes, x->frames);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaMemsetAsync(x->kmax2, 0, (size_t)x->H * 4, cs);
    if (e == cudaSuccess) {
        const int64_t rows = N * x->H;
        const int rpb = 8 * (32 / (x->d / 8));   // rows a 256-thread block takes per step
        int grid = (int)std::min<int64_t>((rows + rpb - 1) / rpb, 148 * 8);
        if (x->d == 128)
            lvsa_kbound_kernel<128><<<grid, 256, 0, cs>>>(static_cast<const __nv_bfloat16*>(K), rows, x->H, x->kmax2);
        else
            lvsa_kbound_kernel<64><<<grid, 256, 0, cs>>>(static_cast<const __nv_bfloat16*>(K), rows, x->H, x->kmax2);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        FrameArgs fa{x->tiles, x->count, x->masktab, x->maxt};
        e = launch_attend_frames_bf16(x->H, x->d, fa, m, T, x->P, x->kmax2, x->consts,
                                      static_cast<__nv_bfloat16*>(out),
                                      (float)((double)x->scale * 1.4426950408889634), x->stats, cs);
    }
    if (e != cudaSuccess) return cuda_status(e);
    x->last_T = T;
    return TC_OK;
}

tc_status tc_lvsa_frames(tc_lvsa_handle x, int32_t* T_out, int32_t* nframes, int32_t* frames) {
    if (!valid(x)) return TC_EINVAL;
    if (cudaStreamSynchronize(x->last_stream) != cudaSuccess) {
        cudaGetLastError();
        return TC_ECUDA;
    }
    if (T_out) *T_out = x->last_T;
    cudaError_t e = cudaSuccess;
    if (nframes && x->last_T) e = cudaMemcpy(nframes, x->nframes, (size_t)x->last_T * 4, cudaMemcpyDeviceToHost);
    for (int t = 0; frames && e == cudaSuccess && t < x->last_T; ++t)
        e = cudaMemcpy(frames + (int64_t)t * x->last_T, x->frames + (int64_t)t * x->last_T, (size_t)x->last_T * 4,
                       cudaMemcpyDeviceToHost);
    return cuda_status(e);
}

tc_status tc_lvsa_sync(tc_lvsa_handle x) {
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

void tc_lvsa_destroy(tc_lvsa_handle x) {
    if (!valid(x)) return;
    cudaDeviceSynchronize();
    cudaGetLastError();
    delete x;
}

}  // extern "C"
