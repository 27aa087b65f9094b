// Host runtime of the TempCache C ABI (include/tempcache.h): handle lifetime,
// argument checks, device memory, staging, tensor maps, and the launch sequence of
// the commit and attention kernels. All compute happens in the kernels.
#include "../../include/tempcache.h"
#include "tc_internal.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

namespace tc {

// ---- allocation with host-side fault injection (TC_FAULT_ALLOC_AT=n fails the
// n-th allocation of the process, counting from 1), used by the failure tests.
std::atomic<int> g_alloc_calls{0};   // handles may be created from several host threads

cudaError_t dev_alloc(void** p, size_t bytes) {
    const int call = ++g_alloc_calls;
    const char* f = std::getenv("TC_FAULT_ALLOC_AT");
    if (f && std::atoi(f) == call) {
        *p = nullptr;
        return cudaErrorMemoryAllocation;
    }
    return cudaMalloc(p, bytes < 16 ? 16 : bytes);
}

// ---- bf16 rounding (round to nearest, ties to even) of a finite float
float round_bf16(float x) {
    uint32_t u;
    std::memcpy(&u, &x, 4);
    const uint32_t lsb = (u >> 16) & 1u;
    u = (u + 0x7fffu + lsb) & 0xffff0000u;
    float y;
    std::memcpy(&y, &u, 4);
    return y;
}

bool is_bf16_value(float x) {
    uint32_t u;
    std::memcpy(&u, &x, 4);
    return (u & 0xffffu) == 0u;
}

// Default hyperplanes: N(0,1) draws rounded to bf16. Uniforms from SplitMix64
// (Steele, Lea and Flood, 2014) turned into normals by the Box-Muller transform.
void default_hyperplanes(uint64_t seed, int n, std::vector<float>& out) {
    uint64_t state = seed ^ 0x5eed7c0de5ca1ab1ull;
    auto next = [&]() {
        uint64_t z = (state += 0x9e3779b97f4a7c15ull);
        z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
        z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
        return z ^ (z >> 31);
    };
    auto uniform = [&]() { return ((next() >> 11) + 0.5) * (1.0 / 9007199254740992.0); };  // (0,1)
    out.resize(n);
    for (int i = 0; i < n; i += 2) {
        const double u1 = uniform(), u2 = uniform();
        const double r = std::sqrt(-2.0 * std::log(u1));
        out[i] = round_bf16((float)(r * std::cos(2.0 * M_PI * u2)));
        if (i + 1 < n) out[i + 1] = round_bf16((float)(r * std::sin(2.0 * M_PI * u2)));
    }
}

// cuTensorMapEncodeTiled, fetched through the runtime so the library needs no
// link-time dependency on the driver library.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool get_encoder() {
    if (g_encode) return true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return false;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    return true;
}

// 3-D bf16 map with a 128-byte swizzle; dims/strides innermost first, strides in bytes.
bool encode3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
              uint32_t b0, uint32_t b1, uint32_t b2) {
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {s1, s2};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t es[3] = {1, 1, 1};
    return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

using namespace tc;

namespace {

constexpr uint32_t kMagic = 0x7c7ca5e1u;

inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// p[h * stride + i] = v for i < n, h < rows (one launch over all heads).
__global__ void fill_f32(float* p, int64_t n, int rows, int64_t stride, float v) {
    for (int h = blockIdx.y; h < rows; h += gridDim.y)
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
            p[(int64_t)h * stride + i] = v;
}

}  // namespace

struct tc_ctx {
    uint32_t magic = kMagic;
    int H = 0, d = 0, nbits = 0, esize = 2;
    float tau = 0.f, scale = 0.f;
    tc_dtype dtype = TC_BF16;
    bool intra = false;            // commits also match inside the chunk
    bool mean = false;             // entry keys are running means of their members' keys
    int32_t* claim = nullptr;      // [H << nbits] bucket claims of the re-bucketing (running-mean keys)
    int64_t capacity = 0, capP = 0;
    int device = 0;
    CacheView c{};
    StageView s{};
    int32_t* ctr = nullptr;
    Stats* stats = nullptr;
    float* R = nullptr;
    float* Rnorm = nullptr;
    std::vector<float> Rhost;
    std::vector<float> Rnorm_host; // |R_b| rounded up
    std::vector<int64_t> m_upper;  // per-head upper bound of the committed size
    int64_t T_staged = 0, last_commit_T = 0;
    bool appended = false;
    uint64_t launches = 0;
    cudaStream_t last_stream = nullptr;
    tc_status sticky = TC_OK;
    AttnMaps maps{};
    int64_t maps_T = -1;
    // The previous launch of this handle, when it was an attention call: its
    // stream and buffers decide whether the next attention call may overlap it.
    bool prev_attend = false;
    cudaStream_t prev_stream = nullptr;
    const char* prev_q = nullptr;
    const char* prev_out = nullptr;
    size_t prev_bytes = 0;
    std::vector<void*> owned;

    tc_status alloc(void** p, size_t bytes) {
        if (dev_alloc(p, bytes) != cudaSuccess) {
            cudaGetLastError();
            return TC_ENOMEM;
        }
        owned.push_back(*p);
        return TC_OK;
    }
    void free_staging() {
        void* ptrs[] = {s.Ks,     s.Vs,     s.scode,  s.sbias,  s.match,  s.lmatch, s.dest,  s.lcode,
                        s.lnext,  s.wcnt,   s.touched, s.bsim,  s.cbnext, s.crnext, s.ichead, s.ictail,
                        s.icnext, s.moved,  s.movedold};
        for (void* p : ptrs) {
            if (!p) continue;
            owned.erase(std::remove(owned.begin(), owned.end(), p), owned.end());
            cudaFree(p);
        }
        const int64_t T = s.T;
        s = StageView{};
        s.T = T;
    }
    ~tc_ctx() {
        for (void* p : owned) cudaFree(p);
        magic = 0;
    }
};

namespace {

bool valid(tc_handle h) { return h != nullptr && h->magic == kMagic; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tc_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return TC_OK;
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? TC_ENOMEM : TC_ECUDA;
}

// Fold the device's sticky error bits into the handle (caller has synchronised).
tc_status refresh_sticky(tc_ctx* x) {
    Stats st{};
    if (cudaMemcpy(&st, x->stats, sizeof(Stats), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        x->sticky = TC_ECUDA;
    } else if (st.error_bits & kErrTimeout) {
        x->sticky = TC_ETIMEOUT;
    } else if (st.error_bits & kErrBucketList) {
        x->sticky = TC_ESTATE;
    }
    return x->sticky;
}

tc_status ensure_staging(tc_ctx* x, int64_t T) {
    if (x->s.Ks && round_up(T, 128) <= x->s.TmaxP) return TC_OK;
    if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
    x->free_staging();
    const int64_t P = round_up(T, 128);
    const size_t rowsH = (size_t)x->H * P;
    tc_ctx& c = *x;
    tc_status st = TC_OK;
    if ((st = c.alloc(&c.s.Ks, rowsH * x->d * x->esize)) || (st = c.alloc(&c.s.Vs, rowsH * x->d * x->esize)) ||
        (st = c.alloc((void**)&c.s.scode, rowsH * 4)) || (st = c.alloc((void**)&c.s.sbias, P * 4)) ||
        (st = c.alloc((void**)&c.s.match, rowsH * 4)) || (st = c.alloc((void**)&c.s.lmatch, rowsH * 4)) ||
        (st = c.alloc((void**)&c.s.dest, rowsH * 4)) ||
        (st = c.alloc((void**)&c.s.lcode, rowsH * 4)) || (st = c.alloc((void**)&c.s.lnext, rowsH * 4)) ||
        (st = c.alloc((void**)&c.s.wcnt, rowsH / 32 * 4)) || (st = c.alloc((void**)&c.s.touched, rowsH * 4)) ||
        (st = c.alloc((void**)&c.s.bsim, rowsH * 8)) || (st = c.alloc((void**)&c.s.cbnext, rowsH * 4)) ||
        (st = c.alloc((void**)&c.s.crnext, rowsH * 4)) || (st = c.alloc((void**)&c.s.ichead, rowsH * 4)) ||
        (st = c.alloc((void**)&c.s.ictail, rowsH * 4)) || (st = c.alloc((void**)&c.s.icnext, rowsH * 4)) ||
        (x->mean && ((st = c.alloc((void**)&c.s.moved, rowsH * 4)) || (st = c.alloc((void**)&c.s.movedold, rowsH * 4))))) {
        x->free_staging();
        return st;
    }
    // Zero the staging keys and values once: rows past the staged chunk are only
    // ever read as masked attention operands and must hold finite values.
    // The window counts start at zero and the in-chunk member chains empty (-1);
    // every commit leaves them so.
    if (cudaMemset(c.s.Ks, 0, rowsH * x->d * x->esize) != cudaSuccess ||
        cudaMemset(c.s.Vs, 0, rowsH * x->d * x->esize) != cudaSuccess ||
        cudaMemset(c.s.wcnt, 0, rowsH / 32 * 4) != cudaSuccess ||
        cudaMemset(c.s.ichead, 0xff, rowsH * 4) != cudaSuccess)
        return cuda_status(cudaGetLastError());
    x->s.TmaxP = P;
    x->maps_T = -1;
    return TC_OK;
}

tc_status encode_stage_maps(tc_ctx* x) {
    if (x->dtype != TC_BF16 || x->s.T == x->maps_T || x->s.T == 0) return TC_OK;
    const uint64_t d = x->d;
    const bool ok = encode3d(&x->maps.ks, x->s.Ks, d, x->s.T, x->H, d * 2, x->s.TmaxP * d * 2, 64, 128, 1) &&
                    encode3d(&x->maps.vs, x->s.Vs, d, x->s.T, x->H, d * 2, x->s.TmaxP * d * 2, 64, 128, 1);
    if (!ok) return TC_ECUDA;
    x->maps_T = x->s.T;
    return TC_OK;
}

// Commit the staged chunk: apply the decisions its staging took. When the worst case
// could overflow the capacity, first synchronise and read the staging's verdict; a
// refused commit launches nothing and leaves the chunk staged with its decisions.
tc_status commit_staged(tc_ctx* x, cudaStream_t st) {
    if (x->T_staged == 0) return TC_OK;
    int64_t worst = 0;
    for (int64_t m : x->m_upper) worst = std::max(worst, m);
    if (worst + x->T_staged > x->capacity) {
        if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_status(cudaGetLastError());
        std::vector<int32_t> ctr(kCtrInts(x->H));
        if (cudaMemcpy(ctr.data(), x->ctr, ctr.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
            return cuda_status(cudaGetLastError());
        if (ctr[2 * x->H]) return TC_ECAPACITY;
        for (int h = 0; h < x->H; ++h) x->m_upper[h] = ctr[x->H + h];
    } else {
        for (auto& m : x->m_upper) m += x->T_staged;
    }
    StageView s = x->s;
    s.T = x->T_staged;
    int launches = 0;
    cudaError_t e = launch_commit(x->c, s, (int)x->dtype, x->mean, x->R, x->Rnorm, x->ctr, x->claim, x->stats,
                                  &launches, st);
    x->launches += launches;
    if (e != cudaSuccess) return cuda_status(e);
    x->last_commit_T = x->T_staged;
    x->T_staged = 0;
    return TC_OK;
}

tc_status check_call(tc_handle h) {
    if (!valid(h)) return TC_EINVAL;
    if (h->sticky != TC_OK) return h->sticky;
    if (cudaSetDevice(h->device) != cudaSuccess) return cuda_status(cudaGetLastError());
    return TC_OK;
}

}  // namespace

extern "C" {

const char* tc_status_string(tc_status s) {
    switch (s) {
        case TC_OK: return "ok";
        case TC_EINVAL: return "invalid argument or handle";
        case TC_ENOMEM: return "out of memory";
        case TC_ECAPACITY: return "commit would exceed the per-head cache capacity";
        case TC_ECUDA: return "CUDA error";
        case TC_ESTATE: return "call not valid in the current state";
        case TC_ETIMEOUT: return "kernel wait timed out";
        case TC_ENOTIMPL: return "not implemented";
        case TC_EDEVICE: return "no usable sm_100 device";
    }
    return "unknown status";
}

tc_status tc_create(int32_t H, int32_t d, int32_t nbits, float tau, int64_t capacity, tc_handle* out) {
    return tc_create_ex(H, d, nbits, tau, capacity, nullptr, out);
}

tc_status tc_create_ex(int32_t H, int32_t d, int32_t nbits, float tau, int64_t capacity, const tc_options* opt,
                       tc_handle* out) {
    if (!out) return TC_EINVAL;
    *out = nullptr;
    tc_options o{TC_BF16, 0, 0.f, nullptr, 0, 0};
    if (opt) o = *opt;
    if (H < 1 || H > 4096 || (d != 64 && d != 128) || nbits < 1 || nbits > 24 || !(tau >= -1.f && tau <= 2.f) ||
        capacity < 1 || capacity > (int64_t)1 << 30 || (o.dtype != TC_BF16 && o.dtype != TC_F32) ||
        !(o.softmax_scale >= 0.f) || !std::isfinite(o.softmax_scale) || (o.intra_chunk != 0 && o.intra_chunk != 1) ||
        (o.key_mode != 0 && o.key_mode != 1) || (o.key_mode == 1 && o.intra_chunk == 1))
        return TC_EINVAL;
    if (o.hyperplanes) {
        for (int i = 0; i < nbits * d; ++i)
            if (!std::isfinite(o.hyperplanes[i]) || !is_bf16_value(o.hyperplanes[i])) return TC_EINVAL;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TC_EDEVICE;
    }
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
        cudaGetLastError();
        return TC_EDEVICE;
    }
    if (prop.major != 10) return TC_EDEVICE;
    if (o.dtype == TC_BF16 && !get_encoder()) return TC_ECUDA;

    tc_ctx* x = new (std::nothrow) tc_ctx;
    if (!x) return TC_ENOMEM;
    x->H = H;
    x->d = d;
    x->nbits = nbits;
    x->tau = tau;
    x->dtype = o.dtype;
    x->intra = o.intra_chunk != 0;
    x->mean = o.key_mode == 1;
    x->esize = (o.dtype == TC_BF16) ? 2 : 4;
    x->capacity = capacity;
    x->capP = round_up(capacity, 128);
    x->scale = (o.softmax_scale > 0.f) ? o.softmax_scale : (float)(1.0 / std::sqrt((double)d));
    x->device = dev;
    x->m_upper.assign(H, 0);
    if (o.hyperplanes)
        x->Rhost.assign(o.hyperplanes, o.hyperplanes + (size_t)nbits * d);
    else
        default_hyperplanes(o.seed, nbits * d, x->Rhost);

    // Memory budget: refuse early instead of failing halfway.
    const size_t rows = (size_t)H * x->capP;
    const bool k32 = x->mean && o.dtype == TC_BF16;   // fp32 key means beside the bf16 keys
    const size_t need = rows * d * (2 * x->esize + 4 + (k32 ? 4 : 0)) + rows * (4 * 7 + 1) +
                        ((size_t)H << nbits) * 4 * (x->mean ? 2 : 1);
    size_t fr = 0, tot = 0;
    if (cudaMemGetInfo(&fr, &tot) != cudaSuccess) {
        cudaGetLastError();
        delete x;
        return TC_ECUDA;
    }
    if (need + (64u << 20) > fr) {
        delete x;
        return TC_ENOMEM;
    }
    CacheView& c = x->c;
    c.H = H;
    c.d = d;
    c.nbits = nbits;
    c.capP = x->capP;
    c.capacity = capacity;
    tc_status st = TC_OK;
    if ((st = x->alloc(&c.Kc, rows * d * x->esize)) || (st = x->alloc(&c.Vc, rows * d * x->esize)) ||
        (st = x->alloc((void**)&c.V32, rows * d * 4)) || (st = x->alloc((void**)&c.cnt, rows * 4)) ||
        (st = x->alloc((void**)&c.bias2, rows * 4)) || (st = x->alloc((void**)&c.code, rows * 4)) ||
        (st = x->alloc((void**)&c.bnext, rows * 4)) || (st = x->alloc((void**)&c.bhead, ((size_t)H << nbits) * 4)) ||
        (st = x->alloc((void**)&c.knorm64, rows * 8)) || (st = x->alloc((void**)&c.kspan, rows)) || (st = x->alloc((void**)&c.lhead, rows * 4)) ||
        (st = x->alloc((void**)&c.M, (size_t)H * 4)) || (st = x->alloc((void**)&c.kmax2, (size_t)H * 4)) ||
        (st = x->alloc((void**)&c.kmax2s, 4)) || (st = x->alloc((void**)&c.bmax, (size_t)H * 4)) ||
        (x->intra && (st = x->alloc((void**)&c.cbhead, ((size_t)H << nbits) * 4))) ||
        (k32 && (st = x->alloc((void**)&c.K32, rows * d * 4))) ||
        (x->mean && (st = x->alloc((void**)&x->claim, ((size_t)H << nbits) * 4))) ||
        (st = x->alloc((void**)&x->ctr, (size_t)kCtrInts(H) * 4)) ||
        (st = x->alloc((void**)&x->stats, sizeof(Stats))) ||
        (st = x->alloc((void**)&x->R, (size_t)nbits * d * 4)) || (st = x->alloc((void**)&x->Rnorm, nbits * 4))) {
        delete x;
        return st;
    }
    // Rows past the committed entries stay zero (finite attention operands) with
    // log2 n = -inf (masked); empty buckets hold -1.
    if (x->mean && !k32) c.K32 = static_cast<float*>(c.Kc);   // fp32 storage: the keys are the means
    std::vector<float> rnorm(nbits);
    for (int b = 0; b < nbits; ++b) {
        double s2 = 0.0;
        for (int i = 0; i < d; ++i) s2 += (double)x->Rhost[(size_t)b * d + i] * x->Rhost[(size_t)b * d + i];
        rnorm[b] = std::nextafter((float)std::sqrt(s2), INFINITY);
    }
    cudaError_t e = cudaSuccess;
    if ((e = cudaMemset(c.Kc, 0, rows * d * x->esize)) || (e = cudaMemset(c.Vc, 0, rows * d * x->esize)) ||
        (e = cudaMemset(c.V32, 0, rows * d * 4)) || (e = cudaMemset(c.cnt, 0, rows * 4)) ||
        (e = cudaMemset(c.code, 0, rows * 4)) || (e = cudaMemset(c.bnext, 0xff, rows * 4)) ||
        (e = cudaMemset(c.bhead, 0xff, ((size_t)H << nbits) * 4)) || (e = cudaMemset(c.knorm64, 0, rows * 8)) || (e = cudaMemset(c.kspan, 0, rows)) ||
        (e = cudaMemset(c.lhead, 0xff, rows * 4)) ||
        (e = cudaMemset(c.M, 0, (size_t)H * 4)) || (e = cudaMemset(c.kmax2, 0, (size_t)H * 4)) ||
        (e = cudaMemset(c.kmax2s, 0, 4)) || (e = cudaMemset(c.bmax, 0, (size_t)H * 4)) ||
        (x->intra && (e = cudaMemset(c.cbhead, 0xff, ((size_t)H << nbits) * 4))) || (e = cudaMemset(x->ctr, 0, (size_t)kCtrInts(H) * 4)) ||
        (k32 && (e = cudaMemset(c.K32, 0, rows * d * 4))) ||
        (x->mean && (e = cudaMemset(x->claim, 0, ((size_t)H << nbits) * 4))) ||
        (e = cudaMemset(x->stats, 0, sizeof(Stats))) ||
        (e = cudaMemcpy(x->R, x->Rhost.data(), (size_t)nbits * d * 4, cudaMemcpyHostToDevice)) ||
        (e = cudaMemcpy(x->Rnorm, rnorm.data(), nbits * 4, cudaMemcpyHostToDevice))) {
        delete x;
        return cuda_status(e);
    }
    x->Rnorm_host = rnorm;
    fill_f32<<<1024, 256>>>(c.bias2, (int64_t)rows, 1, 0, -INFINITY);
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) {
        delete x;
        return cuda_status(e);
    }
    if (x->dtype == TC_BF16) {
        const bool ok = encode3d(&x->maps.kc, c.Kc, d, x->capP, H, (uint64_t)d * 2, (uint64_t)x->capP * d * 2, 64,
                                 128, 1) &&
                        encode3d(&x->maps.vc, c.Vc, d, x->capP, H, (uint64_t)d * 2, (uint64_t)x->capP * d * 2, 64,
                                 128, 1);
        if (!ok) {
            delete x;
            return TC_ECUDA;
        }
    }
    *out = x;
    return TC_OK;
}

tc_status tc_append_chunk(tc_handle x, const void* K, const void* V, int64_t T, tc_stream stream) {
    tc_status st = check_call(x);
    if (st) return st;
    if (!K || !V || !aligned16(K) || !aligned16(V) || T < 1 || T > ((int64_t)1 << 28) ||
        T * x->H >= ((int64_t)1 << 31))   // the kernels index rows t H + h in 32 bits
        return TC_EINVAL;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    x->last_stream = cs;
    x->prev_attend = false;
    if ((st = commit_staged(x, cs))) return st;
    if ((st = ensure_staging(x, T))) return st;
    x->s.T = T;
    if ((st = encode_stage_maps(x))) return st;
    cudaError_t e = cudaMemsetAsync(x->c.kmax2s, 0, 4, cs);   // the staged keys' bound starts over
    int launches = 0;
    if (e == cudaSuccess)
        e = launch_stage(x->c, x->s, (int)x->dtype, x->intra, x->mean, K, V, x->R, x->Rhost.data(),
                         x->Rnorm_host.data(), x->tau, x->ctr, x->stats, &launches, cs);
    x->launches += launches;
    if (e != cudaSuccess) return cuda_status(e);
    x->T_staged = T;
    x->appended = true;
    return TC_OK;
}

tc_status tc_flush(tc_handle x, tc_stream stream) {
    tc_status st = check_call(x);
    if (st) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    x->last_stream = cs;
    x->prev_attend = false;
    if ((st = commit_staged(x, cs))) return st;
    x->s.T = 0;
    return TC_OK;
}

tc_status tc_attend(tc_handle x, const void* Q, int64_t Tq, void* out, tc_stream stream) {
    tc_status st = check_call(x);
    if (st) return st;
    if (!Q || !out || !aligned16(Q) || !aligned16(out) || Tq < 1 || Tq > ((int64_t)1 << 28)) return TC_EINVAL;
    const size_t bytes = (size_t)Tq * x->H * x->d * x->esize;
    const char* q = static_cast<const char*>(Q);
    const char* o = static_cast<const char*>(out);
    if (q < o + bytes && o < q + bytes) return TC_EINVAL;
    if (!x->appended) return TC_ESTATE;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    x->last_stream = cs;
    StageView s = x->s;
    s.T = x->T_staged;
    const float scale_log2 = (float)((double)x->scale * 1.4426950408889634);
    cudaError_t e;
    if (x->dtype == TC_BF16) {
        AttnMaps m = x->maps;
        if (!encode3d(&m.q, Q, x->d, x->H, Tq, (uint64_t)x->d * 2, (uint64_t)x->H * x->d * 2, 64, 1, 128))
            return TC_EINVAL;
        // Consecutive attention calls only read the cache and staging buffers, so the
        // next may start while the previous drains, unless their buffers interact.
        auto overlaps = [](const char* a, size_t na, const char* b, size_t nb) { return a < b + nb && b < a + na; };
        const bool overlap = x->prev_attend && x->prev_stream == cs && !overlaps(o, bytes, x->prev_out, x->prev_bytes) &&
                             !overlaps(o, bytes, x->prev_q, x->prev_bytes) &&
                             !overlaps(q, bytes, x->prev_out, x->prev_bytes);
        e = launch_attend_bf16(x->c, s, m, Tq, static_cast<__nv_bfloat16*>(out), scale_log2, x->stats, overlap,
                               cs);
        x->prev_attend = (e == cudaSuccess);
        x->prev_stream = cs;
        x->prev_q = q;
        x->prev_out = o;
        x->prev_bytes = bytes;
    } else {
        e = launch_attend_f32(x->c, s, static_cast<const float*>(Q), Tq, static_cast<float*>(out), scale_log2, cs);
    }
    x->launches += 1;
    return cuda_status(e);
}

tc_status tc_reset(tc_handle x, tc_stream stream) {
    tc_status st = check_call(x);
    if (st) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    x->last_stream = cs;
    x->prev_attend = false;
    // Rows at or past the committed size only need log2 n = -inf (masked) and finite
    // keys/values, which the previous rollout left there; the bucket lists restart.
    int64_t upto = 0;
    for (int64_t m : x->m_upper) upto = std::max(upto, m);
    upto = std::min(round_up(upto, 128), x->capP);
    cudaError_t e = cudaMemsetAsync(x->c.bhead, 0xff, ((size_t)x->H << x->nbits) * 4, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(x->c.M, 0, (size_t)x->H * 4, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(x->ctr, 0, (size_t)kCtrInts(x->H) * 4, cs);
    if (e == cudaSuccess && x->T_staged > 0) {
        // a staged chunk's decisions are dropped: its merge lists on committed entries,
        // in-chunk member chains and bucket groups
        e = cudaMemsetAsync(x->c.lhead, 0xff, (size_t)x->H * x->capP * 4, cs);
        if (e == cudaSuccess) e = cudaMemsetAsync(x->s.ichead, 0xff, (size_t)x->H * x->s.TmaxP * 4, cs);
        if (e == cudaSuccess && x->intra) e = cudaMemsetAsync(x->c.cbhead, 0xff, ((size_t)x->H << x->nbits) * 4, cs);
    }
    if (e == cudaSuccess) e = cudaMemsetAsync(x->c.kmax2, 0, (size_t)x->H * 4, cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(x->c.bmax, 0, (size_t)x->H * 4, cs);
    if (e == cudaSuccess && upto > 0) {
        dim3 grid((unsigned)std::min<int64_t>((upto + 255) / 256, 64), (unsigned)std::min(x->H, 1024));
        fill_f32<<<grid, 256, 0, cs>>>(x->c.bias2, upto, x->H, x->capP, -INFINITY);
        e = cudaGetLastError();
        x->launches += 1;
    }
    if (e != cudaSuccess) return cuda_status(e);
    std::fill(x->m_upper.begin(), x->m_upper.end(), 0);
    x->T_staged = 0;
    x->s.T = 0;
    x->last_commit_T = 0;
    x->appended = false;
    return TC_OK;
}

tc_status tc_sync(tc_handle x) {
    if (!valid(x)) return TC_EINVAL;
    if (cudaSetDevice(x->device) != cudaSuccess) return cuda_status(cudaGetLastError());
    if (cudaStreamSynchronize(x->last_stream) != cudaSuccess) {
        cudaGetLastError();
        x->sticky = TC_ECUDA;
        return x->sticky;
    }
    return refresh_sticky(x);
}

tc_status tc_cache_size(tc_handle x, int64_t* sizes_H) {
    tc_status st = tc_sync(x);
    if (st) return st;
    if (!sizes_H) return TC_EINVAL;
    std::vector<int32_t> M(x->H);
    if (cudaMemcpy(M.data(), x->c.M, (size_t)x->H * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return cuda_status(cudaGetLastError());
    for (int h = 0; h < x->H; ++h) sizes_H[h] = M[h];
    return TC_OK;
}

void tc_destroy(tc_handle x) {
    if (!valid(x)) return;
    cudaSetDevice(x->device);
    cudaDeviceSynchronize();
    cudaGetLastError();
    delete x;
}

tc_status tc_debug_last_commit(tc_handle x, int64_t* T_out, uint32_t* codes_HT, int32_t* match_HT,
                               int32_t* dest_HT) {
    tc_status st = tc_sync(x);
    if (st) return st;
    const int64_t T = x->last_commit_T;
    if (T_out) *T_out = T;
    if (T == 0) return TC_OK;
    for (int h = 0; h < x->H; ++h) {
        const size_t off = (size_t)h * x->s.TmaxP;
        cudaError_t e = cudaSuccess;
        if (codes_HT && (e = cudaMemcpy(codes_HT + h * T, x->s.lcode + off, T * 4, cudaMemcpyDeviceToHost)))
            return cuda_status(e);
        if (match_HT && (e = cudaMemcpy(match_HT + h * T, x->s.lmatch + off, T * 4, cudaMemcpyDeviceToHost)))
            return cuda_status(e);
        if (dest_HT && (e = cudaMemcpy(dest_HT + h * T, x->s.dest + off, T * 4, cudaMemcpyDeviceToHost)))
            return cuda_status(e);
    }
    return TC_OK;
}

tc_status tc_debug_staged_codes(tc_handle x, int64_t* T_out, uint32_t* codes_HT) {
    tc_status st = tc_sync(x);
    if (st) return st;
    const int64_t T = x->T_staged;
    if (T_out) *T_out = T;
    if (T == 0 || !codes_HT) return TC_OK;
    for (int h = 0; h < x->H; ++h) {
        cudaError_t e =
            cudaMemcpy(codes_HT + h * T, x->s.scode + (size_t)h * x->s.TmaxP, T * 4, cudaMemcpyDeviceToHost);
        if (e) return cuda_status(e);
    }
    return TC_OK;
}

tc_status tc_export_cache(tc_handle x, int32_t head, void* K, float* V32, int32_t* n, uint32_t* code) {
    tc_status st = tc_sync(x);
    if (st) return st;
    if (head < 0 || head >= x->H) return TC_EINVAL;
    int32_t M = 0;
    if (cudaMemcpy(&M, x->c.M + head, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return cuda_status(cudaGetLastError());
    const size_t row = (size_t)head * x->capP;
    cudaError_t e = cudaSuccess;
    if (K && (e = cudaMemcpy(K, static_cast<char*>(x->c.Kc) + row * x->d * x->esize, (size_t)M * x->d * x->esize,
                             cudaMemcpyDeviceToHost)))
        return cuda_status(e);
    if (V32 && (e = cudaMemcpy(V32, x->c.V32 + row * x->d, (size_t)M * x->d * 4, cudaMemcpyDeviceToHost)))
        return cuda_status(e);
    if (n && (e = cudaMemcpy(n, x->c.cnt + row, (size_t)M * 4, cudaMemcpyDeviceToHost))) return cuda_status(e);
    if (code && (e = cudaMemcpy(code, x->c.code + row, (size_t)M * 4, cudaMemcpyDeviceToHost)))
        return cuda_status(e);
    return TC_OK;
}

tc_status tc_export_key_means(tc_handle x, int32_t head, float* K32) {
    tc_status st = tc_sync(x);
    if (st) return st;
    if (head < 0 || head >= x->H || !K32) return TC_EINVAL;
    if (!x->mean) return TC_ESTATE;
    int32_t M = 0;
    if (cudaMemcpy(&M, x->c.M + head, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return cuda_status(cudaGetLastError());
    const size_t row = (size_t)head * x->capP;
    if (cudaMemcpy(K32, x->c.K32 + row * x->d, (size_t)M * x->d * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return cuda_status(cudaGetLastError());
    return TC_OK;
}

tc_status tc_get_hyperplanes(tc_handle x, float* R) {
    if (!valid(x) || !R) return TC_EINVAL;
    std::memcpy(R, x->Rhost.data(), x->Rhost.size() * sizeof(float));
    return TC_OK;
}

tc_status tc_stats(tc_handle x, uint64_t* kernel_launches, uint64_t* hash_rechecks, uint64_t* match_rechecks) {
    if (!valid(x)) return TC_EINVAL;
    if (kernel_launches) *kernel_launches = x->launches;
    if (hash_rechecks || match_rechecks) {
        tc_status st = tc_sync(x);
        if (st) return st;
        Stats s{};
        if (cudaMemcpy(&s, x->stats, sizeof(Stats), cudaMemcpyDeviceToHost) != cudaSuccess)
            return cuda_status(cudaGetLastError());
        if (hash_rechecks) *hash_rechecks = s.hash_rechecks;
        if (match_rechecks) *match_rechecks = s.match_rechecks;
    }
    return TC_OK;
}

}  // extern "C"
