// Biased flash attention over [committed cache | staged chunk] on sm_100a tensor cores.
//
// out_t = sum_j exp(s_tj) v_j / sum_j exp(s_tj), s_tj = scale <q_t,k_j> + ln n_j for
// committed entries (n_j = group size) and + 0 for staged tokens. FAST-AR technical
// summary, section 2.A: Lemma 5.1 makes averaged values with a logit shift by the
// group size exact for identical keys. Computed in base 2: x = s * log2(e).
//
// One CTA = 128 query rows of one head and owns the SM's 512 TMEM columns:
//   S0 [0,128), S1 [128,256)  scores of consecutive key tiles (P overwrites its S)
//   O  [256, 256+D)           fp32 output accumulator
// Warp roles (224 threads):
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r); one pass per key
//              tile with an upper-bound reference max, lazy rescaling of O (only when
//              the reference grows by more than 2^8), P written as bf16 over S.
//   warp 4     TMA producer for Q and the K ring (2 stages); TMEM allocator.
//   warp 5     MMA issuer: S_{i+1} = Q K_{i+1}^T is issued before O += P_i V_i, so
//              the tensor core computes the next scores while softmax works on P_i.
//   warp 6     TMA producer for the V ring (2 stages).
// Operands come by 3-D TMA (64-column, 128-byte-swizzled boxes) straight from the
// token-major Q and the head-major cache/staging buffers. Every mbarrier wait is
// bounded (2 s); a timeout sets an error bit and the CTA drains its own copies and
// MMAs before releasing TMEM.
#include "tc_internal.h"

#include <math.h>

namespace tc {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kThreads = 224;
constexpr uint64_t kTimeoutNs = 2000000000ull;

template <int D>
struct Cfg {
    static constexpr int NB = D / 64;                 // 64-column swizzle boxes per row
    static constexpr int BOX = 128 * 128;             // bytes of one 128-row box
    static constexpr int TILE = NB * BOX;             // bytes of a Q, K or V tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;                // 2 stages
    static constexpr int OFF_V = 3 * TILE;            // 2 stages
    static constexpr int OFF_BIAS = 5 * TILE;         // 2 x 128 floats
    static constexpr int OFF_BMAX = OFF_BIAS + 2 * 128 * 4;  // 2 x 4 floats
    static constexpr int OFF_BAR = OFF_BMAX + 2 * 4 * 4;
    static constexpr int NBAR = 16;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 32 + 1024;  // + slack for 1024-B alignment
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t O_COL = 256;
    // Instruction descriptors, kind::f16: bits 4-5 D format (1 = f32), 7-9 A format
    // (1 = bf16), 10-12 B format (1 = bf16), 15/16 A/B major (0 = K, 1 = MN),
    // 17-22 N>>3, 24-28 M>>4.
    static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                                         ((uint32_t)(kBM >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
};

// mbarriers: Q full; K full/empty x2; V full/empty x2; S full x2; P full x2; PV done; drain.
enum { B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 3, B_VFULL = 5, B_VEMPTY = 7, B_SFULL = 9, B_PFULL = 11, B_ODONE = 13,
       B_DRAIN = 14 };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on phase `parity`; false after kTimeoutNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try(bar, parity)) {
        if (global_ns() - t0 > kTimeoutNs) return false;
    }
    return true;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100 version
// bits [46,48) = 1. Addresses and offsets are in 16-byte units.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

#define TC_LD32(taddr, r)                                                                                    \
    asm volatile(                                                                                            \
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17," \
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                                     \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),    \
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),           \
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),         \
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),         \
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])                                                              \
        : "r"(taddr))

#define TC_ST32(taddr, r)                                                                                    \
    asm volatile(                                                                                            \
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16," \
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),                      \
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),   \
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),       \
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),      \
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])                   \
        : "memory")

#define TC_ST16(taddr, r)                                                                                    \
    asm volatile(                                                                                            \
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" \
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),  \
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])           \
        : "memory")

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void up2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
    return m;
}
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Barrier 1 over the 128 softmax threads with an AND of `v` across them.
__device__ __forceinline__ bool bar_and_128(bool v) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)v)
        : "memory");
    return res != 0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attend_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                   const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKs,
                   const __grid_constant__ CUtensorMap tmVs, const int32_t* __restrict__ Mdev,
                   const float* __restrict__ bias2, int64_t capP, const float* __restrict__ sbias, int64_t Ts,
                   int64_t Tq, int H, __nv_bfloat16* __restrict__ out, float scale_log2, Stats* stats) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    float* sBias = reinterpret_cast<float*>(smem + C::OFF_BIAS);
    float* sBmax = reinterpret_cast<float*>(smem + C::OFF_BMAX);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int q0 = blockIdx.x * kBM;
    const int Mh = Mdev[h];
    const int nc = (Mh + kBN - 1) / kBN;
    const int ntiles = nc + (int)((Ts + kBN - 1) / kBN);

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_QFULL], 1);
        for (int s2 = 0; s2 < 2; ++s2) {
            mbar_init(&bars[B_KFULL + s2], 1);
            mbar_init(&bars[B_KEMPTY + s2], 1);
            mbar_init(&bars[B_VFULL + s2], 1);
            mbar_init(&bars[B_VEMPTY + s2], 1);
            mbar_init(&bars[B_SFULL + s2], 1);
            mbar_init(&bars[B_PFULL + s2], 128);
        }
        mbar_init(&bars[B_ODONE], 1);
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 4) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Let the next attention call on this stream start filling SMs as this grid
    // drains (it only reads what this kernel reads).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const uint32_t tO = tmem + C::O_COL;
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint8_t* sV = smem + C::OFF_V;

    if (warp == 4 || warp == 6) {
        // ---------------------------------------------------------------- producers (lane 0)
        if (lane == 0) {
            const bool kside = (warp == 4);
            uint8_t* ring = kside ? sK : sV;
            uint64_t* full = &bars[kside ? B_KFULL : B_VFULL];
            uint64_t* empty = &bars[kside ? B_KEMPTY : B_VEMPTY];
            const CUtensorMap* mc = kside ? &tmKc : &tmVc;
            const CUtensorMap* ms = kside ? &tmKs : &tmVs;
            if (kside) {
                mbar_expect_tx(&bars[B_QFULL], C::TILE);
                for (int b = 0; b < C::NB; ++b) tma_load_3d(sQ + b * C::BOX, &tmQ, 64 * b, h, q0, &bars[B_QFULL]);
            }
            int last = -1;
            for (int i = 0; i < ntiles && !*abort_flag; ++i) {
                const int st = i & 1;
                if (i >= 2 && !mbar_wait(&empty[st], ((i >> 1) - 1) & 1)) { *abort_flag = 1; break; }
                const bool cache = i < nc;
                const int row0 = (cache ? i : i - nc) * kBN;
                mbar_expect_tx(&full[st], C::TILE);
                for (int b = 0; b < C::NB; ++b)
                    tma_load_3d(ring + st * C::TILE + b * C::BOX, cache ? mc : ms, 64 * b, row0, h, &full[st]);
                last = i;
            }
            // Drain: the copies issued here land before the CTA can exit (already true
            // on the normal path, where the MMA thread consumed them all).
            if (kside) mbar_wait(&bars[B_QFULL], 0);
            for (int i = (last >= 1 ? last - 1 : 0); i <= last; ++i) mbar_wait(&full[i & 1], (i >> 1) & 1);
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer (lane 0)
        if (lane == 0) {
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = mbar_wait(&bars[B_QFULL], 0);
            auto issue_qk = [&](int j) -> bool {
                const int st = j & 1;
                // S_st held P_{j-2}: wait until O += P_{j-2} V_{j-2} has retired.
                if (j >= 2 && !mbar_wait(&bars[B_ODONE], (j - 2) & 1)) return false;
                if (!mbar_wait(&bars[B_KFULL + st], (j >> 1) & 1)) return false;
                tc_fence_after();
                const uint32_t aKs = aK + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tmem + st * 128, sdesc(aQ + off, 16, 1024), sdesc(aKs + off, 16, 1024), C::IDESC_QK,
                           kk > 0);
                }
                tc_commit(&bars[B_SFULL + st]);
                tc_commit(&bars[B_KEMPTY + st]);
                return true;
            };
            if (ok && ntiles > 0) ok = issue_qk(0);
            for (int i = 0; i < ntiles && ok && !*abort_flag; ++i) {
                if (i + 1 < ntiles && !(ok = issue_qk(i + 1))) break;
                const int st = i & 1;
                if (!mbar_wait(&bars[B_PFULL + st], (i >> 1) & 1)) { ok = false; break; }
                if (!mbar_wait(&bars[B_VFULL + st], (i >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t aVs = aV + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ts(tO, tmem + st * 128 + kk * 8, sdesc(aVs + kk * 2048, C::BOX, 1024), C::IDESC_PV,
                           (i > 0 || kk > 0));
                tc_commit(&bars[B_VEMPTY + st]);
                tc_commit(&bars[B_ODONE]);
            }
            if (!ok) *abort_flag = 1;
            // Drain: every MMA issued here retires before TMEM is released.
            tc_commit(&bars[B_DRAIN]);
            mbar_wait(&bars[B_DRAIN], 0);
        }
    } else {
        // ---------------------------------------------------------------- softmax (warps 0-3)
        // Control flow stays uniform across the 128 threads: tcgen05.ld/st are
        // warp-collective, so every decision that guards them is reduced first.
        const int r = threadIdx.x;  // query row within the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const float* bias_h = bias2 + (int64_t)h * capP;
        auto bias_of = [&](int i) -> float {
            return (i < nc) ? bias_h[(int64_t)i * kBN + r] : sbias[(int64_t)(i - nc) * kBN + r];
        };
        const uint64_t c2 = pk2(scale_log2, scale_log2);
        float m_run = -INFINITY, l_run = 0.f;
        float bnext = (ntiles > 0) ? bias_of(0) : 0.f;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            const int st = i & 1;
            float* bb = sBias + st * kBN;
            bb[r] = bnext;
            float wm = bnext;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
            if (lane == 0) sBmax[st * 4 + warp] = wm;
            const bool got = !*abort_flag && mbar_wait(&bars[B_SFULL + st], (i >> 1) & 1);
            if (!bar_and_128(got)) { ok = false; break; }   // also publishes bb[] and the bias maxima
            if (i + 1 < ntiles) bnext = bias_of(i + 1);
            tc_fence_after();
            const uint32_t tS = tmem + st * 128 + lane_base;
            uint32_t sr[kBN];
            TC_LD32(tS + 0, (sr + 0));
            TC_LD32(tS + 32, (sr + 32));
            TC_LD32(tS + 64, (sr + 64));
            TC_LD32(tS + 96, (sr + 96));
            tc_wait_ld();
            // Reference max: an upper bound of this tile's row max, (max raw score) *
            // scale + (max shift of the tile). p = 2^(x - m) stays <= 2^8 below.
            float smax = -INFINITY;
#pragma unroll
            for (int j = 0; j < kBN; j += 2) smax = max3(smax, __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
            const float4 bm4 = *reinterpret_cast<const float4*>(sBmax + st * 4);
            const float ub = fmaf(smax, scale_log2, fmaxf(fmaxf(bm4.x, bm4.y), fmaxf(bm4.z, bm4.w)));
            if (i == 0) {
                m_run = ub;
            } else {
                // Lazy rescaling: O and l keep the old reference until it would grow by
                // more than 8 (a factor 256), then both are scaled by alpha.
                const bool need = ub > m_run + 8.f;
                if (__any_sync(0xffffffffu, need)) {
                    const bool w = mbar_wait(&bars[B_ODONE], (i - 1) & 1);
                    if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; }
                    if (ok) {
                        const float alpha = need ? ex2(m_run - ub) : 1.f;
                        if (need) { l_run *= alpha; m_run = ub; }
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t o[32];
                            TC_LD32(tO + lane_base + 32 * c, o);
                            tc_wait_ld();
#pragma unroll
                            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
                            TC_ST32(tO + lane_base + 32 * c, o);
                        }
                        tc_wait_st();
                    }
                }
            }
            // p = 2^(s * scale + log2 n - m): packed fp32x2 FMA/ADD, MUFU ex2, bf16 pack.
            const uint64_t negm2 = pk2(-m_run, -m_run);
            uint64_t sum2 = pk2(0.f, 0.f);
            uint32_t pk[kBN / 2];
#pragma unroll
            for (int j = 0; j < kBN; j += 4) {
                const float4 b4 = *reinterpret_cast<const float4*>(bb + j);
                const uint64_t x01 = fma2(pk2(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), c2,
                                          add2(pk2(b4.x, b4.y), negm2));
                const uint64_t x23 = fma2(pk2(__uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3])), c2,
                                          add2(pk2(b4.z, b4.w), negm2));
                float a0, a1, a2, a3;
                up2(x01, a0, a1);
                up2(x23, a2, a3);
                const float p0 = ex2(a0), p1 = ex2(a1), p2 = ex2(a2), p3 = ex2(a3);
                sum2 = add2(sum2, add2(pk2(p0, p1), pk2(p2, p3)));
                pk[j / 2] = cvt_bf16x2(p0, p1);
                pk[j / 2 + 1] = cvt_bf16x2(p2, p3);
            }
            float s0, s1;
            up2(sum2, s0, s1);
            l_run += s0 + s1;
            TC_ST32(tS + 0, (pk + 0));
            TC_ST32(tS + 32, (pk + 32));
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[B_PFULL + st]);
        }
        const bool fin = ok && ntiles > 0 && mbar_wait(&bars[B_ODONE], (ntiles - 1) & 1);
        if (bar_and_128(fin)) {
            tc_fence_after();
            const float inv = 1.f / l_run;
            const int64_t row = q0 + r;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                TC_LD32(tO + lane_base + 32 * c, o);
                tc_wait_ld();
                if (row < Tq) {
                    uint4* dst = reinterpret_cast<uint4*>(out + (row * H + h) * D + 32 * c);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = cvt_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                        w.y = cvt_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                        w.z = cvt_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                        w.w = cvt_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
                        dst[v] = w;
                    }
                }
            }
        } else {
            *abort_flag = 1;
        }
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(&stats->error_bits, 2u);
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
    }
    // When this grid was allowed to start before the previous one finished, it
    // completes only after that one: whatever follows on the stream sees both done.
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D>
cudaError_t launch_t(const CacheView& c, const StageView& s, const AttnMaps& m, int64_t Tq, __nv_bfloat16* out,
                     float scale_log2, Stats* stats, bool overlap_prev, cudaStream_t st) {
    using C = Cfg<D>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(attend_bf16_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((Tq + kBM - 1) / kBM), (unsigned)c.H);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = overlap_prev ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attend_bf16_kernel<D>, m.q, m.kc, m.vc, m.ks, m.vs, (const int32_t*)c.M,
                              (const float*)c.bias2, c.capP, (const float*)s.sbias, s.T, Tq, c.H, out, scale_log2,
                              stats);
}

}  // namespace

cudaError_t launch_attend_bf16(const CacheView& c, const StageView& s, const AttnMaps& maps, int64_t Tq,
                               __nv_bfloat16* out, float scale_log2, Stats* stats, bool overlap_prev,
                               cudaStream_t st) {
    return c.d == 128 ? launch_t<128>(c, s, maps, Tq, out, scale_log2, stats, overlap_prev, st)
                      : launch_t<64>(c, s, maps, Tq, out, scale_log2, stats, overlap_prev, st);
}

}  // namespace tc
