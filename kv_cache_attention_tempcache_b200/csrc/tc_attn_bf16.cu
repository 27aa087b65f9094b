// Biased flash attention over [committed cache | staged chunk] on sm_100a tensor cores.
//
// out_t = sum_j exp(s_tj) v_j / sum_j exp(s_tj), s_tj = scale <q_t,k_j> + ln n_j for
// committed entries (n_j = group size) and + 0 for staged tokens. FAST-AR technical
// summary, section 2.A: Lemma 5.1 makes averaged values with a logit shift by the
// group size exact for identical keys. Computed in base 2: x = s * log2(e).
//
// One CTA = 128 query rows of one head; two CTAs share an SM so one CTA's softmax
// overlaps the other's MMAs. Warp roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r); online softmax in
//              fp32 with lazy rescaling of O (only when the running max grows by
//              more than 2^8); writes P as bf16 into TMEM over S.
//   warp 4     TMA producer (Q once, then one K and one V tile per step) and TMEM
//              allocator.
//   warp 5     MMA issuer: S = Q K^T (SS form, both K-major), O += P V (P from
//              TMEM, V MN-major), fp32 accumulators in TMEM.
// TMEM (256 columns): S/P at columns [0,128), O at [128, 128+D).
// Shared memory: Q, K, V tiles of 128 rows, 128-byte swizzled boxes of 64 columns.
// Every mbarrier wait is bounded (2 s); a timeout sets an error bit and the CTA
// drains its own copies and MMAs before releasing TMEM.
#include "tc_internal.h"

#include <math.h>

namespace tc {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kThreads = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;

template <int D>
struct Cfg {
    static constexpr int NB = D / 64;                 // 64-column swizzle boxes per row
    static constexpr int BOX = 128 * 128;             // bytes of one 128-row box
    static constexpr int TILE = NB * BOX;             // bytes of a Q, K or V tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;
    static constexpr int OFF_V = 2 * TILE;
    static constexpr int OFF_BIAS = 3 * TILE;         // 2 x 128 floats
    static constexpr int OFF_BAR = OFF_BIAS + 2 * 128 * 4;
    static constexpr int NBAR = 10;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 32 + 1024;  // + slack for 1024-B alignment
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t O_COL = 128;
    // Instruction descriptors, kind::f16: bits 4-5 D format (1 = f32), 7-9 A format
    // (1 = bf16), 10-12 B format (1 = bf16), 15/16 A/B major (0 = K, 1 = MN),
    // 17-22 N>>3, 24-28 M>>4.
    static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                                         ((uint32_t)(kBM >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
};

enum { B_QFULL = 0, B_KFULL, B_KEMPTY, B_VFULL, B_VEMPTY, B_SFULL, B_PFULL, B_ORDY, B_DRAIN };

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
__global__ void __launch_bounds__(kThreads, 2)
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
        mbar_init(&bars[B_KFULL], 1);
        mbar_init(&bars[B_KEMPTY], 1);
        mbar_init(&bars[B_VFULL], 1);
        mbar_init(&bars[B_VEMPTY], 1);
        mbar_init(&bars[B_SFULL], 1);
        mbar_init(&bars[B_PFULL], 128);
        mbar_init(&bars[B_ORDY], 1);
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
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem + C::S_COL;
    const uint32_t tO = tmem + C::O_COL;
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint8_t* sV = smem + C::OFF_V;

    if (warp == 4) {
        // ---------------------------------------------------------------- producer (lane 0)
        if (lane == 0) {
            int lastK = -1, lastV = -1;
            mbar_expect_tx(&bars[B_QFULL], C::TILE);
            for (int b = 0; b < C::NB; ++b) tma_load_3d(sQ + b * C::BOX, &tmQ, 64 * b, h, q0, &bars[B_QFULL]);
            for (int i = 0; i < ntiles && !*abort_flag; ++i) {
                const bool cache = i < nc;
                const int row0 = (cache ? i : i - nc) * kBN;
                const CUtensorMap* mk = cache ? &tmKc : &tmKs;
                const CUtensorMap* mv = cache ? &tmVc : &tmVs;
                if (i > 0 && !mbar_wait(&bars[B_KEMPTY], (i - 1) & 1)) { *abort_flag = 1; break; }
                mbar_expect_tx(&bars[B_KFULL], C::TILE);
                for (int b = 0; b < C::NB; ++b) tma_load_3d(sK + b * C::BOX, mk, 64 * b, row0, h, &bars[B_KFULL]);
                lastK = i;
                if (i > 0 && !mbar_wait(&bars[B_VEMPTY], (i - 1) & 1)) { *abort_flag = 1; break; }
                mbar_expect_tx(&bars[B_VFULL], C::TILE);
                for (int b = 0; b < C::NB; ++b) tma_load_3d(sV + b * C::BOX, mv, 64 * b, row0, h, &bars[B_VFULL]);
                lastV = i;
            }
            // Drain: every issued copy has landed before the CTA can exit (already
            // true on the normal path, where the MMA thread consumed them all).
            mbar_wait(&bars[B_QFULL], 0);
            if (lastK >= 0) mbar_wait(&bars[B_KFULL], lastK & 1);
            if (lastV >= 0) mbar_wait(&bars[B_VFULL], lastV & 1);
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer (lane 0)
        if (lane == 0) {
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = mbar_wait(&bars[B_QFULL], 0);
            for (int i = 0; i < ntiles && ok && !*abort_flag; ++i) {
                // S/P of step i-1 must be consumed by its PV before S is overwritten.
                if (i > 0 && !mbar_wait(&bars[B_ORDY], (i - 1) & 1)) { ok = false; break; }
                if (!mbar_wait(&bars[B_KFULL], i & 1)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tS, sdesc(aQ + off, 16, 1024), sdesc(aK + off, 16, 1024), C::IDESC_QK, kk > 0);
                }
                tc_commit(&bars[B_SFULL]);
                tc_commit(&bars[B_KEMPTY]);
                if (!mbar_wait(&bars[B_PFULL], i & 1)) { ok = false; break; }
                if (!mbar_wait(&bars[B_VFULL], i & 1)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ts(tO, tS + kk * 8, sdesc(aV + kk * 2048, C::BOX, 1024), C::IDESC_PV, (i > 0 || kk > 0));
                tc_commit(&bars[B_VEMPTY]);
                tc_commit(&bars[B_ORDY]);
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
        float m_run = -INFINITY, l_run = 0.f;
        float bnext = (ntiles > 0) ? bias_of(0) : 0.f;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            float* bb = sBias + (i & 1) * kBN;
            bb[r] = bnext;
            const bool got = !*abort_flag && mbar_wait(&bars[B_SFULL], i & 1);
            if (!bar_and_128(got)) { ok = false; break; }   // also publishes bb[] to the group
            if (i + 1 < ntiles) bnext = bias_of(i + 1);
            tc_fence_after();
            // Pass 1: row max of x = s * scale * log2(e) + log2 n, 32 columns at a time.
            float mx = -INFINITY;
#pragma unroll 1
            for (int cc = 0; cc < kBN / 32; ++cc) {
                uint32_t xr[32];
                TC_LD32(tS + lane_base + 32 * cc, xr);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) mx = fmaxf(mx, fmaf(__uint_as_float(xr[j]), scale_log2, bb[32 * cc + j]));
            }
            const float m_new = fmaxf(m_run, mx);
            if (i == 0) {
                m_run = m_new;
            } else {
                // Lazy rescaling: O and l keep the old reference max until the row max
                // grows by more than 8 (a factor 256), then both are scaled by alpha.
                const bool need = m_new > m_run + 8.f;
                if (__any_sync(0xffffffffu, need)) {
                    const bool w = mbar_wait(&bars[B_ORDY], (i - 1) & 1);
                    if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; }
                    if (ok) {
                        const float alpha = need ? exp2f(m_run - m_new) : 1.f;
                        if (need) { l_run *= alpha; m_run = m_new; }
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
            // Pass 2: p = 2^(x - m), row sum, bf16 P written over S. Chunk cc of P
            // (columns 16cc..16cc+15) only covers S columns already read.
            float sum = 0.f;
#pragma unroll 1
            for (int cc = 0; cc < kBN / 32; ++cc) {
                uint32_t xr[32];
                TC_LD32(tS + lane_base + 32 * cc, xr);
                tc_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float p0 = exp2f(fmaf(__uint_as_float(xr[2 * j]), scale_log2, bb[32 * cc + 2 * j]) - m_run);
                    const float p1 =
                        exp2f(fmaf(__uint_as_float(xr[2 * j + 1]), scale_log2, bb[32 * cc + 2 * j + 1]) - m_run);
                    sum += p0 + p1;
                    pk[j] = pack_bf16(p0, p1);
                }
                TC_ST16(tS + lane_base + 16 * cc, pk);
            }
            l_run += sum;
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[B_PFULL]);
        }
        const bool fin = ok && ntiles > 0 && mbar_wait(&bars[B_ORDY], (ntiles - 1) & 1);
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
                        w.x = pack_bf16(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
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
}

template <int D>
cudaError_t launch_t(const CacheView& c, const StageView& s, const AttnMaps& m, int64_t Tq,
                     __nv_bfloat16* out, float scale_log2, Stats* stats, cudaStream_t st) {
    using C = Cfg<D>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(attend_bf16_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid((unsigned)((Tq + kBM - 1) / kBM), (unsigned)c.H);
    attend_bf16_kernel<D><<<grid, kThreads, C::SMEM, st>>>(m.q, m.kc, m.vc, m.ks, m.vs, c.M, c.bias2, c.capP,
                                                           s.sbias, s.T, Tq, c.H, out, scale_log2, stats);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_bf16(const CacheView& c, const StageView& s, const AttnMaps& maps, int64_t Tq,
                               __nv_bfloat16* out, float scale_log2, Stats* stats, cudaStream_t st) {
    return c.d == 128 ? launch_t<128>(c, s, maps, Tq, out, scale_log2, stats, st)
                      : launch_t<64>(c, s, maps, Tq, out, scale_log2, stats, st);
}

}  // namespace tc
