// Biased flash attention over [committed cache | staged chunk] on sm_100a tensor cores.
//
// out_t = sum_j exp(s_tj) v_j / sum_j exp(s_tj), s_tj = scale <q_t,k_j> + ln n_j for
// committed entries (n_j = group size) and + 0 for staged tokens. FAST-AR technical
// summary, section 2.A: Lemma 5.1 makes averaged values with a logit shift by the
// group size exact for identical keys. Computed in base 2: x = s * log2(e).
//
// Three modes share the kernel: self-attention over the TempCache (as above); AnnCA
// cross-attention, where a CTA's keys are the prompt tokens kept for its frame (no
// shift); and AnnSA same-bucket self-attention over a block put in bucket order, where a
// CTA visits only the key tiles spanning its rows' buckets and masks every other bucket.
//
// One CTA = 128 query rows of one head, one CTA per SM (attend_bf16_duo_kernel below):
// tcgen05.mma (kind::f16, cta_group::1) with operands staged by 3-D TMA in 128-byte
// swizzled shared memory and fp32 accumulators in TMEM; two softmax teams on alternate
// key tiles over a three-buffer score ring; one shared output accumulator. Every
// mbarrier wait is bounded (2 s); a timeout sets an error bit and the CTA drains its
// own copies and products before releasing TMEM.
#include "tc_internal.h"

#include <math.h>

namespace tc {

namespace {

constexpr int kBM = 128;                        // query rows per CTA
constexpr int kBN = 128;                        // keys per tile
constexpr int kRK = 3, kRV = 2;                 // K and V ring stages
constexpr int kThreads = 32 * (16 + 4);         // 16 softmax warps, 4 control warps
constexpr uint64_t kTimeoutNs = 2000000000ull;

template <int D>
struct Cfg {
    static constexpr int NB = D / 64;                 // 64-column swizzle boxes per row
    static constexpr int BOX = 128 * 128;             // bytes of one 128-row box
    static constexpr int TILE = NB * BOX;             // bytes of a Q, K or V tile
    static constexpr uint32_t TMEM_COLS = 512;
    // Instruction descriptors, kind::f16: bits 4-5 D format (1 = f32), 7-9 A format
    // (1 = bf16), 10-12 B format (1 = bf16), 15/16 A/B major (0 = K, 1 = MN),
    // 17-22 N>>3, 24-28 M>>4.
    static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                                         ((uint32_t)(kBM >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
};

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

// One arrival worth `count` (a warp arriving for its lanes after a __syncwarp).
__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
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

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait on phase `parity` (a non-suspending test first: the common case is a phase
// that has already completed); false after kTimeoutNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return true;
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

#define TC_LD16(taddr, r)                                                                                    \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];" \
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),    \
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),           \
                   "=r"(r[15])                                                                                       \
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

// Named barrier `id` over `count` threads with an AND of `v` across them.
__device__ __forceinline__ bool bar_and(int id, int count, bool v) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)v), "r"(id), "r"(count)
        : "memory");
    return res != 0;
}

// mbarriers and shared-memory layout: Q tile, K ring (3 stages), V ring (2 stages); per
// team the log2 n row of three tiles [3][128] and their quarter maxima [3][4]; per team
// the halves' reference bounds [2][half][128]; the teams' references [team][128]; the
// epilogue row sums [4][128].
enum { U_QFULL = 0, U_KFULL = 1, U_KEMPTY = 4, U_VFULL = 7, U_VEMPTY = 9, U_SFULL = 11, U_PFULL = 14,
       U_ODONE = 20, U_DRAIN = 23, U_MREADY = 25, U_NBAR = 27 };   // P full: per buffer and half
template <int D>
struct CfgU {
    using C = Cfg<D>;
    static constexpr int TILE = C::TILE;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;
    static constexpr int OFF_V = (1 + kRK) * TILE;
    static constexpr int OFF_BIAS = (1 + kRK + kRV) * TILE;   // [team][3][128] log2 n
    static constexpr int OFF_BMAX = OFF_BIAS + 2 * 3 * 128 * 4; // [team][3][4]
    static constexpr int OFF_UB = OFF_BMAX + 2 * 3 * 4 * 4;     // [team][2][half][128]
    static constexpr int OFF_MREF = OFF_UB + 2 * 2 * 2 * 128 * 4;  // [team][128]
    static constexpr int OFF_L = OFF_MREF + 2 * 128 * 4;        // [4][128]
    static constexpr int OFF_BAR = OFF_L + 4 * 128 * 4;
    static constexpr int OFF_MISC = OFF_BAR + U_NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 32 + 1024;
    static_assert(SMEM <= 232448, "shared memory per block");
    static constexpr uint32_t O_COL = 384;
};

// One CTA = 128 query rows of one head.
//   TMEM: score buffers S_b = [128 b, 128 b + 128) (tile i uses b = i mod 3) and one
//         output accumulator O = [384, 384 + D).
//   warps 0-15  softmax. With the fixed reference (every row's logit bound <= 40, the
//               common case) all sixteen warps take every tile: thread (t, g, r) owns key
//               columns [32 (2 t + g), 32 (2 t + g) + 32) of query row r (TMEM lane r).
//               Otherwise two teams of eight warps: team t takes tiles t, t + 2, ...;
//               thread (t, g, r) owns columns [64 g, 64 g + 64) of query row r, so every
//               SM sub-partition runs two warps of each team and the teams' phases
//               interleave. Per tile the halves agree on an upper bound of
//               the row max (max raw score * scale + max log2 n) at a team barrier.
//               The reference m is shared by both teams and changes lazily: tile i keeps
//               the reference of tile i - 1 (published by the other team through shared
//               memory and an mbarrier) unless its bound exceeds it by more than 8, and
//               then O is rescaled once PV of tile i - 1 has retired. Row sums stay per
//               thread, rescaled when the reference moves. P (bf16) goes over the first
//               32 S columns of each half.
//   warp 16     TMEM allocator; lane 0 TMA producer for Q and the K ring (3 stages).
//   warp 17     lane 0 issues S_b = Q K_i^T once K_i has landed and PV of tile i - 3 has
//               retired (up to three tiles ahead).
//   warp 18     lane 0 TMA producer for the V ring (2 stages).
//   warp 19     lane 0 issues O += P_i V_i in tile order.
enum { kSelf = 0, kCross = 1, kSparse = 2, kFrames = 3 };   // kernel modes (see the prologue)

// A bucket code as a float's bits -> logit shift 0 when it equals the row's code, else
// -inf (same-bucket mask of the sparse mode).
__device__ __forceinline__ float4 mask4(float4 c, uint32_t gq) {
    return make_float4(__float_as_uint(c.x) == gq ? 0.f : -INFINITY, __float_as_uint(c.y) == gq ? 0.f : -INFINITY,
                       __float_as_uint(c.z) == gq ? 0.f : -INFINITY, __float_as_uint(c.w) == gq ? 0.f : -INFINITY);
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
attend_bf16_duo_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                       const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKs,
                       const __grid_constant__ CUtensorMap tmVs, const int32_t* __restrict__ Mdev,
                       const float* __restrict__ bias2, const float* __restrict__ kmax2c,
                       const float* __restrict__ kmax2s, const float* __restrict__ bmaxh, int64_t capP,
                       const float* __restrict__ sbias, int64_t Ts, int64_t Tq, int H, int Pf, int Ff,
                       const SparseArgs sp, const FrameArgs fa, __nv_bfloat16* __restrict__ out, float scale_log2,
                       Stats* stats) {
    constexpr bool CROSS = MODE == kCross;
    constexpr bool SPARSE = MODE == kSparse;
    constexpr bool FRAMES = MODE == kFrames;
    using C = Cfg<D>;
    using L = CfgU<D>;
    constexpr int kWK = 16, kWQK = 17, kWV = 18, kWPV = 19;
    constexpr int QC = D / 4;   // output columns per softmax thread
    constexpr int HC = D / 2;   // O columns a half rescales
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    float* sBias = reinterpret_cast<float*>(smem + L::OFF_BIAS);
    float* sBmax = reinterpret_cast<float*>(smem + L::OFF_BMAX);
    float* sUb = reinterpret_cast<float*>(smem + L::OFF_UB);
    float* sMref = reinterpret_cast<float*>(smem + L::OFF_MREF);
    float* sL = reinterpret_cast<float*>(smem + L::OFF_L);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    volatile int* sFixed = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8);   // fixed reference in use

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    // Self-attention: CTA x covers query rows [128 x, 128 x + 128) of all Tq, the keys
    // are committed entries (slot h of the cache arrays) then staged tokens.
    // Cross-attention: the query rows are Ff frames of Pf rows; CTA x covers rows of one
    // frame f, and the keys are the kept prompt tokens of slot h Ff + f, nothing staged.
    // Sparse (same-bucket) self-attention: rows are in bucket order (packed, head-major);
    // CTA x covers packed rows [128 x, 128 x + 128) of head h, the keys are the packed
    // tiles [kt0, kt1) that hold its rows' buckets, masked per element to the same bucket.
    // Frame mask (LVSA): the query rows are frames of Pf rows; CTA x covers rows of one
    // frame f, and its keys are the token-major tiles listed for f (the frames f attends
    // to, each run of consecutive frames tiled from its first row), rows past a run's end
    // shifted by -inf.
    int q0, zc, kt0 = 0, nsp = 0;
    int64_t qend;
    const int2* ftab = nullptr;
    if constexpr (FRAMES) {
        asm volatile("griddepcontrol.wait;" ::: "memory");   // the tile lists of this call
        const int tpf = (Pf + kBM - 1) / kBM;
        const int f = blockIdx.x / tpf;
        q0 = f * Pf + (blockIdx.x - f * tpf) * kBM;
        qend = (int64_t)(f + 1) * Pf;
        zc = h;
        ftab = fa.tiles + (int64_t)f * fa.maxt;
        nsp = fa.count[f];
    } else if constexpr (SPARSE) {
        asm volatile("griddepcontrol.wait;" ::: "memory");   // the packing kernel's output
        q0 = blockIdx.x * kBM;
        qend = Tq;
        zc = h;
        const int2 kr = sp.tiles[(int64_t)h * sp.nqt + blockIdx.x];
        kt0 = kr.x;
        nsp = kr.y - kr.x;
    } else if constexpr (CROSS) {
        // launched as a programmatic dependent of the kernel that packs the keys: wait
        // for it before reading anything it writes
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const int tpf = (Pf + kBM - 1) / kBM;
        const int f = blockIdx.x / tpf;
        q0 = f * Pf + (blockIdx.x - f * tpf) * kBM;
        qend = (int64_t)(f + 1) * Pf;
        zc = h * Ff + f;
    } else {
        q0 = blockIdx.x * kBM;
        qend = Tq;
        zc = h;
    }
    const int nc = (SPARSE || FRAMES) ? nsp : (Mdev[zc] + kBN - 1) / kBN;
    const int ntiles = nc + ((CROSS || SPARSE || FRAMES) ? 0 : (int)((Ts + kBN - 1) / kBN));
    if constexpr (CROSS) {
        if (ntiles == 0) {   // no key: the rows are the empty sum, zero
            constexpr int W = D / 8;   // 16-byte words per row
            for (int i = threadIdx.x; i < kBM * W; i += kThreads) {
                const int64_t row = q0 + i / W;
                if (row < qend)
                    reinterpret_cast<uint4*>(out + (row * H + h) * D)[i % W] = make_uint4(0u, 0u, 0u, 0u);
            }
            asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
            asm volatile("griddepcontrol.wait;" ::: "memory");
            return;
        }
    }

    if (threadIdx.x == 0) {
        mbar_init(&bars[U_QFULL], 1);
        for (int s2 = 0; s2 < kRK; ++s2) {
            mbar_init(&bars[U_KFULL + s2], 1);
            mbar_init(&bars[U_KEMPTY + s2], 1);
        }
        for (int s2 = 0; s2 < kRV; ++s2) {
            mbar_init(&bars[U_VFULL + s2], 1);
            mbar_init(&bars[U_VEMPTY + s2], 1);
        }
        for (int b = 0; b < 3; ++b) {
            mbar_init(&bars[U_SFULL + b], 1);
            mbar_init(&bars[U_PFULL + 2 * b], 128);
            mbar_init(&bars[U_PFULL + 2 * b + 1], 128);
            mbar_init(&bars[U_ODONE + b], 1);
        }
        mbar_init(&bars[U_DRAIN], 1);
        mbar_init(&bars[U_DRAIN + 1], 1);
        mbar_init(&bars[U_MREADY], 128);
        mbar_init(&bars[U_MREADY + 1], 128);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kWK) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const uint32_t tO = tmem + L::O_COL;
    uint8_t* sQ = smem + L::OFF_Q;
    uint8_t* sK = smem + L::OFF_K;
    uint8_t* sV = smem + L::OFF_V;

    if ((warp == kWK || warp == kWV) && lane == 0) {
        // ---------------------------------------------------------------- TMA producers
        const bool kside = warp == kWK;
        const int nst = kside ? kRK : kRV;
        uint8_t* ring = kside ? sK : sV;
        uint64_t* full = &bars[kside ? U_KFULL : U_VFULL];
        uint64_t* empty = &bars[kside ? U_KEMPTY : U_VEMPTY];
        const CUtensorMap* mc = kside ? &tmKc : &tmVc;
        const CUtensorMap* ms = kside ? &tmKs : &tmVs;
        if (kside) {
            mbar_expect_tx(&bars[U_QFULL], C::TILE);
            for (int b = 0; b < C::NB; ++b) {
                if constexpr (SPARSE)   // packed queries, head-major
                    tma_load_3d(sQ + b * C::BOX, &tmQ, 64 * b, q0, h, &bars[U_QFULL]);
                else
                    tma_load_3d(sQ + b * C::BOX, &tmQ, 64 * b, h, q0, &bars[U_QFULL]);
            }
        }
        int last = -1;
        for (int i = 0; i < ntiles && !*abort_flag; ++i) {
            const int st = i % nst;
            if (i >= nst && !mbar_wait(&empty[st], ((i / nst) - 1) & 1)) { *abort_flag = 1; break; }
            const bool cache = i < nc;
            mbar_expect_tx(&full[st], C::TILE);
            if constexpr (FRAMES) {   // token-major keys and values
                const int row0 = ftab[i].x;
                for (int b = 0; b < C::NB; ++b)
                    tma_load_3d(ring + st * C::TILE + b * C::BOX, mc, 64 * b, h, row0, &full[st]);
            } else {
                const int row0 = ((cache ? i : i - nc) + kt0) * kBN;
                for (int b = 0; b < C::NB; ++b)
                    tma_load_3d(ring + st * C::TILE + b * C::BOX, cache ? mc : ms, 64 * b, row0, cache ? zc : h,
                                &full[st]);
            }
            last = i;
        }
        if (kside) mbar_wait(&bars[U_QFULL], 0);
        for (int i = (last >= nst - 1 ? last - nst + 1 : 0); i <= last; ++i) mbar_wait(&full[i % nst], (i / nst) & 1);
    } else if (warp == kWQK && lane == 0) {
        // ---------------------------------------------------------------- QK issuer
        const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
        bool ok = mbar_wait(&bars[U_QFULL], 0);
        for (int j = 0; ok && j < ntiles && !*abort_flag; ++j) {
            const int b = j % 3, st = j % kRK;
            if (j >= 3 && !mbar_wait(&bars[U_ODONE + b], ((j - 3) / 3) & 1)) { ok = false; break; }
            if (!mbar_wait(&bars[U_KFULL + st], (j / kRK) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t aKs = aK + st * C::TILE;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                mma_ss(tmem + b * 128, sdesc(aQ + off, 16, 1024), sdesc(aKs + off, 16, 1024), C::IDESC_QK, kk > 0);
            }
            tc_commit(&bars[U_SFULL + b]);
            tc_commit(&bars[U_KEMPTY + st]);
        }
        if (!ok) *abort_flag = 1;
        tc_commit(&bars[U_DRAIN]);
        mbar_wait(&bars[U_DRAIN], 0);
    } else if (warp == kWPV && lane == 0) {
        // ---------------------------------------------------------------- PV issuer
        // O += P_i V_i. With the online reference keys [16 kk, 16 kk + 16) of P sit at
        // column 128 b + 64 (kk / 4) + 8 (kk % 4), each half's probabilities over its own
        // first S columns, and both halves must be done (a tile may rescale all of O
        // first). With the fixed reference they sit at 128 b + 32 (kk / 2) + 8 (kk % 2),
        // each quarter's over its own first columns, and the keys of quarters 0-1 go in as
        // soon as those are written.
        const uint32_t aV = smem_u32(sV);
        bool ok = true, fixed = false;
        for (int i = 0; i < ntiles && !*abort_flag; ++i) {
            const int b = i % 3, st = i % kRV;
            if (!mbar_wait(&bars[U_PFULL + 2 * b], (i / 3) & 1)) { ok = false; break; }
            if (i == 0) fixed = *sFixed != 0;   // written before the first P
            if (!fixed && !mbar_wait(&bars[U_PFULL + 2 * b + 1], (i / 3) & 1)) { ok = false; break; }
            if (!mbar_wait(&bars[U_VFULL + st], (i / kRV) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t aVs = aV + st * C::TILE;
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
                if (kk == 4 && fixed) {
                    if (!mbar_wait(&bars[U_PFULL + 2 * b + 1], (i / 3) & 1)) { ok = false; break; }
                    tc_fence_after();
                }
                const uint32_t pcol = fixed ? 32 * (kk >> 1) + 8 * (kk & 1) : 64 * (kk >> 2) + 8 * (kk & 3);
                mma_ts(tO, tmem + b * 128 + pcol, sdesc(aVs + kk * 2048, C::BOX, 1024), C::IDESC_PV,
                       (i > 0 || kk > 0));
            }
            if (!ok) break;
            tc_commit(&bars[U_VEMPTY + st]);
            tc_commit(&bars[U_ODONE + b]);
        }
        if (!ok) *abort_flag = 1;
        tc_commit(&bars[U_DRAIN + 1]);
        mbar_wait(&bars[U_DRAIN + 1], 0);
    } else if (warp < 16) {
        // ---------------------------------------------------------------- softmax teams
        const int t = warp >> 3;             // team
        const int g = (warp >> 2) & 1;       // half: columns [64 g, 64 g + 64)
        const int wt = warp & 3;             // TMEM lane quarter (= SM sub-partition)
        const int r = wt * 32 + lane;        // query row within the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(wt * 32) << 16;
        const uint32_t tOh = tO + HC * g + lane_base;
        // (sparse mode: the "bias" rows are the packed rows' bucket codes, as float bits,
        // and turn into 0 / -inf by comparison with the row's own code gq)
        const float* bias_h = SPARSE ? reinterpret_cast<const float*>(sp.grp) + (int64_t)h * sp.Tp + (int64_t)kt0 * kBN
                                     : bias2 + (int64_t)zc * capP;
        const uint32_t gq = SPARSE ? sp.grp[(int64_t)h * sp.Tp + q0 + r] : 0u;
        auto bias_of = [&](int i) -> float {
            if constexpr (FRAMES) return fa.masktab[ftab[i].y * kBN + r];
            return (i < nc) ? bias_h[(int64_t)i * kBN + r] : sbias[(int64_t)(i - nc) * kBN + r];
        };
        // Half 0 stages the log2 n row of each of its team's tiles and its quarter maxima
        // (three buffers: a fast thread may stage two tiles ahead of a slow one's reads).
        auto stage_bias = [&](int buf, float v) {
            sBias[(t * 3 + buf) * 128 + r] = v;
            float wm = v;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
            if (lane == 0) sBmax[(t * 3 + buf) * 4 + wt] = wm;
        };
        const uint64_t c2 = pk2(scale_log2, scale_log2);
        float m_run = -INFINITY, l_run = 0.f;   // l_run is relative to m_run
        // A fixed reference per row from the Cauchy-Schwarz bound of its logits,
        //   |x_j - log2 n_j| = |s_j| scale log2 e <= |q| max|k| scale log2 e,   log2 n_j >= 0,
        // rounded up past the fp32 errors of the norms and of the product (mfix below, which
        // adds max log2 n). When every row of the CTA has mfix <= 40, every unmasked logit
        // lies in [-40, 40]: p = 2^x needs no reference at all (the reference 0), cannot
        // overflow (p <= 2^40, a row sum <= 2^40 times the key count) and is never near the
        // fp32 flush to zero (p >= 2^-40), so the tiles need no max pass, no agreement
        // between threads and no rescaling. Otherwise the CTA runs the lazy online
        // reference below.
        bool ok = mbar_wait(&bars[U_QFULL], 0);
        float q2 = 0.f;
        {
            const uint8_t* qrow = sQ + r * 128;
#pragma unroll 1
            for (int bx = 0; bx < C::NB; ++bx) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 w4 = *reinterpret_cast<const uint4*>(qrow + bx * C::BOX + ((ch ^ (r & 7)) << 4));
                    const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float lo = __uint_as_float(wd[e2] << 16), hi = __uint_as_float(wd[e2] & 0xffff0000u);
                        q2 = fmaf(lo, lo, fmaf(hi, hi, q2));
                    }
                }
            }
        }
        const float mfix = sqrtf(q2 * fmaxf(kmax2c[h], kmax2s[0])) * scale_log2 * (1.f + 1.f / 256.f) +
                           bmaxh[h] + 1.f / 256.f;
        const bool fixed = bar_and(3, 512, ok && mfix <= 40.f);   // uniform over the CTA
        if (threadIdx.x == 0) *sFixed = fixed ? 1 : 0;             // before thread 0's first P
        if (fixed) {
            // No max pass and no agreement between threads: all sixteen warps take every
            // tile, thread (t, g, r) the key columns [32 (2 t + g), 32 (2 t + g) + 32) of row
            // r, so a tile's exponentials spread over the whole SM. P goes over the first 16
            // columns of each quarter; the PV issuer starts the keys of quarters 0-1 (team 0)
            // once those are written.
            m_run = 0.f;
            const int qc = 32 * (2 * t + g);
            auto bias_row = [&](int i) -> const float* {
                if constexpr (FRAMES) return fa.masktab + ftab[i].y * kBN + qc;
                return ((i < nc) ? bias_h + (int64_t)i * kBN : sbias + (int64_t)(i - nc) * kBN) + qc;
            };
            if (lane == 0 && ntiles > 0) asm volatile("prefetch.global.L1 [%0];" ::"l"(bias_row(0)));
            uint64_t sumA = pk2(0.f, 0.f), sumB = pk2(0.f, 0.f);
            for (int i = 0; i < ntiles; ++i) {
                const int b = i % 3;
                const bool got = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&bars[U_SFULL + b], (i / 3) & 1));
                if (!got) { ok = false; *abort_flag = 1; break; }
                tc_fence_after();
                if (lane == 0 && i + 1 < ntiles) asm volatile("prefetch.global.L1 [%0];" ::"l"(bias_row(i + 1)));
                const uint32_t tS = tmem + b * 128 + qc + lane_base;
                const float4* brow = reinterpret_cast<const float4*>(bias_row(i));   // (codes when sparse)
                uint32_t sr[32];
                TC_LD32(tS, sr);
                tc_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 b4 = __ldg(brow + j / 4);
                    if constexpr (SPARSE) b4 = mask4(b4, gq);
                    const uint64_t x01 =
                        fma2(pk2(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), c2, pk2(b4.x, b4.y));
                    const uint64_t x23 =
                        fma2(pk2(__uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3])), c2, pk2(b4.z, b4.w));
                    float a0, a1, a2, a3;
                    up2(x01, a0, a1);
                    up2(x23, a2, a3);
                    const float p0 = ex2(a0), p1 = ex2(a1), p2 = ex2(a2), p3 = ex2(a3);
                    sumA = add2(sumA, pk2(p0, p1));
                    sumB = add2(sumB, pk2(p2, p3));
                    pk[j / 2] = cvt_bf16x2(p0, p1);
                    pk[j / 2 + 1] = cvt_bf16x2(p2, p3);
                }
                TC_ST16(tS, pk);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_n(&bars[U_PFULL + 2 * b + t], 16);   // 8 warps x 16 = 128
            }
            float s0, s1, s2, s3;
            up2(sumA, s0, s1);
            up2(sumB, s2, s3);
            l_run = (s0 + s1) + (s2 + s3);
        } else {
        float bnext = 0.f;
        if (g == 0) {
            if (t < ntiles) stage_bias(0, bias_of(t));
            if (t + 2 < ntiles) bnext = bias_of(t + 2);
        }
        ok = bar_and(1 + t, 256, true) && ok;
        int k = 0;
        for (int i = t; i < ntiles; i += 2, ++k) {
            const int b = i % 3, bb = k % 3, u = k & 1;
            // (warp-uniform: the TMEM loads below are warp-collective)
            const bool got = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&bars[U_SFULL + b], (i / 3) & 1));
            tc_fence_after();
            const uint32_t tS = tmem + b * 128 + 64 * g + lane_base;
            float smax = -INFINITY;
            if (got) {
                uint32_t sr[64];
                TC_LD32(tS, (sr + 0));
                TC_LD32(tS + 32, (sr + 32));
                tc_wait_ld();
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if constexpr (SPARSE) {   // only the row's own bucket counts towards its bound
                    const float* ch = sBias + (t * 3 + bb) * 128 + 64 * g;
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (__float_as_uint(ch[j]) != gq) sr[j] = __float_as_uint(-INFINITY);
                }
                if constexpr (FRAMES) {   // rows of frames outside A(t) do not count either
                    const float* ch = sBias + (t * 3 + bb) * 128 + 64 * g;
#pragma unroll
                    for (int j = 0; j < 64; ++j) sr[j] = __float_as_uint(__uint_as_float(sr[j]) + ch[j]);
                }
#pragma unroll
                for (int j = 0; j < 64; j += 8) {
                    m4[0] = max3(m4[0], __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
                    m4[1] = max3(m4[1], __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]));
                    m4[2] = max3(m4[2], __uint_as_float(sr[j + 4]), __uint_as_float(sr[j + 5]));
                    m4[3] = max3(m4[3], __uint_as_float(sr[j + 6]), __uint_as_float(sr[j + 7]));
                }
                smax = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
            }
            const float2 bm = (SPARSE || FRAMES) ? make_float2(0.f, 0.f)
                                                 : *reinterpret_cast<const float2*>(sBmax + (t * 3 + bb) * 4 + 2 * g);
            sUb[((t * 2 + u) * 2 + g) * 128 + r] = fmaf(smax, scale_log2, fmaxf(bm.x, bm.y));
            if (g == 0 && i + 2 < ntiles) stage_bias((k + 1) % 3, bnext);
            if (!bar_and(1 + t, 256, got)) { ok = false; break; }
            if (g == 0 && i + 4 < ntiles) bnext = bias_of(i + 4);
            const float ub = fmaxf(sUb[((t * 2 + u) * 2 + 0) * 128 + r], sUb[((t * 2 + u) * 2 + 1) * 128 + r]);
            // The reference of tile i - 1, decided by the other team. In the sparse mode a
            // tile may hold no key of a row's bucket (bound -inf), so the first reference
            // is the row's own logit, which is finite and never above the row's maximum.
            float mprev = SPARSE ? sp.xself[(int64_t)h * sp.Tp + q0 + r] : -INFINITY;
            if (i > 0) {
                const bool w = mbar_wait(&bars[U_MREADY + (t ^ 1)], ((i - 1) >> 1) & 1);
                if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; }
                mprev = sMref[(t ^ 1) * 128 + r];
            }
            const bool raise = (!SPARSE && i == 0) || ub > mprev + 8.f;
            const float mnew = raise ? ub : mprev;
            if (g == 0) {
                sMref[t * 128 + r] = mnew;
                mbar_arrive(&bars[U_MREADY + t]);
            }
            // O holds tiles < i relative to mprev: rescale it once PV of tile i - 1 retired.
            if (i > 0 && __any_sync(0xffffffffu, raise)) {
                const bool w = mbar_wait(&bars[U_ODONE + (i - 1) % 3], ((i - 1) / 3) & 1);
                if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; }
                if (ok) {
                    const float alpha = raise ? ex2(mprev - mnew) : 1.f;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < HC / 32; ++c) {
                        uint32_t o[32];
                        TC_LD32(tOh + 32 * c, o);
                        tc_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
                        TC_ST32(tOh + 32 * c, o);
                    }
                    tc_wait_st();
                }
            }
            if (mnew != m_run) {   // my row sum follows the reference
                l_run = (l_run > 0.f) ? l_run * ex2(m_run - mnew) : 0.f;
                m_run = mnew;
            }
            // p = 2^(s * scale + log2 n - m) over my 64 columns in two chunks of 32.
            const uint64_t negm2 = pk2(-m_run, -m_run);
            uint64_t sumA = pk2(0.f, 0.f), sumB = pk2(0.f, 0.f);
            const float* bh = sBias + (t * 3 + bb) * 128 + 64 * g;
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t sr[32];
                TC_LD32(tS + 32 * h2, sr);
                tc_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 b4 = *reinterpret_cast<const float4*>(bh + 32 * h2 + j);
                    if constexpr (SPARSE) b4 = mask4(b4, gq);
                    const uint64_t x01 = fma2(pk2(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), c2,
                                              add2(pk2(b4.x, b4.y), negm2));
                    const uint64_t x23 = fma2(pk2(__uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3])), c2,
                                              add2(pk2(b4.z, b4.w), negm2));
                    float a0, a1, a2, a3;
                    up2(x01, a0, a1);
                    up2(x23, a2, a3);
                    const float p0 = ex2(a0), p1 = ex2(a1), p2 = ex2(a2), p3 = ex2(a3);
                    sumA = add2(sumA, pk2(p0, p1));
                    sumB = add2(sumB, pk2(p2, p3));
                    pk[j / 2] = cvt_bf16x2(p0, p1);
                    pk[j / 2 + 1] = cvt_bf16x2(p2, p3);
                }
                TC_ST16(tS + 16 * h2, pk);
            }
            float s0, s1, s2, s3;
            up2(sumA, s0, s1);
            up2(sumB, s2, s3);
            l_run += (s0 + s1) + (s2 + s3);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[U_PFULL + 2 * b + g]);
        }
        }
        // Epilogue: the last product retires (each commit covers every earlier product of
        // the PV issuer), every row sum moves to the final reference, and thread (t, g, r)
        // writes output columns [QC (2 t + g), QC (2 t + g + 1)) of its row.
        const int lastt = ntiles - 1;
        bool fin = ok && mbar_wait(&bars[U_ODONE + lastt % 3], (lastt / 3) & 1);
        float mfin = 0.f;   // (the fixed reference)
        if (!fixed) {
            fin = fin && mbar_wait(&bars[U_MREADY + (lastt & 1)], (lastt >> 1) & 1);
            mfin = sMref[(lastt & 1) * 128 + r];
        }
        const float lfin = (l_run > 0.f) ? l_run * ex2(m_run - mfin) : 0.f;
        sL[(t * 2 + g) * 128 + r] = lfin;
        if (bar_and(3, 512, fin)) {
            const float inv = 1.f / ((sL[0 * 128 + r] + sL[1 * 128 + r]) + (sL[2 * 128 + r] + sL[3 * 128 + r]));
            tc_fence_after();
            const int col = QC * (2 * t + g);
            uint32_t o[QC];
            if constexpr (QC == 32) TC_LD32(tO + lane_base + col, o);
            else TC_LD16(tO + lane_base + col, o);
            tc_wait_ld();
            const int64_t row = q0 + r;
            if (row < qend) {
                const int64_t tok = SPARSE ? (int64_t)sp.perm[(int64_t)h * sp.Tp + row] : row;
                uint4* dst = reinterpret_cast<uint4*>(out + (tok * H + h) * D + col);
#pragma unroll
                for (int v = 0; v < QC / 8; ++v) {
                    uint4 w4;
                    w4.x = cvt_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                    w4.y = cvt_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                    w4.z = cvt_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                    w4.w = cvt_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
                    dst[v] = w4;
                }
            }
        } else {
            *abort_flag = 1;
        }
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(&stats->error_bits, 2u);
    tc_fence_before();
    __syncthreads();
    if (warp == kWK) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D, int MODE>
cudaError_t set_smem_attr() {
    return smem_attr_once(reinterpret_cast<const void*>(attend_bf16_duo_kernel<D, MODE>), CfgU<D>::SMEM);
}

template <int D>
cudaError_t launch_t(const CacheView& c, const StageView& s, const AttnMaps& m, int64_t Tq, __nv_bfloat16* out,
                     float scale_log2, Stats* stats, bool overlap_prev, cudaStream_t st) {
    cudaError_t e = set_smem_attr<D, kSelf>();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((Tq + kBM - 1) / kBM), (unsigned)c.H);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = CfgU<D>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = overlap_prev ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attend_bf16_duo_kernel<D, kSelf>, m.q, m.kc, m.vc, m.ks, m.vs,
                              (const int32_t*)c.M, (const float*)c.bias2, (const float*)c.kmax2,
                              (const float*)c.kmax2s, (const float*)c.bmax, c.capP, (const float*)s.sbias, s.T, Tq,
                              c.H, (int)Tq, 1, SparseArgs{}, FrameArgs{}, out, scale_log2, stats);
}

// Cross-attention over the kept prompt tokens: grid (F frames x tiles per frame, H),
// launched as a programmatic dependent of the packing kernel (the kernel waits for it
// before its first read).
template <int D>
cudaError_t launch_cross_t(const AnnView& a, const AttnMaps& m, int64_t Tq, int P, int F, __nv_bfloat16* out,
                           float scale_log2, Stats* stats, cudaStream_t st) {
    cudaError_t e = set_smem_attr<D, kCross>();
    if (e != cudaSuccess) return e;
    const int tpf = (P + kBM - 1) / kBM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(F * tpf), (unsigned)a.H);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = CfgU<D>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attend_bf16_duo_kernel<D, kCross>, m.q, m.kc, m.vc, m.kc, m.vc,
                              (const int32_t*)a.nsel, (const float*)a.sbias, (const float*)a.kmax2,
                              (const float*)a.zeros, (const float*)a.zeros, a.Lp, (const float*)nullptr, (int64_t)0,
                              Tq, a.H, P, F, SparseArgs{}, FrameArgs{}, out, scale_log2, stats);
}

// Same-bucket self-attention over packed rows: grid (query tiles, H), a programmatic
// dependent of the packing kernel.
template <int D>
cudaError_t launch_sparse_t(int H, const SparseArgs& sp, const AttnMaps& m, int64_t T, const float* kmax2,
                            const float* zeros, __nv_bfloat16* out, float scale_log2, Stats* stats,
                            cudaStream_t st) {
    cudaError_t e = set_smem_attr<D, kSparse>();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((T + kBM - 1) / kBM), (unsigned)H);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = CfgU<D>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attend_bf16_duo_kernel<D, kSparse>, m.q, m.kc, m.vc, m.kc, m.vc,
                              (const int32_t*)nullptr, (const float*)nullptr, kmax2, zeros, zeros, sp.Tp,
                              (const float*)nullptr, (int64_t)0, T, H, (int)T, 1, sp, FrameArgs{}, out, scale_log2,
                              stats);
}

// Frame-masked attention over token-major Q, K, V: grid (T frames x tiles per frame, H), a
// programmatic dependent of the kernels that list the tiles and bound the keys. `big` holds
// the per-head bound of |k|^2 (read as big[h]) and `zeros` H zeros (no group sizes, no
// staged keys): rows whose logit bound stays small take the fixed softmax reference.
template <int D>
cudaError_t launch_frames_t(int H, const FrameArgs& fa, const AttnMaps& m, int T, int P, const float* big,
                            const float* zeros, __nv_bfloat16* out, float scale_log2, Stats* stats,
                            cudaStream_t st) {
    cudaError_t e = set_smem_attr<D, kFrames>();
    if (e != cudaSuccess) return e;
    const int tpf = (P + kBM - 1) / kBM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(T * tpf), (unsigned)H);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = CfgU<D>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int64_t N = (int64_t)T * P;
    return cudaLaunchKernelEx(&cfg, attend_bf16_duo_kernel<D, kFrames>, m.q, m.kc, m.vc, m.kc, m.vc,
                              (const int32_t*)nullptr, (const float*)nullptr, big, zeros, zeros, (int64_t)0,
                              (const float*)nullptr, (int64_t)0, N, H, P, T, SparseArgs{}, fa, out, scale_log2,
                              stats);
}

}  // namespace

cudaError_t launch_attend_bf16(const CacheView& c, const StageView& s, const AttnMaps& maps, int64_t Tq,
                               __nv_bfloat16* out, float scale_log2, Stats* stats, bool overlap_prev,
                               cudaStream_t st) {
    return c.d == 128 ? launch_t<128>(c, s, maps, Tq, out, scale_log2, stats, overlap_prev, st)
                      : launch_t<64>(c, s, maps, Tq, out, scale_log2, stats, overlap_prev, st);
}

cudaError_t launch_attend_cross_bf16(const AnnView& a, const AttnMaps& maps, int64_t Tq, int P, int F,
                                     __nv_bfloat16* out, float scale_log2, Stats* stats, cudaStream_t st) {
    return a.d == 128 ? launch_cross_t<128>(a, maps, Tq, P, F, out, scale_log2, stats, st)
                      : launch_cross_t<64>(a, maps, Tq, P, F, out, scale_log2, stats, st);
}

cudaError_t launch_attend_frames_bf16(int H, int d, const FrameArgs& fa, const AttnMaps& maps, int T, int P,
                                      const float* big, const float* zeros, __nv_bfloat16* out, float scale_log2,
                                      Stats* stats, cudaStream_t st) {
    return d == 128 ? launch_frames_t<128>(H, fa, maps, T, P, big, zeros, out, scale_log2, stats, st)
                    : launch_frames_t<64>(H, fa, maps, T, P, big, zeros, out, scale_log2, stats, st);
}

cudaError_t launch_attend_sparse_bf16(int H, int d, const SparseArgs& sp, const AttnMaps& maps, int64_t T,
                                      const float* kmax2, const float* zeros, __nv_bfloat16* out,
                                      float scale_log2, Stats* stats, cudaStream_t st) {
    return d == 128 ? launch_sparse_t<128>(H, sp, maps, T, kmax2, zeros, out, scale_log2, stats, st)
                    : launch_sparse_t<64>(H, sp, maps, T, kmax2, zeros, out, scale_log2, stats, st);
}

}  // namespace tc
