// Biased flash attention over [committed cache | staged chunk] on sm_100a tensor cores.
//
// out_t = sum_j exp(s_tj) v_j / sum_j exp(s_tj), s_tj = scale <q_t,k_j> + ln n_j for
// committed entries (n_j = group size) and + 0 for staged tokens. FAST-AR technical
// summary, section 2.A: Lemma 5.1 makes averaged values with a logit shift by the
// group size exact for identical keys. Computed in base 2: x = s * log2(e).
//
// One CTA = 128 query rows of one head and owns the SM's 512 TMEM columns:
//   S_b = [128 b, 128 b + 128), b < kSBuf   scores of key tile i, b = i mod kSBuf;
//                                           P (bf16) overwrites the first 64 columns
//   O   = [128 kSBuf, 128 kSBuf + D)        fp32 output accumulator
//   Q   = [384, 448) when kQinTmem          the query tile as the A operand of QK
// The MMA issuer starts S_{i+1} = Q K_{i+1}^T before O += P_i V_i, so the tensor
// core computes the next scores while softmax works on P_i; with three buffers the
// buffer S_{i+1} overwrites held P_{i-2}, whose product retired long before.
// Warp roles (288 threads):
//   warps 0-7  softmax, two warpgroups: thread (g, r) owns columns [64g, 64g+64) of
//              query row r (TMEM lane r), so every SM sub-partition runs two softmax
//              warps. One pass per key tile with an upper-bound reference max (the
//              halves exchange partial maxima in shared memory), lazy rescaling of O
//              (only when the reference grows by more than 2^8), P written as bf16.
//   warp 8     TMEM allocator; lane 0 is the TMA producer for Q and the K ring
//              (2 stages), lane 1 the producer for the V ring, lane 2 the MMA issuer.
//              The three lanes run independent loops.
// Operands come by 3-D TMA (64-column, 128-byte-swizzled boxes) straight from the
// token-major Q and the head-major cache/staging buffers. Every mbarrier wait is
// bounded (2 s); a timeout sets an error bit and the CTA drains its own copies and
// MMAs before releasing TMEM.
#include "tc_internal.h"

#include <math.h>

#ifndef TC_ATTN_SBUF
#define TC_ATTN_SBUF 3
#endif
#ifndef TC_ATTN_POLY
#define TC_ATTN_POLY 0
#endif
#ifndef TC_ATTN_QTMEM
#define TC_ATTN_QTMEM 0
#endif
#ifndef TC_ATTN_CTLWARPS
#define TC_ATTN_CTLWARPS 3
#endif
#ifndef TC_ATTN_TEAMS
#define TC_ATTN_TEAMS 2
#endif
#ifndef TC_ATTN_SCHED
#define TC_ATTN_SCHED 0
#endif
#ifndef TC_ATTN_KST
#define TC_ATTN_KST 2
#endif
#ifndef TC_ATTN_VST
#define TC_ATTN_VST 2
#endif
#ifndef TC_ATTN_SPLIT
#define TC_ATTN_SPLIT 0
#endif
#ifndef TC_ATTN_RING
#define TC_ATTN_RING 0
#endif
#ifndef TC_ATTN_DUO
#define TC_ATTN_DUO 1
#endif
#ifndef TC_ATTN_ONEPASS
#define TC_ATTN_ONEPASS 0
#endif

namespace tc {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
// Control warps after the 8 softmax warps: with 3, the K producer (and TMEM
// allocator), the MMA issuer and the V producer each have a warp; with 2, the two
// producers share warp 8 (lanes 0 and 1); with 1, the MMA issuer is lane 2 of it.
constexpr int kCtlWarps = TC_ATTN_CTLWARPS;
constexpr int kThreads = 32 * (8 + kCtlWarps);
constexpr int kWarpCtl = 8;                                      // K producer, allocator
constexpr int kWarpMma = kCtlWarps >= 2 ? 9 : 8;
constexpr int kLaneMma = kCtlWarps >= 2 ? 0 : 2;
constexpr int kWarpV = kCtlWarps == 3 ? 10 : 8;
constexpr int kLaneV = kCtlWarps == 3 ? 0 : 1;
constexpr int kSBuf = TC_ATTN_SBUF;            // score buffers in TMEM (2 or 3)
constexpr bool kPoly = TC_ATTN_POLY != 0;       // part of the exponentials on the FMA pipe
constexpr bool kQinTmem = TC_ATTN_QTMEM != 0;   // Q as a TMEM operand (needs kSBuf == 2)
constexpr int kTeams = TC_ATTN_TEAMS;          // 2: teams on alternate key tiles
constexpr int kSched = TC_ATTN_SCHED;          // MMA issue: 0 blocking, 1 polling, 2 polling with backoff
constexpr int kKSt = TC_ATTN_KST;               // K ring stages
constexpr int kVSt = TC_ATTN_VST;               // V ring stages
constexpr bool kSplit = TC_ATTN_SPLIT != 0;      // teams with two threads per query row
constexpr int kThreadsSplit = 32 * (16 + 3);
constexpr bool kRing = TC_ATTN_RING != 0;        // one query tile, 16 softmax warps, three S buffers
constexpr int kThreadsRing = 32 * (16 + 4);
constexpr bool kDuo = TC_ATTN_DUO != 0;          // two teams over the ring, one shared O
constexpr bool kOnePass = TC_ATTN_ONEPASS != 0;  // teams: S read from TMEM once per tile, into registers
static_assert(kSBuf == 2 || kSBuf == 3, "two or three score buffers");
static_assert(kKSt >= 2 && kKSt <= 4 && kVSt >= 2 && kVSt <= 4, "ring depths");
static_assert(!kQinTmem || kSBuf == 2, "Q in TMEM leaves room for two score buffers");
constexpr uint64_t kTimeoutNs = 2000000000ull;

template <int D>
struct Cfg {
    static constexpr int NB = D / 64;                 // 64-column swizzle boxes per row
    static constexpr int BOX = 128 * 128;             // bytes of one 128-row box
    static constexpr int TILE = NB * BOX;             // bytes of a Q, K or V tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;                      // kKSt stages
    static constexpr int OFF_V = (1 + kKSt) * TILE;         // kVSt stages
    static constexpr int OFF_BIAS = (1 + kKSt + kVSt) * TILE;  // 2 x 128 floats
    static constexpr int OFF_BMAX = OFF_BIAS + 2 * 128 * 4;      // 2 x 4 floats
    static constexpr int OFF_PMAX = OFF_BMAX + 2 * 4 * 4;        // 2 x 2 halves x 128 rows
    static constexpr int OFF_LSUM = OFF_PMAX + 2 * 2 * 128 * 4;  // 2 halves x 128 rows
    static constexpr int OFF_BAR = OFF_LSUM + 2 * 128 * 4;
    static constexpr int NBAR = 28;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 32 + 1024;  // + slack for 1024-B alignment
    static_assert(SMEM <= 232448, "shared memory per block");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t O_COL = 128 * kSBuf;
    static constexpr uint32_t Q_COL = 384;
    // Instruction descriptors, kind::f16: bits 4-5 D format (1 = f32), 7-9 A format
    // (1 = bf16), 10-12 B format (1 = bf16), 15/16 A/B major (0 = K, 1 = MN),
    // 17-22 N>>3, 24-28 M>>4.
    static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                                         ((uint32_t)(kBM >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
};

// mbarriers: Q full (TMA), Q in TMEM, K full/empty x4, V full/empty x4, then per
// score buffer: S full, P full, PV done; drain.
enum { B_QFULL = 0, B_QTMEM = 1, B_KFULL = 2, B_KEMPTY = 6, B_VFULL = 10, B_VEMPTY = 14, B_SFULL = 18,
       B_PFULL = 21, B_ODONE = 24, B_DRAIN = 27 };
// With two teams: per team t, S full at B_SFULL + t, P full at B_PFULL + t, PV done at
// B_ODONE + t; team t owns S_t = [128 t, 128 t + 128) and O_t = [256 + 128 t, ...).

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

// Non-blocking probe of phase `parity`.
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

#define TC_LD16(taddr, r)                                                                                    \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];" \
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),    \
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),           \
                   "=r"(r[15])                                                                                       \
                 : "r"(taddr))

#define TC_LD64(taddr, r)                                                                                    \
    asm volatile(                                                                                            \
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17," \
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,"  \
        "%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"         \
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),    \
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),           \
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),         \
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),         \
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]),         \
          "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),         \
          "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),         \
          "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),         \
          "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])          \
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
// 2^x for a pair of floats on the FMA pipe instead of the MUFU unit (the softmax
// needs about one exponential per four tensor-core FLOPs per byte of MUFU
// throughput, so a share of them is computed here). x is clamped to >= -125 so the
// result stays a normal float; larger negative x gives 2^-125 instead of ~0, which
// is negligible against a row sum >= 2^-40. Method: n = round(x) via the 1.5*2^23
// rounding constant, f = x - n in [-1/2, 1/2], 2^f by a cubic fitted to relative
// error on [-1/2, 1/2] (Lawson-weighted least squares, max relative error 7.5e-5),
// then n is added to the exponent field.
constexpr float kExpC0 = 0.9999280571937561f, kExpC1 = 0.6932610869407654f;
constexpr float kExpC2 = 0.2426111102104187f, kExpC3 = 0.055171187967061996f;
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& r0, float& r1) {
    const uint64_t x = pk2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
    const uint64_t t = add2(x, pk2(12582912.f, 12582912.f));       // 1.5 * 2^23 + round(x)
    const uint64_t n = add2(t, pk2(-12582912.f, -12582912.f));     // round(x)
    const uint64_t f = fma2(n, pk2(-1.f, -1.f), x);                 // x - round(x)
    uint64_t q = fma2(f, pk2(kExpC3, kExpC3), pk2(kExpC2, kExpC2));
    q = fma2(q, f, pk2(kExpC1, kExpC1));
    q = fma2(q, f, pk2(kExpC0, kExpC0));
    float q0, q1, t0, t1;
    up2(q, q0, q1);
    up2(t, t0, t1);
    r0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    r1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
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

__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Barrier 3 + t over the 128 threads of softmax team t with an AND of `v`.
__device__ __forceinline__ bool bar_and_team(bool v, int t) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)v), "r"(3 + t)
        : "memory");
    return res != 0;
}

// Named barriers: 0 = __syncthreads; single-stream kernel: 1 = all 256 softmax
// threads; team kernel: 1 + t and 3 + t = team t (128 threads), 5 = both teams. One
// barrier id is never used with two different thread counts.
__device__ __forceinline__ bool bar_and_all(bool v) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 5, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)v)
        : "memory");
    return res != 0;
}

// Barrier 1 over the 256 softmax threads with an AND of `v` across them.
__device__ __forceinline__ bool bar_and_256(bool v) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"((uint32_t)v)
        : "memory");
    return res != 0;
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attend_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                   const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKs,
                   const __grid_constant__ CUtensorMap tmVs, const int32_t* __restrict__ Mdev,
                   const float* __restrict__ bias2, int64_t capP, const float* __restrict__ sbias, int64_t Ts,
                   int64_t Tq, int H, __nv_bfloat16* __restrict__ out, float scale_log2, Stats* stats) {
    using C = Cfg<D>;
    constexpr bool kQT = kQinTmem && D == 128;  // each half row of Q is one 64-column box
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    float* sBias = reinterpret_cast<float*>(smem + C::OFF_BIAS);
    float* sBmax = reinterpret_cast<float*>(smem + C::OFF_BMAX);
    float* sPmax = reinterpret_cast<float*>(smem + C::OFF_PMAX);
    float* sLsum = reinterpret_cast<float*>(smem + C::OFF_LSUM);
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
        mbar_init(&bars[B_QTMEM], 256);
        for (int s2 = 0; s2 < 4; ++s2) {
            mbar_init(&bars[B_KFULL + s2], 1);
            mbar_init(&bars[B_KEMPTY + s2], 1);
            mbar_init(&bars[B_VFULL + s2], 1);
            mbar_init(&bars[B_VEMPTY + s2], 1);
        }
        for (int b = 0; b < kSBuf; ++b) {
            mbar_init(&bars[B_SFULL + b], 1);
            mbar_init(&bars[B_PFULL + b], 256);
            mbar_init(&bars[B_ODONE + b], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kWarpCtl) {
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
    const uint32_t tQ = tmem + C::Q_COL;
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint8_t* sV = smem + C::OFF_V;

    const bool is_kprod = (warp == kWarpCtl && lane == 0);
    const bool is_vprod = (warp == kWarpV && lane == kLaneV);
    if (is_kprod || is_vprod) {
        // ---------------------------------------------------------------- TMA producers
        const bool kside = is_kprod;
        const int nst = kside ? kKSt : kVSt;
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
            const int st = i % nst;
            if (i >= nst && !mbar_wait(&empty[st], ((i / nst) - 1) & 1)) { *abort_flag = 1; break; }
            const bool cache = i < nc;
            const int row0 = (cache ? i : i - nc) * kBN;
            mbar_expect_tx(&full[st], C::TILE);
            for (int b = 0; b < C::NB; ++b)
                tma_load_3d(ring + st * C::TILE + b * C::BOX, cache ? mc : ms, 64 * b, row0, h, &full[st]);
            last = i;
        }
        // Drain: the copies issued here land before the CTA can exit (already true on
        // the normal path, where the MMA thread consumed them all).
        if (kside) mbar_wait(&bars[B_QFULL], 0);
        for (int i = (last >= nst - 1 ? last - nst + 1 : 0); i <= last; ++i) mbar_wait(&full[i % nst], (i / nst) & 1);
    } else if (warp >= 8) {
        // ---------------------------------------------------------------- MMA issuer
        if (warp == kWarpMma && lane == kLaneMma) {
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = kQT ? mbar_wait(&bars[B_QTMEM], 0) : mbar_wait(&bars[B_QFULL], 0);
            auto issue_qk = [&](int j) -> bool {
                const int st = j % kKSt, sb = j % kSBuf;
                // buffer sb held P_{j-kSBuf}: its product must have retired
                if (j >= kSBuf && !mbar_wait(&bars[B_ODONE + sb], ((j / kSBuf) - 1) & 1)) return false;
                if (!mbar_wait(&bars[B_KFULL + st], (j / kKSt) & 1)) return false;
                tc_fence_after();
                const uint32_t aKs = aK + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    if constexpr (kQT)
                        mma_ts(tmem + sb * 128, tQ + kk * 8, sdesc(aKs + off, 16, 1024), C::IDESC_QK, kk > 0);
                    else
                        mma_ss(tmem + sb * 128, sdesc(aQ + off, 16, 1024), sdesc(aKs + off, 16, 1024), C::IDESC_QK,
                               kk > 0);
                }
                tc_commit(&bars[B_SFULL + sb]);
                tc_commit(&bars[B_KEMPTY + st]);
                return true;
            };
            if (ok && ntiles > 0) ok = issue_qk(0);
            for (int i = 0; i < ntiles && ok && !*abort_flag; ++i) {
                if (i + 1 < ntiles && !(ok = issue_qk(i + 1))) break;
                const int st = i % kVSt, sb = i % kSBuf;
                if (!mbar_wait(&bars[B_PFULL + sb], (i / kSBuf) & 1)) { ok = false; break; }
                if (!mbar_wait(&bars[B_VFULL + st], (i / kVSt) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t aVs = aV + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ts(tO, tmem + sb * 128 + kk * 8, sdesc(aVs + kk * 2048, C::BOX, 1024), C::IDESC_PV,
                           (i > 0 || kk > 0));
                tc_commit(&bars[B_VEMPTY + st]);
                tc_commit(&bars[B_ODONE + sb]);
            }
            if (!ok) *abort_flag = 1;
            // Drain: every MMA issued here retires before TMEM is released.
            tc_commit(&bars[B_DRAIN]);
            mbar_wait(&bars[B_DRAIN], 0);
        }
    } else {
        // ---------------------------------------------------------------- softmax (warps 0-7)
        // Control flow stays uniform across the 256 threads: tcgen05.ld/st are
        // warp-collective, so every decision that guards them is reduced first.
        const int g = warp >> 2;          // column half: [64g, 64g+64)
        const int r = threadIdx.x & 127;  // query row within the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        bool ok = true;
        if constexpr (kQT) {
            // Q row r, columns [64g, 64g+64), from the swizzled shared tile into TMEM as
            // 32 bf16 pairs (K-major A operand of the score product).
            const bool qok = __all_sync(0xffffffffu, mbar_wait(&bars[B_QFULL], 0));
            if (qok) {
                const uint8_t* rowp = sQ + g * C::BOX + r * 128;
                uint32_t qv[32];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4*>(rowp + ((c ^ (r & 7)) << 4));
                    qv[4 * c + 0] = v.x; qv[4 * c + 1] = v.y; qv[4 * c + 2] = v.z; qv[4 * c + 3] = v.w;
                }
                TC_ST32(tQ + lane_base + 32 * g, qv);
                tc_wait_st();
            } else {
                ok = false;
            }
            tc_fence_before();
            mbar_arrive(&bars[B_QTMEM]);
        }
        const float* bias_h = bias2 + (int64_t)h * capP;
        auto bias_of = [&](int i) -> float {
            return (i < nc) ? bias_h[(int64_t)i * kBN + r] : sbias[(int64_t)(i - nc) * kBN + r];
        };
        const uint64_t c2 = pk2(scale_log2, scale_log2);
        float m_run = -INFINITY, l_run = 0.f;
        float bnext = (g == 0 && ntiles > 0) ? bias_of(0) : 0.f;
        for (int i = 0; i < ntiles; ++i) {
            const int st = i & 1, sb = i % kSBuf;
            float* bb = sBias + st * kBN;
            if (g == 0) {  // the first half stages the tile's log2 n and its maximum
                bb[r] = bnext;
                float wm = bnext;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
                if (lane == 0) sBmax[st * 4 + warp] = wm;
            }
            const bool got =
                __all_sync(0xffffffffu, ok && !*abort_flag && mbar_wait(&bars[B_SFULL + sb], (i / kSBuf) & 1));
            const uint32_t tS = tmem + sb * 128 + lane_base;
            uint32_t sr[64];
            float pmax = -INFINITY;
            if (got) {
                tc_fence_after();
                TC_LD32(tS + 64 * g, (sr + 0));
                TC_LD32(tS + 64 * g + 32, (sr + 32));
                tc_wait_ld();
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int j = 0; j < 64; j += 8) {
                    m4[0] = max3(m4[0], __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
                    m4[1] = max3(m4[1], __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]));
                    m4[2] = max3(m4[2], __uint_as_float(sr[j + 4]), __uint_as_float(sr[j + 5]));
                    m4[3] = max3(m4[3], __uint_as_float(sr[j + 6]), __uint_as_float(sr[j + 7]));
                }
                pmax = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
            }
            sPmax[(st * 2 + g) * 128 + r] = pmax;
            // Publishes bb[], the bias maxima and the partial row maxima; all S reads
            // of this tile are complete once every thread has passed it.
            if (!bar_and_256(got)) { ok = false; break; }
            if (g == 0 && i + 1 < ntiles) bnext = bias_of(i + 1);
            // Reference max: an upper bound of this tile's row max, (max raw score) *
            // scale + (max shift of the tile). p = 2^(x - m) stays <= 2^8 below.
            const float smax = fmaxf(pmax, sPmax[(st * 2 + (1 - g)) * 128 + r]);
            const float4 bm4 = *reinterpret_cast<const float4*>(sBmax + st * 4);
            const float ub = fmaf(smax, scale_log2, fmaxf(fmaxf(bm4.x, bm4.y), fmaxf(bm4.z, bm4.w)));
            if (i == 0) {
                m_run = ub;
            } else {
                // Lazy rescaling: O and l keep the old reference until it would grow by
                // more than 8 (a factor 256), then both are scaled by alpha. Both halves
                // of a row see the same ub and take the same decision.
                const bool need = ub > m_run + 8.f;
                if (__any_sync(0xffffffffu, need)) {
                    const bool w = mbar_wait(&bars[B_ODONE + (i - 1) % kSBuf], ((i - 1) / kSBuf) & 1);
                    if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; }
                    if (ok) {
                        const float alpha = need ? ex2(m_run - ub) : 1.f;
                        if (need) { l_run *= alpha; m_run = ub; }
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < D / 64; ++c) {
                            const uint32_t ta = tO + lane_base + (D / 2) * g + 32 * c;
                            uint32_t o[32];
                            TC_LD32(ta, o);
                            tc_wait_ld();
#pragma unroll
                            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
                            TC_ST32(ta, o);
                        }
                        tc_wait_st();
                    }
                }
            }
            // p = 2^(s * scale + log2 n - m): packed fp32x2 FMA/ADD, exponentials on MUFU
            // (and, with kPoly, about a third on the FMA pipe), bf16 pairs for P.
            const uint64_t negm2 = pk2(-m_run, -m_run);
            uint64_t sumA = pk2(0.f, 0.f), sumB = pk2(0.f, 0.f);
            uint32_t pk[32];
            const float* bh = bb + 64 * g;
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                const float4 b4 = *reinterpret_cast<const float4*>(bh + j);
                const uint64_t x01 = fma2(pk2(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), c2,
                                          add2(pk2(b4.x, b4.y), negm2));
                const uint64_t x23 = fma2(pk2(__uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3])), c2,
                                          add2(pk2(b4.z, b4.w), negm2));
                float a0, a1, a2, a3;
                up2(x01, a0, a1);
                up2(x23, a2, a3);
                const float p0 = ex2(a0), p1 = ex2(a1);
                float p2, p3;
                if (kPoly && (j / 4) % 3 != 2) {   // 22 of every 64 columns on the FMA pipe
                    exp2_poly2(a2, a3, p2, p3);
                } else {
                    p2 = ex2(a2);
                    p3 = ex2(a3);
                }
                sumA = add2(sumA, pk2(p0, p1));
                sumB = add2(sumB, pk2(p2, p3));
                pk[j / 2] = cvt_bf16x2(p0, p1);
                pk[j / 2 + 1] = cvt_bf16x2(p2, p3);
            }
            float s0, s1, s2, s3;
            up2(sumA, s0, s1);
            up2(sumB, s2, s3);
            l_run += (s0 + s1) + (s2 + s3);
            // P columns [32g, 32g+32) hold this half's 64 probabilities; they overlay
            // S columns both halves have already read (see the barrier above).
            TC_ST32(tS + 32 * g, pk);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[B_PFULL + sb]);
        }
        const bool fin = ok && ntiles > 0 &&
                         mbar_wait(&bars[B_ODONE + (ntiles - 1) % kSBuf], ((ntiles - 1) / kSBuf) & 1);
        sLsum[g * 128 + r] = l_run;
        if (bar_and_256(fin)) {
            tc_fence_after();
            const float inv = 1.f / (sLsum[r] + sLsum[128 + r]);
            const int64_t row = q0 + r;
#pragma unroll 1
            for (int c = 0; c < D / 64; ++c) {
                const int col = (D / 2) * g + 32 * c;
                uint32_t o[32];
                TC_LD32(tO + lane_base + col, o);
                tc_wait_ld();
                if (row < Tq) {
                    uint4* dst = reinterpret_cast<uint4*>(out + (row * H + h) * D + col);
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
    if (warp == kWarpCtl) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
    }
    // When this grid was allowed to start before the previous one finished, it
    // completes only after that one: whatever follows on the stream sees both done.
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attend_bf16_teams_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                         const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKs,
                         const __grid_constant__ CUtensorMap tmVs, const int32_t* __restrict__ Mdev,
                         const float* __restrict__ bias2, int64_t capP,
                         const float* __restrict__ sbias, int64_t Ts, int64_t Tq, int H,
                         __nv_bfloat16* __restrict__ out, float scale_log2, Stats* stats) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    float* sBias = reinterpret_cast<float*>(smem + C::OFF_BIAS);     // 2 teams x 128
    float* sBmax = reinterpret_cast<float*>(smem + C::OFF_BMAX);     // 2 teams x 4 warps
    float* sXch = reinterpret_cast<float*>(smem + C::OFF_PMAX);      // 2 teams x (max, sum) x 128
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
        for (int s2 = 0; s2 < 4; ++s2) {
            mbar_init(&bars[B_KFULL + s2], 1);
            mbar_init(&bars[B_KEMPTY + s2], 1);
            mbar_init(&bars[B_VFULL + s2], 1);
            mbar_init(&bars[B_VEMPTY + s2], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars[B_SFULL + t], 1);
            mbar_init(&bars[B_PFULL + t], 128);
            mbar_init(&bars[B_ODONE + t], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kWarpCtl) {
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
    const uint32_t tO = tmem + 256;
    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint8_t* sV = smem + C::OFF_V;

    const bool is_kprod = (warp == kWarpCtl && lane == 0);
    const bool is_vprod = (warp == kWarpV && lane == kLaneV);
    if (is_kprod || is_vprod) {
        // ---------------------------------------------------------------- TMA producers
        const bool kside = is_kprod;
        const int nst = kside ? kKSt : kVSt;
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
            const int st = i % nst;
            if (i >= nst && !mbar_wait(&empty[st], ((i / nst) - 1) & 1)) { *abort_flag = 1; break; }
            const bool cache = i < nc;
            const int row0 = (cache ? i : i - nc) * kBN;
            mbar_expect_tx(&full[st], C::TILE);
            for (int b = 0; b < C::NB; ++b)
                tma_load_3d(ring + st * C::TILE + b * C::BOX, cache ? mc : ms, 64 * b, row0, h, &full[st]);
            last = i;
        }
        if (kside) mbar_wait(&bars[B_QFULL], 0);
        for (int i = (last >= nst - 1 ? last - nst + 1 : 0); i <= last; ++i) mbar_wait(&full[i % nst], (i / nst) & 1);
    } else if (warp >= 8) {
        // ---------------------------------------------------------------- MMA issuer
        if (warp == kWarpMma && lane == kLaneMma) {
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = mbar_wait(&bars[B_QFULL], 0);
            // S_t = Q K_j^T for tile j of team t = j & 1; the team's buffer held P_{j-2},
            // so O_t += P_{j-2} V_{j-2} must have retired first.
            auto issue_qk = [&](int j) -> bool {
                const int t = j & 1, st = j % kKSt;
                if (j >= 2 && !mbar_wait(&bars[B_ODONE + t], ((j - 2) >> 1) & 1)) return false;
                if (!mbar_wait(&bars[B_KFULL + st], (j / kKSt) & 1)) return false;
                tc_fence_after();
                const uint32_t aKs = aK + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tmem + t * 128, sdesc(aQ + off, 16, 1024), sdesc(aKs + off, 16, 1024), C::IDESC_QK,
                           kk > 0);
                }
                tc_commit(&bars[B_SFULL + t]);
                tc_commit(&bars[B_KEMPTY + st]);
                return true;
            };
            // O_t += P_t V_i for tile i of team t (the team's first tile starts O_t).
            auto issue_pv = [&](int i) -> bool {
                const int t = i & 1, st = i % kVSt;
                if (!mbar_wait(&bars[B_VFULL + st], (i / kVSt) & 1)) return false;
                tc_fence_after();
                const uint32_t aVs = aV + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ts(tO + t * 128, tmem + t * 128 + kk * 8, sdesc(aVs + kk * 2048, C::BOX, 1024), C::IDESC_PV,
                           (i >= 2 || kk > 0));
                tc_commit(&bars[B_VEMPTY + st]);
                tc_commit(&bars[B_ODONE + t]);
                return true;
            };
            int pv = 0, qk = 0;
            if constexpr (kSched == 0) {
                // Blocking schedule: after each PV, queue the other team's PV when its P is
                // ready, then every QK whose buffer is free.
                while (ok && qk < ntiles && qk < 2) ok = issue_qk(qk++);
                while (ok && pv < ntiles && !*abort_flag) {
                    if (!mbar_wait(&bars[B_PFULL + (pv & 1)], (pv >> 1) & 1) || !issue_pv(pv)) { ok = false; break; }
                    ++pv;
                    if (pv < ntiles && mbar_try(&bars[B_PFULL + (pv & 1)], (pv >> 1) & 1)) {
                        if (!issue_pv(pv)) { ok = false; break; }
                        ++pv;
                    }
                    while (ok && qk < ntiles && qk <= pv + 1) ok = issue_qk(qk++);
                }
            } else {
                // Polling schedule: issue whichever product is ready, QK first (it feeds the
                // other team's softmax). QK(j) needs PV(j-2) retired; PV(i) needs P(i).
                uint64_t t_last = global_ns();
                while (ok && pv < ntiles && !*abort_flag) {
                    bool prog = false;
                    if (qk < ntiles && qk < pv + 2) {
                        const int t = qk & 1;
                        if ((qk < 2 || mbar_test(&bars[B_ODONE + t], ((qk - 2) >> 1) & 1)) &&
                            mbar_test(&bars[B_KFULL + qk % kKSt], (qk / kKSt) & 1)) {
                            ok = issue_qk(qk++);
                            prog = true;
                        }
                    }
                    if (ok && pv < qk && mbar_test(&bars[B_PFULL + (pv & 1)], (pv >> 1) & 1) &&
                        mbar_test(&bars[B_VFULL + pv % kVSt], (pv / kVSt) & 1)) {
                        ok = issue_pv(pv++);
                        prog = true;
                    }
                    if (prog) {
                        t_last = global_ns();
                    } else {
                        if constexpr (kSched == 2) __nanosleep(32);
                        if (global_ns() - t_last > kTimeoutNs) ok = false;
                    }
                }
            }
            if (!ok) *abort_flag = 1;
            tc_commit(&bars[B_DRAIN]);
            mbar_wait(&bars[B_DRAIN], 0);
        }
    } else {
        // ---------------------------------------------------------------- softmax teams (warps 0-7)
        const int t = warp >> 2;          // team: key tiles i = t, t + 2, ...
        const int r = threadIdx.x & 127;  // query row within the tile = TMEM lane
        const int wt = warp & 3;
        const uint32_t lane_base = (uint32_t)(wt * 32) << 16;
        const uint32_t tS = tmem + t * 128 + lane_base;
        const uint32_t tOt = tO + t * 128 + lane_base;
        const float* bias_h = bias2 + (int64_t)h * capP;
        auto bias_of = [&](int i) -> float {
            return (i < nc) ? bias_h[(int64_t)i * kBN + r] : sbias[(int64_t)(i - nc) * kBN + r];
        };
        float* bb = sBias + t * kBN;
        const uint64_t c2 = pk2(scale_log2, scale_log2);
        float m_run = -INFINITY, l_run = 0.f;
        float bnext = (t < ntiles) ? bias_of(t) : 0.f;
        bool ok = true;
        for (int i = t; i < ntiles; i += 2) {
            const int k = i >> 1;  // the team's k-th tile
            // The team's log2 n row is staged in shared memory once per tile (one value
            // per thread); this barrier orders the write after every read of the
            // previous tile, the one below publishes it.
            named_bar_sync(1 + t, 128);
            bb[r] = bnext;
            float wm = bnext;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
            if (lane == 0) sBmax[t * 4 + wt] = wm;
            const bool got = !*abort_flag && mbar_wait(&bars[B_SFULL + t], k & 1);
            if (!bar_and_team(got, t)) { ok = false; break; }
            if (i + 2 < ntiles) bnext = bias_of(i + 2);
            tc_fence_after();
            // Row max of the raw scores: with kOnePass the whole 128-column row of S
            // comes into registers with one wait, otherwise 64 columns at a time.
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            uint32_t srow[kOnePass ? 128 : 1];
            if constexpr (kOnePass) {
                TC_LD32(tS, (srow + 0));
                TC_LD32(tS + 32, (srow + 32));
                TC_LD32(tS + 64, (srow + 64));
                TC_LD32(tS + 96, (srow + 96));
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 128; j += 8) {
                    m4[0] = max3(m4[0], __uint_as_float(srow[j]), __uint_as_float(srow[j + 1]));
                    m4[1] = max3(m4[1], __uint_as_float(srow[j + 2]), __uint_as_float(srow[j + 3]));
                    m4[2] = max3(m4[2], __uint_as_float(srow[j + 4]), __uint_as_float(srow[j + 5]));
                    m4[3] = max3(m4[3], __uint_as_float(srow[j + 6]), __uint_as_float(srow[j + 7]));
                }
            } else {
#pragma unroll 1
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t sr[64];
                    TC_LD32(tS + 64 * h2, (sr + 0));
                    TC_LD32(tS + 64 * h2 + 32, (sr + 32));
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 64; j += 8) {
                        m4[0] = max3(m4[0], __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
                        m4[1] = max3(m4[1], __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]));
                        m4[2] = max3(m4[2], __uint_as_float(sr[j + 4]), __uint_as_float(sr[j + 5]));
                        m4[3] = max3(m4[3], __uint_as_float(sr[j + 6]), __uint_as_float(sr[j + 7]));
                    }
                }
            }
            const float smax = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
            // Reference max: an upper bound of this tile's row max, (max raw score) *
            // scale + (max log2 n of the tile). p = 2^(x - m) stays <= 2^8 below.
            const float4 bm4 = *reinterpret_cast<const float4*>(sBmax + t * 4);
            const float ub = fmaf(smax, scale_log2, fmaxf(fmaxf(bm4.x, bm4.y), fmaxf(bm4.z, bm4.w)));
            if (k == 0) {
                m_run = ub;
            } else {
                // Lazy rescaling: O_t and l keep the old reference until it would grow
                // by more than 8 (a factor 256), then both are scaled by alpha.
                const bool need = ub > m_run + 8.f;
                if (__any_sync(0xffffffffu, need)) {
                    const bool w = mbar_wait(&bars[B_ODONE + t], (k - 1) & 1);
                    if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; }
                    if (ok) {
                        const float alpha = need ? ex2(m_run - ub) : 1.f;
                        if (need) { l_run *= alpha; m_run = ub; }
                        tc_fence_after();
if constexpr (kOnePass) {
#pragma unroll 1
                            for (int c = 0; c < D / 16; ++c) {
                                uint32_t o[16];
                                TC_LD16(tOt + 16 * c, o);
                                tc_wait_ld();
#pragma unroll
                                for (int q = 0; q < 16; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
                                TC_ST16(tOt + 16 * c, o);
                            }
                        } else {
#pragma unroll 1
                            for (int c = 0; c < D / 32; ++c) {
                                uint32_t o[32];
                                TC_LD32(tOt + 32 * c, o);
                                tc_wait_ld();
#pragma unroll
                                for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
                                TC_ST32(tOt + 32 * c, o);
                            }
                        }
                        tc_wait_st();
                    }
                }
            }
            // Pass 2, 64 columns at a time: p = 2^(s * scale + log2 n - m) with packed fp32x2
            // FMA/ADD and MUFU ex2 (with kPoly, about a third on the FMA pipe); 32 bf16
            // pairs of P are written over S columns already read.
            const uint64_t negm2 = pk2(-m_run, -m_run);
            uint64_t sumA = pk2(0.f, 0.f), sumB = pk2(0.f, 0.f);
            if constexpr (kOnePass) {
                uint32_t pk[64];
#pragma unroll
                for (int j = 0; j < 128; j += 4) {
                    const float4 b4 = *reinterpret_cast<const float4*>(bb + j);
                    const uint64_t x01 = fma2(pk2(__uint_as_float(srow[j]), __uint_as_float(srow[j + 1])), c2,
                                              add2(pk2(b4.x, b4.y), negm2));
                    const uint64_t x23 = fma2(pk2(__uint_as_float(srow[j + 2]), __uint_as_float(srow[j + 3])), c2,
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
                TC_ST32(tS, pk);
                TC_ST32(tS + 32, (pk + 32));
            } else {
    #pragma unroll 1
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t sr[64];
                    TC_LD32(tS + 64 * h2, (sr + 0));
                    TC_LD32(tS + 64 * h2 + 32, (sr + 32));
                    tc_wait_ld();
                    uint32_t pk[32];
                    const float* bh = bb + 64 * h2;
    #pragma unroll
                    for (int j = 0; j < 64; j += 4) {
                        const float4 b4 = *reinterpret_cast<const float4*>(bh + j);
                        const uint64_t x01 = fma2(pk2(__uint_as_float(sr[j]), __uint_as_float(sr[j + 1])), c2,
                                                  add2(pk2(b4.x, b4.y), negm2));
                        const uint64_t x23 = fma2(pk2(__uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3])), c2,
                                                  add2(pk2(b4.z, b4.w), negm2));
                        float a0, a1, a2, a3;
                        up2(x01, a0, a1);
                        up2(x23, a2, a3);
                        const float p0 = ex2(a0), p1 = ex2(a1);
                        float p2, p3;
                        if (kPoly && (j / 4) % 3 != 2) {
                            exp2_poly2(a2, a3, p2, p3);
                        } else {
                            p2 = ex2(a2);
                            p3 = ex2(a3);
                        }
                        sumA = add2(sumA, pk2(p0, p1));
                        sumB = add2(sumB, pk2(p2, p3));
                        pk[j / 2] = cvt_bf16x2(p0, p1);
                        pk[j / 2 + 1] = cvt_bf16x2(p2, p3);
                    }
                    TC_ST32(tS + 32 * h2, pk);
                }
            }
            float s0, s1, s2, s3;
            up2(sumA, s0, s1);
            up2(sumB, s2, s3);
            l_run += (s0 + s1) + (s2 + s3);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[B_PFULL + t]);
        }
        // Epilogue: both teams' last products retire, then each team writes half of
        // the output columns from O = (O_A 2^(m_A - m) + O_B 2^(m_B - m)) / l.
        const int last = ntiles - 1 - ((ntiles - 1 - t) & 1);   // this team's last tile (or < 0)
        const bool fin = ok && (last < 0 || mbar_wait(&bars[B_ODONE + t], (last >> 1) & 1));
        sXch[(t * 2 + 0) * 128 + r] = m_run;
        sXch[(t * 2 + 1) * 128 + r] = l_run;
        if (bar_and_all(fin)) {
            const float mA = sXch[0 * 128 + r], lA = sXch[1 * 128 + r];
            const float mB = sXch[2 * 128 + r], lB = sXch[3 * 128 + r];
            const float m = fmaxf(mA, mB);
            const float fA = (lA > 0.f) ? ex2(mA - m) : 0.f;   // a team with no tiles contributes 0
            const float fB = (lB > 0.f) ? ex2(mB - m) : 0.f;
            const float inv = 1.f / (lA * fA + lB * fB);
            const float wA = fA * inv, wB = fB * inv;
            const bool haveB = ntiles > 1;
            tc_fence_after();
            const int64_t row = q0 + r;
#pragma unroll 1
            for (int c = 0; c < D / 64; ++c) {
                const int col = (D / 2) * t + 32 * c;
                uint32_t oa[32], ob[32];
                TC_LD32(tO + lane_base + col, oa);
                if (haveB) TC_LD32(tO + 128 + lane_base + col, ob);
                tc_wait_ld();
                if (row < Tq) {
                    uint4* dst = reinterpret_cast<uint4*>(out + (row * H + h) * D + col);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        float e[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            e[q] = __uint_as_float(oa[8 * v + q]) * wA +
                                   (haveB ? __uint_as_float(ob[8 * v + q]) * wB : 0.f);
                        uint4 w;
                        w.x = cvt_bf16x2(e[0], e[1]);
                        w.y = cvt_bf16x2(e[2], e[3]);
                        w.z = cvt_bf16x2(e[4], e[5]);
                        w.w = cvt_bf16x2(e[6], e[7]);
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
    if (warp == kWarpCtl) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS)
                     : "memory");
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
}


// Shared-memory layout of the split kernel: Q tile, K and V rings, then per team t
// and bias buffer b: log2 n of the tile's keys [t][b][128] and quarter maxima
// [t][b][4]; the halves' reference maxima [t][g][128]; the epilogue exchange
// [t][g][m, l][128]; mbarriers.
template <int D>
struct CfgS {
    using C = Cfg<D>;
    static constexpr int TILE = C::TILE;
    static constexpr int BOX = C::BOX;
    static constexpr int NB = C::NB;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;
    static constexpr int OFF_V = (1 + kKSt) * TILE;
    static constexpr int OFF_BIAS = (1 + kKSt + kVSt) * TILE;   // 2 x 2 x 128 floats
    static constexpr int OFF_BMAX = OFF_BIAS + 2 * 2 * 128 * 4;  // 2 x 2 x 4 floats
    static constexpr int OFF_UB = OFF_BMAX + 2 * 2 * 4 * 4;      // 2 x 2 x 128 floats
    static constexpr int OFF_XCH = OFF_UB + 2 * 2 * 128 * 4;     // 2 x 2 x 2 x 128 floats
    static constexpr int OFF_BAR = OFF_XCH + 2 * 2 * 2 * 128 * 4;
    static constexpr int OFF_MISC = OFF_BAR + C::NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 32 + 1024;
    static_assert(SMEM <= 232448, "shared memory per block");
};

// Split-row teams. Two softmax teams take alternate key tiles (team t: tiles t, t+2,
// ...) with their own score buffer S_t = TMEM [128 t, 128 t + 128) and output
// accumulator O_t = [256 + 128 t, ...). Each team has eight warps: thread (t, g, r)
// owns columns [64 g, 64 g + 64) of query row r, so every SM sub-partition runs four
// softmax warps. The halves agree on a reference max per tile through shared memory
// at one team barrier, keep partial row sums, and each writes its 64 probabilities
// (bf16) over its own first 32 S columns; the PV product reads the A operand for keys
// [64 g, 64 g + 64) from columns [128 t + 64 g, ... + 32). The epilogue merges the
// teams' partial results: O = (O_A 2^(m_A - m) + O_B 2^(m_B - m)) / (l_A 2^.. + l_B 2^..).
// Warps 16, 17, 18: K producer (and TMEM allocator), MMA issuer, V producer.
template <int D>
__global__ void __launch_bounds__(kThreadsSplit, 1)
attend_bf16_split_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                         const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKs,
                         const __grid_constant__ CUtensorMap tmVs, const int32_t* __restrict__ Mdev,
                         const float* __restrict__ bias2, int64_t capP,
                         const float* __restrict__ sbias, int64_t Ts, int64_t Tq, int H,
                         __nv_bfloat16* __restrict__ out, float scale_log2, Stats* stats) {
    using C = Cfg<D>;
    using L = CfgS<D>;
    constexpr int kWK = 16, kWM = 17, kWV = 18;   // control warps
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    float* sBias = reinterpret_cast<float*>(smem + L::OFF_BIAS);   // [t][b][128]
    float* sBmax = reinterpret_cast<float*>(smem + L::OFF_BMAX);   // [t][b][4]
    float* sUb = reinterpret_cast<float*>(smem + L::OFF_UB);       // [t][g][128]
    float* sXch = reinterpret_cast<float*>(smem + L::OFF_XCH);     // [t][g][m,l][128]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int q0 = blockIdx.x * kBM;
    const int Mh = Mdev[h];
    const int nc = (Mh + kBN - 1) / kBN;
    const int ntiles = nc + (int)((Ts + kBN - 1) / kBN);

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_QFULL], 1);
        for (int s2 = 0; s2 < 4; ++s2) {
            mbar_init(&bars[B_KFULL + s2], 1);
            mbar_init(&bars[B_KEMPTY + s2], 1);
            mbar_init(&bars[B_VFULL + s2], 1);
            mbar_init(&bars[B_VEMPTY + s2], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars[B_SFULL + t], 1);
            mbar_init(&bars[B_PFULL + t], 256);
            mbar_init(&bars[B_ODONE + t], 1);
        }
        mbar_init(&bars[B_DRAIN], 1);
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
    const uint32_t tO = tmem + 256;
    uint8_t* sQ = smem + L::OFF_Q;
    uint8_t* sK = smem + L::OFF_K;
    uint8_t* sV = smem + L::OFF_V;

    const bool is_kprod = (warp == kWK && lane == 0);
    const bool is_vprod = (warp == kWV && lane == 0);
    if (is_kprod || is_vprod) {
        // ---------------------------------------------------------------- TMA producers
        const bool kside = is_kprod;
        const int nst = kside ? kKSt : kVSt;
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
            const int st = i % nst;
            if (i >= nst && !mbar_wait(&empty[st], ((i / nst) - 1) & 1)) { *abort_flag = 1; break; }
            const bool cache = i < nc;
            const int row0 = (cache ? i : i - nc) * kBN;
            mbar_expect_tx(&full[st], C::TILE);
            for (int b = 0; b < C::NB; ++b)
                tma_load_3d(ring + st * C::TILE + b * C::BOX, cache ? mc : ms, 64 * b, row0, h, &full[st]);
            last = i;
        }
        if (kside) mbar_wait(&bars[B_QFULL], 0);
        for (int i = (last >= nst - 1 ? last - nst + 1 : 0); i <= last; ++i) mbar_wait(&full[i % nst], (i / nst) & 1);
    } else if (warp >= 16) {
        // ---------------------------------------------------------------- MMA issuer
        if (warp == kWM && lane == 0) {
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = mbar_wait(&bars[B_QFULL], 0);
            // S_t = Q K_j^T for tile j of team t = j & 1; S_t held P_{j-2}, so
            // O_t += P_{j-2} V_{j-2} must have retired first.
            auto issue_qk = [&](int j) -> bool {
                const int t = j & 1, st = j % kKSt;
                if (j >= 2 && !mbar_wait(&bars[B_ODONE + t], ((j - 2) >> 1) & 1)) return false;
                if (!mbar_wait(&bars[B_KFULL + st], (j / kKSt) & 1)) return false;
                tc_fence_after();
                const uint32_t aKs = aK + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                    mma_ss(tmem + t * 128, sdesc(aQ + off, 16, 1024), sdesc(aKs + off, 16, 1024), C::IDESC_QK,
                           kk > 0);
                }
                tc_commit(&bars[B_SFULL + t]);
                tc_commit(&bars[B_KEMPTY + st]);
                return true;
            };
            // O_t += P_t V_i; keys [16 kk, 16 kk + 16) of P sit at TMEM column
            // 128 t + 64 (kk / 4) + 8 (kk % 4) (each half's P over its own S columns).
            auto issue_pv = [&](int i) -> bool {
                const int t = i & 1, st = i % kVSt;
                if (!mbar_wait(&bars[B_VFULL + st], (i / kVSt) & 1)) return false;
                tc_fence_after();
                const uint32_t aVs = aV + st * C::TILE;
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_ts(tO + t * 128, tmem + t * 128 + 64 * (kk >> 2) + 8 * (kk & 3),
                           sdesc(aVs + kk * 2048, C::BOX, 1024), C::IDESC_PV, (i >= 2 || kk > 0));
                tc_commit(&bars[B_VEMPTY + st]);
                tc_commit(&bars[B_ODONE + t]);
                return true;
            };
            int pv = 0, qk = 0;
            while (ok && qk < ntiles && qk < 2) ok = issue_qk(qk++);
            while (ok && pv < ntiles && !*abort_flag) {
                if (!mbar_wait(&bars[B_PFULL + (pv & 1)], (pv >> 1) & 1) || !issue_pv(pv)) { ok = false; break; }
                ++pv;
                if (pv < ntiles && mbar_try(&bars[B_PFULL + (pv & 1)], (pv >> 1) & 1)) {
                    if (!issue_pv(pv)) { ok = false; break; }
                    ++pv;
                }
                while (ok && qk < ntiles && qk <= pv + 1) ok = issue_qk(qk++);
            }
            if (!ok) *abort_flag = 1;
            tc_commit(&bars[B_DRAIN]);
            mbar_wait(&bars[B_DRAIN], 0);
        }
    } else {
        // ---------------------------------------------------------------- softmax (warps 0-15)
        const int t = warp >> 3;             // team: key tiles i = t, t + 2, ...
        const int g = (warp >> 2) & 1;       // half: key columns [64 g, 64 g + 64) of each tile
        const int wt = warp & 3;             // TMEM lane quarter (= SM sub-partition)
        const int r = wt * 32 + lane;        // query row within the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(wt * 32) << 16;
        const uint32_t tS = tmem + t * 128 + 64 * g + lane_base;   // my S columns, then my P
        const uint32_t tOg = tO + t * 128 + (D / 2) * g + lane_base;  // my O columns
        const float* bias_h = bias2 + (int64_t)h * capP;
        auto bias_of = [&](int i) -> float {
            return (i < nc) ? bias_h[(int64_t)i * kBN + r] : sbias[(int64_t)(i - nc) * kBN + r];
        };
        // Half 0 stages each tile's log2 n row (one value per thread) and its quarter maxima.
        auto stage_bias = [&](int b, float v) {
            sBias[(t * 2 + b) * 128 + r] = v;
            float wm = v;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
            if (lane == 0) sBmax[(t * 2 + b) * 4 + wt] = wm;
        };
        const uint64_t c2 = pk2(scale_log2, scale_log2);
        float m_run = -INFINITY, l_run = 0.f;
        float bnext = 0.f;
        if (g == 0) {
            if (t < ntiles) stage_bias(0, bias_of(t));
            if (t + 2 < ntiles) bnext = bias_of(t + 2);
        }
        bool ok = bar_and(1 + t, 256, true);
        for (int i = t; i < ntiles; i += 2) {
            const int k = i >> 1;  // the team's k-th tile
            const int b = k & 1;
            // (warp-uniform: the TMEM loads below are warp-collective)
            const bool got = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&bars[B_SFULL + t], k & 1));
            tc_fence_after();
            // Row max over my 64 raw scores, and the reference for this half.
            float smax = -INFINITY;
            if (got) {
                uint32_t sr[64];
                TC_LD32(tS, (sr + 0));
                TC_LD32(tS + 32, (sr + 32));
                tc_wait_ld();
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int j = 0; j < 64; j += 8) {
                    m4[0] = max3(m4[0], __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
                    m4[1] = max3(m4[1], __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]));
                    m4[2] = max3(m4[2], __uint_as_float(sr[j + 4]), __uint_as_float(sr[j + 5]));
                    m4[3] = max3(m4[3], __uint_as_float(sr[j + 6]), __uint_as_float(sr[j + 7]));
                }
                smax = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
            }
            const float2 bm = *reinterpret_cast<const float2*>(sBmax + (t * 2 + b) * 4 + 2 * g);
            sUb[(t * 2 + g) * 128 + r] = fmaf(smax, scale_log2, fmaxf(bm.x, bm.y));
            // Stage the log2 n row of the team's next tile into the other buffer. Its
            // previous contents were last read in the team's previous tile, which every
            // thread finished before S could be refilled.
            if (g == 0 && i + 2 < ntiles) stage_bias(b ^ 1, bnext);
            if (!bar_and(1 + t, 256, got)) { ok = false; break; }
            if (g == 0 && i + 4 < ntiles) bnext = bias_of(i + 4);
            // Reference max: an upper bound of the row max of this tile, (max raw score)
            // * scale + (max log2 n), agreed by both halves. p = 2^(x - m) <= 2^8 below.
            const float ub = fmaxf(sUb[(t * 2 + 0) * 128 + r], sUb[(t * 2 + 1) * 128 + r]);
            if (k == 0) {
                m_run = ub;
            } else {
                // Lazy rescaling: O_t and l keep the old reference until it would grow by
                // more than 8 (a factor 256); then both halves scale their parts by alpha.
                const bool need = ub > m_run + 8.f;
                if (__any_sync(0xffffffffu, need)) {
                    const bool w = mbar_wait(&bars[B_ODONE + t], (k - 1) & 1);
                    if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; }
                    if (ok) {
                        const float alpha = need ? ex2(m_run - ub) : 1.f;
                        if (need) { l_run *= alpha; m_run = ub; }
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < D / 64; ++c) {
                            uint32_t o[32];
                            TC_LD32(tOg + 32 * c, o);
                            tc_wait_ld();
#pragma unroll
                            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
                            TC_ST32(tOg + 32 * c, o);
                        }
                        tc_wait_st();
                    }
                }
            }
            // p = 2^(s * scale + log2 n - m) over my 64 columns in two chunks of 32,
            // packed fp32x2 FMA/ADD and MUFU ex2; 16 bf16 pairs per chunk go over S
            // columns already read.
            const uint64_t negm2 = pk2(-m_run, -m_run);
            uint64_t sumA = pk2(0.f, 0.f), sumB = pk2(0.f, 0.f);
            const float* bh = sBias + (t * 2 + b) * 128 + 64 * g;
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
                uint32_t sr[32];
                TC_LD32(tS + 32 * h2, sr);
                tc_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 b4 = *reinterpret_cast<const float4*>(bh + 32 * h2 + j);
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
            mbar_arrive(&bars[B_PFULL + t]);
        }
        // Epilogue: both teams' last products retire; thread (t, g) writes output
        // columns [D/4 (2t + g), D/4 (2t + g + 1)) of its row.
        const int lastt = ntiles - 1 - ((ntiles - 1 - t) & 1);   // this team's last tile (or < 0)
        const bool fin = ok && (lastt < 0 || mbar_wait(&bars[B_ODONE + t], (lastt >> 1) & 1));
        sXch[((t * 2 + g) * 2 + 0) * 128 + r] = m_run;
        sXch[((t * 2 + g) * 2 + 1) * 128 + r] = l_run;
        if (bar_and(3, 512, fin)) {
            const float mA = sXch[(0 * 2 + 0) * 128 + r];
            const float lA = sXch[(0 * 2 + 1) * 128 + r] + sXch[(2 * 1 + 1) * 128 + r];
            const float mB = sXch[(4 + 0) * 128 + r];
            const float lB = sXch[(4 + 1) * 128 + r] + sXch[(6 + 1) * 128 + r];
            const float m = fmaxf(mA, mB);
            const float fA = (lA > 0.f) ? ex2(mA - m) : 0.f;   // a team with no tiles contributes 0
            const float fB = (lB > 0.f) ? ex2(mB - m) : 0.f;
            const float inv = 1.f / (lA * fA + lB * fB);
            const float wA = fA * inv, wB = fB * inv;
            const bool haveB = ntiles > 1;
            tc_fence_after();
            const int64_t row = q0 + r;
            constexpr int QC = D / 4;   // output columns per thread
            const int col = QC * (2 * t + g);
            uint32_t oa[QC], ob[QC];
            if constexpr (QC == 32) {
                TC_LD32(tO + lane_base + col, oa);
                if (haveB) TC_LD32(tO + 128 + lane_base + col, ob);
            } else {
                TC_LD16(tO + lane_base + col, oa);
                if (haveB) TC_LD16(tO + 128 + lane_base + col, ob);
            }
            tc_wait_ld();
            if (row < Tq) {
                uint4* dst = reinterpret_cast<uint4*>(out + (row * H + h) * D + col);
#pragma unroll
                for (int v = 0; v < QC / 8; ++v) {
                    float e[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        e[q] = __uint_as_float(oa[8 * v + q]) * wA + (haveB ? __uint_as_float(ob[8 * v + q]) * wB : 0.f);
                    uint4 w4;
                    w4.x = cvt_bf16x2(e[0], e[1]);
                    w4.y = cvt_bf16x2(e[2], e[3]);
                    w4.z = cvt_bf16x2(e[4], e[5]);
                    w4.w = cvt_bf16x2(e[6], e[7]);
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


// ---------------------------------------------------------------------------- ring kernel
// Shared-memory layout: Q tile, K ring (3 stages), V ring (2 stages); log2 n of the
// keys of three tiles [3][128] and their quarter maxima [3][4]; the quarters' reference
// maxima [2][4][128]; the epilogue row sums [4][128]; mbarriers.
constexpr int kRK = 3, kRV = 2;
enum { R_QFULL = 0, R_KFULL = 1, R_KEMPTY = 4, R_VFULL = 7, R_VEMPTY = 9, R_SFULL = 11, R_PFULL = 14,
       R_ODONE = 17, R_DRAIN = 20, R_NBAR = 22 };
template <int D>
struct CfgR {
    using C = Cfg<D>;
    static constexpr int TILE = C::TILE;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE;
    static constexpr int OFF_V = (1 + kRK) * TILE;
    static constexpr int OFF_BIAS = (1 + kRK + kRV) * TILE;   // 3 x 128 floats
    static constexpr int OFF_BMAX = OFF_BIAS + 3 * 128 * 4;    // 3 x 4 floats
    static constexpr int OFF_UB = OFF_BMAX + 3 * 4 * 4;        // 2 x 4 x 128 floats
    static constexpr int OFF_L = OFF_UB + 2 * 4 * 128 * 4;     // 4 x 128 floats
    static constexpr int OFF_BAR = OFF_L + 4 * 128 * 4;
    static constexpr int OFF_MISC = OFF_BAR + R_NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 32 + 1024;
    static_assert(SMEM <= 232448, "shared memory per block");
    static constexpr uint32_t O_COL = 384;   // S_b = [128 b, 128 b + 128), b < 3; O = [384, 384 + D)
};

// One CTA = 128 query rows of one head; the key tiles are processed in order.
//   TMEM: three score buffers S_b (tile i uses b = i mod 3) and one output
//         accumulator O; P (bf16) overwrites the S columns its quarter has read.
//   warps 0-15  softmax: thread (q, r) owns columns [32 q, 32 q + 32) of query row r
//               (TMEM lane r), four softmax warps per SM sub-partition. Per tile: S
//               into registers once, a reference max agreed by the four quarters at
//               one barrier (upper bound: max raw score * scale + max log2 n), lazy
//               rescaling of O and the row sums (only when the reference grows by more
//               than 2^8), p = 2^(x - m) with packed fp32x2 math and MUFU ex2, P written
//               as bf16 over its own first 16 S columns.
//   warp 16     TMEM allocator; lane 0 TMA producer for Q and the K ring.
//   warp 17     lane 0 issues S_b = Q K_i^T once K_i has landed and PV of tile i - 3
//               (the last reader of S_b) has retired: up to three tiles ahead.
//   warp 18     lane 0 TMA producer for the V ring.
//   warp 19     lane 0 issues O += P_i V_i once P_i is written.
// Two issuing threads keep the tensor pipe fed while either waits on a barrier;
// each commit tracks the products its own thread issued.
template <int D>
__global__ void __launch_bounds__(kThreadsRing, 1)
attend_bf16_ring_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                        const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKs,
                        const __grid_constant__ CUtensorMap tmVs, const int32_t* __restrict__ Mdev,
                        const float* __restrict__ bias2, int64_t capP,
                        const float* __restrict__ sbias, int64_t Ts, int64_t Tq, int H,
                        __nv_bfloat16* __restrict__ out, float scale_log2, Stats* stats) {
    using C = Cfg<D>;
    using L = CfgR<D>;
    constexpr int kWK = 16, kWQK = 17, kWV = 18, kWPV = 19;
    constexpr int QC = D / 4;   // output (and rescale) columns per softmax thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    float* sBias = reinterpret_cast<float*>(smem + L::OFF_BIAS);   // [3][128]
    float* sBmax = reinterpret_cast<float*>(smem + L::OFF_BMAX);   // [3][4]
    float* sUb = reinterpret_cast<float*>(smem + L::OFF_UB);       // [2][4][128]
    float* sL = reinterpret_cast<float*>(smem + L::OFF_L);         // [4][128]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int q0 = blockIdx.x * kBM;
    const int Mh = Mdev[h];
    const int nc = (Mh + kBN - 1) / kBN;
    const int ntiles = nc + (int)((Ts + kBN - 1) / kBN);

    if (threadIdx.x == 0) {
        mbar_init(&bars[R_QFULL], 1);
        for (int s2 = 0; s2 < kRK; ++s2) {
            mbar_init(&bars[R_KFULL + s2], 1);
            mbar_init(&bars[R_KEMPTY + s2], 1);
        }
        for (int s2 = 0; s2 < kRV; ++s2) {
            mbar_init(&bars[R_VFULL + s2], 1);
            mbar_init(&bars[R_VEMPTY + s2], 1);
        }
        for (int b = 0; b < 3; ++b) {
            mbar_init(&bars[R_SFULL + b], 1);
            mbar_init(&bars[R_PFULL + b], 512);
            mbar_init(&bars[R_ODONE + b], 1);
        }
        mbar_init(&bars[R_DRAIN], 1);
        mbar_init(&bars[R_DRAIN + 1], 1);
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
        uint64_t* full = &bars[kside ? R_KFULL : R_VFULL];
        uint64_t* empty = &bars[kside ? R_KEMPTY : R_VEMPTY];
        const CUtensorMap* mc = kside ? &tmKc : &tmVc;
        const CUtensorMap* ms = kside ? &tmKs : &tmVs;
        if (kside) {
            mbar_expect_tx(&bars[R_QFULL], C::TILE);
            for (int b = 0; b < C::NB; ++b) tma_load_3d(sQ + b * C::BOX, &tmQ, 64 * b, h, q0, &bars[R_QFULL]);
        }
        int last = -1;
        for (int i = 0; i < ntiles && !*abort_flag; ++i) {
            const int st = i % nst;
            if (i >= nst && !mbar_wait(&empty[st], ((i / nst) - 1) & 1)) { *abort_flag = 1; break; }
            const bool cache = i < nc;
            const int row0 = (cache ? i : i - nc) * kBN;
            mbar_expect_tx(&full[st], C::TILE);
            for (int b = 0; b < C::NB; ++b)
                tma_load_3d(ring + st * C::TILE + b * C::BOX, cache ? mc : ms, 64 * b, row0, h, &full[st]);
            last = i;
        }
        if (kside) mbar_wait(&bars[R_QFULL], 0);
        for (int i = (last >= nst - 1 ? last - nst + 1 : 0); i <= last; ++i) mbar_wait(&full[i % nst], (i / nst) & 1);
    } else if (warp == kWQK && lane == 0) {
        // ---------------------------------------------------------------- QK issuer
        const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK);
        bool ok = mbar_wait(&bars[R_QFULL], 0);
        for (int j = 0; ok && j < ntiles && !*abort_flag; ++j) {
            const int b = j % 3, st = j % kRK;
            if (j >= 3 && !mbar_wait(&bars[R_ODONE + b], ((j - 3) / 3) & 1)) { ok = false; break; }
            if (!mbar_wait(&bars[R_KFULL + st], (j / kRK) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t aKs = aK + st * C::TILE;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
                mma_ss(tmem + b * 128, sdesc(aQ + off, 16, 1024), sdesc(aKs + off, 16, 1024), C::IDESC_QK, kk > 0);
            }
            tc_commit(&bars[R_SFULL + b]);
            tc_commit(&bars[R_KEMPTY + st]);
        }
        if (!ok) *abort_flag = 1;
        tc_commit(&bars[R_DRAIN]);
        mbar_wait(&bars[R_DRAIN], 0);
    } else if (warp == kWPV && lane == 0) {
        // ---------------------------------------------------------------- PV issuer
        // O += P_i V_i; keys [16 kk, 16 kk + 16) of P sit at column 128 b + 32 (kk / 2) +
        // 8 (kk % 2): each quarter's probabilities over its own first S columns.
        const uint32_t aV = smem_u32(sV);
        bool ok = true;
        for (int i = 0; i < ntiles && !*abort_flag; ++i) {
            const int b = i % 3, st = i % kRV;
            if (!mbar_wait(&bars[R_PFULL + b], (i / 3) & 1)) { ok = false; break; }
            if (!mbar_wait(&bars[R_VFULL + st], (i / kRV) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t aVs = aV + st * C::TILE;
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
                mma_ts(tO, tmem + b * 128 + 32 * (kk >> 1) + 8 * (kk & 1), sdesc(aVs + kk * 2048, C::BOX, 1024),
                       C::IDESC_PV, (i > 0 || kk > 0));
            tc_commit(&bars[R_VEMPTY + st]);
            tc_commit(&bars[R_ODONE + b]);
        }
        if (!ok) *abort_flag = 1;
        tc_commit(&bars[R_DRAIN + 1]);
        mbar_wait(&bars[R_DRAIN + 1], 0);
    } else if (warp < 16) {
        // ---------------------------------------------------------------- softmax (warps 0-15)
        const int q = warp >> 2;             // column quarter
        const int wt = warp & 3;             // TMEM lane quarter (= SM sub-partition)
        const int r = wt * 32 + lane;        // query row within the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(wt * 32) << 16;
        const uint32_t tOq = tO + QC * q + lane_base;
        const float* bias_h = bias2 + (int64_t)h * capP;
        auto bias_of = [&](int i) -> float {
            return (i < nc) ? bias_h[(int64_t)i * kBN + r] : sbias[(int64_t)(i - nc) * kBN + r];
        };
        // Quarter 0 stages each tile's log2 n row (one value per thread) and its quarter maxima.
        auto stage_bias = [&](int b, float v) {
            sBias[b * 128 + r] = v;
            float wm = v;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
            if (lane == 0) sBmax[b * 4 + wt] = wm;
        };
        const uint64_t c2 = pk2(scale_log2, scale_log2);
        float m_run = -INFINITY, l_run = 0.f;
        float bnext = 0.f;
        if (q == 0) {
            stage_bias(0, bias_of(0));
            if (1 < ntiles) bnext = bias_of(1);
        }
        bool ok = bar_and(1, 512, true);
        for (int i = 0; i < ntiles; ++i) {
            const int b = i % 3, u = i & 1;
            // (warp-uniform: the TMEM loads below are warp-collective)
            const bool got = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&bars[R_SFULL + b], (i / 3) & 1));
            tc_fence_after();
            const uint32_t tS = tmem + b * 128 + 32 * q + lane_base;
            uint32_t sr[32];
            float smax = -INFINITY;
            if (got) {
                TC_LD32(tS, sr);
                tc_wait_ld();
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                    m4[0] = max3(m4[0], __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
                    m4[1] = max3(m4[1], __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]));
                    m4[2] = max3(m4[2], __uint_as_float(sr[j + 4]), __uint_as_float(sr[j + 5]));
                    m4[3] = max3(m4[3], __uint_as_float(sr[j + 6]), __uint_as_float(sr[j + 7]));
                }
                smax = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) sr[j] = 0u;
            }
            sUb[(u * 4 + q) * 128 + r] = fmaf(smax, scale_log2, sBmax[b * 4 + q]);
            // Stage the next tile's log2 n row. Its buffer was last read two tiles ago,
            // before the previous barrier.
            if (q == 0 && i + 1 < ntiles) stage_bias((i + 1) % 3, bnext);
            if (!bar_and(1, 512, got)) { ok = false; break; }
            if (q == 0 && i + 2 < ntiles) bnext = bias_of(i + 2);
            // Reference max: an upper bound of the row max of this tile, agreed by the
            // four quarters. p = 2^(x - m) <= 2^8 below.
            const float ub = fmaxf(fmaxf(sUb[(u * 4 + 0) * 128 + r], sUb[(u * 4 + 1) * 128 + r]),
                                   fmaxf(sUb[(u * 4 + 2) * 128 + r], sUb[(u * 4 + 3) * 128 + r]));
            if (i == 0) {
                m_run = ub;
            } else {
                // Lazy rescaling: O and l keep the old reference until it would grow by more
                // than 8 (a factor 256); then, once PV of the previous tile has retired,
                // each quarter scales its O columns and its partial row sum by alpha.
                const bool need = ub > m_run + 8.f;
                if (__any_sync(0xffffffffu, need)) {
                    const bool w = mbar_wait(&bars[R_ODONE + (i - 1) % 3], ((i - 1) / 3) & 1);
                    if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; }
                    if (ok) {
                        const float alpha = need ? ex2(m_run - ub) : 1.f;
                        if (need) { l_run *= alpha; m_run = ub; }
                        tc_fence_after();
                        uint32_t o[QC];
                        if constexpr (QC == 32) TC_LD32(tOq, o);
                        else TC_LD16(tOq, o);
                        tc_wait_ld();
#pragma unroll
                        for (int c = 0; c < QC; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        if constexpr (QC == 32) TC_ST32(tOq, o);
                        else TC_ST16(tOq, o);
                        tc_wait_st();
                    }
                }
            }
            // p = 2^(s * scale + log2 n - m) over my 32 columns: packed fp32x2 FMA/ADD and
            // MUFU ex2; 16 bf16 pairs go over the first 16 of my S columns.
            const uint64_t negm2 = pk2(-m_run, -m_run);
            uint64_t sumA = pk2(0.f, 0.f), sumB = pk2(0.f, 0.f);
            const float* bh = sBias + b * 128 + 32 * q;
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 b4 = *reinterpret_cast<const float4*>(bh + j);
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
            TC_ST16(tS, pk);
            float s0, s1, s2, s3;
            up2(sumA, s0, s1);
            up2(sumB, s2, s3);
            l_run += (s0 + s1) + (s2 + s3);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[R_PFULL + b]);
        }
        // Epilogue: the last product retires (products retire in order: each commit
        // covers every earlier product of the issuing thread), the quarters add their
        // row sums, and thread (q, r) writes output columns [QC q, QC q + QC).
        const int lastt = ntiles - 1;
        const bool fin = ok && mbar_wait(&bars[R_ODONE + lastt % 3], (lastt / 3) & 1);
        sL[q * 128 + r] = l_run;
        if (bar_and(1, 512, fin)) {
            const float inv = 1.f / ((sL[0 * 128 + r] + sL[1 * 128 + r]) + (sL[2 * 128 + r] + sL[3 * 128 + r]));
            tc_fence_after();
            uint32_t o[QC];
            if constexpr (QC == 32) TC_LD32(tOq, o);
            else TC_LD16(tOq, o);
            tc_wait_ld();
            const int64_t row = q0 + r;
            if (row < Tq) {
                uint4* dst = reinterpret_cast<uint4*>(out + (row * H + h) * D + QC * q);
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


// ---------------------------------------------------------------------------- duo kernel
// Two softmax teams over a three-buffer score ring with one shared output accumulator.
enum { U_QFULL = 0, U_KFULL = 1, U_KEMPTY = 4, U_VFULL = 7, U_VEMPTY = 9, U_SFULL = 11, U_PFULL = 14,
       U_ODONE = 17, U_DRAIN = 20, U_MREADY = 22, U_NBAR = 24 };
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
//   warps 0-15  softmax, two teams of eight warps: team t takes tiles t, t + 2, ...;
//               thread (t, g, r) owns columns [64 g, 64 g + 64) of query row r (TMEM
//               lane r), so every SM sub-partition runs two warps of each team and the
//               teams' phases interleave. Per tile the halves agree on an upper bound of
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
template <int D>
__global__ void __launch_bounds__(kThreadsRing, 1)
attend_bf16_duo_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                       const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKs,
                       const __grid_constant__ CUtensorMap tmVs, const int32_t* __restrict__ Mdev,
                       const float* __restrict__ bias2, int64_t capP,
                       const float* __restrict__ sbias, int64_t Ts, int64_t Tq, int H,
                       __nv_bfloat16* __restrict__ out, float scale_log2, Stats* stats) {
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

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int q0 = blockIdx.x * kBM;
    const int Mh = Mdev[h];
    const int nc = (Mh + kBN - 1) / kBN;
    const int ntiles = nc + (int)((Ts + kBN - 1) / kBN);

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
            mbar_init(&bars[U_PFULL + b], 256);
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
            for (int b = 0; b < C::NB; ++b) tma_load_3d(sQ + b * C::BOX, &tmQ, 64 * b, h, q0, &bars[U_QFULL]);
        }
        int last = -1;
        for (int i = 0; i < ntiles && !*abort_flag; ++i) {
            const int st = i % nst;
            if (i >= nst && !mbar_wait(&empty[st], ((i / nst) - 1) & 1)) { *abort_flag = 1; break; }
            const bool cache = i < nc;
            const int row0 = (cache ? i : i - nc) * kBN;
            mbar_expect_tx(&full[st], C::TILE);
            for (int b = 0; b < C::NB; ++b)
                tma_load_3d(ring + st * C::TILE + b * C::BOX, cache ? mc : ms, 64 * b, row0, h, &full[st]);
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
        // O += P_i V_i; keys [16 kk, 16 kk + 16) of P sit at column 128 b + 64 (kk / 4) +
        // 8 (kk % 4): each half's probabilities over its own first S columns.
        const uint32_t aV = smem_u32(sV);
        bool ok = true;
        for (int i = 0; i < ntiles && !*abort_flag; ++i) {
            const int b = i % 3, st = i % kRV;
            if (!mbar_wait(&bars[U_PFULL + b], (i / 3) & 1)) { ok = false; break; }
            if (!mbar_wait(&bars[U_VFULL + st], (i / kRV) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t aVs = aV + st * C::TILE;
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
                mma_ts(tO, tmem + b * 128 + 64 * (kk >> 2) + 8 * (kk & 3), sdesc(aVs + kk * 2048, C::BOX, 1024),
                       C::IDESC_PV, (i > 0 || kk > 0));
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
        const float* bias_h = bias2 + (int64_t)h * capP;
        auto bias_of = [&](int i) -> float {
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
        float bnext = 0.f;
        if (g == 0) {
            if (t < ntiles) stage_bias(0, bias_of(t));
            if (t + 2 < ntiles) bnext = bias_of(t + 2);
        }
        bool ok = bar_and(1 + t, 256, true);
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
#pragma unroll
                for (int j = 0; j < 64; j += 8) {
                    m4[0] = max3(m4[0], __uint_as_float(sr[j]), __uint_as_float(sr[j + 1]));
                    m4[1] = max3(m4[1], __uint_as_float(sr[j + 2]), __uint_as_float(sr[j + 3]));
                    m4[2] = max3(m4[2], __uint_as_float(sr[j + 4]), __uint_as_float(sr[j + 5]));
                    m4[3] = max3(m4[3], __uint_as_float(sr[j + 6]), __uint_as_float(sr[j + 7]));
                }
                smax = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
            }
            const float2 bm = *reinterpret_cast<const float2*>(sBmax + (t * 3 + bb) * 4 + 2 * g);
            sUb[((t * 2 + u) * 2 + g) * 128 + r] = fmaf(smax, scale_log2, fmaxf(bm.x, bm.y));
            if (g == 0 && i + 2 < ntiles) stage_bias((k + 1) % 3, bnext);
            if (!bar_and(1 + t, 256, got)) { ok = false; break; }
            if (g == 0 && i + 4 < ntiles) bnext = bias_of(i + 4);
            const float ub = fmaxf(sUb[((t * 2 + u) * 2 + 0) * 128 + r], sUb[((t * 2 + u) * 2 + 1) * 128 + r]);
            // The reference of tile i - 1, decided by the other team.
            float mprev = -INFINITY;
            if (i > 0) {
                const bool w = mbar_wait(&bars[U_MREADY + (t ^ 1)], ((i - 1) >> 1) & 1);
                if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; }
                mprev = sMref[(t ^ 1) * 128 + r];
            }
            const bool raise = i == 0 || ub > mprev + 8.f;
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
                    const float4 b4 = *reinterpret_cast<const float4*>(bh + 32 * h2 + j);
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
            mbar_arrive(&bars[U_PFULL + b]);
        }
        // Epilogue: the last product retires (each commit covers every earlier product of
        // the PV issuer), every row sum moves to the final reference, and thread (t, g, r)
        // writes output columns [QC (2 t + g), QC (2 t + g + 1)) of its row.
        const int lastt = ntiles - 1;
        bool fin = ok && mbar_wait(&bars[U_ODONE + lastt % 3], (lastt / 3) & 1);
        fin = fin && mbar_wait(&bars[U_MREADY + (lastt & 1)], (lastt >> 1) & 1);
        const float mfin = sMref[(lastt & 1) * 128 + r];
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
            if (row < Tq) {
                uint4* dst = reinterpret_cast<uint4*>(out + (row * H + h) * D + col);
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

template <int D>
cudaError_t launch_t(const CacheView& c, const StageView& s, const AttnMaps& m, int64_t Tq, __nv_bfloat16* out,
                     float scale_log2, Stats* stats, bool overlap_prev, cudaStream_t st) {
    using C = Cfg<D>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = kDuo ? cudaFuncSetAttribute(attend_bf16_duo_kernel<D>,
                                                    cudaFuncAttributeMaxDynamicSharedMemorySize, CfgU<D>::SMEM)
                        : kRing ? cudaFuncSetAttribute(attend_bf16_ring_kernel<D>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, CfgR<D>::SMEM)
                        : kSplit ? cudaFuncSetAttribute(attend_bf16_split_kernel<D>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, CfgS<D>::SMEM)
                        : kTeams == 2 ? cudaFuncSetAttribute(attend_bf16_teams_kernel<D>,
                                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM)
                                      : cudaFuncSetAttribute(attend_bf16_kernel<D>,
                                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((Tq + kBM - 1) / kBM), (unsigned)c.H);
    cfg.blockDim = dim3((kDuo || kRing) ? kThreadsRing : kSplit ? kThreadsSplit : kThreads);
    cfg.dynamicSmemBytes = kDuo ? CfgU<D>::SMEM : kRing ? CfgR<D>::SMEM : kSplit ? CfgS<D>::SMEM : C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = overlap_prev ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if constexpr (kDuo)
        return cudaLaunchKernelEx(&cfg, attend_bf16_duo_kernel<D>, m.q, m.kc, m.vc, m.ks, m.vs,
                                  (const int32_t*)c.M, (const float*)c.bias2, c.capP,
                                  (const float*)s.sbias, s.T, Tq, c.H, out, scale_log2, stats);
    else if constexpr (kRing)
        return cudaLaunchKernelEx(&cfg, attend_bf16_ring_kernel<D>, m.q, m.kc, m.vc, m.ks, m.vs,
                                  (const int32_t*)c.M, (const float*)c.bias2, c.capP,
                                  (const float*)s.sbias, s.T, Tq, c.H, out, scale_log2, stats);
    else if constexpr (kSplit)
        return cudaLaunchKernelEx(&cfg, attend_bf16_split_kernel<D>, m.q, m.kc, m.vc, m.ks, m.vs,
                                  (const int32_t*)c.M, (const float*)c.bias2, c.capP,
                                  (const float*)s.sbias, s.T, Tq, c.H, out, scale_log2, stats);
    else if constexpr (kTeams == 2)
        return cudaLaunchKernelEx(&cfg, attend_bf16_teams_kernel<D>, m.q, m.kc, m.vc, m.ks, m.vs,
                                  (const int32_t*)c.M, (const float*)c.bias2, c.capP,
                                  (const float*)s.sbias, s.T, Tq, c.H, out, scale_log2, stats);
    else
        return cudaLaunchKernelEx(&cfg, attend_bf16_kernel<D>, m.q, m.kc, m.vc, m.ks, m.vs, (const int32_t*)c.M,
                                  (const float*)c.bias2, c.capP, (const float*)s.sbias, s.T, Tq, c.H, out,
                                  scale_log2, stats);
}

}  // namespace

cudaError_t launch_attend_bf16(const CacheView& c, const StageView& s, const AttnMaps& maps, int64_t Tq,
                               __nv_bfloat16* out, float scale_log2, Stats* stats, bool overlap_prev,
                               cudaStream_t st) {
    return c.d == 128 ? launch_t<128>(c, s, maps, Tq, out, scale_log2, stats, overlap_prev, st)
                      : launch_t<64>(c, s, maps, Tq, out, scale_log2, stats, overlap_prev, st);
}

}  // namespace tc
