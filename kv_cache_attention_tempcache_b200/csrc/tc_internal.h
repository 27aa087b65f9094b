// Internal declarations shared by the TempCache host runtime and its kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>
#include <set>
#include <utility>
#include <vector>

namespace tc {

// Device state of one TempCache. Per-head arrays have a padded row stride
// capP = round_up(capacity, 128) so a 128-row attention tile never leaves its head.
struct CacheView {
    int H, d, nbits;
    int64_t capP;          // padded capacity per head
    int64_t capacity;      // usable entries per head
    void* Kc;              // [H][capP][d] storage type, entry keys (the attention operand)
    float* K32;            // [H][capP][d] fp32 key means with running-mean keys (bf16 storage; the
                           // same array as Kc with fp32 storage); null with representative keys
    void* Vc;              // [H][capP][d] storage type, value means (attention operand)
    float* V32;            // [H][capP][d] fp32 value means (master copy)
    int32_t* cnt;          // [H][capP] group sizes n
    float* bias2;          // [H][capP] log2(n); -inf for unused rows
    uint32_t* code;        // [H][capP]
    int32_t* bnext;        // [H][capP] next older entry in the same bucket, -1 ends
    int32_t* bhead;        // [H][2^nbits] newest entry of each bucket, -1 = empty
    double* knorm64;       // [H][capP] |k|^2 of each entry, fp64 summed in index order
    uint8_t* kspan;        // [H][capP] exponent span of each bf16 key (exact-sum rule of the search), <= 255
    int32_t* lhead;        // [H][capP] newest token merging into the entry in this commit (-1 between commits)
    int32_t* M;            // [H] committed entries
    // Upper bounds for the attention's fixed softmax reference (floats >= 0, raised with
    // integer atomicMax on their bits): |k|^2 of any committed entry per head, |k|^2 of
    // any staged token (all heads), log2 n of any committed entry per head.
    float* kmax2;          // [H]
    float* kmax2s;         // [1] (cleared before each staging)
    float* bmax;           // [H]
    int32_t* cbhead;       // [H][2^nbits] newest staged token of each bucket during a commit that matches
                           // inside the chunk (-1 between commits); null when that mode is off
};

struct StageView {
    int64_t TmaxP;         // staging rows per head (multiple of 128)
    int64_t T;             // tokens staged (or being committed)
    void* Ks;              // [H][TmaxP][d]
    void* Vs;              // [H][TmaxP][d]
    uint32_t* scode;       // [H][TmaxP] hash codes of the staged tokens
    float* sbias;          // [TmaxP] 0 for t < T, -inf beyond
    int32_t* match;        // [H][TmaxP] merge target or -1 of each staged token, decided at staging
                           // (the cache cannot change between staging and commit)
    int32_t* lmatch;       // [H][TmaxP] merge targets of the last committed chunk
    int32_t* dest;         // [H][TmaxP] entry each token ended in (last commit)
    uint32_t* lcode;       // [H][TmaxP] codes of the last committed chunk
    int32_t* lnext;        // [H][TmaxP] next (older) token of the same merge list
    int32_t* wcnt;         // [H][TmaxP/32] unmatched tokens per 32-token window (0 between commits)
    int32_t* touched;      // [H][TmaxP] entries with at least one merge
    // matching inside the chunk (see the dedupe kernel):
    double* bsim;          // [H][TmaxP] best committed similarity of each token (-inf: none)
    int32_t* cbnext;       // [H][TmaxP] next older staged token with the same code
    int32_t* crnext;       // [H][TmaxP] next token that created an entry in the same bucket
    int32_t* ichead;       // [H][TmaxP] first token merging into the entry this token created (-1: none)
    int32_t* ictail;       // [H][TmaxP] last such token
    int32_t* icnext;       // [H][TmaxP] next token merging into the same new entry
    // running-mean keys: entries whose merged key changed code in the last commit
    int32_t* moved;        // [H][TmaxP] entry
    uint32_t* movedold;    // [H][TmaxP] its code before the commit
};

// Per-commit counters (int32). The staging kernels of a chunk fill them and the last
// kernel of that chunk's commit clears them (the host clears them on a reset):
//   ctr[0, H)        entries touched by merges, per head
//   ctr[H, 2H)       cache size after the commit, per head
//   ctr[2H]          abort flag: some head would exceed its capacity
//   ctr[2H+1]        ticket of the staging kernel that publishes the sizes
//   ctr[2H+2]        ticket of the commit kernel
//   ctr[2H+3]        ticket of the last re-bucketing kernel (running-mean keys)
//   ctr[2H+4, 3H+4)  entries whose key changed code, per head (running-mean keys)
__host__ __device__ constexpr int kCtrInts(int H) { return 3 * H + 4; }

// Sticky device-side statistics and error bits.
enum : unsigned { kErrBucketList = 1u, kErrTimeout = 2u };
struct Stats {
    unsigned long long hash_rechecks;
    unsigned long long match_rechecks;
    unsigned int error_bits;
    unsigned int pad;
};

// Launchers (tc_commit.cu). launch_stage copies, hashes and searches the chunk s.T
// (plus the in-chunk dedupe when intra); launch_commit applies the staged chunk's
// decisions (plus the re-bucketing with running-mean keys). R: device normals;
// Rhost, Rnorm_host: host copies of the normals and of |R_b| (rounded up).
cudaError_t launch_stage(const CacheView& c, const StageView& s, int dtype, bool intra, bool mean, const void* K,
                         const void* V, const float* R, const float* Rhost, const float* Rnorm_host, float tau,
                         int32_t* ctr, Stats* stats, int* launches, cudaStream_t st);
cudaError_t launch_commit(const CacheView& c, const StageView& s, int dtype, bool mean, const float* R,
                          const float* Rnorm, int32_t* ctr, int32_t* claim, Stats* stats, int* launches,
                          cudaStream_t st);

// Launchers (tc_attn_f32.cu, tc_attn_bf16.cu).
cudaError_t launch_attend_f32(const CacheView& c, const StageView& s, const float* Q,
                              int64_t Tq, float* out, float scale_log2, cudaStream_t st);

struct AttnMaps {
    CUtensorMap q, kc, vc, ks, vs;
};
cudaError_t launch_attend_bf16(const CacheView& c, const StageView& s, const AttnMaps& maps,
                               int64_t Tq, __nv_bfloat16* out, float scale_log2, Stats* stats,
                               bool overlap_prev, cudaStream_t st);


// Device state of one AnnCA cross-attention layer (tc_annca.cu). The prompt is kept
// head-major with a padded row stride Lp = round_up(L, 128); the query block being
// attended holds F frames, and (head h, frame f) is slot z = h F + f of the per-frame
// arrays, each Lp rows long.
struct AnnView {
    int H, d, nbits;
    int L;                 // prompt tokens
    int64_t Lp;            // padded prompt rows per head (and per slot)
    __nv_bfloat16* Kh;     // [H][Lp][d] prompt keys
    __nv_bfloat16* Vh;     // [H][Lp][d] prompt values
    uint32_t* pcode;       // [H][Lp] hash codes of the prompt keys
    uint32_t* pcs;         // [H][Lp] the same codes in ascending order
    int32_t* pix;          // [H][Lp] prompt token of each sorted code (ties by token)
    int32_t* prun;         // [H][Lp] first sorted position of each prompt token's code
    int32_t* ptab;         // [H][2^nbits] first sorted position of each code, -1 if the prompt has
                           // none (nbits <= 16; null otherwise: binary search in pcs)
    float* kmax2;          // [H] upper bound of |k|^2 over the prompt keys
    float* zeros;          // [H] zeros: log2 n bound and staged-key bound of the attention
    int64_t Tmax;          // query rows the per-query arrays hold
    uint32_t* qcode;       // [Tmax][H] hash codes of the last query block (token-major)
    int64_t Zmax;          // slots the per-frame arrays hold
    uint32_t* keep;        // [Zmax][Lp] per slot, one stamp per bucket of the prompt, at the
                           // bucket's first sorted position: equal to gen when a query of the
                           // slot has that code in the current call
    uint32_t gen;          // stamp of the current call (>= 1; the stamps start at 0)
    int32_t* nsel;         // [Zmax] kept prompt tokens per slot
    int32_t* sidx;         // [Zmax][Lp] kept prompt tokens in ascending order
    __nv_bfloat16* Ks;     // [Zmax][Lp][d] kept keys, packed; rows up to the next multiple of 128 zeroed
    __nv_bfloat16* Vs;     // [Zmax][Lp][d] kept values, packed the same way
    float* sbias;          // [Zmax][Lp] 0 for kept rows, -inf for the rest of the last tile
};

// AnnSA (same-bucket self-attention) arrays read by the attention kernel's sparse mode:
// the tokens of one block in bucket order per head ("packed" rows, Tp = round_up(T, 128)).
struct SparseArgs {
    const int2* tiles;     // [H][nqt] key tiles [x, y) holding the buckets of each query tile
    const uint32_t* grp;   // [H][Tp] bucket code of each packed row (0xffffffff past T)
    const int32_t* perm;   // [H][Tp] token of each packed row
    const float* xself;    // [H][Tp] the row's own logit, scale log2(e) <q, k>
    int64_t Tp;            // row stride per head (>= round_up(T, 128))
    int nqt;               // Tp / 128, the row stride of tiles
};

// LVSA frame-mask arrays read by the attention kernel's frame mode (tc_lvsa.cu): per query
// frame, the key tiles that cover the frames it attends to.
struct FrameArgs {
    const int2* tiles;     // [T][maxt] (first token row, valid rows <= 128) of each key tile
    const int32_t* count;  // [T] key tiles of each query frame
    const float* masktab;  // [129][128]: row v holds 0 in its first v columns, -inf after
    int maxt;
};

// Launchers (tc_annca.cu, tc_attn_bf16.cu).
cudaError_t launch_annca_prompt(const AnnView& a, const void* Kp, const void* Vp, const float* R,
                                const float* Rnorm, Stats* stats, cudaStream_t st);
// R: device normals (fp64 re-checks); Rhost, Rnorm_host: host copies, passed to the
// hash kernel by value.
cudaError_t launch_annca_select(const AnnView& a, const void* Q, int64_t Tq, int P, int F, const float* R,
                                const float* Rhost, const float* Rnorm_host, Stats* stats, cudaStream_t st);
cudaError_t launch_attend_cross_bf16(const AnnView& a, const AttnMaps& maps, int64_t Tq, int P, int F,
                                     __nv_bfloat16* out, float scale_log2, Stats* stats, cudaStream_t st);
// maps.q / maps.kc / maps.vc: token-major Q, K, V [T P, H, d] (box 64 x 1 x 128).
cudaError_t launch_attend_frames_bf16(int H, int d, const FrameArgs& fa, const AttnMaps& maps, int T, int P,
                                      const float* big, const float* zeros, __nv_bfloat16* out, float scale_log2,
                                      Stats* stats, cudaStream_t st);
// maps.q: packed queries [H][Tp][d]; maps.kc / maps.vc: packed keys and values, same shape.
cudaError_t launch_attend_sparse_bf16(int H, int d, const SparseArgs& sp, const AttnMaps& maps, int64_t T,
                                      const float* kmax2, const float* zeros, __nv_bfloat16* out,
                                      float scale_log2, Stats* stats, cudaStream_t st);
// Bucket order and packing of one block for the sparse attention (tc_annca.cu).
struct SparseBufs {
    int H, d;
    int64_t T, Tp;          // tokens; row stride per head of the packed arrays (>= round_up(T, 128))
    const uint32_t* codes;  // [T][H] bucket codes (token-major)
    int32_t* perm;          // [H][Tp]
    uint32_t* grp;          // [H][Tp]
    int2* tiles;            // [H][Tp/128]
    float* xself;           // [H][Tp]
    __nv_bfloat16* Qs;      // [H][Tp][d]
    __nv_bfloat16* Ks;
    __nv_bfloat16* Vs;
    float* kmax2;           // [H], cleared by the ordering kernel
    int32_t* bcnt;          // [H][blocks][2^nbits] per-block code counts of the ordering (short codes)
};
cudaError_t launch_annsa_pack(const SparseBufs& b, int nbits, const void* Q, const void* K, const void* V,
                              float scale_log2, cudaStream_t st);

// Raises a kernel's dynamic shared-memory limit once per (device, kernel): function
// attributes belong to each device's copy of the kernel, so a process that drives several
// GPUs needs the call on each of them.
inline cudaError_t smem_attr_once(const void* kern, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<int, const void*>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({dev, kern})) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert({dev, kern});
    return e;
}

// Host helpers (tc_runtime.cu).
cudaError_t dev_alloc(void** p, size_t bytes);   // cudaMalloc with the TC_FAULT_ALLOC_AT injection
float round_bf16(float x);
bool is_bf16_value(float x);
void default_hyperplanes(uint64_t seed, int n, std::vector<float>& out);
bool get_encoder();
// 3-D bf16 tensor map with a 128-byte swizzle; dims and box innermost first, strides in bytes.
bool encode3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
              uint32_t b0, uint32_t b1, uint32_t b2);

}  // namespace tc
