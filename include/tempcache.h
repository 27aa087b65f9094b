/*
 * tempcache.h - C ABI of the TempCache step on one NVIDIA B200 (sm_100a).
 *
 * TempCache (FAST-AR technical summary, section 2.A "TempCache", pt and fr pages)
 * compresses the temporal KV cache of an autoregressive video-diffusion attention
 * layer: every new key is hashed with locality-sensitive hashing, matched top-1
 * against the earlier cache entries, and merged into its match when their
 * similarity clears a threshold (values averaged, group size n counted); keys
 * that find no match are appended. Attention then runs over the compressed cache
 * plus the current chunk and shifts each cache logit by ln n, which Lemma 5.1 of
 * the paper states is exact when the merged keys are identical.
 *
 * Conventions for every call below
 *   - Token-major tensors K, V, Q, out are row-major [T, H, d] arrays in DEVICE
 *     memory, in the handle's storage type (bf16 or fp32), 16-byte aligned and
 *     contiguous. The caller owns them; the library reads K and V only inside the
 *     stream-ordered work it enqueues and copies them into its own memory.
 *   - tc_stream is a cudaStream_t value (NULL = the legacy default stream). Calls
 *     on one handle must use one stream at a time; handles are not thread-safe.
 *   - Host-detectable errors (bad argument, wrong state, out of memory) return at
 *     once and change nothing. Errors seen by a kernel are sticky: the next call
 *     that synchronises (tc_sync, tc_cache_size, the export calls) returns them,
 *     and every later call returns them too.
 *   - Every call returns TC_EINVAL for a NULL or destroyed handle.
 */
#ifndef TEMPCACHE_H
#define TEMPCACHE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tc_ctx* tc_handle;
typedef void* tc_stream;

typedef enum {
    TC_OK = 0,
    TC_EINVAL = 1,     /* bad argument or handle                                   */
    TC_ENOMEM = 2,     /* device or host allocation failed                         */
    TC_ECAPACITY = 3,  /* a commit would exceed the per-head capacity              */
    TC_ECUDA = 4,      /* a CUDA runtime or driver call failed                     */
    TC_ESTATE = 5,     /* call not valid in the current state                      */
    TC_ETIMEOUT = 6,   /* a kernel gave up waiting on one of its own barriers      */
    TC_ENOTIMPL = 7,   /* combination of options the library does not support      */
    TC_EDEVICE = 8     /* no usable sm_100 device                                  */
} tc_status;

typedef enum { TC_BF16 = 0, TC_F32 = 1 } tc_dtype;

typedef struct {
    tc_dtype dtype;            /* storage and I/O type of K, V, Q, out                  */
    uint64_t seed;             /* seed of the default hyperplanes                      */
    float softmax_scale;       /* 0 selects 1/sqrt(d)                                  */
    const float* hyperplanes;  /* HOST [nbits*d] hash normals, each value exactly
                                  representable in bf16; NULL = N(0,1) draws from seed,
                                  rounded to bf16. Copied during the call.              */
    int32_t intra_chunk;       /* 0: a commit matches its tokens against the entries
                                  committed before it only (section 2.A read as a
                                  snapshot). 1: tokens are taken in ascending t and also
                                  match entries created earlier in the same commit, so
                                  duplicates inside one chunk merge too (the other
                                  reading of the same passage). Costs one more kernel and
                                  4 * 2^nbits bytes per head.                             */
    int32_t key_mode;          /* 0: an entry keeps the key that created it (section 2.A
                                  says values are averaged; keys are read as kept). 1: an
                                  entry's key is the running mean of its members' keys,
                                  k <- (n k + sum k_t) / (n + m) in fp32 in ascending t
                                  (the other reading of the same passage); the entry's
                                  code is recomputed from the new key and it moves to that
                                  bucket for later commits, attention uses the mean key.
                                  Requires intra_chunk = 0. Costs 4 d bytes per entry
                                  (bf16 storage), 4 * 2^nbits bytes per head and two more
                                  kernels per commit.                                      */
} tc_options;

/*
 * tc_create / tc_create_ex - allocate a TempCache for one attention layer.
 *   H         heads (>= 1); every head has its own cache.
 *   d         head dimension: 64 or 128.
 *   nbits     hash bits, 1..24 (section 2.A: locality-sensitive hashing; the hash
 *             family is sign-of-random-hyperplane, 2^nbits buckets per head).
 *   tau       cosine threshold for a merge, -1 <= tau <= 2 (section 2.A: merges
 *             use a similarity threshold). tau > 1 never merges (dense cache).
 *   capacity  cache entries per head (>= 1). All device memory for `capacity`
 *             entries is allocated here.
 * tc_create uses bf16 storage, seed 0 and scale 1/sqrt(d).
 * On success *out owns every device buffer of the cache; release it with
 * tc_destroy. On failure *out is set to NULL. Returns TC_EDEVICE when the
 * current device is not an sm_100 part.
 */
tc_status tc_create(int32_t H, int32_t d, int32_t nbits, float tau, int64_t capacity,
                    tc_handle* out);
tc_status tc_create_ex(int32_t H, int32_t d, int32_t nbits, float tau, int64_t capacity,
                       const tc_options* opt, tc_handle* out);

/*
 * tc_append_chunk - feed the next chunk of T new tokens, K and V [T, H, d].
 * First commits the chunk staged by the previous call, then stages this chunk.
 * Staging copies the chunk into the library's head-major staging buffer, hashes
 * its keys and takes every merge decision (section 2.A: each new key is matched
 * top-1 in its hash bucket among the entries committed before its commit, which
 * are already final at staging; a match at cosine >= tau merges). The commit
 * applies them: v <- (n v + sum v_t)/(n + m), n <- n + m for merges, unmatched
 * keys appended in token order. Attention sees a staged chunk raw, with logit
 * shift 0.
 * Asynchronous on `stream`, except when the committed cache might overflow its
 * capacity: then the call synchronises to learn the outcome and, if the commit
 * would overflow, returns TC_ECAPACITY with the cache unchanged, the previous
 * chunk still staged and this chunk not accepted.
 * T >= 1 and T * H < 2^31. Returns TC_EINVAL for NULL or misaligned K or V.
 */
tc_status tc_append_chunk(tc_handle h, const void* K, const void* V, int64_t T,
                          tc_stream stream);

/*
 * tc_attend - biased attention of Q [Tq, H, d] over the committed cache entries
 * (logit shift ln n_j) and the staged chunk (shift 0); writes out [Tq, H, d].
 * out_t = sum_j exp(s_tj) v_j / sum_j exp(s_tj), s_tj = scale <q_t, k_j> + shift_j,
 * no mask (section 2.A with Lemma 5.1: averaged values plus a logit shift by the
 * group size reproduce attention over the identical keys they replace).
 * bf16 handles compute QK^T and PV on tensor cores with fp32 accumulation and an
 * fp32 softmax whose reference per query row is a bound of its logits (|q| times
 * the largest key norm, scaled, plus the largest ln n) when that bound is small
 * enough to rule out underflow, else a running maximum; fp32 handles compute in
 * fp32 throughout.
 * Asynchronous on `stream`. Tq >= 1. Returns TC_ESTATE before the first
 * tc_append_chunk. out must not overlap Q.
 */
tc_status tc_attend(tc_handle h, const void* Q, int64_t Tq, void* out, tc_stream stream);

/* tc_flush - commit the staged chunk (if any) and stage nothing. Same capacity
 * behaviour as tc_append_chunk. */
tc_status tc_flush(tc_handle h, tc_stream stream);

/* tc_reset - empty the cache and drop any staged chunk, keeping every allocation
 * (start a new rollout). Asynchronous on `stream`. */
tc_status tc_reset(tc_handle h, tc_stream stream);

/* tc_cache_size - synchronise and write the committed entry count of every head
 * to the HOST array sizes_H [H]. */
tc_status tc_cache_size(tc_handle h, int64_t* sizes_H);

/* tc_sync - synchronise the handle's last stream and return its sticky status. */
tc_status tc_sync(tc_handle h);

/* tc_destroy - free every buffer of the handle. NULL-safe. Synchronises. */
void tc_destroy(tc_handle h);

/* tc_status_string - static description of a status code. */
const char* tc_status_string(tc_status s);

/* ---- inspection (host buffers; every call synchronises) -------------------- */

/* Codes, merge targets (-1 = appended) and final entry index of every token of the
 * last committed chunk, as HOST arrays [H * T] (head-major); *T_out receives T
 * (0 if nothing was committed). Any array pointer may be NULL. */
tc_status tc_debug_last_commit(tc_handle h, int64_t* T_out, uint32_t* codes_HT,
                               int32_t* match_HT, int32_t* dest_HT);

/* Hash codes of the staged chunk, HOST [H * T_staged]; *T_out receives T_staged. */
tc_status tc_debug_staged_codes(tc_handle h, int64_t* T_out, uint32_t* codes_HT);

/* Committed entries of head `head` (count from tc_cache_size) into HOST arrays:
 * K [M*d] in the storage type, V32 [M*d] fp32 running means, n [M], code [M].
 * Any pointer may be NULL. */
tc_status tc_export_cache(tc_handle h, int32_t head, void* K, float* V32, int32_t* n,
                          uint32_t* code);

/* Running-mean keys (key_mode 1): the fp32 key means of head `head`'s committed
 * entries, HOST K32 [M*d]. TC_ESTATE for a handle with representative keys. */
tc_status tc_export_key_means(tc_handle h, int32_t head, float* K32);

/* The hash normals in use, HOST [nbits * d]. */
tc_status tc_get_hyperplanes(tc_handle h, float* R);

/* Kernels this handle has launched so far; hash bits that needed the exact fp64
 * re-check (the fp32 sign was inside its rounding bound); and similarity sums that
 * took the sequential index-order fp64 path (bf16 rows outside the exact-sum
 * exponent range, or fp32 decisions inside their rounding bound). */
tc_status tc_stats(tc_handle h, uint64_t* kernel_launches, uint64_t* hash_rechecks,
                   uint64_t* match_rechecks);

/* ---- allocation-free entry point -------------------------------------------- */

/*
 * tc_merge_means_noalloc - average matched rows into running means, allocating
 * nothing. The paper has no counterpart to this call: it exists for callers that
 * may not allocate device memory once they are running, such as inference
 * runtimes that reserve a single fixed arena at start-up, or plugins inside a
 * framework whose allocator owns the whole device. It is the library's merge step
 * (values averaged, counts added) on buffers the caller owns:
 *   for every destination row j, with S_j = { i : target[i] == j } in ascending i,
 *     mean[j]  <- (count[j] * mean[j] + sum_{i in S_j} src[i]) / (count[j] + |S_j|)
 *     count[j] <- count[j] + |S_j|
 *   summed in fp32 in ascending i, so the result does not depend on scheduling.
 *   src     DEVICE [n_src, d] in src_dtype (bf16 or fp32), read only.
 *   target  DEVICE [n_src] int32 destination row or -1 (skip); values outside
 *           [0, n_dst) are skipped too.
 *   mean    DEVICE [n_dst, d] fp32, updated in place; count DEVICE [n_dst] int32,
 *           updated in place. Rows no source targets are left as they are. A row
 *           with count 0 that some source targets becomes the plain mean of its
 *           sources (its old contents, even NaN, are not read into the result).
 *   d       64 or 128.
 *   src and target must not overlap mean or count, nor mean overlap count
 *   (TC_EINVAL otherwise).
 * Limits: n_src <= 65536 and n_dst <= 262144; larger sizes return TC_EINVAL and
 * launch nothing. Scratch lives in a fixed device array of about 3.4 MB that every
 * GPU loading the library holds until the process exits; the call never calls
 * cudaMalloc, cudaFree or any allocating routine. The first call in each CUDA
 * context looks up that array's device address in that context and caches it per
 * context (a device reset or another current context triggers a new lookup); make
 * that first call before any stream capture. All calls share the array: calls whose
 * GPU work overlaps (other streams or host threads on the same device) race and
 * corrupt each other's results, so keep them ordered.
 * Asynchronous on `stream`; returns TC_ECUDA if a launch fails.
 */
tc_status tc_merge_means_noalloc(const void* src, tc_dtype src_dtype, const int32_t* target,
                                 int32_t n_src, int32_t d, float* mean, int32_t* count,
                                 int32_t n_dst, tc_stream stream);

/* ---- AnnCA: cross-attention over the prompt tokens a frame shares buckets with -- */

/*
 * AnnCA (FAST-AR technical summary, section 2.B "AnnCA", pt and fr pages): the
 * latent queries of a frame and the prompt keys are hashed into one space; a prompt
 * token is kept for the frame when its bucket holds at least one of the frame's
 * queries, and the frame's cross-attention runs over the kept tokens only. Here
 * the hash is the sign of nbits random hyperplanes (the TempCache hash, with the
 * cross-attention layer's own normals, shared by the heads), buckets are exact
 * codes, and the kept set is decided per frame and per head. A frame whose queries
 * share no bucket with the prompt gets zero output rows (the empty sum).
 * Same conventions as above; bf16 only.
 */
typedef struct tc_annca_ctx* tc_annca_handle;

/*
 * tc_annca_create - a cross-attention layer with H heads of dimension d (64 or
 * 128) and nbits hash bits (1..24). opt may be NULL (seed 0, scale 1/sqrt(d));
 * opt->dtype must be TC_BF16 (TC_F32 returns TC_ENOTIMPL) and opt->intra_chunk 0.
 * Allocates nothing until the prompt is set. *out is NULL on failure.
 */
tc_status tc_annca_create(int32_t H, int32_t d, int32_t nbits, const tc_options* opt,
                          tc_annca_handle* out);

/*
 * tc_annca_set_prompt - the prompt keys and values, Kp and Vp DEVICE [L, H, d]
 * bf16, 1 <= L <= 4096. The library copies them into its own memory, hashes the
 * keys and sorts their codes, all on `stream`; the caller may free Kp and Vp once
 * that work has run. Growing L past the largest earlier value reallocates (and
 * synchronises first).
 */
tc_status tc_annca_set_prompt(tc_annca_handle h, const void* Kp, const void* Vp, int32_t L,
                              tc_stream stream);

/*
 * tc_annca_attend - cross-attention of the query block Q DEVICE [Tq, H, d] bf16,
 * Tq = F P: F frames of P consecutive tokens (frame f is rows f P .. f P + P - 1).
 * For frame f and head h the kept tokens are the prompt tokens whose code equals
 * the code of at least one query of that frame and head; then
 *   out_t = sum_{l kept} exp(scale <q_t, k_l>) v_l / sum_{l kept} exp(scale <q_t, k_l>)
 * on tensor cores (bf16 products, fp32 accumulation and softmax), and zero rows
 * where nothing is kept. Writes out DEVICE [Tq, H, d] bf16, which must not overlap
 * Q. Asynchronous on `stream`: one hash-and-mark kernel, one packing kernel and the
 * attention kernel. Returns TC_ESTATE before a prompt is set and TC_EINVAL unless
 * P >= 1, Tq is a positive multiple of P and Tq * H < 2^31. Growing Tq or F past the largest
 * earlier value reallocates (and synchronises first).
 */
tc_status tc_annca_attend(tc_annca_handle h, const void* Q, int64_t Tq, int32_t P, void* out,
                          tc_stream stream);

/*
 * tc_annca_kept - inspection of the last tc_annca_attend (HOST buffers; synchronises).
 * *T_out receives its Tq, *F_out its F and *L_out the prompt length (0 before any). counts [H*F]: kept tokens of slot
 * h F + f; index [H*F*L]: slot z's kept prompt tokens in ascending order in
 * index[z*L .. z*L + counts[z]) (the rest unspecified); qcodes [H*Tq] head-major
 * query codes; pcodes [H*L] prompt codes. Any array pointer may be NULL.
 */
tc_status tc_annca_kept(tc_annca_handle h, int64_t* T_out, int64_t* F_out, int32_t* L_out,
                        int32_t* counts, int32_t* index, uint32_t* qcodes, uint32_t* pcodes);

/*
 * tc_annsa_attend - AnnSA (FAST-AR technical summary, section 2.C "AnnSA", pt and fr
 * pages): self-attention of the block whose cross-attention the last tc_annca_attend
 * of this handle pruned, restricted to the buckets that pruning found. Token t's bucket
 * in head h is the code of its AnnCA query there; its self-attention query sees only
 * the keys of the tokens in its own bucket:
 *   out_t = sum_{j: b(j) = b(t)} exp(scale <q_t, k_j>) v_j / sum_{same j} exp(...)
 * (never empty: t is in its own bucket). Q, K, V, out DEVICE [T, H, d] bf16 are the
 * self-attention projections of the same T tokens; out must not overlap Q, K or V.
 * The tokens are put in bucket order per head and packed; the attention runs every
 * 128-row query tile against the 128-row key tiles spanning its buckets, on tensor
 * cores with the same-bucket mask applied per element (block-sparse).
 * Asynchronous on `stream` (an ordering kernel, a packing kernel and the attention
 * kernel). Returns TC_ESTATE unless the last tc_annca_attend had Tq == T, and
 * TC_EINVAL unless 1 <= T <= 16384. Growing T past the largest earlier value
 * reallocates (and synchronises first).
 */
tc_status tc_annsa_attend(tc_annca_handle h, const void* Q, const void* K, const void* V,
                          int64_t T, void* out, tc_stream stream);

/* tc_annca_get_hyperplanes - the hash normals in use, HOST [nbits * d]. */
tc_status tc_annca_get_hyperplanes(tc_annca_handle h, float* R);

/* tc_annca_sync - synchronise the handle's last stream and return its sticky status
 * (TC_ETIMEOUT if an attention kernel gave up on one of its barriers). */
tc_status tc_annca_sync(tc_annca_handle h);

/* tc_annca_destroy - free every buffer of the handle. NULL-safe. Synchronises. */
void tc_annca_destroy(tc_annca_handle h);

/* ---- LVSA: frame-masked attention for long videos --------------------------- */

/*
 * LVSA (LVSA technical summary, section 2 "Mecanismo Central"): query frame t attends only
 * to the frames A(t) = G_s u W(t). G_s = { g : g = step (mod T_per) } are the global frames
 * of denoising step `step` (over T_per consecutive steps every frame is one exactly once);
 * W(t) grows from {t} one frame at a time, on the side with fewer frames added so far
 * (right first on a tie, the other side at the video's edge), until |G_s u W(t)| >= C or
 * it covers all T frames. Query tokens of frame t attend (bidirectionally, plain softmax,
 * bf16 tensor cores) to every token of the frames in A(t).
 */
typedef struct tc_lvsa_ctx* tc_lvsa_handle;

/* tc_lvsa_create - H heads of dimension d (64 or 128), P tokens per frame (>= 1), anchor
 * period T_per (>= 1), budget C frames (>= 1), softmax_scale 0 = 1/sqrt(d). */
tc_status tc_lvsa_create(int32_t H, int32_t d, int32_t P, int32_t T_per, int32_t C,
                         float softmax_scale, tc_lvsa_handle* out);

/* tc_lvsa_attend - Q, K, V, out DEVICE [T P, H, d] bf16 (frame f = rows f P .. f P + P - 1),
 * out not overlapping Q, K or V; step >= 0. Asynchronous on `stream` (a tile-list kernel
 * and the attention kernel). Growing T past the largest earlier value reallocates (and
 * synchronises first). TC_EINVAL unless T >= 1 and T P H < 2^31. */
tc_status tc_lvsa_attend(tc_lvsa_handle h, const void* Q, const void* K, const void* V,
                         int32_t T, int32_t step, void* out, tc_stream stream);

/* tc_lvsa_frames - inspection of the last call (HOST buffers; synchronises): *T_out its T,
 * nframes [T] = |A(t)|, frames [T*T] = A(t) ascending in frames[t*T .. t*T + nframes[t]). */
tc_status tc_lvsa_frames(tc_lvsa_handle h, int32_t* T_out, int32_t* nframes, int32_t* frames);

/* tc_lvsa_sync - synchronise the last stream; returns the sticky status (TC_ETIMEOUT if
 * the attention kernel gave up on one of its barriers). */
tc_status tc_lvsa_sync(tc_lvsa_handle h);

/* tc_lvsa_destroy - free every buffer of the handle. NULL-safe. Synchronises. */
void tc_lvsa_destroy(tc_lvsa_handle h);

#ifdef __cplusplus
}
#endif

#endif /* TEMPCACHE_H */
