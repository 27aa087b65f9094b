"""Plain fp64 CPU oracle of the TempCache step.  TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke() check and the benchmark's CPU-baseline leg
may import this module. The product path (the CUDA library and its Python
binding) never imports or calls it, and it shares no code with that path.

What it computes (FAST-AR technical summary, section 2.A "TempCache"; the same
passage appears on the French page, section 2.A): each new key of the current
chunk is hashed with locality-sensitive hashing, its top-1 nearest neighbour among
the earlier cache entries is found, near-duplicates are merged under a similarity
threshold with their values averaged, and attention then shifts each merged
logit by the group size, which Lemma 5.1 states is exact for identical keys.

The pages give prose only. Every step below is the plainest reading of it; each
silent point is marked READING.

 1. Hyperplanes R [nbits, d]: an input (the caller draws them).
 2. Code of a key k: bit b = 1 iff <R_b, k> >= 0 (READING: zero maps to 1);
    code = sum_b bit_b * 2^b. Dots are fp64 sums taken in index order 0..d-1.
 3. Candidates of a new key: the entries committed before this commit whose code
    equals the key's code (READING: one hash table, exact bucket, snapshot).
 4. Similarity: cosine dot / sqrt(|k|^2 |e|^2) with the three sums as in 2,
    then one fp64 multiply, square root and divide; a zero-norm side gives 0.
    The entry's key is the first key that created it and never changes (READING).
 5. Top-1: largest similarity; exact ties go to the lowest entry index (READING).
 6. Merge iff sim >= tau, with tau the fp32 threshold widened to fp64 (READING).
 7. Merge: entry j with matched tokens S_j gets v <- (n v + sum_{t in S_j} v_t)
    / (n + |S_j|), n <- n + |S_j| (Lemma 5.1: values averaged). Several tokens may
    merge into one entry (READING).
 8. Append: unmatched tokens become new entries in ascending t with n = 1. Tokens
    of one chunk are not matched against each other (READING: snapshot). If any
    head would exceed its capacity the whole commit is refused and nothing
    changes (READING: the pages give no eviction policy).
 9. Deferred commit (READING): the chunk passed to append_chunk(c) is committed at
    the next append_chunk or at flush(); until then attention sees it raw.
8b. Variant (option intra_chunk; the open point of 8 read the other way): the
    tokens of a commit are taken in ascending t and the candidates of token t
    also include the entries created by earlier tokens of the same commit (same
    code). A token that merges into such an entry joins its group: the entry's
    value is the mean of its creating token and every later member, n their
    count. Committed entries precede new ones in index order, so exact ties
    still go to the lowest entry index.
8c. Variant (option key_mode="mean"; the other half of the open point of 4): an
    entry's key is the running mean of its members' keys, kept in fp32 the way a
    device merge keeps means: k <- (n k + sum_{t in S} k_t) / (n + m), the sum taken
    in fp32 in ascending t and every operation rounded to fp32 (READING). After the
    commit the entry's code is recomputed from its new key (step 2) and it moves to
    that bucket for later commits; matches inside one commit still see the keys as
    they were before it (snapshot). Attention uses the mean key. Identical keys give
    a mean equal to each of them exactly (bf16 keys, counts below 2^16), so Lemma
    5.1's case is unchanged.
10. Attention: out_t = sum_j w_tj v_j / sum_j w_tj with
    w_tj = exp(scale <q_t, k_j> + b_j - max), b_j = ln n_j for committed entries
    and 0 for staged tokens, scale = 1/sqrt(d), no mask (READING: the logit shift
    "by the group size" is + ln n, the only shift that makes Lemma 5.1 exact).

Parity pins live in tests/test_oracle_pins.py. The hash (2) and the threshold
(6) follow the reading above; the pages fix no hash family or threshold, so
their agreement with the paper itself is "parity unpinned" beyond the textbook
SimHash collision law and the special cases tested there.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


class CapacityExceeded(RuntimeError):
    """A commit would push some head past its capacity; nothing was changed."""


# ----------------------------------------------------------------------------- step 2, 4

def seq_dot(A, B) -> np.ndarray:
    """Row-wise dot products accumulated in fp64 in index order i = 0 .. d-1.

    A and B broadcast against each other over their leading axes; the last axis
    is the one summed. The inputs of this method are bf16 or fp32 values, whose
    pairwise products are exact in fp64, so only the additions round.
    """
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    shape = np.broadcast_shapes(A.shape[:-1], B.shape[:-1])
    s = np.zeros(shape, dtype=np.float64)
    for i in range(A.shape[-1]):
        s = s + A[..., i] * B[..., i]
    return s


def simhash_codes(R, X) -> np.ndarray:
    """Sign-of-random-hyperplane code of each row of X [N, d] (step 2).

    FAST-AR summary, section 2.A: the nearest neighbour is found with
    locality-sensitive hashing. Bit b is set iff <R_b, x> >= 0.
    """
    R = np.asarray(R, dtype=np.float64)
    X = np.asarray(X, dtype=np.float64)
    nbits = R.shape[0]
    proj = seq_dot(X[:, None, :], R[None, :, :])          # [N, nbits]
    bits = (proj >= 0.0).astype(np.uint64)
    weights = np.left_shift(np.uint64(1), np.arange(nbits, dtype=np.uint64))
    return (bits * weights).sum(axis=1).astype(np.uint32)


def cosine_similarity(A, B) -> np.ndarray:
    """Row-wise cosine of A and B (step 4); 0 where either row has zero norm."""
    dot = seq_dot(A, B)
    na = seq_dot(A, A)
    nb = seq_dot(B, B)
    out = np.zeros(dot.shape, dtype=np.float64)
    ok = (na > 0.0) & (nb > 0.0)
    out[ok] = dot[ok] / np.sqrt(na[ok] * nb[ok])
    return out


# ----------------------------------------------------------------------------- step 3, 5, 6

def top1_in_bucket(keys, codes, cache_keys, cache_codes):
    """Top-1 cosine neighbour of every new key among the same-code cache entries.

    Returns (best [T] int64, best_sim [T] fp64); best = -1 and best_sim = -inf
    where the bucket is empty. Exact ties resolve to the lowest entry index.
    """
    keys = np.asarray(keys, dtype=np.float64)
    codes = np.asarray(codes, dtype=np.uint32)
    cache_keys = np.asarray(cache_keys, dtype=np.float64)
    cache_codes = np.asarray(cache_codes, dtype=np.uint32)
    T = keys.shape[0]
    best = np.full(T, -1, dtype=np.int64)
    best_sim = np.full(T, -np.inf, dtype=np.float64)
    if T == 0 or cache_keys.shape[0] == 0:
        return best, best_sim
    order = np.argsort(cache_codes, kind="stable")
    sorted_codes = cache_codes[order]
    lo = np.searchsorted(sorted_codes, codes, side="left")
    hi = np.searchsorted(sorted_codes, codes, side="right")
    count = hi - lo
    if count.sum() == 0:
        return best, best_sim
    token = np.repeat(np.arange(T), count)
    # position of each (token, candidate) pair inside its bucket range
    starts = np.repeat(lo, count)
    offset = np.arange(token.size) - np.repeat(np.cumsum(count) - count, count)
    entry = order[starts + offset]
    sims = cosine_similarity(keys[token], cache_keys[entry])
    # sort pairs by token, then similarity descending, then entry ascending
    perm = np.lexsort((entry, -sims, token))
    token_sorted = token[perm]
    first = np.ones(perm.size, dtype=bool)
    first[1:] = token_sorted[1:] != token_sorted[:-1]
    winners = perm[first]
    best[token[winners]] = entry[winners]
    best_sim[token[winners]] = sims[winners]
    return best, best_sim


def new_entry_members(u, match_row, e) -> np.ndarray:
    """Tokens of an entry created inside a commit (step 8b): its creating token u
    and every later token whose match is the new entry e, in ascending t."""
    return np.concatenate([[u], np.nonzero(np.asarray(match_row) == e)[0]]).astype(np.int64)


def mean_key_fp32(key, n, members) -> np.ndarray:
    """Step 8c: (n key + sum of members' keys) / (n + m), the member sum taken in
    ascending order in fp32 and every operation rounded to fp32; returned as fp64
    holding the fp32 values."""
    acc = np.zeros(np.asarray(key).shape, dtype=np.float32)
    for row in np.asarray(members):
        acc = (acc + np.asarray(row, dtype=np.float32)).astype(np.float32)
    num = (np.float32(n) * np.asarray(key, dtype=np.float32)).astype(np.float32)
    num = (num + acc).astype(np.float32)
    return (num / np.float32(n + len(members))).astype(np.float32).astype(np.float64)


def merge_decision(best, best_sim, tau) -> np.ndarray:
    """match = best where sim >= tau (tau as fp32 widened to fp64), else -1."""
    tau64 = np.float64(np.float32(tau))
    best = np.asarray(best, dtype=np.int64)
    return np.where((best >= 0) & (np.asarray(best_sim) >= tau64), best, -1)


# ----------------------------------------------------------------------------- step 10

def biased_attention(Q, K, V, bias, scale) -> np.ndarray:
    """softmax(scale * Q K^T + bias) V for one head, in fp64.

    Q [Tq, d], K [L, d], V [L, d], bias [L]. Lemma 5.1 (FAST-AR summary, 2.A):
    an entry standing for n identical keys enters with logit shift ln n.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    logits = scale * (Q @ K.T) + np.asarray(bias, dtype=np.float64)[None, :]
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    return (w @ V) / w.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------- state

@dataclass
class HeadState:
    d: int
    keys: np.ndarray = None      # [M, d] representative keys (exact input values)
    values: np.ndarray = None    # [M, d] fp64 running means
    counts: np.ndarray = None    # [M] int64 group sizes n
    codes: np.ndarray = None     # [M] uint32

    def __post_init__(self):
        self.keys = np.zeros((0, self.d))
        self.values = np.zeros((0, self.d))
        self.counts = np.zeros(0, dtype=np.int64)
        self.codes = np.zeros(0, dtype=np.uint32)

    @property
    def size(self) -> int:
        return int(self.counts.shape[0])


@dataclass
class CommitRecord:
    codes: np.ndarray   # [H, T] uint32 codes of the committed chunk
    match: np.ndarray   # [H, T] int64 merge target or -1
    dest: np.ndarray    # [H, T] int64 entry each token ends up in
    sizes: np.ndarray = field(default=None)  # [H] cache sizes after the commit


class OracleTempCache:
    """The TempCache state machine with the library's verbs, in fp64 on the CPU.

    K, V, Q are [T, H, d] arrays of the exact values the GPU sees (bf16 or fp32
    values widened to fp64).
    """

    def __init__(self, H, d, nbits, tau, capacity, hyperplanes, scale=None, intra_chunk=False,
                 key_mode="representative"):
        self.intra_chunk = bool(intra_chunk)
        if key_mode not in ("representative", "mean"):
            raise ValueError("key_mode is 'representative' or 'mean'")
        if key_mode == "mean" and self.intra_chunk:
            raise NotImplementedError("running-mean keys are defined for the snapshot commit")
        self.key_mode = key_mode
        self.H, self.d, self.nbits = int(H), int(d), int(nbits)
        self.tau = float(tau)
        self.capacity = int(capacity)
        self.R = np.asarray(hyperplanes, dtype=np.float64).reshape(self.nbits, self.d)
        self.scale = (1.0 / np.sqrt(self.d)) if scale is None else float(scale)
        self.heads = [HeadState(self.d) for _ in range(self.H)]
        self.staged = None   # (K [H,T,d], V [H,T,d], codes [H,T])
        self.committed_tokens = 0

    # -- staging (step 2 happens when a chunk arrives) --------------------------
    def _stage(self, K, V):
        K = np.asarray(K, dtype=np.float64).transpose(1, 0, 2).copy()   # [H,T,d]
        V = np.asarray(V, dtype=np.float64).transpose(1, 0, 2).copy()
        codes = np.stack([simhash_codes(self.R, K[h]) for h in range(self.H)])
        self.staged = (K, V, codes)

    # -- commit (steps 3-8) -----------------------------------------------------
    def _commit(self) -> CommitRecord | None:
        if self.staged is None:
            return None
        if self.intra_chunk:
            return self._commit_intra()
        K, V, codes = self.staged
        T = K.shape[1]
        match = np.full((self.H, T), -1, dtype=np.int64)
        for h, st in enumerate(self.heads):
            best, sim = top1_in_bucket(K[h], codes[h], st.keys, st.codes)
            match[h] = merge_decision(best, sim, self.tau)
        unmatched = match < 0
        new_sizes = np.array([st.size for st in self.heads]) + unmatched.sum(axis=1)
        if np.any(new_sizes > self.capacity):
            raise CapacityExceeded(f"commit needs {int(new_sizes.max())} entries, capacity {self.capacity}")
        dest = match.copy()
        for h, st in enumerate(self.heads):
            # step 7: merges, values averaged with the old group
            targets = np.unique(match[h][match[h] >= 0])
            for j in targets:
                grp = np.nonzero(match[h] == j)[0]
                n_old = st.counts[j]
                total = n_old * st.values[j] + V[h, grp].sum(axis=0)
                st.counts[j] = n_old + grp.size
                st.values[j] = total / st.counts[j]
                if self.key_mode == "mean":   # step 8c
                    st.keys[j] = mean_key_fp32(st.keys[j], n_old, K[h, grp])
                    st.codes[j] = simhash_codes(self.R, st.keys[j][None, :])[0]
            # step 8: append unmatched tokens in ascending t
            new = np.nonzero(unmatched[h])[0]
            dest[h, new] = st.size + np.arange(new.size)
            st.keys = np.concatenate([st.keys, K[h, new]])
            st.values = np.concatenate([st.values, V[h, new]])
            st.counts = np.concatenate([st.counts, np.ones(new.size, dtype=np.int64)])
            st.codes = np.concatenate([st.codes, codes[h, new]])
        self.committed_tokens += T
        self.staged = None
        return CommitRecord(codes=codes.copy(), match=match, dest=dest, sizes=self.cache_size())

    def _commit_intra(self) -> CommitRecord:
        """Step 8b: tokens in ascending t, candidates = committed entries of the
        token's code (snapshot, as in 3) plus the entries created earlier in this
        commit with the same code; ties to the lowest entry index."""
        K, V, codes = self.staged
        T = K.shape[1]
        tau64 = np.float64(np.float32(self.tau))
        match = np.full((self.H, T), -1, dtype=np.int64)
        created = []
        for h, st in enumerate(self.heads):
            best, sim = top1_in_bucket(K[h], codes[h], st.keys, st.codes)
            M0 = st.size
            new_of_code = {}     # code -> [(entry index, creating token)] in creation order
            made = []
            for t in range(T):
                bj, bs = int(best[t]), float(sim[t])
                for e, u in new_of_code.get(int(codes[h, t]), []):
                    s_ = float(cosine_similarity(K[h, t][None, :], K[h, u][None, :])[0])
                    if s_ > bs:
                        bj, bs = e, s_
                if bj >= 0 and bs >= tau64:
                    match[h, t] = bj
                else:
                    e = M0 + len(made)
                    made.append(t)
                    new_of_code.setdefault(int(codes[h, t]), []).append((e, t))
            created.append(made)
        new_sizes = np.array([st.size + len(c) for st, c in zip(self.heads, created)])
        if np.any(new_sizes > self.capacity):
            raise CapacityExceeded(f"commit needs {int(new_sizes.max())} entries, capacity {self.capacity}")
        dest = match.copy()
        for h, st in enumerate(self.heads):
            M0 = st.size
            made = created[h]
            dest[h, made] = M0 + np.arange(len(made))
            # committed targets: step 7
            for j in np.unique(match[h][(match[h] >= 0) & (match[h] < M0)]):
                grp = np.nonzero(match[h] == j)[0]
                n_old = st.counts[j]
                total = n_old * st.values[j] + V[h, grp].sum(axis=0)
                st.counts[j] = n_old + grp.size
                st.values[j] = total / st.counts[j]
            # new entries: creating token plus later members
            keys = np.zeros((len(made), self.d))
            vals = np.zeros((len(made), self.d))
            cnts = np.zeros(len(made), dtype=np.int64)
            for k, u in enumerate(made):
                members = new_entry_members(u, match[h], M0 + k)
                keys[k] = K[h, u]
                vals[k] = V[h, members].sum(axis=0) / members.size
                cnts[k] = members.size
            st.keys = np.concatenate([st.keys, keys])
            st.values = np.concatenate([st.values, vals])
            st.counts = np.concatenate([st.counts, cnts])
            st.codes = np.concatenate([st.codes, codes[h, made].astype(np.uint32)])
        self.committed_tokens += T
        self.staged = None
        return CommitRecord(codes=codes.copy(), match=match, dest=dest, sizes=self.cache_size())

    # -- public verbs -----------------------------------------------------------
    def append_chunk(self, K, V) -> CommitRecord | None:
        """Commit the staged chunk (if any), then stage (K, V) [T, H, d]."""
        rec = self._commit()
        self._stage(K, V)
        return rec

    def flush(self) -> CommitRecord | None:
        return self._commit()

    def cache_size(self) -> np.ndarray:
        return np.array([st.size for st in self.heads], dtype=np.int64)

    def _head_kv(self, h):
        st = self.heads[h]
        keys, values = st.keys, st.values
        bias = np.log(st.counts.astype(np.float64))
        if self.staged is not None:
            K, V, _ = self.staged
            keys = np.concatenate([keys, K[h]])
            values = np.concatenate([values, V[h]])
            bias = np.concatenate([bias, np.zeros(K.shape[1])])
        return keys, values, bias

    def attend(self, Q, rows=None) -> np.ndarray:
        """Biased attention of Q [Tq, H, d] over committed entries + staged chunk.

        With `rows` given, only those query rows are computed; the result is then
        [len(rows), H, d].
        """
        if self.committed_tokens == 0 and self.staged is None:
            raise RuntimeError("attend before any chunk was appended")
        Q = np.asarray(Q, dtype=np.float64)
        if rows is not None:
            Q = Q[np.asarray(rows)]
        out = np.zeros(Q.shape, dtype=np.float64)
        for h in range(self.H):
            keys, values, bias = self._head_kv(h)
            out[:, h] = biased_attention(Q[:, h], keys, values, bias, self.scale)
        return out

    def export_head(self, h):
        st = self.heads[h]
        return st.keys.copy(), st.values.copy(), st.counts.copy(), st.codes.copy()
