"""Plain fp64 CPU oracle of AnnSA self-attention.  TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke() check and the benchmark's CPU-baseline leg
may import this module. The product path never imports or calls it, and it
shares no code with that path.

What it computes (FAST-AR technical summary, section 2.C "AnnSA"; the French page,
section 2.C, says the same): the semantic buckets found while pruning the
cross-attention are reused, and the self-attention query of every token only
attends to the keys of tokens in its own bucket, which turns the quadratic
self-attention into a block-sparse one.

The pages give prose only; every silent point is marked READING.

 1. Bucket of a token: its AnnCA query code in the same head (annca_oracle, step 1),
    i.e. the bucket the cross-attention pruning put it in (READING: "reusing the
    buckets"; heads keep their own buckets).
 2. Tokens: the T tokens of the query block whose buckets were found, attending to
    each other (READING: the block's own self-attention; the pages say nothing about
    a cache here).
 3. out_t = softmax(scale <q_t, k_j>) over the tokens j with bucket(j) = bucket(t),
    times v_j; scale = 1/sqrt(d). A token is in its own bucket, so the set is never
    empty (READING: exact same-bucket mask; block-sparse is how it is computed).

Parity pins live in tests/test_annsa_pins.py.
"""
from __future__ import annotations

import numpy as np

from .tempcache_oracle import biased_attention


def same_bucket_groups(buckets) -> list:
    """Step 3's key sets for one head: the token indices of every bucket, ascending."""
    buckets = np.asarray(buckets)
    return [np.nonzero(buckets == c)[0] for c in np.unique(buckets)]


def annsa_attention(Q, K, V, buckets, scale=None) -> np.ndarray:
    """AnnSA self-attention of one block. Q, K, V [T, H, d]; buckets [H, T] (the AnnCA
    query codes of the block). Returns out [T, H, d] in fp64."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    T, H, d = Q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((T, H, d), dtype=np.float64)
    for h in range(H):
        for g in same_bucket_groups(buckets[h]):
            out[g, h, :] = biased_attention(Q[g, h, :], K[g, h, :], V[g, h, :], np.zeros(g.size), scale)
    return out
