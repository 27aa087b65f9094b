"""Plain fp64 CPU oracle of AnnCA cross-attention.  TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke() check and the benchmark's CPU-baseline leg
may import this module. The product path never imports or calls it, and it
shares no code with that path.

What it computes (FAST-AR technical summary, section 2.B "AnnCA"; the French page,
section 2.B, says the same): the latent queries of the current frame and the
prompt keys are projected into one shared hashed space; a prompt token is kept for
the frame when it shares a bucket with at least one query of that frame, and the
prompt tokens without such a bucket are pruned for that frame. Cross-attention
then runs over the kept prompt tokens only.

The pages give prose only; every silent point is marked READING.

 1. Hash: the sign-of-random-hyperplane code of the TempCache oracle (step 2 of
    tempcache_oracle), with the cross-attention layer's own hyperplanes R
    [nbits, d], one set shared by all heads (READING: the pages name "LSH or
    quantization" and no family).
 2. Frame: the P consecutive query tokens f*P .. f*P+P-1 of the [T, H, d] query
    block, T = F*P (READING: the block is the chunk being denoised, frame-major).
 3. Kept set of frame f, head h: prompt tokens l whose code equals the code of at
    least one query of frame f in head h (READING: one table, exact bucket, per
    head, as the heads have their own queries and keys).
 4. Attention: out_t = softmax(scale <q_t, k_l>) over the kept l, times v_l;
    scale = 1/sqrt(d), no logit shift (READING: plain cross-attention).
 5. Empty kept set: the output rows of that frame and head are zero, the sum
    over no prompt token (READING: the pages do not say).
 6. The prompt is fixed for the rollout and hashed once (READING).

Parity pins live in tests/test_annca_pins.py.
"""
from __future__ import annotations

import numpy as np

from .tempcache_oracle import biased_attention, simhash_codes


def kept_prompt_tokens(query_codes, prompt_codes) -> np.ndarray:
    """Step 3 for one head: keep[f, l] = code of prompt token l occurs among the
    codes of frame f's queries.

    query_codes [F, P], prompt_codes [L]; returns bool [F, L].
    """
    query_codes = np.asarray(query_codes, dtype=np.uint32)
    prompt_codes = np.asarray(prompt_codes, dtype=np.uint32)
    F = query_codes.shape[0]
    keep = np.zeros((F, prompt_codes.shape[0]), dtype=bool)
    for f in range(F):
        keep[f] = np.isin(prompt_codes, np.unique(query_codes[f]))
    return keep


def annca_cross_attention(Q, Kp, Vp, R, P, scale=None):
    """AnnCA cross-attention of one query block (steps 1-5).

    Q [T, H, d] with T = F*P; Kp, Vp [L, H, d] the prompt keys and values; R
    [nbits, d] the hyperplanes. Returns (out [T, H, d] fp64, keep [H, F, L] bool,
    query codes [H, T] u32, prompt codes [H, L] u32).
    """
    Q = np.asarray(Q, dtype=np.float64)
    Kp = np.asarray(Kp, dtype=np.float64)
    Vp = np.asarray(Vp, dtype=np.float64)
    T, H, d = Q.shape
    if T % P:
        raise ValueError("the query block must hold whole frames")
    F = T // P
    L = Kp.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((T, H, d), dtype=np.float64)
    keep = np.zeros((H, F, L), dtype=bool)
    qcodes = np.zeros((H, T), dtype=np.uint32)
    pcodes = np.zeros((H, L), dtype=np.uint32)
    for h in range(H):
        qcodes[h] = simhash_codes(R, Q[:, h, :])
        pcodes[h] = simhash_codes(R, Kp[:, h, :])
        keep[h] = kept_prompt_tokens(qcodes[h].reshape(F, P), pcodes[h])
        for f in range(F):
            rows = slice(f * P, (f + 1) * P)
            sel = np.nonzero(keep[h, f])[0]
            if sel.size == 0:
                continue   # step 5: zero rows
            out[rows, h, :] = biased_attention(Q[rows, h, :], Kp[sel, h, :], Vp[sel, h, :],
                                               np.zeros(sel.size), scale)
    return out, keep, qcodes, pcodes
