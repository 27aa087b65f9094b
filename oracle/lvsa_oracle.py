"""Plain fp64 CPU oracle of the LVSA frame mask.  TEST INFRASTRUCTURE ONLY.

Only the tests, the package's smoke() check and the benchmark's CPU-baseline leg
may import this module. The product path never imports or calls it, and it
shares no code with that path.

What it computes (LVSA technical summary, section 2 "Metodologia: Long Video Sparse
Attention", "Mecanismo Central"): a query frame t attends only to the frames
A(t) = G u W(t) instead of all T frames, where
  * G is a set of periodic global frames that, at denoising step s, is shifted by
    s mod T_per, so that over T_per consecutive steps every frame is a global
    anchor exactly once, and
  * W(t) is a local window around t that is extended when it overlaps global
    frames, so that every query frame attends to about C frames (the budget).

The pages give prose only; every silent point is marked READING.

 1. G_s = { g in [0, T) : g = s (mod T_per) } (READING: one anchor every T_per frames,
    the grid offset by s mod T_per).
 2. W(t) grows from {t} one frame at a time, on the side with fewer frames added so
    far (right first on a tie; the other side when one side reaches the video's
    edge), until |G_s u W(t)| >= C or it covers all T frames (READING: "a local
    window extended to compensate the overlap so that |A(t)| ~ C": the smallest such
    window, centred on t where the edges allow; with no overlap this is the centred
    window of C - |G_s| frames).
 3. A(t) = G_s u W(t); so |A(t)| = C whenever |G_s u {t}| <= C <= T.
 4. Attention: query tokens of frame t attend to every token of the frames in A(t)
    (bidirectional), softmax(scale <q, k>) v, scale = 1/sqrt(d); a frame is P
    consecutive tokens of the [T P, H, d] sequence (READING).

Parity pins live in tests/test_lvsa_pins.py.
"""
from __future__ import annotations

import numpy as np

from .tempcache_oracle import biased_attention


def global_frames(T, T_per, s) -> np.ndarray:
    """Step 1: the rotating global anchors G_s, ascending."""
    return np.array([g for g in range(T) if g % T_per == s % T_per], dtype=np.int64)


def local_window(T, t, G, C):
    """Step 2: (lo, hi) with W(t) = [lo, hi], grown from {t} until |G u W| >= C."""
    Gs = set(int(g) for g in G)
    lo = hi = t
    left = right = 0

    def size():
        return len(Gs | set(range(lo, hi + 1)))

    while size() < C and (lo > 0 or hi < T - 1):
        if hi < T - 1 and (right <= left or lo == 0):
            hi += 1
            right += 1
        else:
            lo -= 1
            left += 1
    return lo, hi


def attended_frames(T, T_per, C, s) -> list:
    """Step 3: A(t) for every query frame t, as sorted arrays."""
    G = global_frames(T, T_per, s)
    out = []
    for t in range(T):
        lo, hi = local_window(T, t, G, C)
        out.append(np.array(sorted(set(G.tolist()) | set(range(lo, hi + 1))), dtype=np.int64))
    return out


def lvsa_attention(Q, K, V, P, T_per, C, s, scale=None) -> np.ndarray:
    """Step 4: Q, K, V [T P, H, d] -> out [T P, H, d] in fp64."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    N, H, d = Q.shape
    if N % P:
        raise ValueError("the sequence must hold whole frames")
    T = N // P
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    A = attended_frames(T, T_per, C, s)
    out = np.zeros((N, H, d), dtype=np.float64)
    for t in range(T):
        keys = np.concatenate([np.arange(f * P, (f + 1) * P) for f in A[t]])
        rows = slice(t * P, (t + 1) * P)
        for h in range(H):
            out[rows, h] = biased_attention(Q[rows, h], K[keys, h], V[keys, h], np.zeros(keys.size), scale)
    return out
