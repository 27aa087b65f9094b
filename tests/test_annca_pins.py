"""Pins of the AnnCA oracle against facts fixed outside the oracle itself.

FAST-AR summary, section 2.B "AnnCA": a prompt token is kept for a frame when it
shares a hash bucket with at least one query of that frame; the others are pruned
for that frame, and cross-attention runs over the kept tokens. The pins:
  * the kept sets recomputed by brute force with exact integer arithmetic on
    integer-valued vectors (Python ints, no numpy, no oracle code);
  * when every prompt token is kept, the output is textbook softmax attention
    (torch's own routine, fp64);
  * hyperplanes equal to coordinate axes make the code the sign pattern of a
    vector, so the kept sets of hand-built frames are known in advance, and the
    output of each frame is textbook attention over exactly those tokens;
  * a frame whose every query is the negation of every prompt key shares no
    bucket with the prompt (every bit flips) and gets zero rows;
  * positive scaling of the queries changes no code, hence no kept set.
The last section plants mistakes in the oracle and checks that a pin catches each.
"""
import numpy as np
import pytest
import torch

import oracle.annca_oracle as ann
from synthetic import CROSS_CONFIGS, CrossWorkload


def f64(x):
    return x.to(torch.float64).cpu().numpy()


def sdpa(Q, K, V, scale):
    """Textbook softmax attention of one head by torch's routine: Q [n,d], K/V [m,d]."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(np.ascontiguousarray(Q))[None, None], torch.from_numpy(np.ascontiguousarray(K))[None, None],
        torch.from_numpy(np.ascontiguousarray(V))[None, None], scale=scale)
    return out[0, 0].numpy()


# ----------------------------------------------------------------------------- pins

def pin_brute_force_kept_sets(mod):
    rng = np.random.default_rng(5)
    H, d, P, F, L, nbits = 2, 6, 5, 3, 9, 3
    R = rng.integers(-3, 4, size=(nbits, d))
    Q = rng.integers(-2, 3, size=(F * P, H, d))
    Kp = rng.integers(-2, 3, size=(L, H, d))
    # one query lies exactly on a hyperplane (zero projection counts as bit 1)
    Q[0, 0] = 0
    Q[0, 0, 0], Q[0, 0, 1] = R[0, 1], -R[0, 0]
    Q[0, 0, 2:] = 0
    Vp = rng.standard_normal((L, H, d))

    def code(x):
        c = 0
        for b in range(nbits):
            s = sum(int(R[b][i]) * int(x[i]) for i in range(d))
            if s >= 0:
                c |= 1 << b
        return c

    _, keep, qc, pc = mod.annca_cross_attention(Q.astype(float), Kp.astype(float), Vp, R.astype(float), P)
    for h in range(H):
        for f in range(F):
            frame_codes = {code(Q[f * P + p, h]) for p in range(P)}
            for l in range(L):
                assert bool(keep[h, f, l]) == (code(Kp[l, h]) in frame_codes), (h, f, l)
        assert [int(c) for c in qc[h]] == [code(Q[t, h]) for t in range(F * P)]
        assert [int(c) for c in pc[h]] == [code(Kp[l, h]) for l in range(L)]


def pin_all_kept_is_dense_attention(mod):
    rng = np.random.default_rng(6)
    H, d, L, F, nbits = 2, 16, 7, 2, 5
    P = L + 4
    R = rng.standard_normal((nbits, d))
    Kp = rng.standard_normal((L, H, d))
    Vp = rng.standard_normal((L, H, d))
    Q = rng.standard_normal((F * P, H, d))
    for f in range(F):   # every frame holds a positive multiple of every prompt key
        Q[f * P: f * P + L] = Kp * (1.5 + f)
    out, keep, _, _ = mod.annca_cross_attention(Q, Kp, Vp, R, P)
    assert keep.all()
    for h in range(H):
        np.testing.assert_allclose(out[:, h], sdpa(Q[:, h], Kp[:, h], Vp[:, h], 1 / np.sqrt(d)), rtol=0, atol=1e-12)


def axis_case():
    """Hyperplanes = coordinate axes 0..3 of d = 8: the code is the sign pattern of
    the first four coordinates. Prompt tokens carry the patterns A, B, C; frame 0
    shows A only, frame 1 shows B and C, frame 2 shows a fourth pattern D."""
    d, nbits, H, P = 8, 4, 1, 6
    R = np.zeros((nbits, d))
    R[np.arange(nbits), np.arange(nbits)] = 1.0
    sign = {"A": [1, 1, -1, -1], "B": [-1, 1, 1, -1], "C": [1, -1, 1, 1], "D": [-1, -1, -1, 1]}
    rng = np.random.default_rng(7)

    def vec(p):
        v = rng.uniform(0.5, 2.0, d) * np.array(sign[p] + [1] * 4)
        v[4:] = rng.standard_normal(4)
        return v

    kinds = ["A", "B", "C", "A", "C", "B", "A", "C"]
    Kp = np.stack([vec(k) for k in kinds])[:, None, :]
    Vp = rng.standard_normal((len(kinds), H, d))
    frames = [["A"] * 6, ["B", "C", "B", "C", "C", "B"], ["D"] * 6]
    Q = np.stack([vec(k) for fr in frames for k in fr])[:, None, :]
    expect = np.array([[k == "A" for k in kinds], [k in ("B", "C") for k in kinds], [False] * len(kinds)])
    return Q, Kp, Vp, R, P, expect


def pin_frames_pruned_independently(mod):
    Q, Kp, Vp, R, P, expect = axis_case()
    out, keep, _, _ = mod.annca_cross_attention(Q, Kp, Vp, R, P)
    np.testing.assert_array_equal(keep[0], expect)
    d = Q.shape[-1]
    for f in range(2):
        sel = np.nonzero(expect[f])[0]
        rows = slice(f * P, (f + 1) * P)
        np.testing.assert_allclose(out[rows, 0], sdpa(Q[rows, 0], Kp[sel, 0], Vp[sel, 0], 1 / np.sqrt(d)),
                                   rtol=0, atol=1e-12)
    np.testing.assert_array_equal(out[2 * P:, 0], 0.0)


def pin_negated_queries_share_no_bucket(mod):
    rng = np.random.default_rng(8)
    H, d, L, P, nbits = 1, 12, 5, 4, 6
    R = rng.standard_normal((nbits, d))
    k = rng.standard_normal(d)
    Kp = np.stack([k * s for s in (1.0, 0.5, 2.0, 3.0, 0.25)])[:, None, :]
    Vp = rng.standard_normal((L, H, d))
    Q = np.concatenate([np.tile(k, (P, 1)), np.tile(-k, (P, 1))])[:, None, :]
    out, keep, _, _ = mod.annca_cross_attention(Q, Kp, Vp, R, P)
    assert keep[0, 0].all() and not keep[0, 1].any()
    np.testing.assert_array_equal(out[P:], 0.0)
    np.testing.assert_allclose(out[:P, 0], sdpa(Q[:P, 0], Kp[:, 0], Vp[:, 0], 1 / np.sqrt(d)), rtol=0, atol=1e-12)


def pin_positive_scaling(mod):
    cfg = CROSS_CONFIGS["annca-tiny"]
    w = CrossWorkload(cfg)
    Kp, Vp = w.prompt()
    Q = f64(w.queries(0))
    R = f64(w.hyperplanes())
    _, keep1, qc1, _ = mod.annca_cross_attention(Q, f64(Kp), f64(Vp), R, cfg.P)
    _, keep2, qc2, _ = mod.annca_cross_attention(Q * 4.0, f64(Kp), f64(Vp), R, cfg.P)
    np.testing.assert_array_equal(qc1, qc2)
    np.testing.assert_array_equal(keep1, keep2)
    assert 0 < keep1.sum() < keep1.size   # the synthetic prompt is pruned, but not away


PINS = [pin_brute_force_kept_sets, pin_all_kept_is_dense_attention, pin_frames_pruned_independently,
        pin_negated_queries_share_no_bucket, pin_positive_scaling]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_annca_oracle_pin(pin):
    pin(ann)


# ----------------------------------------------------------------------------- planted mistakes

class Planted:
    """The oracle module with one function replaced."""

    def __init__(self, **repl):
        self.repl = repl

    def __enter__(self):
        self.saved = {k: getattr(ann, k) for k in self.repl}
        for k, v in self.repl.items():
            setattr(ann, k, v)
        return ann

    def __exit__(self, *a):
        for k, v in self.saved.items():
            setattr(ann, k, v)


def _kept_over_whole_block(qcodes, pcodes):
    keep = np.isin(np.asarray(pcodes), np.unique(qcodes))
    return np.tile(keep, (np.asarray(qcodes).shape[0], 1))


def _kept_frames_reversed(qcodes, pcodes):
    return np.stack([np.isin(pcodes, np.unique(q)) for q in np.asarray(qcodes)[::-1]])


def _kept_strict_sign(qcodes, pcodes):
    return np.stack([np.isin(pcodes, np.unique(q) ^ 1) for q in np.asarray(qcodes)])


@pytest.mark.parametrize("mistake,pin", [
    (_kept_over_whole_block, pin_frames_pruned_independently),
    (_kept_frames_reversed, pin_frames_pruned_independently),
    (_kept_strict_sign, pin_brute_force_kept_sets),
])
def test_planted_kept_set_mistake_is_caught(mistake, pin):
    with Planted(kept_prompt_tokens=mistake) as mod:
        with pytest.raises(AssertionError):
            pin(mod)


def test_planted_fallback_on_empty_frame_is_caught():
    real = ann.biased_attention

    def attention_over_everything_when_empty(Qf, K, V, bias, scale):
        return real(Qf, K, V, bias, scale)

    def annca_dense_when_empty(Q, Kp, Vp, R, P, scale=None):
        out, keep, qc, pc = ANNCA(Q, Kp, Vp, R, P, scale)
        T, H, d = Q.shape
        for h in range(H):
            for f in range(T // P):
                if not keep[h, f].any():   # the mistake: fall back to the whole prompt
                    rows = slice(f * P, (f + 1) * P)
                    out[rows, h] = attention_over_everything_when_empty(
                        Q[rows, h], Kp[:, h], Vp[:, h], np.zeros(Kp.shape[0]), 1 / np.sqrt(d))
        return out, keep, qc, pc

    with Planted(annca_cross_attention=annca_dense_when_empty) as mod:
        with pytest.raises(AssertionError):
            pin_negated_queries_share_no_bucket(mod)


ANNCA = ann.annca_cross_attention
