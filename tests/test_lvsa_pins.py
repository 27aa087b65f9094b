"""Pins of the LVSA frame-mask oracle against facts fixed outside the oracle itself.

LVSA technical summary, section 2 "Mecanismo Central": A(t) = G u W(t); the global
frames rotate with the denoising step so that over T_per consecutive steps every frame
is an anchor exactly once; the local window is extended over anchors so that every
query frame attends to about C frames. The pins:
  * the rotation property, counted over T_per consecutive steps (the page's own claim);
  * the budget: |A(t)| = C whenever |G u {t}| <= C <= T;
  * A(t) holds t and every anchor, and W(t) is one interval around t, minimal: either
    end frame removed (if it is neither t nor an anchor) leaves fewer than C frames;
  * C >= T: every frame sees every frame, so the output is textbook attention (torch);
  * the output equals torch's masked attention with a token mask built by a plain
    double loop over the frame sets.
The last section plants mistakes in the oracle and checks that a pin catches each.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle.lvsa_oracle as lv

CASES = [(T, T_per, C) for T in (1, 5, 12, 29) for T_per in (1, 3, 7) for C in (1, 4, 9, 40)]


def sdpa(Q, K, V, scale, mask=None):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]  # noqa: E731
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), attn_mask=m, scale=scale)[0, 0].numpy()


def pin_rotation(mod):
    for T, T_per, _ in CASES:
        for s0 in (0, 5):
            seen = np.zeros(T, int)
            for s in range(s0, s0 + T_per):
                for g in mod.global_frames(T, T_per, s):
                    seen[g] += 1
            assert (seen == 1).all(), (T, T_per, s0, seen)


def pin_budget_and_shape(mod):
    for T, T_per, C in CASES:
        for s in range(T_per):
            G = set(mod.global_frames(T, T_per, s).tolist())
            A = mod.attended_frames(T, T_per, C, s)
            for t in range(T):
                a = set(A[t].tolist())
                assert t in a and G <= a
                lo, hi = mod.local_window(T, t, sorted(G), C)
                assert lo <= t <= hi and a == G | set(range(lo, hi + 1))
                if len(G | {t}) <= C <= T:
                    assert len(a) == C, (T, T_per, C, s, t, len(a))
                    for end in (lo, hi):   # minimal: dropping an end frame loses the budget
                        if end != t and end not in G:
                            assert len(a - {end}) < C


def pin_whole_budget_is_dense(mod):
    rng = np.random.default_rng(1)
    T, P, H, d = 5, 3, 2, 8
    Q, K, V = (rng.standard_normal((T * P, H, d)) for _ in range(3))
    out = mod.lvsa_attention(Q, K, V, P, T_per=2, C=T, s=1)
    for h in range(H):
        np.testing.assert_allclose(out[:, h], sdpa(Q[:, h], K[:, h], V[:, h], 1 / np.sqrt(d)), rtol=0, atol=1e-12)


def pin_brute_force_mask(mod):
    rng = np.random.default_rng(2)
    T, P, H, d, T_per, C = 11, 3, 2, 8, 4, 5
    Q, K, V = (rng.standard_normal((T * P, H, d)) for _ in range(3))
    for s in range(T_per):
        out = mod.lvsa_attention(Q, K, V, P, T_per, C, s)
        A = mod.attended_frames(T, T_per, C, s)
        mask = np.zeros((T * P, T * P), bool)
        for i, j in itertools.product(range(T * P), range(T * P)):
            mask[i, j] = (j // P) in set(A[i // P].tolist())
        for h in range(H):
            np.testing.assert_allclose(out[:, h], sdpa(Q[:, h], K[:, h], V[:, h], 1 / np.sqrt(d), mask),
                                       rtol=0, atol=1e-12)


PINS = [pin_rotation, pin_budget_and_shape, pin_whole_budget_is_dense, pin_brute_force_mask]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_lvsa_oracle_pin(pin):
    pin(lv)


# ----------------------------------------------------------------------------- planted mistakes

class Planted:
    def __init__(self, **repl):
        self.repl = repl

    def __enter__(self):
        self.saved = {k: getattr(lv, k) for k in self.repl}
        for k, v in self.repl.items():
            setattr(lv, k, v)
        return lv

    def __exit__(self, *a):
        for k, v in self.saved.items():
            setattr(lv, k, v)


REAL_WINDOW = lv.local_window
REAL_ATTENDED = lv.attended_frames


def _fixed_grid(T, T_per, s):
    """Mistake: anchors do not rotate with the step."""
    return np.arange(0, T, T_per, dtype=np.int64)


def _window_not_extended(T, t, G, C):
    """Mistake: the window keeps C - |G| frames however many anchors it overlaps."""
    w = max(1, C - len(G))
    lo = max(0, min(t - (w - 1) // 2, T - w))
    return lo, min(T - 1, lo + w - 1)


def _anchors_left_out(T, T_per, C, s):
    """Mistake: A(t) = W(t) only."""
    G = lv.global_frames(T, T_per, s)
    return [np.arange(*(lambda lh: (lh[0], lh[1] + 1))(REAL_WINDOW(T, t, G, C))) for t in range(T)]


@pytest.mark.parametrize("repl,pin", [
    ({"global_frames": _fixed_grid}, pin_rotation),
    ({"local_window": _window_not_extended}, pin_budget_and_shape),
    ({"attended_frames": _anchors_left_out}, pin_budget_and_shape),
])
def test_planted_mask_mistake_is_caught(repl, pin):
    with Planted(**repl) as mod:
        with pytest.raises(AssertionError):
            pin(mod)
