"""Pins of the AnnSA oracle against facts fixed outside the oracle itself.

FAST-AR summary, section 2.C "AnnSA": every token's query attends only to the keys
of tokens in its own semantic bucket. The pins:
  * one bucket for every token: textbook softmax attention (torch's routine);
  * every token alone in its bucket: out_t = v_t exactly;
  * brute force: a dense mask built by a pure-Python double loop over the buckets,
    applied through torch's masked attention routine;
  * equivariance: permuting the tokens permutes the output rows;
  * buckets are labels only: renaming them changes nothing.
The last section plants mistakes in the oracle and checks that a pin catches each.
"""
import numpy as np
import pytest
import torch

import oracle.annsa_oracle as sa


def sdpa(Q, K, V, scale, mask=None):
    """Textbook attention of one head by torch: Q, K, V [T, d]; mask [T, T] bool (True = attend)."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))[None, None]  # noqa: E731
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), attn_mask=m, scale=scale)[0, 0].numpy()


def block(T=23, H=2, d=16, nb=5, seed=0):
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.standard_normal((T, H, d)) for _ in range(3))
    buckets = rng.integers(0, nb, size=(H, T)).astype(np.uint32) * 977   # sparse labels
    return Q, K, V, buckets


def pin_one_bucket_is_dense(mod):
    Q, K, V, _ = block()
    out = mod.annsa_attention(Q, K, V, np.full((2, Q.shape[0]), 7, np.uint32))
    for h in range(2):
        np.testing.assert_allclose(out[:, h], sdpa(Q[:, h], K[:, h], V[:, h], 1 / 4.0), rtol=0, atol=1e-12)


def pin_singletons_return_own_value(mod):
    Q, K, V, _ = block()
    T = Q.shape[0]
    out = mod.annsa_attention(Q, K, V, np.tile(np.arange(T, dtype=np.uint32), (2, 1)))
    np.testing.assert_array_equal(out, V)


def pin_brute_force_mask(mod):
    Q, K, V, buckets = block(seed=3)
    T, H, d = Q.shape
    out = mod.annsa_attention(Q, K, V, buckets)
    for h in range(H):
        mask = np.zeros((T, T), bool)
        for i in range(T):
            for j in range(T):
                mask[i, j] = int(buckets[h][i]) == int(buckets[h][j])
        np.testing.assert_allclose(out[:, h], sdpa(Q[:, h], K[:, h], V[:, h], 1 / np.sqrt(d), mask),
                                   rtol=0, atol=1e-12)


def pin_permutation_equivariance(mod):
    Q, K, V, buckets = block(seed=4)
    perm = np.random.default_rng(9).permutation(Q.shape[0])
    a = mod.annsa_attention(Q, K, V, buckets)
    b = mod.annsa_attention(Q[perm], K[perm], V[perm], buckets[:, perm])
    np.testing.assert_allclose(b, a[perm], rtol=0, atol=1e-12)


def pin_labels_only(mod):
    Q, K, V, buckets = block(seed=5)
    renamed = (buckets.astype(np.int64) * 31 + 5).astype(np.uint32)
    np.testing.assert_allclose(mod.annsa_attention(Q, K, V, renamed), mod.annsa_attention(Q, K, V, buckets),
                               rtol=0, atol=1e-12)


PINS = [pin_one_bucket_is_dense, pin_singletons_return_own_value, pin_brute_force_mask,
        pin_permutation_equivariance, pin_labels_only]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_annsa_oracle_pin(pin):
    pin(sa)


# ----------------------------------------------------------------------------- planted mistakes

class Planted:
    def __init__(self, **repl):
        self.repl = repl

    def __enter__(self):
        self.saved = {k: getattr(sa, k) for k in self.repl}
        for k, v in self.repl.items():
            setattr(sa, k, v)
        return sa

    def __exit__(self, *a):
        for k, v in self.saved.items():
            setattr(sa, k, v)


REAL_GROUPS = sa.same_bucket_groups


def _groups_drop_first(buckets):
    """Mistake: the first token of every bucket with company left out."""
    return [g if g.size == 1 else g[1:] for g in REAL_GROUPS(buckets)]


def _groups_bucket_order_not_token(buckets):
    """Mistake: groups cut as consecutive runs of the token order."""
    b = np.asarray(buckets)
    cuts = np.nonzero(b[1:] != b[:-1])[0] + 1
    return np.split(np.arange(b.size), cuts)


def _groups_merge_neighbours(buckets):
    """Mistake: buckets whose labels are adjacent in sorted order merged pairwise."""
    u = np.unique(np.asarray(buckets))
    out = []
    for i in range(0, u.size, 2):
        out.append(np.nonzero(np.isin(buckets, u[i:i + 2]))[0])
    return out


@pytest.mark.parametrize("mistake,pin", [
    (_groups_drop_first, pin_brute_force_mask),
    (_groups_bucket_order_not_token, pin_brute_force_mask),
    (_groups_merge_neighbours, pin_brute_force_mask),
])
def test_planted_grouping_mistake_is_caught(mistake, pin):
    with Planted(same_bucket_groups=mistake) as mod:
        with pytest.raises(AssertionError):
            pin(mod)


def test_planted_wrong_scale_is_caught():
    real = sa.annsa_attention

    def unscaled(Q, K, V, buckets, scale=None):
        return real(Q, K, V, buckets, scale=1.0)

    with Planted(annsa_attention=unscaled) as mod:
        with pytest.raises(AssertionError):
            pin_one_bucket_is_dense(mod)
