"""Pins of the CPU oracle against facts fixed outside the oracle itself.

The pages (FAST-AR technical summary, section 2.A "TempCache") state the method in
prose only, so the pins are: a hand-derived worked example (tests/golden), Lemma
5.1 as a closed form (merged + shifted attention equals uncompressed attention
for identical keys), textbook attention through torch's own kernel, brute-force
top-1 search on tiny inputs, conservation invariants, and the textbook SimHash
collision law. The last section plants mistakes in the oracle and checks that a
pin catches each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.tempcache_oracle as orc
from oracle import OracleTempCache, CapacityExceeded
from synthetic import CONFIGS, Workload, round_to_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(x):
    return x.to(torch.float64).cpu().numpy()


def sdpa_reference(Q, K, V, scale):
    """Plain softmax attention by torch's own routine, fp64 on the CPU. Q [Tq,H,d]."""
    q = torch.from_numpy(np.ascontiguousarray(Q.transpose(1, 0, 2)))[None]
    k = torch.from_numpy(np.ascontiguousarray(K.transpose(1, 0, 2)))[None]
    v = torch.from_numpy(np.ascontiguousarray(V.transpose(1, 0, 2)))[None]
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)
    return out[0].numpy().transpose(1, 0, 2)


def small_cfg(**kw):
    base = CONFIGS["wan1.3b"].replace(H=2, d=64, P=48, F=2, chunks=6, S=24, nbits=6,
                                      capacity=10_000, seed=77)
    return base.replace(**kw)


# ----------------------------------------------------------------------------- golden

def test_golden_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "tiny_hand_example.json")))
    o = OracleTempCache(g["H"], g["d"], g["nbits"], g["tau"], 100, np.array(g["hyperplanes"]),
                        scale=g["scale"])
    recs = []
    for c, ch in enumerate(g["chunks"]):
        K = np.array(ch["K"], float)[:, None, :]
        V = np.array(ch["V"], float)[:, None, :]
        recs.append(o.append_chunk(K, V))
        assert list(o.staged[2][0]) == g["expected_codes"][c]
        if c == 2:   # appending chunk C commits chunk B
            keys, vals, cnt, _ = o.export_head(0)
            exp = g["expected_after_chunk_B_commit"]
            np.testing.assert_array_equal(keys, exp["keys"])
            np.testing.assert_array_equal(vals, exp["values"])
            np.testing.assert_array_equal(cnt, exp["counts"])
    for item in g["attend_with_C_staged"]:
        out = o.attend(np.array(item["q"], float)[None, None, :])
        np.testing.assert_allclose(out[0, 0], np.array(item["out_num"]) / item["out_den"],
                                   rtol=0, atol=1e-14)
    recs.append(o.flush())
    for rec, exp in zip(recs[1:], g["expected_commits"]):
        assert list(rec.match[0]) == exp["match"]
        assert list(rec.dest[0]) == exp["dest"]
        assert int(rec.sizes[0]) == exp["size"]
    _, vals, cnt, _ = o.export_head(0)
    np.testing.assert_array_equal(vals, g["expected_after_chunk_C_commit"]["values"])
    np.testing.assert_array_equal(cnt, g["expected_after_chunk_C_commit"]["counts"])
    for item in g["attend_after_flush"]:
        out = o.attend(np.array(item["q"], float)[None, None, :])
        np.testing.assert_allclose(out[0, 0], np.array(item["out_num"]) / item["out_den"],
                                   rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------- Lemma 5.1

def run_lemma(cfg, calls_per_chunk=2, intra_chunk=False):
    """Max |oracle - uncompressed softmax attention| over a rollout with exact duplicates."""
    w = Workload(cfg)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()),
                        intra_chunk=intra_chunk)
    hist_k, hist_v, worst, merged = [], [], 0.0, 0
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        rec = o.append_chunk(f64(K), f64(V))
        if rec is not None:
            merged += int((rec.match >= 0).sum())
        hist_k.append(f64(K))
        hist_v.append(f64(V))
        Kh, Vh = np.concatenate(hist_k), np.concatenate(hist_v)
        for a in range(calls_per_chunk):
            Q = f64(w.queries(c, a))
            ref = sdpa_reference(Q, Kh, Vh, 1.0 / math.sqrt(cfg.d))
            worst = max(worst, float(np.abs(o.attend(Q) - ref).max()))
    return worst, merged, o


def test_lemma51_exact_duplicates_equal_uncompressed_attention():
    cfg = small_cfg(sigma=0.0, tau=1.0 - 1e-6, p_stay=0.7)
    worst, merged, o = run_lemma(cfg)
    assert merged > 0, "the rollout must exercise merges"
    assert o.cache_size().max() < o.committed_tokens, "the cache must be compressed"
    assert worst < 1e-9


def test_no_merge_reduces_to_textbook_attention():
    cfg = small_cfg(tau=2.0)  # a threshold above 1 never merges: every n is 1
    w = Workload(cfg)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()))
    hist_k, hist_v = [], []
    for c in range(3):
        K, V = w.next_chunk()
        o.append_chunk(f64(K), f64(V))
        hist_k.append(f64(K))
        hist_v.append(f64(V))
        Q = f64(w.queries(c, 0))
        ref = sdpa_reference(Q, np.concatenate(hist_k), np.concatenate(hist_v), 1 / math.sqrt(cfg.d))
        assert np.abs(o.attend(Q) - ref).max() < 1e-12


def test_deferred_commit_first_attend_sees_raw_chunk():
    cfg = small_cfg()
    w = Workload(cfg)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()))
    K, V = w.next_chunk()
    assert o.append_chunk(f64(K), f64(V)) is None
    assert o.cache_size().sum() == 0
    Q = f64(w.queries(0, 0))
    ref = sdpa_reference(Q, f64(K), f64(V), 1 / math.sqrt(cfg.d))
    assert np.abs(o.attend(Q) - ref).max() < 1e-12


# ----------------------------------------------------------------------------- top-1

def brute_force_match(keys, codes, cache_keys, cache_codes, tau):
    """Pure-Python top-1: scan every entry, keep equal codes, cosine by loops."""
    tau64 = float(np.float32(tau))
    out = []
    for t in range(len(keys)):
        k = [float(x) for x in keys[t]]
        best, best_sim = -1, -math.inf
        for j in range(len(cache_keys)):
            if int(cache_codes[j]) != int(codes[t]):
                continue
            e = [float(x) for x in cache_keys[j]]
            dot = nk = ne = 0.0
            for a, b in zip(k, e):
                dot += a * b
                nk += a * a
                ne += b * b
            sim = dot / math.sqrt(nk * ne) if (nk > 0 and ne > 0) else 0.0
            if sim > best_sim:          # strict: the first (lowest) index wins ties
                best, best_sim = j, sim
        out.append(best if (best >= 0 and best_sim >= tau64) else -1)
    return np.array(out)


def tiny_clustered_keys(rng, protos, n, noise, dup_frac):
    """Noisy copies of a few prototypes, some replaced by exact power-of-two multiples."""
    idx = rng.integers(0, protos.shape[0], n)
    x = protos[idx] + noise * rng.standard_normal((n, protos.shape[1]))
    dup = rng.random(n) < dup_frac
    x[dup] = protos[idx[dup]] * (2.0 ** rng.integers(0, 3, dup.sum()))[:, None]
    return round_to_bf16(torch.from_numpy(x).float()).double().numpy()


def tiny_top1_case(seed):
    rng = np.random.default_rng(seed)
    d, nbits = 8, 2
    R = round_to_bf16(torch.from_numpy(rng.standard_normal((nbits, d))).float()).double().numpy()
    protos = round_to_bf16(torch.from_numpy(rng.standard_normal((6, d))).float()).double().numpy()
    cache = tiny_clustered_keys(rng, protos, 60, 0.05, 0.3)
    new = tiny_clustered_keys(rng, protos, 40, 0.05, 0.3)
    return R, cache, new


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_top1_equals_brute_force(seed):
    R, cache, new = tiny_top1_case(seed)
    cache_codes = orc.simhash_codes(R, cache)
    codes = orc.simhash_codes(R, new)
    for tau in (0.95, 0.5, -1.0):
        best, sim = orc.top1_in_bucket(new, codes, cache, cache_codes)
        got = orc.merge_decision(best, sim, tau)
        want = brute_force_match(new, codes, cache, cache_codes, tau)
        np.testing.assert_array_equal(got, want)
    # the case must contain exact ties that the tie-break decides
    best, sim = orc.top1_in_bucket(new, codes, cache, cache_codes)
    assert (sim == 1.0).sum() > 0


# ----------------------------------------------------------------------------- invariants

def test_conservation_and_order_invariants():
    cfg = small_cfg(chunks=5)
    w = Workload(cfg)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()))
    committed_v = [np.zeros((0, cfg.d)) for _ in range(cfg.H)]
    committed_k = [np.zeros((0, cfg.d)) for _ in range(cfg.H)]
    staged = None
    for c in range(cfg.chunks + 1):
        if c < cfg.chunks:
            K, V = w.next_chunk()
            rec = o.append_chunk(f64(K), f64(V))
        else:
            rec = o.flush()
        if staged is not None:
            for h in range(cfg.H):
                committed_k[h] = np.concatenate([committed_k[h], staged[0][:, h]])
                committed_v[h] = np.concatenate([committed_v[h], staged[1][:, h]])
        staged = (f64(K), f64(V)) if c < cfg.chunks else None
        for h in range(cfg.H):
            keys, vals, cnt, _ = o.export_head(h)
            # (i) each committed token counted once
            assert cnt.sum() == committed_v[h].shape[0] == o.committed_tokens
            # (ii) n-weighted values add up to the committed values
            np.testing.assert_allclose((cnt[:, None] * vals).sum(0), committed_v[h].sum(0),
                                       rtol=0, atol=1e-9)
            # (iii) entry keys are committed keys, in order of first appearance
            pos = [int(np.nonzero((committed_k[h] == k).all(1))[0][0]) for k in keys]
            assert pos == sorted(pos)
            if rec is not None:
                # dest points at the entry the token ended in
                assert (rec.dest[h] >= 0).all() and (rec.dest[h] < keys.shape[0]).all()


def test_exact_duplicates_entry_count_matches_snapshot_dedupe():
    cfg = small_cfg(sigma=0.0, tau=1.0 - 1e-6, chunks=5)
    w = Workload(cfg)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()))
    seen = [set() for _ in range(cfg.H)]
    expected = np.zeros(cfg.H, dtype=int)
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        o.append_chunk(f64(K), f64(V))
        o.flush()
        Kn = f64(K)
        for h in range(cfg.H):
            snapshot = set(seen[h])
            for t in range(cfg.T):
                key = Kn[t, h].tobytes()
                if key not in snapshot:
                    expected[h] += 1          # snapshot: duplicates inside one chunk all append
                seen[h].add(key)
        np.testing.assert_array_equal(o.cache_size(), expected)


def test_capacity_refusal_leaves_state_unchanged():
    cfg = small_cfg()
    w = Workload(cfg)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, capacity=cfg.T + 5,
                        hyperplanes=f64(w.hyperplanes()))
    K0, V0 = w.next_chunk()
    o.append_chunk(f64(K0), f64(V0))
    K1, V1 = w.next_chunk()
    o.append_chunk(f64(K1), f64(V1))            # commits chunk 0: T entries
    before = [o.export_head(h) for h in range(cfg.H)]
    staged_before = o.staged
    K2, V2 = w.next_chunk()
    with pytest.raises(CapacityExceeded):
        o.append_chunk(f64(K2), f64(V2))        # chunk 1 cannot fit
    assert o.staged is staged_before
    for h in range(cfg.H):
        for a, b in zip(before[h], o.export_head(h)):
            np.testing.assert_array_equal(a, b)


# ----------------------------------------------------------------------------- hash

AXIS_X = np.array([[1, -1, 0, 2, -0.5, 0, 3, -2],
                   [0, 0, 0, 0, 0, 0, 0, 0],
                   [-1, -1, -1, -1, -1, -1, -1, -1]], dtype=float)


def axis_codes_ok():
    """Axis hyperplanes: bit b of x is [x_b >= 0], including exact zeros."""
    want = [sum((1 << b) for b in range(8) if AXIS_X[i, b] >= 0) for i in range(3)]
    return list(orc.simhash_codes(np.eye(8), AXIS_X)) == want


def test_simhash_axis_hyperplanes_closed_form():
    assert axis_codes_ok()


def test_simhash_collision_law():
    """P[bit differs] = angle / pi for Gaussian hyperplanes (Charikar 2002)."""
    rng = np.random.default_rng(5)
    d, nbits, n = 32, 24, 4000
    R = rng.standard_normal((nbits, d))
    for theta in (0.2, 0.8, 1.6):
        a = rng.standard_normal((n, d))
        u = rng.standard_normal((n, d))
        u -= (u * a).sum(1, keepdims=True) / (a * a).sum(1, keepdims=True) * a
        a /= np.linalg.norm(a, axis=1, keepdims=True)
        u /= np.linalg.norm(u, axis=1, keepdims=True)
        b = np.cos(theta) * a + np.sin(theta) * u
        diff = orc.simhash_codes(R, a) ^ orc.simhash_codes(R, b)
        frac = np.unpackbits(diff.view(np.uint8)).sum() / (n * nbits)
        sd = math.sqrt(theta / math.pi * (1 - theta / math.pi) / (n * nbits))
        # hyperplanes are shared across pairs, so allow more than the iid spread
        assert abs(frac - theta / math.pi) < 10 * sd + 0.01


def test_cosine_special_cases():
    a = np.array([[1.0, 2.0, -3.0], [0.0, 0.0, 0.0], [1.5, -2.0, 0.25]])
    b = np.array([[2.0, 4.0, -6.0], [1.0, 1.0, 1.0], [-1.5, 2.0, -0.25]])
    np.testing.assert_array_equal(orc.cosine_similarity(a, b), [1.0, 0.0, -1.0])


def test_seq_dot_is_index_ordered():
    # in index order (1e16 + 1) rounds back to 1e16, so the sum is 0; the exact sum is 1
    a = np.array([[1e16, 1.0, -1e16]])
    assert orc.seq_dot(a, np.ones((1, 3)))[0] == 0.0
    assert math.fsum([1e16, 1.0, -1e16]) == 1.0


# ----------------------------------------------------------------------------- planted mistakes

def test_planted_mistake_zero_bias_breaks_lemma(monkeypatch):
    real = orc.biased_attention
    monkeypatch.setattr(orc, "biased_attention",
                        lambda Q, K, V, bias, scale: real(Q, K, V, np.zeros_like(bias), scale))
    worst, merged, _ = run_lemma(small_cfg(sigma=0.0, tau=1.0 - 1e-6, p_stay=0.7, chunks=3), 1)
    assert merged > 0 and worst > 1e-3


def test_planted_mistake_highest_index_tie_break_is_caught(monkeypatch):
    real = orc.top1_in_bucket

    def flipped(keys, codes, cache_keys, cache_codes):
        # same search over a reversed cache, indices mapped back: ties go to the highest index
        M = len(cache_keys)
        best, sim = real(keys, codes, cache_keys[::-1], cache_codes[::-1])
        return np.where(best >= 0, M - 1 - best, -1), sim

    monkeypatch.setattr(orc, "top1_in_bucket", flipped)
    R, cache, new = tiny_top1_case(0)
    cc, c = orc.simhash_codes(R, cache), orc.simhash_codes(R, new)
    best, sim = orc.top1_in_bucket(new, c, cache, cc)
    assert (orc.merge_decision(best, sim, 0.95) != brute_force_match(new, c, cache, cc, 0.95)).any()


def test_planted_mistake_strict_sign_is_caught(monkeypatch):
    def strict(R, X):
        proj = orc.seq_dot(np.asarray(X, float)[:, None, :], np.asarray(R, float)[None])
        return ((proj > 0) * (1 << np.arange(R.shape[0]))).sum(1).astype(np.uint32)

    monkeypatch.setattr(orc, "simhash_codes", strict)
    assert not axis_codes_ok()


def conservation_error(cfg, oracle_factory=OracleTempCache):
    """max |sum_j n_j v_j - sum of committed values| over heads after a flushed rollout."""
    w = Workload(cfg)
    o = oracle_factory(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()))
    sums = np.zeros((cfg.H, cfg.d))
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        o.append_chunk(f64(K), f64(V))
        sums += f64(V).sum(0)
    o.flush()
    return max(np.abs((o.export_head(h)[2][:, None] * o.export_head(h)[1]).sum(0) - sums[h]).max()
               for h in range(cfg.H))


def test_conservation_error_is_rounding_only():
    assert conservation_error(small_cfg(chunks=3)) < 1e-9


def test_planted_mistake_dropping_old_group_breaks_conservation():
    class DropsOldGroup(OracleTempCache):
        """Planted mistake: a merged entry keeps only the new tokens' mean."""

        def _commit(self):
            staged = self.staged
            rec = super()._commit()
            if rec is not None:
                V = staged[1]
                for h in range(self.H):
                    for j in np.unique(rec.match[h][rec.match[h] >= 0]):
                        grp = rec.match[h] == j
                        self.heads[h].values[j] = V[h, grp].mean(0)
                        self.heads[h].counts[j] = grp.sum()
            return rec

    assert conservation_error(small_cfg(chunks=3), DropsOldGroup) > 1e-3


# ----------------------------------------------------------------------------- intra-chunk variant (8b)

def test_intra_exact_duplicates_entry_count_equals_distinct_keys():
    """With exact duplicates and matching inside a commit, every distinct key seen so
    far is exactly one entry (a plain set of key bytes counts them)."""
    cfg = small_cfg(sigma=0.0, tau=1.0 - 1e-6, chunks=5)
    w = Workload(cfg)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()),
                        intra_chunk=True)
    seen = [set() for _ in range(cfg.H)]
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        o.append_chunk(f64(K), f64(V))
        o.flush()
        Kn = f64(K)
        for h in range(cfg.H):
            seen[h].update(Kn[t, h].tobytes() for t in range(cfg.T))
        np.testing.assert_array_equal(o.cache_size(), [len(x) for x in seen])
    assert o.cache_size().max() <= cfg.S


def test_intra_lemma51_exact_duplicates_equal_uncompressed_attention():
    cfg = small_cfg(sigma=0.0, tau=1.0 - 1e-6, p_stay=0.7)
    worst, merged, o = run_lemma(cfg, intra_chunk=True)
    assert merged > 0
    assert worst < 1e-9


def test_intra_conservation_and_order():
    cfg = small_cfg(chunks=4, sigma=0.02, tau=0.99)
    w = Workload(cfg)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()),
                        intra_chunk=True)
    snap = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()))
    all_k = [np.zeros((0, cfg.d)) for _ in range(cfg.H)]
    all_v = [np.zeros((0, cfg.d)) for _ in range(cfg.H)]
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        rec = o.append_chunk(f64(K), f64(V))
        snap.append_chunk(f64(K), f64(V))
        o.flush()
        snap.flush()
        for h in range(cfg.H):
            all_k[h] = np.concatenate([all_k[h], f64(K)[:, h]])
            all_v[h] = np.concatenate([all_v[h], f64(V)[:, h]])
            keys, vals, cnt, _ = o.export_head(h)
            assert cnt.sum() == all_v[h].shape[0]
            np.testing.assert_allclose((cnt[:, None] * vals).sum(0), all_v[h].sum(0), rtol=0, atol=1e-9)
            pos = [int(np.nonzero((all_k[h] == k).all(1))[0][0]) for k in keys]
            assert pos == sorted(pos)
    # matching inside a commit can only merge more
    assert (o.cache_size() <= snap.cache_size()).all() and (o.cache_size() < snap.cache_size()).any()


def test_planted_mistake_intra_without_creating_token_breaks_conservation(monkeypatch):
    """Averaging a new entry's later members without its creating token is caught."""
    cfg = small_cfg(chunks=3, sigma=0.0, tau=1.0 - 1e-6)
    real = orc.new_entry_members
    monkeypatch.setattr(orc, "new_entry_members", lambda u, row, e: real(u, row, e)[1:] if (row == e).any()
                        else real(u, row, e))
    w = Workload(cfg)
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, f64(w.hyperplanes()),
                        intra_chunk=True)
    total = np.zeros(cfg.d)
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        o.append_chunk(f64(K), f64(V))
        o.flush()
        total += f64(V)[:, 0].sum(0)
    _, vals, cnt, _ = o.export_head(0)
    assert np.abs((cnt[:, None] * vals).sum(0) - total).max() > 1e-6


# ----------------------------------------------------------------------------- running-mean keys (step 8c)

def _rollout(cfg, key_mode, chunks=None):
    w = Workload(cfg)
    R = f64(w.hyperplanes())
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, R, key_mode=key_mode)
    recs = []
    for _ in range(chunks or cfg.chunks):
        K, V = w.next_chunk()
        recs.append(o.append_chunk(f64(K), f64(V)))
    recs.append(o.flush())
    return o, [r for r in recs if r is not None], R


def test_mean_keys_of_identical_duplicates_change_nothing():
    cfg = small_cfg(sigma=0.0, tau=1.0 - 1e-6, S=12, chunks=5)
    a, ra, _ = _rollout(cfg, "representative")
    b, rb, _ = _rollout(cfg, "mean")
    for x, y in zip(ra, rb):
        np.testing.assert_array_equal(x.match, y.match)
        np.testing.assert_array_equal(x.dest, y.dest)
    for h in range(cfg.H):
        for u, v in zip(a.export_head(h), b.export_head(h)):
            np.testing.assert_array_equal(u, v)
    assert sum(int((r.match >= 0).sum()) for r in rb) > 0   # there were merges


def _exact_code(R, key):
    from fractions import Fraction
    code = 0
    for b in range(R.shape[0]):
        s = sum(Fraction(float(R[b, i])) * Fraction(float(key[i])) for i in range(R.shape[1]))
        code |= int(s >= 0) << b
    return code


def test_mean_keys_codes_follow_their_keys():
    cfg = small_cfg(d=16, nbits=5, sigma=0.3, tau=0.8, S=6, chunks=4, P=24)
    o, recs, R = _rollout(cfg, "mean")
    moved = 0
    for h in range(cfg.H):
        keys, _, cnt, codes = o.export_head(h)
        for k, c in zip(keys, codes):
            assert int(c) == _exact_code(R, k)
        np.testing.assert_array_equal(keys, keys.astype(np.float32).astype(np.float64))   # fp32 values
        moved += int((cnt > 1).sum())
    assert moved > 0


def test_mean_keys_conserve_the_key_sum():
    cfg = small_cfg(d=16, nbits=5, sigma=0.3, tau=0.8, S=6, chunks=4, P=24)
    w = Workload(cfg)
    total = np.zeros((cfg.H, cfg.d))
    for _ in range(cfg.chunks):
        K, _ = w.next_chunk()
        total += f64(K).sum(axis=0)
    o, _, _ = _rollout(cfg, "mean")
    for h in range(cfg.H):
        keys, _, cnt, _ = o.export_head(h)
        got = (cnt[:, None] * keys).sum(axis=0)
        assert np.abs(got - total[h]).max() <= 1e-4 * np.abs(total[h]).max() * cfg.T


def test_mean_keys_worked_example():
    """Hand geometry (one head, d = 2, one hyperplane along y, tau = 0.85): keys at 0, 20
    and 40 degrees in three chunks. The 20-degree key merges into the first entry
    (cos 20 = 0.94). With representative keys the 40-degree key then sees the 0-degree
    key (cos 40 = 0.77 < 0.85) and is appended; with running-mean keys it sees their mean
    at about 10 degrees (cos 30 = 0.87 >= 0.85) and merges too."""
    def unit(deg):
        return round_to_bf16(torch.tensor([[math.cos(math.radians(deg)), math.sin(math.radians(deg))]])).double().numpy()

    R = np.array([[0.0, 1.0]])
    ks = [unit(0), unit(20), unit(40)]
    sizes = {}
    for mode in ("representative", "mean"):
        o = OracleTempCache(1, 2, 1, 0.85, 10, R, key_mode=mode)
        for k in ks:
            o.append_chunk(k[:, None, :], np.ones((1, 1, 2)))
        o.flush()
        sizes[mode] = int(o.cache_size()[0])
        if mode == "mean":
            keys, _, cnt, _ = o.export_head(0)
            assert cnt.tolist() == [3]
            np.testing.assert_allclose(keys[0], (ks[0][0] + ks[1][0] + ks[2][0]) / 3, rtol=0, atol=1e-6)
    assert sizes == {"representative": 2, "mean": 1}


def test_planted_stale_code_is_caught(monkeypatch):
    real = orc.simhash_codes
    calls = {"n": 0}

    def stale_after_merge(R, X):
        calls["n"] += 1
        out = real(R, X)
        return out ^ np.uint32(1) if np.asarray(X).shape[0] == 1 else out   # the mean key's code corrupted

    monkeypatch.setattr(orc, "simhash_codes", stale_after_merge)
    with pytest.raises(AssertionError):
        test_mean_keys_codes_follow_their_keys()


def test_planted_mean_without_old_count_is_caught(monkeypatch):
    real = orc.mean_key_fp32
    monkeypatch.setattr(orc, "mean_key_fp32", lambda key, n, members: real(key, 1, members))
    with pytest.raises(AssertionError):
        test_mean_keys_conserve_the_key_sum()
