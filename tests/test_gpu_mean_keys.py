"""GPU parity of running-mean keys (option key_mode="mean") against the fp64 oracle.

FAST-AR technical summary, section 2.A: keys merge under a similarity threshold and
values are averaged; with running-mean keys the entry's key is averaged too (the
oracle's step 8c): k <- (n k + sum k_t) / (n + m) in fp32 in ascending t, the code is
recomputed from the new key and the entry moves to that bucket for later commits.

Rules: codes, merge targets, entry indices, sizes, counts and cache codes bit-exact;
the fp32 key means bit-exact (same fp32 operations in the same order); value means
within 1e-3; attention within max-abs 2e-2 / mean-abs 2e-3 (bf16 storage, whose
keys are the bf16 roundings of the means) or 1e-5 (fp32 storage).
"""
import numpy as np
import pytest
import torch

from synthetic import CONFIGS
from tests.gpu_harness import run_parity

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN, F32_TOL, V32_TOL = 2e-2, 2e-3, 1e-5, 1e-3


def assert_exact(rep):
    assert rep.code_mismatch == 0, rep
    assert rep.match_mismatch == 0, rep
    assert rep.dest_mismatch == 0, rep
    assert rep.size_mismatch == 0, rep
    assert rep.key_mismatch == 0, rep
    assert rep.count_mismatch == 0, rep
    assert rep.v32_max_err <= V32_TOL, rep


def small(**kw):
    # ragged: T = 2 * 200 = 400 tokens; a loose threshold makes merges of distinct keys
    # (and so mean keys that are not bf16 values, and codes that change) common
    base = CONFIGS["wan1.3b"].replace(H=3, P=200, F=2, chunks=6, S=96, nbits=10, capacity=4000, seed=41,
                                      tau=0.9, sigma=0.12)
    return base.replace(**kw)


def test_mean_keys_small_bf16():
    cfg = small()
    rep, tc, o = run_parity(cfg, attends=2, key_mode="mean")
    assert_exact(rep)
    assert rep.merges > 0
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep
    # some merged keys are no longer bf16 values: the fp32 chain of the search ran
    keys = [o.export_head(h)[0] for h in range(cfg.H)]
    nonbf16 = sum(int(((k.astype(np.float32).view(np.uint32) & 0xFFFF) != 0).any(axis=1).sum()) for k in keys)
    assert nonbf16 > 0
    assert tc.stats()["match_rechecks"] > 0


def test_mean_keys_longer_rollout():
    cfg = small(chunks=10, tau=0.85, sigma=0.15, nbits=12)
    rep, tc, o = run_parity(cfg, attends=1, key_mode="mean")
    assert_exact(rep)
    assert rep.merges > 0
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_mean_key_that_changes_bucket_is_found_there():
    # Members of an entry share its code, and a convex combination of keys on one side
    # of a hyperplane stays on that side, so a mean key changes code only through the
    # fp32 rounding of the mean. Hand-built case, one hyperplane R = (1, -3, 0, ...):
    # keys (3y, y) lie exactly on it (bit 1); the fp32 mean of these three lands just
    # below it (bit 0), so the entry must move to bucket 0, where the probe of the third
    # chunk finds it (with representative keys the probe is appended instead).
    from kv_cache_attention_tempcache_b200 import TempCache
    from oracle import OracleTempCache
    from tests.gpu_harness import f64

    d = 64
    R = np.zeros((1, d), np.float32)
    R[0, 0], R[0, 1] = 1.0, -3.0

    def rows(*pairs):
        x = torch.zeros(len(pairs), 1, d)
        for i, (a, b) in enumerate(pairs):
            x[i, 0, 0], x[i, 0, 1] = a, b
        return x.to(torch.bfloat16)

    chunks = [rows((0.03515625, 0.01171875), (-1.0, 1.0)),
              rows((0.00439453125, 0.00146484375), (0.64453125, 0.21484375)),
              rows((0.2265625, 0.076171875))]
    g = torch.Generator().manual_seed(0)
    tc = TempCache(1, d, 1, 0.9, 100, hyperplanes=R, key_mode="mean")
    o = OracleTempCache(1, d, 1, 0.9, 100, R.astype(np.float64), key_mode="mean")
    matches = []
    for K in chunks:
        V = torch.randn(K.shape, generator=g).to(torch.bfloat16)
        rec = o.append_chunk(f64(K), f64(V))
        tc.append_chunk(K.cuda(), V.cuda())
        if rec is not None:
            codes, match, dest = tc.last_commit()
            assert np.array_equal(codes, rec.codes) and np.array_equal(match, rec.match)
            assert np.array_equal(dest, rec.dest)
    rec = o.flush()
    tc.flush()
    codes, match, dest = tc.last_commit()
    assert np.array_equal(match, rec.match) and int(match[0, 0]) == 0   # the probe found the moved entry
    k, v32, n, code = tc.export_cache(0)
    k_ref, v_ref, n_ref, c_ref = o.export_head(0)
    assert np.array_equal(k.astype(np.float64), k_ref) and np.array_equal(n, n_ref)
    assert np.array_equal(code, c_ref) and int(code[0]) == 0
    assert np.abs(v32 - v_ref).max() <= V32_TOL


def test_mean_keys_d64_and_wide_codes():
    cfg = small(d=64, nbits=20, chunks=4)
    rep, _, _ = run_parity(cfg, attends=1, key_mode="mean")
    assert_exact(rep)
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_mean_keys_f32_storage():
    cfg = CONFIGS["tiny-f32"].replace(tau=0.9, sigma=0.1)
    rep, _, _ = run_parity(cfg, attends=2, key_mode="mean")
    assert_exact(rep)
    assert rep.merges > 0
    assert rep.attn_max_err <= F32_TOL, rep


def test_mean_keys_identical_keys_equal_representative():
    # sigma = 0: every merged key equals its entry's key, so the mean key is the key
    # itself and the state equals the representative-key state
    cfg = small(sigma=0.0, tau=1.0 - 1e-6, chunks=5)
    rep_m, tc_m, _ = run_parity(cfg, attends=1, key_mode="mean")
    rep_r, tc_r, _ = run_parity(cfg, attends=1)
    assert_exact(rep_m)
    assert np.array_equal(tc_m.cache_size(), tc_r.cache_size())
    for h in range(cfg.H):
        a = tc_m.export_cache(h)
        b = tc_r.export_cache(h)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[2], b[2]) and np.array_equal(a[3], b[3])


def test_mean_keys_wan13b_shape():
    cfg = CONFIGS["wan1.3b"]
    rows = np.unique(np.concatenate([np.arange(0, 40), np.arange(4600, 4680),
                                     np.random.default_rng(5).integers(0, 4680, 136)]))
    rep, tc, o = run_parity(cfg, chunks=8, attends=1, rows=rows, oracle_heads=[0, 11], attn_chunks={0, 7},
                            key_mode="mean")
    assert_exact(rep)
    assert rep.merges > 0
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_mean_keys_need_the_snapshot_commit():
    from kv_cache_attention_tempcache_b200 import TempCache, TempCacheError
    with pytest.raises(TempCacheError):
        TempCache(2, 128, 8, 0.9, 100, intra_chunk=True, key_mode="mean")
