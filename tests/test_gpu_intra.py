"""GPU parity of matching inside a commit (option intra_chunk) against the oracle.

The oracle takes the tokens of a commit in ascending t and lets each one match the
entries committed before and the entries created by earlier tokens of the same
commit (its step 8b); the CUDA path must produce the same codes, merge targets,
entry indices, sizes, keys, counts and codes bit for bit, value means within 1e-3
and attention within the bf16 / fp32 tolerances.
"""
import numpy as np
import pytest
import torch

from synthetic import CONFIGS, Workload
from tests.gpu_harness import f64, run_parity
from tests.test_gpu_parity import BF16_MAX, BF16_MEAN, F32_TOL, V32_TOL, assert_exact, small_bf16

pytestmark = pytest.mark.gpu


def test_intra_small_bf16_rollout_ragged():
    cfg = small_bf16(sigma=0.03, tau=0.97)
    rep, tc, _ = run_parity(cfg, attends=2, intra_chunk=True)
    assert_exact(rep)
    assert rep.merges > 0
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_intra_tiny_f32():
    cfg = CONFIGS["tiny-f32"]
    rep, tc, _ = run_parity(cfg, attends=2, intra_chunk=True)
    assert_exact(rep)
    assert rep.attn_max_err <= F32_TOL, rep


def test_intra_exact_duplicates_one_entry_per_distinct_key():
    cfg = CONFIGS["long-rollout-dup"].replace(H=2, P=300, chunks=5, S=128, capacity=10_000)
    rep, tc, _ = run_parity(cfg, attends=1, intra_chunk=True)
    assert_exact(rep)
    assert max(max(s) for s in rep.sizes) <= cfg.S
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_intra_identical_keys_one_bucket_scan_path():
    # every token carries the same key: one bucket of hundreds of tokens per head,
    # so the dedupe visits members by scanning; the whole chunk collapses into one entry
    from kv_cache_attention_tempcache_b200 import TempCache
    from oracle import OracleTempCache

    H, d, T = 2, 128, 300
    g = torch.Generator(device="cpu").manual_seed(5)
    key = torch.randn(1, 1, d, generator=g).to(torch.bfloat16)
    R = torch.randn(8, d, generator=g).to(torch.bfloat16).float().numpy()
    tc = TempCache(H, d, 8, 0.95, 10_000, hyperplanes=R, intra_chunk=True)
    o = OracleTempCache(H, d, 8, 0.95, 10_000, R.astype(np.float64), intra_chunk=True)
    for c in range(3):
        K = key.expand(T, H, d).contiguous()
        V = torch.randn(T, H, d, generator=g).to(torch.bfloat16)
        rec = o.append_chunk(f64(K), f64(V))
        tc.append_chunk(K.cuda(), V.cuda())
        if rec is not None:
            _, match, dest = tc.last_commit()
            assert (match == rec.match).all() and (dest == rec.dest).all()
        Q = torch.randn(64, H, d, generator=g).to(torch.bfloat16)
        err = np.abs(f64(tc.attend(Q.cuda())) - o.attend(f64(Q)))
        assert err.max() <= BF16_MAX
    tc.flush()
    o.flush()
    assert (tc.cache_size() == 1).all() and (o.cache_size() == 1).all()
    for h in range(H):
        K, V32, n, code = tc.export_cache(h)
        k, v, nr, cr = o.export_head(h)
        assert (n == nr).all() and np.abs(V32 - v).max() <= V32_TOL


def test_intra_wan13b_full_shape_sampled():
    cfg = CONFIGS["wan1.3b"]
    rows = np.unique(np.concatenate([np.arange(0, 40), np.arange(4600, 4680),
                                     np.random.default_rng(1).integers(0, 4680, 136)]))
    rep, tc, _ = run_parity(cfg, chunks=4, attends=1, rows=rows, state_heads=[0, 11], check_every_state=False,
                            intra_chunk=True)
    assert_exact(rep)
    assert rep.merges > 0
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_intra_capacity_refusal_is_repeatable():
    from kv_cache_attention_tempcache_b200 import TempCache, CapacityError

    from oracle import OracleTempCache

    cfg = small_bf16(chunks=3)
    # a capacity that holds chunk 0 but not chunk 1 (sizes from the oracle)
    wo = Workload(cfg, device="cuda")
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, 10 ** 6, wo.hyperplanes().double().numpy(),
                        intra_chunk=True)
    for _ in range(2):
        K, V = wo.next_chunk()
        o.append_chunk(f64(K), f64(V))
    s0 = o.cache_size().copy()
    o.flush()
    cap = int(s0.max()) + 1
    assert (o.cache_size() > cap).any()
    w = Workload(cfg, device="cuda")
    tc = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cap, hyperplanes=w.hyperplanes().numpy(), intra_chunk=True)
    K0, V0 = w.next_chunk()
    tc.append_chunk(K0, V0)
    K1, V1 = w.next_chunk()
    tc.append_chunk(K1, V1)        # commits chunk 0
    before = [tc.export_cache(h) for h in range(cfg.H)]
    for _ in range(2):             # the refused commit leaves nothing behind, so it refuses again
        with pytest.raises(CapacityError):
            tc.flush()
        for h in range(cfg.H):
            for a, b in zip(before[h], tc.export_cache(h)):
                assert np.array_equal(a, b)
