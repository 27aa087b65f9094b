"""GPU parity at the full shapes of every synthetic workload, through the C ABI.

Each test runs the CUDA TempCache over every head at the workload's own sizes and
follows a few heads with the fp64 CPU oracle (heads are independent in the method
and in both implementations, so the oracle may run a subset). Rules as in
test_gpu_parity.py: codes, merge targets, entry indices, sizes, keys, counts and
cache codes bit-exact at every commit; value means within 1e-3; attention on sampled
query rows (the first rows, the ragged last tile and random rows) within max-abs
2e-2 and mean-abs 2e-3.

Workloads: Wan-2.1-1.3B-shaped layer over its whole 40-chunk rollout; the 160-chunk
long rollout; its exact-duplicate variant, whose compressed attention must equal
plain softmax attention over the whole uncompressed history (FAST-AR technical
summary, section 2.A, Lemma 5.1); the Wan-14B 720p-shaped layer; the low-redundancy
stress workload until the cache holds more than 100 000 entries per head and the
capacity pre-check has to wait for the commit's outcome.
"""
import numpy as np
import pytest
import torch

from oracle import biased_attention
from synthetic import CONFIGS
from tests.gpu_harness import f64, run_parity

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN, V32_TOL = 2e-2, 2e-3, 1e-3


def sample_rows(T, seed=0):
    last = T - T % 128 if T % 128 else T - 128
    return np.unique(np.concatenate([np.arange(0, 40), np.arange(max(last - 8, 0), T),
                                     np.random.default_rng(seed).integers(0, T, 136)]))


def assert_exact(rep):
    assert rep.code_mismatch == 0, rep
    assert rep.match_mismatch == 0, rep
    assert rep.dest_mismatch == 0, rep
    assert rep.size_mismatch == 0, rep
    assert rep.key_mismatch == 0, rep
    assert rep.count_mismatch == 0, rep
    assert rep.v32_max_err <= V32_TOL, rep


def assert_attention(rep, checks):
    assert rep.attn_checks == checks, rep
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_wan13b_whole_rollout():
    # all 40 chunks of the benchmarked workload: every commit bit-exact on three heads,
    # their caches compared after every commit, attention at chunks 1, 20 and 40
    cfg = CONFIGS["wan1.3b"]
    rep, tc, o = run_parity(cfg, attends=1, rows=sample_rows(cfg.T), oracle_heads=[0, 5, 11],
                            attn_chunks={0, 19, 39})
    assert_exact(rep)
    assert rep.commits == cfg.chunks and rep.merges > 0
    assert_attention(rep, 3)
    assert tc.stats()["match_rechecks"] > 0   # the exact re-check path ran on real near-ties
    assert int(o.cache_size().min()) > 3 * cfg.S


def test_long_rollout_160_chunks():
    cfg = CONFIGS["long-rollout"]
    rep, tc, o = run_parity(cfg, attends=1, rows=sample_rows(cfg.T, 1), oracle_heads=[0, 7],
                            attn_chunks={0, 79, 159}, check_every_state=False)
    assert_exact(rep)
    assert rep.commits == cfg.chunks
    assert_attention(rep, 3)
    # the cache grows ever more slowly: fewer than 1% of a chunk's tokens are new at the end
    growth = np.diff(np.asarray(rep.sizes), axis=0)[-10:]
    assert growth.max() < 0.01 * cfg.T


def test_long_rollout_exact_duplicates_equal_dense_history():
    # sigma = 0: merged keys are identical, so by Lemma 5.1 attention over the compressed
    # cache (+ln n) equals plain softmax attention over every token appended so far
    cfg = CONFIGS["long-rollout-dup"]
    heads = [0, 6]
    rows = sample_rows(cfg.T, 2)
    hist_k, hist_v = [], []
    checked = []

    def on_chunk(c, tc, o, w, K, V):
        hist_k.append(K[:, heads].clone())
        hist_v.append(V[:, heads].clone())
        if c not in (39, 79, 159):
            return
        Q = w.queries(c, 0)
        out = tc.attend(Q)
        Kh = torch.cat(hist_k).cpu()
        Vh = torch.cat(hist_v).cpu()
        q = f64(Q[torch.as_tensor(rows, device=Q.device)])
        got = f64(out[torch.as_tensor(rows, device=out.device)])
        for i, h in enumerate(heads):
            Kd = Kh[:, i].to(torch.float64).numpy()
            Vd = Vh[:, i].to(torch.float64).numpy()
            ref = biased_attention(q[:, h], Kd, Vd, np.zeros(Kd.shape[0]), 1.0 / np.sqrt(cfg.d))
            err = np.abs(got[:, h] - ref)
            checked.append((c, h, float(err.max()), float(err.mean())))

    rep, tc, o = run_parity(cfg, attends=0, oracle_heads=heads, check_every_state=False, on_chunk=on_chunk)
    assert_exact(rep)
    assert len(checked) == 3 * len(heads)
    for c, h, mx, mn in checked:
        assert mx <= BF16_MAX and mn <= BF16_MEAN, (c, h, mx, mn)
    sizes = np.asarray(rep.sizes)
    assert (sizes[-1] == sizes[-20]).all()               # the cache stopped growing
    assert sizes[-1].max() < cfg.T * cfg.chunks // 50    # compressed more than 50x


def test_wan14b_720p_first_chunks():
    cfg = CONFIGS["wan14b-720p"]
    rep, tc, o = run_parity(cfg, chunks=8, attends=1, rows=sample_rows(cfg.T, 3), oracle_heads=[0, 19, 39],
                            attn_chunks={0, 3, 7}, check_every_state=False)
    assert_exact(rep)
    assert rep.commits == 8 and rep.merges > 0
    assert_attention(rep, 3)


def test_low_redundancy_large_cache():
    # nbits 18, capacity 262 144: past chunk 56 the host can no longer prove that a
    # commit fits and waits for its outcome; the cache ends above 100 000 entries per head
    cfg = CONFIGS["low-redundancy"]
    rep, tc, o = run_parity(cfg, chunks=60, attends=1, rows=sample_rows(cfg.T, 4), oracle_heads=[0, 7],
                            attn_chunks={20, 59}, check_every_state=False)
    assert_exact(rep)
    assert rep.commits == 60
    assert_attention(rep, 2)
    assert int(o.cache_size().min()) > 100_000
    assert int(tc.cache_size().min()) > 100_000
