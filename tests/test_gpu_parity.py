"""GPU parity: the CUDA TempCache against the fp64 CPU oracle on seeded workloads.

Rules (integer results bit-exact; floats within the stated tolerances):
  hash codes, merge targets, entry indices, cache sizes, keys, counts and codes of
  the cache: bit-exact;
  fp32 value means: 1e-3 absolute;
  attention: max-abs 2e-2 and mean-abs 2e-3 for bf16 storage, 1e-5 for fp32.
"""
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from synthetic import CONFIGS, Workload
from tests.gpu_harness import f64, run_parity

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


def test_tiny_f32_full_rollout():
    cfg = CONFIGS["tiny-f32"]
    rep, tc, _ = run_parity(cfg, attends=cfg.attends)
    assert_exact(rep)
    assert rep.merges > 0
    assert rep.attn_max_err <= F32_TOL, rep


def small_bf16(**kw):
    # ragged: T = 2 * 200 = 400 tokens, not a multiple of the 128-row tiles
    base = CONFIGS["wan1.3b"].replace(H=3, P=200, F=2, chunks=6, S=96, nbits=10, capacity=4000, seed=11)
    return base.replace(**kw)


def test_small_bf16_rollout_ragged():
    cfg = small_bf16()
    rep, tc, _ = run_parity(cfg, attends=2)
    assert_exact(rep)
    assert rep.merges > 0
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_small_bf16_d64():
    cfg = small_bf16(d=64, nbits=8)
    rep, _, _ = run_parity(cfg, attends=1)
    assert_exact(rep)
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_f32_d128():
    cfg = small_bf16(dtype="f32", chunks=4)
    rep, _, _ = run_parity(cfg, attends=1)
    assert_exact(rep)
    assert rep.attn_max_err <= F32_TOL, rep


@pytest.mark.parametrize("tau", [-1.0, 2.0])
def test_threshold_extremes(tau):
    # tau = -1 merges every token that finds a candidate; tau = 2 never merges (dense cache)
    cfg = small_bf16(tau=tau, chunks=4)
    rep, tc, o = run_parity(cfg, attends=1)
    assert_exact(rep)
    if tau > 1:
        assert rep.merges == 0 and int(o.cache_size().sum()) == cfg.H * cfg.T * cfg.chunks
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


@pytest.mark.parametrize("nbits", [1, 24])
def test_hash_width_extremes(nbits):
    cfg = small_bf16(nbits=nbits, chunks=3, H=2)
    rep, _, _ = run_parity(cfg, attends=1)
    assert_exact(rep)
    assert rep.attn_max_err <= BF16_MAX, rep


def test_single_token_chunks_and_single_query():
    cfg = small_bf16(P=1, F=1, chunks=5, S=3)
    rep, _, _ = run_parity(cfg, attends=1)
    assert_exact(rep)
    assert rep.attn_max_err <= BF16_MAX, rep


def test_degenerate_identical_keys_large_groups():
    # every token carries the same key: one bucket, ties everywhere, merge groups
    # larger than a warp (exercises the ordered-selection merge path)
    from kv_cache_attention_tempcache_b200 import TempCache
    from oracle import OracleTempCache

    H, d, T = 2, 128, 300
    g = torch.Generator(device="cpu").manual_seed(3)
    key = torch.randn(1, 1, d, generator=g).to(torch.bfloat16)
    R = torch.randn(8, d, generator=g).to(torch.bfloat16).float().numpy()
    tc = TempCache(H, d, 8, 0.95, 10_000, hyperplanes=R)
    o = OracleTempCache(H, d, 8, 0.95, 10_000, R.astype(np.float64))
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
    for h in range(H):
        K, V32, n, code = tc.export_cache(h)
        k, v, nr, cr = o.export_head(h)
        assert (n == nr).all() and np.abs(V32 - v).max() <= V32_TOL


def test_large_logits_take_the_running_reference():
    # queries x8: every row's Cauchy-Schwarz bound of its logits is ~130 > 40, so each
    # CTA runs the lazy online softmax reference (handover between the teams, O
    # rescaled when the reference moves) over merged entries and a ragged staged tile
    cfg = small_bf16(chunks=5)
    rep, _, _ = run_parity(cfg, attends=2, q_scale=8.0)
    assert_exact(rep)
    assert rep.merges > 0
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_logits_near_the_fixed_bound():
    # queries x1.55: the rows' Cauchy-Schwarz bounds are ~30-38, under the fixed-reference
    # limit, so the CTAs take p = 2^x with no reference at magnitudes up to ~2^38
    cfg = small_bf16(chunks=5)
    rep, _, _ = run_parity(cfg, attends=2, q_scale=1.55)
    assert_exact(rep)
    assert rep.attn_max_err <= BF16_MAX and rep.attn_mean_err <= BF16_MEAN, rep


def test_large_key_norms_take_the_running_reference():
    # the same branch reached from the key side: keys scaled x6 and rounded to bf16
    # (both sides see the rounded values), queries of norm sqrt(d)
    from kv_cache_attention_tempcache_b200 import TempCache
    from oracle import OracleTempCache

    cfg = small_bf16(chunks=4, H=2)
    w = Workload(cfg, device="cuda")
    R = w.hyperplanes()
    tc = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, hyperplanes=R.numpy())
    o = OracleTempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, R.double().numpy())
    worst, tot, n = 0.0, 0.0, 0
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        K = (K.float() * 6.0).to(torch.bfloat16)
        rec = o.append_chunk(f64(K), f64(V))
        tc.append_chunk(K, V)
        if rec is not None:
            _, match, dest = tc.last_commit()
            assert np.array_equal(match, rec.match) and np.array_equal(dest, rec.dest)
        Q = w.queries(c, 0)
        err = np.abs(f64(tc.attend(Q)) - o.attend(f64(Q)))
        worst = max(worst, float(err.max()))
        tot += float(err.sum())
        n += err.size
    assert worst <= BF16_MAX and tot / n <= BF16_MEAN


def test_exact_duplicates_equal_dense_attention():
    # Lemma 5.1 end to end on the GPU: with identical keys merged, the compressed
    # attention equals attention over the full uncompressed history
    cfg = CONFIGS["long-rollout-dup"].replace(H=2, P=512, chunks=5, S=256, capacity=10_000)
    from kv_cache_attention_tempcache_b200 import TempCache

    w = Workload(cfg, device="cuda")
    R = w.hyperplanes()
    tc = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, hyperplanes=R.numpy())
    hist_k, hist_v = [], []
    worst, mean = 0.0, 0.0
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        tc.append_chunk(K, V)
        hist_k.append(K.float())
        hist_v.append(V.float())
        Q = w.queries(c, 0)
        out = tc.attend(Q).float()
        Kh, Vh = torch.cat(hist_k), torch.cat(hist_v)
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q.float().transpose(0, 1)[None], Kh.transpose(0, 1)[None], Vh.transpose(0, 1)[None],
            scale=1 / math.sqrt(cfg.d))[0].transpose(0, 1)
        err = (out - ref).abs()
        worst = max(worst, float(err.max()))
        mean = max(mean, float(err.mean()))
    sizes = tc.cache_size()
    assert sizes.max() < cfg.T * (cfg.chunks - 1)   # compressed
    assert worst <= BF16_MAX and mean <= BF16_MEAN


def test_capacity_overflow_is_refused_and_state_kept():
    from kv_cache_attention_tempcache_b200 import TempCache, CapacityError

    cfg = small_bf16(chunks=3)
    w = Workload(cfg, device="cuda")
    tc = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.T + 3, hyperplanes=w.hyperplanes().numpy())
    K0, V0 = w.next_chunk()
    tc.append_chunk(K0, V0)
    K1, V1 = w.next_chunk()
    tc.append_chunk(K1, V1)        # commits chunk 0 (T entries)
    before = [tc.export_cache(h) for h in range(cfg.H)]
    Q = w.queries(1, 0)
    out_before = tc.attend(Q).clone()
    K2, V2 = w.next_chunk()
    with pytest.raises(CapacityError):
        tc.append_chunk(K2, V2)    # chunk 1 does not fit
    for h in range(cfg.H):
        for a, b in zip(before[h], tc.export_cache(h)):
            assert np.array_equal(a, b)
    # chunk 1 is still staged: attention is unchanged
    assert torch.equal(tc.attend(Q), out_before)


def test_deterministic_across_runs():
    cfg = small_bf16(chunks=4)
    outs = []
    for _ in range(2):
        from kv_cache_attention_tempcache_b200 import TempCache
        w = Workload(cfg, device="cuda")
        tc = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, hyperplanes=w.hyperplanes().numpy())
        res = []
        for c in range(cfg.chunks):
            K, V = w.next_chunk()
            tc.append_chunk(K, V)
            res.append(tc.attend(w.queries(c, 0)).clone())
        tc.flush()
        res.append(torch.from_numpy(tc.export_cache(0)[1]))
        outs.append(res)
    for a, b in zip(*outs):
        assert torch.equal(a.cpu(), b.cpu())


def test_attend_before_append_and_bad_pointers():
    from kv_cache_attention_tempcache_b200 import TempCache, TempCacheError, TC_ESTATE, TC_EINVAL, lib

    tc = TempCache(2, 128, 8, 0.9, 100)
    Q = torch.zeros(4, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TempCacheError) as e:
        tc.attend(Q)
    assert e.value.status == TC_ESTATE
    raw = torch.zeros(4 * 2 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    mis = raw.data_ptr() + 2  # not 16-byte aligned
    assert lib.tc_append_chunk(tc.handle, mis, mis, 4, None) == TC_EINVAL


def test_default_hyperplanes_are_bf16_normals():
    from kv_cache_attention_tempcache_b200 import TempCache

    a = TempCache(1, 128, 24, 0.9, 10, seed=5).hyperplanes()
    b = TempCache(1, 128, 24, 0.9, 10, seed=5).hyperplanes()
    c = TempCache(1, 128, 24, 0.9, 10, seed=6).hyperplanes()
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert np.all((a.view(np.uint32) & 0xFFFF) == 0)
    assert abs(a.mean()) < 0.05 and abs(a.std() - 1) < 0.05


def test_injected_allocation_failure_reports_enomem():
    code = ("import os, torch, ctypes\n"
            "torch.zeros(1, device='cuda')\n"
            "import kv_cache_attention_tempcache_b200 as m\n"
            "h = ctypes.c_void_p()\n"
            "st = m.lib.tc_create(2, 128, 8, 0.9, 1000, ctypes.byref(h))\n"
            "print(st, bool(h.value))\n")
    env = dict(os.environ, TC_FAULT_ALLOC_AT="3")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))), timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.split() == ["2", "False"]
