"""GPU parity of AnnCA cross-attention against the CPU oracle, through the C ABI.

Kept sets, query codes and prompt codes are integer results: bit-exact. The
attention output is bf16 tensor-core arithmetic with fp32 accumulation: max-abs
error <= 2e-2 and mean-abs error <= 2e-3 against the fp64 oracle, the bound the
TempCache attention tests use (bf16 output rounding alone is up to 2^-9 relative).
"""
import numpy as np
import pytest
import torch

from oracle import annca_cross_attention
from oracle.tempcache_oracle import biased_attention, simhash_codes
from oracle.annca_oracle import kept_prompt_tokens
from synthetic import CROSS_CONFIGS, CrossWorkload

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def f64(x):
    return x.detach().to(torch.float64).cpu().numpy()


def run_case(cfg, calls=1, prompt=None, queries=None):
    from kv_cache_attention_tempcache_b200 import AnnCA
    torch.cuda.set_device(0)
    w = CrossWorkload(cfg, device="cuda")
    R = w.hyperplanes()
    ann = AnnCA(cfg.H, cfg.d, cfg.nbits, hyperplanes=R.numpy())
    Kp, Vp = prompt if prompt is not None else w.prompt()
    ann.set_prompt(Kp, Vp)
    results = []
    for c in range(calls):
        Q = queries[c] if queries is not None else w.queries(c)
        out = ann.attend(Q, cfg.P)
        keep, qc, pc = ann.kept()
        ref, rkeep, rqc, rpc = annca_cross_attention(f64(Q), f64(Kp), f64(Vp), R.double().numpy(), cfg.P)
        np.testing.assert_array_equal(pc, rpc)
        np.testing.assert_array_equal(qc, rqc)
        np.testing.assert_array_equal(keep, rkeep)
        err = np.abs(f64(out) - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (c, err.max(), err.mean())
        results.append((out, rkeep, ref))
    ann.close()
    return results


def test_tiny_frames_narrower_than_a_tile():
    # P = 96 < 128: every attention tile straddles two frames
    res = run_case(CROSS_CONFIGS["annca-tiny"], calls=2)
    keep = res[0][1]
    assert 0 < keep.sum() < keep.size


def test_several_tiles_with_ragged_tails():
    # kept sets longer than one 128-key tile, frames of 2.3 tiles, d = 128
    cfg = CROSS_CONFIGS["annca-tiny"].replace(H=3, d=128, P=300, F=2, L=700, C=6, A=3, nbits=4, seed=2011)
    res = run_case(cfg)
    counts = res[0][1].sum(-1)
    assert counts.max() > 256 and (counts % 128 != 0).any()


def test_frame_with_no_shared_bucket_gets_zero_rows():
    cfg = CROSS_CONFIGS["annca-tiny"].replace(F=2, seed=2012)
    w = CrossWorkload(cfg, device="cuda")
    Kp, Vp = w.prompt()
    Q = w.queries(0)
    # head 0: every prompt key is a positive multiple of one vector k (one code), and
    # every query of frame 1 is -k, whose code is the complement: no shared bucket
    k = Kp[0, 0].float()
    Kp = Kp.clone()
    Kp[:, 0] = (k[None, :] * torch.linspace(0.5, 2.0, cfg.L, device="cuda")[:, None]).to(torch.bfloat16)
    Q = Q.clone()
    Q[:10, 0] = k.to(torch.bfloat16)[None, :]            # frame 0 shows the prompt's direction
    Q[cfg.P:, 0] = (-k).to(torch.bfloat16)[None, :]      # frame 1 only its opposite
    out, keep, _ = run_case(cfg, prompt=(Kp, Vp), queries=[Q])[0]
    assert not keep[0, 1].any() and keep[0, 0].any()
    assert torch.count_nonzero(out[cfg.P:, 0]).item() == 0


def test_prompt_regrowth_and_repeated_calls():
    from kv_cache_attention_tempcache_b200 import AnnCA
    cfg = CROSS_CONFIGS["annca-tiny"].replace(seed=2013)
    w = CrossWorkload(cfg, device="cuda")
    R = w.hyperplanes()
    ann = AnnCA(cfg.H, cfg.d, cfg.nbits, hyperplanes=R.numpy())
    for L in (40, 300, 90):   # grows (reallocates), then shrinks (reuses)
        w2 = CrossWorkload(cfg.replace(L=L), device="cuda")
        Kp, Vp = w2.prompt()
        ann.set_prompt(Kp, Vp)
        for c in range(2):
            Q = w2.queries(c)
            out = ann.attend(Q, cfg.P)
            keep, qc, pc = ann.kept()
            ref, rkeep, _, _ = annca_cross_attention(f64(Q), f64(Kp), f64(Vp), R.double().numpy(), cfg.P)
            np.testing.assert_array_equal(keep, rkeep)
            err = np.abs(f64(out) - ref)
            assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (L, c, err.max())
    ann.close()


def test_argument_errors():
    import kv_cache_attention_tempcache_b200 as m
    cfg = CROSS_CONFIGS["annca-tiny"]
    ann = m.AnnCA(cfg.H, cfg.d, cfg.nbits)
    Q = torch.zeros(cfg.T, cfg.H, cfg.d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.TempCacheError) as e:
        ann.attend(Q, cfg.P)                      # no prompt yet
    assert e.value.status == m.TC_ESTATE
    Kp = torch.randn(cfg.L, cfg.H, cfg.d, device="cuda").to(torch.bfloat16)
    ann.set_prompt(Kp, Kp.clone())
    with pytest.raises(m.TempCacheError) as e:
        ann.attend(Q, cfg.P + 1)                  # not whole frames
    assert e.value.status == m.TC_EINVAL
    big = torch.zeros(4097, cfg.H, cfg.d, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.TempCacheError) as e:
        ann.set_prompt(big, big)                  # longer than the sort holds
    assert e.value.status == m.TC_EINVAL
    ann.attend(Q, cfg.P)                          # still usable
    ann.sync()
    ann.close()


def test_full_size_wan13b_prompt_pruning():
    """The Wan-2.1-1.3B-shaped layer (12 heads, 3 frames of 1560 tokens, 512 prompt
    tokens), in the launch configuration the benchmark times: every code and kept set
    exact, attention checked on sampled query rows of every head and frame."""
    from kv_cache_attention_tempcache_b200 import AnnCA
    cfg = CROSS_CONFIGS["annca-wan1.3b"]
    torch.cuda.set_device(0)
    w = CrossWorkload(cfg, device="cuda")
    R = w.hyperplanes()
    R64 = R.double().numpy()
    ann = AnnCA(cfg.H, cfg.d, cfg.nbits, hyperplanes=R.numpy())
    Kp, Vp = w.prompt()
    ann.set_prompt(Kp, Vp)
    Q = w.queries(0)
    out = ann.attend(Q, cfg.P)
    keep, qc, pc = ann.kept()
    Qn, Kn, Vn, On = f64(Q), f64(Kp), f64(Vp), f64(out)
    rng = np.random.default_rng(3)
    errs = []
    for h in range(cfg.H):
        rqc = simhash_codes(R64, Qn[:, h])
        rpc = simhash_codes(R64, Kn[:, h])
        np.testing.assert_array_equal(qc[h], rqc)
        np.testing.assert_array_equal(pc[h], rpc)
        rkeep = kept_prompt_tokens(rqc.reshape(cfg.F, cfg.P), rpc)
        np.testing.assert_array_equal(keep[h], rkeep)
        for f in range(cfg.F):
            sel = np.nonzero(rkeep[f])[0]
            rows = f * cfg.P + rng.choice(cfg.P, 24, replace=False)
            ref = biased_attention(Qn[rows, h], Kn[sel, h], Vn[sel, h], np.zeros(sel.size), 1 / np.sqrt(cfg.d))
            errs.append(np.abs(On[rows, h] - ref))
    err = np.concatenate([e.ravel() for e in errs])
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    frac = keep.sum() / keep.size
    assert 0.05 < frac < 0.5, frac   # the synthetic prompt is pruned, not emptied
    ann.close()
