"""GPU parity of AnnSA (same-bucket self-attention) against the CPU oracle, through the C ABI.

The buckets are the AnnCA query codes of the same block (checked bit-exact by the AnnCA
tests); the oracle here recomputes them itself from the pages' definition. The output
is bf16 tensor-core arithmetic: max-abs error <= 2e-2, mean-abs <= 2e-3 against fp64.
"""
import numpy as np
import pytest
import torch

from oracle import annca_cross_attention, annsa_attention
from synthetic import CROSS_CONFIGS, CrossWorkload

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def f64(x):
    return x.detach().to(torch.float64).cpu().numpy()


def run(cfg, q_scale=1.0, calls=1):
    from kv_cache_attention_tempcache_b200 import AnnCA
    torch.cuda.set_device(0)
    w = CrossWorkload(cfg, device="cuda")
    R = w.hyperplanes()
    ann = AnnCA(cfg.H, cfg.d, cfg.nbits, hyperplanes=R.numpy())
    Kp, Vp = w.prompt()
    ann.set_prompt(Kp, Vp)
    sizes = []
    for c in range(calls):
        Qc = w.queries(c)
        ann.attend(Qc, cfg.P)
        Q, K, V = w.self_qkv(c)
        if q_scale != 1.0:
            Q = (Q.float() * q_scale).to(torch.bfloat16)
        out = ann.self_attend(Q, K, V)
        _, _, qcodes, _ = annca_cross_attention(f64(Qc), f64(Kp), f64(Vp), R.double().numpy(), cfg.P)
        ref = annsa_attention(f64(Q), f64(K), f64(V), qcodes)
        err = np.abs(f64(out) - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (c, err.max(), err.mean())
        sizes.append([np.unique(qcodes[h], return_counts=True)[1] for h in range(cfg.H)])
    ann.sync()
    ann.close()
    return sizes


def test_tiny_block():
    run(CROSS_CONFIGS["annca-tiny"], calls=2)


def test_buckets_spanning_several_tiles():
    cfg = CROSS_CONFIGS["annca-tiny"].replace(H=3, d=128, P=300, F=2, L=64, C=4, A=2, nbits=3, seed=3011)
    sizes = run(cfg)
    assert max(s.max() for s in sizes[0]) > 256   # a bucket wider than two key tiles


def test_mostly_singleton_buckets():
    cfg = CROSS_CONFIGS["annca-tiny"].replace(nbits=24, sigma=1.0, seed=3012)
    sizes = run(cfg)
    assert sum((s == 1).sum() for s in sizes[0]) > 0


@pytest.mark.parametrize("nbits", [10, 12, 14])
def test_every_ordering_path(nbits):
    # codes of <= 10 bits are ordered by per-warp segment counts, <= 13 by one shared count,
    # wider ones by a sort; a ragged token count (2 x 700) in each
    cfg = CROSS_CONFIGS["annca-tiny"].replace(H=2, d=128, P=700, F=2, nbits=nbits, sigma=0.5,
                                              seed=3020 + nbits)
    run(cfg)


@pytest.mark.parametrize("P", [5, 129])
def test_blocks_with_few_tokens(P):
    # T = 5 leaves most of the eight ordering blocks of a head empty; T = 129 puts one token
    # past the first 128-row tile
    cfg = CROSS_CONFIGS["annca-tiny"].replace(H=2, P=P, F=1, nbits=6, seed=3030 + P)
    run(cfg)


def test_largest_block():
    # T = 16 383, one short of the largest block: every warp of the ordering takes all of
    # its 32-token steps
    cfg = CROSS_CONFIGS["annca-tiny"].replace(H=1, d=128, P=5461, F=3, nbits=10, sigma=0.5, seed=3040)
    run(cfg)


def test_large_logits_take_the_running_reference():
    # |q| max|k| scale log2(e) ~ 130 > 40: the kernel cannot use the fixed softmax
    # reference and starts each row's running reference at its own logit
    run(CROSS_CONFIGS["annca-tiny"].replace(seed=3013), q_scale=8.0)


def test_state_and_argument_errors():
    import kv_cache_attention_tempcache_b200 as m
    cfg = CROSS_CONFIGS["annca-tiny"]
    w = CrossWorkload(cfg, device="cuda")
    ann = m.AnnCA(cfg.H, cfg.d, cfg.nbits, hyperplanes=w.hyperplanes().numpy())
    Q, K, V = w.self_qkv(0)
    with pytest.raises(m.TempCacheError) as e:
        ann.self_attend(Q, K, V)                  # no AnnCA call yet: no buckets
    assert e.value.status == m.TC_ESTATE
    Kp, Vp = w.prompt()
    ann.set_prompt(Kp, Vp)
    ann.attend(w.queries(0), cfg.P)
    with pytest.raises(m.TempCacheError) as e:
        ann.self_attend(Q[:-cfg.P], K[:-cfg.P], V[:-cfg.P])   # not the block AnnCA pruned
    assert e.value.status == m.TC_ESTATE
    ann.self_attend(Q, K, V)
    ann.sync()
    ann.close()


def test_full_size_wan13b_block():
    """The Wan-2.1-1.3B-shaped block (12 heads, 3 x 1560 tokens, 10-bit buckets), in the
    launch configuration the benchmark times, compared in full."""
    run(CROSS_CONFIGS["annca-wan1.3b"])
