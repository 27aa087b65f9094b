"""GPU parity of LVSA frame-masked attention against the CPU oracle, through the C ABI.

The frame sets A(t) are integer results: bit-exact. The output is bf16 tensor-core
arithmetic: max-abs error <= 2e-2, mean-abs <= 2e-3 against fp64.
"""
import numpy as np
import pytest
import torch

from oracle import attended_frames, lvsa_attention

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def f64(x):
    return x.detach().to(torch.float64).cpu().numpy()


def run(T, P, H, d, T_per, C, steps, q_scale=1.0, seed=0):
    from kv_cache_attention_tempcache_b200 import LVSA
    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(seed)
    Q, K, V = (torch.randn(T * P, H, d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    if q_scale != 1.0:
        Q = (Q.float() * q_scale).to(torch.bfloat16)
    lv = LVSA(H, d, P, T_per, C)
    for s in steps:
        out = lv.attend(Q, K, V, s)
        got = lv.frames()
        exp = attended_frames(T, T_per, C, s)
        assert all(np.array_equal(a, b) for a, b in zip(got, exp))
        err = np.abs(f64(out) - lvsa_attention(f64(Q), f64(K), f64(V), P, T_per, C, s))
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (s, err.max(), err.mean())
    lv.sync()
    lv.close()


def test_frames_narrower_than_a_tile():
    run(T=7, P=100, H=2, d=64, T_per=3, C=4, steps=range(3))


def test_frames_of_several_tiles():
    run(T=12, P=300, H=2, d=128, T_per=5, C=5, steps=(0, 7))


def test_budget_covering_the_video_is_dense():
    run(T=5, P=64, H=1, d=128, T_per=2, C=9, steps=(1,))


def test_large_logits():
    run(T=6, P=128, H=2, d=128, T_per=3, C=3, steps=(2,), q_scale=8.0)
