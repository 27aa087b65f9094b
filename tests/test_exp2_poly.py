"""The attention kernel computes part of its 2^x on the FMA pipe with its own cubic
(see exp2_poly2 in csrc/tc_attn_bf16.cu). This replays the same fp32 steps with the
coefficients read from the source and bounds the error against the exact 2^x."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cache_attention_tempcache_b200", "csrc", "tc_attn_bf16.cu")


def coefficients():
    text = open(SRC).read()
    return [np.float32(float(re.search(rf"kExpC{k} = ([0-9.eE+-]+)f", text).group(1))) for k in range(4)]


def exp2_poly_fp32(x):
    c0, c1, c2, c3 = coefficients()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    f = (x - n).astype(f32)
    q = (f * c3 + c2).astype(f32)
    q = (q * f + c1).astype(f32)
    q = (q * f + c0).astype(f32)
    bits = q.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_exp2_poly_relative_error():
    x = np.concatenate([np.linspace(-125, 9, 2_000_001, dtype=np.float64),
                        np.random.default_rng(0).uniform(-30, 8, 200_000)]).astype(np.float32)
    got = exp2_poly_fp32(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert np.max(np.abs(got / want - 1)) < 1e-4


def test_exp2_poly_clamps_large_negative_inputs():
    x = np.array([-np.inf, -1e30, -200, -126], dtype=np.float32)
    got = exp2_poly_fp32(x)
    assert np.all(got == exp2_poly_fp32(np.array([-125.0], dtype=np.float32))[0])
    assert np.all(got < 1e-37)
