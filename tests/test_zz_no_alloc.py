"""tc_merge_means_noalloc: the merge step for callers that cannot allocate device
memory while running (fixed-arena inference runtimes, plugins inside a framework
that owns the device allocator). Its scratch is a fixed array inside the library.

The test drives the regular path (tc_append_chunk commits a chunk with merges),
then replays the same merges through the allocation-free call on copies of the
pre-commit means and counts, for two heads in a row, and requires the same means
(within the value-mean tolerance 1e-3 used by the parity tests; the arithmetic
order is the same, so they agree bit for bit in practice) and identical counts.
This file is collected last so that a failure here leaves every other test run.
"""
import ctypes

import numpy as np
import pytest
import torch

from synthetic import CONFIGS, Workload

pytestmark = pytest.mark.gpu


def test_noalloc_merge_matches_the_commit_path():
    import kv_cache_attention_tempcache_b200 as m
    from kv_cache_attention_tempcache_b200 import TempCache

    cfg = CONFIGS["wan1.3b"].replace(H=3, P=400, F=2, chunks=3, S=120, nbits=10, capacity=5000, seed=31)
    w = Workload(cfg, device="cuda")
    tc = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, hyperplanes=w.hyperplanes().numpy())
    K0, V0 = w.next_chunk()
    K1, V1 = w.next_chunk()
    K2, V2 = w.next_chunk()
    tc.append_chunk(K0, V0)
    tc.append_chunk(K1, V1)                      # commits chunk 0
    before = [tc.export_cache(h) for h in range(cfg.H)]
    tc.append_chunk(K2, V2)                      # commits chunk 1, with merges
    _, match, _ = tc.last_commit()
    after = [tc.export_cache(h) for h in range(cfg.H)]
    assert (match >= 0).sum() > 0

    for h in (0, 1):                             # two calls in a row
        _, v32_b, n_b, _ = before[h]
        _, v32_a, n_a, _ = after[h]
        M0 = n_b.shape[0]
        src = V1[:, h, :].contiguous()           # bf16 values of the committed chunk
        target = torch.from_numpy(match[h].astype(np.int32)).cuda()
        mean = torch.from_numpy(v32_b.copy()).cuda()
        count = torch.from_numpy(n_b.copy()).cuda()
        st = m.lib.tc_merge_means_noalloc(src.data_ptr(), m.TC_BF16, target.data_ptr(), src.shape[0], cfg.d,
                                          mean.data_ptr(), count.data_ptr(), M0,
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == m.TC_OK
        torch.cuda.synchronize()
        assert np.array_equal(count.cpu().numpy(), n_a[:M0])
        assert np.abs(mean.cpu().numpy() - v32_a[:M0]).max() <= 1e-3


def test_noalloc_merge_rejects_sizes_beyond_its_scratch():
    import kv_cache_attention_tempcache_b200 as m

    buf = torch.zeros(16, dtype=torch.float32, device="cuda")
    p = buf.data_ptr()
    assert m.lib.tc_merge_means_noalloc(p, m.TC_F32, p, 65537, 128, p, p, 10, None) == m.TC_EINVAL
    assert m.lib.tc_merge_means_noalloc(p, m.TC_F32, p, 10, 128, p, p, 262145, None) == m.TC_EINVAL


def _expected(src, target, mean, count):
    """Sequential fp32 reference: sources summed in ascending index, then the mean update."""
    mean = mean.copy()
    count = count.copy()
    for j in np.unique(target[(target >= 0) & (target < mean.shape[0])]):
        ids = np.nonzero(target == j)[0]
        acc = np.zeros(mean.shape[1], np.float32)
        for i in ids:
            acc = (acc + src[i].astype(np.float32)).astype(np.float32)
        n = np.float32(count[j])
        ft = np.float32(count[j] + ids.size)
        if count[j] == 0:
            mean[j] = (acc / ft).astype(np.float32)
        else:
            mean[j] = (((n * mean[j]).astype(np.float32) + acc).astype(np.float32) / ft).astype(np.float32)
        count[j] += ids.size
    return mean, count


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 128), ("f32", 128)])
def test_noalloc_merge_long_groups_in_source_order(dtype, d):
    # one destination gets > 256 sources (scan path), one > 32 (shared-memory order),
    # the rest small groups; a destination with count 0 holds NaN that must not leak
    import kv_cache_attention_tempcache_b200 as m

    rng = np.random.default_rng(7 + d)
    n_src, n_dst = 3000, 400
    target = rng.integers(-1, n_dst, n_src).astype(np.int32)
    target[rng.choice(n_src, 700, replace=False)] = 5      # > 256 sources
    target[rng.choice(np.nonzero(target != 5)[0], 100, replace=False)] = 17   # > 32 sources
    src32 = rng.standard_normal((n_src, d)).astype(np.float32)
    if dtype == "bf16":
        src_t = torch.from_numpy(src32).to(torch.bfloat16)
        src_np = src_t.float().numpy()
        code = m.TC_BF16
    else:
        src_t = torch.from_numpy(src32)
        src_np = src32
        code = m.TC_F32
    mean0 = rng.standard_normal((n_dst, d)).astype(np.float32)
    count0 = rng.integers(0, 9, n_dst).astype(np.int32)
    count0[17] = 0
    mean0[17] = np.nan
    exp_mean, exp_count = _expected(src_np, target, mean0, count0)
    src_d = src_t.cuda()
    tgt_d = torch.from_numpy(target).cuda()
    for _ in range(2):   # two calls in a row on fresh copies
        mean = torch.from_numpy(mean0.copy()).cuda()
        count = torch.from_numpy(count0.copy()).cuda()
        st = m.lib.tc_merge_means_noalloc(src_d.data_ptr(), code, tgt_d.data_ptr(), n_src, d, mean.data_ptr(),
                                          count.data_ptr(), n_dst,
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == m.TC_OK
        torch.cuda.synchronize()
        assert np.array_equal(count.cpu().numpy(), exp_count)
        got = mean.cpu().numpy()
        assert np.isfinite(got[17]).all()
        assert np.abs(got - exp_mean).max() <= 1e-3
        assert np.array_equal(got, exp_mean)   # same operations in the same order


def test_noalloc_merge_rejects_overlapping_buffers():
    import kv_cache_attention_tempcache_b200 as m

    buf = torch.zeros(64 * 128, dtype=torch.float32, device="cuda")
    tgt = torch.zeros(16, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(8, dtype=torch.int32, device="cuda")
    p = buf.data_ptr()
    # src rows [0, 16 * 64) overlap mean rows starting at the same address
    assert m.lib.tc_merge_means_noalloc(p, m.TC_F32, tgt.data_ptr(), 16, 64, p, cnt.data_ptr(), 8,
                                        None) == m.TC_EINVAL
    # target overlaps count
    assert m.lib.tc_merge_means_noalloc(p, m.TC_F32, tgt.data_ptr(), 16, 64, p + 16 * 64 * 4, tgt.data_ptr(), 8,
                                        None) == m.TC_EINVAL
