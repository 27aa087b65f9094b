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
