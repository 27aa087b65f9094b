"""Host tensors through the public API: inputs copied on the package's H2D stream and
outputs read back on its D2H stream, overlapping the kernels of neighbouring calls, give
the same bits as the device-tensor path."""
import pytest
import torch

from synthetic import CONFIGS, Workload

pytestmark = pytest.mark.gpu


def test_host_tensors_match_device_tensors():
    from kv_cache_attention_tempcache_b200 import TempCache

    torch.cuda.set_device(0)
    cfg = CONFIGS["wan1.3b"].replace(H=4, P=1560, F=3, chunks=6, nbits=16, capacity=40_000, seed=4101)
    w = Workload(cfg, device="cuda")
    R = w.hyperplanes().numpy()
    dev = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, hyperplanes=R)
    host = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, hyperplanes=R)
    pairs = []
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        dev.append_chunk(K, V)
        host.append_chunk(K.cpu().pin_memory(), V.cpu().pin_memory())
        for a in range(2):
            Q = w.queries(c, a)
            oh = torch.empty(Q.shape, dtype=Q.dtype).pin_memory()
            pairs.append((dev.attend(Q), host.attend(Q.cpu().pin_memory(), out=oh)))
    host.sync()
    torch.cuda.synchronize()
    for i, (od, oh) in enumerate(pairs):
        assert torch.equal(od.cpu(), oh), i
    assert (dev.cache_size() == host.cache_size()).all()
    dev.close()
    host.close()
