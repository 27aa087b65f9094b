"""Drives the CUDA TempCache and the CPU oracle side by side on one seeded workload.

Used by the GPU parity tests and by the smoke check. Inputs come from the shared
generator (synthetic/); expected values come only from oracle/.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

from oracle import OracleTempCache
from synthetic import Workload


def f64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to(torch.float64).cpu().numpy()


@dataclass
class ParityReport:
    commits: int = 0
    tokens: int = 0
    code_mismatch: int = 0
    match_mismatch: int = 0
    dest_mismatch: int = 0
    size_mismatch: int = 0
    key_mismatch: int = 0
    count_mismatch: int = 0
    v32_max_err: float = 0.0
    attn_max_err: float = 0.0
    attn_mean_err: float = 0.0
    attn_checks: int = 0
    merges: int = 0
    sizes: list = field(default_factory=list)
    records: list = field(default_factory=list)   # the oracle's commit records (keep_records=True)


def compare_state(tc, o, rep: ParityReport, heads, oracle_heads):
    """Cache contents of GPU heads `heads` against the oracle, whose head i is GPU head
    oracle_heads[i]."""
    sizes_gpu = tc.cache_size()[list(oracle_heads)]
    sizes_ref = o.cache_size()
    rep.size_mismatch += int((sizes_gpu != sizes_ref).sum())
    for i, h in enumerate(oracle_heads):
        if h not in heads:
            continue
        K, V32, n, code = tc.export_cache(h)
        k_ref, v_ref, n_ref, c_ref = o.export_head(i)
        if K.shape[0] != k_ref.shape[0]:
            rep.key_mismatch += 1
            continue
        rep.key_mismatch += int((K.astype(np.float64) != k_ref).any(axis=1).sum())
        rep.count_mismatch += int((n != n_ref).sum()) + int((code != c_ref).sum())
        if V32.size:
            rep.v32_max_err = max(rep.v32_max_err, float(np.abs(V32.astype(np.float64) - v_ref).max()))


def run_parity(cfg, chunks=None, attends=1, rows=None, state_heads=None, flush=True, device="cuda",
               check_every_state=True, intra_chunk=False, oracle_heads=None, attn_chunks=None, q_scale=1.0,
               key_mode="representative", on_chunk=None, keep_records=False):
    """Run `chunks` chunks through both implementations and collect the differences.

    rows: query rows checked per attend (None = all). oracle_heads: the heads the oracle
    follows (None = all; heads are independent, so the oracle may run a subset while the
    GPU runs every head). state_heads: heads whose cache contents are compared (None =
    every oracle head). attn_chunks: chunk indices whose attention is checked (None =
    all; the GPU attends in every chunk). q_scale: queries multiplied by this factor
    (then rounded to the storage type) to reach large logits. on_chunk(c, tc, o, w, K, V)
    is called after each chunk's attention with that chunk's keys and values.
    """
    from kv_cache_attention_tempcache_b200 import TempCache

    chunks = cfg.chunks if chunks is None else chunks
    oh = list(range(cfg.H)) if oracle_heads is None else list(oracle_heads)
    w = Workload(cfg, device=device)
    R = w.hyperplanes()
    extra = {} if key_mode == "representative" else {"key_mode": key_mode}
    tc = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, dtype=cfg.dtype, hyperplanes=R.numpy(),
                   intra_chunk=intra_chunk, **extra)
    o = OracleTempCache(len(oh), cfg.d, cfg.nbits, cfg.tau, cfg.capacity, R.double().numpy(),
                        intra_chunk=intra_chunk, key_mode=key_mode)
    heads = set(oh if state_heads is None else state_heads)
    rep = ParityReport()
    sum_abs, n_abs = 0.0, 0
    sel = None if rows is None else np.asarray(rows)

    def check_commit(rec):
        if keep_records:
            rep.records.append(rec)
        codes, match, dest = tc.last_commit()
        rep.commits += 1
        rep.tokens += rec.match.size
        rep.merges += int((rec.match >= 0).sum())
        rep.code_mismatch += int((codes[oh] != rec.codes).sum())
        rep.match_mismatch += int((match[oh] != rec.match).sum())
        rep.dest_mismatch += int((dest[oh] != rec.dest).sum())

    for c in range(chunks):
        K, V = w.next_chunk()
        rec = o.append_chunk(f64(K[:, oh]), f64(V[:, oh]))
        tc.append_chunk(K, V)
        rep.code_mismatch += int((tc.staged_codes()[oh] != o.staged[2]).sum())
        if rec is not None:
            check_commit(rec)
            if check_every_state or c == chunks - 1:
                compare_state(tc, o, rep, heads, oh)
            rep.sizes.append(o.cache_size().tolist())
        for a in range(attends):
            Q = w.queries(c, a)
            if q_scale != 1.0:
                Q = (Q.float() * q_scale).to(Q.dtype)
            out = tc.attend(Q)
            if attn_chunks is not None and c not in attn_chunks:
                continue
            ref = o.attend(f64(Q[:, oh]), rows=sel)
            got = out[:, oh] if sel is None else out[torch.as_tensor(sel, device=out.device)][:, oh]
            err = np.abs(f64(got) - ref)
            rep.attn_max_err = max(rep.attn_max_err, float(err.max()))
            sum_abs += float(err.sum())
            n_abs += err.size
            rep.attn_checks += 1
        if on_chunk is not None:
            on_chunk(c, tc, o, w, K, V)
    if flush:
        rec = o.flush()
        tc.flush()
        if rec is not None:
            check_commit(rec)
            compare_state(tc, o, rep, heads, oh)
    rep.attn_mean_err = sum_abs / max(n_abs, 1)
    tc.sync()
    return rep, tc, o
