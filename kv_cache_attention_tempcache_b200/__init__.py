"""TempCache on B200: Python binding of the C-ABI library libtempcache.so.

FAST-AR's TempCache (technical summary, section 2.A) compresses the temporal KV
cache of an autoregressive video-diffusion attention layer: new keys are hashed
with sign-of-random-hyperplane LSH, matched top-1 against the cache inside their
bucket, merged into their match above a cosine threshold (values averaged, count n
kept) or appended; attention then runs over the compressed cache plus the current
chunk with a +ln n logit shift per cache entry.

This module only marshals arguments: torch tensors supply device memory and the
current CUDA stream, and every step runs in the library's CUDA kernels. There is
no CPU fallback; without the built library the import fails.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libtempcache.so")

TC_OK, TC_EINVAL, TC_ENOMEM, TC_ECAPACITY, TC_ECUDA, TC_ESTATE, TC_ETIMEOUT, TC_ENOTIMPL, TC_EDEVICE = range(9)
TC_BF16, TC_F32 = 0, 1

API = [
    "tc_create", "tc_create_ex", "tc_append_chunk", "tc_attend", "tc_flush", "tc_reset", "tc_cache_size", "tc_sync",
    "tc_destroy", "tc_status_string", "tc_debug_last_commit", "tc_debug_staged_codes", "tc_export_cache",
    "tc_get_hyperplanes", "tc_stats", "tc_merge_means_noalloc", "tc_export_key_means",
    "tc_annca_create", "tc_annca_set_prompt", "tc_annca_attend", "tc_annca_kept", "tc_annca_get_hyperplanes",
    "tc_annca_sync", "tc_annca_destroy", "tc_annsa_attend",
    "tc_lvsa_create", "tc_lvsa_attend", "tc_lvsa_frames", "tc_lvsa_sync", "tc_lvsa_destroy",
]


class TCOptions(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("seed", ctypes.c_uint64), ("softmax_scale", ctypes.c_float),
                ("hyperplanes", ctypes.POINTER(ctypes.c_float)), ("intra_chunk", ctypes.c_int32),
                ("key_mode", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libtempcache.so is not built ({LIB_PATH}); run "
                          "`python kv_cache_attention_tempcache_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    H = ctypes.c_void_p
    i32, i64, f32, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
    sig = {
        "tc_create": (ctypes.c_int, [i32, i32, i32, f32, i64, ctypes.POINTER(H)]),
        "tc_create_ex": (ctypes.c_int, [i32, i32, i32, f32, i64, ctypes.POINTER(TCOptions), ctypes.POINTER(H)]),
        "tc_append_chunk": (ctypes.c_int, [H, vp, vp, i64, vp]),
        "tc_attend": (ctypes.c_int, [H, vp, i64, vp, vp]),
        "tc_flush": (ctypes.c_int, [H, vp]),
        "tc_reset": (ctypes.c_int, [H, vp]),
        "tc_cache_size": (ctypes.c_int, [H, ctypes.POINTER(i64)]),
        "tc_sync": (ctypes.c_int, [H]),
        "tc_destroy": (None, [H]),
        "tc_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "tc_debug_last_commit": (ctypes.c_int, [H, ctypes.POINTER(i64), vp, vp, vp]),
        "tc_debug_staged_codes": (ctypes.c_int, [H, ctypes.POINTER(i64), vp]),
        "tc_export_cache": (ctypes.c_int, [H, i32, vp, vp, vp, vp]),
        "tc_get_hyperplanes": (ctypes.c_int, [H, vp]),
        "tc_export_key_means": (ctypes.c_int, [H, i32, vp]),
        "tc_stats": (ctypes.c_int, [H, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64),
                                    ctypes.POINTER(ctypes.c_uint64)]),
        "tc_merge_means_noalloc": (ctypes.c_int, [vp, ctypes.c_int, vp, i32, i32, vp, vp, i32, vp]),
        "tc_annca_create": (ctypes.c_int, [i32, i32, i32, ctypes.POINTER(TCOptions), ctypes.POINTER(H)]),
        "tc_annca_set_prompt": (ctypes.c_int, [H, vp, vp, i32, vp]),
        "tc_annca_attend": (ctypes.c_int, [H, vp, i64, i32, vp, vp]),
        "tc_annca_kept": (ctypes.c_int, [H, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i32), vp, vp,
                                          vp, vp]),
        "tc_annca_get_hyperplanes": (ctypes.c_int, [H, vp]),
        "tc_annca_sync": (ctypes.c_int, [H]),
        "tc_annca_destroy": (None, [H]),
        "tc_annsa_attend": (ctypes.c_int, [H, vp, vp, vp, i64, vp, vp]),
        "tc_lvsa_create": (ctypes.c_int, [i32, i32, i32, i32, i32, f32, ctypes.POINTER(H)]),
        "tc_lvsa_attend": (ctypes.c_int, [H, vp, vp, vp, i32, i32, vp, vp]),
        "tc_lvsa_frames": (ctypes.c_int, [H, ctypes.POINTER(i32), vp, vp]),
        "tc_lvsa_sync": (ctypes.c_int, [H]),
        "tc_lvsa_destroy": (None, [H]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class TempCacheError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.tc_status_string(status).decode()} (status {status})")


class CapacityError(TempCacheError):
    pass


def _check(status: int, where: str):
    if status == TC_OK:
        return
    if status == TC_ECAPACITY:
        raise CapacityError(status, where)
    raise TempCacheError(status, where)


def _np_ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class _HostCopies:
    """Side streams for host tensors, one pair per device. A host input is copied on the
    H2D stream and the current stream waits for that copy; a host output is filled on the
    D2H stream once the current stream has produced it. The kernels of one call then
    overlap the transfers of the next (and of the previous call's result). The device
    copies are tied to the streams that use them (record_stream), so the caching allocator
    reuses their memory only after that work."""

    _per_device = {}

    def __init__(self, dev: int):
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)

    @classmethod
    def get(cls) -> "_HostCopies":
        dev = torch.cuda.current_device()
        if dev not in cls._per_device:
            cls._per_device[dev] = cls(dev)
        return cls._per_device[dev]

    def to_device(self, x: torch.Tensor) -> torch.Tensor:
        cur = torch.cuda.current_stream()
        with torch.cuda.stream(self.h2d):
            xd = x.to("cuda", non_blocking=True)
        cur.wait_stream(self.h2d)
        xd.record_stream(cur)
        return xd

    def to_host(self, xd: torch.Tensor, out: torch.Tensor):
        self.d2h.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.d2h):
            out.copy_(xd, non_blocking=True)
        xd.record_stream(self.d2h)

    def join(self):
        cur = torch.cuda.current_stream()
        cur.wait_stream(self.h2d)
        cur.wait_stream(self.d2h)

    def synchronize(self):
        self.h2d.synchronize()
        self.d2h.synchronize()


def host_copy_streams():
    """(H2D stream, D2H stream) that host inputs and outputs of this package use on the
    current device. A caller timing an end-to-end region makes the H2D stream wait for its
    start event so that no copy begins before it."""
    io = _HostCopies.get()
    return io.h2d, io.d2h


def join_host_copies():
    """Make the current stream wait for every host copy issued so far on this device."""
    _HostCopies.get().join()


def _to_device(x: torch.Tensor) -> torch.Tensor:
    return x if x.is_cuda else _HostCopies.get().to_device(x)


def _out_for(Q: torch.Tensor, out: torch.Tensor | None):
    """(device output to compute into, host tensor to fill afterwards or None)."""
    if out is None:
        return torch.empty_like(Q), None
    if out.shape != Q.shape or out.dtype != Q.dtype:
        raise ValueError("out must match Q in shape and dtype")
    if out.is_cuda:
        return out, None
    return torch.empty_like(Q), out


def _finish(out: torch.Tensor, host: torch.Tensor | None) -> torch.Tensor:
    if host is None:
        return out
    _HostCopies.get().to_host(out, host)
    return host


class TempCache:
    """One attention layer's TempCache on the current CUDA device.

    K, V, Q are [T, H, d] torch tensors in the storage dtype (torch.bfloat16 or
    torch.float32). CUDA tensors are used in place. CPU tensors (the end-to-end path;
    pinned memory for asynchronous copies) are copied to the device on a side stream that
    the current stream waits for; a CPU `out` of attend() is filled from a second side
    stream after the kernels, and holds the result once sync() or join_host_copies() and
    the current stream have completed.
    """

    def __init__(self, H: int, d: int, nbits: int, tau: float, capacity: int, dtype: str = "bf16",
                 seed: int = 0, softmax_scale: float = 0.0, hyperplanes=None, intra_chunk: bool = False,
                 key_mode: str = "representative"):
        if key_mode not in ("representative", "mean"):
            raise ValueError("key_mode is 'representative' or 'mean'")
        self.H, self.d, self.nbits = int(H), int(d), int(nbits)
        self.dtype = dtype
        self.key_mode = key_mode
        self.torch_dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        opt = TCOptions()
        opt.dtype = TC_BF16 if dtype == "bf16" else TC_F32
        opt.seed = int(seed)
        opt.softmax_scale = float(softmax_scale)
        opt.intra_chunk = 1 if intra_chunk else 0
        opt.key_mode = 1 if key_mode == "mean" else 0
        self._R = None
        if hyperplanes is not None:
            R = np.ascontiguousarray(np.asarray(hyperplanes, dtype=np.float32).reshape(-1))
            self._R = R
            opt.hyperplanes = R.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        self._h = ctypes.c_void_p()
        _check(lib.tc_create_ex(self.H, self.d, self.nbits, float(tau), int(capacity), ctypes.byref(opt),
                                ctypes.byref(self._h)), "tc_create_ex")
        self._keep = []

    # -- helpers ---------------------------------------------------------------
    def _dev(self, x: torch.Tensor, name: str) -> torch.Tensor:
        if x.dtype != self.torch_dtype:
            raise TypeError(f"{name} must be {self.torch_dtype}, got {x.dtype}")
        if x.dim() != 3 or x.shape[1] != self.H or x.shape[2] != self.d:
            raise ValueError(f"{name} must be [T, {self.H}, {self.d}], got {tuple(x.shape)}")
        return _to_device(x.contiguous())

    @staticmethod
    def _stream():
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    @property
    def handle(self):
        return self._h

    # -- verbs -----------------------------------------------------------------
    def append_chunk(self, K: torch.Tensor, V: torch.Tensor):
        K = self._dev(K, "K")
        V = self._dev(V, "V")
        if K.shape != V.shape:
            raise ValueError("K and V shapes differ")
        self._keep = [K, V]  # the kernels read them asynchronously on the stream
        _check(lib.tc_append_chunk(self._h, K.data_ptr(), V.data_ptr(), K.shape[0], self._stream()),
               "tc_append_chunk")

    def attend(self, Q: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        Q = self._dev(Q, "Q")
        out, host = _out_for(Q, out)
        _check(lib.tc_attend(self._h, Q.data_ptr(), Q.shape[0], out.data_ptr(), self._stream()), "tc_attend")
        return _finish(out, host)

    def flush(self):
        _check(lib.tc_flush(self._h, self._stream()), "tc_flush")

    def reset(self):
        """Empty the cache (new rollout); allocations are kept."""
        _check(lib.tc_reset(self._h, self._stream()), "tc_reset")

    def sync(self):
        _check(lib.tc_sync(self._h), "tc_sync")
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            _HostCopies.get().synchronize()

    def join_host_copies(self):
        join_host_copies()

    def cache_size(self) -> np.ndarray:
        out = np.zeros(self.H, dtype=np.int64)
        _check(lib.tc_cache_size(self._h, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))), "tc_cache_size")
        return out

    def last_commit(self):
        """(codes, match, dest) of the last committed chunk as [H, T] arrays."""
        T = ctypes.c_int64()
        _check(lib.tc_debug_last_commit(self._h, ctypes.byref(T), None, None, None), "tc_debug_last_commit")
        n = T.value
        codes = np.zeros((self.H, n), np.uint32)
        match = np.zeros((self.H, n), np.int32)
        dest = np.zeros((self.H, n), np.int32)
        if n:
            _check(lib.tc_debug_last_commit(self._h, ctypes.byref(T), _np_ptr(codes), _np_ptr(match),
                                            _np_ptr(dest)), "tc_debug_last_commit")
        return codes, match, dest

    def staged_codes(self) -> np.ndarray:
        T = ctypes.c_int64()
        _check(lib.tc_debug_staged_codes(self._h, ctypes.byref(T), None), "tc_debug_staged_codes")
        codes = np.zeros((self.H, T.value), np.uint32)
        if T.value:
            _check(lib.tc_debug_staged_codes(self._h, ctypes.byref(T), _np_ptr(codes)), "tc_debug_staged_codes")
        return codes

    def export_cache(self, head: int):
        """(K [M,d] as fp32, V32 [M,d], n [M], code [M]) of one head's committed entries.
        With running-mean keys K holds the fp32 key means."""
        M = int(self.cache_size()[head])
        K = np.zeros((M, self.d), np.uint16 if self.dtype == "bf16" else np.float32)
        V = np.zeros((M, self.d), np.float32)
        n = np.zeros(M, np.int32)
        code = np.zeros(M, np.uint32)
        _check(lib.tc_export_cache(self._h, head, _np_ptr(K), _np_ptr(V), _np_ptr(n), _np_ptr(code)),
               "tc_export_cache")
        if self.dtype == "bf16":
            K = (K.astype(np.uint32) << 16).view(np.float32)
        if self.key_mode == "mean":
            K = np.zeros((M, self.d), np.float32)
            _check(lib.tc_export_key_means(self._h, head, _np_ptr(K)), "tc_export_key_means")
        return K, V, n, code

    def hyperplanes(self) -> np.ndarray:
        R = np.zeros((self.nbits, self.d), np.float32)
        _check(lib.tc_get_hyperplanes(self._h, _np_ptr(R)), "tc_get_hyperplanes")
        return R

    def stats(self):
        a, b, c = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
        _check(lib.tc_stats(self._h, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)), "tc_stats")
        return {"kernel_launches": a.value, "hash_rechecks": b.value, "match_rechecks": c.value}

    def launch_count(self) -> int:
        a = ctypes.c_uint64()
        _check(lib.tc_stats(self._h, ctypes.byref(a), None, None), "tc_stats")
        return a.value

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib.tc_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class AnnCA:
    """AnnCA cross-attention of one layer on the current CUDA device (bf16).

    FAST-AR summary, section 2.B: for every frame of a query block, only the prompt
    tokens that share a hash bucket with one of the frame's queries take part in the
    frame's cross-attention. Kp, Vp are [L, H, d] and Q is [F*P, H, d] torch.bfloat16
    tensors; CPU tensors are copied to the device on the current stream first.
    """

    def __init__(self, H: int, d: int, nbits: int, seed: int = 0, softmax_scale: float = 0.0, hyperplanes=None):
        self.H, self.d, self.nbits = int(H), int(d), int(nbits)
        opt = TCOptions()
        opt.dtype = TC_BF16
        opt.seed = int(seed)
        opt.softmax_scale = float(softmax_scale)
        opt.intra_chunk = 0
        self._R = None
        if hyperplanes is not None:
            self._R = np.ascontiguousarray(np.asarray(hyperplanes, dtype=np.float32).reshape(-1))
            opt.hyperplanes = self._R.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        self._h = ctypes.c_void_p()
        _check(lib.tc_annca_create(self.H, self.d, self.nbits, ctypes.byref(opt), ctypes.byref(self._h)),
               "tc_annca_create")
        self._keep = []

    def _dev(self, x: torch.Tensor, name: str) -> torch.Tensor:
        if x.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be torch.bfloat16, got {x.dtype}")
        if x.dim() != 3 or x.shape[1] != self.H or x.shape[2] != self.d:
            raise ValueError(f"{name} must be [n, {self.H}, {self.d}], got {tuple(x.shape)}")
        return _to_device(x.contiguous())

    def set_prompt(self, Kp: torch.Tensor, Vp: torch.Tensor):
        Kp = self._dev(Kp, "Kp")
        Vp = self._dev(Vp, "Vp")
        if Kp.shape != Vp.shape:
            raise ValueError("Kp and Vp shapes differ")
        self._keep = [Kp, Vp]
        _check(lib.tc_annca_set_prompt(self._h, Kp.data_ptr(), Vp.data_ptr(), Kp.shape[0], TempCache._stream()),
               "tc_annca_set_prompt")

    def attend(self, Q: torch.Tensor, P: int, out: torch.Tensor | None = None) -> torch.Tensor:
        Q = self._dev(Q, "Q")
        out, host = _out_for(Q, out)
        _check(lib.tc_annca_attend(self._h, Q.data_ptr(), Q.shape[0], int(P), out.data_ptr(), TempCache._stream()),
               "tc_annca_attend")
        return _finish(out, host)

    def kept(self):
        """Inspection of the last attend: (keep [H, F, L] bool, query codes [H, T], prompt codes [H, L])."""
        T, F, L = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
        _check(lib.tc_annca_kept(self._h, ctypes.byref(T), ctypes.byref(F), ctypes.byref(L), None, None, None, None),
               "tc_annca_kept")
        T, F, L = T.value, F.value, L.value
        counts = np.zeros(self.H * F, np.int32)
        index = np.zeros(self.H * F * L, np.int32)
        qcodes = np.zeros((self.H, T), np.uint32)
        pcodes = np.zeros((self.H, L), np.uint32)
        _check(lib.tc_annca_kept(self._h, None, None, None, _np_ptr(counts), _np_ptr(index), _np_ptr(qcodes),
                                 _np_ptr(pcodes)), "tc_annca_kept")
        keep = np.zeros((self.H, F, L), bool)
        for z in range(self.H * F):
            ids = index[z * L: z * L + counts[z]]
            if counts[z] > 1 and not np.all(np.diff(ids) > 0):
                raise TempCacheError(TC_ESTATE, "tc_annca_kept: kept list not ascending")
            keep[z // F, z % F, ids] = True
        return keep, qcodes, pcodes

    def self_attend(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                    out: torch.Tensor | None = None) -> torch.Tensor:
        """AnnSA (FAST-AR summary, section 2.C): self-attention of the block the last
        attend() pruned, each token seeing only the tokens of its own AnnCA bucket."""
        Q = self._dev(Q, "Q")
        K = self._dev(K, "K")
        V = self._dev(V, "V")
        if not (Q.shape == K.shape == V.shape):
            raise ValueError("Q, K and V shapes differ")
        out, host = _out_for(Q, out)
        self._keep_sa = [Q, K, V]
        _check(lib.tc_annsa_attend(self._h, Q.data_ptr(), K.data_ptr(), V.data_ptr(), Q.shape[0], out.data_ptr(),
                                   TempCache._stream()), "tc_annsa_attend")
        return _finish(out, host)

    def hyperplanes(self) -> np.ndarray:
        R = np.zeros((self.nbits, self.d), np.float32)
        _check(lib.tc_annca_get_hyperplanes(self._h, _np_ptr(R)), "tc_annca_get_hyperplanes")
        return R

    def sync(self):
        _check(lib.tc_annca_sync(self._h), "tc_annca_sync")
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            _HostCopies.get().synchronize()

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib.tc_annca_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class LVSA:
    """LVSA frame-masked attention (LVSA summary, section 2): query frame t attends only to
    the rotating global frames of the step and a local window around t extended to C
    frames in all. Q, K, V are [T*P, H, d] torch.bfloat16 tensors."""

    def __init__(self, H: int, d: int, P: int, T_per: int, C: int, softmax_scale: float = 0.0):
        self.H, self.d, self.P = int(H), int(d), int(P)
        self._h = ctypes.c_void_p()
        _check(lib.tc_lvsa_create(self.H, self.d, self.P, int(T_per), int(C), float(softmax_scale),
                                  ctypes.byref(self._h)), "tc_lvsa_create")

    def attend(self, Q, K, V, step: int, out=None):
        t = []
        for x, name in ((Q, "Q"), (K, "K"), (V, "V")):
            if x.dtype != torch.bfloat16 or x.dim() != 3 or x.shape[1] != self.H or x.shape[2] != self.d:
                raise ValueError(f"{name} must be [T*P, {self.H}, {self.d}] bfloat16")
            t.append(_to_device(x.contiguous()))
        Q, K, V = t
        if Q.shape[0] % self.P:
            raise ValueError("Q must hold whole frames")
        out, host = _out_for(Q, out)
        self._keep = [Q, K, V]
        _check(lib.tc_lvsa_attend(self._h, Q.data_ptr(), K.data_ptr(), V.data_ptr(), Q.shape[0] // self.P,
                                  int(step), out.data_ptr(), TempCache._stream()), "tc_lvsa_attend")
        return _finish(out, host)

    def frames(self):
        """A(t) of the last call, as a list of arrays."""
        T = ctypes.c_int32()
        _check(lib.tc_lvsa_frames(self._h, ctypes.byref(T), None, None), "tc_lvsa_frames")
        T = T.value
        n = np.zeros(T, np.int32)
        f = np.zeros(T * T, np.int32)
        if T:
            _check(lib.tc_lvsa_frames(self._h, None, _np_ptr(n), _np_ptr(f)), "tc_lvsa_frames")
        return [f[t * T: t * T + n[t]].copy() for t in range(T)]

    def sync(self):
        _check(lib.tc_lvsa_sync(self._h), "tc_lvsa_sync")
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            _HostCopies.get().synchronize()

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib.tc_lvsa_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
