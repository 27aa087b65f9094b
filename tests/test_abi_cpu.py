"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/tempcache.h declares, and rejects bad arguments before touching
the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tempcache.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tc_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def tcmod():
    import kv_cache_attention_tempcache_b200 as m
    return m


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("tc_create", "tc_append_chunk", "tc_attend", "tc_cache_size", "tc_destroy"):
        assert required in names


def test_library_exports_every_declared_symbol(tcmod):
    lib = ctypes.CDLL(tcmod.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(tcmod.API) == set(declared_functions())


def test_status_strings(tcmod):
    for s in range(9):
        assert tcmod.lib.tc_status_string(s)
    assert tcmod.lib.tc_status_string(99) == b"unknown status"


@pytest.mark.parametrize("args", [
    (0, 128, 16, 0.95, 100),       # H < 1
    (4, 96, 16, 0.95, 100),        # d not 64/128
    (4, 128, 0, 0.95, 100),        # nbits < 1
    (4, 128, 25, 0.95, 100),       # nbits > 24
    (4, 128, 16, -1.5, 100),       # tau < -1
    (4, 128, 16, 2.5, 100),        # tau > 2
    (4, 128, 16, float("nan"), 100),
    (4, 128, 16, 0.95, 0),         # capacity < 1
])
def test_create_rejects_bad_arguments(tcmod, args):
    h = ctypes.c_void_p()
    assert tcmod.lib.tc_create(*args, ctypes.byref(h)) == tcmod.TC_EINVAL
    assert not h.value


def test_create_rejects_non_bf16_hyperplanes(tcmod):
    import numpy as np
    R = np.full(2 * 64, 0.1, dtype=np.float32)  # 0.1 is not a bf16 value
    opt = tcmod.TCOptions()
    opt.dtype = tcmod.TC_BF16
    opt.hyperplanes = R.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
    h = ctypes.c_void_p()
    assert tcmod.lib.tc_create_ex(1, 64, 2, 0.9, 10, ctypes.byref(opt), ctypes.byref(h)) == tcmod.TC_EINVAL


def test_null_handle_is_rejected_everywhere(tcmod):
    L, E = tcmod.lib, tcmod.TC_EINVAL
    buf = (ctypes.c_int64 * 4)()
    assert L.tc_append_chunk(None, None, None, 1, None) == E
    assert L.tc_attend(None, None, 1, None, None) == E
    assert L.tc_flush(None, None) == E
    assert L.tc_reset(None, None) == E
    assert L.tc_cache_size(None, buf) == E
    assert L.tc_sync(None) == E
    assert L.tc_debug_last_commit(None, None, None, None, None) == E
    assert L.tc_debug_staged_codes(None, None, None) == E
    assert L.tc_export_cache(None, 0, None, None, None, None) == E
    assert L.tc_get_hyperplanes(None, None) == E
    assert L.tc_stats(None, None, None, None) == E
    L.tc_destroy(None)  # NULL-safe


def test_create_without_device_reports_it(tcmod):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    st = tcmod.lib.tc_create(2, 128, 16, 0.95, 1000, ctypes.byref(h))
    assert st in (tcmod.TC_EDEVICE, tcmod.TC_ECUDA)
    assert not h.value


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference runs the CPU oracle and prints one JSON line with the
    keys the benchmark contract names (no GPU needed)."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([x for x in out.stdout.splitlines() if x.startswith("{")][-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


@pytest.mark.parametrize("args", [
    (0, 128, 10),      # H < 1
    (4, 96, 10),       # d not 64/128
    (4, 128, 0),       # nbits < 1
    (4, 128, 25),      # nbits > 24
])
def test_annca_create_rejects_bad_arguments(tcmod, args):
    h = ctypes.c_void_p()
    assert tcmod.lib.tc_annca_create(*args, None, ctypes.byref(h)) == tcmod.TC_EINVAL
    assert not h.value


def test_annca_is_bf16_only(tcmod):
    opt = tcmod.TCOptions()
    opt.dtype = tcmod.TC_F32
    h = ctypes.c_void_p()
    assert tcmod.lib.tc_annca_create(4, 128, 10, ctypes.byref(opt), ctypes.byref(h)) == tcmod.TC_ENOTIMPL
    opt.dtype = tcmod.TC_BF16
    opt.intra_chunk = 1   # a TempCache option, meaningless here
    assert tcmod.lib.tc_annca_create(4, 128, 10, ctypes.byref(opt), ctypes.byref(h)) == tcmod.TC_EINVAL


def test_annca_calls_reject_a_null_handle(tcmod):
    lib = tcmod.lib
    assert lib.tc_annca_set_prompt(None, None, None, 1, None) == tcmod.TC_EINVAL
    assert lib.tc_annca_attend(None, None, 1, 1, None, None) == tcmod.TC_EINVAL
    assert lib.tc_annca_kept(None, None, None, None, None, None, None, None) == tcmod.TC_EINVAL
    assert lib.tc_annca_sync(None) == tcmod.TC_EINVAL
    lib.tc_annca_destroy(None)


def test_annsa_rejects_a_null_handle(tcmod):
    assert tcmod.lib.tc_annsa_attend(None, None, None, None, 1, None, None) == tcmod.TC_EINVAL


@pytest.mark.parametrize("args", [
    (0, 128, 1560, 4, 21, 0.0),     # H < 1
    (12, 96, 1560, 4, 21, 0.0),     # d not 64/128
    (12, 128, 0, 4, 21, 0.0),       # P < 1
    (12, 128, 1560, 0, 21, 0.0),    # T_per < 1
    (12, 128, 1560, 4, 0, 0.0),     # C < 1
    (12, 128, 1560, 4, 21, -1.0),   # negative scale
])
def test_lvsa_create_rejects_bad_arguments(tcmod, args):
    h = ctypes.c_void_p()
    assert tcmod.lib.tc_lvsa_create(*args, ctypes.byref(h)) == tcmod.TC_EINVAL
    assert not h.value


def test_lvsa_calls_reject_a_null_handle(tcmod):
    lib = tcmod.lib
    assert lib.tc_lvsa_attend(None, None, None, None, 1, 0, None, None) == tcmod.TC_EINVAL
    assert lib.tc_lvsa_frames(None, None, None, None) == tcmod.TC_EINVAL
    assert lib.tc_lvsa_sync(None) == tcmod.TC_EINVAL
    lib.tc_lvsa_destroy(None)
