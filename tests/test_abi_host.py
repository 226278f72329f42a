"""The C-ABI library loads without a GPU, exports every symbol the header declares, and
rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tri.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tri_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from rope_aware_key_tri_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("tri_create", "tri_destroy", "tri_calibrate_load", "tri_prune", "tri_score",
              "tri_calibrate_estimate", "tri_append", "tri_get_error", "tri_status_str",
              "tri_set_offset_combine", "tri_decode_attention", "tri_get_failed_units", "tri_set_test_fault"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from rope_aware_key_tri_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for n in _declared():
        assert n in exported, n
        assert hasattr(lib, n), n
    # nothing but the C ABI is exported
    assert all(s.startswith("tri_") for s in exported if not s.startswith("_")), \
        sorted(s for s in exported if not s.startswith("tri_"))[:10]


def test_host_validation_without_device(lib):
    from rope_aware_key_tri_b200 import tri
    assert tri.status_str(tri.TRI_EINVAL).startswith("TRI_EINVAL")
    assert tri.tri_version() >= 100
    kv = tri.tri_kv()
    assert lib.tri_prune(None, ctypes.byref(kv), None, 1, None) == tri.TRI_EINVAL
    assert lib.tri_score(None, ctypes.byref(kv), None, None, None, None) == tri.TRI_EINVAL
    assert lib.tri_destroy(None) == tri.TRI_OK
    assert lib.tri_set_tuning(None, 0, 0) == tri.TRI_EINVAL
    assert lib.tri_set_offset_combine(None, tri.TRI_OFFSETS_MAX) == tri.TRI_EINVAL
    assert tri.tri_calibrate_estimate(None, None, 1, 1, 1, 128, 0, None, None, None, None) == tri.TRI_EINVAL
    assert lib.tri_append(None, ctypes.byref(kv), None, None, None, None) == tri.TRI_EINVAL
    assert lib.tri_append_advance(None, ctypes.byref(kv), None, None, None, None) == tri.TRI_EINVAL
    assert lib.tri_calibrate_load(None, 1, 1, 1, 64, ctypes.c_double(1e4), 0, None, None, None, None, 1) \
        == tri.TRI_EINVAL
    code = ctypes.c_int32(7)
    unit = ctypes.c_int64(7)
    assert lib.tri_get_error(None, None, ctypes.byref(code), ctypes.byref(unit)) == tri.TRI_EINVAL
    assert code.value == 0 and unit.value == -1
    assert tri.tri_decode_attention(None, kv, 0, 0, None) == tri.TRI_EINVAL
    n = ctypes.c_int32(5)
    assert lib.tri_get_failed_units(None, None, None, 0, ctypes.byref(n)) == tri.TRI_EINVAL and n.value == 0
    assert lib.tri_set_test_fault(None, -1, 0) == tri.TRI_EINVAL


def test_create_without_gpu_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    st = lib.tri_create(ctypes.byref(h), 0)
    assert st in (3, 1, 6)  # ECUDA (no device), EINVAL or EUNSUPPORTED; never a crash
    assert not h.value
