"""CPU-side checks of the C-ABI library: it builds for sm_100a, loads without a
GPU, exports every symbol include/nc.h declares, and rejects bad arguments on
the host before touching the device."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import kv_cache_transformer_b200 as nc
from kv_cache_transformer_b200 import build as ncbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(nc_\w+)\s*\(", src))
    return names


def test_library_builds_and_exports_every_declared_symbol():
    path = ncbuild.build()
    assert os.path.exists(path)
    declared = _declared()
    assert {"nc_model_create", "nc_prefill", "nc_decode_step", "nc_kv_fork"} <= declared
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (nc_\w+)", out))
    missing = declared - exported
    assert not missing, f"declared but not exported: {missing}"
    assert set(nc.EXPORTS) == declared
    L = nc.lib()
    for name in declared:
        assert getattr(L, name) is not None


def test_no_cpu_fallback_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(nc, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(nc, "_lib", None)
    with pytest.raises(RuntimeError):
        nc.lib()


class Cfg:
    def __init__(self, **kw):
        base = dict(depth=1, d_model=128, n_head=2, n_kv_head=1, head_dim=64, mlp_hidden=256, vocab=64,
                    rope_base=10000.0, softcap=15.0, norm_eps=1e-6, dtype="f32")
        base.update(kw)
        self.__dict__.update(base)


def _blob(c):
    d, qd, kd = c.d_model, c.n_head * c.head_dim, c.n_kv_head * c.head_dim
    n = 2 * c.vocab * d + c.depth * (qd * d + 2 * kd * d + d * qd + 2 * c.mlp_hidden * d)
    return np.zeros(n, dtype=np.float32 if c.dtype == "f32" else np.uint16)


@pytest.mark.parametrize("kw,msg", [
    (dict(head_dim=63, n_head=2, d_model=126), "even"),
    (dict(n_head=3), "n_head * head_dim"),
    (dict(n_kv_head=3, n_head=2, d_model=128), "n_kv_head"),
    (dict(vocab=0), "non-positive"),
    (dict(dtype=7), "dtype"),
])
def test_model_create_rejects_bad_config_on_host(kw, msg):
    c = Cfg(**kw)
    cfg = nc.make_config(c)
    h = ctypes.c_void_p()
    blob = np.zeros(16, np.float32)
    rc = nc.lib().nc_model_create(ctypes.byref(cfg), ctypes.c_void_p(blob.ctypes.data), blob.nbytes,
                                  ctypes.byref(h))
    assert rc == nc.NC_EINVAL
    assert msg in nc.nc_last_error()
    assert not h.value


def test_model_create_rejects_blob_size_mismatch():
    c = Cfg()
    blob = _blob(c)
    with pytest.raises(nc.NcError) as e:
        nc.nc_model_create(c, blob[:-1])
    assert e.value.code == nc.NC_EINVAL and "blob has" in str(e.value)


def test_calls_reject_null_handles():
    L = nc.lib()
    assert L.nc_prefill(None, None, None, 1, 1, 0, None, None, None, None) == nc.NC_EINVAL
    assert L.nc_decode_step(None, None, None, None, 1, None, None, None, None) == nc.NC_EINVAL
    assert L.nc_kv_fork(None, 0, None, 0, 1, None) == nc.NC_EINVAL
    assert L.nc_kv_create(None, 1, 1, ctypes.byref(ctypes.c_void_p())) == nc.NC_EINVAL
    assert L.nc_kv_lengths(None, 1, None) == nc.NC_EINVAL
    assert L.nc_device_status(None, None) == nc.NC_EINVAL
    L.nc_model_destroy(None)
    L.nc_kv_destroy(None)
