"""CPU oracle for the nanochat-style KV-cache Engine forward pass.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg are the only callers. The CUDA engine never imports,
links or executes anything here, and this package imports nothing from it.

The arithmetic lives in ``nc_oracle.c`` (plain C, double precision, OpenMP
over independent outputs), compiled with gcc into ``libnc_oracle.so``. This
module is argument marshalling only.

Parity status: every function is pinned by ``tests/test_oracle_pins.py``
(closed forms, invariants, brute force and the pages' own figures). The
model as a whole has no printed worked example on the pages (no weights, no
logits), so end-to-end agreement with nanochat's trained model is unpinned;
what is pinned is agreement with the feature list's definitions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nc_oracle.c")
_LIB = os.path.join(_HERE, "libnc_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile nc_oracle.c into libnc_oracle.so with gcc (-O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("depth", "d_model", "n_head", "n_kv_head", "head_dim", "mlp_hidden", "vocab")] + \
               [(n, ctypes.c_double) for n in ("rope_base", "softcap", "norm_eps")] + \
               [("dtype", ctypes.c_int)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            vp, ip, dp, i32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_int
            L.orc_model_create.restype = vp
            L.orc_model_create.argtypes = [ctypes.POINTER(_Cfg), vp]
            L.orc_model_destroy.argtypes = [vp]
            L.orc_model_num_params.restype = ctypes.c_size_t
            L.orc_model_num_params.argtypes = [vp]
            L.orc_seq_create.restype = vp
            L.orc_seq_create.argtypes = [vp, ip]
            L.orc_seq_destroy.argtypes = [vp]
            L.orc_seq_len.restype = ip
            L.orc_seq_len.argtypes = [vp]
            L.orc_seq_copy.restype = ip
            L.orc_seq_copy.argtypes = [vp, vp, vp]
            L.orc_step.restype = ip
            L.orc_step.argtypes = [vp, vp, ip, ip, vp]
            L.orc_forward_full.restype = ip
            L.orc_forward_full.argtypes = [vp, vp, ip, ip, ip, vp, vp]
            L.orc_rmsnorm.argtypes = [vp, ip, dp, vp]
            L.orc_rope.argtypes = [vp, ip, dp, dp]
            L.orc_softcap.restype = dp
            L.orc_softcap.argtypes = [dp, dp]
            L.orc_attend.argtypes = [vp, vp, vp, ip, ip, ip, vp]
            L.orc_argmax.restype = i32
            L.orc_argmax.argtypes = [vp, vp, ip]
            L.orc_num_threads.restype = ip
            L.orc_sample_topk.restype = i32
            L.orc_sample_topk.argtypes = [vp, vp, ip, ctypes.c_float, ip]
            L.orc_set_threads.argtypes = [ip]
            L.orc_set_threads.restype = None
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    return int(lib().orc_num_threads())


def sample_topk(z, g=None, temperature: float = 1.0, top_k: int = 0) -> int:
    """Sampled pick over fp32 logits z [n]: argmax over the top_k largest z of
    fl(fl(z / temperature) + g) (g fp32 Gumbel noise or None), lowest index on
    ties; temperature 0 is argmax z. See orc_sample_topk in nc_oracle.c."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    gg = None if g is None else np.ascontiguousarray(g, dtype=np.float32)
    return int(lib().orc_sample_topk(_p(z), None if gg is None else _p(gg), z.size, float(temperature), int(top_k)))


def set_threads(n: int) -> None:
    """Threads of the oracle's parallel loops (results do not depend on it)."""
    lib().orc_set_threads(int(n))


# ---------------------------------------------------------------- primitives
def rmsnorm(x, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    lib().orc_rmsnorm(_p(x), x.size, eps, _p(y))
    return y


def rope(v, pos: float, base: float) -> np.ndarray:
    v = np.array(v, dtype=np.float64, copy=True)
    lib().orc_rope(_p(v), v.size, float(pos), float(base))
    return v


def softcap(z: float, cap: float) -> float:
    return float(lib().orc_softcap(float(z), float(cap)))


def attend(q, K, V) -> np.ndarray:
    """One head: q [hd], K/V [n, hd] -> y [hd]."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    n, hd = K.shape
    y = np.empty(hd, dtype=np.float64)
    lib().orc_attend(_p(q), _p(K), _p(V), n, hd, hd, _p(y))
    return y


def argmax(v, g=None) -> int:
    v = np.ascontiguousarray(v, dtype=np.float64)
    gp = None
    if g is not None:
        g = np.ascontiguousarray(g, dtype=np.float32)
        gp = _p(g)
    return int(lib().orc_argmax(_p(v), gp, v.size))


# ----------------------------------------------------------------- the model
class OracleModel:
    """The oracle's model over a caller-held weight blob (kept alive here)."""

    def __init__(self, cfg, blob: np.ndarray):
        self.cfg = cfg
        self.blob = np.ascontiguousarray(blob)
        c = _Cfg(cfg.depth, cfg.d_model, cfg.n_head, cfg.n_kv_head, cfg.head_dim, cfg.mlp_hidden,
                 cfg.vocab, cfg.rope_base, cfg.softcap, cfg.norm_eps, 0 if cfg.dtype == "f32" else 1)
        want = np.float32 if cfg.dtype == "f32" else np.uint16
        if self.blob.dtype != want:
            raise TypeError(f"blob dtype {self.blob.dtype} does not match config dtype {cfg.dtype}")
        self._h = lib().orc_model_create(ctypes.byref(c), _p(self.blob))
        if not self._h:
            raise ValueError("orc_model_create rejected the config")
        if int(lib().orc_model_num_params(self._h)) != self.blob.size:
            lib().orc_model_destroy(self._h)
            self._h = None
            raise ValueError("blob size does not match the config")

    def __del__(self):
        if getattr(self, "_h", None):
            lib().orc_model_destroy(self._h)
            self._h = None

    def new_seq(self, max_seq: int) -> "OracleSeq":
        return OracleSeq(self, max_seq)

    def forward_full(self, tokens, pos0: int = 0, all_positions: bool = True, fill=None) -> np.ndarray:
        tokens = np.ascontiguousarray(tokens, dtype=np.int32)
        T = tokens.size
        V = self.cfg.vocab
        out = np.empty((T, V) if all_positions else (V,), dtype=np.float64)
        rc = lib().orc_forward_full(self._h, _p(tokens), T, pos0, 1 if all_positions else 0, _p(out),
                                    fill._h if fill is not None else None)
        if rc != 0:
            raise ValueError("orc_forward_full failed")
        return out


class OracleSeq:
    """One sequence's KV cache in the oracle."""

    def __init__(self, model: OracleModel, max_seq: int):
        self.model = model
        self._h = lib().orc_seq_create(model._h, max_seq)
        if not self._h:
            raise MemoryError("orc_seq_create")

    def __del__(self):
        if getattr(self, "_h", None):
            lib().orc_seq_destroy(self._h)
            self._h = None

    @property
    def length(self) -> int:
        return int(lib().orc_seq_len(self._h))

    def step(self, token: int, pos: int | None = None) -> np.ndarray:
        """Feed one token (RoPE position defaults to the current length)."""
        if pos is None:
            pos = self.length
        out = np.empty(self.model.cfg.vocab, dtype=np.float64)
        if lib().orc_step(self.model._h, self._h, int(token), int(pos), _p(out)) != 0:
            raise ValueError("orc_step failed (cache full or bad token)")
        return out

    def prefill(self, tokens, all_positions: bool = False) -> np.ndarray:
        """Fill the empty cache with `tokens` (positions 0..T-1) via the layer-major
        forward; returns last-position logits (or all positions)."""
        return self.model.forward_full(tokens, 0, all_positions, fill=self)

    def copy_from(self, other: "OracleSeq"):
        if lib().orc_seq_copy(self.model._h, other._h, self._h) != 0:
            raise ValueError("orc_seq_copy: destination too small")
