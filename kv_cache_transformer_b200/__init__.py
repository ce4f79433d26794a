"""Python binding of libnc.so, the B200 KV-cache Transformer inference engine.

Argument marshalling only: every step of prefill, decode and fork runs in the
library's CUDA kernels (see include/nc.h for the contract of each call). torch
provides device memory and streams. The functions keep the C names:

    nc_model_create(cfg, blob)                 -> model handle
    nc_kv_create(model, max_batch, max_seq)    -> cache handle
    nc_prefill(model, kv, tokens[B,T], logits_mode, logits, next, noise, stream)
    nc_decode_step(model, kv, tokens[B], positions[B], noise, logits, next, stream)
    nc_kv_fork(src, src_seq, dst, dst_first, n, stream)
    nc_kv_lengths(kv, n) / nc_device_status(model) / nc_last_error()

plus ``Model`` and ``KVCache`` wrappers that own the handles. There is no
fallback: if libnc.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnc.so")

NC_OK, NC_EINVAL, NC_ERANGE, NC_ENOMEM, NC_ECUDA, NC_EUNSUP = 0, 1, 2, 3, 4, 5
NC_DEV_BAD_TOKEN, NC_DEV_BAD_POSITION, NC_DEV_TIMEOUT = 1, 2, 4
NC_F32, NC_BF16 = 0, 1

# every symbol include/nc.h declares
EXPORTS = (
    "nc_model_create", "nc_model_destroy", "nc_device_status", "nc_kv_create", "nc_kv_destroy",
    "nc_kv_lengths", "nc_prefill", "nc_decode_step", "nc_kv_fork", "nc_last_error",
    "nc_profile_enable", "nc_profile_read", "nc_launch_count", "nc_gemm_bf16",
    "nc_attention_prefill_bf16", "nc_attention_decode_workspace_bytes", "nc_attention_decode_bf16",
    "nc_attention_decode_bf16_static", "nc_decode_trace", "nc_kv_set_sampling", "nc_sample_topk",
    "nc_kv_fork_shared", "nc_prefill_extend",
)
NC_EPI_STORE, NC_EPI_RELU2, NC_EPI_RESID, NC_EPI_SOFTCAP = 0, 1, 2, 3
NC_K_GEMM, NC_K_ATTN, NC_K_HEAD, NC_K_MISC, NC_K_STEP, NC_K_COUNT = 0, 1, 2, 3, 4, 5
K_CLASS_NAMES = ("gemm", "attn", "head", "misc", "step")


class NcError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"nc error {code}: {msg}")
        self.code = code


class nc_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("depth", "d_model", "n_head", "n_kv_head", "head_dim", "mlp_hidden", "vocab")] + \
               [(n, ctypes.c_float) for n in ("rope_base", "softcap", "norm_eps")] + [("dtype", ctypes.c_int)]


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load libnc.so (raises if it is not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is not built: run `python -m kv_cache_transformer_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            L.nc_model_create.argtypes = [ctypes.POINTER(nc_config), vp, sz, ctypes.POINTER(vp)]
            L.nc_model_destroy.argtypes = [vp]
            L.nc_model_destroy.restype = None
            L.nc_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
            L.nc_kv_create.argtypes = [vp, i, i, ctypes.POINTER(vp)]
            L.nc_kv_destroy.argtypes = [vp]
            L.nc_kv_destroy.restype = None
            L.nc_kv_lengths.argtypes = [vp, i, vp]
            L.nc_prefill.argtypes = [vp, vp, vp, i, i, i, vp, vp, vp, vp]
            L.nc_prefill_extend.argtypes = [vp, vp, vp, i, i, i, vp, vp, vp, vp]
            L.nc_decode_step.argtypes = [vp, vp, vp, vp, i, vp, vp, vp, vp]
            L.nc_kv_fork.argtypes = [vp, i, vp, i, i, vp]
            L.nc_kv_fork_shared.argtypes = [vp, i, vp, i, i, vp]
            L.nc_last_error.restype = ctypes.c_char_p
            L.nc_last_error.argtypes = []
            L.nc_profile_enable.argtypes = [vp, i]
            L.nc_profile_read.argtypes = [vp, vp, vp]
            L.nc_launch_count.argtypes = []
            L.nc_launch_count.restype = ctypes.c_ulonglong
            L.nc_gemm_bf16.argtypes = [vp, i, vp, i, i, i, i, vp, i, ctypes.c_float, vp]
            L.nc_attention_prefill_bf16.argtypes = [vp, vp, vp, i, i, i, i, i, vp, vp]
            L.nc_attention_decode_workspace_bytes.argtypes = [i, i]
            L.nc_attention_decode_workspace_bytes.restype = ctypes.c_size_t
            L.nc_attention_decode_bf16.argtypes = [vp, vp, vp, vp, i, i, i, vp, vp, sz, vp]
            L.nc_attention_decode_bf16_static.argtypes = [vp, vp, vp, vp, i, i, i, vp, vp]
            L.nc_decode_trace.argtypes = [vp, vp, sz, ctypes.POINTER(i), ctypes.POINTER(i)]
            L.nc_kv_set_sampling.argtypes = [vp, ctypes.c_float, i]
            L.nc_sample_topk.argtypes = [vp, i, i, ctypes.c_longlong, vp, ctypes.c_float, i, vp, vp]
            for name in EXPORTS:
                if name not in ("nc_model_destroy", "nc_kv_destroy", "nc_last_error", "nc_launch_count",
                                "nc_attention_decode_workspace_bytes"):
                    getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def nc_last_error() -> str:
    return lib().nc_last_error().decode()


def _check(rc: int):
    if rc != NC_OK:
        raise NcError(rc, nc_last_error())


def _dptr(t, dtype=None, numel=None, name="tensor"):
    """Device pointer of a CUDA torch tensor (or None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs {numel}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def make_config(cfg) -> nc_config:
    """nc_config from any object with the nc_config field names (dtype 'f32'/'bf16' or 0/1)."""
    dt = cfg.dtype
    if isinstance(dt, str):
        dt = NC_F32 if dt == "f32" else NC_BF16
    return nc_config(cfg.depth, cfg.d_model, cfg.n_head, cfg.n_kv_head, cfg.head_dim, cfg.mlp_hidden, cfg.vocab,
                     float(cfg.rope_base), float(cfg.softcap), float(cfg.norm_eps), int(dt))


# ------------------------------------------------------------------ C names
def nc_model_create(cfg, blob: np.ndarray) -> ctypes.c_void_p:
    c = make_config(cfg)
    blob = np.ascontiguousarray(blob)
    h = ctypes.c_void_p()
    _check(lib().nc_model_create(ctypes.byref(c), ctypes.c_void_p(blob.ctypes.data), blob.nbytes, ctypes.byref(h)))
    return h


def nc_model_destroy(h):
    lib().nc_model_destroy(h)


def nc_device_status(h) -> int:
    v = ctypes.c_uint32()
    _check(lib().nc_device_status(h, ctypes.byref(v)))
    return int(v.value)


def nc_kv_create(model_h, max_batch: int, max_seq: int) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib().nc_kv_create(model_h, int(max_batch), int(max_seq), ctypes.byref(h)))
    return h


def nc_kv_destroy(h):
    lib().nc_kv_destroy(h)


def nc_kv_lengths(kv_h, n: int) -> np.ndarray:
    out = np.zeros(n, dtype=np.int32)
    _check(lib().nc_kv_lengths(kv_h, int(n), ctypes.c_void_p(out.ctypes.data)))
    return out


def nc_prefill(model_h, kv_h, tokens, logits_mode: int = 0, logits=None, next=None, noise=None, stream=None,
               vocab: int | None = None):
    import torch
    B, T = tokens.shape
    V = vocab
    _check(lib().nc_prefill(
        model_h, kv_h, _dptr(tokens, torch.int32, name="tokens"), int(B), int(T), int(logits_mode),
        _dptr(logits, torch.float32, None if V is None else (B * T * V if logits_mode else B * V), "logits"),
        _dptr(next, torch.int32, B, "next"),
        _dptr(noise, torch.float32, None if V is None else B * V, "noise"), _stream(stream)))


def nc_prefill_extend(model_h, kv_h, tokens, logits_mode: int = 0, logits=None, next=None, noise=None, stream=None,
                      vocab: int | None = None):
    import torch
    B, T = tokens.shape
    V = vocab
    _check(lib().nc_prefill_extend(
        model_h, kv_h, _dptr(tokens, torch.int32, name="tokens"), int(B), int(T), int(logits_mode),
        _dptr(logits, torch.float32, None if V is None else (B * T * V if logits_mode else B * V), "logits"),
        _dptr(next, torch.int32, B, "next"),
        _dptr(noise, torch.float32, None if V is None else B * V, "noise"), _stream(stream)))


def nc_decode_step(model_h, kv_h, tokens, positions, noise=None, logits=None, next=None, stream=None,
                   vocab: int | None = None):
    import torch
    B = tokens.numel()
    V = vocab
    _check(lib().nc_decode_step(
        model_h, kv_h, _dptr(tokens, torch.int32, name="tokens"), _dptr(positions, torch.int32, B, "positions"),
        int(B), _dptr(noise, torch.float32, None if V is None else B * V, "noise"),
        _dptr(logits, torch.float32, None if V is None else B * V, "logits"),
        _dptr(next, torch.int32, B, "next"), _stream(stream)))


def nc_kv_fork(src_h, src_seq: int, dst_h, dst_first: int, n: int, stream=None):
    _check(lib().nc_kv_fork(src_h, int(src_seq), dst_h, int(dst_first), int(n), _stream(stream)))


def nc_kv_set_sampling(kv_h, temperature: float = 1.0, top_k: int = 0):
    _check(lib().nc_kv_set_sampling(kv_h, float(temperature), int(top_k)))


def nc_sample_topk(logits, next, noise=None, temperature: float = 1.0, top_k: int = 0, stream=None):
    """next[b] = sampled pick over fp32 CUDA logits [B, V] (rows may be strided: logits.stride(0))."""
    import torch
    B, V = logits.shape
    if logits.dtype != torch.float32 or logits.stride(1) != 1 or not logits.is_cuda:
        raise TypeError("logits must be a CUDA float32 tensor with unit inner stride")
    _check(lib().nc_sample_topk(ctypes.c_void_p(logits.data_ptr()), int(B), int(V), int(logits.stride(0)),
                                _dptr(noise, torch.float32, B * V, "noise"), float(temperature), int(top_k),
                                _dptr(next, torch.int32, B, "next"), _stream(stream)))


def nc_decode_trace(kv_h, buf=None):
    """Point the whole-step decode kernel's phase timestamps at `buf` (a CUDA
    int64 tensor of at least grid * phases * 8 elements), or turn them off
    (buf=None). -> (grid, phases)."""
    import torch
    g, p = ctypes.c_int(), ctypes.c_int()
    ptr = None if buf is None else _dptr(buf, torch.int64, name="trace buffer")
    n = 0 if buf is None else buf.numel()
    _check(lib().nc_decode_trace(kv_h, ptr, n, ctypes.byref(g), ctypes.byref(p)))
    return g.value, p.value


def nc_kv_fork_shared(src_h, src_seq: int, dst_h, dst_first: int, n: int, stream=None):
    _check(lib().nc_kv_fork_shared(src_h, int(src_seq), dst_h, int(dst_first), int(n), _stream(stream)))


def nc_profile_enable(model_h, on: bool = True):
    _check(lib().nc_profile_enable(model_h, 1 if on else 0))


def nc_profile_read(model_h):
    """-> (ms[NC_K_COUNT], launches[NC_K_COUNT]) per kernel class since the last read."""
    ms = np.zeros(NC_K_COUNT, dtype=np.float64)
    n = np.zeros(NC_K_COUNT, dtype=np.int64)
    _check(lib().nc_profile_read(model_h, ctypes.c_void_p(ms.ctypes.data), ctypes.c_void_p(n.ctypes.data)))
    return ms, n


def nc_launch_count() -> int:
    return int(lib().nc_launch_count())


def nc_gemm_bf16(A, W, out, epi: int = NC_EPI_STORE, cap: float = 15.0, stream=None):
    """out (epi) A @ W.T for bf16 CUDA tensors A [M, K] (row pitch A.stride(0)) and W [N, K]."""
    import torch
    M, K = A.shape
    N = W.shape[0]
    if A.dtype != torch.bfloat16 or W.dtype != torch.bfloat16 or A.stride(1) != 1 or not W.is_contiguous():
        raise TypeError("A and W must be bf16 with unit inner stride (W contiguous)")
    if W.shape[1] != K or out.shape[0] < M or out.stride(1) != 1:
        raise ValueError("shape mismatch")
    _check(lib().nc_gemm_bf16(ctypes.c_void_p(A.data_ptr()), A.stride(0), ctypes.c_void_p(W.data_ptr()), M, N, K,
                              int(epi), ctypes.c_void_p(out.data_ptr()), out.stride(0), float(cap), _stream(stream)))


def nc_attention_prefill_bf16(q, k, v, y, stream=None):
    """Causal MQA: q, y bf16 [B, T, H, hd]; k, v bf16 [B, max_seq, hd] (CUDA, contiguous)."""
    import torch
    B, T, H, hd = q.shape
    if k.shape[0] != B or k.shape[2] != hd or k.shape != v.shape or y.shape != q.shape:
        raise ValueError("shape mismatch")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (y, "y")):
        _dptr(t, torch.bfloat16, name=n)
    _check(lib().nc_attention_prefill_bf16(_dptr(q), _dptr(k), _dptr(v), B, T, H, hd, k.shape[1], _dptr(y),
                                           _stream(stream)))


def nc_attention_decode_workspace_bytes(B: int, max_seq: int) -> int:
    return int(lib().nc_attention_decode_workspace_bytes(int(B), int(max_seq)))


def nc_attention_decode_bf16(q, k, v, pos, y, workspace, stream=None):
    """Decode MQA: q, y bf16 [B, H, 128]; k, v bf16 [B, max_seq, 128]; pos int32 [B];
    workspace: a zero-filled CUDA byte tensor of nc_attention_decode_workspace_bytes(B, max_seq)."""
    import torch
    B, H, hd = q.shape
    if hd != 128 or k.shape[0] != B or k.shape[2] != 128 or k.shape != v.shape or y.shape != q.shape:
        raise ValueError("shape mismatch")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (y, "y")):
        _dptr(t, torch.bfloat16, name=n)
    _check(lib().nc_attention_decode_bf16(_dptr(q), _dptr(k), _dptr(v), _dptr(pos, torch.int32, B, "pos"), B, H,
                                          k.shape[1], _dptr(y), _dptr(workspace), workspace.numel() *
                                          workspace.element_size(), _stream(stream)))


def nc_attention_decode_bf16_static(q, k, v, pos, y, stream=None):
    """nc_attention_decode_bf16 using the library's static scratch (no workspace, no allocation)."""
    import torch
    B, H, hd = q.shape
    if hd != 128 or k.shape[0] != B or k.shape[2] != 128 or k.shape != v.shape or y.shape != q.shape:
        raise ValueError("shape mismatch")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (y, "y")):
        _dptr(t, torch.bfloat16, name=n)
    _check(lib().nc_attention_decode_bf16_static(_dptr(q), _dptr(k), _dptr(v), _dptr(pos, torch.int32, B, "pos"), B,
                                                 H, k.shape[1], _dptr(y), _stream(stream)))


# ----------------------------------------------------------------- wrappers
class Model:
    """A model on the current CUDA device (weights copied from a host blob)."""

    def __init__(self, cfg, blob: np.ndarray):
        self.cfg = cfg
        self.vocab = cfg.vocab
        self._h = nc_model_create(cfg, blob)

    def close(self):
        if getattr(self, "_h", None):
            nc_model_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def status(self) -> int:
        return nc_device_status(self._h)

    def profile(self, on: bool = True):
        nc_profile_enable(self._h, on)

    def profile_read(self):
        return nc_profile_read(self._h)

    def kv(self, max_batch: int, max_seq: int) -> "KVCache":
        return KVCache(self, max_batch, max_seq)

    def prefill(self, kv: "KVCache", tokens, logits_mode: int = 0, logits=None, next=None, noise=None, stream=None):
        nc_prefill(self._h, kv.handle, tokens, logits_mode, logits, next, noise, stream, vocab=self.vocab)

    def extend(self, kv: "KVCache", tokens, logits_mode: int = 0, logits=None, next=None, noise=None, stream=None):
        """Append tokens [B, T] to sequences 0..B-1 at their current lengths (nc_prefill_extend)."""
        nc_prefill_extend(self._h, kv.handle, tokens, logits_mode, logits, next, noise, stream, vocab=self.vocab)

    def decode_step(self, kv: "KVCache", tokens, positions, noise=None, logits=None, next=None, stream=None):
        nc_decode_step(self._h, kv.handle, tokens, positions, noise, logits, next, stream, vocab=self.vocab)


class KVCache:
    def __init__(self, model: Model, max_batch: int, max_seq: int):
        self.model = model  # keeps the model alive
        self.max_batch, self.max_seq = max_batch, max_seq
        self._h = nc_kv_create(model.handle, max_batch, max_seq)

    def close(self):
        if getattr(self, "_h", None):
            nc_kv_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def lengths(self, n: int | None = None) -> np.ndarray:
        return nc_kv_lengths(self._h, self.max_batch if n is None else n)

    def fork_to(self, src_seq: int, dst: "KVCache", dst_first: int, n: int, stream=None):
        nc_kv_fork(self._h, src_seq, dst.handle, dst_first, n, stream)

    def fork_shared_to(self, src_seq: int, dst: "KVCache", dst_first: int, n: int, stream=None):
        """Fork sequence src_seq into dst[dst_first:dst_first+n] sharing its prefix rows (nc_kv_fork_shared)."""
        nc_kv_fork_shared(self._h, src_seq, dst.handle, dst_first, n, stream)

    def set_sampling(self, temperature: float = 1.0, top_k: int = 0):
        """Sampled token pick for later prefill/decode calls on this cache (see nc_kv_set_sampling)."""
        nc_kv_set_sampling(self._h, temperature, top_k)

    def trace(self, buf=None):
        """Phase timestamps of later decode steps into `buf` (see nc_decode_trace)."""
        return nc_decode_trace(self._h, buf)
