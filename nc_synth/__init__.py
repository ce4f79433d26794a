"""Seeded synthetic inputs shared by the CUDA engine's tests/bench and the CPU oracle.

This package draws random numbers and lays them out; it computes nothing of
the model itself. It holds:

* ``ModelConfig`` and the five workload presets (tiny fp32 check model; d20,
  d26, d30 bf16 models whose widths follow the single-depth-knob rule
  d_model = 64*depth, head_dim = 128, n_head = d_model/128, mlp_hidden =
  4*d_model -- the nanochat pages say widths are derived from depth but print
  no formula; this is the reading that reproduces their "d20 ~ 560M" count
  for the MHA variant).
* the weight-blob layout (tensor order) and a seeded N(0, 0.02) blob maker;
* Zipf(s=1.1) / uniform token ids and Gumbel noise.

Random numbers come from ``ncgen.c`` (splitmix64, counter-indexed), compiled
on first use with gcc into ``libncsynth.so`` next to this file.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ncgen.c")
_LIB = os.path.join(_HERE, "libncsynth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ncgen.c into libncsynth.so (gcc, OpenMP). Returns the path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _get():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i64, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
            vp = ctypes.c_void_p
            lib.ncg_splitmix64_at.restype = u64
            lib.ncg_splitmix64_at.argtypes = [u64, u64]
            lib.ncg_stream_base.restype = u64
            lib.ncg_stream_base.argtypes = [u64, u64]
            lib.ncg_uniform01.argtypes = [u64, u64, i64, vp]
            lib.ncg_normal.argtypes = [u64, u64, i64, dbl, vp, vp]
            lib.ncg_round_bf16.argtypes = [vp, i64, vp]
            lib.ncg_tokens_uniform.argtypes = [u64, u64, i64, ctypes.c_int, vp]
            lib.ncg_tokens_zipf.restype = ctypes.c_int
            lib.ncg_tokens_zipf.argtypes = [u64, u64, i64, ctypes.c_int, dbl, vp]
            lib.ncg_gumbel.argtypes = [u64, u64, i64, vp]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


# ----------------------------------------------------------------------------
# configs
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class ModelConfig:
    depth: int
    d_model: int
    n_head: int
    n_kv_head: int
    head_dim: int
    mlp_hidden: int
    vocab: int
    rope_base: float = 10000.0
    softcap: float = 15.0
    norm_eps: float = 1e-6
    dtype: str = "bf16"  # "f32" | "bf16": storage type of the weights

    @property
    def np_dtype(self):
        return np.float32 if self.dtype == "f32" else np.uint16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


def depth_config(depth: int, vocab: int = 65536, dtype: str = "bf16", n_kv_head: int = 1) -> ModelConfig:
    d = 64 * depth
    return ModelConfig(depth=depth, d_model=d, n_head=d // 128, n_kv_head=n_kv_head, head_dim=128,
                       mlp_hidden=4 * d, vocab=vocab, dtype=dtype)


TINY = ModelConfig(depth=2, d_model=128, n_head=2, n_kv_head=1, head_dim=64, mlp_hidden=512,
                   vocab=512, dtype="f32")
D20 = depth_config(20)
D26 = depth_config(26)
D30 = depth_config(30)
# d20 with one KV head per query head (multi-head attention): the 560M count
D20_MHA = depth_config(20, n_kv_head=10)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One benchmark/parity workload: a model plus its synthetic request shape."""
    name: str
    model: ModelConfig
    batch: int            # sequences prefilled (before any fork)
    prompt_len: int       # tokens per prompt
    decode_steps: int     # greedy decode steps after the prompt
    token_dist: str       # "uniform" | "zipf"
    weight_seed: int = 0
    token_seed: int = 1
    fork: int = 0         # >0: the prefilled sequence is forked to this many samples
    noise_seed: int = -1  # >=0: Gumbel noise [samples, vocab] per step from this seed


WORKLOADS = {
    "tiny": Workload("tiny", TINY, batch=1, prompt_len=16, decode_steps=16, token_dist="uniform",
                     token_seed=1),
    "d20_prefill": Workload("d20_prefill", D20, batch=8, prompt_len=2048, decode_steps=0,
                            token_dist="zipf", token_seed=1),
    "d20_decode": Workload("d20_decode", D20, batch=32, prompt_len=2048, decode_steps=128,
                           token_dist="zipf", token_seed=2),
    "d26_latency": Workload("d26_latency", D26, batch=1, prompt_len=1024, decode_steps=512,
                            token_dist="zipf", token_seed=3),
    "d30_rollout": Workload("d30_rollout", D30, batch=1, prompt_len=256, decode_steps=256,
                            token_dist="zipf", token_seed=4, fork=16, noise_seed=5),
    # the d20 shapes with multi-head attention (10 KV heads: the 560M model)
    "d20_mha_prefill": Workload("d20_mha_prefill", D20_MHA, batch=8, prompt_len=2048, decode_steps=0,
                                token_dist="zipf", token_seed=1),
    "d20_mha_decode": Workload("d20_mha_decode", D20_MHA, batch=32, prompt_len=2048, decode_steps=128,
                               token_dist="zipf", token_seed=2),
}


# ----------------------------------------------------------------------------
# weight blob
# ----------------------------------------------------------------------------
def tensor_list(cfg: ModelConfig):
    """Blob tensor order: (name, rows, cols), each row-major [out, in].

    wte[V,d]; per layer Wq[H*hd,d], Wk[Hkv*hd,d], Wv[Hkv*hd,d], Wo[d,H*hd],
    Wfc[F,d], Wproj[d,F]; then the untied lm_head Wlm[V,d].
    """
    d, hd = cfg.d_model, cfg.head_dim
    out = [("wte", cfg.vocab, d)]
    for l in range(cfg.depth):
        out += [
            (f"h{l}.wq", cfg.n_head * hd, d),
            (f"h{l}.wk", cfg.n_kv_head * hd, d),
            (f"h{l}.wv", cfg.n_kv_head * hd, d),
            (f"h{l}.wo", d, cfg.n_head * hd),
            (f"h{l}.wfc", cfg.mlp_hidden, d),
            (f"h{l}.wproj", d, cfg.mlp_hidden),
        ]
    out.append(("wlm", cfg.vocab, d))
    return out


def param_count(cfg: ModelConfig) -> int:
    return sum(r * c for _, r, c in tensor_list(cfg))


def tensor_offsets(cfg: ModelConfig):
    """name -> (element offset, rows, cols) inside the flat blob."""
    off, res = 0, {}
    for name, r, c in tensor_list(cfg):
        res[name] = (off, r, c)
        off += r * c
    return res


def make_blob(cfg: ModelConfig, seed: int = 0, std: float = 0.02) -> np.ndarray:
    """Flat weight blob: every tensor i.i.d. N(0, std^2), stream id = its index in
    the blob order. f32 configs give float32; bf16 configs give uint16 bf16 bits
    (round-to-nearest-even of the same fp32 draws)."""
    lib = _get()
    total = param_count(cfg)
    blob = np.empty(total, dtype=cfg.np_dtype)
    off = 0
    for sid, (_, r, c) in enumerate(tensor_list(cfg)):
        n = r * c
        view = blob[off:off + n]
        if cfg.dtype == "f32":
            lib.ncg_normal(seed, sid, n, std, _ptr(view), None)
        else:
            lib.ncg_normal(seed, sid, n, std, None, _ptr(view))
        off += n
    return blob


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 bits, nearest-even (the generator's own rounding)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _get().ncg_round_bf16(_ptr(x), x.size, _ptr(out))
    return out


# ----------------------------------------------------------------------------
# tokens and noise
# ----------------------------------------------------------------------------
def tokens_uniform(seed: int, shape, vocab: int, stream: int = 0) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), dtype=np.int32)
    _get().ncg_tokens_uniform(seed, stream, out.size, vocab, _ptr(out))
    return out.reshape(shape)


def tokens_zipf(seed: int, shape, vocab: int, s: float = 1.1, stream: int = 0) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), dtype=np.int32)
    if _get().ncg_tokens_zipf(seed, stream, out.size, vocab, s, _ptr(out)) != 0:
        raise MemoryError("ncg_tokens_zipf")
    return out.reshape(shape)


def prompt_tokens(w: Workload) -> np.ndarray:
    """[batch, prompt_len] int32 prompt ids for a workload."""
    shape = (w.batch, w.prompt_len)
    if w.token_dist == "zipf":
        return tokens_zipf(w.token_seed, shape, w.model.vocab)
    return tokens_uniform(w.token_seed, shape, w.model.vocab)


def gumbel(seed: int, shape, stream: int = 0) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), dtype=np.float32)
    _get().ncg_gumbel(seed, stream, out.size, _ptr(out))
    return out.reshape(shape)


def uniform01(seed: int, n: int, stream: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _get().ncg_uniform01(seed, stream, n, _ptr(out))
    return out


def splitmix64_at(state: int, i: int) -> int:
    return int(_get().ncg_splitmix64_at(state, i))
