"""Kernel-level parity: the tcgen05 GEMM entry point (nc_gemm_bf16) against a
float64 CPU matmul of the same bf16 operands, for every epilogue, ragged and
full-size shapes, on CTA pairs and on the one-CTA kernel; rows outside M must
stay untouched."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _ref(A, W, rows=None):
    import torch
    a = A.cpu().double() if rows is None else A.cpu().double()[rows]
    return a @ W.cpu().double().T


def _apply(epi, acc, prev, cap=15.0):
    import kv_cache_transformer_b200 as nc
    if epi == nc.NC_EPI_STORE:
        return acc
    if epi == nc.NC_EPI_RELU2:
        return np.maximum(acc, 0) ** 2
    if epi == nc.NC_EPI_RESID:
        return prev + acc
    return cap * np.tanh(acc / cap)


def _tol(epi, want, K):
    # bf16 outputs carry one rounding (relative 2^-8); fp32 outputs only the
    # accumulation error of K fp32 partial sums, which grows like sqrt(K)
    if epi in (0, 1):
        return 2.0 ** -8 * np.abs(want) + 1e-4
    return 3e-6 * np.sqrt(K) * (1 + np.abs(want))


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 64),      # one tile, one k-block
    (129, 256, 64),      # one CTA pair: the second CTA holds a single valid row
    (256, 512, 128),     # exactly one 256-row pair tile per column block
    (300, 1536, 1280),   # ragged M, d20 QKV width
    (257, 1920, 1664),   # ragged M and N (d26 QKV), K not a multiple of 128
    (1000, 5120, 1280),  # d20 MLP fc
    (640, 1280, 5120),   # d20 MLP proj (long K)
    (96, 512, 128),      # M < 128: generic kernel
])
@pytest.mark.parametrize("epi", [0, 1, 2, 3])
def test_gemm_bf16_matches_float64(M, N, K, epi):
    import torch
    import kv_cache_transformer_b200 as nc
    g = torch.Generator().manual_seed(M * 7 + N + K + epi)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    out_dtype = torch.bfloat16 if epi in (0, 1) else torch.float32
    pad = 3
    prev = torch.randn(M + pad, N, generator=g).to(out_dtype)
    out = prev.clone().cuda()
    nc.nc_gemm_bf16(A.cuda(), W.cuda(), out, epi)
    torch.cuda.synchronize()
    got = out.cpu().double().numpy()
    acc = _ref(A, W).numpy()
    want = _apply(epi, acc, prev[:M].double().numpy())
    err = np.abs(got[:M] - want)
    assert np.all(err <= _tol(epi, want, K)), f"max err {err.max():.3g}"
    assert torch.equal(out[M:].cpu(), prev[M:]), "rows beyond M were written"


_ONE_CTA_CHECK = r"""
import sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import kv_cache_transformer_b200 as nc
from tests.test_kernels_gpu import _ref, _apply, _tol
bad = []
for M, N, K in [(300, 1536, 1280), (257, 1920, 1664), (640, 1280, 5120)]:
    for epi in (0, 1, 2, 3):
        g = torch.Generator().manual_seed(M + N + K + epi)
        A = torch.randn(M, K, generator=g).to(torch.bfloat16)
        W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
        dt = torch.bfloat16 if epi in (0, 1) else torch.float32
        prev = torch.randn(M, N, generator=g).to(dt)
        out = prev.clone().cuda()
        nc.nc_gemm_bf16(A.cuda(), W.cuda(), out, epi)
        torch.cuda.synchronize()
        want = _apply(epi, _ref(A, W).numpy(), prev.double().numpy())
        if not np.all(np.abs(out.cpu().double().numpy() - want) <= _tol(epi, want, K)):
            bad.append((M, N, K, epi))
print(bad)
sys.exit(1 if bad else 0)
"""


def test_gemm_one_cta_kernel_on_pair_shapes():
    """Shapes of more than 128 rows run on CTA pairs (tcgen05.mma.cta_group::2);
    NC_GEMM_PAIR=0 selects the one-CTA kernel for every shape. Its results on
    the same ragged shapes, in a process of its own."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, NC_GEMM_PAIR="0")
    r = subprocess.run([sys.executable, "-c", _ONE_CTA_CHECK, root], env=env, cwd=root,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr


def test_gemm_bf16_full_size_sampled_rows():
    # d20 prefill MLP fc at full size (M = 8 x 2048): sampled rows only
    import torch
    import kv_cache_transformer_b200 as nc
    M, N, K = 16384, 5120, 1280
    g = torch.Generator().manual_seed(5)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nc.nc_gemm_bf16(A.cuda(), W.cuda(), out, nc.NC_EPI_RELU2)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(M, 96, replace=False))
    rows[-1] = M - 1
    want = np.maximum(_ref(A, W, torch.from_numpy(rows)).numpy(), 0) ** 2
    got = out.cpu()[torch.from_numpy(rows)].double().numpy()
    assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-4)


def _attn_ref(q, k, v, T):
    """Causal MQA in float64: q [B,T,H,hd], k/v [B,S,hd] (first T rows used)."""
    import torch
    qd = q.double().permute(0, 2, 1, 3)                  # B,H,T,hd
    kd, vd = k.double()[:, :T], v.double()[:, :T]        # B,T,hd
    s = torch.einsum("bhtd,bjd->bhtj", qd, kd) / np.sqrt(q.shape[-1])
    mask = torch.ones(T, T, dtype=torch.bool).triu(1)
    s = s.masked_fill(mask, float("-inf"))
    p = torch.softmax(s, dim=-1)
    return torch.einsum("bhtj,bjd->bhtd", p, vd).permute(0, 2, 1, 3)


@pytest.mark.parametrize("B,T,H,hd,extra", [
    (1, 1, 10, 128, 0),      # one position: y = v0
    (2, 130, 10, 128, 6),    # two key tiles, ragged, cache longer than T
    (1, 2048, 10, 128, 0),   # d20 prompt length: 16 key tiles, 160 row tiles
    (2, 300, 13, 128, 20),   # d26 heads: rows per tile span partial positions
    (3, 77, 15, 128, 3),     # d30 heads, last row tile partial
    (2, 50, 2, 64, 0),       # head_dim 64: generic kernel
    (8, 1024, 10, 128, 0),   # 640 row tiles: each CTA of the persistent kernel runs several
])
def test_attention_prefill_matches_float64(B, T, H, hd, extra):
    import torch
    import kv_cache_transformer_b200 as nc
    g = torch.Generator().manual_seed(B * 1000 + T + H)
    S = T + extra
    q = torch.randn(B, T, H, hd, generator=g).to(torch.bfloat16)
    k = torch.randn(B, S, hd, generator=g).to(torch.bfloat16)
    v = torch.randn(B, S, hd, generator=g).to(torch.bfloat16)
    y = torch.full((B, T, H, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    nc.nc_attention_prefill_bf16(q.cuda(), k.cuda(), v.cuda(), y)
    torch.cuda.synchronize()
    want = _attn_ref(q, k, v, T).numpy()
    got = y.cpu().double().numpy()
    err = np.abs(got - want)
    assert np.all(np.isfinite(got))
    assert np.all(err <= 1e-2 + 2.0 ** -8 * np.abs(want)), f"max err {err.max():.3g}"


@pytest.mark.parametrize("B,T,H", [(2, 600, 10), (1, 2048, 4)])
def test_attention_prefill_growing_scores_rescale_the_output(B, T, H):
    """Keys whose norm grows along the sequence push every row's running max
    up tile after tile, so the online softmax rescales its output again and
    again (the random-key cases above rarely need it)."""
    import torch
    import kv_cache_transformer_b200 as nc
    g = torch.Generator().manual_seed(7 * T + H)
    q = torch.randn(B, T, H, 128, generator=g).to(torch.bfloat16)
    ramp = (1.0 + torch.arange(T, dtype=torch.float32) / 48.0).view(1, T, 1)
    k = (torch.randn(B, T, 128, generator=g) * ramp).to(torch.bfloat16)
    v = torch.randn(B, T, 128, generator=g).to(torch.bfloat16)
    y = torch.full((B, T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    nc.nc_attention_prefill_bf16(q.cuda(), k.cuda(), v.cuda(), y)
    torch.cuda.synchronize()
    want = _attn_ref(q, k, v, T).numpy()
    got = y.cpu().double().numpy()
    err = np.abs(got - want)
    assert np.all(np.isfinite(got))
    assert np.all(err <= 1e-2 + 2.0 ** -8 * np.abs(want)), f"max err {err.max():.3g}"


def _decode_ref(q, k, v, pos):
    import torch
    out = torch.zeros(q.shape, dtype=torch.float64)
    for b in range(q.shape[0]):
        n = int(pos[b]) + 1
        s = q[b].double() @ k[b, :n].double().T / np.sqrt(128.0)
        out[b] = torch.softmax(s, dim=-1) @ v[b, :n].double()
    return out


@pytest.mark.parametrize("B,H,max_seq", [(1, 13, 1536), (7, 10, 300), (32, 10, 2176), (5, 15, 64)])
def test_attention_decode_matches_float64(B, H, max_seq):
    import torch
    import kv_cache_transformer_b200 as nc
    g = torch.Generator().manual_seed(B * 31 + H + max_seq)
    q = torch.randn(B, H, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(B, max_seq, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(B, max_seq, 128, generator=g).to(torch.bfloat16)
    pos = torch.randint(0, max_seq, (B,), generator=g, dtype=torch.int32)
    pos[0] = max_seq - 1
    if B > 1:
        pos[1] = 0
    ws = torch.zeros(nc.nc_attention_decode_workspace_bytes(B, max_seq), dtype=torch.uint8, device="cuda")
    y = torch.full((B, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    for _ in range(2):  # the workspace is reusable as the call leaves it
        nc.nc_attention_decode_bf16(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), y, ws)
        torch.cuda.synchronize()
        want = _decode_ref(q, k, v, pos).numpy()
        got = y.cpu().double().numpy()
        err = np.abs(got - want)
        assert np.all(np.isfinite(got))
        assert np.all(err <= 1e-2 + 2.0 ** -8 * np.abs(want)), f"max err {err.max():.3g}"
