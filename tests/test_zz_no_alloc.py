"""The allocation-free decode attention entry point.

nc_attention_decode_bf16_static exists for callers that cannot allocate
device memory themselves: a serving runtime whose allocator owns all of it, a
plugin host that offers no workspace hook, a deployment with a fixed device
footprint. It keeps its scratch in a static array inside the library instead
of a caller workspace. This test calls it through the C ABI and checks that
its output matches the workspace entry point (nc_attention_decode_bf16) on
the same inputs, for two calls in a row: the array keeps the previous call's
contents, and the second call must not be affected by them. It also checks
the size limit. The file sorts last so that a run stopping at the first
failure has already run every other test; it needs no state from them.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _inputs(seed, B, H, max_seq):
    import torch
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, max_seq, 128, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, max_seq, 128, generator=g).to(torch.bfloat16).cuda()
    pos = torch.randint(0, max_seq, (B,), generator=g, dtype=torch.int32)
    pos[0] = max_seq - 1
    return q, k, v, pos.cuda()


def test_static_scratch_decode_attention_matches_workspace_entry_point():
    import torch
    import kv_cache_transformer_b200 as nc
    for call, (B, H, max_seq) in enumerate([(32, 10, 2176), (7, 13, 900)]):
        q, k, v, pos = _inputs(100 + call, B, H, max_seq)
        ws = torch.zeros(nc.nc_attention_decode_workspace_bytes(B, max_seq), dtype=torch.uint8, device="cuda")
        y_ws = torch.full((B, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        y_st = torch.full((B, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        nc.nc_attention_decode_bf16(q, k, v, pos, y_ws, ws)
        nc.nc_attention_decode_bf16_static(q, k, v, pos, y_st)
        torch.cuda.synchronize()
        a = y_ws.cpu().double().numpy()
        b = y_st.cpu().double().numpy()
        assert np.all(np.isfinite(b)), f"call {call}: non-finite output"
        err = np.abs(a - b)
        assert np.all(err <= 1e-2 + 2.0 ** -8 * np.abs(a)), f"call {call}: max diff {err.max():.3g}"


def test_static_scratch_rejects_sizes_beyond_its_limit():
    import torch
    import kv_cache_transformer_b200 as nc
    q, k, v, pos = _inputs(7, 33, 4, 64)
    y = torch.empty((33, 4, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nc.NcError) as e:
        nc.nc_attention_decode_bf16_static(q, k, v, pos, y)
    assert e.value.code == nc.NC_EINVAL and "static scratch limit" in str(e.value)
