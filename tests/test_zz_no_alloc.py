"""The allocation-free decode attention entry point.

nc_attention_decode_bf16_static exists for callers that cannot allocate
device memory themselves: a serving runtime whose allocator owns all of it, a
plugin host that offers no workspace hook, a deployment with a fixed device
footprint. It keeps its scratch in a static array inside the library instead
of a caller workspace. This test calls it through the C ABI, for two calls in
a row per shape (the array keeps the previous call's contents, and a call
must not be affected by them), and checks its output

  - bit for bit against the workspace entry point (nc_attention_decode_bf16):
    both run the same kernel with the same split plan, so any difference
    would come from stale scratch;
  - against a float64 softmax-attention of the same bf16 inputs, within the
    tolerance of the other attention tests.

One shape (one sequence, 8192 cache rows) makes the split planner grow the
key chunk to stay within 16 splits, the array's limit. It also checks the
size limit. The file sorts last so that a run stopping at the first failure
has already run every other test; it needs no state from them.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _inputs(seed, B, H, max_seq):
    import torch
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(B, max_seq, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(B, max_seq, 128, generator=g).to(torch.bfloat16)
    pos = torch.randint(0, max_seq, (B,), generator=g, dtype=torch.int32)
    pos[0] = max_seq - 1
    return q, k, v, pos


def _ref(q, k, v, pos):
    """Single-token attention in float64: softmax(q . k_j / sqrt(128)) over j <= pos."""
    import torch
    out = torch.zeros(q.shape, dtype=torch.float64)
    for b in range(q.shape[0]):
        n = int(pos[b]) + 1
        s = q[b].double() @ k[b, :n].double().T / np.sqrt(128.0)
        out[b] = torch.softmax(s, dim=-1) @ v[b, :n].double()
    return out.numpy()


@pytest.mark.parametrize("B,H,max_seq", [(32, 10, 2176), (7, 13, 900), (1, 15, 8192)])
def test_static_scratch_decode_attention_matches_workspace_entry_point(B, H, max_seq):
    import torch
    import kv_cache_transformer_b200 as nc
    for call in range(2):
        q, k, v, pos = _inputs(100 * B + 7 * call + max_seq, B, H, max_seq)
        qd, kd, vd, pd = q.cuda(), k.cuda(), v.cuda(), pos.cuda()
        ws = torch.zeros(nc.nc_attention_decode_workspace_bytes(B, max_seq), dtype=torch.uint8, device="cuda")
        y_ws = torch.full((B, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        y_st = torch.full((B, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        nc.nc_attention_decode_bf16(qd, kd, vd, pd, y_ws, ws)
        nc.nc_attention_decode_bf16_static(qd, kd, vd, pd, y_st)
        torch.cuda.synchronize()
        assert torch.equal(y_st, y_ws), f"call {call}: static and workspace outputs differ"
        got = y_st.cpu().double().numpy()
        want = _ref(q, k, v, pos)
        assert np.all(np.isfinite(got)), f"call {call}: non-finite output"
        err = np.abs(got - want)
        assert np.all(err <= 1e-2 + 2.0 ** -8 * np.abs(want)), f"call {call}: max err {err.max():.3g}"


def test_static_scratch_rejects_sizes_beyond_its_limit():
    import torch
    import kv_cache_transformer_b200 as nc
    q, k, v, pos = (t.cuda() for t in _inputs(7, 33, 4, 64))
    y = torch.empty((33, 4, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nc.NcError) as e:
        nc.nc_attention_decode_bf16_static(q, k, v, pos, y)
    assert e.value.code == nc.NC_EINVAL and "static scratch limit" in str(e.value)
