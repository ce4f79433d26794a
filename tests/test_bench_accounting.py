"""The roofline figures bench.py reports rest on its algorithmic FLOP and byte
counts. They are re-derived here by hand from the d20 shapes (d = 1280,
10 query heads and 1 KV head of 128, MLP 5120, vocab 65,536, depth 20), and
the reference arm's JSON line is checked on a tiny oracle sample."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

D, H, HD, F, V, L = 1280, 10, 128, 5120, 65536, 20
# per layer: Wq [H*128, d], Wk and Wv [128, d], Wo [d, H*128], Wfc [F, d], Wproj [d, F]
LAYER_PARAMS = (H * HD) * D + 2 * HD * D + D * (H * HD) + F * D + D * F
LINEAR_PARAMS = L * LAYER_PARAMS  # 334,233,600


def test_layer_parameter_count_by_hand():
    assert LAYER_PARAMS == 1_966_080 + 1_638_400 + 2 * 6_553_600
    # with both embeddings this is the d20 parameter count of the one-KV-head model
    assert LINEAR_PARAMS + 2 * V * D == 502_005_760


def test_prefill_flops_d20_8x2048():
    import bench
    import nc_synth as syn
    cfg = syn.D20
    fl = bench.prefill_flops(cfg, 8, 2048)
    M = 8 * 2048
    assert fl["gemm"] == 2 * M * LINEAR_PARAMS                     # 10.95 TFLOP
    assert fl["gemm"] / (4 * L) == pytest.approx(136_902_082_560)  # per GEMM launch, 80 launches
    # causal attention: query t sees t+1 keys; QK^T and PV are 2*128 FLOP each per (head, key)
    causal_pairs = sum(t + 1 for t in range(2048))
    assert fl["attn"] == L * 8 * H * 4 * HD * causal_pairs           # 1.719 TFLOP
    assert fl["head"] == 2 * 8 * D * V                               # last position of each prompt


def test_decode_bytes_d20_32_sequences():
    import bench
    import nc_synth as syn
    cfg = syn.D20
    ctx = 2048 + (128 + 1) / 2.0  # mean context over the 128 timed steps
    by = bench.decode_bytes(cfg, 32, ctx)
    assert by["weights_linear"] == 2 * LINEAR_PARAMS
    assert by["weights_head"] == 2 * V * D
    assert by["kv_read"] == pytest.approx(L * 32 * ctx * 2 * HD * 2)  # K and V rows, bf16
    assert by["kv_write"] == L * 32 * 2 * HD * 2                      # the new K and V rows
    assert by["logits"] == 4 * 32 * V
    assert by["total"] == pytest.approx(1_537_179_648)


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1", "--ref-tokens", "4"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "config"):
        assert k in line, k
    assert line["value"] > 0 and line["unit"] == "tok/s"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
