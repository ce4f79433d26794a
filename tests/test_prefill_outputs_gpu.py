"""GPU parity of the outputs around the token pick: every-position logits of
bf16 models (the tcgen05 GEMM with the softcap epilogue), the next token with
additive noise on each of the library's argmax paths, and the tie rule
(lowest index wins) on logits that tie exactly.

Paths covered (nc.h, nc_prefill):
  logits_mode 0, bf16, B <= 32  -> fused final norm + lm_head + softcap + argmax
  logits_mode 1, bf16           -> norm + softcap GEMM over all rows, then the
                                   row argmax kernel
  fp32 model                    -> generic head, then the row argmax kernel
  decode step, bf16             -> the whole-step kernel's head and merge
"""
import numpy as np
import pytest

import nc_synth as syn
import oracle as orc
from nc_harness import Run, check_logits, check_token, tol_for

pytestmark = pytest.mark.gpu

SMALL = syn.ModelConfig(depth=2, d_model=256, n_head=2, n_kv_head=1, head_dim=128, mlp_hidden=512, vocab=1024,
                        dtype="bf16")
_blobs = {}


def blob_for(cfg):
    if cfg not in _blobs:
        _blobs[cfg] = syn.make_blob(cfg, 0)
    return _blobs[cfg]


def first_argmax(z: np.ndarray) -> int:
    """Index of the largest value, the lowest one among equals (the rule nc.h states)."""
    return int(np.flatnonzero(z == z.max())[0])


@pytest.mark.parametrize("cfg,B,T,seqs", [
    (syn.D20, 2, 136, [0, 1]),  # 272 rows: two full 128-row tiles and a partial one
    (syn.D30, 1, 130, [0]),     # 15 heads, d 1920: partial last 256-column tile
])
def test_bf16_all_position_logits_match_oracle(cfg, B, T, seqs):
    prompts = syn.tokens_zipf(41, (B, T), cfg.vocab)
    run = Run(cfg, blob_for(cfg), B, T + 1)
    lg, nxt = run.prefill(prompts, all_logits=True)
    assert run.status() == 0
    om = orc.OracleModel(cfg, blob_for(cfg))
    for b in seqs:
        ref = om.new_seq(T + 1).prefill(prompts[b], all_positions=True)
        check_logits(lg[b], ref, tol_for(cfg), f"seq {b} all positions")
        assert int(nxt[b]) == first_argmax(lg[b, -1]), f"seq {b}: next token is not the argmax of its logits"
        check_token(int(nxt[b]), ref[-1], None, f"seq {b}")


@pytest.mark.parametrize("cfg,B,T,mode", [
    (SMALL, 3, 40, 0),      # fused lm_head + argmax with noise
    (SMALL, 3, 40, 1),      # all-position logits, then the row argmax with noise
    (syn.D20, 2, 24, 0),    # fused path over 512 vocabulary tiles
    (syn.TINY, 2, 17, 0),   # fp32 model: generic head, row argmax
])
def test_prefill_next_token_with_noise(cfg, B, T, mode):
    prompts = syn.tokens_zipf(43, (B, T), cfg.vocab)
    noise = syn.gumbel(5, (B, cfg.vocab), stream=3)
    run = Run(cfg, blob_for(cfg), B, T + 1)
    lg, nxt = run.prefill(prompts, all_logits=bool(mode), noise=noise)
    assert run.status() == 0
    last = lg[:, -1] if mode else lg
    om = orc.OracleModel(cfg, blob_for(cfg))
    for b in range(B):
        # the pick is the argmax of the kernel's own logits + noise, in fp32
        z = (last[b].astype(np.float32) + noise[b].astype(np.float32)).astype(np.float32)
        assert int(nxt[b]) == first_argmax(z), f"seq {b}: token {nxt[b]} != argmax(logits + noise)"
        ref = om.new_seq(T + 1).prefill(prompts[b])
        check_logits(last[b], ref, tol_for(cfg), f"seq {b}")
        check_token(int(nxt[b]), ref, noise[b], f"seq {b} with noise")


def _paired_head_blob(cfg):
    """The model's blob with lm_head rows duplicated in pairs (row 2k+1 = row
    2k), so every logit has an exact twin at the next index."""
    blob = blob_for(cfg).copy()
    off, rows, cols = syn.tensor_offsets(cfg)["wlm"]
    w = blob[off:off + rows * cols].reshape(rows, cols)
    w[1::2] = w[0::2]
    return blob


@pytest.mark.parametrize("cfg", [SMALL, syn.TINY])
def test_exact_ties_pick_the_lowest_index(cfg):
    B, T, steps = 3, 20, 3
    blob = _paired_head_blob(cfg)
    prompts = syn.tokens_zipf(47, (B, T), cfg.vocab)
    # noise tied in the same pairs keeps every tie through the noisy pick
    noise = np.repeat(syn.gumbel(5, (B, cfg.vocab // 2), stream=9), 2, axis=1)

    def check(lg, nxt, nz, what):
        for b in range(B):
            assert np.array_equal(lg[b, 0::2], lg[b, 1::2]), f"{what} seq {b}: twin rows gave different logits"
            z = lg[b] if nz is None else (lg[b].astype(np.float32) + nz[b].astype(np.float32)).astype(np.float32)
            want = first_argmax(z)
            assert want % 2 == 0
            assert int(nxt[b]) == want, f"{what} seq {b}: token {nxt[b]}, the lowest tied index is {want}"

    for mode in (0, 1):
        for nz in (None, noise):
            run = Run(cfg, blob, B, T + steps + 1)
            lg, nxt = run.prefill(prompts, all_logits=bool(mode), noise=nz)
            check(lg[:, -1] if mode else lg, nxt, nz, f"prefill mode {mode} noise {nz is not None}")
            cur = nxt.copy()
            for s in range(steps):
                lg2, n2 = run.decode(cur, np.full(B, T + s, np.int32), nz)
                check(lg2, n2, nz, f"decode step {s} noise {nz is not None}")
                cur = n2
            assert run.status() == 0


@pytest.mark.parametrize("temp,k,pad", [(0.0, 0, 96), (1.0, 0, 96), (1.0, 50, 96), (0.7, 1000, 96), (1.3, 1, 96),
                                         (0.9, 65535, 96), (1.0, 50, 3), (0.7, 1000, 3)])
def test_sample_topk_kernel_matches_oracle(temp, k, pad):
    """nc_sample_topk against the oracle's pick on the same fp32 logits and
    noise: the decision is taken in fp32 on both sides, so it must agree
    exactly; rows carry exact ties, some of them on the top-k cut."""
    import torch
    import kv_cache_transformer_b200 as nc
    B, V = 5, 65536
    rng = np.random.default_rng(int(1000 * temp) + k)
    z = (rng.standard_normal((B, V)) * 3).astype(np.float32)
    z[1, :] = np.float32(1.25)                     # every logit tied
    z[2, 1000:3000] = z[2].max()                   # a block of tied maxima wider than k
    z[3, ::7] = np.float32(0.5)                    # many ties in the middle of the order
    z[4, 5] = np.float32(-0.0)
    z[4, 6] = np.float32(0.0)
    noise = syn.gumbel(17, (B, V), stream=int(10 * temp) + k)
    stride = V + pad                               # rows of a wider logits buffer (pad 3: rows not 16-byte aligned)
    buf = torch.zeros((B, stride), dtype=torch.float32)
    buf[:, :V] = torch.from_numpy(z)
    lg = buf.cuda()[:, :V]
    nxt = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    nc.nc_sample_topk(lg, nxt, torch.from_numpy(noise).cuda(), temp, k)
    torch.cuda.synchronize()
    got = nxt.cpu().numpy()
    for b in range(B):
        want = orc.sample_topk(z[b], noise[b], temp, k)
        assert int(got[b]) == want, f"row {b}: kernel {got[b]}, oracle {want}"


@pytest.mark.parametrize("temp,k", [(0.8, 20), (0.0, 0)])
def test_engine_sampling_in_prefill_and_decode(temp, k):
    """nc_kv_set_sampling: the engine's next tokens are the sampled pick over
    the logits it returns (prefill and the whole-step decode), and those
    logits still match the oracle."""
    cfg = SMALL
    B, T, steps = 4, 30, 3
    prompts = syn.tokens_zipf(49, (B, T), cfg.vocab)
    run = Run(cfg, blob_for(cfg), B, T + steps + 1)
    run.kv.set_sampling(temp, k)
    noise = syn.gumbel(5, (B, cfg.vocab), stream=20)
    lg, nxt = run.prefill(prompts, noise=noise)
    om = orc.OracleModel(cfg, blob_for(cfg))
    seqs = [om.new_seq(T + steps + 1) for _ in range(B)]
    for b in range(B):
        check_logits(lg[b], seqs[b].prefill(prompts[b]), tol_for(cfg), f"prefill seq {b}")
        assert int(nxt[b]) == orc.sample_topk(lg[b], noise[b], temp, k)
    cur = nxt.copy()
    for s in range(steps):
        nz = syn.gumbel(5, (B, cfg.vocab), stream=21 + s)
        lg2, n2 = run.decode(cur, np.full(B, T + s, np.int32), nz)
        for b in range(B):
            check_logits(lg2[b], seqs[b].step(int(cur[b])), tol_for(cfg), f"step {s} seq {b}")
            assert int(n2[b]) == orc.sample_topk(lg2[b], nz[b], temp, k), f"step {s} seq {b}"
        cur = n2
    assert run.status() == 0
