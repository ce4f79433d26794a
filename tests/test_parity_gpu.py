"""GPU parity: the CUDA engine (through the C ABI) against the CPU oracle on the
same seeded inputs, logits element by element, tokens where unique."""
import numpy as np
import pytest

import nc_synth as syn
import oracle as orc
from nc_harness import (GAP, Run, check_logits, check_token, greedy_session, tol_for, top2_gap)

pytestmark = pytest.mark.gpu

_blobs = {}


def blob_for(cfg, seed=0):
    key = (cfg, seed)
    if key not in _blobs:
        _blobs[key] = syn.make_blob(cfg, seed)
    return _blobs[key]


def test_tiny_fp32_prefill_all_positions_and_16_decode_steps():
    w = syn.WORKLOADS["tiny"]
    worst = greedy_session(w.model, blob_for(w.model), syn.prompt_tokens(w), w.decode_steps, [0],
                           all_logits=True)
    assert worst <= 1e-3


def test_tiny_batch_with_ragged_prompt_length():
    cfg = syn.TINY
    prompts = syn.tokens_uniform(9, (3, 37), cfg.vocab)
    greedy_session(cfg, blob_for(cfg), prompts, 5, [0, 1, 2], all_logits=True)


@pytest.mark.parametrize("cfg,B,T,steps,seqs", [
    (syn.D20, 3, 160, 3, [0, 2]),
    (syn.D26, 1, 72, 3, [0]),
    (syn.D30, 2, 40, 2, [1]),
    # >= 128 prompt rows: the fused prefill epilogues, with a partial last
    # 256-column tile of the residual (d 1664, 1920) and of the qkv projection
    # (15 and 17 heads of 128) and a partial last 128-row tile
    (syn.D26, 2, 100, 2, [1]),
    (syn.D30, 1, 130, 1, [0]),
])
def test_bf16_models_short_context(cfg, B, T, steps, seqs):
    prompts = syn.tokens_zipf(21, (B, T), cfg.vocab)
    worst = greedy_session(cfg, blob_for(cfg), prompts, steps, seqs)
    assert worst <= 0.05


def test_ragged_positions_in_one_decode_step():
    cfg = syn.TINY
    blob = blob_for(cfg)
    prompts = syn.tokens_uniform(4, (3, 11), cfg.vocab)
    run = Run(cfg, blob, 3, 40)
    _, nxt = run.prefill(prompts)
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(40) for _ in range(3)]
    for b in range(3):
        seqs[b].prefill(prompts[b])
    # advance sequence 0 alone by two tokens
    pos = np.array([11, 11, 11], np.int32)
    cur = nxt.copy()
    for _ in range(2):
        l, n = run.decode(cur[:1], pos[:1])
        ref = seqs[0].step(int(cur[0]))
        check_logits(l[0], ref, 1e-3, "seq 0 alone")
        cur[0] = n[0]
        pos[0] += 1
    assert list(run.kv.lengths(3)) == [13, 11, 11]
    l, n = run.decode(cur, pos)
    for b in range(3):
        ref = seqs[b].step(int(cur[b]))
        check_logits(l[b], ref, 1e-3, f"ragged seq {b}")
        check_token(int(n[b]), ref, None, f"ragged seq {b}")
    assert list(run.kv.lengths(3)) == [14, 12, 12]
    assert run.status() == 0


def test_fork_then_gumbel_sampling_matches_oracle():
    cfg = syn.TINY
    blob = blob_for(cfg)
    import kv_cache_transformer_b200 as nc
    import torch
    prompt = syn.tokens_uniform(5, (1, 20), cfg.vocab)
    src = Run(cfg, blob, 1, 32)
    _, nxt = src.prefill(prompt)
    n = 4
    dst = src.model.kv(n + 1, 32)  # destinations 1..4; row 0 stays empty
    src.kv.fork_to(0, dst, 1, n)
    assert list(dst.lengths(n + 1)) == [0, 20, 20, 20, 20]
    om = orc.OracleModel(cfg, blob)
    base = om.new_seq(32)
    base.prefill(prompt[0])
    refs = [om.new_seq(32) for _ in range(n)]
    for r in refs:
        r.copy_from(base)
    cur = np.full(n, int(nxt[0]), np.int32)
    for step in range(6):
        noise = syn.gumbel(syn.WORKLOADS["d30_rollout"].noise_seed, (n, cfg.vocab), stream=step)
        # decode rows 1..4 of dst: feed row 0 a bad position so it is skipped
        tok = np.concatenate([[0], cur]).astype(np.int32)
        pos = np.concatenate([[999], np.full(n, 20 + step)]).astype(np.int32)
        t = torch.from_numpy(tok).cuda()
        p = torch.from_numpy(pos).cuda()
        nz = torch.from_numpy(np.concatenate([np.zeros((1, cfg.vocab), np.float32), noise])).cuda()
        logits = torch.empty((n + 1, cfg.vocab), device="cuda")
        nx = torch.full((n + 1,), -1, dtype=torch.int32, device="cuda")
        src.model.decode_step(dst, t, p, nz, logits, nx)
        torch.cuda.synchronize()
        lg, nn = logits.cpu().numpy(), nx.cpu().numpy()
        assert nn[0] == -1
        for i in range(n):
            ref = refs[i].step(int(cur[i]))
            check_logits(lg[i + 1], ref, 1e-3, f"fork sample {i} step {step}")
            check_token(int(nn[i + 1]), ref, noise[i], f"fork sample {i} step {step}")
        cur = nn[1:].copy()
    assert src.model.status() == nc.NC_DEV_BAD_POSITION  # only row 0's planted position
    dst.close()


def test_bad_position_skips_sequence_and_raises_status():
    cfg = syn.TINY
    import kv_cache_transformer_b200 as nc
    run = Run(cfg, blob_for(cfg), 2, 16)
    _, nxt = run.prefill(syn.tokens_uniform(6, (2, 5), cfg.vocab))
    l, n = run.decode(nxt, np.array([5, 9], np.int32))
    assert np.all(np.isnan(l[1])) and n[1] == -1   # untouched
    assert np.all(np.isfinite(l[0])) and n[0] >= 0
    assert list(run.kv.lengths(2)) == [6, 5]
    assert run.status() == nc.NC_DEV_BAD_POSITION
    assert run.status() == 0  # read clears
    # position at the end of the cache is rejected too
    l, n = run.decode(np.array([n[0], 3], np.int32), np.array([6, 16], np.int32))
    assert run.status() == nc.NC_DEV_BAD_POSITION


def test_bad_token_is_clamped_and_flagged():
    cfg = syn.TINY
    import kv_cache_transformer_b200 as nc
    run = Run(cfg, blob_for(cfg), 1, 8)
    p = np.array([[1, 2, cfg.vocab + 5]], np.int32)
    lg, _ = run.prefill(p)
    assert np.all(np.isfinite(lg))
    assert run.status() == nc.NC_DEV_BAD_TOKEN


def test_prefill_replaces_previous_contents_and_errors_leave_state():
    cfg = syn.TINY
    import kv_cache_transformer_b200 as nc
    import torch
    blob = blob_for(cfg)
    run = Run(cfg, blob, 2, 24)
    run.prefill(syn.tokens_uniform(7, (2, 20), cfg.vocab))
    p2 = syn.tokens_uniform(8, (2, 9), cfg.vocab)
    lg, _ = run.prefill(p2)
    assert list(run.kv.lengths(2)) == [9, 9]
    om = orc.OracleModel(cfg, blob)
    for b in range(2):
        check_logits(lg[b], om.forward_full(p2[b], all_positions=False), 1e-3, f"re-prefill seq {b}")
    # host-side range errors change nothing
    too_long = torch.zeros((1, 25), dtype=torch.int32, device="cuda")
    with pytest.raises(nc.NcError) as e:
        run.model.prefill(run.kv, too_long)
    assert e.value.code == nc.NC_ERANGE
    too_many = torch.zeros((3, 4), dtype=torch.int32, device="cuda")
    with pytest.raises(nc.NcError) as e:
        run.model.prefill(run.kv, too_many)
    assert e.value.code == nc.NC_ERANGE
    assert list(run.kv.lengths(2)) == [9, 9]
