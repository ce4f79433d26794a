"""GPU parity of the sm_100a decode path (bf16, head_dim 128, one KV head,
B <= 32): batch sizes around the MMA widths, CUDA-graph replay with in-place
tokens and implicit positions, ragged and invalid positions, fork + Gumbel
sampling, batch invariance, and the d20 decode workload at full context."""
import numpy as np
import pytest

import nc_synth as syn
import oracle as orc
from nc_harness import TOL_BF16, Run, check_logits, check_token, greedy_session

pytestmark = pytest.mark.gpu

# small bf16 model on the fast decode path (hd 128, one KV head)
SMALL = syn.ModelConfig(depth=2, d_model=256, n_head=2, n_kv_head=1, head_dim=128, mlp_hidden=512, vocab=1024,
                        dtype="bf16")
_blobs = {}


def blob_for(cfg):
    if cfg not in _blobs:
        _blobs[cfg] = syn.make_blob(cfg, 0)
    return _blobs[cfg]


@pytest.mark.parametrize("B", [1, 5, 16, 17, 32])
def test_small_bf16_decode_batch_sizes(B):
    prompts = syn.tokens_zipf(30 + B, (B, 40), SMALL.vocab)
    greedy_session(SMALL, blob_for(SMALL), prompts, 4, list(range(B)))


def test_graph_replay_inplace_tokens_and_implicit_positions():
    import torch
    cfg, blob = SMALL, blob_for(SMALL)
    B, T, steps = 4, 33, 8
    prompts = syn.tokens_zipf(7, (B, T), cfg.vocab)
    run = Run(cfg, blob, B, T + steps + 1)
    _, nxt = run.prefill(prompts)
    tok = torch.from_numpy(nxt.astype(np.int32)).cuda()      # also receives the next tokens
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(T + steps + 1) for _ in range(B)]
    for b in range(B):
        seqs[b].prefill(prompts[b])
    for s in range(steps):
        fed = tok.cpu().numpy().copy()
        run.model.decode_step(run.kv, tok, None, None, logits, tok)
        torch.cuda.synchronize()
        lg, nn = logits.cpu().numpy(), tok.cpu().numpy()
        for b in range(B):
            ref = seqs[b].step(int(fed[b]))
            check_logits(lg[b], ref, TOL_BF16, f"replay step {s} seq {b}")
            check_token(int(nn[b]), ref, None, f"replay step {s} seq {b}")
    assert list(run.kv.lengths(B)) == [T + steps] * B
    assert run.status() == 0


def test_ragged_and_invalid_positions_bf16():
    import kv_cache_transformer_b200 as nc
    cfg, blob = SMALL, blob_for(SMALL)
    prompts = syn.tokens_zipf(4, (3, 21), cfg.vocab)
    run = Run(cfg, blob, 3, 40)
    _, nxt = run.prefill(prompts)
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(40) for _ in range(3)]
    for b in range(3):
        seqs[b].prefill(prompts[b])
    pos = np.array([21, 21, 21], np.int32)
    cur = nxt.copy()
    for _ in range(3):  # sequence 0 alone
        l, n = run.decode(cur[:1], pos[:1])
        check_logits(l[0], seqs[0].step(int(cur[0])), TOL_BF16, "seq 0 alone")
        cur[0] = n[0]
        pos[0] += 1
    # one wrong position (seq 2): skipped, outputs untouched, status raised
    bad = pos.copy()
    bad[2] += 5
    l, n = run.decode(cur, bad)
    assert np.all(np.isnan(l[2])) and n[2] == -1
    for b in range(2):
        ref = seqs[b].step(int(cur[b]))
        check_logits(l[b], ref, TOL_BF16, f"ragged seq {b}")
        check_token(int(n[b]), ref, None, f"ragged seq {b}")
    assert list(run.kv.lengths(3)) == [25, 22, 21]
    assert run.status() == nc.NC_DEV_BAD_POSITION
    # every sequence continues from its real length
    cur[:2] = n[:2]
    l, n = run.decode(cur, np.array([25, 22, 21], np.int32))
    for b in range(3):
        check_logits(l[b], seqs[b].step(int(cur[b])), TOL_BF16, f"seq {b} after the skip")
    assert list(run.kv.lengths(3)) == [26, 23, 22]
    assert run.status() == 0


def test_fork_then_gumbel_sampling_bf16():
    import torch
    cfg, blob = SMALL, blob_for(SMALL)
    prompt = syn.tokens_zipf(5, (1, 30), cfg.vocab)
    src = Run(cfg, blob, 1, 48)
    _, nxt = src.prefill(prompt)
    n = 8
    dst = src.model.kv(n, 48)
    src.kv.fork_to(0, dst, 0, n)
    om = orc.OracleModel(cfg, blob)
    base = om.new_seq(48)
    base.prefill(prompt[0])
    refs = [om.new_seq(48) for _ in range(n)]
    for r in refs:
        r.copy_from(base)
    cur = np.full(n, int(nxt[0]), np.int32)
    seen = set()
    for step in range(6):
        noise = syn.gumbel(syn.WORKLOADS["d30_rollout"].noise_seed, (n, cfg.vocab), stream=step)
        t = torch.from_numpy(cur).cuda()
        nz = torch.from_numpy(noise).cuda()
        logits = torch.empty((n, cfg.vocab), device="cuda")
        nx = torch.full((n,), -1, dtype=torch.int32, device="cuda")
        src.model.decode_step(dst, t, None, nz, logits, nx)
        torch.cuda.synchronize()
        lg, nn = logits.cpu().numpy(), nx.cpu().numpy()
        for i in range(n):
            ref = refs[i].step(int(cur[i]))
            check_logits(lg[i], ref, TOL_BF16, f"sample {i} step {step}")
            check_token(int(nn[i]), ref, noise[i], f"sample {i} step {step}")
        seen |= set(nn.tolist())
        cur = nn.copy()
    assert len(seen) > 1  # the noise makes the samples differ
    assert src.model.status() == 0
    dst.close()


def test_decode_batch_invariance_d20():
    cfg = syn.D20
    blob = blob_for(cfg)
    prompts = syn.tokens_zipf(12, (32, 64), cfg.vocab)
    big = Run(cfg, blob, 32, 80)
    lgb, nb = big.prefill(prompts)
    # two sequences: 128 prefill rows, the same tensor-core path as the batch of 32
    one = Run(cfg, blob, 2, 80)
    lg1, n1 = one.prefill(prompts[6:8])
    assert np.max(np.abs(lgb[7] - lg1[1])) <= 1e-6
    d_big, _ = big.decode(nb, np.full(32, 64, np.int32))
    d_one, _ = one.decode(nb[6:8], np.array([64, 64], np.int32))
    assert np.max(np.abs(d_big[7] - d_one[1])) <= 1e-4


def test_d20_decode_workload_full_context_sampled():
    """The d20 decode workload (32 sequences prefilled to 2048 Zipf tokens) on
    the GPU; the oracle replays sequence 31 at full context for 2 steps."""
    w = syn.WORKLOADS["d20_decode"]
    cfg = w.model
    prompts = syn.prompt_tokens(w)
    worst = greedy_session(cfg, blob_for(cfg), prompts, 2, [31], max_seq=w.prompt_len + w.decode_steps)
    assert worst <= TOL_BF16


@pytest.mark.parametrize("cfg,B,T,steps", [(SMALL, 5, 40, 4), (syn.D20, 3, 70, 3)])
def test_per_kernel_decode_path_matches_oracle(monkeypatch, cfg, B, T, steps):
    """The decode step as one launch per layer step (the path a cache takes
    when the whole-step kernel cannot be placed), forced with the
    NC_DECODE_STEP_KERNEL=0 switch, against the oracle."""
    import kv_cache_transformer_b200 as nc
    monkeypatch.setenv("NC_DECODE_STEP_KERNEL", "0")
    blob = blob_for(cfg)
    prompts = syn.tokens_zipf(60 + B, (B, T), cfg.vocab)
    run = Run(cfg, blob, B, T + steps + 1)
    _, nxt = run.prefill(prompts)
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(T + steps + 1) for _ in range(B)]
    for b in range(B):
        seqs[b].prefill(prompts[b])
    cur = nxt.copy()
    run.model.profile(True)
    run.model.profile_read()
    for s in range(steps):
        lg, nn = run.decode(cur, np.full(B, T + s, np.int32))
        for b in (0, B - 1):
            ref = seqs[b].step(int(cur[b]))
            check_logits(lg[b], ref, TOL_BF16, f"per-kernel step {s} seq {b}")
            check_token(int(nn[b]), ref, None, f"per-kernel step {s} seq {b}")
        for b in range(1, B - 1):
            seqs[b].step(int(cur[b]))
        cur = nn
    _, launches = run.model.profile_read()
    run.model.profile(False)
    assert launches[nc.NC_K_STEP] == 0 and launches[nc.NC_K_GEMM] == 4 * cfg.depth * steps
    assert run.status() == 0


def test_decode_step_trace_fills_and_fits_the_event_time():
    """nc_decode_trace: every CTA stamps every phase, phases follow one
    another, the kernel's span lies inside the event-timed step, and tracing
    does not change the results."""
    import torch
    cfg = syn.D20
    blob = blob_for(cfg)
    B, T = 4, 16
    prompts = syn.tokens_zipf(66, (B, T), cfg.vocab)
    a, b_ = Run(cfg, blob, B, T + 3), Run(cfg, blob, B, T + 3)
    _, na = a.prefill(prompts)
    _, nb = b_.prefill(prompts)
    assert np.array_equal(na, nb)
    # one untraced step first: the traced one is not the cache's first launch
    _, na = a.decode(na, np.full(B, T, np.int32))
    _, nb = b_.decode(nb, np.full(B, T, np.int32))
    T += 1
    grid, P = a.kv.trace(None)
    assert grid > 0 and P == 3 + 5 * cfg.depth
    buf = torch.zeros(grid * P * 8, dtype=torch.int64, device="cuda")
    a.kv.trace(buf)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    la, ta = a.decode(na, np.full(B, T, np.int32))
    e1.record()
    torch.cuda.synchronize()
    a.kv.trace(None)
    lb, tb = b_.decode(nb, np.full(B, T, np.int32))
    assert np.array_equal(la, lb) and np.array_equal(ta, tb), "tracing changed the results"
    tr = buf.cpu().numpy().reshape(grid, P, 8)
    assert np.all(tr[:, :, 0] > 0) and np.all(tr[:, :, 4] > 0), "a CTA skipped a phase stamp"
    assert np.all(tr[:, :, 4] >= tr[:, :, 0])
    assert np.all(np.diff(tr[:, :, 0], axis=1) >= 0), "phase starts out of order"
    span_us = (tr[:, -1, 4].max() - tr[:, 0, 0].min()) / 1e3
    event_us = 1e3 * e0.elapsed_time(e1)
    assert 0.5 * event_us <= span_us <= event_us, (span_us, event_us)
    assert a.status() == 0


def test_d26_latency_workload_sampled():
    """The d26 latency workload's shape (one sequence, 1024-token Zipf prompt,
    greedy steps on the whole-step kernel), every logit against the oracle
    for the first decode steps."""
    w = syn.WORKLOADS["d26_latency"]
    cfg = w.model
    worst = greedy_session(cfg, blob_for(cfg), syn.prompt_tokens(w), 3, [0], max_seq=w.prompt_len + w.decode_steps)
    assert worst <= TOL_BF16


@pytest.mark.parametrize("shared", [False, True])
def test_d30_rollout_workload_sampled(shared):
    """The d30 rollout workload's shape: a 256-token prompt prefilled once,
    forked to 16 samples (copied, or sharing the prompt's rows), decode steps
    picking argmax(logits + Gumbel noise) with the workload's noise; samples 0
    and 15 replayed by the oracle."""
    import torch
    w = syn.WORKLOADS["d30_rollout"]
    cfg, blob = w.model, blob_for(w.model)
    n, T, max_seq, steps = w.fork, w.prompt_len, w.prompt_len + w.decode_steps, 3
    src = Run(cfg, blob, 1, max_seq)
    _, nxt = src.prefill(syn.prompt_tokens(w))
    dst = src.model.kv(n, max_seq)
    (src.kv.fork_shared_to if shared else src.kv.fork_to)(0, dst, 0, n)
    om = orc.OracleModel(cfg, blob)
    base = om.new_seq(max_seq)
    base.prefill(syn.prompt_tokens(w)[0])
    refs = {i: om.new_seq(max_seq) for i in (0, n - 1)}
    for r in refs.values():
        r.copy_from(base)
    cur = np.full(n, int(nxt[0]), np.int32)
    for s in range(steps):
        noise = syn.gumbel(w.noise_seed, (n, cfg.vocab), stream=s)
        t = torch.from_numpy(cur).cuda()
        lg = torch.full((n, cfg.vocab), float("nan"), dtype=torch.float32, device="cuda")
        nx = torch.full((n,), -1, dtype=torch.int32, device="cuda")
        src.model.decode_step(dst, t, None, torch.from_numpy(noise).cuda(), lg, nx)
        torch.cuda.synchronize()
        lg, nx = lg.cpu().numpy(), nx.cpu().numpy()
        for i, r in refs.items():
            ref = r.step(int(cur[i]))
            check_logits(lg[i], ref, TOL_BF16, f"sample {i} step {s}")
            check_token(int(nx[i]), ref, noise[i], f"sample {i} step {s}")
        cur = nx.copy()
    assert src.status() == 0
    dst.close()
