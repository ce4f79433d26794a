"""GPU parity of grouped-query and multi-head attention (n_kv_head > 1): the
H query heads form Hkv groups of G = H/Hkv heads, each group reading one KV
head. The oracle's attention takes head h's keys from KV head h // G (its MQA
= MHA pin fixes the grouping), and every logit of the engine is compared with
it: prefill at all positions through the fused tcgen05 layers (where a
128-row Q tile holds whole positions of a group) or the generic attention (G =
5), decode through the whole-step kernel, including batches with more
(sequence, KV head) pairs than CTAs, ragged positions, shared-prefix forks and
chunks appended to the cache."""
import numpy as np
import pytest

import nc_synth as syn
import oracle as orc
from nc_harness import Run, check_logits, check_token, greedy_session, tol_for

pytestmark = pytest.mark.gpu


def _cfg(d, H, Hkv, F=None, V=1024, depth=2):
    return syn.ModelConfig(depth=depth, d_model=d, n_head=H, n_kv_head=Hkv, head_dim=128, mlp_hidden=F or 2 * d,
                           vocab=V, dtype="bf16")


GQA2 = _cfg(512, 4, 2)     # G = 2
MHA4 = _cfg(512, 4, 4)     # G = 1
GQA5 = _cfg(1280, 10, 2)   # G = 5: 128 Q rows hold no whole positions, prefill attention on the generic kernel
MHA8 = _cfg(1024, 8, 8)    # 32 sequences x 8 KV heads = 256 attention pairs, more than the CTAs
_blobs = {}


def blob_for(cfg):
    if cfg not in _blobs:
        _blobs[cfg] = syn.make_blob(cfg, 0)
    return _blobs[cfg]


def _launches(run, fn):
    run.model.profile(True)
    run.model.profile_read()
    out = fn()
    _, launches = run.model.profile_read()
    run.model.profile(False)
    return out, launches


@pytest.mark.parametrize("cfg,B,T,fused", [
    (GQA2, 2, 136, True),
    (MHA4, 3, 100, True),
    (GQA5, 2, 136, False),
    (syn.D20_MHA, 2, 136, True),   # the 560M d20 model
])
def test_prefill_all_positions_and_decode_match_oracle(cfg, B, T, fused):
    import kv_cache_transformer_b200 as nc
    blob = blob_for(cfg)
    prompts = syn.tokens_zipf(90, (B, T), cfg.vocab)
    steps = 4
    run = Run(cfg, blob, B, T + steps + 1)
    (lg, nxt), pl = _launches(run, lambda: run.prefill(prompts, all_logits=True))
    # the fused layer sequence launches one norm (layer 0) instead of three per layer
    assert (pl[nc.NC_K_MISC] < 3 * cfg.depth) == fused
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(T + steps + 1) for _ in range(B)]
    tol = tol_for(cfg)
    for b in range(B):
        ref = seqs[b].prefill(prompts[b], all_positions=True)
        check_logits(lg[b], ref, tol, f"prefill seq {b} (all positions)")
        check_token(int(nxt[b]), ref[-1], None, f"prefill seq {b}")
    cur = nxt.copy()
    for s in range(steps):
        (l, n), dl = _launches(run, lambda: run.decode(cur, np.full(B, T + s, np.int32)))
        assert dl[nc.NC_K_STEP] == 1, "decode did not run the whole-step kernel"
        for b in range(B):
            ref = seqs[b].step(int(cur[b]))
            check_logits(l[b], ref, tol, f"decode seq {b} step {s}")
            check_token(int(n[b]), ref, None, f"decode seq {b} step {s}")
        cur = n
    assert run.status() == 0


def test_decode_with_more_attention_pairs_than_ctas_and_ragged_positions():
    """32 sequences x 8 KV heads: each CTA takes two attention units (one key
    split each); the first half of the batch runs one step ahead."""
    cfg, blob = MHA8, blob_for(MHA8)
    B, T, steps = 32, 40, 3
    prompts = syn.tokens_zipf(91, (B, T), cfg.vocab)
    run = Run(cfg, blob, B, T + steps + 2)
    _, nxt = run.prefill(prompts)
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(T + steps + 2) for _ in range(B)]
    for b in range(B):
        seqs[b].prefill(prompts[b])
    tol = tol_for(cfg)
    cur = nxt.copy()
    l, n = run.decode(cur[:16], np.full(16, T, np.int32))
    for b in range(16):
        check_logits(l[b], seqs[b].step(int(cur[b])), tol, f"half-batch step seq {b}")
    cur[:16] = n
    for s in range(steps):
        pos = np.array([T + 1 + s] * 16 + [T + s] * 16, np.int32)
        noise = syn.gumbel(5, (B, cfg.vocab), stream=500 + s)
        l, n = run.decode(cur, pos, noise)
        for b in range(B):
            ref = seqs[b].step(int(cur[b]))
            check_logits(l[b], ref, tol, f"step {s} seq {b}")
            check_token(int(n[b]), ref, noise[b], f"step {s} seq {b}")
        cur = n
    assert run.status() == 0


def test_more_pairs_than_ctas_dealt_in_rounds():
    """With more (sequence, KV head) units than CTAs the decode step deals the
    key tiles evenly; NC_DECODE_TILE_DEAL=0 keeps the rounds of key splits
    that it falls back to when the deal does not fit. The test above, run in
    a process of its own with the rounds."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, NC_DECODE_TILE_DEAL="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_gqa_gpu.py::test_decode_with_more_attention_pairs_than_ctas_and_ragged_positions"],
                       env=env, cwd=root, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_d20_mha_batch32_decode_sampled_sequences():
    """The d20 MHA model at batch 32: 320 (sequence, KV head) attention pairs
    over the CTAs; sequences 0, 13 and 31 replayed by the oracle."""
    cfg, blob = syn.D20_MHA, blob_for(syn.D20_MHA)
    B, T, steps = 32, 72, 2
    prompts = syn.tokens_zipf(92, (B, T), cfg.vocab)
    worst = greedy_session(cfg, blob, prompts, steps, check_seqs=(0, 13, 31))
    assert worst <= tol_for(cfg)


@pytest.mark.parametrize("cfg", [GQA2, MHA8])
def test_shared_prefix_fork_equals_copy(cfg):
    blob = blob_for(cfg)
    T, n, steps, max_seq = 150, 5, 3, 170  # 128 shared rows
    prompt = syn.tokens_zipf(93, (1, T), cfg.vocab)
    src = Run(cfg, blob, 1, max_seq)
    _, nxt = src.prefill(prompt)
    copy = src.model.kv(n, max_seq)
    share = src.model.kv(n, max_seq)
    src.kv.fork_to(0, copy, 0, n)
    src.kv.fork_shared_to(0, share, 0, n)
    om = orc.OracleModel(cfg, blob)
    base = om.new_seq(max_seq)
    base.prefill(prompt[0])
    refs = [om.new_seq(max_seq) for _ in range(n)]
    for r in refs:
        r.copy_from(base)
    import torch
    cur = np.full(n, int(nxt[0]), np.int32)
    for s in range(steps):
        noise = syn.gumbel(5, (n, cfg.vocab), stream=600 + s)
        outs = []
        for kv in (copy, share):
            t = torch.from_numpy(cur).cuda()
            nz = torch.from_numpy(noise).cuda()
            lg = torch.full((n, cfg.vocab), float("nan"), dtype=torch.float32, device="cuda")
            nx = torch.full((n,), -1, dtype=torch.int32, device="cuda")
            src.model.decode_step(kv, t, None, nz, lg, nx)
            torch.cuda.synchronize()
            outs.append((lg.cpu().numpy(), nx.cpu().numpy()))
        (lc, nc_), (ls, ns) = outs
        assert np.array_equal(lc, ls), f"step {s}: shared-prefix logits differ from the copy's"
        assert np.array_equal(nc_, ns)
        for i in range(n):
            ref = refs[i].step(int(cur[i]))
            check_logits(ls[i], ref, tol_for(cfg), f"sample {i} step {s}")
            check_token(int(ns[i]), ref, noise[i], f"sample {i} step {s}")
        cur = ns.copy()
    assert src.status() == 0
    copy.close()
    share.close()


def test_chunk_appended_to_gqa_cache():
    import torch
    cfg, blob = GQA2, blob_for(GQA2)
    B, T0, T1 = 2, 40, 19
    run = Run(cfg, blob, B, T0 + T1 + 4)
    prompts = syn.tokens_zipf(94, (B, T0), cfg.vocab)
    chunk = syn.tokens_zipf(95, (B, T1), cfg.vocab)
    _, nxt = run.prefill(prompts)
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(T0 + T1 + 4) for _ in range(B)]
    for b in range(B):
        seqs[b].prefill(prompts[b])
    lg = torch.full((B, T1, cfg.vocab), float("nan"), dtype=torch.float32, device="cuda")
    nx = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    run.model.extend(run.kv, torch.from_numpy(chunk).cuda(), 1, lg, nx)
    torch.cuda.synchronize()
    lg = lg.cpu().numpy()
    for b in range(B):
        for t in range(T1):
            check_logits(lg[b, t], seqs[b].step(int(chunk[b, t])), tol_for(cfg), f"chunk seq {b} position {t}")
    l, _ = run.decode(nx.cpu().numpy(), np.full(B, T0 + T1, np.int32))
    for b in range(B):
        check_logits(l[b], seqs[b].step(int(nx[b])), tol_for(cfg), f"decode after the chunk seq {b}")
    assert run.status() == 0


def test_fused_chunk_on_gqa_cache():
    """160 chunk rows on a grouped-query cache: the fused layers with per-sequence
    offsets put each KV head of the chunk at its slot of the cache rows."""
    import kv_cache_transformer_b200 as nc
    import torch
    cfg, blob = GQA2, blob_for(GQA2)
    B, T0, T1 = 2, 33, 80
    run = Run(cfg, blob, B, T0 + T1 + 2)
    prompts = syn.tokens_zipf(96, (B, T0), cfg.vocab)
    chunk = syn.tokens_zipf(97, (B, T1), cfg.vocab)
    _, nxt = run.prefill(prompts)
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(T0 + T1 + 2) for _ in range(B)]
    for b in range(B):
        seqs[b].prefill(prompts[b])
    lg = torch.full((B, T1, cfg.vocab), float("nan"), dtype=torch.float32, device="cuda")
    nx = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    (_, launches) = _launches(run, lambda: (run.model.extend(run.kv, torch.from_numpy(chunk).cuda(), 1, lg, nx),
                                            torch.cuda.synchronize()))
    assert launches[nc.NC_K_MISC] < 2 + 3 * cfg.depth, "the chunk did not take the fused layers"
    lg = lg.cpu().numpy()
    for b in range(B):
        for t in range(T1):
            check_logits(lg[b, t], seqs[b].step(int(chunk[b, t])), tol_for(cfg), f"chunk seq {b} position {t}")
    l, _ = run.decode(nx.cpu().numpy(), np.full(B, T0 + T1, np.int32))
    for b in range(B):
        check_logits(l[b], seqs[b].step(int(nx[b])), tol_for(cfg), f"decode after the chunk seq {b}")
    assert run.status() == 0
