"""GPU parity of chunked prefill (nc_prefill_extend): tokens appended to
sequences that already hold a prompt, earlier chunks or decode steps, each at
its own current length. The oracle replays the same tokens one at a time
through its cache (orc_step, pinned to the full recompute), and every logit of
the chunk is compared, then decoding continues from the extended caches."""
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


def _extend(run, tokens, all_logits=False, noise=None):
    import torch
    B, T = tokens.shape
    V = run.cfg.vocab
    tok = torch.from_numpy(np.ascontiguousarray(tokens, np.int32)).cuda()
    logits = torch.full((B, T, V) if all_logits else (B, V), float("nan"), dtype=torch.float32, device="cuda")
    nxt = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    nz = None if noise is None else torch.from_numpy(noise).cuda()
    run.model.extend(run.kv, tok, 1 if all_logits else 0, logits, nxt, nz)
    torch.cuda.synchronize()
    return logits.cpu().numpy(), nxt.cpu().numpy()


@pytest.mark.parametrize("cfg,B,T0,T1,T2", [
    (SMALL, 3, 40, 17, 9),      # two chunks after the prompt
    (syn.TINY, 2, 16, 10, 5),   # fp32 model
    (syn.D20, 2, 48, 80, 3),    # 160 chunk rows: the tensor-core GEMMs on the chunk
])
def test_chunks_after_prompt_and_ragged_decode_match_oracle(cfg, B, T0, T1, T2):
    blob = blob_for(cfg)
    max_seq = T0 + T1 + T2 + 8
    prompts = syn.tokens_zipf(81, (B, T0), cfg.vocab)
    chunk1 = syn.tokens_zipf(82, (B, T1), cfg.vocab)
    chunk2 = syn.tokens_zipf(83, (B, T2), cfg.vocab)
    run = Run(cfg, blob, B, max_seq)
    _, nxt = run.prefill(prompts)
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(max_seq) for _ in range(B)]
    for b in range(B):
        seqs[b].prefill(prompts[b])
    # sequence 0 alone takes two decode steps, so the chunk starts at ragged lengths
    cur = nxt.copy()
    for s in range(2):
        l, n = run.decode(cur[:1], np.array([T0 + s], np.int32))
        check_logits(l[0], seqs[0].step(int(cur[0])), tol_for(cfg), f"pre-chunk decode {s}")
        cur[0] = n[0]
    tol = tol_for(cfg)
    lg, nx = _extend(run, chunk1, all_logits=True)
    for b in range(B):
        for t in range(T1):
            ref = seqs[b].step(int(chunk1[b, t]))
            check_logits(lg[b, t], ref, tol, f"chunk 1 seq {b} position {t}")
        check_token(int(nx[b]), ref, None, f"chunk 1 seq {b}")
    noise = syn.gumbel(5, (B, cfg.vocab), stream=40)
    lg, nx = _extend(run, chunk2, noise=noise)
    for b in range(B):
        for t in range(T2):
            ref = seqs[b].step(int(chunk2[b, t]))
        check_logits(lg[b], ref, tol, f"chunk 2 seq {b}")
        check_token(int(nx[b]), ref, noise[b], f"chunk 2 seq {b}")
    lens = [T0 + 2 + T1 + T2] + [T0 + T1 + T2] * (B - 1)
    assert list(run.kv.lengths(B)) == lens
    # decoding continues from the extended caches
    l, n = run.decode(nx, np.array(lens, np.int32))
    for b in range(B):
        check_logits(l[b], seqs[b].step(int(nx[b])), tol, f"decode after the chunks seq {b}")
    assert run.status() == 0


def test_chunk_that_does_not_fit_is_skipped():
    import kv_cache_transformer_b200 as nc
    cfg, blob = SMALL, blob_for(SMALL)
    run = Run(cfg, blob, 2, 50)
    run.prefill(syn.tokens_zipf(84, (2, 30), cfg.vocab))
    l, _ = run.decode(np.array([1, 2], np.int32), np.array([30, 30], np.int32))
    run.decode(np.array([3], np.int32), np.array([31], np.int32))  # sequence 0 at 32, sequence 1 at 31
    _extend(run, syn.tokens_zipf(85, (2, 19), cfg.vocab))            # 32 + 19 > 50: sequence 0 skipped
    assert list(run.kv.lengths(2)) == [32, 50]
    assert run.status() == nc.NC_DEV_BAD_POSITION


def test_chunk_on_a_shared_prefix_sample():
    cfg, blob = SMALL, blob_for(SMALL)
    T, max_seq = 140, 200
    prompt = syn.tokens_zipf(86, (1, T), cfg.vocab)
    run = Run(cfg, blob, 3, max_seq)
    run.prefill(prompt)
    run.kv.fork_shared_to(0, run.kv, 1, 2)  # samples 1, 2 read rows 0..127 of sequence 0
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(max_seq) for _ in range(3)]
    seqs[0].prefill(prompt[0])
    for r in seqs[1:]:
        r.copy_from(seqs[0])
    chunk = syn.tokens_zipf(87, (3, 21), cfg.vocab)
    lg, _ = _extend(run, chunk, all_logits=True)
    for b in range(3):
        for t in range(21):
            ref = seqs[b].step(int(chunk[b, t]))
            check_logits(lg[b, t], ref, tol_for(cfg), f"seq {b} position {t}")
    assert run.status() == 0


def _misc_launches(run, fn):
    import kv_cache_transformer_b200 as nc
    run.model.profile(True)
    run.model.profile_read()
    out = fn()
    _, launches = run.model.profile_read()
    run.model.profile(False)
    return out, launches[nc.NC_K_MISC]


def test_fused_chunk_with_a_sequence_that_does_not_fit():
    """180 chunk rows take the fused tensor-core layers (RoPE/QK norm and the
    cache append in the QKV epilogue, the tcgen05 attention with per-sequence
    offsets); sequence 0, one decode step ahead, does not fit and must keep
    its cache and length."""
    import kv_cache_transformer_b200 as nc
    cfg, blob = SMALL, blob_for(SMALL)
    B, T0, T1, max_seq = 3, 40, 60, 100
    run = Run(cfg, blob, B, max_seq)
    prompts = syn.tokens_zipf(88, (B, T0), cfg.vocab)
    _, nxt = run.prefill(prompts)
    om = orc.OracleModel(cfg, blob)
    seqs = [om.new_seq(max_seq) for _ in range(B)]
    for b in range(B):
        seqs[b].prefill(prompts[b])
    l, n = run.decode(nxt[:1], np.array([T0], np.int32))  # sequence 0 at 41: 41 + 60 > 100
    check_logits(l[0], seqs[0].step(int(nxt[0])), tol_for(cfg), "decode before the chunk")
    chunk = syn.tokens_zipf(89, (B, T1), cfg.vocab)
    (lg, _), misc = _misc_launches(run, lambda: _extend(run, chunk, all_logits=True))
    assert misc < 2 + 3 * cfg.depth, "the chunk did not take the fused layers"
    assert list(run.kv.lengths(B)) == [T0 + 1, T0 + T1, T0 + T1]
    assert run.status() == nc.NC_DEV_BAD_POSITION
    for b in (1, 2):
        for t in range(T1):
            check_logits(lg[b, t], seqs[b].step(int(chunk[b, t])), tol_for(cfg), f"chunk seq {b} position {t}")
    # the skipped sequence's cache is intact: its next decode step matches
    l, _ = run.decode(n[:1], np.array([T0 + 1], np.int32))
    check_logits(l[0], seqs[0].step(int(n[0])), tol_for(cfg), "sequence 0 after the skipped chunk")
    assert run.status() == 0
