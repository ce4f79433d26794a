"""GPU parity of the shared-prefix fork (nc_kv_fork_shared): forked samples
read the prompt's key/value rows from the source sequence instead of copies.
It must be observationally a copy: decode steps give logits bit-identical to
those after nc_kv_fork on the same inputs, and the oracle's copied sequences
(orc_seq_copy) agree within the usual tolerance. Covered on the three
attention paths: the whole-step kernel (bf16), the per-kernel decode launches
(NC_DECODE_STEP_KERNEL=0) and the generic kernels (fp32 model); plus the
link rules (a shared source cannot be replaced, one prefix cache per cache,
the source cache outliving its handle)."""
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


def _decode(model, kv, cur, noise):
    import torch
    B = cur.size
    t = torch.from_numpy(np.ascontiguousarray(cur, np.int32)).cuda()
    nz = torch.from_numpy(np.ascontiguousarray(noise, np.float32)).cuda()
    logits = torch.full((B, model.vocab), float("nan"), dtype=torch.float32, device="cuda")
    nx = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    model.decode_step(kv, t, None, nz, logits, nx)
    torch.cuda.synchronize()
    return logits.cpu().numpy(), nx.cpu().numpy()


@pytest.mark.parametrize("cfg,per_kernel", [(SMALL, False), (SMALL, True), (syn.TINY, False)])
def test_shared_fork_equals_copy_fork(monkeypatch, cfg, per_kernel):
    if per_kernel:
        monkeypatch.setenv("NC_DECODE_STEP_KERNEL", "0")
    blob = blob_for(cfg)
    T, n, steps, max_seq = 150, 6, 5, 170  # 128 shared rows, 22 copied
    prompt = syn.tokens_zipf(71, (1, T), cfg.vocab)
    src = Run(cfg, blob, 1, max_seq)
    _, nxt = src.prefill(prompt)
    copy = src.model.kv(n, max_seq)
    share = src.model.kv(n, max_seq)
    src.kv.fork_to(0, copy, 0, n)
    src.kv.fork_shared_to(0, share, 0, n)
    assert list(share.lengths(n)) == [T] * n
    om = orc.OracleModel(cfg, blob)
    base = om.new_seq(max_seq)
    base.prefill(prompt[0])
    refs = [om.new_seq(max_seq) for _ in range(n)]
    for r in refs:
        r.copy_from(base)
    cur = np.full(n, int(nxt[0]), np.int32)
    for s in range(steps):
        noise = syn.gumbel(5, (n, cfg.vocab), stream=100 + s)
        lc, nc_ = _decode(src.model, copy, cur, noise)
        ls, ns = _decode(src.model, share, cur, noise)
        assert np.array_equal(lc, ls), f"step {s}: shared-prefix logits differ from the copy's"
        assert np.array_equal(nc_, ns)
        for i in (0, n - 1):
            ref = refs[i].step(int(cur[i]))
            check_logits(ls[i], ref, tol_for(cfg), f"sample {i} step {s}")
            check_token(int(ns[i]), ref, noise[i], f"sample {i} step {s}")
        for i in range(1, n - 1):
            refs[i].step(int(cur[i]))
        cur = ns.copy()
    assert src.status() == 0
    copy.close()
    share.close()


def test_shared_fork_within_one_cache_and_chained():
    """Source and samples in one cache (the source keeps decoding), then a
    second generation forked from a sample (it reads the same prefix), and a
    copy fork of a sample (its shared rows resolved through the prefix)."""
    cfg, blob = SMALL, blob_for(SMALL)
    T, max_seq = 200, 230  # 192 shared rows
    prompt = syn.tokens_zipf(73, (1, T), cfg.vocab)
    run = Run(cfg, blob, 5, max_seq)
    _, nxt = run.prefill(prompt)
    run.kv.fork_shared_to(0, run.kv, 1, 4)
    om = orc.OracleModel(cfg, blob)
    refs = [om.new_seq(max_seq) for _ in range(5)]
    refs[0].prefill(prompt[0])
    for r in refs[1:]:
        r.copy_from(refs[0])
    cur = np.full(5, int(nxt[0]), np.int32)
    for s in range(3):
        noise = syn.gumbel(5, (5, cfg.vocab), stream=200 + s)
        lg, nn = _decode(run.model, run.kv, cur, noise)
        for i in range(5):
            check_logits(lg[i], refs[i].step(int(cur[i])), tol_for(cfg), f"seq {i} step {s}")
        cur = nn.copy()
    # second generation: from sample 2 (which reads seq 0's rows), shared and copied
    gen2 = run.model.kv(2, max_seq)
    run.kv.fork_shared_to(2, gen2, 0, 1)
    run.kv.fork_to(2, gen2, 1, 1)
    r2 = [om.new_seq(max_seq), om.new_seq(max_seq)]
    for r in r2:
        r.copy_from(refs[2])
    c2 = np.full(2, int(cur[2]), np.int32)
    for s in range(2):
        # one noise row for both: the two forks must pick the same tokens
        noise = np.repeat(syn.gumbel(5, (1, cfg.vocab), stream=300 + s), 2, axis=0)
        lg, nn = _decode(run.model, gen2, c2, noise)
        errs = []
        for i in range(2):
            ref = r2[i].step(int(c2[i]))
            errs.append(float(np.max(np.abs(lg[i] - ref))))
        assert max(errs) <= tol_for(cfg), f"gen2 step {s}: max |logit error| shared {errs[0]:.3g}, copied {errs[1]:.3g}"
        assert np.array_equal(lg[0], lg[1]), "shared and copied second-generation forks differ"
        c2 = nn.copy()
    assert run.status() == 0
    gen2.close()


def test_shared_source_cannot_be_replaced_and_outlives_its_handle():
    import torch
    import kv_cache_transformer_b200 as nc
    cfg, blob = SMALL, blob_for(SMALL)
    T, max_seq = 100, 120
    prompt = syn.tokens_zipf(75, (1, T), cfg.vocab)
    src = Run(cfg, blob, 1, max_seq)
    _, nxt = src.prefill(prompt)
    dst = src.model.kv(3, max_seq)
    src.kv.fork_shared_to(0, dst, 0, 3)
    tok = torch.from_numpy(prompt.astype(np.int32)).cuda()
    with pytest.raises(nc.NcError) as e:
        src.model.prefill(src.kv, tok)
    assert e.value.code == nc.NC_EINVAL and "shared prefix" in str(e.value)
    other = src.model.kv(1, max_seq)
    other.close()
    with pytest.raises(nc.NcError):
        dst.fork_to(0, src.kv, 0, 1)  # a fork into the shared source replaces it
    # a second prefix cache for dst while its links to src live
    src2 = src.model.kv(1, max_seq)
    src.model.prefill(src2, tok)
    with pytest.raises(nc.NcError) as e:
        src2.fork_shared_to(0, dst, 0, 1)
    assert "another cache" in str(e.value)
    # the source handle goes away first: dst keeps reading its rows
    src.kv.close()
    om = orc.OracleModel(cfg, blob)
    ref = om.new_seq(max_seq)
    ref.prefill(prompt[0])
    cur = np.full(3, int(nxt[0]), np.int32)
    lg, _ = _decode(src.model, dst, cur, np.zeros((3, cfg.vocab), np.float32))
    check_logits(lg[2], ref.step(int(cur[2])), tol_for(cfg), "after the source handle was closed")
    # replacing every sample ends the links: src2 may now lend its prefix
    src.model.prefill(dst, torch.from_numpy(syn.tokens_zipf(76, (3, 10), cfg.vocab)).cuda())
    src2.fork_shared_to(0, dst, 0, 1)
    assert src.model.status() == 0
    dst.close()
    src2.close()
