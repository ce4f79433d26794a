"""Shared helpers for the GPU parity tests: run the CUDA engine through the
C ABI and replay the same tokens through the CPU oracle (teacher forcing),
comparing logits element by element and tokens where the oracle's top-2 gap
makes the choice unique."""
from __future__ import annotations

import numpy as np

import nc_synth as syn
import oracle as orc

TOL_F32 = 1e-3   # max |logit| error, fp32 tiny model
TOL_BF16 = 0.05  # max |logit| error, bf16 models (oracle reads the same rounded weights)
GAP = 0.1        # token ids must match where the oracle's top-2 gap exceeds this


def tol_for(cfg) -> float:
    return TOL_F32 if cfg.dtype == "f32" else TOL_BF16


def top2_gap(v: np.ndarray) -> float:
    p = np.partition(v, -2)[-2:]
    return float(p[1] - p[0])


def check_logits(gpu: np.ndarray, ref: np.ndarray, tol: float, what: str):
    err = float(np.max(np.abs(gpu.astype(np.float64) - ref)))
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite logits"
    assert err <= tol, f"{what}: max |logit error| {err:.3g} > {tol}"
    return err


def check_token(gpu_tok: int, ref_logits: np.ndarray, noise: np.ndarray | None, what: str):
    z = ref_logits + (noise.astype(np.float64) if noise is not None else 0.0)
    if top2_gap(z) > GAP:
        assert gpu_tok == int(orc.argmax(ref_logits, noise)), f"{what}: token {gpu_tok} != oracle"


class Run:
    """One engine session (model + cache) plus the record of what it produced."""

    def __init__(self, cfg, blob, max_batch: int, max_seq: int):
        import kv_cache_transformer_b200 as nc
        self.cfg, self.blob = cfg, blob
        self.model = nc.Model(cfg, blob)
        self.kv = self.model.kv(max_batch, max_seq)

    def prefill(self, prompts: np.ndarray, all_logits: bool = False, noise=None):
        import torch
        B, T = prompts.shape
        V = self.cfg.vocab
        tok = torch.from_numpy(np.ascontiguousarray(prompts, np.int32)).cuda()
        logits = torch.empty((B, T, V) if all_logits else (B, V), dtype=torch.float32, device="cuda")
        nxt = torch.full((B,), -1, dtype=torch.int32, device="cuda")
        nz = None if noise is None else torch.from_numpy(noise).cuda()
        self.model.prefill(self.kv, tok, 1 if all_logits else 0, logits, nxt, nz)
        torch.cuda.synchronize()
        return logits.cpu().numpy(), nxt.cpu().numpy()

    def decode(self, tokens: np.ndarray, positions: np.ndarray, noise=None):
        import torch
        B = tokens.size
        V = self.cfg.vocab
        t = torch.from_numpy(np.ascontiguousarray(tokens, np.int32)).cuda()
        p = torch.from_numpy(np.ascontiguousarray(positions, np.int32)).cuda()
        logits = torch.full((B, V), float("nan"), dtype=torch.float32, device="cuda")
        nxt = torch.full((B,), -1, dtype=torch.int32, device="cuda")
        nz = None if noise is None else torch.from_numpy(np.ascontiguousarray(noise, np.float32)).cuda()
        self.model.decode_step(self.kv, t, p, nz, logits, nxt)
        torch.cuda.synchronize()
        return logits.cpu().numpy(), nxt.cpu().numpy()

    def status(self) -> int:
        return self.model.status()


def greedy_session(cfg, blob, prompts: np.ndarray, steps: int, check_seqs, all_logits=False, max_seq=None):
    """Prefill `prompts` [B,T], decode `steps` greedy steps on the GPU; replay the
    GPU's tokens through the oracle for sequences `check_seqs` and compare every
    logits row. Returns the max error seen."""
    B, T = prompts.shape
    run = Run(cfg, blob, B, max_seq or (T + steps + 1))
    lg, nxt = run.prefill(prompts, all_logits)
    fed = []
    step_logits = []
    cur = nxt.copy()
    for s in range(steps):
        fed.append(cur.copy())
        l, n = run.decode(cur, np.full(B, T + s, np.int32))
        step_logits.append(l)
        cur = n
    assert run.status() == 0
    tol = tol_for(cfg)
    om = orc.OracleModel(cfg, blob)
    worst = 0.0
    for b in check_seqs:
        seq = om.new_seq(T + steps + 1)
        if all_logits:
            ref = seq.prefill(prompts[b], all_positions=True)
            worst = max(worst, check_logits(lg[b], ref, tol, f"prefill seq {b} (all positions)"))
            ref_last = ref[-1]
        else:
            ref_last = seq.prefill(prompts[b])
            worst = max(worst, check_logits(lg[b], ref_last, tol, f"prefill seq {b}"))
        check_token(int(nxt[b]), ref_last, None, f"prefill seq {b}")
        for s in range(steps):
            ref = seq.step(int(fed[s][b]))
            worst = max(worst, check_logits(step_logits[s][b], ref, tol, f"decode seq {b} step {s}"))
            nt = int(fed[s + 1][b]) if s + 1 < steps else None
            if nt is not None:
                check_token(nt, ref, None, f"decode seq {b} step {s}")
    return worst
