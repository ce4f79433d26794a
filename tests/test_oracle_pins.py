"""Pins for the CPU oracle: it is checked against what the nanochat pages and
the mathematics fix, never against itself.

The pages (the launch Q&A in "Karpathy再放大招：8000行代碼復現ChatGPT全棧..."
listing the architecture) name the features but print no formulas, weights or
logits. Each test below fixes one feature through a closed form, an invariant
that only the stated feature satisfies, a special case that reduces to a
simpler computation, or a figure the pages print (tests/golden/). Every test
is chosen so that a plausible slip -- a dropped term, a wrong sign or index,
a transposed operand -- fails at least one of them.
"""
import dataclasses
import json
import math
import os

import numpy as np
import pytest

import nc_synth as syn
import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")
RNG = np.random.default_rng(1234)


# ------------------------------------------------------------------ RMSNorm
def test_rmsnorm_closed_form_rms():
    # feature "RMSNorm without learnable params": y = x / sqrt(mean(x^2)+eps)
    # has RMS exactly sqrt(m / (m + eps)), m = mean(x^2).
    for eps in (0.0, 1e-6, 0.5):
        x = RNG.normal(size=37) * 3.0
        y = orc.rmsnorm(x, eps)
        m = np.mean(x * x)
        assert math.isclose(np.sqrt(np.mean(y * y)), math.sqrt(m / (m + eps)), rel_tol=1e-14)
        assert np.all(np.sign(y) == np.sign(x))  # a positive per-row scale


def test_rmsnorm_unit_rms_and_hand_example():
    y = orc.rmsnorm([3.0, 4.0], 0.0)   # mean square 12.5
    r = math.sqrt(12.5)
    assert np.allclose(y, [3.0 / r, 4.0 / r], rtol=0, atol=1e-15)
    x = RNG.normal(size=128)
    assert abs(np.sqrt(np.mean(orc.rmsnorm(x, 0.0) ** 2)) - 1.0) < 1e-15
    # no gain: scale invariant
    assert np.allclose(orc.rmsnorm(7.5 * x, 0.0), orc.rmsnorm(x, 0.0), atol=1e-14)


# --------------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    v = RNG.normal(size=64)
    assert np.array_equal(orc.rope(v, 0, 10000.0), v)


def test_rope_direction_and_pairing():
    # one pair, theta_0 = base^0 = 1: (1, 0) at position 1 -> (cos 1, sin 1)
    assert np.allclose(orc.rope([1.0, 0.0], 1, 10000.0), [math.cos(1), math.sin(1)], atol=1e-15)
    # hd = 4: pairs are (0, 2) and (1, 3); theta_1 = 10000^(-2/4) = 0.01
    p = 25
    out = orc.rope([0.0, 1.0, 0.0, 0.0], p, 10000.0)
    assert np.allclose(out, [0.0, math.cos(0.01 * p), 0.0, math.sin(0.01 * p)], atol=1e-15)
    out = orc.rope([1.0, 0.0, 0.0, 0.0], p, 10000.0)
    assert np.allclose(out, [math.cos(p), 0.0, math.sin(p), 0.0], atol=1e-15)


def test_rope_preserves_pair_norms_and_composes():
    hd = 128
    v = RNG.normal(size=hd)
    r = orc.rope(v, 1234, 10000.0)
    half = hd // 2
    assert np.allclose(np.hypot(r[:half], r[half:]), np.hypot(v[:half], v[half:]), rtol=1e-13)
    assert np.allclose(orc.rope(orc.rope(v, 300, 10000.0), 77, 10000.0), orc.rope(v, 377, 10000.0),
                       atol=1e-12)


def test_rope_dot_depends_only_on_relative_position():
    hd = 128
    q, k = RNG.normal(size=hd), RNG.normal(size=hd)
    for m, n, c in ((5, 2, 100), (0, 9, 1000), (2047, 1, 31)):
        a = orc.rope(q, m, 10000.0) @ orc.rope(k, n, 10000.0)
        b = orc.rope(q, m + c, 10000.0) @ orc.rope(k, n + c, 10000.0)
        assert math.isclose(a, b, rel_tol=1e-11, abs_tol=1e-11)


def test_qk_norm_commutes_with_rope():
    v = RNG.normal(size=128) * 2
    a = orc.rmsnorm(orc.rope(v, 517, 10000.0), 1e-6)
    b = orc.rope(orc.rmsnorm(v, 1e-6), 517, 10000.0)
    assert np.allclose(a, b, atol=1e-14)


# ---------------------------------------------------------------- attention
def test_attention_single_key_returns_value():
    q, K, V = RNG.normal(size=16), RNG.normal(size=(1, 16)), RNG.normal(size=(1, 16))
    assert np.allclose(orc.attend(q, K, V), V[0], atol=1e-15)


def test_attention_identical_keys_average_values():
    k = RNG.normal(size=16)
    K = np.tile(k, (9, 1))
    V = RNG.normal(size=(9, 16))
    assert np.allclose(orc.attend(RNG.normal(size=16), K, V), V.mean(0), atol=1e-14)


def test_attention_weights_sum_to_one():
    n, hd = 50, 32
    y = orc.attend(RNG.normal(size=hd) * 5, RNG.normal(size=(n, hd)), np.ones((n, hd)))
    assert np.allclose(y, 1.0, atol=1e-14)


def test_attention_scale_is_inverse_sqrt_hd():
    # scores s0 = a/sqrt(hd) * |q| and s1 = 0; choose them to differ by ln 3, so
    # the softmax weights are exactly 3/4 and 1/4.
    hd = 64
    q = np.zeros(hd); q[0] = 1.0
    K = np.zeros((2, hd)); K[0, 0] = math.log(3.0) * math.sqrt(hd)
    V = RNG.normal(size=(2, hd))
    assert np.allclose(orc.attend(q, K, V), 0.75 * V[0] + 0.25 * V[1], atol=1e-14)


def test_attention_is_a_function_of_the_key_set():
    n, hd = 12, 16
    q, K, V = RNG.normal(size=hd), RNG.normal(size=(n, hd)), RNG.normal(size=(n, hd))
    perm = RNG.permutation(n)
    assert np.allclose(orc.attend(q, K, V), orc.attend(q, K[perm], V[perm]), atol=1e-14)


# ------------------------------------------------------------ softcap, pick
def test_softcap_bounds_and_values():
    cap = 15.0
    z = np.linspace(-100, 100, 2001)
    out = np.array([orc.softcap(v, cap) for v in z])
    assert np.all(np.abs(out) < cap)
    assert orc.softcap(0.0, cap) == 0.0
    assert math.isclose(orc.softcap(cap * math.atanh(0.5), cap), cap / 2, rel_tol=1e-14)
    assert math.isclose(orc.softcap(1e-6, cap), 1e-6, rel_tol=1e-12)  # slope 1 at 0
    assert np.allclose(out, -out[::-1], atol=0)  # odd


def test_argmax_lowest_index_and_noise():
    v = np.array([1.0, 3.0, 2.0, 3.0])
    assert orc.argmax(v) == 1
    assert orc.argmax(v, np.array([0, 0, 1.5, 0], np.float32)) == 2
    assert orc.argmax(np.zeros(5)) == 0


# ------------------------------------------------------------- the model
CFG = syn.TINY
BLOB = syn.make_blob(CFG, seed=0)


def _model(cfg=CFG, blob=BLOB):
    return orc.OracleModel(cfg, blob)


def _tensor(blob, cfg, name):
    off, r, c = syn.tensor_offsets(cfg)[name]
    return blob[off:off + r * c].reshape(r, c)


def _toks(T, seed=7):
    return syn.tokens_uniform(seed, (T,), CFG.vocab)


def test_incremental_decode_equals_full_recompute():
    m = _model()
    toks = _toks(24)
    full = m.forward_full(toks)
    s = m.new_seq(32)
    inc = np.stack([s.step(t) for t in toks])
    assert np.max(np.abs(full - inc)) < 1e-10
    # cache-filled prefill, then steps, equals the full forward over T+3
    s2 = m.new_seq(32)
    last = s2.prefill(toks[:20])
    assert np.max(np.abs(last - full[19])) < 1e-10
    for t in range(20, 24):
        assert np.max(np.abs(s2.step(toks[t]) - full[t])) < 1e-10


def test_causal_prefix_unaffected_by_future_tokens():
    m = _model()
    a, b = _toks(16, seed=7), _toks(16, seed=8)
    b[:9] = a[:9]
    assert np.max(np.abs(m.forward_full(a)[:9] - m.forward_full(b)[:9])) < 1e-12
    assert np.max(np.abs(m.forward_full(a)[9:] - m.forward_full(b)[9:])) > 1e-3


def test_no_positional_embedding_only_relative_positions():
    # RoPE and no absolute position embedding: shifting every position by c
    # leaves all logits unchanged.
    m = _model()
    toks = _toks(16)
    base = m.forward_full(toks, pos0=0)
    for c in (1, 37, 1000):
        assert np.max(np.abs(m.forward_full(toks, pos0=c) - base)) < 1e-9


def test_mqa_equals_mha_with_replicated_kv_head():
    H = CFG.n_head
    mha = dataclasses.replace(CFG, n_kv_head=H)
    parts = []
    for name, r, c in syn.tensor_list(CFG):
        t = _tensor(BLOB, CFG, name)
        if name.endswith(".wk") or name.endswith(".wv"):
            t = np.tile(t, (H, 1))
        parts.append(t.ravel())
    blob_mha = np.concatenate(parts)
    toks = _toks(12)
    a = _model().forward_full(toks)
    b = orc.OracleModel(mha, blob_mha).forward_full(toks)
    assert np.max(np.abs(a - b)) < 1e-12


def test_gqa_equals_mha_with_each_kv_head_repeated_for_its_group():
    # four query heads in two groups: heads 0, 1 read KV head 0, heads 2, 3
    # read KV head 1 (head h reads KV head h // (H / Hkv)); the MHA model
    # with each KV head's Wk, Wv rows repeated for its group computes the same
    # function, while a model with the heads interleaved (h % Hkv) does not
    gqa = syn.ModelConfig(depth=1, d_model=256, n_head=4, n_kv_head=2, head_dim=64, mlp_hidden=1024, vocab=512,
                          dtype="f32")
    blob = syn.make_blob(gqa, 31)
    H, Hkv, hd = gqa.n_head, gqa.n_kv_head, gqa.head_dim
    G = H // Hkv
    mha = dataclasses.replace(gqa, n_kv_head=H)
    grouped, interleaved = [], []
    for name, r, c in syn.tensor_list(gqa):
        t = _tensor(blob, gqa, name)
        if name.endswith(".wk") or name.endswith(".wv"):
            heads = t.reshape(Hkv, hd, c)
            grouped.append(np.repeat(heads, G, axis=0).ravel())
            interleaved.append(np.tile(heads, (G, 1, 1)).ravel())
        else:
            grouped.append(t.ravel())
            interleaved.append(t.ravel())
    toks = syn.tokens_uniform(11, (10,), gqa.vocab)
    a = orc.OracleModel(gqa, blob).forward_full(toks)
    b = orc.OracleModel(mha, np.concatenate(grouped)).forward_full(toks)
    wrong = orc.OracleModel(mha, np.concatenate(interleaved)).forward_full(toks)
    assert np.max(np.abs(a - b)) < 1e-12
    assert np.max(np.abs(a - wrong)) > 1e-6


def _edited(edits):
    blob = BLOB.copy()
    for name, fn in edits.items():
        off, r, c = syn.tensor_offsets(CFG)[name]
        blob[off:off + r * c] = fn(blob[off:off + r * c].reshape(r, c)).astype(np.float32).ravel()
    return blob


def test_depth_zero_is_norm_embed_norm_head_softcap():
    cfg0 = dataclasses.replace(CFG, depth=0)
    wte, wlm = _tensor(BLOB, CFG, "wte"), _tensor(BLOB, CFG, "wlm")
    blob0 = np.concatenate([wte.ravel(), wlm.ravel()])
    toks = _toks(5)
    got = orc.OracleModel(cfg0, blob0).forward_full(toks)
    for i, t in enumerate(toks):
        h = orc.rmsnorm(orc.rmsnorm(wte[t].astype(np.float64), 1e-6), 1e-6)
        z = wlm.astype(np.float64) @ h  # library matmul as one step
        want = np.array([orc.softcap(v, CFG.softcap) for v in z])
        assert np.max(np.abs(got[i] - want)) < 1e-12


def test_blocks_with_zero_output_projections_are_identity():
    # With Wo = Wproj = 0 each block adds nothing: pins the residual form.
    zero = lambda w: np.zeros_like(w)
    edits = {}
    for l in range(CFG.depth):
        edits[f"h{l}.wo"] = zero
        edits[f"h{l}.wproj"] = zero
    toks = _toks(8)
    got = orc.OracleModel(CFG, _edited(edits)).forward_full(toks)
    cfg0 = dataclasses.replace(CFG, depth=0)
    blob0 = np.concatenate([_tensor(BLOB, CFG, "wte").ravel(), _tensor(BLOB, CFG, "wlm").ravel()])
    want = orc.OracleModel(cfg0, blob0).forward_full(toks)
    assert np.max(np.abs(got - want)) < 1e-12


def test_mlp_is_relu_squared():
    # relu(c z)^2 = c^2 relu(z)^2 for c > 0: scaling Wfc by c equals scaling
    # Wproj by c^2 (a plain relu would give c, a gelu neither).
    c = 1.7
    toks = _toks(10)
    a = orc.OracleModel(CFG, _edited({f"h{l}.wfc": (lambda w: w * c) for l in range(CFG.depth)}))
    b = orc.OracleModel(CFG, _edited({f"h{l}.wproj": (lambda w: w * c * c) for l in range(CFG.depth)}))
    assert np.max(np.abs(a.forward_full(toks) - b.forward_full(toks))) < 1e-5
    # and negative pre-activations contribute nothing: flipping every Wfc row
    # sign gives a different model
    d = orc.OracleModel(CFG, _edited({f"h{l}.wfc": (lambda w: -w) for l in range(CFG.depth)}))
    assert np.max(np.abs(d.forward_full(toks) - _model().forward_full(toks))) > 1e-3


def test_norm_after_embedding_and_qk_norm():
    toks = _toks(10)
    base = _model().forward_full(toks)
    # embedding rows scaled by 4: the norm after the embedding removes it
    got = orc.OracleModel(CFG, _edited({"wte": lambda w: w * 4.0})).forward_full(toks)
    assert np.max(np.abs(got - base)) < 1e-4
    # q and k scaled by 3: QK norm removes it (attention unchanged)
    ed = {}
    for l in range(CFG.depth):
        ed[f"h{l}.wq"] = lambda w: w * 3.0
        ed[f"h{l}.wk"] = lambda w: w * 3.0
    got = orc.OracleModel(CFG, _edited(ed)).forward_full(toks)
    assert np.max(np.abs(got - base)) < 1e-4
    # v scaled by 3 is NOT removed (values are not normed)
    got = orc.OracleModel(CFG, _edited({"h0.wv": lambda w: w * 3.0})).forward_full(toks)
    assert np.max(np.abs(got - base)) > 1e-3


def test_first_position_ignores_queries_and_keys():
    # one key at position 0: softmax weight 1 whatever q.k is
    toks = _toks(6)
    ed = {f"h{l}.{n}": (lambda w: RNG.normal(size=w.shape) * 0.05) for l in range(CFG.depth) for n in ("wq", "wk")}
    a = _model().forward_full(toks)
    b = orc.OracleModel(CFG, _edited(ed)).forward_full(toks)
    assert np.max(np.abs(a[0] - b[0])) < 1e-12
    assert np.max(np.abs(a[1:] - b[1:])) > 1e-4


def test_logits_within_softcap_and_fork_copy():
    m = _model()
    toks = _toks(12)
    out = m.forward_full(toks)
    assert np.all(np.abs(out) < CFG.softcap)
    s = m.new_seq(20)
    s.prefill(toks[:8])
    f = m.new_seq(20)
    f.copy_from(s)
    assert f.length == 8
    for t in toks[8:]:
        assert np.array_equal(s.step(t), f.step(t))


def test_bf16_blob_is_read_as_rounded_values():
    cfg = dataclasses.replace(CFG, dtype="bf16")
    bits = syn.f32_to_bf16_bits(BLOB)
    wide = syn.bf16_bits_to_f32(bits)
    toks = _toks(6)
    a = orc.OracleModel(cfg, bits).forward_full(toks)
    b = orc.OracleModel(CFG, wide).forward_full(toks)
    assert np.array_equal(a, b)


# ------------------------------------------------------- the pages' figures
def test_pages_figures_pin_the_width_reading():
    g = json.load(open(GOLDEN))
    assert syn.D20.vocab == g["vocab"]["value"]
    # widths from depth: d = 64*depth, hd = 128, F = 4d. With one KV head per
    # query head (MHA) d20 has 560,988,160 params, the pages' "~560M"; the MQA
    # model the feature list names has 502,005,760.
    mha = syn.depth_config(20, n_kv_head=syn.D20.n_head)
    n_mha = syn.param_count(mha)
    assert n_mha == 560_988_160
    assert abs(n_mha / g["d20_params"]["value"] - 1) < g["d20_params"]["approx_rel"]
    assert syn.param_count(syn.D20) == 502_005_760
    assert syn.param_count(syn.D26) == 949_092_352
    assert syn.param_count(syn.D30) == 1_372_323_840
    # Chinchilla 20:1 and 6ND
    tokens = g["d20_tokens"]["chinchilla_ratio"] * g["d20_params"]["value"]
    assert tokens == g["d20_tokens"]["value"]
    flops = 6 * n_mha * tokens
    assert abs(flops / g["d20_train_flops"]["value"] - 1) < g["d20_train_flops"]["approx_rel"]
    # the oracle's own parameter count agrees with the blob layout
    m = orc.OracleModel(syn.TINY, BLOB)
    assert BLOB.size == syn.param_count(syn.TINY) == 491_520


# ------------------------------------------------------ sampled token pick
def _first_max(a):
    return int(np.flatnonzero(a == a.max())[0])


def test_sample_topk_special_cases_reduce_to_argmax():
    # temperature 0: the greedy pick, whatever the noise and k
    z = RNG.standard_normal(300).astype(np.float32)
    g = syn.gumbel(11, (300,), stream=1)
    assert orc.sample_topk(z, g, 0.0, 7) == _first_max(z)
    # k = 1: only the largest logit is a candidate
    assert orc.sample_topk(z, g, 0.6, 1) == _first_max(z)
    # k = n (and k = 0), temperature 1: argmax of z + g, the pick the engine
    # makes without sampling parameters
    want = _first_max((z + g).astype(np.float32))
    assert orc.sample_topk(z, g, 1.0, 0) == want == orc.sample_topk(z, g, 1.0, 300)
    # no noise: any temperature > 0 and any k keep the greedy pick
    assert orc.sample_topk(z, None, 2.5, 40) == _first_max(z)


def test_sample_topk_membership_and_ties():
    z = np.array([3.0, 5.0, 5.0, 5.0, 1.0], np.float32)
    # k = 2 keeps the two lowest indices of the three tied 5s: index 3 is out
    # however large its noise, and equal scores go to the lower index
    assert orc.sample_topk(z, np.array([0, 0, 0, 9, 0], np.float32), 1.0, 2) == 1
    assert orc.sample_topk(z, np.array([0, 0, 0.5, 9, 0], np.float32), 1.0, 2) == 2
    # k = 3 lets index 3 in
    assert orc.sample_topk(z, np.array([0, 0, 0, 9, 0], np.float32), 1.0, 3) == 3
    # the lowest logit can win only once it is a candidate
    g = np.array([0, 0, 0, 0, 50], np.float32)
    assert orc.sample_topk(z, g, 1.0, 4) != 4 and orc.sample_topk(z, g, 1.0, 5) == 4


def test_sample_topk_draws_follow_the_tempered_topk_softmax():
    # Gumbel-max: with i.i.d. standard Gumbel noise the pick is distributed as
    # softmax(z / T) over the top-k logits and never picks outside them
    z = np.array([0.5, 2.0, 1.0, -1.0, 1.5, 0.2], np.float32)
    T, k, n = 0.8, 4, 40000
    g = syn.gumbel(21, (n, z.size), stream=0)
    counts = np.bincount([orc.sample_topk(z, g[i], T, k) for i in range(n)], minlength=z.size)
    keep = np.argsort(-z, kind="stable")[:k]
    p = np.zeros(z.size)
    e = np.exp((z[keep].astype(np.float64) - z.max()) / T)
    p[keep] = e / e.sum()
    freq = counts / n
    assert np.all(counts[p == 0] == 0)
    assert np.all(np.abs(freq - p) <= 4.5 * np.sqrt(p * (1 - p) / n) + 1e-3), (freq, p)
