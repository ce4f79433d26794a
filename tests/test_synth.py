"""Pins for the seeded input generators (splitmix64 test vectors, distribution
moments, bf16 round-to-nearest-even, determinism)."""
import math

import numpy as np

import nc_synth as syn


def test_splitmix64_published_vectors():
    # splitmix64 seeded with 0 and with 1234567 (published reference outputs)
    assert syn.splitmix64_at(0, 0) == 0xE220A8397B1DCDAF
    assert syn.splitmix64_at(0, 1) == 0x6E789E6AA1B965F4
    assert syn.splitmix64_at(0, 2) == 0x06C45D188009454F
    assert syn.splitmix64_at(1234567, 0) == 6457827717110365317
    assert syn.splitmix64_at(1234567, 1) == 3203168211198807973


def test_uniform_and_normal_moments():
    u = syn.uniform01(3, 1 << 20)
    assert 0.0 < u.min() and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 2e-3
    cfg = syn.ModelConfig(depth=0, d_model=1024, n_head=8, n_kv_head=1, head_dim=128, mlp_hidden=4096,
                          vocab=512, dtype="f32")
    w = syn.make_blob(cfg, seed=0)
    assert abs(w.mean()) < 1e-4
    assert abs(w.std() - 0.02) < 1e-4
    # approximately Gaussian tails: ~0.27% beyond 3 sigma
    assert abs(np.mean(np.abs(w) > 0.06) - 0.0027) < 5e-4


def test_blob_deterministic_and_bf16_is_rne_of_f32():
    cfg32 = syn.TINY
    cfg16 = syn.ModelConfig(**{**syn.TINY.__dict__, "dtype": "bf16"})
    a, b = syn.make_blob(cfg32, 0), syn.make_blob(cfg32, 0)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, syn.make_blob(cfg32, 1))
    bits = syn.make_blob(cfg16, 0)
    assert np.array_equal(bits, syn.f32_to_bf16_bits(a))
    assert np.max(np.abs(syn.bf16_bits_to_f32(bits) - a) / np.abs(a)) <= 2.0 ** -8


def test_bf16_round_nearest_even_cases():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-8 + 2**-20, -1.0 - 2**-8, 2**-7],
                 dtype=np.float32)
    got = syn.f32_to_bf16_bits(x)
    assert list(got) == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xBF80, 0x3C00]


def test_zipf_tokens():
    V, s = 65536, 1.1
    t = syn.tokens_zipf(11, (1 << 18,), V, s)
    assert t.min() >= 0 and t.max() < V
    H = np.sum(np.arange(1, V + 1, dtype=np.float64) ** -s)
    for r in (1, 2, 10):
        p = r ** -s / H
        assert abs(np.mean(t == r - 1) - p) < 4 * math.sqrt(p / t.size) + 1e-4


def test_uniform_tokens_and_gumbel():
    t = syn.tokens_uniform(1, (4, 1000), 512)
    assert t.shape == (4, 1000) and t.min() >= 0 and t.max() < 512
    g = syn.gumbel(5, (1 << 20,)).astype(np.float64)
    assert abs(g.mean() - 0.5772156649) < 5e-3
    assert abs(g.var() - math.pi ** 2 / 6) < 2e-2


def test_workload_presets():
    w = syn.WORKLOADS
    assert w["tiny"].model.dtype == "f32" and w["tiny"].prompt_len == 16 and w["tiny"].decode_steps == 16
    assert (w["d20_prefill"].batch, w["d20_prefill"].prompt_len) == (8, 2048)
    assert (w["d20_decode"].batch, w["d20_decode"].decode_steps) == (32, 128)
    assert w["d30_rollout"].fork == 16 and w["d30_rollout"].noise_seed == 5
    p = syn.prompt_tokens(w["tiny"])
    assert p.shape == (1, 16) and p.dtype == np.int32
