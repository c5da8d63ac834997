"""Pins of the seeded input generator (shared by both sides of every parity
test): published SplitMix64 values, bf16 rounding cases, and the closed-form
moments of the distributions the workloads use."""
import math

import numpy as np

from free_ffn_activation_b200 import synth as S


def test_splitmix64_published_first_output():
    # SplitMix64 seeded with state 0 emits 0xE220A8397B1DCDAF first, and with
    # state 1234567 emits 6457827717110365317, 3203168211198807973, ...
    # (the reference sequence of Vigna's splitmix64.c / Java's SplittableRandom).
    z = S._mix(np.array([S._GOLDEN], dtype=np.uint64))
    assert int(z[0]) == 0xE220A8397B1DCDAF
    with np.errstate(over="ignore"):
        st = np.uint64(1234567) + np.arange(1, 3, dtype=np.uint64) * S._GOLDEN
    got = S._mix(st)
    assert [int(v) for v in got] == [6457827717110365317, 3203168211198807973]


def test_counter_based_and_chunk_invariant():
    a = S.raw_u64(7, "w_up", 0, 1000)
    b = S.raw_u64(7, "w_up", 500, 500)
    assert np.array_equal(a[500:], b)
    assert not np.array_equal(S.raw_u64(7, "w_up", 0, 100), S.raw_u64(7, "w_gate", 0, 100))
    assert not np.array_equal(S.raw_u64(7, "w_up", 0, 100), S.raw_u64(8, "w_up", 0, 100))
    n1 = S._normal_chunk(3, "s", 0, 101)
    n2 = np.concatenate([S._normal_chunk(3, "s", 0, 37), S._normal_chunk(3, "s", 37, 64)])
    assert np.array_equal(n1, n2)


def test_bf16_round_to_nearest_even():
    f = np.array([1.0, 1.0 / 3.0, -2.0, 0.0], dtype=np.float32)
    assert list(S.to_bf16(f)) == [0x3F80, 0x3EAB, 0xC000, 0x0000]
    ties = np.array([0x3F808000, 0x3F818000, 0x3F808001], dtype=np.uint32).view(np.float32)
    assert list(S.to_bf16(ties)) == [0x3F80, 0x3F82, 0x3F81]
    h = np.arange(0, 0x7F80, 97, dtype=np.uint16)
    assert np.array_equal(S.to_bf16(S.bf16_to_f32(h)), h)


def _mc_check(samples, fn, expected, n_batches=100):
    est = np.array([fn(b) for b in np.array_split(samples, n_batches)])
    se = est.std(ddof=1) / math.sqrt(n_batches)
    assert abs(est.mean() - expected) < 5 * se, (est.mean(), expected, se)


def test_laplace_energy_retention_closed_form():
    # Prox deep-dive blog, "Why the SwiGLU intermediate state": for a Laplace
    # variable, dropping the smallest 70% by magnitude keeps about 87.9% of the
    # squared energy. With |X| ~ Exp(1) and cut t = ln(10/3) the exact value is
    # 0.3 * ((1 + t)^2 + 1) / 2 = 0.878624.
    t = math.log(10.0 / 3.0)
    closed = 0.3 * ((1.0 + t) ** 2 + 1.0) / 2.0
    assert abs(closed - 0.878624) < 1e-6
    assert round(closed, 3) == 0.879
    v = S.laplace(0, "retention", 10_000_000)

    def retained(b):
        a = np.sort(np.abs(b))
        k = int(0.7 * a.size)
        return float((a[k:] ** 2).sum() / (a ** 2).sum())

    _mc_check(v, retained, closed)


def test_laplace_and_normal_moments():
    v = S.laplace(1, "mom", 2_000_000)
    _mc_check(v, lambda b: float(np.abs(b).mean()), 1.0)   # E|X| = b
    _mc_check(v, lambda b: float((b ** 2).mean()), 2.0)    # Var = 2 b^2
    _mc_check(v, lambda b: float(b.mean()), 0.0)
    n = S.normal(2, "mom", 2_000_000, sigma=0.02)
    _mc_check(n, lambda b: float((b ** 2).mean()), 0.02 ** 2)
    _mc_check(n, lambda b: float((b ** 4).mean()), 3 * 0.02 ** 4)
    _mc_check(n, lambda b: float(b.mean()), 0.0)


def test_layer_and_token_recipes():
    spec = S.LayerSpec(256, 768, sigma=0.02, seed=0)
    L = S.make_layer(spec)
    assert L["w_up_cm"].shape == (768, 256) and L["w_down"].shape == (768, 256)
    assert L["w_up_cm"].dtype == np.uint16
    w = S.bf16_to_f32(L["w_gate_cm"]).astype(np.float64)
    assert abs(w.std() - 0.02) < 0.02 * 0.01
    L2 = S.make_layer(S.LayerSpec(256, 768, sigma=0.02, seed=0, layer=1))
    assert not np.array_equal(L["w_up_cm"], L2["w_up_cm"])
    x = S.make_tokens(64, 4096, outlier_frac=0.001)
    idx = S.outlier_channels(0, 4096, 0.001)
    assert len(idx) == 4
    xf = np.abs(S.bf16_to_f32(x))
    others = np.delete(xf, idx, axis=1)
    assert xf[:, idx].mean() > 10 * others.mean()
    xc = S.make_tokens(64, 4096, stream="x_cal")
    assert not np.array_equal(x[:, :8], xc[:, :8])
