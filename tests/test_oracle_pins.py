"""Pins of the CPU oracle against what the Prox pages and the mathematics fix.

Each test names the passage it follows. None of them retypes the oracle's
formula: the checks are special cases that reduce to library routines
(numpy matmul, scipy's logistic function, numpy SVD), hand-worked values,
brute force over all subsets on tiny inputs, closed forms and invariants.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import expit

import oracle
from free_ffn_activation_b200 import synth as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(h):
    return S.bf16_to_f32(h).astype(np.float64)


def dense_swiglu(x, L):
    """Textbook dense SwiGLU FFN(x) = (x W_up (.) SiLU(x W_gate)) W_down
    (translated arXiv page, section 2.1), evaluated with numpy matmul and
    scipy's logistic sigmoid. W_up = w_up_cm^T in the pages' orientation."""
    xd = f64(x)
    u = xd @ f64(L["w_up_cm"]).T
    g = xd @ f64(L["w_gate_cm"]).T
    return (u * g * expit(g)) @ f64(L["w_down"])


def small_layer(d, f, seed=0, sigma=0.02, layer=0):
    return S.make_layer(S.LayerSpec(d, f, sigma=sigma, seed=seed, layer=layer))


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# --------------------------------------------------------------------------
# INT4 proxy quantisation (blog, "Stage 1": symmetric per-row INT4 copies)
# --------------------------------------------------------------------------

def _golden_rows():
    rows = []
    for line in open(os.path.join(GOLDEN, "int4_rows.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        w, sc, by = [p.strip() for p in line.split("|")]
        rows.append(([float(v) for v in w.split()], int(sc, 16), bytes.fromhex(by)))
    return rows


def test_int4_hand_worked_rows():
    rows = _golden_rows()
    W = np.array([r[0] for r in rows], dtype=np.float64)  # [d_model][d_ff]
    w_bf16 = S.to_bf16(W)
    assert np.array_equal(f64(w_bf16), W)  # fixture values are exact in bf16
    q, s = oracle.quantize_proxy(np.ascontiguousarray(w_bf16.T))  # channel-major in
    for i, (_, scale_bits, packed) in enumerate(rows):
        assert int(s[i:i + 1].view(np.uint32)[0]) == scale_bits, i
        assert bytes(q[i]) == packed, (i, bytes(q[i]).hex())


def test_int4_properties_random():
    L = small_layer(64, 256)
    q, s = oracle.quantize_proxy(L["w_up_cm"])
    W = f64(L["w_up_cm"]).T  # [d_model][d_ff]
    lo = (q & 0xF).astype(np.int64)
    hi = (q >> 4).astype(np.int64)
    codes = np.empty((64, 256), dtype=np.int64)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    codes = np.where(codes >= 8, codes - 16, codes)
    assert codes.min() >= -7 and codes.max() <= 7
    assert np.all(np.abs(codes).max(axis=1) == 7)          # row max maps to +-7
    rec = codes * s.astype(np.float64)[:, None]
    assert np.all(np.abs(rec - W) <= 0.5 * s[:, None] * (1 + 1e-6))   # half-step error
    # symmetric: negating the weights negates every code and keeps the scales
    qn, sn = oracle.quantize_proxy(np.ascontiguousarray(L["w_up_cm"] ^ np.uint16(0x8000)))
    assert np.array_equal(sn, s)
    cn = np.empty((64, 256), dtype=np.int64)
    cn[:, 0::2] = (qn & 0xF)
    cn[:, 1::2] = (qn >> 4)
    cn = np.where(cn >= 8, cn - 16, cn)
    assert np.array_equal(cn, -codes)


# --------------------------------------------------------------------------
# Stage 2 and the dense special case (blog "Stage 2"; arXiv section 2.1)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("d,f", [(64, 192), (256, 768)])
def test_zero_thresholds_give_dense_swiglu(d, f):
    L = small_layer(d, f, seed=3)
    # exact ties with a zero threshold: a channel with all-zero up weights has
    # s~ = 0 exactly and an input coordinate equal to 0 has |x_i| = 0; the
    # masks use >= (blog "Stage 1"), so both are kept at tau = 0.
    L["w_up_cm"][[1, f - 2], :] = 0
    P = oracle.make_proxy(L)
    x = S.make_tokens(5, d, seed=3)
    x[:, 3] = 0
    out = oracle.forward(x, 0.0, 0.0, L, P)
    assert out["s_proxy"][:, 1].tolist() == [0.0] * 5
    assert out["mask_x"].all() and out["mask_s"].all()
    assert rel(out["y"], dense_swiglu(x, L)) < 1e-12


def test_stage2_uses_full_x_whatever_tau_x():
    # Stage 2 computes Pi_out(x, W, m_s) on the full x (blog "Stage 2"), so with
    # tau_s = 0 the output is the dense SwiGLU even when tau_x masks inputs.
    L = small_layer(128, 384, seed=4)
    P = oracle.make_proxy(L)
    x = S.make_tokens(4, 128, seed=4)
    out = oracle.forward(x, 1.0, 0.0, L, P)
    assert 0.2 < out["mask_x"].mean() < 0.6
    assert out["mask_s"].all()
    assert rel(out["y"], dense_swiglu(x, L)) < 1e-12


def test_masked_output_matches_diag_formulation():
    # y = Pi_in(s_sp, W_down, m_s) equals (s (.) m) W_down with s the exact
    # dense intermediate state (blog "Why the SwiGLU intermediate state": the
    # output is the sum over channels of s_i W_down[i, :]).
    L = small_layer(96, 256, seed=5)
    P = oracle.make_proxy(L)
    x = S.make_tokens(3, 96, seed=5)
    rng = np.random.default_rng(0)
    m = (rng.random((3, 256)) < 0.3).astype(np.uint8)
    out = oracle.forward(x, 0.5, 0.0, L, P, mask_s_in=m)
    xd = f64(x)
    u = xd @ f64(L["w_up_cm"]).T
    g = xd @ f64(L["w_gate_cm"]).T
    s = u * g * expit(g)
    assert rel(out["y"], (s * m) @ f64(L["w_down"])) < 1e-12
    assert rel(out["s_exact"], s * m) < 1e-12


def test_error_isolation_output_depends_only_on_mask():
    # Proxy values never reach the output (blog "Ranking" / "Stage 2"): with the
    # channel mask fixed, a different proxy gives the same y bit for bit.
    L = small_layer(64, 128, seed=6)
    P = oracle.make_proxy(L)
    P_bad = oracle.make_proxy(small_layer(64, 128, seed=99))
    x = S.make_tokens(2, 64, seed=6)
    m = oracle.forward(x, 0.7, 1e-4, L, P)["mask_s"]
    y1 = oracle.forward(x, 0.7, 1e-4, L, P, mask_s_in=m)["y"]
    y2 = oracle.forward(x, 0.7, 1e-4, L, P_bad, mask_s_in=m)["y"]
    assert np.array_equal(y1, y2)


# --------------------------------------------------------------------------
# Stage 1 proxy (blog "Stage 1"; arXiv section 2.2 input-sparse projection)
# --------------------------------------------------------------------------

def _int4_exact_layer(d, f, seed):
    """Weights that INT4 represents exactly: W[i,j] = 2^-e_i * q_ij with
    integer |q| <= 7 and a +-7 in every row, so W~ = W."""
    rng = np.random.default_rng(seed)
    qv = rng.integers(-7, 8, size=(d, f))
    qv[np.arange(d), rng.integers(0, f, size=d)] = 7 * rng.choice([-1, 1], size=d)
    e = rng.integers(3, 9, size=d)
    W = qv * (2.0 ** -e)[:, None]
    w_cm = np.ascontiguousarray(S.to_bf16(W).T)
    assert np.array_equal(f64(w_cm).T, W)
    return W, qv, e, w_cm


def test_proxy_with_exact_int4_weights_is_input_sparse_product():
    d, f = 48, 64
    Wu, qu, eu, wu_cm = _int4_exact_layer(d, f, 1)
    Wg, qg, eg, wg_cm = _int4_exact_layer(d, f, 2)
    qup, sup = oracle.quantize_proxy(wu_cm)
    qgt, sgt = oracle.quantize_proxy(wg_cm)
    assert np.array_equal(sup.astype(np.float64), 2.0 ** -eu)
    x = S.make_tokens(1, d, seed=7)[0]
    xd = f64(x)
    for tau in (0.0, 0.6, 1.5):
        o = oracle.stage1(x, tau, qup, sup, qgt, sgt, 0.0)
        keep = o["mask_x"].astype(bool)
        # Pi_in(x, W, m) = x_[I(m)] W_[I(m), :]
        assert rel(o["u"], xd[keep] @ Wu[keep, :]) < 1e-13
        assert rel(o["g"], xd[keep] @ Wg[keep, :]) < 1e-13
        assert rel(o["s"], o["u"] * o["g"] * expit(o["g"])) < 1e-13
        if tau == 0.0:
            assert keep.all()


def test_input_sparsity_residual_bound():
    # blog "Ranking": ||xW - x_sp W||_2 = ||rW||_2 <= ||r||_2 ||W||_2 with
    # r = x - x_sp; ||W||_2 is the spectral norm (numpy SVD).
    d, f = 64, 96
    Wu, _, _, wu_cm = _int4_exact_layer(d, f, 11)
    Wg, _, _, wg_cm = _int4_exact_layer(d, f, 12)
    qup, sup = oracle.quantize_proxy(wu_cm)
    qgt, sgt = oracle.quantize_proxy(wg_cm)
    norm2 = np.linalg.norm(Wu, 2)
    for seed in range(20):
        x = S.make_tokens(1, d, seed=100 + seed)[0]
        full = oracle.stage1(x, 0.0, qup, sup, qgt, sgt, 0.0)["u"]
        sp = oracle.stage1(x, 0.9, qup, sup, qgt, sgt, 0.0)
        r = f64(x) * (1 - sp["mask_x"])
        lhs = np.linalg.norm(full - sp["u"])
        assert lhs <= np.linalg.norm(r) * norm2 * (1 + 1e-12)
        assert lhs > 0


def test_magnitude_mask_minimises_residual_bruteforce():
    # blog "Ranking": at a fixed keep count, keeping the largest |x_i| minimises
    # the l2 residual. d = 8, every subset of every size enumerated.
    d, f = 8, 16
    L = small_layer(d, f, seed=8)
    P = oracle.make_proxy(L)
    for seed in range(10):
        x = S.make_tokens(1, d, seed=200 + seed)[0]
        xd = f64(x)
        mags = np.sort(np.unique(np.abs(xd)))[::-1]
        for k in range(1, len(mags) + 1):
            tau = mags[k - 1]
            m = oracle.stage1(x, tau, P["q_up"], P["s_up"], P["q_gate"], P["s_gate"], 0.0)["mask_x"]
            kept = int(m.sum())
            best = min(itertools.combinations(range(d), kept),
                       key=lambda c: (np.linalg.norm(np.delete(xd, list(c))), c))
            res_mask = np.linalg.norm(xd * (1 - m))
            assert abs(res_mask - np.linalg.norm(np.delete(xd, list(best)))) < 1e-15
            assert kept >= k


def test_channel_mask_bruteforce_d8_f16():
    # blog "Stage 1": [m_s]_j = 1[|s~_j| >= tau_s]. Setting tau_s to the k-th
    # largest |s~| must select the size-k subset with the largest total |s~|
    # (enumerating all C(16, k) subsets), and y must match the diag(m) form.
    d, f = 8, 16
    L = small_layer(d, f, seed=9, sigma=0.5)
    P = oracle.make_proxy(L)
    x = S.make_tokens(1, d, seed=9)[0]
    base = oracle.stage1(x, 0.5, P["q_up"], P["s_up"], P["q_gate"], P["s_gate"], 0.0)
    sabs = np.abs(base["s"])
    assert len(np.unique(sabs)) == f
    order = np.sort(sabs)[::-1]
    xd = f64(x)
    u = xd @ f64(L["w_up_cm"]).T
    g = xd @ f64(L["w_gate_cm"]).T
    s_exact = u * g * expit(g)
    for k in range(1, f + 1):
        tau = float(np.float32(order[k - 1]))
        if tau > order[k - 1]:   # fp32 rounding up would drop the k-th channel
            tau = float(np.nextafter(np.float32(order[k - 1]), np.float32(0)))
        o = oracle.stage1(x, 0.5, P["q_up"], P["s_up"], P["q_gate"], P["s_gate"], tau)
        best = max(itertools.combinations(range(f), k), key=lambda c: sabs[list(c)].sum())
        want = np.zeros(f, np.uint8)
        want[list(best)] = 1
        assert np.array_equal(o["mask_s"], want), k
        y = oracle.forward(x, 0.5, tau, L, P)["y"][0]
        assert rel(y, (s_exact * want) @ f64(L["w_down"])) < 1e-13


def test_batch_forward_equals_per_token_and_thread_invariant():
    L = small_layer(128, 256, seed=10)
    P = oracle.make_proxy(L)
    x = S.make_tokens(6, 128, seed=10)
    a = oracle.forward(x, 0.7, 1e-4, L, P, n_threads=1)
    b = oracle.forward(x, 0.7, 1e-4, L, P, n_threads=4)
    for key in ("y", "mask_x", "mask_s", "s_proxy", "s_exact"):
        assert np.array_equal(a[key], b[key]), key
    for t in range(6):
        o = oracle.stage1(x[t], 0.7, P["q_up"], P["s_up"], P["q_gate"], P["s_gate"], 1e-4)
        assert np.array_equal(o["mask_s"], a["mask_s"][t])
        _, y = oracle.stage2(x[t], L["w_up_cm"], L["w_gate_cm"], L["w_down"], o["mask_s"])
        assert np.array_equal(y, a["y"][t])


# --------------------------------------------------------------------------
# Calibration (blog "Stage 1": offline per-layer thresholds; "Evidence":
# thresholds from calibration activations) -- exact order statistic reading
# --------------------------------------------------------------------------

def test_order_statistic_definition_bruteforce():
    rng = np.random.default_rng(1)
    for n in (1, 2, 7, 10, 33):
        v = rng.standard_normal(n) * 3
        for keep in (0.0, 0.1, 0.3, 0.5, 0.7, 1.0):
            tau = oracle.order_statistic(v, keep)
            rank = oracle.quantile_rank(n, keep)
            exact = math.floor((1 - Fraction(str(keep))) * n)   # rational arithmetic
            assert rank == min(n - 1, max(0, exact))
            a = np.abs(v)
            t64 = np.sort(a)[rank]
            assert tau == float(np.float32(t64))
            assert (a < t64).sum() <= rank < (a <= t64).sum()


def test_calibrated_keep_fractions():
    L = small_layer(256, 768, seed=0)
    P = oracle.make_proxy(L)
    xc = S.make_tokens(256, 256, stream="x_cal")
    tx, ts = oracle.calibrate(xc, P, 0.5, 0.3)
    ax = np.abs(f64(xc))
    assert abs((ax >= tx).mean() - 0.5) < 0.01
    sv = np.stack([oracle.stage1(xc[t], tx, P["q_up"], P["s_up"], P["q_gate"], P["s_gate"], 0.0)["s"]
                   for t in range(256)])
    n = sv.size
    assert abs((np.abs(sv) >= ts).mean() - 0.3) <= 3.0 / n
    # held-out tokens keep roughly the same fractions
    x = S.make_tokens(64, 256)
    o = oracle.forward(x, tx, ts, L, P)
    assert abs(o["mask_x"].mean() - 0.5) < 0.02
    assert abs(o["mask_s"].mean() - 0.3) < 0.03


# --------------------------------------------------------------------------
# Compute budget (blog "Compute budget")
# --------------------------------------------------------------------------

def test_budget_split_matches_printed_value():
    s1, s2 = oracle.allocate(0.7)
    assert s1 == pytest.approx(0.7)
    assert abs(s2 - 0.7667) < 5e-5          # printed: s2 ~= 0.7667
    assert oracle.effective_sparsity(s1, s2) == pytest.approx(0.7, abs=1e-12)
    # e = 1 - C/3 with C = 2 alpha (1 - s1) + 3 (1 - s2)
    for e in (0.4, 0.5, 0.6, 0.7, 0.8):
        s1, s2 = oracle.allocate(e)
        assert 0.0 <= s1 <= 0.7 + 1e-12
        cost = 2 * (1 / 3) * (1 - s1) + 3 * (1 - s2)
        assert 1 - cost / 3 == pytest.approx(e, abs=1e-12)


# ---------------------------------------------------------------------------
# Stack pre-norm (the stacked-layer benchmark on top of the Prox FFN; not on
# the Prox pages): x = bf16(h / sqrt(mean(h^2) + eps)), unit gain
# ---------------------------------------------------------------------------

def _bf16_bits(v):
    return int(np.array([v], np.float32).view(np.uint32)[0] >> 16)


def test_rmsnorm_closed_forms():
    # one nonzero coordinate: mean(h^2) = 1 for h = (2, 0, 0, 0), so x = h
    x = oracle.rmsnorm_bf16(np.array([[2, 0, 0, 0]], np.float32), eps=0.0)
    assert x.tolist() == [[_bf16_bits(2.0), 0, 0, 0]]
    # a constant c with eps = 3 c^2: x = c / sqrt(4 c^2) = 1/2, any d and c
    for c, d in [(3.0, 8), (0.125, 16), (-5.0, 4)]:
        x = oracle.rmsnorm_bf16(np.full((1, d), c, np.float32), eps=3 * c * c)
        assert (x == _bf16_bits(0.5 if c > 0 else -0.5)).all()
    # alternating signs of one magnitude normalise to +-1 exactly
    h = np.array([[7, -7, 7, -7, 7, -7]], np.float32)
    assert oracle.rmsnorm_bf16(h, eps=0.0).tolist() == [[_bf16_bits(v) for v in (1, -1) * 3]]


def test_rmsnorm_scale_invariance():
    # with eps = 0 the norm is invariant under exact (power-of-two) scaling
    rng = np.random.default_rng(3)
    h = rng.standard_normal((4, 256)).astype(np.float32)
    a = oracle.rmsnorm_bf16(h, eps=0.0)
    for k in (0.25, 8.0, 1024.0):
        assert np.array_equal(oracle.rmsnorm_bf16(h * np.float32(k), eps=0.0), a)


def test_rmsnorm_ties_to_even_and_eps():
    # eps chosen so that mean(h^2) + eps = 1 exactly: x is h rounded to bf16,
    # and 1 + 2^-8, 1 + 3 * 2^-8 sit exactly halfway between bf16 neighbours
    t0, t1 = 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8
    h = np.array([[t0, t1, -t0, 0.5]], np.float32)
    eps = 1.0 - float(np.mean(h.astype(np.float64) ** 2))
    x = oracle.rmsnorm_bf16(h, eps=eps)
    assert x.tolist() == [[_bf16_bits(1.0), _bf16_bits(1.0 + 2.0 ** -6),
                           _bf16_bits(-1.0), _bf16_bits(0.5)]]


# ---------------------------------------------------------------------------
# GeGLU variant (blog, "Evidence": GeGLU-style models): the gate activation is
# GELU(z) = z Phi(z); reading adopted: the exact (erf) GELU
# ---------------------------------------------------------------------------

def dense_geglu(x, L):
    """Textbook dense GeGLU FFN(x) = (x W_up (.) GELU(x W_gate)) W_down with
    GELU(z) = z Phi(z), Phi the standard normal CDF from scipy."""
    from scipy.stats import norm
    xd = f64(x)
    u = xd @ f64(L["w_up_cm"]).T
    g = xd @ f64(L["w_gate_cm"]).T
    return (u * g * norm.cdf(g)) @ f64(L["w_down"])


def test_zero_thresholds_give_dense_geglu():
    L = small_layer(32, 64, seed=5)
    P = oracle.make_proxy(L)
    x = S.make_tokens(4, 32, seed=5)
    out = oracle.forward(x, 0.0, 0.0, L, P, act=oracle.ACT_GEGLU)
    assert rel(out["y"], dense_geglu(x, L)) < 1e-12
    # and the SwiGLU output differs (the activation is really switched)
    assert rel(out["y"], dense_swiglu(x, L)) > 1e-3


def test_geglu_proxy_state_identity():
    # GELU(z) - GELU(-z) = z exactly in the reals (Phi(z) + Phi(-z) = 1): the
    # proxy state s~ = u~ GELU(g~) of a layer and of the same layer with the
    # gate negated differ by u~ g~ channel by channel
    L = small_layer(32, 64, seed=6)
    Lneg = dict(L)
    Lneg["w_gate_cm"] = L["w_gate_cm"] ^ np.uint16(0x8000)   # exact negation of bf16
    P, Pn = oracle.make_proxy(L), oracle.make_proxy(Lneg)
    x = S.make_tokens(1, 32, seed=6)[0]
    a = oracle.stage1(x, 0.0, P["q_up"], P["s_up"], P["q_gate"], P["s_gate"], 0.0,
                      act=oracle.ACT_GEGLU)
    b = oracle.stage1(x, 0.0, Pn["q_up"], Pn["s_up"], Pn["q_gate"], Pn["s_gate"], 0.0,
                      act=oracle.ACT_GEGLU)
    assert np.allclose(b["g"], -a["g"], rtol=0, atol=0)
    assert np.allclose(a["s"] - b["s"], a["u"] * a["g"], rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------
# Histogram calibration (blog, "Evidence": at most 200,000 samples and a
# 4,096-bin histogram per layer; readings: every k-th sample, equal bins over
# [0, max], tau = the lower edge of the bin holding the rank-floor sample)
# ---------------------------------------------------------------------------

def test_hist_quantile_hand_worked():
    # 0..15 in 4 bins of width 3.75: counts 4, 4, 4, 4 (15 itself in the top
    # bin); keep 0.5 -> rank 8 -> third bin -> tau = 2 * 3.75
    v = np.arange(16, dtype=np.float32)
    assert oracle.hist_quantile(v, 0.5, bins=4) == 7.5
    # keep 1.0 -> rank 0 -> first bin -> 0; keep 0.0 -> rank 15 (clamped) -> top bin
    assert oracle.hist_quantile(v, 1.0, bins=4) == 0.0
    assert oracle.hist_quantile(v, 0.0, bins=4) == 11.25
    # signs do not matter, and an all-zero input gives 0
    assert oracle.hist_quantile(-v, 0.5, bins=4) == 7.5
    assert oracle.hist_quantile(np.zeros(8, np.float32), 0.5) == 0.0


def test_hist_quantile_subsamples_every_kth():
    # 10 values, at most 4 samples -> every 3rd: 0, 1, 2, 3 (the 100s are
    # skipped); 3 bins of width 1 -> counts 1, 1, 2; rank floor(0.5 * 4) = 2
    v = np.array([0, 100, 100, 1, 100, 100, 2, 100, 100, 3], np.float32)
    assert oracle.hist_quantile(v, 0.5, max_samples=4, bins=3) == 2.0
    # without the budget the 100s dominate
    assert oracle.hist_quantile(v, 0.5, max_samples=1000, bins=3) > 50.0


def test_hist_quantile_brackets_the_order_statistic():
    # with every value sampled, the histogram threshold is the lower edge of
    # the bin that holds the exact rank-floor((1-keep) n) value
    rng = np.random.default_rng(7)
    for n, keep in [(5000, 0.5), (20001, 0.3), (777, 0.9)]:
        v = rng.laplace(size=n).astype(np.float32)
        th = oracle.hist_quantile(v, keep)
        tx = oracle.order_statistic(v.astype(np.float64), keep)
        w = np.float32(np.abs(v).max()) / np.float32(4096)
        assert th <= tx < th + w * 1.0001, (n, keep, th, tx, w)


# ---------------------------------------------------------------------------
# bf16-proxy ablation (blog, "Evidence", ablation A1: the proxy at full
# precision instead of INT4): the proxy is the original weight
# ---------------------------------------------------------------------------

def test_bf16_proxy_at_zero_tau_x_is_the_exact_state():
    # with every input kept, Stage 1 with the bf16 proxy computes the same
    # sums in the same order as Stage 2's exact u and g: s~ == s bit for bit
    L = small_layer(64, 256, seed=2)
    P = oracle.make_proxy_bf16(L)
    x = S.make_tokens(3, 64, seed=2)
    out = oracle.forward(x, 0.0, 0.0, L, P)
    assert np.array_equal(out["s_proxy"], out["s_exact"])


def test_bf16_proxy_masked_state_matches_numpy():
    # with tau_x > 0 the proxy state is (x (.) m_x) W_up  (.) SiLU((x (.) m_x) W_gate)
    L = small_layer(64, 256, seed=4)
    P = oracle.make_proxy_bf16(L)
    x = S.make_tokens(4, 64, seed=4)
    tau_x = 0.7
    out = oracle.forward(x, tau_x, 0.0, L, P)
    xd = f64(x)
    xm = np.where(np.abs(xd) >= tau_x, xd, 0.0)
    u = xm @ f64(L["w_up_cm"]).T
    g = xm @ f64(L["w_gate_cm"]).T
    assert rel(out["s_proxy"], u * g * expit(g)) < 1e-12
