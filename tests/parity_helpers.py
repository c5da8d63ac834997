"""Shared pieces of the GPU parity tests: one layer case with its oracle
proxies and thresholds, and the comparison of a device forward with the
oracle under the parity bars (Prox pages' method):
  * m_x: bit-exact (same inputs, same fp32 thresholds).
  * m_s and the ascending kept-channel lists: bit-exact except on channels
    whose oracle |s~| lies within 1e-3 * tau_s of tau_s (the "band"); band
    channels must be fewer than 0.1% of all channels on large samples.
  * y: the oracle's Stage 2 fed the device's m_s; per token
    ||y_gpu - y_ref||_2 / ||y_ref||_2 <= 2e-3.
"""
import numpy as np

import oracle
from free_ffn_activation_b200 import prox as P
from free_ffn_activation_b200 import synth as S

BAND = 1e-3
Y_TOL = 2e-3


def to_dev_bf16(a, dev):
    return P.as_bf16(a, dev).contiguous()


class Case:
    """One layer with its oracle proxies, device layer and thresholds."""

    def __init__(self, d, f, n_tok, n_cal, sigma=0.02, seed=0, outlier=0.0, layer=0,
                 keep_x=0.5, keep_s=0.3, dev="cuda", act=oracle.ACT_SWIGLU,
                 proxy_kind=P.PROXY_INT4):
        self.spec = S.LayerSpec(d, f, sigma=sigma, seed=seed, layer=layer)
        self.L = S.make_layer(self.spec)
        self.Por = (oracle.make_proxy_bf16(self.L) if proxy_kind == P.PROXY_BF16
                    else oracle.make_proxy(self.L))
        self.dev = dev
        self.act = act
        self.layer = P.ProxLayer.from_weights(self.L["w_up_cm"], self.L["w_gate_cm"],
                                              self.L["w_down"], device=dev, activation=act,
                                              proxy_kind=proxy_kind)
        self.x = S.make_tokens(n_tok, d, seed=seed, stream="x_eval", outlier_frac=outlier)
        self.x_cal = S.make_tokens(n_cal, d, seed=seed, stream="x_cal", outlier_frac=outlier)
        self.keep_x, self.keep_s = keep_x, keep_s
        self.tau_x, self.tau_s = oracle.calibrate(self.x_cal, self.Por, keep_x, keep_s, act=act)

    def xdev(self, rows=None):
        x = self.x if rows is None else self.x[rows]
        return to_dev_bf16(x, self.dev)


def check_forward(case, rows, out, tag=""):
    """Compare a device ForwardOut for tokens `rows` with the oracle."""
    x = case.x[rows]
    ref = oracle.forward(x, case.tau_x, case.tau_s, case.L, case.Por, act=case.act)
    mx = out.mask_x.cpu().numpy()
    ms = out.mask_s.cpu().numpy()
    idx = out.idx_s.cpu().numpy()
    cnt = out.count_s.cpu().numpy()
    assert np.array_equal(mx, ref["mask_x"]), f"{tag} mask_x differs"
    sabs = np.abs(ref["s_proxy"])
    band = np.abs(sabs - case.tau_s) <= BAND * case.tau_s
    diff = ms != ref["mask_s"]
    assert not np.any(diff & ~band), f"{tag} m_s differs outside the band"
    n_band = int(band.sum())
    if band.size >= 20000:   # the 0.1% rule is a rate: checked on large samples
        assert n_band < 1e-3 * band.size, f"{tag} band holds {n_band} of {band.size}"
    for t in range(len(rows)):
        kept = np.flatnonzero(ms[t])
        assert cnt[t] == kept.size
        assert np.array_equal(idx[t, :cnt[t]], kept), f"{tag} idx_s token {t}"
    y_ref = oracle.forward(x, case.tau_x, case.tau_s, case.L, case.Por, mask_s_in=ms,
                           want=(), act=case.act)["y"]
    y = out.y.cpu().numpy().astype(np.float64)
    num = np.linalg.norm(y - y_ref, axis=1)
    den = np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    worst = float((num / den).max())
    assert worst <= Y_TOL, f"{tag} y rel err {worst}"
    print(f"[parity{tag}] tokens={len(rows)} band={n_band}/{band.size} "
          f"mask_s diffs={int(diff.sum())} y_rel_max={worst:.2e} "
          f"keep_x={mx.mean():.3f} keep_s={ms.mean():.3f}")
    return worst
