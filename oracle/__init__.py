"""CPU oracle of the Prox two-stage sparse SwiGLU FFN (fp64, plain C).

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library
never calls it and it never calls the CUDA library.

Each function wraps one routine of ``prox_oracle.c`` (which cites the Prox
pages step by step) and takes/returns numpy arrays in the library's storage
formats: bf16 as uint16 bit patterns, proxies as packed uint8 plus fp32
scales. Outputs are fp64 where the method produces real numbers.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(_build.build())
        _declare(_lib)
    return _lib


_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")


class _Opt:
    """ndpointer that also accepts None (NULL)."""

    def __init__(self, base):
        self.base = base

    def from_param(self, obj):
        if obj is None:
            return None
        return self.base.from_param(obj)


def _declare(L):
    i, f, d = C.c_int, C.c_float, C.c_double
    L.oracle_quantize_proxy.argtypes = [i, i, _u16p, _u8p, _f32p]
    L.oracle_quantize_proxy.restype = None
    L.oracle_stage1_token.argtypes = [i, i, _u16p, f, _u8p, _f32p, _u8p, _f32p, f,
                                      _Opt(_u8p), _Opt(_f64p), _Opt(_f64p), _Opt(_f64p),
                                      _Opt(_u8p), i, _Opt(_u16p), _Opt(_u16p)]
    L.oracle_stage1_token.restype = None
    L.oracle_stage2_token.argtypes = [i, i, _u16p, _u16p, _u16p, _u16p, _u8p,
                                      _Opt(_f64p), _f64p, i]
    L.oracle_stage2_token.restype = None
    L.oracle_forward.argtypes = [i, i, i, _u16p, f, f, _u16p, _u16p, _u16p, _u8p, _f32p,
                                 _u8p, _f32p, _Opt(_u8p), _Opt(_u8p), _Opt(_u8p),
                                 _Opt(_f64p), _Opt(_f64p), _f64p, i, i, _Opt(_u16p), _Opt(_u16p)]
    L.oracle_forward.restype = C.c_int
    L.oracle_quantile_rank.argtypes = [C.c_long, d]
    L.oracle_quantile_rank.restype = C.c_long
    L.oracle_order_statistic.argtypes = [_f64p, C.c_long, d]
    L.oracle_order_statistic.restype = C.c_float
    L.oracle_calibrate.argtypes = [i, i, i, _u16p, _u8p, _f32p, _u8p, _f32p, d, d,
                                   C.POINTER(C.c_float), C.POINTER(C.c_float), i, i,
                                   _Opt(_u16p), _Opt(_u16p)]
    L.oracle_calibrate.restype = None
    L.oracle_hist_quantile.argtypes = [_f32p, C.c_long, d, C.c_long, i]
    L.oracle_hist_quantile.restype = C.c_float
    L.oracle_calibrate_hist.argtypes = [i, i, i, _u16p, _u8p, _f32p, _u8p, _f32p, d, d,
                                        C.c_long, i, C.POINTER(C.c_float),
                                        C.POINTER(C.c_float), i, i, _Opt(_u16p), _Opt(_u16p)]
    L.oracle_calibrate_hist.restype = None
    L.oracle_rmsnorm_bf16.argtypes = [i, _f32p, d, _u16p]
    L.oracle_rmsnorm_bf16.restype = None
    L.oracle_allocate.argtypes = [d, d, d, d, C.POINTER(C.c_double), C.POINTER(C.c_double)]
    L.oracle_allocate.restype = None
    L.oracle_effective_sparsity.argtypes = [d, d, d]
    L.oracle_effective_sparsity.restype = C.c_double


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def quantize_proxy(w_cm: np.ndarray):
    """Per-row symmetric INT4 copy of a channel-major weight [d_ff][d_model].
    Returns (q [d_model][d_ff/2] uint8, scale [d_model] fp32)."""
    d_ff, d_model = w_cm.shape
    q = np.zeros((d_model, d_ff // 2), dtype=np.uint8)
    s = np.zeros(d_model, dtype=np.float32)
    lib().oracle_quantize_proxy(d_model, d_ff, _u16(w_cm), q, s)
    return q, s


ACT_SWIGLU, ACT_GEGLU = 0, 1   # gate activation: SiLU (SwiGLU) or GELU (GeGLU)


def stage1(x, tau_x, q_up, s_up, q_gate, s_gate, tau_s, act=ACT_SWIGLU, pw_up=None,
           pw_gate=None):
    """Stage 1 for one token. Returns dict mask_x, u, g, s (fp64), mask_s.
    With pw_up/pw_gate (bf16 [d_ff][d_model]) the proxy is those weights."""
    d_model = x.shape[-1]
    d_ff = q_up.shape[1] * 2
    out = dict(mask_x=np.zeros(d_model, np.uint8), u=np.zeros(d_ff), g=np.zeros(d_ff),
               s=np.zeros(d_ff), mask_s=np.zeros(d_ff, np.uint8))
    lib().oracle_stage1_token(d_model, d_ff, _u16(x), float(tau_x), q_up, s_up, q_gate,
                              s_gate, float(tau_s), out["mask_x"], out["u"], out["g"],
                              out["s"], out["mask_s"], int(act), _opt16(pw_up), _opt16(pw_gate))
    return out


def _opt16(a):
    return None if a is None else _u16(a)


def stage2(x, w_up_cm, w_gate_cm, w_down, mask_s, act=ACT_SWIGLU):
    """Stage 2 for one token given its channel mask. Returns (s_exact, y)."""
    d_ff, d_model = w_up_cm.shape
    s = np.zeros(d_ff)
    y = np.zeros(d_model)
    lib().oracle_stage2_token(d_model, d_ff, _u16(x), _u16(w_up_cm), _u16(w_gate_cm),
                              _u16(w_down), np.ascontiguousarray(mask_s, np.uint8), s, y,
                              int(act))
    return s, y


def forward(x, tau_x, tau_s, layer: dict, proxy: dict, mask_s_in=None, n_threads=0,
            want=("mask_x", "mask_s", "s_proxy", "s_exact"), act=ACT_SWIGLU):
    """Forward over a batch x [b][d_model]. ``layer`` holds w_up_cm, w_gate_cm,
    w_down; ``proxy`` holds q_up, s_up, q_gate, s_gate. With ``mask_s_in``
    [b][d_ff] Stage 2 uses that mask instead of the oracle's own.
    Returns a dict with y [b][d_model] fp64, the requested extras and
    ``threads``."""
    x = _u16(np.atleast_2d(x))
    b, d_model = x.shape
    d_ff = layer["w_up_cm"].shape[0]
    out = {"y": np.zeros((b, d_model))}
    if "mask_x" in want:
        out["mask_x"] = np.zeros((b, d_model), np.uint8)
    if "mask_s" in want:
        out["mask_s"] = np.zeros((b, d_ff), np.uint8)
    if "s_proxy" in want:
        out["s_proxy"] = np.zeros((b, d_ff))
    if "s_exact" in want:
        out["s_exact"] = np.zeros((b, d_ff))
    ms_in = None if mask_s_in is None else np.ascontiguousarray(mask_s_in, np.uint8)
    out["threads"] = lib().oracle_forward(
        d_model, d_ff, b, x, float(tau_x), float(tau_s), _u16(layer["w_up_cm"]),
        _u16(layer["w_gate_cm"]), _u16(layer["w_down"]), proxy["q_up"], proxy["s_up"],
        proxy["q_gate"], proxy["s_gate"], ms_in, out.get("mask_x"), out.get("mask_s"),
        out.get("s_proxy"), out.get("s_exact"), out["y"], int(n_threads), int(act),
        _opt16(proxy.get("pw_up")), _opt16(proxy.get("pw_gate")))
    return out


def quantile_rank(n: int, keep: float) -> int:
    return lib().oracle_quantile_rank(int(n), float(keep))


def order_statistic(v: np.ndarray, keep: float) -> float:
    v = np.ascontiguousarray(v, dtype=np.float64).ravel()
    return float(np.float32(lib().oracle_order_statistic(v, v.size, float(keep))))


def calibrate(x_cal, proxy: dict, keep_x: float, keep_s: float, n_threads=0, act=ACT_SWIGLU):
    """Thresholds (tau_x, tau_s) as fp32 values (returned as Python floats)."""
    x_cal = _u16(np.atleast_2d(x_cal))
    n, d_model = x_cal.shape
    d_ff = proxy["q_up"].shape[1] * 2
    tx, ts = C.c_float(), C.c_float()
    lib().oracle_calibrate(d_model, d_ff, n, x_cal, proxy["q_up"], proxy["s_up"],
                           proxy["q_gate"], proxy["s_gate"], float(keep_x), float(keep_s),
                           C.byref(tx), C.byref(ts), int(n_threads), int(act),
                           _opt16(proxy.get("pw_up")), _opt16(proxy.get("pw_gate")))
    return tx.value, ts.value


HIST_SAMPLES, HIST_BINS = 200_000, 4096   # the pages' per-layer calibration budget


def hist_quantile(v, keep: float, max_samples: int = HIST_SAMPLES,
                  bins: int = HIST_BINS) -> float:
    """Histogram threshold of |v| (fp32 values, pooled order) for `keep`."""
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    return float(lib().oracle_hist_quantile(v, v.size, float(keep), int(max_samples), int(bins)))


def calibrate_hist(x_cal, proxy: dict, keep_x: float, keep_s: float,
                   max_samples: int = HIST_SAMPLES, bins: int = HIST_BINS, n_threads=0, act=0):
    """Histogram thresholds (tau_x, tau_s): each from at most max_samples pooled
    magnitudes and a histogram of `bins` bins (see oracle_hist_quantile)."""
    x_cal = _u16(np.atleast_2d(x_cal))
    n, d_model = x_cal.shape
    d_ff = proxy["q_up"].shape[1] * 2
    tx, ts = C.c_float(), C.c_float()
    lib().oracle_calibrate_hist(d_model, d_ff, n, x_cal, proxy["q_up"], proxy["s_up"],
                                proxy["q_gate"], proxy["s_gate"], float(keep_x), float(keep_s),
                                int(max_samples), int(bins), C.byref(tx), C.byref(ts),
                                int(n_threads), int(act), _opt16(proxy.get("pw_up")),
                                _opt16(proxy.get("pw_gate")))
    return tx.value, ts.value


def rmsnorm_bf16(h, eps: float = 1e-6) -> np.ndarray:
    """Stack pre-norm: bf16 bits of h / sqrt(mean(h^2) + eps) per row of h (fp32)."""
    h = np.ascontiguousarray(np.atleast_2d(h), dtype=np.float32)
    out = np.empty(h.shape, dtype=np.uint16)
    for t in range(h.shape[0]):
        lib().oracle_rmsnorm_bf16(h.shape[1], h[t], float(eps), out[t])
    return out


def allocate(e: float, alpha: float = 1.0 / 3.0, s1_max: float = 0.7,
             s2_anchor: float = 0.7):
    s1, s2 = C.c_double(), C.c_double()
    lib().oracle_allocate(e, alpha, s1_max, s2_anchor, C.byref(s1), C.byref(s2))
    return s1.value, s2.value


def effective_sparsity(s1: float, s2: float, alpha: float = 1.0 / 3.0) -> float:
    return lib().oracle_effective_sparsity(s1, s2, alpha)


def make_proxy_bf16(layer: dict) -> dict:
    """The bf16-proxy ablation: the proxy is the original bf16 weight (the INT4
    codes and scales below are unused placeholders of the right shapes)."""
    d_ff, d_model = layer["w_up_cm"].shape
    z8 = np.zeros((d_model, d_ff // 2), np.uint8)
    z32 = np.zeros(d_model, np.float32)
    return {"q_up": z8, "s_up": z32, "q_gate": z8, "s_gate": z32,
            "pw_up": layer["w_up_cm"], "pw_gate": layer["w_gate_cm"]}


def make_proxy(layer: dict) -> dict:
    q_up, s_up = quantize_proxy(layer["w_up_cm"])
    q_gate, s_gate = quantize_proxy(layer["w_gate_cm"])
    return {"q_up": q_up, "s_up": s_up, "q_gate": q_gate, "s_gate": s_gate}
