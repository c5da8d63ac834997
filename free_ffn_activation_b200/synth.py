"""Seeded synthetic inputs for the Prox sparse SwiGLU FFN.

This module is the only code shared by the CUDA path's callers and the CPU
oracle's callers. It holds no step of the method: it draws random numbers,
shapes them into the distributions the workloads ask for, and rounds them to
bf16 storage. Nothing here masks, quantises, thresholds or multiplies weights.

Generator
---------
Every value is a pure function of ``(seed, stream, index)``:

* ``splitmix64``: the published SplitMix64 output function (Steele, Lea and
  Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014):
  ``z = key + (index + 1) * 0x9E3779B97F4A7C15`` followed by the two
  xor-shift-multiply rounds and a final xor-shift.
* ``key(seed, stream)``: SplitMix64 of the seed, xor the 64-bit FNV-1a hash of
  the stream name, mixed once more. Streams are named (``"w_up"``,
  ``"x_eval"``...), so adding a stream never shifts another one.
* uniform in the open interval (0, 1): ``((z >> 11) + 0.5) * 2**-53``.
* normal: Box-Muller on consecutive uniform pairs (cos for even indices,
  sin for odd ones).
* Laplace(0, b): ``-b * sign(v) * ln(1 - 2|v|)`` with ``v = u - 1/2``.

bf16 storage: fp64 -> fp32 (round to nearest even) -> bf16 (round to nearest
even on the upper 16 bits). The result is a ``uint16`` array holding bf16 bit
patterns, which is what both the library and the oracle consume.

Workload recipes (shapes, distributions, outlier placement) live in
``LayerSpec`` / ``make_layer`` / ``make_tokens``; the stream names make the
calibration tokens and the evaluation tokens disjoint.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def _fnv1a64(name: str) -> int:
    h = 0xCBF29CE484222325
    for b in name.encode():
        h ^= b
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def stream_key(seed: int, stream: str) -> np.uint64:
    """64-bit key of a named stream under a seed."""
    with np.errstate(over="ignore"):
        k = _mix(np.array([np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + _GOLDEN], dtype=np.uint64))
        k = _mix(k ^ np.uint64(_fnv1a64(stream)))
    return k[0]


def raw_u64(seed: int, stream: str, start: int, count: int) -> np.ndarray:
    """SplitMix64 outputs ``start .. start+count-1`` of a stream."""
    key = stream_key(seed, stream)
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(key + idx * _GOLDEN)


def uniform(seed: int, stream: str, start: int, count: int) -> np.ndarray:
    """Uniform draws in (0, 1), fp64."""
    z = raw_u64(seed, stream, start, count)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def _normal_chunk(seed: int, stream: str, start: int, count: int) -> np.ndarray:
    # element i uses the uniform pair (2*(i//2), 2*(i//2)+1)
    p0 = start // 2
    p1 = (start + count + 1) // 2
    u = uniform(seed, stream, 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
    r = np.sqrt(-2.0 * np.log(u[:, 0]))
    th = 2.0 * np.pi * u[:, 1]
    pairs = np.empty((p1 - p0, 2), dtype=np.float64)
    pairs[:, 0] = r * np.cos(th)
    pairs[:, 1] = r * np.sin(th)
    flat = pairs.reshape(-1)
    off = start - 2 * p0
    return flat[off: off + count]


def _laplace_chunk(seed: int, stream: str, start: int, count: int) -> np.ndarray:
    v = uniform(seed, stream, start, count) - 0.5
    return -np.sign(v) * np.log1p(-2.0 * np.abs(v))


def _chunked(fn, seed: int, stream: str, count: int, out_fn) -> np.ndarray:
    """Evaluate ``fn`` over [0, count) in chunks on a thread pool."""
    out = np.empty(count, dtype=np.uint16 if out_fn is not None else np.float64)
    starts = list(range(0, count, _CHUNK))

    def work(s):
        n = min(_CHUNK, count - s)
        v = fn(seed, stream, s, n)
        out[s: s + n] = out_fn(v) if out_fn is not None else v

    workers = max(1, min(len(starts), os.cpu_count() or 1))
    if workers == 1:
        for s in starts:
            work(s)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(work, starts))
    return out


def normal(seed: int, stream: str, count: int, sigma: float = 1.0) -> np.ndarray:
    return _chunked(_normal_chunk, seed, stream, count, None) * sigma


def laplace(seed: int, stream: str, count: int, b: float = 1.0) -> np.ndarray:
    return _chunked(_laplace_chunk, seed, stream, count, None) * b


def to_bf16(v: np.ndarray) -> np.ndarray:
    """fp64/fp32 values -> bf16 bit patterns (uint16), round to nearest even."""
    bits = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((bits >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    return ((bits + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, stream: str, count: int, sigma: float) -> np.ndarray:
    return _chunked(lambda s, st, a, n: _normal_chunk(s, st, a, n) * sigma,
                    seed, stream, count, to_bf16)


# ---------------------------------------------------------------------------
# workload recipes
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class LayerSpec:
    """One SwiGLU FFN layer: shapes, weight std and the seed of its streams."""
    d_model: int
    d_ff: int
    sigma: float = 0.02
    seed: int = 0
    layer: int = 0

    def stream(self, name: str) -> str:
        return f"L{self.layer}/{name}"


def make_layer(spec: LayerSpec) -> dict:
    """bf16 weights of one layer, in the storage layouts the library takes.

    ``w_up_cm``, ``w_gate_cm``: [d_ff][d_model], channel j is row j.
    ``w_down``: [d_ff][d_model], row j multiplies intermediate channel j.
    Entries are i.i.d. N(0, sigma^2) rounded to bf16.
    """
    n = spec.d_model * spec.d_ff
    shape = (spec.d_ff, spec.d_model)
    return {
        "w_up_cm": normal_bf16(spec.seed, spec.stream("w_up"), n, spec.sigma).reshape(shape),
        "w_gate_cm": normal_bf16(spec.seed, spec.stream("w_gate"), n, spec.sigma).reshape(shape),
        "w_down": normal_bf16(spec.seed, spec.stream("w_down"), n, spec.sigma).reshape(shape),
    }


def outlier_channels(seed: int, d_model: int, frac: float) -> np.ndarray:
    """Fixed input coordinates that carry outliers: round(frac * d_model) of
    them (at least one when frac > 0), picked by a seeded permutation."""
    k = int(round(frac * d_model))
    if frac > 0:
        k = max(k, 1)
    if k == 0:
        return np.zeros(0, dtype=np.int64)
    u = uniform(seed, "outlier_channels", 0, d_model)
    return np.sort(np.argsort(u, kind="stable")[:k])


def make_tokens(n: int, d_model: int, seed: int = 0, stream: str = "x_eval",
                outlier_frac: float = 0.0, outlier_scale: float = 20.0) -> np.ndarray:
    """``n`` decode tokens, bf16 [n][d_model], entries Laplace(0, 1).

    With ``outlier_frac > 0`` a fixed set of coordinates (the same for every
    token, drawn by ``outlier_channels``) is multiplied by ``outlier_scale``
    before rounding, mimicking the fixed outlier channels of real hidden
    states."""
    v = laplace(seed, stream, n * d_model).reshape(n, d_model)
    if outlier_frac > 0:
        v[:, outlier_channels(seed, d_model, outlier_frac)] *= outlier_scale
    return to_bf16(v)
