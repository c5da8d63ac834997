"""Thin Python binding of libprox (C ABI in ``include/prox.h``).

Argument marshalling only: every step of the method runs in the CUDA
kernels behind the C ABI. Tensors are torch CUDA tensors (PyTorch supplies
device memory and streams); calls are enqueued on the current torch stream.
If ``libprox.so`` is missing or cannot be loaded, the first call raises: there
is no fallback of any kind.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libprox.so")

PROX_OK, PROX_EINVAL, PROX_ENOMEM, PROX_ECUDA, PROX_ETIMEOUT, PROX_EDEVICE = range(6)

ABI_FUNCTIONS = (
    "prox_quantize_proxy", "prox_workspace_bytes", "prox_ffn_forward", "prox_proxy_state",
    "prox_max_batch_per_pass", "prox_ffn_stage1", "prox_ffn_stage2",
    "prox_calibrate_workspace_bytes", "prox_calibrate", "prox_allocate",
    "prox_last_device_status", "prox_status_str", "prox_set_stage2_engine",
    "prox_set_stage1_engine",
)

# Stage-2 and Stage-1 engines (prox_set_stage2_engine, prox_set_stage1_engine)
ENGINE_AUTO, ENGINE_SIMT, ENGINE_TC = 0, 1, 2


class ProxError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} (status {status})")


class _Layer(C.Structure):
    _fields_ = [("d_model", C.c_int), ("d_ff", C.c_int),
                ("w_up_cm", C.c_void_p), ("w_gate_cm", C.c_void_p), ("w_down", C.c_void_p),
                ("q_up", C.c_void_p), ("q_gate", C.c_void_p),
                ("s_up", C.c_void_p), ("s_gate", C.c_void_p), ("activation", C.c_int),
                ("proxy_kind", C.c_int)]


ACT_SWIGLU, ACT_GEGLU = 0, 1   # PROX_ACT_SWIGLU, PROX_ACT_GEGLU
PROXY_INT4, PROXY_BF16 = 0, 1  # PROX_PROXY_INT4, PROX_PROXY_BF16


_lib = None


def lib() -> C.CDLL:
    """The loaded libprox (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libprox.so not built ({LIB_PATH}); run "
                              "`python -m free_ffn_activation_b200.build` or __graft_entry__.build()")
        L = C.CDLL(LIB_PATH)
        vp, i, f, d, sz = C.c_void_p, C.c_int, C.c_float, C.c_double, C.c_size_t
        L.prox_quantize_proxy.argtypes = [i, i, vp, vp, vp, vp]
        L.prox_workspace_bytes.argtypes = [i, i, i]
        L.prox_workspace_bytes.restype = sz
        L.prox_ffn_forward.argtypes = [C.POINTER(_Layer), vp, i, f, f, vp, vp, vp, vp, vp, vp, sz, vp]
        L.prox_ffn_forward_static.argtypes = [C.POINTER(_Layer), vp, i, f, f, vp, vp, vp, vp,
                                               vp, vp]
        L.prox_rmsnorm_bf16.argtypes = [i, i, vp, f, vp, vp]
        L.prox_bf16_proxy.argtypes = [i, i, vp, vp, vp]
        L.prox_ffn_block.argtypes = [C.POINTER(_Layer), vp, i, f, f, f, vp, vp, vp, vp, vp, vp,
                                     vp, sz, vp]
        L.prox_proxy_state.argtypes = [C.POINTER(_Layer), vp, i, f, vp, vp, vp, sz, vp]
        L.prox_calibrate_workspace_bytes.argtypes = [i, i, i]
        L.prox_calibrate_workspace_bytes.restype = sz
        L.prox_calibrate.argtypes = [C.POINTER(_Layer), vp, i, d, d, C.POINTER(C.c_float),
                                     C.POINTER(C.c_float), vp, sz, vp]
        L.prox_calibrate_histogram.argtypes = [C.POINTER(_Layer), vp, i, d, d, C.c_long, i,
                                               C.POINTER(C.c_float), C.POINTER(C.c_float), vp,
                                               sz, vp]
        L.prox_allocate.argtypes = [d, d, d, d, C.POINTER(C.c_double), C.POINTER(C.c_double)]
        L.prox_last_device_status.argtypes = [vp, sz, vp, C.POINTER(C.c_uint32)]
        L.prox_status_str.argtypes = [i]
        L.prox_status_str.restype = C.c_char_p
        L.prox_set_stage2_engine.argtypes = [i]
        L.prox_set_stage2_engine.restype = C.c_int
        L.prox_set_stage1_engine.argtypes = [i]
        L.prox_set_stage1_engine.restype = C.c_int
        L.prox_max_batch_per_pass.argtypes = [i]
        L.prox_max_batch_per_pass.restype = C.c_int
        L.prox_ffn_stage1.argtypes = [C.POINTER(_Layer), vp, i, f, f, vp, vp, vp, vp, sz, vp]
        L.prox_ffn_stage2.argtypes = [C.POINTER(_Layer), vp, i, vp, vp, vp, vp, sz, vp]
        L.prox_static_last_device_status.argtypes = [vp, C.POINTER(C.c_uint32)]
        L.prox_test_set_wait.argtypes = [C.c_uint32, i]
        L.prox_test_set_wait.restype = None
        L.prox_test_set_stamps.argtypes = [vp]
        L.prox_test_set_stamps.restype = None
        L.prox_test_set_skip.argtypes = [i, i]
        L.prox_test_set_skip.restype = None
        for name in ("prox_quantize_proxy", "prox_ffn_forward", "prox_ffn_forward_static",
                     "prox_rmsnorm_bf16", "prox_ffn_block", "prox_calibrate_histogram",
                     "prox_bf16_proxy",
                     "prox_proxy_state",
                     "prox_ffn_stage1", "prox_ffn_stage2",
                     "prox_calibrate", "prox_allocate", "prox_last_device_status",
                     "prox_static_last_device_status"):
            getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().prox_status_str(int(status)).decode()


def _check(status: int, what: str):
    if status != PROX_OK:
        raise ProxError(status, what)


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, shape, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def as_bf16(a, device=None) -> torch.Tensor:
    """bf16 tensor from a uint16 bit-pattern array/tensor or a bf16 tensor."""
    if isinstance(a, torch.Tensor):
        t = a if a.dtype == torch.bfloat16 else a.view(torch.bfloat16)
    else:
        import numpy as np
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t


# ---------------------------------------------------------------------------
# layer + proxies
# ---------------------------------------------------------------------------

@dataclass
class ProxLayer:
    """Device tensors of one layer, in libprox's layouts (see prox.h)."""
    w_up_cm: torch.Tensor      # bf16 [d_ff][d_model]
    w_gate_cm: torch.Tensor    # bf16 [d_ff][d_model]
    w_down: torch.Tensor       # bf16 [d_ff][d_model]
    q_up: torch.Tensor         # uint8 [d_ff/256][d_model][128] (block-tiled)
    q_gate: torch.Tensor
    s_up: torch.Tensor         # fp32 [d_model]
    s_gate: torch.Tensor
    activation: int = 0        # ACT_SWIGLU (SiLU gate) or ACT_GEGLU (GELU gate)
    proxy_kind: int = 0        # PROXY_INT4, or PROXY_BF16: q_* are bf16 tiles
                               # uint16 [d_ff/256][d_model][256], s_* unused (None)

    @property
    def d_model(self) -> int:
        return self.w_up_cm.shape[1]

    @property
    def d_ff(self) -> int:
        return self.w_up_cm.shape[0]

    def cstruct(self) -> _Layer:
        d, f = self.d_model, self.d_ff
        if self.proxy_kind == PROXY_BF16:
            checks = (("q_up", torch.int16, (f // 256, d, 256)),
                      ("q_gate", torch.int16, (f // 256, d, 256)))
        else:
            checks = (("q_up", torch.uint8, (f // 256, d, 128)),
                      ("q_gate", torch.uint8, (f // 256, d, 128)), ("s_up", torch.float32, (d,)),
                      ("s_gate", torch.float32, (d,)))
        for name, dt, shp in (("w_up_cm", torch.bfloat16, (f, d)), ("w_gate_cm", torch.bfloat16, (f, d)),
                              ("w_down", torch.bfloat16, (f, d))) + checks:
            _need(getattr(self, name), dt, shp, name)
        return _Layer(d, f, _ptr(self.w_up_cm), _ptr(self.w_gate_cm), _ptr(self.w_down),
                      _ptr(self.q_up), _ptr(self.q_gate), _ptr(self.s_up), _ptr(self.s_gate),
                      int(self.activation), int(self.proxy_kind))

    @staticmethod
    def from_weights(w_up_cm, w_gate_cm, w_down, device="cuda",
                     activation: int = ACT_SWIGLU, proxy_kind: int = PROXY_INT4) -> "ProxLayer":
        """Upload bf16 weights and build their proxies (INT4, or the bf16
        ablation's tiled copies) on the device."""
        up, gate, down = (as_bf16(w, device).contiguous() for w in (w_up_cm, w_gate_cm, w_down))
        if proxy_kind == PROXY_BF16:
            return ProxLayer(up, gate, down, bf16_proxy(up), bf16_proxy(gate), None, None,
                             int(activation), PROXY_BF16)
        q_up, s_up = quantize_proxy(up)
        q_gate, s_gate = quantize_proxy(gate)
        return ProxLayer(up, gate, down, q_up, q_gate, s_up, s_gate, int(activation))


def bf16_proxy(w_cm: torch.Tensor) -> torch.Tensor:
    """prox_bf16_proxy: block-tiled copy [d_ff/256][d_model][256] (int16 view of
    bf16) of a channel-major bf16 weight [d_ff][d_model]."""
    f, d = w_cm.shape
    _need(w_cm, torch.bfloat16, (f, d), "w_cm")
    q = torch.empty((f // 256, d, 256), dtype=torch.int16, device=w_cm.device)
    _check(lib().prox_bf16_proxy(d, f, _ptr(w_cm), _ptr(q), _stream(w_cm.device)),
           "prox_bf16_proxy")
    return q


def quantize_proxy(w_cm: torch.Tensor):
    """INT4 proxy of a channel-major bf16 weight [d_ff][d_model] ->
    (q uint8 [d_ff/256][d_model][128] block-tiled, scale fp32 [d_model])."""
    f, d = w_cm.shape
    _need(w_cm, torch.bfloat16, (f, d), "w_cm")
    q = torch.empty((f // 256, d, 128), dtype=torch.uint8, device=w_cm.device)
    s = torch.empty((d,), dtype=torch.float32, device=w_cm.device)
    _check(lib().prox_quantize_proxy(d, f, _ptr(w_cm), _ptr(q), _ptr(s), _stream(w_cm.device)),
           "prox_quantize_proxy")
    return q, s


# ---------------------------------------------------------------------------
# forward / stage 1 / calibration
# ---------------------------------------------------------------------------

def workspace_bytes(d_model: int, d_ff: int, batch: int) -> int:
    return int(lib().prox_workspace_bytes(d_model, d_ff, batch))


def workspace(d_model: int, d_ff: int, batch: int, device="cuda") -> torch.Tensor:
    """A zero-filled forward workspace (reusable across calls on one stream)."""
    n = workspace_bytes(d_model, d_ff, batch)
    if n == 0:
        raise ProxError(PROX_EINVAL, "prox_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


@dataclass
class ForwardOut:
    y: torch.Tensor
    mask_x: torch.Tensor | None
    mask_s: torch.Tensor | None
    idx_s: torch.Tensor | None
    count_s: torch.Tensor | None


def ffn_forward(layer: ProxLayer, x: torch.Tensor, tau_x: float, tau_s: float,
                ws: torch.Tensor | None = None, *, want_masks: bool = True,
                out: ForwardOut | None = None) -> ForwardOut:
    """Prox forward for x bf16 [batch][d_model] -> ForwardOut (y fp32)."""
    d, f = layer.d_model, layer.d_ff
    if x.dim() == 1:
        x = x.unsqueeze(0)
    b = x.shape[0]
    _need(x, torch.bfloat16, (b, d), "x")
    dev = x.device
    if ws is None:
        ws = workspace(d, f, b, dev)
    if out is None:
        out = ForwardOut(
            y=torch.empty((b, d), dtype=torch.float32, device=dev),
            mask_x=torch.empty((b, d), dtype=torch.uint8, device=dev) if want_masks else None,
            mask_s=torch.empty((b, f), dtype=torch.uint8, device=dev) if want_masks else None,
            idx_s=torch.empty((b, f), dtype=torch.int32, device=dev) if want_masks else None,
            count_s=torch.empty((b,), dtype=torch.int32, device=dev) if want_masks else None)
    cl = layer.cstruct()
    _check(lib().prox_ffn_forward(C.byref(cl), _ptr(x), b, float(tau_x), float(tau_s), _ptr(out.y),
                                  _ptr(out.mask_x), _ptr(out.mask_s), _ptr(out.idx_s),
                                  _ptr(out.count_s), _ptr(ws), ws.numel(), _stream(dev)),
           "prox_ffn_forward")
    return out


def ffn_forward_static(layer: ProxLayer, x: torch.Tensor, tau_x: float, tau_s: float,
                       *, want_masks: bool = True) -> ForwardOut:
    """prox_ffn_forward_static: the forward on the library's static workspace."""
    d, f = layer.d_model, layer.d_ff
    if x.dim() == 1:
        x = x.unsqueeze(0)
    b = x.shape[0]
    _need(x, torch.bfloat16, (b, d), "x")
    dev = x.device
    out = ForwardOut(
        y=torch.empty((b, d), dtype=torch.float32, device=dev),
        mask_x=torch.empty((b, d), dtype=torch.uint8, device=dev) if want_masks else None,
        mask_s=torch.empty((b, f), dtype=torch.uint8, device=dev) if want_masks else None,
        idx_s=torch.empty((b, f), dtype=torch.int32, device=dev) if want_masks else None,
        count_s=torch.empty((b,), dtype=torch.int32, device=dev) if want_masks else None)
    cl = layer.cstruct()
    _check(lib().prox_ffn_forward_static(C.byref(cl), _ptr(x), b, float(tau_x), float(tau_s),
                                         _ptr(out.y), _ptr(out.mask_x), _ptr(out.mask_s),
                                         _ptr(out.idx_s), _ptr(out.count_s), _stream(dev)),
           "prox_ffn_forward_static")
    return out


STATIC_WORKSPACE_BYTES = 2 << 20  # PROX_STATIC_WORKSPACE_BYTES


def rmsnorm_bf16(h: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    """prox_rmsnorm_bf16: bf16 h / sqrt(mean(h^2) + eps) per row of fp32 h."""
    if h.dim() == 1:
        h = h.unsqueeze(0)
    b, d = h.shape
    _need(h, torch.float32, (b, d), "h")
    x = torch.empty((b, d), dtype=torch.bfloat16, device=h.device)
    _check(lib().prox_rmsnorm_bf16(d, b, _ptr(h), float(eps), _ptr(x), _stream(h.device)),
           "prox_rmsnorm_bf16")
    return x


def ffn_block(layer: ProxLayer, h_in: torch.Tensor, tau_x: float, tau_s: float,
              eps: float = 1e-6, h_out: torch.Tensor | None = None,
              ws: torch.Tensor | None = None, *, want_masks: bool = True):
    """prox_ffn_block: one pre-norm stack layer, h_out = h_in + FFN(RMSNorm(h_in)).
    Returns (h_out, x, ForwardOut with y=None and the masks)."""
    d, f = layer.d_model, layer.d_ff
    if h_in.dim() == 1:
        h_in = h_in.unsqueeze(0)
    b = h_in.shape[0]
    _need(h_in, torch.float32, (b, d), "h_in")
    dev = h_in.device
    if h_out is None:
        h_out = torch.empty_like(h_in)
    if ws is None:
        ws = workspace(d, f, b, dev)
    x = torch.empty((b, d), dtype=torch.bfloat16, device=dev)
    out = ForwardOut(
        y=None,
        mask_x=torch.empty((b, d), dtype=torch.uint8, device=dev) if want_masks else None,
        mask_s=torch.empty((b, f), dtype=torch.uint8, device=dev) if want_masks else None,
        idx_s=torch.empty((b, f), dtype=torch.int32, device=dev) if want_masks else None,
        count_s=torch.empty((b,), dtype=torch.int32, device=dev) if want_masks else None)
    cl = layer.cstruct()
    _check(lib().prox_ffn_block(C.byref(cl), _ptr(h_in), b, float(tau_x), float(tau_s),
                                float(eps), _ptr(h_out), _ptr(x), _ptr(out.mask_x),
                                _ptr(out.mask_s), _ptr(out.idx_s), _ptr(out.count_s), _ptr(ws),
                                ws.numel(), _stream(dev)),
           "prox_ffn_block")
    return h_out, x, out


def ffn_block_raw(layer_struct: _Layer, h_in_ptr: int, batch: int, tau_x: float, tau_s: float,
                  eps: float, h_out_ptr: int, x_ptr: int, ws_ptr: int, ws_bytes: int,
                  stream: int) -> None:
    """prox_ffn_block with raw device pointers (no masks)."""
    _check(lib().prox_ffn_block(C.byref(layer_struct), h_in_ptr, batch, float(tau_x),
                                float(tau_s), float(eps), h_out_ptr, x_ptr, None, None, None,
                                None, ws_ptr, ws_bytes, stream),
           "prox_ffn_block")


def ffn_forward_raw(layer_struct: _Layer, x_ptr: int, batch: int, tau_x: float, tau_s: float,
                    y_ptr: int, ws_ptr: int, ws_bytes: int, stream: int, mask_x=None,
                    mask_s=None, idx_s=None, count_s=None) -> None:
    """The C ABI call with raw device pointers (no tensor checks)."""
    _check(lib().prox_ffn_forward(C.byref(layer_struct), x_ptr, batch, float(tau_x), float(tau_s),
                                  y_ptr, mask_x, mask_s, idx_s, count_s, ws_ptr, ws_bytes, stream),
           "prox_ffn_forward")


def max_batch_per_pass(d_model: int) -> int:
    return int(lib().prox_max_batch_per_pass(int(d_model)))


def set_stage2_engine(engine: int) -> int:
    """Select the Stage-2 engine (ENGINE_AUTO, ENGINE_SIMT, ENGINE_TC) for
    later forward calls in this process; returns the previous one."""
    prev = int(lib().prox_set_stage2_engine(int(engine)))
    if prev < 0:
        raise ProxError(PROX_EINVAL, f"prox_set_stage2_engine({engine})")
    return prev


def set_stage1_engine(engine: int) -> int:
    """Select the Stage-1 engine (ENGINE_AUTO, ENGINE_SIMT, ENGINE_TC) for
    later calls in this process; returns the previous one."""
    prev = int(lib().prox_set_stage1_engine(int(engine)))
    if prev < 0:
        raise ProxError(PROX_EINVAL, f"prox_set_stage1_engine({engine})")
    return prev


class stage1_engine:
    """Context manager: run the enclosed calls with one Stage-1 engine."""

    def __init__(self, engine: int):
        self.engine = engine

    def __enter__(self):
        self.prev = set_stage1_engine(self.engine)
        return self

    def __exit__(self, *exc):
        set_stage1_engine(self.prev)
        return False


class stage2_engine:
    """Context manager: run the enclosed calls with one Stage-2 engine."""

    def __init__(self, engine: int):
        self.engine = engine

    def __enter__(self):
        self.prev = set_stage2_engine(self.engine)
        return self

    def __exit__(self, *exc):
        set_stage2_engine(self.prev)
        return False


def ffn_stage1_raw(layer_struct: _Layer, x_ptr: int, batch: int, tau_x: float, tau_s: float,
                   y_clear_ptr, ws_ptr: int, ws_bytes: int, stream: int, mask_x=None,
                   mask_s=None) -> None:
    """prox_ffn_stage1 with raw device pointers."""
    _check(lib().prox_ffn_stage1(C.byref(layer_struct), x_ptr, batch, float(tau_x), float(tau_s),
                                 y_clear_ptr, mask_x, mask_s, ws_ptr, ws_bytes, stream),
           "prox_ffn_stage1")


def ffn_stage2_raw(layer_struct: _Layer, x_ptr: int, batch: int, y_ptr: int, ws_ptr: int,
                   ws_bytes: int, stream: int, idx_s=None, count_s=None) -> None:
    """prox_ffn_stage2 with raw device pointers."""
    _check(lib().prox_ffn_stage2(C.byref(layer_struct), x_ptr, batch, y_ptr, idx_s, count_s,
                                 ws_ptr, ws_bytes, stream), "prox_ffn_stage2")


def proxy_state(layer: ProxLayer, x: torch.Tensor, tau_x: float, ws: torch.Tensor | None = None):
    """Stage 1 alone: (s~ fp32 [batch][d_ff], mask_x uint8 [batch][d_model])."""
    d, f = layer.d_model, layer.d_ff
    if x.dim() == 1:
        x = x.unsqueeze(0)
    b = x.shape[0]
    _need(x, torch.bfloat16, (b, d), "x")
    if ws is None:
        ws = workspace(d, f, b, x.device)
    s = torch.empty((b, f), dtype=torch.float32, device=x.device)
    mx = torch.empty((b, d), dtype=torch.uint8, device=x.device)
    cl = layer.cstruct()
    _check(lib().prox_proxy_state(C.byref(cl), _ptr(x), b, float(tau_x), _ptr(s), _ptr(mx),
                                  _ptr(ws), ws.numel(), _stream(x.device)), "prox_proxy_state")
    return s, mx


def calibrate(layer: ProxLayer, x_cal: torch.Tensor, keep_x: float, keep_s: float):
    """Thresholds (tau_x, tau_s) from calibration vectors x_cal bf16 [n][d_model]."""
    n, d = x_cal.shape
    _need(x_cal, torch.bfloat16, (n, layer.d_model), "x_cal")
    nbytes = int(lib().prox_calibrate_workspace_bytes(layer.d_model, layer.d_ff, n))
    if nbytes == 0:
        raise ProxError(PROX_EINVAL, "prox_calibrate_workspace_bytes")
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=x_cal.device)
    tx, ts = C.c_float(), C.c_float()
    cl = layer.cstruct()
    _check(lib().prox_calibrate(C.byref(cl), _ptr(x_cal), n, float(keep_x), float(keep_s),
                                C.byref(tx), C.byref(ts), _ptr(ws), nbytes, _stream(x_cal.device)),
           "prox_calibrate")
    return tx.value, ts.value


HIST_SAMPLES, HIST_BINS = 200_000, 4096   # the pages' per-layer calibration budget


def calibrate_histogram(layer: ProxLayer, x_cal: torch.Tensor, keep_x: float, keep_s: float,
                        max_samples: int = HIST_SAMPLES, bins: int = HIST_BINS):
    """Histogram thresholds (tau_x, tau_s): see prox_calibrate_histogram."""
    n, d = x_cal.shape
    _need(x_cal, torch.bfloat16, (n, layer.d_model), "x_cal")
    nbytes = int(lib().prox_calibrate_workspace_bytes(layer.d_model, layer.d_ff, n))
    if nbytes == 0:
        raise ProxError(PROX_EINVAL, "prox_calibrate_workspace_bytes")
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=x_cal.device)
    tx, ts = C.c_float(), C.c_float()
    cl = layer.cstruct()
    _check(lib().prox_calibrate_histogram(C.byref(cl), _ptr(x_cal), n, float(keep_x),
                                          float(keep_s), int(max_samples), int(bins),
                                          C.byref(tx), C.byref(ts), _ptr(ws), nbytes,
                                          _stream(x_cal.device)),
           "prox_calibrate_histogram")
    return tx.value, ts.value


def allocate(e: float, alpha: float = 1.0 / 3.0, s1_max: float = 0.7, s2_anchor: float = 0.7):
    """(s1, s2) for a target effective sparsity e (host only)."""
    s1, s2 = C.c_double(), C.c_double()
    _check(lib().prox_allocate(float(e), float(alpha), float(s1_max), float(s2_anchor),
                               C.byref(s1), C.byref(s2)), "prox_allocate")
    return s1.value, s2.value


def last_device_status(ws: torch.Tensor) -> tuple[int, int]:
    """(status, raw flags) of the device status word; clears it."""
    flags = C.c_uint32()
    st = lib().prox_last_device_status(_ptr(ws), ws.numel(), _stream(ws.device), C.byref(flags))
    return st, flags.value


def static_last_device_status(device=None) -> tuple[int, int]:
    """(status, raw flags) of the static array's status word (the array of
    ffn_forward_static on the current device); clears it."""
    flags = C.c_uint32()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = lib().prox_static_last_device_status(_stream(dev), C.byref(flags))
    return st, flags.value


SKIP_OFF, SKIP_STAGE1_TC, SKIP_STAGE2_TC = 0, 1, 3


def test_set_skip(where: int, position: int = -1) -> None:
    """Test hook (prox_testing.h): one arrival in CTA 0 of a tensor-core
    kernel never happens, so that its bounded wait runs out."""
    lib().prox_test_set_skip(int(where), int(position))


def test_set_wait(wait_us: int = 0, skip_position: int = -1) -> None:
    """Test hook (prox_testing.h): shorter bounded waits / one unfilled stage."""
    lib().prox_test_set_wait(int(wait_us), int(skip_position))


STAMP_SLOTS = 16
# stamp slots that hold a minimum over CTAs (all others hold a maximum)
STAMP_MIN_SLOTS = (0, 1, 8, 9, 12)


def stamp_buffer(n_passes: int, device) -> torch.Tensor:
    """Zeroed int64 [n_passes][16] buffer for prox_test_set_stamps."""
    return torch.zeros((n_passes, STAMP_SLOTS), dtype=torch.int64, device=device)


def reset_stamps(buf: torch.Tensor) -> None:
    """Minimum slots to all ones (as unsigned), maximum slots to zero."""
    buf.zero_()
    buf[:, list(STAMP_MIN_SLOTS)] = -1


def test_set_stamps(ptr: int) -> None:
    """Measurement hook (prox_testing.h): passes launched while ptr != 0
    record phase stamps at that device address (16 uint64 slots)."""
    lib().prox_test_set_stamps(C.c_void_p(int(ptr)) if ptr else None)


def untile_proxy(q):
    """Block-tiled offset-binary proxy [d_ff/256][d_model][128] -> row-major
    two's complement nibbles [d_model][d_ff/2] (numpy arrays or tensors):
    the bytes reordered, and q + 8 turned back into q & 0xF by flipping bit 3
    of each nibble."""
    C, d, _ = q.shape
    if isinstance(q, torch.Tensor):
        return q.permute(1, 0, 2).reshape(d, C * 128) ^ 0x88
    return q.transpose(1, 0, 2).reshape(d, C * 128) ^ 0x88


def touched_bytes(d_model: int, d_ff: int, k_x: int, k_s: int,
                  proxy_kind: int = PROXY_INT4) -> int:
    """Weight bytes one token's forward reads: the kept rows of both proxies
    (INT4 with their scales, or bf16) and three bf16 rows per kept channel."""
    proxy = 2 * k_x * d_ff * 2 if proxy_kind == PROXY_BF16 else 2 * k_x * (d_ff // 2) + 2 * k_x * 4
    return proxy + 3 * k_s * d_model * 2


__all__ = ["ProxLayer", "ProxError", "quantize_proxy", "workspace", "workspace_bytes",
           "ffn_forward", "ffn_forward_static", "STATIC_WORKSPACE_BYTES", "ffn_forward_raw",
           "ffn_stage1_raw", "ffn_stage2_raw", "rmsnorm_bf16", "ffn_block", "ffn_block_raw",
           "calibrate_histogram", "bf16_proxy", "PROXY_INT4", "PROXY_BF16",
           "max_batch_per_pass", "set_stage2_engine", "stage2_engine", "set_stage1_engine",
           "stage1_engine", "ENGINE_AUTO",
           "ENGINE_SIMT", "ENGINE_TC", "proxy_state", "calibrate", "allocate",
           "last_device_status", "static_last_device_status", "touched_bytes", "untile_proxy",
           "as_bf16"]
