"""The C-ABI library loads, exports every symbol include/*.h declares, and
rejects bad arguments on the host before any CUDA call (runs without a GPU)."""
import ctypes as C
import glob
import os
import re

import pytest

from free_ffn_activation_b200 import prox as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(prox_\w+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


def test_headers_declare_the_boundary():
    names = declared_functions()
    for n in ("prox_quantize_proxy", "prox_calibrate", "prox_ffn_forward", "prox_workspace_bytes",
              "prox_last_device_status", "prox_status_str", "prox_proxy_state", "prox_allocate"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = C.CDLL(P.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_only_abi_symbols_exported():
    out = os.popen(f"nm -D --defined-only {P.LIB_PATH}").read()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(declared_functions()), exported ^ set(declared_functions())


def test_status_strings():
    for s in range(6):
        assert P.status_str(s)
    assert "time" in P.status_str(P.PROX_ETIMEOUT)


def test_workspace_sizes():
    assert P.workspace_bytes(4096, 12288, 1) > 0
    assert P.workspace_bytes(4096, 12288, 8) > P.workspace_bytes(4096, 12288, 1)
    assert P.workspace_bytes(4096, 12288, 100) == P.workspace_bytes(4096, 12288, 8)
    assert P.workspace_bytes(8192, 28672, 16) > 0
    for d, f in ((255, 768), (256, 100), (0, 768), (16384, 768), (256, -256)):
        assert P.workspace_bytes(d, f, 1) == 0
    assert P.workspace_bytes(256, 768, -1) == 0
    assert P.lib().prox_calibrate_workspace_bytes(256, 768, 0) == 0
    assert P.lib().prox_calibrate_workspace_bytes(256, 768, 256) > 256 * 768 * 4


def _fake_layer(d=256, f=768, **override):
    base = 1 << 20
    fields = dict(d_model=d, d_ff=f, w_up_cm=base, w_gate_cm=base * 2, w_down=base * 3,
                  q_up=base * 4, q_gate=base * 5, s_up=base * 6, s_gate=base * 7)
    fields.update(override)
    return P._Layer(**fields)


def _fwd(layer, x=1 << 24, batch=1, tau_x=0.5, tau_s=0.1, y=1 << 25, ws=1 << 26, ws_bytes=1 << 30):
    return P.lib().prox_ffn_forward(C.byref(layer) if layer is not None else None, x, batch,
                                    tau_x, tau_s, y, None, None, None, None, ws, ws_bytes, None)


def test_forward_validation_before_launch():
    L = _fake_layer()
    assert _fwd(None) == P.PROX_EINVAL
    assert _fwd(_fake_layer(d=300)) == P.PROX_EINVAL
    assert _fwd(_fake_layer(f=700)) == P.PROX_EINVAL
    assert _fwd(_fake_layer(w_down=None)) == P.PROX_EINVAL
    assert _fwd(_fake_layer(q_gate=(1 << 20) + 4)) == P.PROX_EINVAL   # misaligned
    assert _fwd(L, tau_x=float("nan")) == P.PROX_EINVAL
    assert _fwd(L, tau_s=-1.0) == P.PROX_EINVAL
    assert _fwd(L, tau_s=float("inf")) == P.PROX_EINVAL
    assert _fwd(L, batch=-1) == P.PROX_EINVAL
    assert _fwd(L, x=None) == P.PROX_EINVAL
    assert _fwd(L, y=None) == P.PROX_EINVAL
    assert _fwd(L, ws=None) == P.PROX_EINVAL
    assert _fwd(L, batch=0) == P.PROX_OK            # nothing to do, nothing launched
    lib = P.lib()
    for k in range(4):   # optional outputs must be aligned when given
        outs = [None] * 4
        outs[k] = (1 << 27) + 8
        assert lib.prox_ffn_forward(C.byref(L), 1 << 24, 1, 0.5, 0.1, 1 << 25, *outs,
                                    1 << 26, 1 << 30, None) == P.PROX_EINVAL


def test_other_entry_points_validate():
    lib = P.lib()
    assert lib.prox_quantize_proxy(256, 768, None, 1 << 20, 1 << 21, None) == P.PROX_EINVAL
    assert lib.prox_quantize_proxy(250, 768, 1 << 20, 1 << 21, 1 << 22, None) == P.PROX_EINVAL
    L = _fake_layer()
    tx, ts = C.c_float(), C.c_float()
    assert lib.prox_calibrate(C.byref(L), 1 << 20, 0, 0.5, 0.3, C.byref(tx), C.byref(ts),
                              1 << 21, 1 << 30, None) == P.PROX_EINVAL
    assert lib.prox_calibrate(C.byref(L), 1 << 20, 4, 1.5, 0.3, C.byref(tx), C.byref(ts),
                              1 << 21, 1 << 30, None) == P.PROX_EINVAL
    assert lib.prox_calibrate(C.byref(L), 1 << 20, 4, 0.5, 0.3, None, C.byref(ts),
                              1 << 21, 1 << 30, None) == P.PROX_EINVAL
    assert lib.prox_calibrate(C.byref(L), 1 << 20, 4, 0.5, 0.3, C.byref(tx), C.byref(ts),
                              1 << 21, 16, None) == P.PROX_ENOMEM
    assert lib.prox_proxy_state(C.byref(L), 1 << 20, 1, -0.5, 1 << 21, None, 1 << 22, 1 << 30,
                                None) == P.PROX_EINVAL
    assert lib.prox_last_device_status(None, 0, None, None) == P.PROX_EINVAL


def test_budget_split_entry_point():
    # blog "Compute budget": e = 0.7, alpha = 1/3, s1 capped at 0.7 -> s2 ~= 0.7667
    s1, s2 = P.allocate(0.7)
    assert s1 == pytest.approx(0.7) and abs(s2 - 0.7667) < 5e-5
    import oracle
    for e in (0.3, 0.45, 0.6, 0.7, 0.85):
        assert P.allocate(e) == pytest.approx(oracle.allocate(e), abs=1e-15)
    with pytest.raises(P.ProxError):
        P.allocate(1.5)
    with pytest.raises(P.ProxError):
        P.allocate(0.5, alpha=0.0)


def test_stack_entry_points_validate_before_launch():
    lib = P.lib()
    base = 1 << 20
    L = P._Layer(d_model=256, d_ff=768, w_up_cm=base, w_gate_cm=base * 2, w_down=base * 3,
                 q_up=base * 4, q_gate=base * 5, s_up=base * 6, s_gate=base * 7)
    # rmsnorm: bad shape, negative or non-finite eps, null or misaligned pointers
    assert lib.prox_rmsnorm_bf16(250, 1, base, 1e-6, base * 2, None) == P.PROX_EINVAL
    assert lib.prox_rmsnorm_bf16(256, 1, base, -1.0, base * 2, None) == P.PROX_EINVAL
    assert lib.prox_rmsnorm_bf16(256, 1, base, float("nan"), base * 2, None) == P.PROX_EINVAL
    assert lib.prox_rmsnorm_bf16(256, 1, None, 1e-6, base * 2, None) == P.PROX_EINVAL
    assert lib.prox_rmsnorm_bf16(256, 1, base + 4, 1e-6, base * 2, None) == P.PROX_EINVAL
    assert lib.prox_rmsnorm_bf16(256, 0, None, 1e-6, None, None) == P.PROX_OK
    # block: x_out is required, eps checked, workspace size checked
    ws = P.lib().prox_workspace_bytes(256, 768, 1)
    args = lambda **k: dict(dict(h_in=base * 8, tau_x=0.5, tau_s=0.1, eps=1e-6, h_out=base * 9,
                                 x_out=base * 10, ws=base * 11, wsb=ws), **k)
    def call(a):
        return lib.prox_ffn_block(C.byref(L), a["h_in"], 1, a["tau_x"], a["tau_s"], a["eps"],
                                  a["h_out"], a["x_out"], None, None, None, None, a["ws"],
                                  a["wsb"], None)
    assert call(args(x_out=None)) == P.PROX_EINVAL
    assert call(args(eps=-1e-6)) == P.PROX_EINVAL
    assert call(args(h_in=None)) == P.PROX_EINVAL
    assert call(args(tau_s=float("inf"))) == P.PROX_EINVAL
    assert call(args(wsb=ws - 1)) == P.PROX_ENOMEM


def test_unknown_activation_rejected():
    base = 1 << 20
    L = P._Layer(d_model=256, d_ff=768, w_up_cm=base, w_gate_cm=base * 2, w_down=base * 3,
                 q_up=base * 4, q_gate=base * 5, s_up=base * 6, s_gate=base * 7, activation=2)
    st = P.lib().prox_ffn_forward(C.byref(L), 1 << 24, 1, 0.5, 0.1, 1 << 25, None, None, None,
                                  None, 1 << 26, 1 << 30, None)
    assert st == P.PROX_EINVAL
    L.activation = P.ACT_GEGLU
    assert P.lib().prox_quantize_proxy(250, 768, base, base, base, None) == P.PROX_EINVAL


def test_calibrate_histogram_validates():
    base = 1 << 20
    L = P._Layer(d_model=256, d_ff=768, w_up_cm=base, w_gate_cm=base * 2, w_down=base * 3,
                 q_up=base * 4, q_gate=base * 5, s_up=base * 6, s_gate=base * 7)
    tx, ts = C.c_float(), C.c_float()
    wsb = P.lib().prox_calibrate_workspace_bytes(256, 768, 4)
    call = lambda ms, bins, wb=wsb: P.lib().prox_calibrate_histogram(
        C.byref(L), base * 8, 4, 0.5, 0.3, ms, bins, C.byref(tx), C.byref(ts), base * 9, wb, None)
    assert call(0, 4096) == P.PROX_EINVAL          # no samples
    assert call(200000, 4000) == P.PROX_EINVAL     # bins not a multiple of 1024
    assert call(200000, 131072) == P.PROX_EINVAL   # too many bins
    assert call(200000, 4096, wsb - 1) == P.PROX_ENOMEM


def test_stage1_engine_switch():
    prev = P.set_stage1_engine(P.ENGINE_SIMT)
    try:
        assert P.set_stage1_engine(P.ENGINE_TC) == P.ENGINE_SIMT
        assert P.lib().prox_set_stage1_engine(-3) == -1          # unknown: nothing changes
        with P.stage1_engine(P.ENGINE_AUTO):
            assert P.set_stage1_engine(P.ENGINE_AUTO) == P.ENGINE_AUTO
        assert P.set_stage1_engine(P.ENGINE_AUTO) == P.ENGINE_TC
    finally:
        P.set_stage1_engine(prev)


def test_stage2_engine_switch():
    prev = P.set_stage2_engine(P.ENGINE_SIMT)
    try:
        assert P.set_stage2_engine(P.ENGINE_TC) == P.ENGINE_SIMT
        assert P.lib().prox_set_stage2_engine(7) == -1          # unknown: nothing changes
        assert P.set_stage2_engine(P.ENGINE_AUTO) == P.ENGINE_TC
        with P.stage2_engine(P.ENGINE_SIMT):
            assert P.set_stage2_engine(P.ENGINE_SIMT) == P.ENGINE_SIMT
        assert P.set_stage2_engine(P.ENGINE_AUTO) == P.ENGINE_AUTO
    finally:
        P.set_stage2_engine(prev)


def test_workspace_holds_tensor_core_buffers():
    # every pass: status word, per-block counts, union list and per-token lists;
    # passes of <= 4 tokens add the tensor-core Stage 1's int64 proxy sums and
    # block counters (2*B*f*8 + C*4 bytes); passes of >= 4 tokens the
    # tensor-core Stage 2's partial sums, split counters, s tiles and union
    # positions (f*2*B*4 + (f/64)*4 + (f/64)*2048 + f*4 bytes)
    d, f = 4096, 12288
    C = f // 256

    def lists(B):
        return 256 + C * 4 + C * B * 4 + C * 256 * 4 + B * f * 4

    def s1_tc(B):
        return 2 * B * f * 8 + C * 4

    def s2_tc(B):
        return f * 2 * B * 4 + (f // 64) * 4 + (f // 64) * 2048 + f * 4

    assert P.workspace_bytes(d, f, 1) >= lists(1) + s1_tc(1)
    assert P.workspace_bytes(d, f, 2) >= lists(2) + s1_tc(2)
    assert P.workspace_bytes(d, f, 4) >= lists(4) + s1_tc(4) + s2_tc(4)
    assert P.workspace_bytes(d, f, 8) >= lists(8) + s2_tc(8)
    assert P.workspace_bytes(d, f, 1000) <= P.STATIC_WORKSPACE_BYTES
    assert P.workspace_bytes(d, f, 4) <= P.STATIC_WORKSPACE_BYTES
