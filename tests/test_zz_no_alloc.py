"""prox_ffn_forward_static: the forward on the library's own file-scope
workspace (no allocation by the caller or the library), for callers that
cannot allocate device memory of their own. Kept in its own file, collected
after the others, so it also runs after every other GPU test has used the
device; it passes alone in a fresh process too."""
import ctypes as C

import numpy as np
import pytest
import torch

from free_ffn_activation_b200 import prox as P
from free_ffn_activation_b200 import synth as S
from parity_helpers import Case, check_forward


def test_static_workspace_limit_rejected_before_any_launch():
    # d_model 256 x d_ff 262144 needs more than the 2 MiB array: PROX_ENOMEM,
    # decided on the host from the shape alone (no device work, no GPU needed)
    assert P.lib().prox_workspace_bytes(256, 262144, 1) > P.STATIC_WORKSPACE_BYTES
    base = 1 << 20
    L = P._Layer(d_model=256, d_ff=262144, w_up_cm=base, w_gate_cm=base * 2, w_down=base * 3,
                 q_up=base * 4, q_gate=base * 5, s_up=base * 6, s_gate=base * 7)
    st = P.lib().prox_ffn_forward_static(C.byref(L), 1 << 24, 1, 0.5, 0.1, 1 << 25,
                                         None, None, None, None, None)
    assert st == P.PROX_ENOMEM
    # the 4096 x 12288 layer fits at any batch (passes of at most 8 tokens)
    assert P.lib().prox_workspace_bytes(4096, 12288, 1000) <= P.STATIC_WORKSPACE_BYTES


def _same_results(a, b, n_tok):
    torch.cuda.synchronize()
    assert torch.equal(a.mask_x, b.mask_x) and torch.equal(a.mask_s, b.mask_s)
    assert torch.equal(a.count_s, b.count_s)
    for t in range(n_tok):
        n = int(a.count_s[t])
        assert n > 0 and torch.equal(a.idx_s[t, :n], b.idx_s[t, :n])
    # y is summed across CTAs with fp32 atomics: equal up to summation order
    rel = (torch.linalg.norm(a.y - b.y) / torch.linalg.norm(a.y)).item()
    assert np.isfinite(rel) and rel < 1e-5


@pytest.mark.gpu
def test_static_forward_matches_workspace_forward(gpu):
    d, f = 1024, 4096
    L = S.make_layer(S.LayerSpec(d, f, sigma=0.02, seed=11))
    layer = P.ProxLayer.from_weights(L["w_up_cm"], L["w_gate_cm"], L["w_down"], device=gpu)
    x_cal = P.as_bf16(S.make_tokens(128, d, seed=11, stream="x_cal"), gpu)
    tau_x, tau_s = P.calibrate(layer, x_cal, 0.5, 0.3)
    x = P.as_bf16(S.make_tokens(3, d, seed=11), gpu)
    for _ in range(2):  # two calls in a row on the same static array
        a = P.ffn_forward(layer, x, tau_x, tau_s)
        b = P.ffn_forward_static(layer, x, tau_x, tau_s)
        _same_results(a, b, 3)
    assert P.static_last_device_status() == (P.PROX_OK, 0)


@pytest.fixture(scope="module")
def c2s(gpu):
    # the 4096 x 12288 layer with 0.1% x20 outlier coordinates, thresholds from
    # 128 calibration vectors (oracle)
    return Case(4096, 12288, 16, 128, outlier=0.001)


@pytest.mark.gpu
def test_static_forward_matches_oracle_tensor_core_stage2(c2s):
    # passes of 8 tokens run the tensor-core union Stage 2, whose partial sums,
    # split counters and s tiles live in the static array: two calls in a row
    # (the second reuses the array the first left behind), each against the
    # oracle and against the forward on a caller-owned workspace
    rows = list(range(8))
    x = c2s.xdev(rows)
    for k in range(2):
        b = P.ffn_forward_static(c2s.layer, x, c2s.tau_x, c2s.tau_s)
        a = P.ffn_forward(c2s.layer, x, c2s.tau_x, c2s.tau_s)
        _same_results(a, b, 8)
        check_forward(c2s, rows, b, f" static b=8 call {k}")
    # one token per call (the CUDA-core Stage 2), also against the oracle
    outs = [P.ffn_forward_static(c2s.layer, c2s.xdev([t]), c2s.tau_x, c2s.tau_s) for t in rows]
    merged = P.ForwardOut(*(torch.cat([getattr(o, k) for o in outs]) for k in
                            ("y", "mask_x", "mask_s", "idx_s", "count_s")))
    check_forward(c2s, rows, merged, " static b=1")
    assert P.static_last_device_status() == (P.PROX_OK, 0)


@pytest.mark.gpu
def test_static_timeout_is_observable(c2s):
    # a bounded wait that gives up (test hook: CTA 0's Stage-2 producer never
    # fills one ring stage, waits bounded to 2 ms) is reported by the static
    # array's status reader, which clears it; the next call is whole again
    x = c2s.xdev([3])
    try:
        P.test_set_wait(2000, 2)
        P.ffn_forward_static(c2s.layer, x, c2s.tau_x, c2s.tau_s)
        st, flags = P.static_last_device_status()
    finally:
        P.test_set_wait(0, -1)
    assert st == P.PROX_ETIMEOUT and flags != 0
    assert P.static_last_device_status() == (P.PROX_OK, 0)
    out = P.ffn_forward_static(c2s.layer, x, c2s.tau_x, c2s.tau_s)
    check_forward(c2s, [3], out, " static after timeout")
