"""prox_ffn_forward_static: the forward on the library's own file-scope
workspace (no allocation by the caller or the library). Kept in its own file,
collected after the others, so it also runs after every other GPU test has
used the device."""
import ctypes as C

import numpy as np
import pytest
import torch

from free_ffn_activation_b200 import prox as P
from free_ffn_activation_b200 import synth as S


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
        torch.cuda.synchronize()
        assert torch.equal(a.mask_x, b.mask_x) and torch.equal(a.mask_s, b.mask_s)
        assert torch.equal(a.count_s, b.count_s)
        for t in range(3):
            n = int(a.count_s[t])
            assert n > 0 and torch.equal(a.idx_s[t, :n], b.idx_s[t, :n])
        # y is summed across CTAs with fp32 atomics: equal up to summation order
        rel = (torch.linalg.norm(a.y - b.y) / torch.linalg.norm(a.y)).item()
        assert np.isfinite(rel) and rel < 1e-5
