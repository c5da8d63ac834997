"""Parity of a pre-norm layer stack (prox_ffn_block) with the fp64 oracle.

The stack (the stacked-layer benchmark built on the Prox FFN): x = bf16 of
RMSNorm(h) with unit gain and eps 1e-6, h <- h + FFN(x), the residual stream
in fp32. Thresholds are calibrated depth-sequentially by the oracle: layer l's
tau_x and tau_s come from the calibration vectors after layers 0..l-1.

Checked layer by layer on the device's own layer input:
  * x: the oracle's bf16 RMSNorm of the device's h, equal on >= 99% of the
    coordinates and never more than one bf16 step apart (the device sums the
    squares in fp32);
  * the FFN on that x: the same bars as a single forward (masks bit-exact
    outside the 1e-3 * tau_s band, y = h_out - h_in within 2e-3 relative of
    the oracle's Stage 2 fed the device's channel mask).
"""
import numpy as np
import pytest
import torch

import oracle
from free_ffn_activation_b200 import prox as P
from free_ffn_activation_b200 import synth as S

pytestmark = pytest.mark.gpu

EPS = 1e-6
BAND = 1e-3
Y_TOL = 2e-3


class Stack:
    def __init__(self, d, f, n_layers, n_tok, n_cal, sigma=0.02, dev="cuda"):
        self.d, self.f = d, f
        self.L, self.Por, self.layers, self.tau = [], [], [], []
        h_cal = S.bf16_to_f32(S.make_tokens(n_cal, d, seed=0, stream="x_cal"))
        for ell in range(n_layers):
            L = S.make_layer(S.LayerSpec(d, f, sigma=sigma, seed=0, layer=ell))
            Por = oracle.make_proxy(L)
            x_cal = oracle.rmsnorm_bf16(h_cal, EPS)
            tx, ts = oracle.calibrate(x_cal, Por, 0.5, 0.3)
            y = oracle.forward(x_cal, tx, ts, L, Por, want=())["y"]
            h_cal = (h_cal.astype(np.float64) + y).astype(np.float32)
            self.L.append(L)
            self.Por.append(Por)
            self.tau.append((tx, ts))
            self.layers.append(P.ProxLayer.from_weights(L["w_up_cm"], L["w_gate_cm"],
                                                        L["w_down"], device=dev))
        self.h0 = S.bf16_to_f32(S.make_tokens(n_tok, d, seed=0, stream="x_eval"))


def _bits(x_bf16: torch.Tensor) -> np.ndarray:
    return x_bf16.view(torch.int16).cpu().numpy().view(np.uint16)


def check_layer(st, ell, h_in, h_out, x, out):
    tx, ts = st.tau[ell]
    L, Por = st.L[ell], st.Por[ell]
    # the pre-norm
    xb = _bits(x)
    xr = oracle.rmsnorm_bf16(h_in, EPS)
    step = np.abs(xb.astype(np.int32) - xr.astype(np.int32))
    same_sign = (xb >> 15) == (xr >> 15)
    assert np.all((step <= 1) & (same_sign | (step == 0))), f"layer {ell}: x off by > 1 step"
    assert (step == 0).mean() >= 0.99, f"layer {ell}: x differs on {(step != 0).mean():.4f}"
    # the FFN on the device's x
    ref = oracle.forward(xb, tx, ts, L, Por)
    assert np.array_equal(out.mask_x.cpu().numpy(), ref["mask_x"]), f"layer {ell}: mask_x"
    ms = out.mask_s.cpu().numpy()
    band = np.abs(np.abs(ref["s_proxy"]) - ts) <= BAND * ts
    assert not np.any((ms != ref["mask_s"]) & ~band), f"layer {ell}: mask_s outside band"
    cnt, idx = out.count_s.cpu().numpy(), out.idx_s.cpu().numpy()
    for t in range(ms.shape[0]):
        kept = np.flatnonzero(ms[t])
        assert cnt[t] == kept.size and np.array_equal(idx[t, :cnt[t]], kept)
    y_ref = oracle.forward(xb, tx, ts, L, Por, mask_s_in=ms, want=())["y"]
    y = h_out.astype(np.float64) - h_in.astype(np.float64)
    rel = np.linalg.norm(y - y_ref, axis=1) / np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    assert rel.max() <= Y_TOL, f"layer {ell}: y rel err {rel.max()}"
    return float(rel.max()), int(band.sum()), int((ms != ref["mask_s"]).sum())


def run_stack(st, dev, in_place=False, batch_rows=None):
    h = torch.from_numpy(st.h0 if batch_rows is None else st.h0[batch_rows]).to(dev)
    for ell, layer in enumerate(st.layers):
        tx, ts = st.tau[ell]
        h_in = h.cpu().numpy()
        h_out, x, out = P.ffn_block(layer, h, tx, ts, EPS, h_out=h if in_place else None)
        torch.cuda.synchronize()
        rel, nb, nd = check_layer(st, ell, h_in, h_out.cpu().numpy(), x, out)
        print(f"[stack layer {ell}] tokens={h.shape[0]} y_rel_max={rel:.2e} band={nb} "
              f"mask_s diffs={nd}")
        h = h_out


@pytest.fixture(scope="module")
def small(gpu):
    # three 256 x 768 layers with their own seeds, 16 tokens, 64 calibration vectors
    return Stack(256, 768, 3, 16, 64)


@pytest.fixture(scope="module")
def qwen(gpu):
    # the first two layers of the 36-layer 4096 x 12288 stack, 2 tokens
    return Stack(4096, 12288, 2, 2, 64)


def test_stack_small_batched(small, gpu):
    run_stack(small, gpu)


def test_stack_small_token_by_token_in_place(small, gpu):
    for t in range(4):
        run_stack(small, gpu, in_place=True, batch_rows=[t])


def test_stack_qwen_shape_two_layers(qwen, gpu):
    run_stack(qwen, gpu)


def test_rmsnorm_entry_matches_block_input(small, gpu):
    h = torch.from_numpy(small.h0).to(gpu)
    x = P.rmsnorm_bf16(h, EPS)
    _, xb, _ = P.ffn_block(small.layers[0], h, *small.tau[0], EPS)
    torch.cuda.synchronize()
    assert torch.equal(x, xb)
