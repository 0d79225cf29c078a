"""The backward of Conv1D + RG-LRU (rglru_backward, bf16 IO) against the float64 oracle's
reverse-mode derivative, which the oracle tests pin to central differences of the forward."""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_rnn_conv1d_b200 import inputs, rglru

from _util import f64, rel

pytestmark = pytest.mark.gpu
DEV = "cuda"

# bf16 IO: dy, y (h_{t−1}), ∂z and the gate-GEMM ∂u are rounded to bf16 (8 significant
# bits) on their way between kernels, as the forward's y is. The bound is the forward's
# 2e-2, except for the weight gradients ∂W = Σ_t ∂z_tᵀ u_t: each product there has two bf16
# operands (relative rounding up to 2^-9 each, on top of ∂z's own error of a few 2^-9)
# summed over the tokens in float32, so the error relative to the entries' rms does not
# shrink with more tokens and its maximum over R² entries reaches about 3%: 4e-2 for them.
TOL = 2e-2
TOL_W = 4e-2
KEYS = ("dx", "dconv_state0", "dconv_w", "dconv_b", "dW_a", "db_a", "dW_x", "db_x", "dLambda", "dh0")


def _tol(k):
    return TOL_W if k in ("dW_a", "dW_x") else TOL


def _problem(B, T, R, with_state, seed):
    w = inputs.make_forward(B, T, R, torch.bfloat16, seed=seed)
    g = torch.Generator("cpu").manual_seed(seed + 101)
    w.params.b_a = torch.randn(R, generator=g) * 0.5
    w.params.b_x = torch.randn(R, generator=g) * 0.5
    h0 = torch.randn(B, R, generator=g) if with_state else None
    st0 = torch.randn(B, 3, R, generator=g).to(torch.bfloat16) if with_state else None
    dy = torch.randn(B, T, R, generator=g).to(torch.bfloat16)
    dh_T = torch.randn(B, R, generator=g)
    return w, h0, st0, dy, dh_T


def _dev(t):
    return None if t is None else t.to(DEV)


@pytest.mark.parametrize("B,T,R,with_state", [(2, 200, 264, True), (1, 65, 8, False), (3, 130, 136, True),
                                               (2, 64, 128, False), (1, 1, 16, True), (2, 1024, 1024, True)])
def test_backward_matches_oracle(B, T, R, with_state):
    w, h0, st0, dy, dh_T = _problem(B, T, R, with_state, seed=B * 1000 + T + R)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    y, _, _ = rglru.forward(p, x, _dev(h0), _dev(st0))
    G = rglru.backward(p, x, y, dy.to(DEV), _dev(h0), dh_T.to(DEV), _dev(st0))
    ws_status = rglru.workspace_status(None)
    ref = oracle.rglru_backward(w.x, w.params.conv_w, w.params.conv_b, w.params.W_a, w.params.b_a, w.params.W_x,
                                w.params.b_x, w.params.Lambda, dy, h0=h0, conv_state0=st0, dh_T=dh_T)
    assert ws_status == 0
    errs = {k: rel(G[k], ref[k]) for k in KEYS}
    print("backward errors", B, T, R, with_state, {k: round(v, 4) for k, v in errs.items()})
    assert all(errs[k] <= _tol(k) for k in KEYS), errs


def test_backward_without_optional_outputs_and_inputs():
    """dh0 and dconv_state0 may be left out (NULL), and h0, dh_T, conv_state0 default to
    zeros: the other gradients are those of the oracle with zeros for them."""
    B, T, R = 2, 96, 136
    w, _, _, dy, _ = _problem(B, T, R, False, seed=7)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    y, _, _ = rglru.forward(p, x)
    G = rglru.backward(p, x, y, dy.to(DEV), want_dh0=False, want_dconv_state0=False)
    assert G["dh0"] is None and G["dconv_state0"] is None
    ref = oracle.rglru_backward(w.x, w.params.conv_w, w.params.conv_b, w.params.W_a, w.params.b_a, w.params.W_x,
                                w.params.b_x, w.params.Lambda, dy)
    for k in ("dx", "dconv_w", "dconv_b", "dW_a", "db_a", "dW_x", "db_x", "dLambda"):
        assert rel(G[k], ref[k]) <= _tol(k), k


def test_backward_of_a_frozen_state():
    """r ≡ 0 (W_a = 0, b_a = −1000): a_t = 1 and √(1 − a_t²) = 0, so h_t = h0, ∂h0 = Σ dy + dh_T
    and no gradient reaches x, the taps, the input gate or Λ."""
    B, T, R = 2, 100, 16
    w, h0, st0, dy, dh_T = _problem(B, T, R, True, seed=3)
    w.params.W_a = torch.zeros(R, R, dtype=torch.bfloat16)
    w.params.b_a = torch.full((R,), -1000.0)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    y, _, _ = rglru.forward(p, x, _dev(h0), _dev(st0))
    G = rglru.backward(p, x, y, dy.to(DEV), _dev(h0), dh_T.to(DEV), _dev(st0))
    expect = f64(dy).sum(axis=1) + f64(dh_T)
    assert np.max(np.abs(f64(G["dh0"]) - expect)) <= 1e-4 * max(1.0, np.max(np.abs(expect)))
    for k in ("dx", "dconv_w", "dconv_b", "dW_x", "db_x", "dLambda", "dconv_state0"):
        assert float(torch.max(torch.abs(G[k].float()))) == 0.0, k


@pytest.mark.parametrize("B,T,R,with_state", [(2, 200, 264, True), (2, 1024, 1024, True), (1, 65, 8, False)])
def test_training_pair_equals_forward_and_backward(B, T, R, with_state):
    """rglru_forward_train gives rglru_forward's outputs bit for bit and saves the gate
    pre-activations the backward would recompute; rglru_backward_saved from them gives
    rglru_backward's gradients — bit for bit for every gradient formed without atomics, to
    float32 summation order for the ones accumulated with atomics (taps, biases, Λ)."""
    w, h0, st0, dy, dh_T = _problem(B, T, R, with_state, seed=B * 100 + T + R + 5)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    y, hT, csT = rglru.forward(p, x, _dev(h0), _dev(st0))
    y2, hT2, csT2, saved = rglru.forward_train(p, x, _dev(h0), _dev(st0))
    assert torch.equal(y, y2) and torch.equal(hT, hT2) and torch.equal(csT, csT2)
    assert saved.numel() == rglru.saved_bytes(B, T, R)
    G = rglru.backward(p, x, y, dy.to(DEV), _dev(h0), dh_T.to(DEV), _dev(st0))
    G2 = rglru.backward(p, x, y2, dy.to(DEV), _dev(h0), dh_T.to(DEV), _dev(st0), saved=saved)
    assert rglru.workspace_status(None) == 0
    for k in ("dx", "dconv_state0", "dW_a", "dW_x", "dh0"):
        assert G[k] is None or torch.equal(G[k], G2[k]), k
    for k in ("dconv_w", "dconv_b", "db_a", "db_x", "dLambda"):
        assert rel(G2[k], G[k]) <= 1e-5, k
    ref = oracle.rglru_backward(w.x, w.params.conv_w, w.params.conv_b, w.params.W_a, w.params.b_a, w.params.W_x,
                                w.params.b_x, w.params.Lambda, dy, h0=h0, conv_state0=st0, dh_T=dh_T)
    assert all(rel(G2[k], ref[k]) <= _tol(k) for k in KEYS if G2[k] is not None)
