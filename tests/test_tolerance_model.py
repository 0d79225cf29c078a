"""The bf16 tolerances against the arithmetic they must absorb (CPU only).

The CUDA path stores its intermediates in bf16 (the block: v = x W_1ᵀ, g = x W_2ᵀ, the
Conv1D output u, h ⊙ GeLU(g), the block output; the layer in addition: both RMSNorm outputs,
the residual stream, the MLP's gate, up, GeLU product and down projection, the output) and
the recurrence coefficients d = 1 − a_t, b_t = √(1 − a_t²)·i_t·u_t in fp16, with float32
arithmetic in between. The model below is the float64 oracle's arithmetic with exactly
those roundings (round to nearest even, torch's casts) and nothing else; the CUDA path is
not involved. Its distance from the unrounded oracle is the error that storage rounding
alone forces on any implementation with these formats, on the seeded parity cases of the
GPU tests. The tolerances must cover it, and the layer's case shows why the layer cannot
be held to the RG-LRU's 2e-2.
"""
import numpy as np
import torch

import oracle
from gated_linear_rnn_conv1d_b200 import inputs

from _util import TOL, TOL_LAYER


def _f(t):
    return t.double().numpy() if torch.is_tensor(t) else np.asarray(t, dtype=np.float64)


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def _fp16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.float16).double().numpy()


def _rms_norm(v, gain, eps=oracle.RMS_EPS):
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps) * _f(gain)


def _block_rounded(x, W_1, W_2, W_o, P):
    """Recurrent block with the storage roundings of the bf16 path."""
    v, g = _bf16(x @ _f(W_1).T), _bf16(x @ _f(W_2).T)
    u, _ = oracle.conv1d_causal(v, _f(P.conv_w), _f(P.conv_b))
    u = _bf16(u)
    r = oracle.sigmoid(u @ _f(P.W_a).T + _f(P.b_a))
    i = oracle.sigmoid(u @ _f(P.W_x).T + _f(P.b_x))
    a_t = oracle.decay_direct(r, _f(P.Lambda))
    d, b = _fp16(1.0 - a_t), _fp16(np.sqrt(1.0 - a_t * a_t) * i * u)
    h, hs = np.zeros((u.shape[0], u.shape[2])), np.empty_like(u)
    for t in range(u.shape[1]):
        h = (1.0 - d[:, t]) * h + b[:, t]
        hs[:, t] = h
    return _bf16(_bf16(hs * oracle.gelu(g)) @ _f(W_o).T)


def test_block_storage_rounding_fits_the_bf16_tolerance():
    w = inputs.make_block(2, 150, 136, 264, torch.bfloat16, seed=6)  # the block's GPU parity case
    P = w.params
    got = _block_rounded(_f(w.x), w.W_1, w.W_2, w.W_o, P)
    ref, _ = oracle.recurrent_block(w.x, w.W_1, w.W_2, w.W_o, P.conv_w, P.conv_b, P.W_a, P.b_a, P.W_x, P.b_x,
                                    P.Lambda)
    err = oracle.max_rel_error(got, ref)
    assert 5e-3 < err <= TOL[torch.bfloat16], err


def test_layer_storage_rounding_fits_the_layer_tolerance_and_not_the_rglru_one():
    w = inputs.make_layer(2, 150, 136, 264, 3, torch.bfloat16, seed=7)  # the layer's GPU parity case
    P, e = w.params, w.extra
    x = _f(w.x)
    o1 = _block_rounded(_bf16(_rms_norm(x, e["norm1_scale"])), w.W_1, w.W_2, w.W_o, P)
    y = _bf16(x + o1)
    n2 = _bf16(_rms_norm(y, e["norm2_scale"]))
    gate, up = _bf16(n2 @ _f(e["W_gate"]).T), _bf16(n2 @ _f(e["W_up"]).T)
    o2 = _bf16(_bf16(oracle.gelu(gate) * up) @ _f(e["W_down"]).T)
    got = _bf16(y + o2)
    ref, _ = oracle.hawk_residual_layer(w.x, e["norm1_scale"], w.W_1, w.W_2, w.W_o, e["norm2_scale"], e["W_gate"],
                                        e["W_up"], e["W_down"], P.conv_w, P.conv_b, P.W_a, P.b_a, P.W_x, P.b_x,
                                        P.Lambda)
    err = oracle.max_rel_error(got, ref)
    assert TOL[torch.bfloat16] < err <= TOL_LAYER, err
    print(f"layer parity case: storage rounding alone gives {err:.17g}")


def test_forward_storage_rounding_fits_the_bf16_tolerance():
    # the RG-LRU forward's bf16 parity case (B=2, T=200, D_RNN=264, non-zero biases, h0 and
    # conv history, as the GPU test draws them): u in bf16 (the gate GEMM's operand, also
    # the u in b_t), d and b in fp16, y in bf16
    B, T, R = 2, 200, 264
    w = inputs.make_forward(B, T, R, torch.bfloat16, seed=0)
    g = torch.Generator("cpu").manual_seed(77)
    P = w.params
    P.b_a = torch.randn(R, generator=g) * 0.5
    P.b_x = torch.randn(R, generator=g) * 0.5
    h0 = torch.randn(B, R, generator=g)
    state0 = torch.randn(B, 3, R, generator=g).to(torch.bfloat16)
    for hist, h_init in ((None, None), (state0, h0)):
        u, _ = oracle.conv1d_causal(w.x, _f(P.conv_w), _f(P.conv_b), None if hist is None else _f(hist))
        u = _bf16(u)
        r = oracle.sigmoid(u @ _f(P.W_a).T + _f(P.b_a))
        i = oracle.sigmoid(u @ _f(P.W_x).T + _f(P.b_x))
        a_t = oracle.decay_direct(r, _f(P.Lambda))
        d, b = _fp16(1.0 - a_t), _fp16(np.sqrt(1.0 - a_t * a_t) * i * u)
        h = np.zeros((B, R)) if h_init is None else _f(h_init)
        ys = np.empty_like(u)
        for t in range(T):
            h = (1.0 - d[:, t]) * h + b[:, t]
            ys[:, t] = h
        y_ref, _, _ = oracle.rglru_forward(w.x, P.conv_w, P.conv_b, P.W_a, P.b_a, P.W_x, P.b_x, P.Lambda,
                                           h0=h_init, conv_state0=hist)
        err = oracle.max_rel_error(_bf16(ys), y_ref)
        print(f"forward parity case, history={hist is not None}: storage rounding alone gives {err:.3e}")
        assert err <= TOL[torch.bfloat16], err
