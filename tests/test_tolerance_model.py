"""The bf16 tolerances against the arithmetic they must absorb (CPU only).

The CUDA path stores its intermediates in bf16 (the forward: the Conv1D output u and y;
the block in addition: v = x W_1ᵀ, g = x W_2ᵀ, h ⊙ GeLU(g), the block output; the layer in
addition: both RMSNorm outputs, the residual stream, the MLP's gate, up, GeLU product and
down projection, the output; the backward: the recomputed pre-activations and ∂z, the
operands of the weight-gradient GEMMs) and the recurrence coefficients d = 1 − a_t (fp16)
and b_t = √(1 − a_t²)·i_t·u_t (bf16), with float32 arithmetic in between. The model
(rounding_model.py) is the float64 oracle's arithmetic with exactly those roundings (round
to nearest even, torch's casts) and nothing else; the CUDA path is not involved. Its distance from the unrounded oracle is the error that storage rounding
alone forces on any implementation with these formats, on the seeded parity cases of the
GPU tests. The tolerances must cover it; the layer's case and the backward's weight
gradients show why those two cannot be held to the RG-LRU's 2e-2.
"""
import numpy as np
import torch

import oracle
import rounding_model as rm
from gated_linear_rnn_conv1d_b200 import inputs

from _util import TOL, TOL_ATTN, TOL_LAYER


def test_block_storage_rounding_fits_the_bf16_tolerance():
    w = inputs.make_block(2, 150, 136, 264, torch.bfloat16, seed=6)  # the block's GPU parity case
    P = w.params
    got, _ = rm.block(w.x, w.W_1, w.W_2, w.W_o, P)
    ref, _ = oracle.recurrent_block(w.x, w.W_1, w.W_2, w.W_o, P.conv_w, P.conv_b, P.W_a, P.b_a, P.W_x, P.b_x,
                                    P.Lambda)
    err = oracle.max_rel_error(got, ref)
    print(f"block parity case: storage rounding alone gives {err:.3e}")
    assert 5e-3 < err <= TOL[torch.bfloat16], err


def test_layer_storage_rounding_fits_the_layer_tolerance_and_not_the_rglru_one():
    w = inputs.make_layer(2, 150, 136, 264, 3, torch.bfloat16, seed=7)  # the layer's GPU parity case
    P, e = w.params, w.extra
    got, _ = rm.layer_from_workload(w)
    ref, _ = oracle.hawk_residual_layer(w.x, e["norm1_scale"], w.W_1, w.W_2, w.W_o, e["norm2_scale"], e["W_gate"],
                                        e["W_up"], e["W_down"], P.conv_w, P.conv_b, P.W_a, P.b_a, P.W_x, P.b_x,
                                        P.Lambda)
    err = oracle.max_rel_error(got, ref)
    print(f"layer parity case: storage rounding alone gives {err:.17g}")
    assert TOL[torch.bfloat16] < err <= TOL_LAYER, err


def test_forward_storage_rounding_fits_the_bf16_tolerance():
    # the RG-LRU forward's bf16 parity case (B=2, T=200, D_RNN=264, non-zero biases, h0 and
    # conv history, as the GPU test draws them): u in bf16 (the gate GEMM's operand, also
    # the u in b_t), d in fp16, b in bf16, y in bf16
    B, T, R = 2, 200, 264
    w = inputs.make_forward(B, T, R, torch.bfloat16, seed=0)
    g = torch.Generator("cpu").manual_seed(77)
    P = w.params
    P.b_a = torch.randn(R, generator=g) * 0.5
    P.b_x = torch.randn(R, generator=g) * 0.5
    h0 = torch.randn(B, R, generator=g)
    state0 = torch.randn(B, 3, R, generator=g).to(torch.bfloat16)
    for hist, h_init in ((None, None), (state0, h0)):
        ys, _ = rm.forward(w.x, P, h_init, hist)
        y_ref, _, _ = oracle.rglru_forward(w.x, P.conv_w, P.conv_b, P.W_a, P.b_a, P.W_x, P.b_x, P.Lambda,
                                           h0=h_init, conv_state0=hist)
        err = oracle.max_rel_error(ys, y_ref)
        print(f"forward parity case, history={hist is not None}: storage rounding alone gives {err:.3e}")
        assert err <= TOL[torch.bfloat16], err


def _backward_problem(B, T, R, with_state, seed):
    # the GPU backward test's draws (same generator, same order)
    w = inputs.make_forward(B, T, R, torch.bfloat16, seed=seed)
    g = torch.Generator("cpu").manual_seed(seed + 101)
    w.params.b_a = torch.randn(R, generator=g) * 0.5
    w.params.b_x = torch.randn(R, generator=g) * 0.5
    h0 = torch.randn(B, R, generator=g) if with_state else None
    st0 = torch.randn(B, 3, R, generator=g).to(torch.bfloat16) if with_state else None
    dy = torch.randn(B, T, R, generator=g).to(torch.bfloat16)
    dh_T = torch.randn(B, R, generator=g)
    return w, h0, st0, dy, dh_T


def test_backward_weight_gradients_storage_rounding_needs_the_wider_bound():
    # The backward's storage formats (rounding_model.backward_weight_gradients). On two of
    # the GPU backward test's cases they alone put ∂W_a above the RG-LRU's 2e-2, inside 4e-2.
    for B, T, R, with_state in ((2, 64, 128, False), (2, 200, 264, True)):
        w, h0, st0, dy, dh_T = _backward_problem(B, T, R, with_state, seed=B * 1000 + T + R)
        P = w.params
        dW_a, dW_x = rm.backward_weight_gradients(w.x, P, dy, h0, st0, dh_T)
        ref = oracle.rglru_backward(w.x, P.conv_w, P.conv_b, P.W_a, P.b_a, P.W_x, P.b_x, P.Lambda, dy, h0=h0,
                                    conv_state0=st0, dh_T=dh_T)
        ea, ex = oracle.max_rel_error(dW_a, ref["dW_a"]), oracle.max_rel_error(dW_x, ref["dW_x"])
        print(f"backward case {(B, T, R)}: storage rounding alone gives dW_a {ea:.4f}, dW_x {ex:.4f}")
        assert TOL[torch.bfloat16] < ea <= 4e-2 and ex <= 4e-2, (ea, ex)


def test_attention_storage_rounding_needs_the_attention_bound():
    # the GPU attention test's first case: B=3, D=256 (two heads), window 128, 300 steps
    B, D, W, steps = 3, 256, 128, 300
    w = inputs.make_attention(D, seed=D + W)
    hw = {k: rm.f(v) for k, v in w.items()}
    W_qkv = np.concatenate([hw["W_q"], hw["W_k"], hw["W_v"]], 0)
    K_o, V_o = np.zeros((B, W, 128)), np.zeros((B, W, 128))
    K_m, V_m = np.zeros((B, W, 128)), np.zeros((B, W, 128))
    errs = []
    for t in range(steps):
        xt = inputs.decode_token(t, B, D)
        out_o, K_o, V_o = oracle.local_attention_step(xt, K_o, V_o, t, hw["W_q"], hw["W_k"], hw["W_v"], hw["W_o"], W)
        errs.append(oracle.max_rel_error(rm.attention_step(xt, K_m, V_m, t, W_qkv, hw["W_o"], W), out_o))
    worst = max(errs)
    print(f"attention case: storage rounding alone gives {worst:.4e} (median {np.median(errs):.3e})")
    assert TOL[torch.bfloat16] < worst <= TOL_ATTN, worst
