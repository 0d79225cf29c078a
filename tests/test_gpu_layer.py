"""Decode form of the Hawk residual layer (rglru_layer_step) on the GPU: against the oracle's
hawk_residual_layer_step at every step, and against the layer's own prefill.

Bounds: the layer's 3e-2 on its output (the recurrent block's bf16 allowance plus the
MLP's five bf16 roundings) and on the float32 state h (its input v_t = bf16(RMSNorm₁(x_t))
W_1ᵀ, rounded to bf16 again, carries two roundings the RG-LRU's own 2e-2 does not cover)."""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_rnn_conv1d_b200 import inputs, rglru

from _util import TOL, TOL_LAYER, f64, host_params64, rel

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer_host(w):
    e = w.extra
    return dict(norm1_scale=f64(e["norm1_scale"]), W_1=f64(w.W_1), W_2=f64(w.W_2), W_o=f64(w.W_o),
                norm2_scale=f64(e["norm2_scale"]), W_gate=f64(e["W_gate"]), W_up=f64(e["W_up"]),
                W_down=f64(e["W_down"]))


# (3, 136, 264): ragged batch, a partial 128-channel block, the 1-SM RG-LRU step kernel
# (R % 128 != 0); (256, 512, 512): a full 256-row decode batch on the split-K step kernel
@pytest.mark.parametrize("B,D,R,M,steps", [(3, 136, 264, 3, 10), (256, 512, 512, 3, 6)])
def test_layer_step_matches_oracle_every_step(B, D, R, M, steps):
    w = inputs.make_layer(B, 1, D, R, M, torch.bfloat16, seed=13)
    p = rglru.Params.from_host(w.params)
    lw = rglru.LayerWeights.from_host(w)
    hp, lh = host_params64(w.params), _layer_host(w)
    ring = torch.zeros(B, 3, R, dtype=torch.bfloat16, device=DEV)
    h = torch.zeros(B, R, device=DEV)
    ws = torch.full((rglru.layer_step_workspace_bytes(B, D, R, M * D),), 0xFF, dtype=torch.uint8, device=DEV)
    ring_o, h_o = np.zeros((B, 3, R)), np.zeros((B, R))
    for k in range(steps):
        xt = inputs.decode_token(k, B, D)
        out = rglru.layer_step(p, lw, xt.to(DEV), ring, h, k, eps=oracle.RMS_EPS, workspace=ws)
        out_o, h_o, ring_o = oracle.hawk_residual_layer_step(xt, ring_o, k, h_o, **lh, **hp)
        assert rglru.workspace_status(ws) == 0
        e_out, e_h = rel(out, out_o), rel(h, h_o)
        print(f"step {k}: out {e_out:.3e} h {e_h:.3e}")
        assert e_out <= TOL_LAYER, (k, e_out)
        # the state's input v_t is two bf16 roundings (RMSNorm₁ output, v_t) away from the
        # oracle's, on top of the RG-LRU's own bf16 allowance: the layer's bound
        assert e_h <= TOL_LAYER, (k, e_h)
        # the ring holds the bf16 v_t = bf16(RMSNorm₁(x_t)) W_1ᵀ the GPU computed (two bf16
        # roundings); the oracle's are unrounded
        assert rel(ring, ring_o) <= TOL[torch.bfloat16], k


def test_layer_steps_equal_layer_forward():
    """T decode steps of the layer from a zero state give the layer's prefill over the same
    T tokens. The two round at different points (the prefill stores the recurrence
    coefficients d in fp16 and b_t in bf16 from the bf16 u; the decode step updates the
    float32 state from the float32 u_t), so they agree to the bf16 bound, not bit for bit."""
    B, T, D, R, M = 2, 24, 136, 264, 3
    w = inputs.make_layer(B, T, D, R, M, torch.bfloat16, seed=14)
    p = rglru.Params.from_host(w.params)
    lw = rglru.LayerWeights.from_host(w)
    x = w.x.to(DEV)
    out_f, h_f = rglru.layer_forward(p, lw, x, eps=oracle.RMS_EPS)
    ring = torch.zeros(B, 3, R, dtype=torch.bfloat16, device=DEV)
    h = torch.zeros(B, R, device=DEV)
    outs = [rglru.layer_step(p, lw, x[:, t].contiguous(), ring, h, t, eps=oracle.RMS_EPS).clone() for t in range(T)]
    assert rglru.workspace_status(None) == 0
    assert rel(torch.stack(outs, 1), out_f) <= TOL[torch.bfloat16]
    assert rel(h, h_f) <= TOL[torch.bfloat16]
