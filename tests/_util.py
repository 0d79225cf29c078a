"""Shared test helpers: float64 views of tensors, the packed gate layout, oracle calls."""
import numpy as np
import torch

import oracle

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}

# Tolerance of the Hawk residual layer's output: out = x + o₁ + o₂ with o₁ the recurrent
# block's output (bf16 allowance 2e-2 of its own scale, as for the block) and o₂ the MLP's,
# which adds five bf16 roundings of O(1) quantities (RMSNorm₂ output, gate, up, GeLU product,
# down projection): 5 · 2⁻⁹ ≈ 1e-2. The two allowances add: 3e-2.
TOL_LAYER = 3e-2

# Tolerance of Griffin's local-attention decode step: its output passes through six bf16
# storage points between the bf16 input and the bf16 output (q, k and v from the fused
# projection; the rotated q and k; the softmax numerators; the merged o; the output
# projection). The float64 oracle with exactly those roundings (rounding_model.attention_step)
# reaches 2.48e-2 on the GPU test's first case (B=3, D=256, window 128, 300 steps; median
# 1.4e-2), which is what the GPU measures there too: the same 3e-2 as the layer's.
TOL_ATTN = 3e-2


def f64(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu").double().numpy()


def unpack_gates(z, R):
    """Packed gate rows [N][pitch] → (z_a [N][R], z_x [N][R]).

    Channel c's recurrence-gate pre-activation sits at column 256·(c//128) + c%128, its
    input-gate pre-activation 128 columns further."""
    z = f64(z)
    c = np.arange(R)
    col_a = 256 * (c // 128) + (c % 128)
    return z[:, col_a], z[:, col_a + 128]


def pack_gates(z_a, z_x, R, dtype, device):
    """Inverse of unpack_gates (unused columns zero)."""
    N = z_a.shape[0]
    pitch = ((R + 127) // 128) * 256
    out = np.zeros((N, pitch))
    c = np.arange(R)
    col_a = 256 * (c // 128) + (c % 128)
    out[:, col_a] = z_a
    out[:, col_a + 128] = z_x
    return torch.from_numpy(out).to(dtype).to(device)


def host_params64(p):
    """float64 numpy copies of a parameter set (so repeated oracle calls skip conversion)."""
    return dict(conv_w=f64(p.conv_w), conv_b=f64(p.conv_b), W_a=f64(p.W_a), b_a=f64(p.b_a), W_x=f64(p.W_x),
                b_x=f64(p.b_x), Lambda=f64(p.Lambda))


def rel(got, ref):
    return oracle.max_rel_error(f64(got), f64(ref))
