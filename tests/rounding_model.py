"""The float64 oracle's arithmetic with the bf16 path's storage roundings, and nothing else.

Test infrastructure (CPU only; no CUDA code is involved). The CUDA path stores some of its
intermediates in narrow formats and does all arithmetic between them in float32:
  * the forward: the Conv1D output u (bf16, the gate GEMM's operand and the u inside b_t),
    the recurrence coefficients d = 1 − a_t (fp16) and b_t = √(1 − a_t²)·i_t·u_t (bf16)
    — not in the fused gate GEMM + scan, which keeps them in registers — and y (bf16);
  * the recurrent block in addition: v = x W_1ᵀ and g = x W_2ᵀ (bf16), the gated product
    h ⊙ GeLU(g) (bf16) and the block output (bf16);
  * the Hawk residual layer in addition: both RMSNorm outputs, the residual stream, the
    MLP's gate and up projections, their GeLU product and the down projection (bf16);
  * the backward: the recomputed pre-activations and ∂z (bf16), h_{t−1} read from the
    forward's bf16 y.
Each function below is the oracle's definition with exactly those roundings (round to
nearest even, through torch's casts) applied where the CUDA path stores a value. Its
distance from the unrounded oracle is the error the storage formats alone force on any
implementation with these formats; its distance from the GPU is the error the kernels add
on top of that (float32 accumulation order, approximate exponentials), which is far smaller.
"""
import numpy as np
import torch

import oracle


def f(t):
    """float64 numpy copy of a tensor or array."""
    return t.double().numpy() if torch.is_tensor(t) else np.asarray(t, dtype=np.float64)


def bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def fp16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.float16).double().numpy()


def rms_norm(v, gain, eps=oracle.RMS_EPS):
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps) * f(gain)


def coefficients(u, P, stored=True):
    """(d, b) as the gate GEMM's epilogue stores them (d fp16, b bf16), from the bf16 u
    [..][R]; unrounded with stored=False (the fused gate GEMM + scan keeps them in
    registers)."""
    r = oracle.sigmoid(u @ f(P.W_a).T + f(P.b_a))
    i = oracle.sigmoid(u @ f(P.W_x).T + f(P.b_x))
    a_t = oracle.decay_direct(r, f(P.Lambda))
    d, b = 1.0 - a_t, np.sqrt(1.0 - a_t * a_t) * i * u
    return (fp16(d), bf16(b)) if stored else (d, b)


def scan(d, b, h0):
    """h_t = (1 − d)·h_{t−1} + b_t over [B][T][R] (unrounded states); returns all h_t, h_T."""
    B, T, R = d.shape
    h = np.zeros((B, R)) if h0 is None else f(h0).copy()
    hs = np.empty_like(d)
    for t in range(T):
        h = (1.0 - d[:, t]) * h + b[:, t]
        hs[:, t] = h
    return hs, h


def forward(x, P, h0=None, conv_state0=None, fused=False):
    """rglru_forward with bf16 IO: returns (y [B][T][R], h_T [B][R]); fused=True for the
    gate GEMM with the scan in its epilogue (T a multiple of 128), whose coefficients are
    never stored."""
    u, _ = oracle.conv1d_causal(f(x), f(P.conv_w), f(P.conv_b), None if conv_state0 is None else f(conv_state0))
    u = bf16(u)
    d, b = coefficients(u, P, stored=not fused)
    hs, h_T = scan(d, b, h0)
    return bf16(hs), h_T


def block(x, W_1, W_2, W_o, P, h0=None):
    """rglru_block_forward: returns (out [B][T][D], h_T)."""
    x = f(x)
    v, g = bf16(x @ f(W_1).T), bf16(x @ f(W_2).T)
    u, _ = oracle.conv1d_causal(v, f(P.conv_w), f(P.conv_b))
    u = bf16(u)
    d, b = coefficients(u, P)
    hs, h_T = scan(d, b, h0)
    return bf16(bf16(hs * oracle.gelu(g)) @ f(W_o).T), h_T


def layer(x, P, W_1, W_2, W_o, norm1_scale, norm2_scale, W_gate, W_up, W_down, h0=None):
    """rglru_layer_forward: returns (out [B][T][D], h_T)."""
    x = f(x)
    o1, h_T = block(bf16(rms_norm(x, norm1_scale)), W_1, W_2, W_o, P, h0)
    y = bf16(x + o1)
    n2 = bf16(rms_norm(y, norm2_scale))
    gate, up = bf16(n2 @ f(W_gate).T), bf16(n2 @ f(W_up).T)
    o2 = bf16(bf16(oracle.gelu(gate) * up) @ f(W_down).T)
    return bf16(y + o2), h_T


def layer_from_workload(w, h0=None):
    e = w.extra
    return layer(w.x, w.params, w.W_1, w.W_2, w.W_o, e["norm1_scale"], e["norm2_scale"], e["W_gate"], e["W_up"],
                 e["W_down"], h0)


def backward_weight_gradients(x, P, dy, h0=None, conv_state0=None, dh_T=None):
    """∂W_a and ∂W_x of rglru_backward: u and the recomputed pre-activations z in bf16,
    h_{t−1} read from the forward's bf16 y (itself from fp16 d, bf16 b), ∂z in bf16 as the
    operand of ∂W = Σ_t ∂z_tᵀ u_t, exact arithmetic elsewhere."""
    cla = 8.0 * -np.log1p(np.exp(-f(P.Lambda)))
    u, _ = oracle.conv1d_causal(f(x), f(P.conv_w), f(P.conv_b), None if conv_state0 is None else f(conv_state0))
    u = bf16(u)
    B, T, R = u.shape
    za, zx = u @ f(P.W_a).T + f(P.b_a), u @ f(P.W_x).T + f(P.b_x)
    y, _ = forward(x, P, h0, conv_state0)
    r, i = oracle.sigmoid(bf16(za)), oracle.sigmoid(bf16(zx))
    la = r * cla
    at, mt = np.exp(la), np.sqrt(-np.expm1(2.0 * la))
    hp = np.concatenate([np.zeros((B, 1, R)) if h0 is None else f(h0)[:, None], y[:, :-1]], axis=1)
    g, a_next = (np.zeros((B, R)) if dh_T is None else f(dh_T)), np.ones((B, R))
    dza, dzx = np.empty_like(u), np.empty_like(u)
    dy = f(dy)
    for t in range(T - 1, -1, -1):
        g = a_next * g + dy[:, t]
        r_over_m = np.divide(r[:, t], mt[:, t], out=np.zeros((B, R)), where=mt[:, t] > 0)
        dlr = g * hp[:, t] * at[:, t] * r[:, t] - g * i[:, t] * u[:, t] * at[:, t] ** 2 * r_over_m
        dza[:, t] = dlr * cla * (1.0 - r[:, t])
        dzx[:, t] = g * mt[:, t] * u[:, t] * i[:, t] * (1.0 - i[:, t])
        a_next = at[:, t]
    dW_a = bf16(dza).reshape(-1, R).T @ u.reshape(-1, R)
    dW_x = bf16(dzx).reshape(-1, R).T @ u.reshape(-1, R)
    return dW_a, dW_x


def rms_rel(got, ref):
    """rms(got − ref) / rms(ref): the typical size of a difference, next to the maximum."""
    got, ref = f(got), f(ref)
    return float(np.sqrt(np.mean((got - ref) ** 2)) / np.sqrt(np.mean(ref ** 2)))


def attention_step(x_t, K, V, pos, W_qkv, W_o, window, chunk=128):
    """rglru_attention_step with the path's roundings: qkv = x W_qkvᵀ (bf16), the rotated q and
    k (bf16; k and v stored in the rings), per 128-slot chunk of the ring the softmax
    numerators 2^(s − m_c) in bf16 (m_c the chunk's maximum) and their sum l_c, the merged
    o = Σ_c 2^(m_c − m) O_c / Σ_c 2^(m_c − m) l_c (bf16), out = o W_oᵀ (bf16). K, V [B][W][128]
    as the oracle holds them (modified in place). Returns out_t."""
    x_t = f(x_t)
    B = x_t.shape[0]
    dh = 128
    H = (f(W_qkv).shape[0] // dh) - 2
    qkv = bf16(x_t @ f(W_qkv).T)
    p = np.array([pos])
    q = bf16(oracle.rope(qkv[:, :H * dh].reshape(B, H, dh), p))
    slot = pos % window
    K[:, slot] = bf16(oracle.rope(qkv[:, None, H * dh:(H + 1) * dh], p)[:, 0])
    V[:, slot] = qkv[:, (H + 1) * dh:]
    n_valid = window if pos >= window - 1 else pos + 1
    s = np.einsum("bhd,bnd->bhn", q, K[:, :n_valid]) / np.sqrt(dh) / np.log(2.0)   # log2 units
    num = np.zeros((B, H, dh))
    den = np.zeros((B, H))
    ms = [s[:, :, c0:c0 + chunk].max(axis=-1) for c0 in range(0, n_valid, chunk)]
    m = np.max(np.stack(ms), axis=0)
    for c, c0 in enumerate(range(0, n_valid, chunk)):
        pc = bf16(np.exp2(s[:, :, c0:c0 + chunk] - ms[c][..., None]))
        w = np.exp2(ms[c] - m)
        num += w[..., None] * np.einsum("bhn,bnd->bhd", pc, V[:, c0:min(c0 + chunk, n_valid)])
        den += w * pc.sum(axis=-1)
    o = bf16((num / den[..., None]).reshape(B, H * dh))
    return bf16(o @ f(W_o).T)


def attention_layer_step(x_t, K, V, pos, w, window):
    """rglru_attention_layer_step with the path's roundings (the attention step above on the
    bf16 RMSNorm output, then the residual adds and the gated MLP as in `layer`). `w` holds
    W_q, W_k, W_v, W_o, the norm gains and the MLP weights. Returns out_t."""
    x = f(x_t)
    W_qkv = np.concatenate([f(w["W_q"]), f(w["W_k"]), f(w["W_v"])], 0)
    o1 = attention_step(bf16(rms_norm(x, w["norm1_scale"])), K, V, pos, W_qkv, w["W_o"], window)
    y = bf16(x + o1)
    n2 = bf16(rms_norm(y, w["norm2_scale"]))
    gate, up = bf16(n2 @ f(w["W_gate"]).T), bf16(n2 @ f(w["W_up"]).T)
    o2 = bf16(bf16(oracle.gelu(gate) * up) @ f(w["W_down"]).T)
    return bf16(y + o2)
