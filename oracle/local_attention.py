"""CPU oracle for Griffin's local (sliding-window) multi-query attention, prefill and decode.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links this
module: only the test suite, the smoke check and the benchmark's CPU-baseline leg use it.
It shares no code with the CUDA path.

The definition, in float64 numpy:
  * "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §时间混合块:
    global MQA — H query heads of width D_head = 128 with H·D_head = D, one key/value head
    shared by all query heads (multi-query attention, Shazeer 2019), no absolute position
    embedding, rotary position embedding (RoPE, Su et al. 2021) as the relative one;
    local sliding-window attention — each position attends only to a fixed number of past
    positions, which bounds the KV cache by the window; everything else as global MQA.
  * "Griffin's Compromise: Combining Gated Linear Recurrence with Local Attention",
    §"Griffin: Attention for Recent Memory, Recurrence for Long-Range Flow": the default
    window is 1024 tokens, and a local-attention residual block follows every two recurrent
    residual blocks.

Readings where the pages are silent (listed with reasons in the design notes): the window
W counts the current position, so position t attends to t−W+1 … t; scores are scaled by
1/√D_head; RoPE rotates the interleaved pairs (x_{2i}, x_{2i+1}) by angle p·θ_i with
θ_i = 10000^(−2i/D_head), applied to queries and keys (not values) at their absolute
positions; the q, k, v and output projections have no bias; the decode cache is a ring of
W slots where slot (p mod W) holds position p.
"""
from __future__ import annotations

import numpy as np

ROPE_BASE = 10000.0
WINDOW = 1024


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def rope(x, positions, base=ROPE_BASE):
    """Rotary position embedding (Su et al.): x [..., P, d] with d even and `positions` [P]
    integer positions. Pair i = (x_{2i}, x_{2i+1}) is rotated by the angle p·θ_i,
    θ_i = base^(−2i/d):  (a, b) ↦ (a cos − b sin, a sin + b cos)."""
    x = _f64(x)
    d = x.shape[-1]
    theta = base ** (-np.arange(0, d, 2, dtype=np.float64) / d)          # [d/2]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]  # [P][d/2]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def local_mqa(q, k, v, window=WINDOW):
    """Sliding-window multi-query attention over a whole sequence.

    q [B][T][H][dh] (already rotated), k, v [B][T][dh] (k rotated): the one key/value head
    is shared by the H query heads. Position t attends to s with t − window < s ≤ t:
        o[b, t, h] = Σ_s softmax_s(q[b,t,h]·k[b,s] / √dh) v[b,s].
    Returns o [B][T][H][dh]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, dh = q.shape
    o = np.empty_like(q)
    for t in range(T):
        s0 = max(0, t - window + 1)
        ks, vs = k[:, s0:t + 1], v[:, s0:t + 1]                  # [B][n][dh]
        sc = np.einsum("bhd,bnd->bhn", q[:, t], ks) / np.sqrt(dh)
        sc = sc - sc.max(axis=-1, keepdims=True)
        p = np.exp(sc)
        p /= p.sum(axis=-1, keepdims=True)
        o[:, t] = np.einsum("bhn,bnd->bhd", p, vs)
    return o


def local_attention(x, W_q, W_k, W_v, W_o, window=WINDOW, pos0=0):
    """The local-MQA temporal-mixing block over a sequence: x [B][T][D] →
    q = x W_qᵀ (H heads of dh), k = x W_kᵀ, v = x W_vᵀ (one head), RoPE on q and k at
    positions pos0 … pos0+T−1, sliding-window attention, out = o W_oᵀ [B][T][D].
    W_q [H·dh][D], W_k, W_v [dh][D], W_o [D][H·dh]."""
    x = _f64(x)
    W_q, W_k, W_v, W_o = _f64(W_q), _f64(W_k), _f64(W_v), _f64(W_o)
    B, T, _ = x.shape
    dh = W_k.shape[0]
    H = W_q.shape[0] // dh
    pos = np.arange(pos0, pos0 + T)
    q = rope((x @ W_q.T).reshape(B, T, H, dh).transpose(0, 2, 1, 3), pos).transpose(0, 2, 1, 3)
    k = rope(x @ W_k.T, pos)
    v = x @ W_v.T
    o = local_mqa(q, k, v, window)
    return o.reshape(B, T, H * dh) @ W_o.T


def local_attention_step(x_t, K_ring, V_ring, pos, W_q, W_k, W_v, W_o, window=WINDOW):
    """One decode step of the local-MQA block at position `pos` on a ring KV cache.

    x_t [B][D]; K_ring, V_ring [B][window][dh]: slot (p mod window) holds the rotated key
    and the value of position p, for the positions seen so far (pos of them). The step
    writes position pos into slot (pos mod window), then attends to the slots holding
    positions max(0, pos − window + 1) … pos. Returns out_t [B][D] and the new rings."""
    x_t = _f64(x_t)
    W_q, W_k, W_v, W_o = _f64(W_q), _f64(W_k), _f64(W_v), _f64(W_o)
    K, V = _f64(K_ring).copy(), _f64(V_ring).copy()
    B, D = x_t.shape
    dh = W_k.shape[0]
    H = W_q.shape[0] // dh
    p = np.array([pos])
    q = rope((x_t @ W_q.T).reshape(B, H, dh), p)                 # one position: rows are heads
    k = rope((x_t @ W_k.T)[:, None, :], p)[:, 0]
    v = x_t @ W_v.T
    slot = pos % window
    K[:, slot], V[:, slot] = k, v
    n = min(pos + 1, window)
    slots = [(pos - j) % window for j in range(n)]                 # the window's positions, newest first
    sc = np.einsum("bhd,bnd->bhn", q, K[:, slots]) / np.sqrt(dh)
    sc = sc - sc.max(axis=-1, keepdims=True)
    w = np.exp(sc)
    w /= w.sum(axis=-1, keepdims=True)
    o = np.einsum("bhn,bnd->bhd", w, V[:, slots])
    return o.reshape(B, H * dh) @ W_o.T, K, V


def griffin_attention_layer(x, norm1_scale, W_q, W_k, W_v, W_o, norm2_scale, W_gate, W_up, W_down,
                            window=WINDOW, eps=None, pos0=0):
    """The residual block of Griffin whose temporal-mixing block is local MQA (§残块, Fig. 2(a),
    with the local-attention block of §时间混合块): each component pre-normed by RMSNorm and
    merged with the skip connection from its own RMSNorm input, as in the Hawk layer:
        y   = x + LocalMQA(RMSNorm₁(x)),   out = y + MLP(RMSNorm₂(y))."""
    from .rglru_oracle import RMS_EPS, gated_mlp, rms_norm
    eps = RMS_EPS if eps is None else eps
    x = _f64(x)
    y = x + local_attention(rms_norm(x, norm1_scale, eps), W_q, W_k, W_v, W_o, window, pos0)
    return y + gated_mlp(rms_norm(y, norm2_scale, eps), W_gate, W_up, W_down)


def griffin_attention_layer_step(x_t, K_ring, V_ring, pos, norm1_scale, W_q, W_k, W_v, W_o, norm2_scale,
                                 W_gate, W_up, W_down, window=WINDOW, eps=None):
    """One decode step of griffin_attention_layer at position `pos` on the ring KV cache of
    local_attention_step. Returns out_t [B][D] and the new rings."""
    from .rglru_oracle import RMS_EPS, gated_mlp, rms_norm
    eps = RMS_EPS if eps is None else eps
    x_t = _f64(x_t)
    o, K, V = local_attention_step(rms_norm(x_t, norm1_scale, eps), K_ring, V_ring, pos, W_q, W_k, W_v, W_o, window)
    y = x_t + o
    return y + gated_mlp(rms_norm(y, norm2_scale, eps), W_gate, W_up, W_down), K, V
