"""CPU oracle for the RG-LRU temporal core: Conv1D(4) → RG-LRU, and the recurrent block.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links this
module: only the test suite, the smoke check and the benchmark's CPU-baseline leg
use it. It shares no code with the CUDA path.

It is the plain definition, written out in float64 with numpy:
  * "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型",
    §实门线性循环单元 (RG-LRU), Eq. (1)–(4) and the paragraph after them:
        r_t = σ(W_a x_t + b_a)                      (1)  recurrence gate
        i_t = σ(W_x x_t + b_x)                      (2)  input gate
        a_t = a^(c·r_t),  a = σ(Λ),  c = 8          (3)
        h_t = a_t ⊙ h_{t-1} + √(1 − a_t²) ⊙ (i_t ⊙ x_t)   (4)
        y_t = h_t
    where the x_t of the RG-LRU is the output of the Conv1D that precedes it.
  * the same page, §循环块 (recurrent block): two D → D_RNN linears; branch 1 is a
    width-4 Conv1D followed by the RG-LRU, branch 2 is GeLU; the branches are
    multiplied elementwise and a final D_RNN → D linear follows.
  * the same page, §残块 (residual block, Fig. 2(a)) and §MLP块 (Fig. 2(b)): RMSNorm
    ahead of the temporal-mixing block and of a gated MLP (two D → M·D linears, GeLU
    on one, elementwise product, M·D → D linear), each merged with its skip connection.
  * "Griffin's Compromise: Combining Gated Linear Recurrence with Local Attention",
    §Hawk: during generation the layer reads and writes only the current token and
    a fixed-size state (the decode step below).

Readings where the pages are silent (each one is listed with its reason in the
design notes): the Conv1D is causal with zero left padding, per channel, with a
bias, tap k multiplying x_{t-3+k}; W_a and W_x are dense D_RNN × D_RNN; GeLU is the
exact erf form; the block and MLP linears have no bias; RMSNorm has a per-channel
gain and ε = 1e-6.

a_t is evaluated as the direct power a**(c*r_t) in float64. The log-space form the
page prescribes for numerical stability is kept as its own function
(decay_log_space) so that the two can be compared.

Parity pins for every function live in the oracle tests (closed forms, invariants,
brute-force sums, library special cases); nothing here is "parity unpinned" except
the readings named above, which no passage of the pages fixes.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

C_DECAY = 8.0      # the scalar constant c of Eq. (3)
CONV_WIDTH = 4     # temporal filter width of the Conv1D (§循环块)


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):          # torch tensor (bf16 upcasts exactly)
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def sigmoid(z):
    """σ(z) = 1 / (1 + e^{-z}), evaluated without overflow for large |z|."""
    z = np.asarray(z, dtype=np.float64)
    out = np.empty_like(z)
    pos = z >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-z[pos]))
    ez = np.exp(z[~pos])
    out[~pos] = ez / (1.0 + ez)
    return out


def conv1d_causal(x, conv_w, conv_b, state=None):
    """Causal depthwise Conv1D of width 4 (§循环块).

    x [B][T][R]; conv_w [4][R], tap k multiplies x_{t-3+k}; conv_b [R];
    state [B][3][R] holds (x_{-3}, x_{-2}, x_{-1}) in time order, zeros if None.
    Returns u [B][T][R] and the new state (the last three inputs, time order).
    """
    x = _f64(x)
    w = _f64(conv_w)
    b = _f64(conv_b)
    B, T, R = x.shape
    hist = np.zeros((B, CONV_WIDTH - 1, R)) if state is None else _f64(state)
    xp = np.concatenate([hist, x], axis=1)          # xp[:, s] = x_{s-3}
    u = np.broadcast_to(b, (B, T, R)).copy()
    for k in range(CONV_WIDTH):
        u += w[k] * xp[:, k:k + T, :]               # x_{t-3+k} sits at xp[:, t+k]
    new_state = xp[:, T:T + CONV_WIDTH - 1, :].copy()
    return u, new_state


def gate_preactivations(u, W_a, b_a, W_x, b_x, channels=None):
    """Arguments of σ in Eq. (1) and (2): z_a = W_a u_t + b_a, z_x = W_x u_t + b_x.

    u [..][R]; W_* [R][R] row-major [out][in]. If `channels` is given, only those
    output channels are formed (rows of W_* and entries of b_*)."""
    u = _f64(u)
    W_a, W_x, b_a, b_x = _f64(W_a), _f64(W_x), _f64(b_a), _f64(b_x)
    if channels is not None:
        W_a, W_x, b_a, b_x = W_a[channels], W_x[channels], b_a[channels], b_x[channels]
    z_a = u @ W_a.T + b_a
    z_x = u @ W_x.T + b_x
    return z_a, z_x


def decay_direct(r, Lambda, c=C_DECAY):
    """Eq. (3) as written: a_t = a^(c r_t) with a = σ(Λ)."""
    return sigmoid(_f64(Lambda)) ** (c * _f64(r))


def decay_log_space(r, Lambda, c=C_DECAY):
    """Eq. (3) in log space: log a_t = c r_t log σ(Λ), log σ(Λ) = −log(1 + e^{−Λ})."""
    Lam = _f64(Lambda)
    log_a = -np.logaddexp(0.0, -Lam)
    return np.exp(c * _f64(r) * log_a)


def rglru_recurrence(a_t, i_t, u, h0):
    """Eq. (4), one time step after another: h_t = a_t h_{t-1} + √(1 − a_t²)(i_t u_t).

    a_t, i_t, u [B][T][R]; h0 [B][R]. Returns y [B][T][R] (y_t = h_t) and h_T."""
    a_t, i_t, u = _f64(a_t), _f64(i_t), _f64(u)
    B, T, R = u.shape
    h = np.zeros((B, R)) if h0 is None else _f64(h0).copy()
    y = np.empty((B, T, R))
    for t in range(T):
        at = a_t[:, t, :]
        h = at * h + np.sqrt(1.0 - at * at) * (i_t[:, t, :] * u[:, t, :])
        y[:, t, :] = h
    return y, h


def rglru_forward(x, conv_w, conv_b, W_a, b_a, W_x, b_x, Lambda, h0=None,
                  conv_state0=None, channels=None, c=C_DECAY):
    """Full-sequence forward: Conv1D(4) then the RG-LRU (Eq. (1)–(4)).

    x [B][T][R]. Returns y [B][T][R'], h_T [B][R'], conv_state_T [B][3][R] where
    R' = len(channels) when only a subset of output channels is formed (each
    channel of the RG-LRU is independent of the others once u is known)."""
    u, conv_state_T = conv1d_causal(x, conv_w, conv_b, conv_state0)
    z_a, z_x = gate_preactivations(u, W_a, b_a, W_x, b_x, channels)
    r = sigmoid(z_a)                                    # Eq. (1)
    i = sigmoid(z_x)                                    # Eq. (2)
    Lam = _f64(Lambda)
    if channels is not None:
        Lam = Lam[channels]
        u = u[..., channels]
    a_t = decay_direct(r, Lam, c)                       # Eq. (3)
    if h0 is not None:
        h0 = _f64(h0)
        if channels is not None:
            h0 = h0[:, channels]
    y, h_T = rglru_recurrence(a_t, i, u, h0)            # Eq. (4)
    return y, h_T, conv_state_T


def ring_to_time_order(ring, step):
    """Decode conv ring [B][3][R]: slot (step mod 3) holds the oldest input x_{t-3},
    slot (step+1) mod 3 holds x_{t-2}, slot (step+2) mod 3 holds x_{t-1}."""
    ring = _f64(ring)
    order = [(step + j) % 3 for j in range(3)]
    return ring[:, order, :]


def rglru_step(x_t, ring, step, h, conv_w, conv_b, W_a, b_a, W_x, b_x, Lambda,
               c=C_DECAY, rows=None):
    """One decode step on a carried state (the layer reads the current token and a
    fixed-size state only).

    x_t [B][R]; ring [B][3][R] (see ring_to_time_order); h [B][R].
    Returns y_t [B][R], the new h, and the new ring, in which slot (step mod 3) now
    holds x_t. `rows` restricts the work to those batch rows (rows are independent).
    """
    x_t = _f64(x_t)
    h = _f64(h)
    ring = _f64(ring)
    if rows is not None:
        x_t, h, ring = x_t[rows], h[rows], ring[rows]
    hist = ring_to_time_order(ring, step)               # (x_{t-3}, x_{t-2}, x_{t-1})
    u, _ = conv1d_causal(x_t[:, None, :], conv_w, conv_b, hist)
    z_a, z_x = gate_preactivations(u, W_a, b_a, W_x, b_x)
    r, i = sigmoid(z_a), sigmoid(z_x)
    a_t = decay_direct(r, Lambda, c)
    y, h_new = rglru_recurrence(a_t, i, u, h)
    new_ring = ring.copy()
    new_ring[:, step % 3, :] = x_t
    return y[:, 0, :], h_new, new_ring


def gelu(x):
    """GeLU in its exact form x Φ(x) = ½ x (1 + erf(x/√2)) (Hendrycks & Gimpel)."""
    x = _f64(x)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def recurrent_block(x, W_1, W_2, W_o, conv_w, conv_b, W_a, b_a, W_x, b_x, Lambda,
                    h0=None, c=C_DECAY):
    """Recurrent block (§循环块, Fig. 2(c)).

    x [B][T][D]; W_1, W_2 [R][D] (D → D_RNN); W_o [D][R] (D_RNN → D).
    Branch 1: v = x W_1ᵀ → Conv1D(4) → RG-LRU → h.  Branch 2: g = x W_2ᵀ → GeLU.
    out = (h ⊙ GeLU(g)) W_oᵀ.  Returns out [B][T][D] and h_T."""
    x = _f64(x)
    v = x @ _f64(W_1).T
    g = x @ _f64(W_2).T
    h, h_T, _ = rglru_forward(v, conv_w, conv_b, W_a, b_a, W_x, b_x, Lambda, h0, c=c)
    p = h * gelu(g)
    out = p @ _f64(W_o).T
    return out, h_T


# ε of RMSNorm: the page gives none; 1e-6 is taken (a reading, listed in the design notes).
RMS_EPS = 1e-6


def rms_norm(x, scale, eps=RMS_EPS):
    """RMSNorm (Zhang & Sennrich, 2019) over the last axis, as the residual block applies
    it ahead of each of its two sub-blocks (§残块, Fig. 2(a)):
        n = x / √(mean_j x_j² + ε) ⊙ scale,   scale [D] a per-channel gain, no bias."""
    x = _f64(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * _f64(scale)


def gated_mlp(x, W_gate, W_up, W_down):
    """Gated MLP block (§MLP块, Fig. 2(b)): two D → M·D linears, GeLU on the first
    (gate) branch, the branches multiplied elementwise, then an M·D → D linear.
    W_gate, W_up [M·D][D]; W_down [D][M·D]; no biases."""
    x = _f64(x)
    return (gelu(x @ _f64(W_gate).T) * (x @ _f64(W_up).T)) @ _f64(W_down).T


def hawk_residual_layer(x, norm1_scale, W_1, W_2, W_o, norm2_scale, W_gate, W_up, W_down,
                        conv_w, conv_b, W_a, b_a, W_x, b_x, Lambda, h0=None, eps=RMS_EPS, c=C_DECAY):
    """One residual block of Hawk (§残块, Fig. 2(a)) with the recurrent block as its
    temporal-mixing block. Two components in sequence, each pre-normed and merged with
    the skip connection from its own RMSNorm input:
        y   = x + RecurrentBlock(RMSNorm₁(x))
        out = y + MLP(RMSNorm₂(y))
    Returns out [B][T][D] and the RG-LRU's h_T."""
    x = _f64(x)
    o, h_T = recurrent_block(rms_norm(x, norm1_scale, eps), W_1, W_2, W_o, conv_w, conv_b, W_a, b_a,
                             W_x, b_x, Lambda, h0, c=c)
    y = x + o
    out = y + gated_mlp(rms_norm(y, norm2_scale, eps), W_gate, W_up, W_down)
    return out, h_T


def hawk_residual_layer_step(x_t, ring, step, h, norm1_scale, W_1, W_2, W_o, norm2_scale, W_gate, W_up,
                             W_down, conv_w, conv_b, W_a, b_a, W_x, b_x, Lambda, eps=RMS_EPS, c=C_DECAY):
    """One decode step of the Hawk residual layer: hawk_residual_layer at a single token
    with the recurrent block's carried state — RMSNorm₁, the block's two linears, one
    RG-LRU decode step (rglru_step: the conv ring holds the last three inputs of the
    Conv1D, i.e. of the x W_1ᵀ branch), the GeLU gate, W_o, the residual add, RMSNorm₂,
    the gated MLP and the second residual add. Every part but the RG-LRU acts on each token
    alone.

    x_t [B][D]; ring [B][3][R]; h [B][R]. Returns out_t [B][D], the new h, the new ring."""
    x_t = _f64(x_t)
    n1 = rms_norm(x_t, norm1_scale, eps)
    v_t = n1 @ _f64(W_1).T
    g_t = n1 @ _f64(W_2).T
    y_t, h_new, ring_new = rglru_step(v_t, ring, step, h, conv_w, conv_b, W_a, b_a, W_x, b_x, Lambda, c=c)
    y = x_t + (y_t * gelu(g_t)) @ _f64(W_o).T
    out = y + gated_mlp(rms_norm(y, norm2_scale, eps), W_gate, W_up, W_down)
    return out, h_new, ring_new


def rglru_backward(x, conv_w, conv_b, W_a, b_a, W_x, b_x, Lambda, dy, h0=None, conv_state0=None,
                   dh_T=None, c=C_DECAY):
    """Gradients of the full-sequence forward (rglru_forward) by reverse-mode
    differentiation of the same definition, step by step, in float64.

    For a scalar loss ℓ with ∂ℓ/∂y = dy [B][T][R] and ∂ℓ/∂h_T = dh_T [B][R] (zero if
    None), returns a dict with dx [B][T][R], dconv_w [4][R], dconv_b [R], dW_a, dW_x
    [R][R], db_a, db_x, dLambda [R], dh0 [B][R] and dconv_state0 [B][3][R].

    The forward, per batch row and channel (Eq. (1)–(4) with log a_t = c r_t log σ(Λ)):
        r_t = σ(z_a,t), i_t = σ(z_x,t), a_t = exp(c r_t L), L = log σ(Λ),
        m_t = √(1 − a_t²), h_t = a_t h_{t-1} + m_t i_t u_t, y_t = h_t.
    Walking t from T−1 down to 0 with g = ∂ℓ/∂h_t (g starts at dh_T and takes dy_t at
    each step): ∂a_t = g h_{t-1}, ∂m_t = g i_t u_t, ∂i_t = g m_t u_t, ∂u_t += g m_t i_t,
    then g ← a_t g for h_{t-1}. Through a_t and m_t (∂m/∂log a = −a²/m):
    ∂log a_t = ∂a_t a_t − ∂m_t a_t²/m_t; ∂r_t = ∂log a_t c L; ∂L += ∂log a_t c r_t;
    ∂z_a = ∂r r(1 − r), ∂z_x = ∂i i(1 − i). Both uses of ∂log a_t carry a factor r_t, so
    they are formed from ∂log a_t·r_t = ∂a_t a_t r_t − ∂m_t a_t² (r_t/m_t), where r_t/m_t → 0
    as r_t → 0 (m_t ≈ √(−2 c r_t L)); at r_t = 0 exactly (a_t = 1, m_t = 0) it is taken as its
    limit 0. Then the two linears and the Conv1D are differentiated as written
    (dΛ = ∂L·σ(−Λ), since L = −log(1 + e^{−Λ})).
    """
    x = _f64(x)
    B, T, R = x.shape
    Wa, Wx = _f64(W_a), _f64(W_x)
    u, _ = conv1d_causal(x, conv_w, conv_b, conv_state0)
    z_a, z_x = gate_preactivations(u, W_a, b_a, W_x, b_x)
    r, i = sigmoid(z_a), sigmoid(z_x)
    Lam = _f64(Lambda)
    L = -np.logaddexp(0.0, -Lam)                        # log σ(Λ)
    a = np.exp(c * r * L)
    m = np.sqrt(1.0 - a * a)
    h_prev0 = np.zeros((B, R)) if h0 is None else _f64(h0)
    y, _ = rglru_recurrence(a, i, u, h_prev0)
    dy = _f64(dy)
    g = np.zeros((B, R)) if dh_T is None else _f64(dh_T).copy()
    dz_a = np.empty((B, T, R))
    dz_x = np.empty((B, T, R))
    du = np.empty((B, T, R))
    dL = np.zeros(R)
    for t in range(T - 1, -1, -1):
        g = g + dy[:, t]
        hp = y[:, t - 1] if t > 0 else h_prev0
        at, mt, it, ut, rt = a[:, t], m[:, t], i[:, t], u[:, t], r[:, t]
        d_a = g * hp
        d_m = g * it * ut
        d_i = g * mt * ut
        du[:, t] = g * mt * it
        r_over_m = np.divide(rt, mt, out=np.zeros_like(rt), where=mt > 0.0)
        d_loga_r = d_a * at * rt - d_m * at * at * r_over_m      # ∂log a_t · r_t
        dz_a[:, t] = d_loga_r * c * L * (1.0 - rt)
        dL += np.sum(d_loga_r * c, axis=0)
        dz_x[:, t] = d_i * it * (1.0 - it)
        g = g * at
    dh0 = g
    zf_a = dz_a.reshape(B * T, R)
    zf_x = dz_x.reshape(B * T, R)
    uf = u.reshape(B * T, R)
    dW_a = zf_a.T @ uf
    dW_x = zf_x.T @ uf
    db_a = zf_a.sum(axis=0)
    db_x = zf_x.sum(axis=0)
    du = du + (zf_a @ Wa + zf_x @ Wx).reshape(B, T, R)
    # Conv1D: u_t = b + Σ_k w_k x_{t-3+k}, history (x_{-3}, x_{-2}, x_{-1}) from conv_state0
    w = _f64(conv_w)
    hist = np.zeros((B, CONV_WIDTH - 1, R)) if conv_state0 is None else _f64(conv_state0)
    xp = np.concatenate([hist, x], axis=1)              # xp[:, s] = x_{s-3}
    dxp = np.zeros_like(xp)
    dconv_w = np.empty((CONV_WIDTH, R))
    for k in range(CONV_WIDTH):
        dconv_w[k] = np.sum(du * xp[:, k:k + T, :], axis=(0, 1))
        dxp[:, k:k + T, :] += w[k] * du
    return {
        "dx": dxp[:, CONV_WIDTH - 1:, :], "dconv_state0": dxp[:, :CONV_WIDTH - 1, :],
        "dconv_w": dconv_w, "dconv_b": du.sum(axis=(0, 1)),
        "dW_a": dW_a, "db_a": db_a, "dW_x": dW_x, "db_x": db_x,
        "dLambda": dL * sigmoid(-Lam), "dh0": dh0,
    }


def max_rel_error(got, ref):
    """Error measure for parity: max_i |g_i − o_i| / max(|o_i|, rms(o)).

    The denominator's floor rms(o) keeps the ratio defined where o crosses zero."""
    got = _f64(got)
    ref = _f64(ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    den = np.maximum(np.abs(ref), rms)
    den = np.where(den == 0.0, 1.0, den)
    return float(np.max(np.abs(got - ref) / den))
