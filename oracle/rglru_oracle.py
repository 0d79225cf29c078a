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
  * "Griffin's Compromise: Combining Gated Linear Recurrence with Local Attention",
    §Hawk: during generation the layer reads and writes only the current token and
    a fixed-size state (the decode step below).

Readings where the pages are silent (each one is listed with its reason in the
design notes): the Conv1D is causal with zero left padding, per channel, with a
bias, tap k multiplying x_{t-3+k}; W_a and W_x are dense D_RNN × D_RNN; GeLU is the
exact erf form; the block linears have no bias.

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
