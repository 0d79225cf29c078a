"""Pins for the CPU oracle: each test checks it against something other than itself.

Sources of truth: hand-worked examples (tests/golden), closed forms that follow from
Eq. (3)-(4) of the RG-LRU section of "Griffin：将门控线性循环与局部注意力混合以实现
高效的语言模型", invariants of the linear recurrence (superposition, split and
step equivalence), brute-force enumeration on tiny inputs, and library routines for
the special cases that reduce to them (torch conv1d, matmul, GeLU, scipy expit).
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from gated_linear_rnn_conv1d_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.txt")


def _parse_golden(path):
    examples, cur = {}, None
    for line in open(path, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("[example"):
            cur = examples.setdefault(line[len("[example"):-1].strip(), {})
            continue
        key, val = (s.strip() for s in line.split("=", 1))
        vals = []
        for v in val.split(","):
            v = v.strip()
            sign = -1.0 if v.startswith("-") else 1.0
            v = v.lstrip("-")
            vals.append(sign * (math.log(3.0) if v == "ln3" else float(v)))
        cur[key] = np.array(vals)
    return examples


def _rng_params(rng, R, lam_lo=4.0, lam_hi=9.0, wscale=None):
    wscale = 1.0 / math.sqrt(R) if wscale is None else wscale
    return dict(
        conv_w=rng.normal(0, 0.5, (4, R)), conv_b=rng.normal(0, 0.5, R),
        W_a=rng.normal(0, wscale, (R, R)), b_a=rng.normal(0, 0.3, R),
        W_x=rng.normal(0, wscale, (R, R)), b_x=rng.normal(0, 0.3, R),
        Lambda=rng.uniform(lam_lo, lam_hi, R),
    )


@pytest.mark.parametrize("name", ["identity_conv", "taps_and_state"])
def test_hand_worked_examples(name):
    ex = _parse_golden(GOLDEN)[name]
    T = ex["x"].size
    x = ex["x"].reshape(1, T, 1)
    y, h_T, _ = oracle.rglru_forward(
        x, ex["conv_w"].reshape(4, 1), ex["conv_b"], np.zeros((1, 1)), ex["b_a"],
        np.zeros((1, 1)), ex["b_x"], ex["Lambda"], h0=ex["h0"].reshape(1, 1))
    np.testing.assert_allclose(y.ravel(), ex["y"], rtol=1e-15, atol=1e-15)
    assert h_T.ravel()[0] == y.ravel()[-1]
    if "u" in ex:
        u, _ = oracle.conv1d_causal(x, ex["conv_w"].reshape(4, 1), ex["conv_b"])
        np.testing.assert_allclose(u.ravel(), ex["u"], rtol=0, atol=1e-15)


def test_sigmoid_matches_scipy():
    z = np.concatenate([np.linspace(-800, 800, 4001), [0.0, -1e-300, 1e-300]])
    np.testing.assert_allclose(oracle.sigmoid(z), expit(z), rtol=1e-15, atol=1e-300)


def test_O1_zero_recurrence_gate_keeps_state_bitwise():
    """r ≡ 0 ⇒ a_t = a^0 = 1 and √(1 − 1) = 0, so h_t = h_0 for every t (the gate's
    'keep history, discard input' end, §门行为)."""
    rng = np.random.default_rng(1)
    B, T, R = 3, 17, 12
    p = _rng_params(rng, R)
    p["W_a"] = np.zeros((R, R))
    p["b_a"] = np.full(R, -1000.0)          # σ(−1000) underflows to exactly 0
    x = rng.normal(size=(B, T, R))
    h0 = rng.normal(size=(B, R))
    y, h_T, _ = oracle.rglru_forward(x, h0=h0, **p)
    assert np.array_equal(y, np.broadcast_to(h0[:, None, :], y.shape))
    assert np.array_equal(h_T, h0)


def test_O2_constant_gates_geometric_sum():
    """W_a = W_x = 0 and zero conv taps ⇒ r, i, u constant; Eq. (4) unrolls to
    h_T = α^T h0 + m i κ (1 − α^T)/(1 − α), α = σ(Λ)^(8σ(b_a)), m = √(1 − α²)."""
    rng = np.random.default_rng(2)
    B, T, R = 2, 300, 5
    kappa = rng.normal(size=R)
    Lam = rng.uniform(-2, 9, R)
    b_a = rng.normal(size=R)
    b_x = rng.normal(size=R)
    h0 = rng.normal(size=(B, R))
    x = rng.normal(size=(B, T, R))
    y, h_T, _ = oracle.rglru_forward(
        x, np.zeros((4, R)), kappa, np.zeros((R, R)), b_a, np.zeros((R, R)), b_x, Lam, h0=h0)
    a = expit(Lam)
    alpha = a ** (8.0 * expit(b_a))
    m = np.sqrt(1.0 - alpha ** 2)
    i = expit(b_x)
    for t in (1, 7, T):
        want = alpha ** t * h0 + m * i * kappa * (1 - alpha ** t) / (1 - alpha)
        np.testing.assert_allclose(y[:, t - 1, :], want, rtol=1e-11, atol=1e-12)


def test_O3_unit_variance_fixed_point():
    """i ≡ 1, constant r, identity conv, x i.i.d. N(0,1), h0 = 0:
    Var(h_t) = (1 − α²) Σ_{k<t} α^{2k} = 1 − α^{2t} (the √(1 − a_t²) normalisation)."""
    rng = np.random.default_rng(3)
    B, T, R = 100, 120, 1000
    Lam = np.full(R, math.log(0.9 ** (1 / 8)) - math.log1p(-(0.9 ** (1 / 8))))
    w = np.zeros((4, R))
    w[3] = 1.0
    x = rng.normal(size=(B, T, R))
    y, _, _ = oracle.rglru_forward(x, w, np.zeros(R), np.zeros((R, R)), np.zeros(R),
                                   np.zeros((R, R)), np.full(R, 1000.0), Lam)
    alpha = 0.9 ** 0.5                      # a^8 = 0.9 and r = 1/2 ⇒ a_t = a^4
    n = B * R
    for t in (1, 10, T):
        var = float(np.mean(y[:, t - 1, :] ** 2))
        want = 1.0 - alpha ** (2 * t)
        se = math.sqrt(2.0 / n) * want
        assert abs(var - want) < 4 * se, (t, var, want)


def test_O4_log_space_equals_direct_power():
    """log-space evaluation of a^(c r) (the page's numerically stable route) equals
    the direct power over the init range of Λ and r ∈ [0, 1]."""
    Lam = np.linspace(4.33, 8.99, 257)[:, None]
    r = np.linspace(0.0, 1.0, 129)[None, :]
    d = oracle.decay_direct(r, Lam)
    l = oracle.decay_log_space(r, Lam)
    assert np.max(np.abs(d - l) / d) <= 1e-14
    # and over a wide range of Λ, including a ≪ 1
    Lam = np.linspace(-30, 30, 601)[:, None]
    d = oracle.decay_direct(r, Lam)
    l = oracle.decay_log_space(r, Lam)
    assert np.max(np.abs(d - l) / np.maximum(d, 1e-300)) <= 1e-12


def test_O5_brute_force_unrolled_sum():
    """h_T = (Π_t a_t) h0 + Σ_k (Π_{t>k} a_t) √(1−a_k²) i_k u_k, enumerated term by term."""
    rng = np.random.default_rng(5)
    for T in range(1, 9):
        B, R = 2, 3
        p = _rng_params(rng, R, lam_lo=-1.0, lam_hi=6.0, wscale=1.0)
        x = rng.normal(size=(B, T, R))
        h0 = rng.normal(size=(B, R))
        y, h_T, _ = oracle.rglru_forward(x, h0=h0, **p)
        for b, c in itertools.product(range(B), range(R)):
            # independent scalar recomputation of the inputs of the sum
            us, ats, ms, iis = [], [], [], []
            for t in range(T):
                u = p["conv_b"][c]
                for k in range(4):
                    s = t - 3 + k
                    if s >= 0:
                        u += p["conv_w"][k][c] * x[b, s, c]
                us.append(u)
            for t in range(T):
                za = p["b_a"][c] + sum(p["W_a"][c][j] * us_j for j, us_j in
                                       enumerate([_u_at(x, p, b, t, jj) for jj in range(R)]))
                zx = p["b_x"][c] + sum(p["W_x"][c][j] * _u_at(x, p, b, t, j) for j in range(R))
                r = 1.0 / (1.0 + math.exp(-za))
                a = 1.0 / (1.0 + math.exp(-p["Lambda"][c]))
                at = math.exp(8.0 * r * math.log(a))
                ats.append(at)
                ms.append(math.sqrt(1.0 - at * at))
                iis.append(1.0 / (1.0 + math.exp(-zx)))
            want = math.prod(ats) * h0[b, c]
            for k in range(T):
                want += math.prod(ats[k + 1:]) * ms[k] * iis[k] * us[k]
            assert abs(h_T[b, c] - want) <= 1e-13 * max(1.0, abs(want)), (T, b, c)


def _u_at(x, p, b, t, c):
    u = p["conv_b"][c]
    for k in range(4):
        s = t - 3 + k
        if s >= 0:
            u += p["conv_w"][k][c] * x[b, s, c]
    return u


def test_O6_conv_matches_torch_conv1d():
    rng = np.random.default_rng(6)
    B, T, R = 3, 37, 16
    x = rng.normal(size=(B, T, R))
    w = rng.normal(size=(4, R))
    bias = rng.normal(size=R)
    u, state = oracle.conv1d_causal(x, w, bias)
    xt = torch.from_numpy(x).permute(0, 2, 1)                  # [B][R][T]
    wt = torch.from_numpy(w).T.reshape(R, 1, 4)                # weight[c][0][k]
    ref = torch.nn.functional.conv1d(xt, wt, torch.from_numpy(bias), padding=3, groups=R)
    ref = ref[..., :T].permute(0, 2, 1).numpy()
    np.testing.assert_allclose(u, ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(state, x[:, T - 3:, :])
    # with a history: equals the conv of the concatenated sequence
    hist = rng.normal(size=(B, 3, R))
    u2, _ = oracle.conv1d_causal(x, w, bias, hist)
    full, _ = oracle.conv1d_causal(np.concatenate([hist, x], axis=1), w, bias)
    np.testing.assert_allclose(u2, full[:, 3:, :], rtol=1e-13, atol=1e-13)


def test_O7_gate_preactivations_match_torch_matmul():
    rng = np.random.default_rng(7)
    B, T, R = 2, 9, 24
    u = rng.normal(size=(B, T, R))
    Wa, Wx = rng.normal(size=(R, R)), rng.normal(size=(R, R))
    ba, bx = rng.normal(size=R), rng.normal(size=R)
    za, zx = oracle.gate_preactivations(u, Wa, ba, Wx, bx)
    ut = torch.from_numpy(u)
    np.testing.assert_allclose(za, (torch.matmul(ut, torch.from_numpy(Wa).T) + torch.from_numpy(ba)).numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(zx, (torch.matmul(ut, torch.from_numpy(Wx).T) + torch.from_numpy(bx)).numpy(), rtol=1e-12, atol=1e-12)
    ch = np.array([5, 0, 23])
    za2, zx2 = oracle.gate_preactivations(u, Wa, ba, Wx, bx, channels=ch)
    np.testing.assert_array_equal(za2, za[..., ch])
    np.testing.assert_array_equal(zx2, zx[..., ch])


def test_O8_superposition_in_h0():
    """y(h0) − y(0) = (Π_{s≤t} a_s) h0: the recurrence is linear in h."""
    rng = np.random.default_rng(8)
    B, T, R = 2, 40, 6
    p = _rng_params(rng, R)
    x = rng.normal(size=(B, T, R))
    h0 = rng.normal(size=(B, R))
    y1, _, _ = oracle.rglru_forward(x, h0=h0, **p)
    y0, _, _ = oracle.rglru_forward(x, h0=None, **p)
    u, _ = oracle.conv1d_causal(x, p["conv_w"], p["conv_b"])
    za, _ = oracle.gate_preactivations(u, p["W_a"], p["b_a"], p["W_x"], p["b_x"])
    at = expit(p["Lambda"]) ** (8.0 * expit(za))
    np.testing.assert_allclose(y1 - y0, np.cumprod(at, axis=1) * h0[:, None, :], rtol=1e-11, atol=1e-14)


def test_O9_step_equals_forward_and_split_equals_whole():
    rng = np.random.default_rng(9)
    B, T, R = 3, 13, 8
    p = _rng_params(rng, R)
    x = rng.normal(size=(B, T, R))
    h0 = rng.normal(size=(B, R))
    y, h_T, st_T = oracle.rglru_forward(x, h0=h0, **p)
    # T decode steps from a zero ring equal the forward pass
    ring, h = np.zeros((B, 3, R)), h0.copy()
    for t in range(T):
        yt, h, ring = oracle.rglru_step(x[:, t, :], ring, t, h, **p)
        np.testing.assert_allclose(yt, y[:, t, :], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h, h_T, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(oracle.ring_to_time_order(ring, T), st_T)
    # forward(0:T1) then forward(T1:T) from the carried (h, conv state) equals forward(0:T)
    for T1 in (1, 5, 12):
        ya, ha, sa = oracle.rglru_forward(x[:, :T1], h0=h0, **p)
        yb, hb, sb = oracle.rglru_forward(x[:, T1:], h0=ha, conv_state0=sa, **p)
        np.testing.assert_allclose(np.concatenate([ya, yb], 1), y, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(hb, h_T, rtol=1e-13, atol=1e-13)
        np.testing.assert_array_equal(sb, st_T)
    # a subset of rows gives the same rows
    yt_all, _, _ = oracle.rglru_step(x[:, 0, :], np.zeros((B, 3, R)), 0, h0, **p)
    yt_sub, _, _ = oracle.rglru_step(x[:, 0, :], np.zeros((B, 3, R)), 0, h0, rows=[2, 0], **p)
    np.testing.assert_array_equal(yt_sub, yt_all[[2, 0]])
    # a subset of channels gives the same channels
    ch = [7, 1]
    ys, hs, _ = oracle.rglru_forward(x, h0=h0, channels=ch, **p)
    np.testing.assert_allclose(ys, y[..., ch], rtol=1e-14, atol=1e-15)


def test_O10_parameter_ranges_of_the_init():
    """a^8 ~ U[0.9, 0.999] ⇒ a ∈ [0.98692, 0.999875]; r ∈ (0, 1) ⇒ a_t ∈ [0.9, 1]."""
    w = inputs.make_forward(1, 64, 256, torch.float32, seed=0)
    a = expit(w.params.Lambda.double().numpy())
    assert a.min() >= 0.9 ** (1 / 8) - 1e-7 and a.max() <= 0.999 ** (1 / 8) + 1e-7
    assert 0.98692 <= a.min() and a.max() <= 0.999875
    y, h_T, _ = oracle.rglru_forward(w.x, w.params.conv_w, w.params.conv_b, w.params.W_a,
                                     w.params.b_a, w.params.W_x, w.params.b_x, w.params.Lambda)
    assert np.isfinite(y).all()
    u, _ = oracle.conv1d_causal(w.x, w.params.conv_w, w.params.conv_b)
    za, _ = oracle.gate_preactivations(u, w.params.W_a, w.params.b_a, w.params.W_x, w.params.b_x)
    at = oracle.decay_direct(oracle.sigmoid(za), w.params.Lambda)
    assert at.min() >= 0.9 - 1e-12 and at.max() <= 1.0


def test_gelu_exact_matches_torch_and_identity():
    x = np.linspace(-12, 12, 2401)
    g = oracle.gelu(x)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    np.testing.assert_allclose(g, ref, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(g - oracle.gelu(-x), x, rtol=1e-14, atol=1e-14)   # xΦ(x)+xΦ(−x) = x


def test_block_zero_gate_branch_and_constant_input_branch():
    """Recurrent block: W_2 = 0 ⇒ GeLU(0) = 0 ⇒ out ≡ 0; W_1 = 0 with W_a = W_x = 0 ⇒
    u ≡ conv bias, so h follows the geometric closed form and out = (h ⊙ GeLU(g)) W_oᵀ."""
    rng = np.random.default_rng(11)
    B, T, D, R = 2, 20, 6, 4
    x = rng.normal(size=(B, T, D))
    W1, W2, Wo = rng.normal(size=(R, D)), rng.normal(size=(R, D)), rng.normal(size=(D, R))
    p = _rng_params(rng, R)
    out, _ = oracle.recurrent_block(x, W1, np.zeros((R, D)), Wo, **p)
    assert np.array_equal(out, np.zeros_like(out))
    p["W_a"] = np.zeros((R, R))
    p["W_x"] = np.zeros((R, R))
    out, h_T = oracle.recurrent_block(x, np.zeros((R, D)), W2, Wo, **p)
    alpha = expit(p["Lambda"]) ** (8.0 * expit(p["b_a"]))
    m, i, kappa = np.sqrt(1 - alpha ** 2), expit(p["b_x"]), p["conv_b"]
    t = np.arange(1, T + 1)[:, None]
    h = m * i * kappa * (1 - alpha ** t) / (1 - alpha)                  # [T][R]
    g = torch.from_numpy(x @ W2.T)
    gel = torch.nn.functional.gelu(g, approximate="none").numpy()
    want = (h[None] * gel) @ Wo.T
    np.testing.assert_allclose(out, want, rtol=1e-11, atol=1e-12)


def test_max_rel_error_definition():
    ref = np.array([1.0, -2.0, 0.0, 4.0])
    rms = math.sqrt((1 + 4 + 0 + 16) / 4)
    got = ref + np.array([0.0, 0.0, 0.1, 0.0])
    assert abs(oracle.max_rel_error(got, ref) - 0.1 / rms) < 1e-15
    got = ref + np.array([0.0, 0.0, 0.0, 0.4])
    assert abs(oracle.max_rel_error(got, ref) - 0.1) < 1e-15


def test_planted_mistakes_are_caught():
    """Plant plausible mistakes in the oracle's arithmetic (on the CPU) and check that
    the pins above would reject each one."""
    ex = _parse_golden(GOLDEN)["taps_and_state"]
    x = ex["x"].reshape(1, -1, 1)

    def run(conv_w):
        y, _, _ = oracle.rglru_forward(x, conv_w.reshape(4, 1), ex["conv_b"], np.zeros((1, 1)),
                                       ex["b_a"], np.zeros((1, 1)), ex["b_x"], ex["Lambda"],
                                       h0=ex["h0"].reshape(1, 1))
        return y.ravel()

    assert np.allclose(run(ex["conv_w"]), ex["y"], rtol=1e-15)
    assert not np.allclose(run(ex["conv_w"][::-1].copy()), ex["y"], rtol=1e-6)   # reversed taps
    # wrong normalisation (1 − a_t instead of 1 − a_t²) changes the hand-worked values
    at, i, h0 = 9 / 16, 0.75, 1.0
    h = h0
    for u in ex["u"]:
        h = at * h + math.sqrt(1 - at) * i * u
    assert abs(h - ex["y"][-1]) > 1e-3


def _bwd_problem(seed, lam_lo, lam_hi, B=2, T=6, R=3):
    rng = np.random.default_rng(seed)
    P = {
        "x": rng.normal(size=(B, T, R)),
        "conv_w": rng.normal(size=(4, R)) * 0.5,
        "conv_b": rng.normal(size=R) * 0.5,
        "W_a": rng.normal(size=(R, R)) / math.sqrt(R),
        "b_a": rng.normal(size=R) * 0.5,
        "W_x": rng.normal(size=(R, R)) / math.sqrt(R),
        "b_x": rng.normal(size=R) * 0.5,
        "Lambda": rng.uniform(lam_lo, lam_hi, size=R),
        "h0": rng.normal(size=(B, R)),
        "conv_state0": rng.normal(size=(B, 3, R)),
    }
    dy = rng.normal(size=(B, T, R))
    dh_T = rng.normal(size=(B, R))
    return P, dy, dh_T


def _loss(P, dy, dh_T):
    y, h_T, _ = oracle.rglru_forward(P["x"], P["conv_w"], P["conv_b"], P["W_a"], P["b_a"], P["W_x"], P["b_x"],
                                     P["Lambda"], h0=P["h0"], conv_state0=P["conv_state0"])
    return float(np.sum(dy * y) + np.sum(dh_T * h_T))


@pytest.mark.parametrize("seed,lam_lo,lam_hi", [(3, 1.0, 4.0), (4, 4.33, 8.99)])
def test_backward_matches_central_differences(seed, lam_lo, lam_hi):
    """The oracle's backward against central differences of the forward oracle — an
    independent derivative of the definition — for every input: x, the taps and bias, W_a,
    b_a, W_x, b_x, Λ (also in the configs' range, where a_t is close to 1 and √(1 − a_t²)
    is small), h0 and the conv history. A dropped term, a wrong sign or a transposed
    operand in the backward shows up here."""
    P, dy, dh_T = _bwd_problem(seed, lam_lo, lam_hi)
    G = oracle.rglru_backward(P["x"], P["conv_w"], P["conv_b"], P["W_a"], P["b_a"], P["W_x"], P["b_x"],
                              P["Lambda"], dy, h0=P["h0"], conv_state0=P["conv_state0"], dh_T=dh_T)
    names = {"x": "dx", "conv_w": "dconv_w", "conv_b": "dconv_b", "W_a": "dW_a", "b_a": "db_a", "W_x": "dW_x",
             "b_x": "db_x", "Lambda": "dLambda", "h0": "dh0", "conv_state0": "dconv_state0"}
    eps = 1e-6
    for name, gname in names.items():
        g = G[gname]
        assert g.shape == P[name].shape, name
        fd = np.empty_like(P[name])
        for idx in np.ndindex(P[name].shape):
            orig = P[name][idx]
            P[name][idx] = orig + eps
            lp = _loss(P, dy, dh_T)
            P[name][idx] = orig - eps
            lm = _loss(P, dy, dh_T)
            P[name][idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        scale = max(float(np.max(np.abs(fd))), 1e-3)
        assert np.max(np.abs(g - fd)) <= 1e-6 * scale, (name, np.max(np.abs(g - fd)), scale)


def test_backward_of_a_frozen_state_is_plain_accumulation():
    """With r ≡ 0 (W_a = 0, b_a = −1000: a_t = 1 and √(1 − a_t²) = 0 exactly) the state
    never changes, h_t = h0, so ∂ℓ/∂h0 = Σ_t dy_t + dh_T and no gradient reaches x, the
    taps or the input gate."""
    B, T, R = 2, 5, 3
    P, dy, dh_T = _bwd_problem(5, 1.0, 4.0, B, T, R)
    P["W_a"][:] = 0.0
    P["b_a"][:] = -1000.0
    G = oracle.rglru_backward(P["x"], P["conv_w"], P["conv_b"], P["W_a"], P["b_a"], P["W_x"], P["b_x"],
                              P["Lambda"], dy, h0=P["h0"], conv_state0=P["conv_state0"], dh_T=dh_T)
    assert np.allclose(G["dh0"], dy.sum(axis=1) + dh_T, rtol=1e-13, atol=1e-13)
    for k in ("dx", "dconv_w", "dconv_b", "dW_x", "db_x", "dLambda"):
        assert np.all(G[k] == 0.0), k


def test_backward_pins_reject_planted_mistakes():
    """Plausible slips in a backward — the derivative of log σ(Λ) taken as σ(Λ) instead of
    σ(−Λ), a weight gradient transposed, ∂h0 missing the first step's decay a_0 — are each
    rejected by the central-difference comparison used above."""
    P, dy, dh_T = _bwd_problem(9, 1.0, 4.0)
    G = oracle.rglru_backward(P["x"], P["conv_w"], P["conv_b"], P["W_a"], P["b_a"], P["W_x"], P["b_x"],
                              P["Lambda"], dy, h0=P["h0"], conv_state0=P["conv_state0"], dh_T=dh_T)

    def fd(name):
        out = np.empty_like(P[name])
        for idx in np.ndindex(P[name].shape):
            orig = P[name][idx]
            P[name][idx] = orig + 1e-6
            lp = _loss(P, dy, dh_T)
            P[name][idx] = orig - 1e-6
            lm = _loss(P, dy, dh_T)
            P[name][idx] = orig
            out[idx] = (lp - lm) / 2e-6
        return out

    def agrees(g, ref):
        return np.max(np.abs(g - ref)) <= 1e-6 * max(float(np.max(np.abs(ref))), 1e-3)

    ref_L, ref_Wa = fd("Lambda"), fd("W_a")
    assert agrees(G["dLambda"], ref_L) and agrees(G["dW_a"], ref_Wa)
    s_pos = 1.0 / (1.0 + np.exp(-P["Lambda"]))
    assert not agrees(G["dLambda"] / (1.0 - s_pos) * s_pos, ref_L)          # σ(Λ) for σ(−Λ)
    assert not agrees(G["dW_a"].T, ref_Wa)                                   # transposed ∂W
    # ∂h0 taken as g_0 (the gradient at h_0) without the last step's decay a_0
    u, _ = oracle.conv1d_causal(P["x"], P["conv_w"], P["conv_b"], P["conv_state0"])
    z_a, _ = oracle.gate_preactivations(u[:, 0], P["W_a"], P["b_a"], P["W_x"], P["b_x"])
    a0 = oracle.decay_direct(oracle.sigmoid(z_a), P["Lambda"])
    ref_h0 = fd("h0")
    assert agrees(G["dh0"], ref_h0)
    assert not agrees(G["dh0"] / a0, ref_h0)


# ------------------------------------------------------------------------------------
# Hawk residual layer: RMSNorm, gated MLP and their wiring around the recurrent block
# ("Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §残块, Fig. 2(a);
# §MLP块, Fig. 2(b)).
def test_rms_norm_worked_example_and_invariants():
    # x = (3, 4): mean square 12.5; gain (1, 2)
    n = oracle.rms_norm(np.array([3.0, 4.0]), np.array([1.0, 2.0]), eps=0.0)
    np.testing.assert_allclose(n, [3 / math.sqrt(12.5), 8 / math.sqrt(12.5)], rtol=1e-15)
    # ε enters under the root: x = (1, 1, 1, 1), ε = 3 ⇒ 1/√(1 + 3) = 1/2
    np.testing.assert_allclose(oracle.rms_norm(np.ones(4), np.ones(4), eps=3.0), 0.5 * np.ones(4), rtol=1e-15)
    # an all-zero row stays zero (ε keeps the root away from zero)
    assert np.array_equal(oracle.rms_norm(np.zeros((2, 8)), np.ones(8)), np.zeros((2, 8)))
    rng = np.random.default_rng(11)
    x = rng.normal(0, 3, (5, 7, 64))
    ones = np.ones(64)
    n = oracle.rms_norm(x, ones, eps=0.0)
    # unit gain, ε = 0: every row has mean square exactly 1 (up to rounding)
    np.testing.assert_allclose(np.mean(n * n, axis=-1), 1.0, rtol=1e-13)
    # scale invariance per row, odd symmetry, and the gain multiplies channel by channel
    c = rng.uniform(0.1, 10, (5, 7, 1))
    np.testing.assert_allclose(oracle.rms_norm(c * x, ones, eps=0.0), n, rtol=1e-12)
    np.testing.assert_allclose(oracle.rms_norm(-x, ones, eps=0.0), -n, rtol=1e-15)
    gam = rng.uniform(0.5, 1.5, 64)
    np.testing.assert_allclose(oracle.rms_norm(x, gam, eps=0.0), n * gam, rtol=1e-15)


def test_gated_mlp_worked_example_and_branch_roles():
    Phi1, Phi2 = 0.8413447460685429, 0.9772498680518208  # standard normal table: Φ(1), Φ(2)
    I2 = np.eye(2)
    # identity gate and down projections, up = 2·I: out_j = GeLU(x_j) · 2 x_j
    out = oracle.gated_mlp(np.array([1.0, -1.0]), I2, 2 * I2, I2)
    np.testing.assert_allclose(out, [2 * Phi1, 2 * (1 - Phi1)], rtol=1e-15)
    # GeLU sits on the gate branch only: swapping the two branches gives GeLU(2)·1 = 2Φ(2)
    swapped = oracle.gated_mlp(np.array([1.0, -1.0]), 2 * I2, I2, I2)
    np.testing.assert_allclose(swapped[0], 2 * Phi2, rtol=1e-15)
    # a zero gate projection zeroes the block (GeLU(0) = 0)
    rng = np.random.default_rng(12)
    x = rng.normal(0, 1, (3, 16))
    Wu, Wd = rng.normal(0, 0.25, (48, 16)), rng.normal(0, 0.15, (16, 48))
    assert np.array_equal(oracle.gated_mlp(x, np.zeros((48, 16)), Wu, Wd), np.zeros((3, 16)))
    # library cross-check: torch's exact GeLU and matmuls in float64
    Wg = rng.normal(0, 0.25, (48, 16))
    xt = torch.from_numpy(x)
    ref = (torch.nn.functional.gelu(xt @ torch.from_numpy(Wg).T) * (xt @ torch.from_numpy(Wu).T)) \
        @ torch.from_numpy(Wd).T
    np.testing.assert_allclose(oracle.gated_mlp(x, Wg, Wu, Wd), ref.numpy(), rtol=1e-12, atol=1e-14)


def test_hawk_layer_worked_example():
    ex = _parse_golden(GOLDEN)["hawk_layer"]
    m = lambda k: ex[k].reshape(1, 1)  # noqa: E731
    out, h_T = oracle.hawk_residual_layer(
        ex["x"].reshape(1, 1, 1), ex["norm1_scale"], m("W_1"), m("W_2"), m("W_o"), ex["norm2_scale"],
        m("W_gate"), m("W_up"), m("W_down"), ex["conv_w"].reshape(4, 1), ex["conv_b"], np.zeros((1, 1)),
        np.zeros(1), np.zeros((1, 1)), np.zeros(1), ex["Lambda"], eps=0.0)
    np.testing.assert_allclose(h_T.ravel(), ex["h_T"], rtol=1e-14)
    np.testing.assert_allclose(out.ravel(), ex["out"], rtol=1e-14)
    # the residual stream between the two components, through the zero-MLP special case
    y, _ = oracle.hawk_residual_layer(
        ex["x"].reshape(1, 1, 1), ex["norm1_scale"], m("W_1"), m("W_2"), m("W_o"), ex["norm2_scale"],
        m("W_gate"), m("W_up"), np.zeros((1, 1)), ex["conv_w"].reshape(4, 1), ex["conv_b"], np.zeros((1, 1)),
        np.zeros(1), np.zeros((1, 1)), np.zeros(1), ex["Lambda"], eps=0.0)
    np.testing.assert_allclose(y.ravel(), ex["y"], rtol=1e-14)


def test_hawk_layer_zero_branches_and_block_special_case():
    rng = np.random.default_rng(13)
    B, T, D, R = 2, 9, 16, 24
    P = _rng_params(rng, R)
    x = rng.normal(0, 1, (B, T, D))
    W_1, W_2 = rng.normal(0, 0.25, (R, D)), rng.normal(0, 0.25, (R, D))
    W_o = rng.normal(0, 0.2, (D, R))
    Wg, Wu, Wd = rng.normal(0, 0.25, (3 * D, D)), rng.normal(0, 0.25, (3 * D, D)), rng.normal(0, 0.15, (D, 3 * D))
    g1, g2 = rng.uniform(0.5, 1.5, D), rng.uniform(0.5, 1.5, D)
    # both output projections zero: the layer is the identity on its input, bitwise
    out, _ = oracle.hawk_residual_layer(x, g1, W_1, W_2, np.zeros((D, R)), g2, Wg, Wu, np.zeros((D, 3 * D)), **P)
    assert np.array_equal(out, x)
    # zero MLP output projection: x plus the recurrent block of the normalised input
    out, h_T = oracle.hawk_residual_layer(x, g1, W_1, W_2, W_o, g2, Wg, Wu, np.zeros((D, 3 * D)), **P)
    n1 = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + oracle.RMS_EPS) * g1
    blk, h_blk = oracle.recurrent_block(n1, W_1, W_2, W_o, **P)
    np.testing.assert_allclose(out, x + blk, rtol=1e-13, atol=1e-13)
    assert np.array_equal(h_T, h_blk)
    # the layer is causal: changing the last step leaves every earlier output unchanged
    x2 = x.copy()
    x2[:, -1, :] += 1.0
    o1, _ = oracle.hawk_residual_layer(x, g1, W_1, W_2, W_o, g2, Wg, Wu, Wd, **P)
    o2, _ = oracle.hawk_residual_layer(x2, g1, W_1, W_2, W_o, g2, Wg, Wu, Wd, **P)
    assert np.array_equal(o1[:, :-1], o2[:, :-1]) and not np.allclose(o1[:, -1], o2[:, -1])


def test_hawk_layer_steps_equal_the_layer_forward():
    # T decode steps from a zero state (h = 0, empty conv ring) reproduce the full-sequence
    # layer at every position; the ring ends holding the last three inputs of the Conv1D
    rng = np.random.default_rng(14)
    B, T, D, R = 2, 7, 16, 24
    P = _rng_params(rng, R)
    x = rng.normal(0, 1, (B, T, D))
    W = dict(norm1_scale=rng.uniform(0.5, 1.5, D), W_1=rng.normal(0, 0.25, (R, D)), W_2=rng.normal(0, 0.25, (R, D)),
             W_o=rng.normal(0, 0.2, (D, R)), norm2_scale=rng.uniform(0.5, 1.5, D),
             W_gate=rng.normal(0, 0.25, (3 * D, D)), W_up=rng.normal(0, 0.25, (3 * D, D)),
             W_down=rng.normal(0, 0.15, (D, 3 * D)))
    ref, h_ref = oracle.hawk_residual_layer(x, **W, **P)
    ring, h = np.zeros((B, 3, R)), np.zeros((B, R))
    for t in range(T):
        out_t, h, ring = oracle.hawk_residual_layer_step(x[:, t], ring, t, h, **W, **P)
        np.testing.assert_allclose(out_t, ref[:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h, h_ref, rtol=1e-12, atol=1e-14)
    n1 = oracle.rms_norm(x, W["norm1_scale"])
    v = n1 @ W["W_1"].T
    np.testing.assert_allclose(oracle.ring_to_time_order(ring, T), v[:, -3:], rtol=1e-14)


def test_hawk_layer_example_rejects_planted_wiring_mistakes():
    # Each plausible slip in wiring the residual layer, built from the oracle's own parts,
    # misses the hand-worked value by far more than rounding.
    ex = _parse_golden(GOLDEN)["hawk_layer"]
    m = lambda k: ex[k].reshape(1, 1)  # noqa: E731
    x = ex["x"].reshape(1, 1, 1)
    P = dict(conv_w=ex["conv_w"].reshape(4, 1), conv_b=ex["conv_b"], W_a=np.zeros((1, 1)), b_a=np.zeros(1),
             W_x=np.zeros((1, 1)), b_x=np.zeros(1), Lambda=ex["Lambda"])
    norm = lambda v, g: oracle.rms_norm(v, g, eps=0.0)  # noqa: E731
    block = lambda n: oracle.recurrent_block(n, m("W_1"), m("W_2"), m("W_o"), **P)[0]  # noqa: E731
    mlp = lambda n: oracle.gated_mlp(n, m("W_gate"), m("W_up"), m("W_down"))  # noqa: E731
    g1, g2 = ex["norm1_scale"], ex["norm2_scale"]
    right = x + block(norm(x, g1))
    right = right + mlp(norm(right, g2))
    np.testing.assert_allclose(right.ravel(), ex["out"], rtol=1e-14)
    planted = {
        "skip from the norm output": (lambda n1: (lambda y: y + mlp(norm(y, g2)))(n1 + block(n1)))(norm(x, g1)),
        "second norm applied to x": (lambda y: y + mlp(norm(x, g2)))(x + block(norm(x, g1))),
        "gains dropped": (lambda y: y + mlp(norm(y, 1.0)))(x + block(norm(x, 1.0))),
        "GeLU on the up branch": (lambda y: y + oracle.gated_mlp(norm(y, g2), m("W_up"), m("W_gate"), m("W_down")))(
            x + block(norm(x, g1))),
        "no second residual": mlp(norm(x + block(norm(x, g1)), g2)),
    }
    for name, out in planted.items():
        assert abs(out.ravel()[0] - ex["out"][0]) > 0.1, name
