"""Pins of the local-attention oracle (oracle/local_attention.py), CPU only.

Sources of truth other than the oracle itself:
  * the hand-worked example `local_attention` in tests/golden/hand_worked.txt (RoPE
    angles, the window's eviction of the oldest key, the 1/√d scale, values not rotated);
  * torch's scaled_dot_product_attention in float64 with a causal mask (the window does
    not bind when T ≤ W) and with an explicit band mask (T > W): library special cases;
  * closed forms: q = 0 gives uniform weights, so each output is the mean of the values
    in its window; RoPE preserves norms and makes q·k depend only on the position
    difference;
  * the ring decode, step after step across several wraps of the ring, equals the
    whole-sequence form;
  * planted mistakes (window one too wide, scale 1/d, RoPE on the values, the pairs rotated
    the wrong way) are each rejected by one of the pins above.
"""
import importlib
import math

import numpy as np
import pytest
import torch

import oracle
la = importlib.import_module("oracle.local_attention")  # the module (the package re-exports a function of that name)

from test_oracle_pins import GOLDEN, _parse_golden


def _sdpa(q, k, v, mask):
    """torch's attention in float64: q [B][T][H][d], k, v [B][T][d] shared by the heads."""
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                      # [B][H][T][d]
    kt = torch.from_numpy(k)[:, None].expand(-1, q.shape[2], -1, -1)
    vt = torch.from_numpy(v)[:, None].expand(-1, q.shape[2], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask))
    return o.permute(0, 2, 1, 3).numpy()


def _band(T, W):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return (j <= i) & (j > i - W)


def _qkv(rng, B, T, H, d):
    return rng.normal(size=(B, T, H, d)), rng.normal(size=(B, T, d)), rng.normal(size=(B, T, d))


def _golden_case(window_fn=None, **kw):
    ex = _parse_golden(GOLDEN)["local_attention"]
    x = ex["x"].reshape(1, -1, 2)
    I2 = np.eye(2)
    fn = window_fn or oracle.local_attention
    return fn(x, I2, I2, I2, I2, int(ex["window"][0]), **kw), ex["out"].reshape(1, -1, 2)


def test_hand_worked_local_attention():
    got, want = _golden_case()
    assert np.allclose(got, want, rtol=0, atol=1e-15)


def test_matches_causal_sdpa_when_the_window_does_not_bind():
    rng = np.random.default_rng(1)
    q, k, v = _qkv(rng, 2, 9, 3, 8)
    o = oracle.local_mqa(q, k, v, window=9)
    assert np.allclose(o, _sdpa(q, k, v, _band(9, 9)), rtol=0, atol=1e-13)
    o1024 = oracle.local_mqa(q, k, v, window=1024)
    assert np.array_equal(o, o1024)


@pytest.mark.parametrize("T,W", [(13, 5), (20, 1), (17, 16)])
def test_matches_band_masked_sdpa(T, W):
    rng = np.random.default_rng(T + W)
    q, k, v = _qkv(rng, 2, T, 4, 8)
    assert np.allclose(oracle.local_mqa(q, k, v, W), _sdpa(q, k, v, _band(T, W)), rtol=0, atol=1e-13)


def test_zero_query_averages_the_window():
    rng = np.random.default_rng(3)
    B, T, H, d, W = 2, 11, 2, 4, 4
    _, k, v = _qkv(rng, B, T, H, d)
    o = oracle.local_mqa(np.zeros((B, T, H, d)), k, v, W)
    for t in range(T):
        mean = v[:, max(0, t - W + 1):t + 1].mean(axis=1)
        for h in range(H):
            assert np.allclose(o[:, t, h], mean, rtol=0, atol=1e-14)


def test_rope_rotation_and_relative_positions():
    rng = np.random.default_rng(4)
    d = 16
    x = rng.normal(size=(5, d))
    r = oracle.rope(x, np.arange(5) * 7)
    assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-14)
    # d = 2, θ_0 = 1: (1, 0) at position p turns to (cos p, sin p)
    e = oracle.rope(np.array([[1.0, 0.0]] * 3), np.array([0, 1, 2]))
    assert np.allclose(e, [[1, 0], [math.cos(1), math.sin(1)], [math.cos(2), math.sin(2)]], atol=1e-15)
    # pair i turns with θ_i = 10000^(-2i/d): the last pair of d = 16 at position 1
    last = oracle.rope(np.eye(d)[None, d - 2], np.array([1]))[0]
    th = 10000.0 ** (-(d - 2) / d)
    assert np.allclose(last[d - 2:], [math.cos(th), math.sin(th)], atol=1e-15)
    # the rotated product depends only on n − m
    q, k = rng.normal(size=(1, d)), rng.normal(size=(1, d))
    dots = [float(oracle.rope(q, np.array([m])) @ oracle.rope(k, np.array([m + 5])).T) for m in (0, 3, 40, 999)]
    assert np.allclose(dots, dots[0], rtol=1e-12)


@pytest.mark.parametrize("T,W", [(11, 4), (9, 9), (10, 3), (7, 1)])
def test_ring_decode_equals_the_sequence_form(T, W):
    rng = np.random.default_rng(T * W)
    B, D, H, d = 2, 12, 3, 4
    Wq, Wk, Wv = rng.normal(size=(H * d, D)), rng.normal(size=(d, D)), rng.normal(size=(d, D))
    Wo = rng.normal(size=(D, H * d))
    x = rng.normal(size=(B, T, D))
    full = oracle.local_attention(x, Wq, Wk, Wv, Wo, W)
    K, V = np.full((B, W, d), np.nan), np.full((B, W, d), np.nan)    # unwritten slots must never be read
    for t in range(T):
        out, K, V = oracle.local_attention_step(x[:, t], K, V, t, Wq, Wk, Wv, Wo, W)
        assert np.allclose(out, full[:, t], rtol=0, atol=1e-12), t
    # the ring holds the last min(T, W) positions' rotated keys and values, slot p mod W
    k_all = oracle.rope(x @ Wk.T, np.arange(T))
    for p in range(max(0, T - W), T):
        assert np.allclose(K[:, p % W], k_all[:, p], atol=1e-13)


def test_griffin_layer_step_equals_the_layer():
    rng = np.random.default_rng(9)
    B, T, D, H, d, W, M = 2, 7, 8, 2, 4, 3, 3
    ws = dict(norm1_scale=rng.uniform(0.5, 1.5, D), W_q=rng.normal(size=(H * d, D)) / 3,
              W_k=rng.normal(size=(d, D)) / 3, W_v=rng.normal(size=(d, D)) / 3, W_o=rng.normal(size=(D, H * d)) / 3,
              norm2_scale=rng.uniform(0.5, 1.5, D), W_gate=rng.normal(size=(M * D, D)) / 3,
              W_up=rng.normal(size=(M * D, D)) / 3, W_down=rng.normal(size=(D, M * D)) / 5)
    x = rng.normal(size=(B, T, D))
    full = oracle.griffin_attention_layer(x, window=W, **ws)
    K, V = np.zeros((B, W, d)), np.zeros((B, W, d))
    for t in range(T):
        out, K, V = oracle.griffin_attention_layer_step(x[:, t], K, V, t, window=W, **ws)
        assert np.allclose(out, full[:, t], atol=1e-12)
    # zero projections on both components leave the residual stream untouched
    z = dict(ws, W_o=np.zeros_like(ws["W_o"]), W_down=np.zeros_like(ws["W_down"]))
    assert np.array_equal(oracle.griffin_attention_layer(x, window=W, **z), x)


# ---- planted mistakes: each variant must fail one of the pins above ---------------------
def _mqa_wide(q, k, v, window):
    return oracle.local_mqa(q, k, v, window + 1)


def _mqa_scale_d(q, k, v, window):
    # scores scaled by 1/d instead of 1/√d: the same as queries shrunk by a further 1/√d
    return oracle.local_mqa(q / math.sqrt(q.shape[-1]), k, v, window)


def _attn_rope_on_v(x, W_q, W_k, W_v, W_o, window, pos0=0):
    T = x.shape[1]
    orig = la.local_mqa

    def mqa(q, k, v, w):
        return orig(q, k, oracle.rope(v, np.arange(pos0, pos0 + T)), w)
    la.local_mqa = mqa
    try:
        return la.local_attention(x, W_q, W_k, W_v, W_o, window, pos0)
    finally:
        la.local_mqa = orig


def _attn_rope_backwards(x, W_q, W_k, W_v, W_o, window, pos0=0):
    orig = la.rope
    la.rope = lambda y, p, base=oracle.ROPE_BASE: orig(y, -np.asarray(p), base)
    try:
        return la.local_attention(x, W_q, W_k, W_v, W_o, window, pos0)
    finally:
        la.rope = orig


@pytest.mark.parametrize("mistake", [_mqa_wide, _mqa_scale_d])
def test_planted_attention_mistakes_are_rejected(mistake):
    rng = np.random.default_rng(5)
    q, k, v = _qkv(rng, 2, 13, 4, 8)
    assert not np.allclose(mistake(q, k, v, 5), _sdpa(q, k, v, _band(13, 5)), atol=1e-6)


@pytest.mark.parametrize("mistake", [_attn_rope_on_v, _attn_rope_backwards])
def test_planted_rope_mistakes_are_rejected(mistake):
    got, want = _golden_case(window_fn=mistake)
    assert not np.allclose(got, want, atol=1e-6)
