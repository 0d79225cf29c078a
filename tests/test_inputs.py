"""The seeded input generators shared by the tests, the bench and the oracle checks: the same
seed gives the same values, and the shortcuts the large tests take draw the same numbers as
the full recipe."""
import torch

from gated_linear_rnn_conv1d_b200 import inputs


def test_attention_only_draw_equals_the_layer_recipe():
    full = inputs.make_attention(256, seed=12)
    att = inputs.make_attention(256, seed=12, layer=False)
    assert set(att) == {"W_q", "W_k", "W_v", "W_o"}
    assert all(torch.equal(att[k], full[k]) for k in att)


def test_generators_are_deterministic():
    a, b = inputs.make_forward(2, 64, 16, seed=3), inputs.make_forward(2, 64, 16, seed=3)
    assert torch.equal(a.x, b.x)
    assert torch.equal(inputs.decode_token(7, 4, 32), inputs.decode_token(7, 4, 32))
    assert not torch.equal(inputs.decode_token(7, 4, 32), inputs.decode_token(8, 4, 32))
