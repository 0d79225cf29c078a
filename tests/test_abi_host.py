"""Host-side checks of librglru.so that need no GPU: it loads, exports every function
include/rglru.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from gated_linear_rnn_conv1d_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rglru.h")


def _declared():
    text = open(HEADER, encoding="utf-8").read()
    return sorted(set(re.findall(r"RGLRU_API\s+[\w\s\*]+?\b(rglru_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = _abi.load()
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in _abi.SIGNATURES, f"binding lacks {n}"


def test_version_and_strerror():
    lib = _abi.load()
    assert lib.rglru_version() == 10000
    for code in range(-8, 1):
        assert lib.rglru_strerror(code)
    assert lib.rglru_strerror(-99) == b"unknown status"


def _fake(addr=0x100000):
    return ctypes.c_void_p(addr)


def _params(addr=0x100000):
    return _abi.RGLRUParams(*([addr] * 7))


def test_argument_errors_are_returned_before_any_launch():
    lib = _abi.load()
    p = _params()
    ws_bytes = lib.rglru_forward_workspace_bytes(1, 64, 256, 1)
    ok_ptr = _fake()
    ws = _fake(0x200000)
    args = lambda **kw: dict(dict(params=ctypes.byref(p), x=ok_ptr, h0=None, st0=None, y=ok_ptr, hT=None, stT=None,
                                  B=1, T=64, R=256, io=1, ws=ws, wsb=ws_bytes), **kw)

    def call(**kw):
        a = args(**kw)
        return lib.rglru_forward(a["params"], a["x"], a["h0"], a["st0"], a["y"], a["hT"], a["stT"], a["B"], a["T"],
                                 a["R"], a["io"], a["ws"], a["wsb"], None)

    assert call(io=7) == -4
    assert call(R=12) == -2
    assert call(R=0) == -2
    assert call(T=0) == -2
    assert call(B=0) == -2
    assert call(params=None) == -1
    assert call(x=None) == -1
    assert call(x=_fake(0x100004)) == -3
    assert call(ws=None) == -5
    assert call(wsb=ws_bytes - 1) == -5
    assert call(ws=_fake(0x200010)) == -3
    bad = _abi.RGLRUParams(0x100000, 0x100000, 0, 0x100000, 0x100000, 0x100000, 0x100000)
    assert call(params=ctypes.byref(bad)) == -1
    # decode takes bf16 only and a non-negative step
    sb = lib.rglru_step_workspace_bytes(4, 256, 1)
    assert sb > 0 and lib.rglru_step_workspace_bytes(4, 256, 0) == 0
    assert lib.rglru_step(ctypes.byref(p), ok_ptr, ok_ptr, ok_ptr, ok_ptr, 4, 256, 0, 0, ws, sb, None) == -4
    assert lib.rglru_step(ctypes.byref(p), ok_ptr, ok_ptr, ok_ptr, ok_ptr, 4, 256, -1, 1, ws, sb, None) == -2
    assert lib.rglru_step(ctypes.byref(p), ok_ptr, None, ok_ptr, ok_ptr, 4, 256, 0, 1, ws, sb, None) == -1
    # GEMM and block
    assert lib.rglru_gemm_bf16(ok_ptr, ok_ptr, ok_ptr, 0, 64, 64, None) == -2
    assert lib.rglru_gemm_bf16(ok_ptr, ok_ptr, ok_ptr, 16, 60, 64, None) == -2
    assert lib.rglru_gemm_bf16(ok_ptr, None, ok_ptr, 16, 64, 64, None) == -1
    bb = lib.rglru_block_workspace_bytes(1, 8, 64, 64, 1)
    assert lib.rglru_block_forward(ctypes.byref(p), ok_ptr, ok_ptr, ok_ptr, ok_ptr, None, ok_ptr, None, 1, 8, 64, 64,
                                   0, ws, bb, None) == -4
    assert lib.rglru_block_forward(ctypes.byref(p), ok_ptr, ok_ptr, ok_ptr, ok_ptr, None, ok_ptr, None, 1, 8, 60, 64,
                                   1, ws, bb, None) == -2


def test_coefficient_stages_reject_bad_arguments_before_any_launch():
    lib = _abi.load()
    p = _params()
    ok_ptr = _fake()
    assert lib.rglru_gate_coeffs(ctypes.byref(p), ok_ptr, ok_ptr, 0, 256, None) == -2
    assert lib.rglru_gate_coeffs(ctypes.byref(p), ok_ptr, ok_ptr, 64, 12, None) == -2
    assert lib.rglru_gate_coeffs(None, ok_ptr, ok_ptr, 64, 256, None) == -1
    assert lib.rglru_gate_coeffs(ctypes.byref(p), None, ok_ptr, 64, 256, None) == -1
    assert lib.rglru_gate_coeffs(ctypes.byref(p), _fake(0x100004), ok_ptr, 64, 256, None) == -3
    wsb = lib.rglru_scan_workspace_bytes(1, 64, 256, 1)
    ws = _fake(0x200000)
    call = lambda **kw: lib.rglru_scan_coeffs(kw.get("g", ok_ptr), kw.get("h0", None), None, kw.get("y", ok_ptr),
                                              None, 1, kw.get("T", 64), kw.get("R", 256), kw.get("ws", ws),
                                              kw.get("wsb", wsb), None)
    assert call(R=12) == -2
    assert call(T=0) == -2
    assert call(g=None) == -1
    assert call(y=_fake(0x100008)) == -3
    assert call(h0=_fake(0x100004)) == -3
    assert call(ws=None) == -5
    assert call(wsb=wsb - 1) == -5


def test_workspace_queries():
    lib = _abi.load()
    assert lib.rglru_forward_workspace_bytes(1, 1, 8, 1) > 0
    assert lib.rglru_forward_workspace_bytes(1, 1, 7, 1) == 0
    # the fused gate-GEMM + scan stage needs 12 B of chunk carries per channel and 128-step chunk
    assert lib.rglru_gate_scan_workspace_bytes(8, 2048, 2048, 1) == 256 + 8 * 16 * 16 * 128 * 12
    assert lib.rglru_gate_scan_workspace_bytes(8, 2000, 2048, 1) == 0
    # otherwise: u (2 B) + packed z (2·2 B per channel) per element, plus chunk carries
    c = lib.rglru_forward_workspace_bytes(8, 2000, 2048, 1)
    assert 8 * 2000 * 2048 * 6 <= c < 8 * 2000 * 2048 * 6 * 1.05
    b = lib.rglru_forward_workspace_bytes(8, 2048, 2048, 0)
    assert b > c
    assert lib.rglru_gate_pitch(256) == 512
    assert lib.rglru_gate_pitch(264) == 768      # partial last 128-channel block
    assert lib.rglru_gate_pitch(5632) == 11264
    assert lib.rglru_gate_pitch(12) == 0
    assert lib.rglru_scan_workspace_bytes(1, 64, 128, 1) > 256
    assert lib.rglru_block_workspace_bytes(4, 4096, 4096, 5632, 1) > 4 * 4096 * 5632 * 2 * 5


def test_backward_rejects_bad_arguments_before_any_launch():
    lib = _abi.load()
    p = _params()
    ok = _fake()
    assert lib.rglru_backward_workspace_bytes(2, 64, 256) > 0
    assert lib.rglru_backward_workspace_bytes(2, 64, 12) == 0
    grads = _abi.RGLRUGrads(*([0x100000] * 10))
    wsb = lib.rglru_backward_workspace_bytes(1, 64, 256)
    ws = _fake(0x200000)

    def call(**kw):
        g = kw.get("g", grads)
        return lib.rglru_backward(kw.get("p", ctypes.byref(p)), kw.get("x", ok), ok, ok, kw.get("h0", None), None,
                                  None, ctypes.byref(g) if g is not None else None, 1, kw.get("T", 64),
                                  kw.get("R", 256), kw.get("ws", ws), kw.get("wsb", wsb), None)
    assert call(R=12) == -2
    assert call(T=0) == -2
    assert call(p=None) == -1
    assert call(x=None) == -1
    assert call(g=None) == -1
    assert call(g=_abi.RGLRUGrads(*([0x100000] * 8 + [None, 0x100000]))) == -1   # dLambda missing
    assert call(g=_abi.RGLRUGrads(*([0x100000] + [0x100008] + [0x100000] * 8))) == -3  # dconv_state0 misaligned
    assert call(h0=_fake(0x100004)) == -3
    assert call(ws=None) == -5
    assert call(wsb=wsb - 1) == -5


def test_training_pair_rejects_bad_arguments_before_any_launch():
    """rglru_forward_train / rglru_backward_saved: a null or misaligned `saved` and the
    checks of the calls they extend, all before anything is launched."""
    lib = _abi.load()
    p = _params()
    ok = _fake()
    assert lib.rglru_saved_bytes(2, 64, 256) == 2 * 64 * lib.rglru_gate_pitch(256) * 2
    assert lib.rglru_saved_bytes(1, 64, 264) == 64 * 768 * 2
    assert lib.rglru_saved_bytes(2, 64, 12) == 0
    assert lib.rglru_saved_bytes(0, 64, 256) == 0
    fwb = lib.rglru_forward_workspace_bytes(1, 64, 256, 1)
    ws = _fake(0x200000)

    def fwd(**kw):
        return lib.rglru_forward_train(kw.get("p", ctypes.byref(p)), kw.get("x", ok), None, None, kw.get("y", ok),
                                       None, None, kw.get("saved", _fake(0x300000)), 1, kw.get("T", 64),
                                       kw.get("R", 256), kw.get("ws", ws), kw.get("wsb", fwb), None)
    assert fwd(saved=None) == -1
    assert fwd(saved=_fake(0x300008)) == -3
    assert fwd(R=12) == -2
    assert fwd(y=None) == -1
    assert fwd(wsb=fwb - 1) == -5
    grads = _abi.RGLRUGrads(*([0x100000] * 10))
    bwb = lib.rglru_backward_workspace_bytes(1, 64, 256)

    def bwd(**kw):
        return lib.rglru_backward_saved(ctypes.byref(p), kw.get("x", ok), ok, ok, None, None, None,
                                        kw.get("saved", _fake(0x300000)), ctypes.byref(grads), 1, 64,
                                        kw.get("R", 256), ws, kw.get("wsb", bwb), None)
    assert bwd(saved=None) == -1
    assert bwd(saved=_fake(0x300004)) == -3
    assert bwd(R=12) == -2
    assert bwd(x=None) == -1
    assert bwd(wsb=bwb - 1) == -5


def test_layer_rejects_bad_arguments_before_any_launch():
    lib = _abi.load()
    p = _params()
    ok_ptr = _fake()
    wb = lib.rglru_layer_workspace_bytes(1, 8, 64, 64, 192, 1)
    assert wb > lib.rglru_block_workspace_bytes(1, 8, 64, 64, 1)
    assert lib.rglru_layer_workspace_bytes(1, 8, 64, 64, 192, 0) == 0
    assert lib.rglru_layer_workspace_bytes(1, 8, 64, 64, 190, 1) == 0
    f = 0x100000
    weights = _abi.RGLRULayerWeights(f, f, f, f, f, f, f, f)
    ws = _fake(0x200000)

    def call(**kw):
        return lib.rglru_layer_forward(
            ctypes.byref(p), kw.get("w", ctypes.byref(weights)), kw.get("x", ok_ptr), None, kw.get("out", _fake(0x300000)),
            None, 1, 8, kw.get("D", 64), 64, kw.get("H", 192), kw.get("eps", 1e-6), kw.get("io", 1),
            kw.get("ws", ws), kw.get("wsb", wb), None)

    assert call(io=0) == -4
    assert call(D=60) == -2
    assert call(H=190) == -2
    assert call(eps=-1.0) == -2
    assert call(eps=float("nan")) == -2
    assert call(out=ok_ptr) == -2  # out must not be x
    assert call(w=None) == -1
    assert call(x=None) == -1
    missing = _abi.RGLRULayerWeights(f, f, f, f, f, f, 0, f)
    assert call(w=ctypes.byref(missing)) == -1
    odd = _abi.RGLRULayerWeights(f, f, f, f, f + 4, f, f, f)
    assert call(w=ctypes.byref(odd)) == -3
    assert call(ws=None) == -5
    assert call(wsb=wb - 1) == -5
    assert call(ws=_fake(0x200010)) == -3


def test_layer_step_rejects_bad_arguments_before_any_launch():
    lib = _abi.load()
    p = _params()
    ok_ptr = _fake()
    wb = lib.rglru_layer_step_workspace_bytes(4, 64, 64, 192, 1)
    assert wb > lib.rglru_step_workspace_bytes(4, 64, 1)
    assert lib.rglru_layer_step_workspace_bytes(4, 64, 64, 192, 0) == 0
    assert lib.rglru_layer_step_workspace_bytes(0, 64, 64, 192, 1) == 0
    f = 0x100000
    weights = _abi.RGLRULayerWeights(f, f, f, f, f, f, f, f)
    ws = _fake(0x200000)

    def call(**kw):
        return lib.rglru_layer_step(
            ctypes.byref(p), kw.get("w", ctypes.byref(weights)), kw.get("x", ok_ptr), kw.get("ring", ok_ptr),
            kw.get("h", ok_ptr), kw.get("out", _fake(0x300000)), 4, kw.get("D", 64), 64, kw.get("H", 192),
            kw.get("step", 0), kw.get("eps", 1e-6), kw.get("io", 1), kw.get("ws", ws), kw.get("wsb", wb), None)

    assert call(io=0) == -4
    assert call(D=12) == -2
    assert call(H=0) == -2
    assert call(step=-1) == -2
    assert call(eps=2.0) == -2
    assert call(out=ok_ptr) == -2
    assert call(ring=None) == -1
    assert call(h=None) == -1
    assert call(w=None) == -1
    assert call(h=_fake(0x100008)) == -3
    assert call(ws=None) == -5
    assert call(wsb=wb - 1) == -5


def test_layer_weights_marshal_every_field_in_header_order():
    import torch
    from gated_linear_rnn_conv1d_b200 import inputs, rglru
    w = inputs.make_layer(1, 4, 16, 24, 3, torch.bfloat16, seed=1)
    lw = rglru.LayerWeights.from_host(w, "cpu")
    assert lw.H == 48 and lw.W_down.shape == (16, 48) and lw.norm1_scale.dtype == torch.float32
    st = lw.struct()
    names = [f for f, _ in _abi.RGLRULayerWeights._fields_]
    assert names == list(rglru.LayerWeights.FIELDS)
    for f in names:
        assert getattr(st, f) == getattr(lw, f).data_ptr()
    assert torch.equal(lw.W_gate, w.extra["W_gate"]) and torch.equal(lw.W_1, w.W_1)
    # the header's struct lists the same fields in the same order
    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "rglru.h"), encoding="utf-8").read()
    body = hdr[hdr.index("typedef struct rglru_layer_weights"):hdr.index("} rglru_layer_weights;")]
    assert re.findall(r"\*\s*(\w+);", body) == names


def test_layer_workspace_sizes_follow_the_documented_layouts():
    lib = _abi.load()
    r256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    for B, T, D, R, H in [(1, 8, 64, 64, 192), (2, 150, 136, 264, 408), (4, 4096, 4096, 5632, 12288)]:
        n = B * T
        blk = lib.rglru_block_workspace_bytes(B, T, D, R, 1)
        assert lib.rglru_layer_workspace_bytes(B, T, D, R, H, 1) == r256(blk) + 3 * r256(n * D * 2) + 2 * r256(n * H * 2)
        stp = lib.rglru_step_workspace_bytes(B, R, 1)
        assert lib.rglru_layer_step_workspace_bytes(B, D, R, H, 1) == (
            r256(stp) + 3 * r256(B * D * 2) + 3 * r256(B * R * 2) + 2 * r256(B * H * 2))


def test_layer_binding_takes_cuda_tensors_only():
    import torch
    from gated_linear_rnn_conv1d_b200 import inputs, rglru
    w = inputs.make_layer(1, 4, 16, 24, 3, torch.bfloat16, seed=1)
    p = rglru.Params.from_host(w.params, "cpu")
    lw = rglru.LayerWeights.from_host(w, "cpu")
    ws = torch.empty(1 << 20, dtype=torch.uint8)
    with pytest.raises(ValueError):
        rglru.layer_forward(p, lw, w.x, workspace=ws, out=torch.empty_like(w.x), h_T=torch.empty(1, 24))
    with pytest.raises(ValueError):
        rglru.layer_step(p, lw, w.x[:, 0].contiguous(), torch.zeros(1, 3, 24, dtype=torch.bfloat16),
                         torch.zeros(1, 24), 0, workspace=ws, out_t=torch.empty(1, 16, dtype=torch.bfloat16))


def test_attention_steps_reject_bad_arguments_before_any_launch():
    lib = _abi.load()
    ok_ptr = _fake()
    B, D, W, Hm = 4, 256, 128, 768
    wb = lib.rglru_attention_step_workspace_bytes(B, D, W)
    assert wb > 0
    assert lib.rglru_attention_step_workspace_bytes(B, 200, W) == 0       # D not a multiple of 128
    assert lib.rglru_attention_step_workspace_bytes(B, 128 * 65, W) == 0   # more than 64 heads
    assert lib.rglru_attention_step_workspace_bytes(B, D, 100) == 0       # window not a multiple of 128
    assert lib.rglru_attention_step_workspace_bytes(0, D, W) == 0
    f = 0x100000
    aw = _abi.RGLRUAttentionWeights(f, f)
    ws = _fake(0x200000)

    def call(**kw):
        return lib.rglru_attention_step(kw.get("w", ctypes.byref(aw)), kw.get("x", ok_ptr), kw.get("k", ok_ptr),
                                        kw.get("v", ok_ptr), kw.get("out", ok_ptr), B, kw.get("D", D),
                                        kw.get("W", W), kw.get("pos", 0), kw.get("ws", ws), kw.get("wsb", wb), None)

    assert call(D=192) == -2
    assert call(W=192) == -2
    assert call(pos=-1) == -2
    assert call(w=None) == -1
    assert call(k=None) == -1
    assert call(v=_fake(0x100004)) == -3
    assert call(ws=None) == -5
    assert call(wsb=wb - 1) == -5
    assert call(ws=_fake(0x200010)) == -3

    lwb = lib.rglru_attention_layer_step_workspace_bytes(B, D, Hm, W)
    assert lwb > wb
    lw = _abi.RGLRUAttentionLayerWeights(f, f, f, f, f, f, f)

    def lcall(**kw):
        return lib.rglru_attention_layer_step(kw.get("w", ctypes.byref(lw)), kw.get("x", ok_ptr), ok_ptr, ok_ptr,
                                              kw.get("out", _fake(0x300000)), B, D, kw.get("H", Hm), W,
                                              kw.get("pos", 0), kw.get("eps", 1e-6), ws, kw.get("wsb", lwb), None)

    assert lcall(out=ok_ptr) == -2         # out_t == x_t
    assert lcall(H=12) == -2
    assert lcall(eps=float("nan")) == -2
    assert lcall(w=None) == -1
    assert lcall(wsb=lwb - 1) == -5


def test_attention_weights_marshal_in_header_order():
    hdr = open(HEADER, encoding="utf-8").read()
    for struct, cls in (("rglru_attention_weights", _abi.RGLRUAttentionWeights),
                        ("rglru_attention_layer_weights", _abi.RGLRUAttentionLayerWeights)):
        end = hdr.index("} " + struct + ";")
        body = hdr[hdr.rindex("typedef struct", 0, end):end]
        assert re.findall(r"\*\s*(\w+);", body) == [f for f, _ in cls._fields_], struct


def test_attention_workspace_sizes_follow_the_documented_layout():
    lib = _abi.load()
    r256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    for B, D, W in [(1, 128, 128), (3, 256, 128), (256, 4096, 1024)]:
        H, nc = D // 128, W // 128
        want = 256 + r256(B * (H + 2) * 128 * 2) + r256(B * H * 128 * 2) + r256(B * nc * H * 128 * 4) + \
            2 * r256(B * nc * H * 4) + r256(B * H * 128 * 2) + 80 * 256 * 256 * 4
        assert lib.rglru_attention_step_workspace_bytes(B, D, W) == want
