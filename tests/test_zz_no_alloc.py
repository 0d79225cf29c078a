"""rglru_scan_noalloc: the scan for callers that cannot allocate device memory (a plugin
handed only its inputs and outputs, a process whose memory is reserved up front, a loop
that must not risk a cudaMalloc synchronising the device). Its scratch is a fixed array
inside the library. Two calls in a row, through the C ABI, must agree with the
workspace-taking rglru_scan within the parity tolerances; the second call checks that
the state the first one leaves behind in the shared array does no harm.

This file is collected last on purpose, and it also passes when run on its own."""
import ctypes

import pytest
import torch

from gated_linear_rnn_conv1d_b200 import _abi, inputs, rglru

from _util import TOL, pack_gates, rel

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(B, T, R, dtype, seed):
    w = inputs.make_forward(B, T, R, dtype, seed=seed)
    g = torch.Generator("cpu").manual_seed(seed + 1)
    w.h0 = torch.randn(B, R, generator=g)
    za = torch.randn(B * T, R, generator=g).double().numpy()
    zx = torch.randn(B * T, R, generator=g).double().numpy()
    return w, pack_gates(za, zx, R, dtype, DEV)


def _noalloc(lib, p, x, z, h0, y, h_T, B, T, R, io):
    st = p.struct()
    return lib.rglru_scan_noalloc(ctypes.byref(st), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(z.data_ptr()),
                                  None, ctypes.c_void_p(h0.data_ptr()), None, ctypes.c_void_p(y.data_ptr()),
                                  ctypes.c_void_p(h_T.data_ptr()), B, T, R, io,
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype,shapes", [
    (torch.bfloat16, [(2, 300, 264), (8, 2048, 2048)]),
    (torch.float32, [(1, 256, 256), (3, 130, 72)]),
])
def test_noalloc_scan_matches_workspace_scan_two_calls_in_a_row(dtype, shapes):
    lib = _abi.load()
    io = _abi.RGLRU_BF16 if dtype == torch.bfloat16 else _abi.RGLRU_F32
    for k, (B, T, R) in enumerate(shapes):
        w, z = _case(B, T, R, dtype, seed=10 + k)
        p = rglru.Params.from_host(w.params)
        x, h0 = w.x.to(DEV), w.h0.to(DEV)
        y_ref, h_ref = rglru.scan(p, x, z, h0)
        y = torch.full_like(x, float("nan"))
        h_T = torch.full((B, R), float("nan"), device=DEV)
        assert _noalloc(lib, p, x, z, h0, y, h_T, B, T, R, io) == 0
        assert lib.rglru_workspace_status(None, None) == 0
        assert rel(y, y_ref) <= TOL[dtype], (B, T, R)
        assert rel(h_T, h_ref) <= TOL[dtype], (B, T, R)


def test_noalloc_scan_rejects_problems_beyond_its_scratch():
    lib = _abi.load()
    B, T, R = 1, 32768, 4096            # 16384 tiles: more than the fixed scratch holds
    x = torch.zeros(B, T, R, dtype=torch.bfloat16, device=DEV)
    z = torch.zeros(B * T, rglru.gate_pitch(R), dtype=torch.bfloat16, device=DEV)
    w = inputs.make_forward(1, 1, R, torch.bfloat16)
    p = rglru.Params.from_host(w.params)
    h0 = torch.zeros(B, R, device=DEV)
    y = torch.empty_like(x)
    h_T = torch.empty(B, R, device=DEV)
    assert _noalloc(lib, p, x, z, h0, y, h_T, B, T, R, _abi.RGLRU_BF16) == _abi.STATUS_CODE["RGLRU_ERR_WORKSPACE"]
