"""rglru_scan_noalloc: the scan for callers that cannot allocate device memory (a plugin
handed only its inputs and outputs, a process whose memory is reserved up front, a loop
that must not risk a cudaMalloc synchronising the device). Its scratch is a fixed array
inside the library. Two calls in a row, through the C ABI, must agree with the
workspace-taking rglru_scan and with the float64 oracle within the parity tolerances; the
second call checks that the state the first one leaves behind in the shared array does no
harm. The largest problem the array holds is run too, so that the size check, the cleared
region and the top of the array are all exercised.

This file is collected last on purpose, and it also passes when run on its own."""
import ctypes

import pytest
import torch

import oracle
from gated_linear_rnn_conv1d_b200 import _abi, inputs, rglru

from _util import TOL, f64, pack_gates, rel, unpack_gates

pytestmark = pytest.mark.gpu
DEV = "cuda"
SCRATCH = 8 << 20


def _tiles(B, T, R, dtype):
    cw = 128 if dtype == torch.bfloat16 else 64
    return B * -(-R // cw) * -(-T // 64)


def _bytes(B, T, R, dtype):
    """The scan's scratch: a 256-byte header, then per tile and channel a 4-byte inclusive
    state (rounded up to 256 bytes in all) and an 8-byte aggregate."""
    cw = 128 if dtype == torch.bfloat16 else 64
    n = _tiles(B, T, R, dtype)
    return 256 + -(-n * cw * 4 // 256) * 256 + n * cw * 8


def _fits(B, T, R, dtype):
    return _bytes(B, T, R, dtype) <= SCRATCH


def _case(B, T, R, dtype, seed):
    w = inputs.make_forward(B, T, R, dtype, seed=seed)
    g = torch.Generator("cpu").manual_seed(seed + 1)
    w.h0 = torch.randn(B, R, generator=g)
    za = torch.randn(B * T, R, generator=g).double().numpy()
    zx = torch.randn(B * T, R, generator=g).double().numpy()
    return w, pack_gates(za, zx, R, dtype, DEV)


def _oracle(w, z, R):
    """The oracle's scan on the same inputs: u = Conv1D(x), the gates from the (rounded) z."""
    B, T, _ = w.x.shape
    za, zx = unpack_gates(z, R)
    u, _ = oracle.conv1d_causal(w.x, w.params.conv_w, w.params.conv_b)
    a_t = oracle.decay_direct(oracle.sigmoid(za.reshape(B, T, R)), f64(w.params.Lambda))
    return oracle.rglru_recurrence(a_t, oracle.sigmoid(zx.reshape(B, T, R)), u, f64(w.h0))


def _noalloc(lib, p, x, z, h0, y, h_T, B, T, R, io):
    st = p.struct()
    return lib.rglru_scan_noalloc(ctypes.byref(st), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(z.data_ptr()),
                                  None, ctypes.c_void_p(h0.data_ptr()), None, ctypes.c_void_p(y.data_ptr()),
                                  ctypes.c_void_p(h_T.data_ptr()), B, T, R, io,
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _run_and_check(lib, dtype, B, T, R, seed):
    io = _abi.RGLRU_BF16 if dtype == torch.bfloat16 else _abi.RGLRU_F32
    w, z = _case(B, T, R, dtype, seed)
    p = rglru.Params.from_host(w.params)
    x, h0 = w.x.to(DEV), w.h0.to(DEV)
    y_ref, h_ref = rglru.scan(p, x, z, h0)
    y = torch.full_like(x, float("nan"))
    h_T = torch.full((B, R), float("nan"), device=DEV)
    assert _noalloc(lib, p, x, z, h0, y, h_T, B, T, R, io) == 0
    assert lib.rglru_scan_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    assert rel(y, y_ref) <= TOL[dtype], (B, T, R)
    assert rel(h_T, h_ref) <= TOL[dtype], (B, T, R)
    y_o, h_o = _oracle(w, z, R)
    assert rel(y, y_o) <= TOL[dtype], (B, T, R)
    assert rel(h_T, h_o) <= TOL[dtype], (B, T, R)


@pytest.mark.parametrize("dtype,shapes", [
    (torch.bfloat16, [(2, 300, 264), (8, 2048, 2048)]),
    (torch.float32, [(1, 256, 256), (3, 130, 72)]),
])
def test_noalloc_scan_matches_workspace_scan_and_oracle_two_calls_in_a_row(dtype, shapes):
    lib = _abi.load()
    for k, (B, T, R) in enumerate(shapes):
        _run_and_check(lib, dtype, B, T, R, seed=10 + k)


def test_noalloc_scan_at_the_largest_problem_its_scratch_holds():
    # 43 rows × 1 channel block × 127 chunks (the last one ragged) = 5461 bf16 tiles:
    # 256 + 5461·(512 + 1024) bytes, 256 bytes below 8 MiB, so the last tile's aggregates lie
    # in the top kilobyte of the array (8 channels keep the oracle's share of the test small)
    B, T, R = 43, 127 * 64 - 5, 8
    assert _tiles(B, T, R, torch.bfloat16) == 5461 and _bytes(B, T, R, torch.bfloat16) == SCRATCH - 256
    lib = _abi.load()
    _run_and_check(lib, torch.bfloat16, B, T, R, seed=21)
    _run_and_check(lib, torch.bfloat16, 2, 300, 264, seed=22)   # and a small call after it


@pytest.mark.parametrize("dtype,B,T,R", [
    (torch.bfloat16, 2, 2731 * 64, 8),   # 5462 bf16 tiles: 1280 bytes more than the array
    (torch.float32, 3, 3641 * 64, 8),    # 10923 float32 tiles of 64 channels: 512 bytes more
    (torch.bfloat16, 1, 32768, 4096),    # the long-sequence workload: 16384 tiles
])
def test_noalloc_scan_rejects_problems_beyond_its_scratch(dtype, B, T, R):
    assert not _fits(B, T, R, dtype)
    lib = _abi.load()
    io = _abi.RGLRU_BF16 if dtype == torch.bfloat16 else _abi.RGLRU_F32
    x = torch.zeros(B, T, R, dtype=dtype, device=DEV)
    z = torch.zeros(B * T, rglru.gate_pitch(R), dtype=dtype, device=DEV)
    w = inputs.make_forward(1, 1, R, dtype)
    p = rglru.Params.from_host(w.params)
    h0 = torch.zeros(B, R, device=DEV)
    y = torch.empty_like(x)
    h_T = torch.empty(B, R, device=DEV)
    assert _noalloc(lib, p, x, z, h0, y, h_T, B, T, R, io) == _abi.STATUS_CODE["RGLRU_ERR_WORKSPACE"]
