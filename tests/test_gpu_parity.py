"""CUDA path vs the float64 oracle, element by element, at sizes that span several tiles
and end in ragged tails; plus the invariants of the recurrence checked on the GPU.

Tolerances (max_i |g−o| / max(|o_i|, rms(o))): 1e-4 on the float32-IO path and 2e-2 on
the bf16-IO path with float32 state, per output tensor."""
import math

import numpy as np
import pytest
import torch

import oracle
from gated_linear_rnn_conv1d_b200 import _abi, inputs, rglru

from _util import TOL, TOL_LAYER, f64, host_params64, pack_gates, rel, unpack_gates

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _wl(B, T, R, dtype, seed=0):
    w = inputs.make_forward(B, T, R, dtype, seed=seed)
    g = torch.Generator("cpu").manual_seed(seed + 77)
    # non-zero biases, initial state and conv history so that every input is exercised
    w.params.b_a = torch.randn(R, generator=g) * 0.5
    w.params.b_x = torch.randn(R, generator=g) * 0.5
    w.h0 = torch.randn(B, R, generator=g)
    w.extra["state0"] = torch.randn(B, 3, R, generator=g).to(dtype)
    return w


def _nan_like(t):
    return torch.full_like(t, float("nan"))


# ------------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype,B,T,R", [(torch.float32, 1, 256, 256), (torch.bfloat16, 2, 77, 264),
                                         (torch.bfloat16, 3, 2, 8), (torch.float32, 2, 100, 72)])
@pytest.mark.parametrize("with_state", [False, True])
def test_conv1d_matches_oracle(dtype, B, T, R, with_state):
    w = _wl(B, T, R, dtype)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    st0 = w.extra["state0"].to(DEV) if with_state else None
    u = _nan_like(x)
    stT = torch.full((B, 3, R), float("nan"), dtype=dtype, device=DEV)
    rglru.conv1d(p, x, st0, u=u, conv_state_T=stT)
    u_ref, st_ref = oracle.conv1d_causal(w.x, w.params.conv_w, w.params.conv_b,
                                         w.extra["state0"] if with_state else None)
    tol = 1e-6 if dtype == torch.float32 else 4e-3
    assert rel(u, u_ref) <= tol
    # the carried conv state is the last three inputs, copied exactly
    assert np.array_equal(f64(stT), st_ref)


@pytest.mark.parametrize("dtype,N,R", [(torch.float32, 256, 256), (torch.bfloat16, 300, 264),
                                       (torch.bfloat16, 128, 128), (torch.bfloat16, 1000, 1040),
                                       (torch.float32, 77, 136)])
def test_gate_projection_matches_oracle(dtype, N, R):
    w = _wl(1, N, R, dtype)
    p = rglru.Params.from_host(w.params)
    g = torch.Generator("cpu").manual_seed(5)
    u = torch.randn(N, R, generator=g).to(dtype)
    z = rglru.gate_proj(p, u.to(DEV))
    za, zx = unpack_gates(z, R)
    ra, rx = oracle.gate_preactivations(u, w.params.W_a, w.params.b_a, w.params.W_x, w.params.b_x)
    tol = 1e-5 if dtype == torch.float32 else 8e-3
    assert rel(za, ra) <= tol and rel(zx, rx) <= tol


@pytest.mark.parametrize("N,R", [(300, 136), (1024, 512), (129, 264)])
def test_gate_coeffs_match_oracle(N, R):
    """rglru_gate_coeffs: d = 1 − a_t (fp16) and b_t = √(1−a_t²)·i_t·u_t (bf16) in the packed
    places."""
    w = _wl(1, N, R, torch.bfloat16)
    p = rglru.Params.from_host(w.params)
    g = torch.Generator("cpu").manual_seed(5)
    u = torch.randn(N, R, generator=g).to(torch.bfloat16)
    co = rglru.gate_coeffs(p, u.to(DEV))
    assert co.dtype == torch.int16
    d, _ = unpack_gates(co.view(torch.float16), R)
    _, b = unpack_gates(co.view(torch.bfloat16), R)
    za, zx = oracle.gate_preactivations(u, w.params.W_a, w.params.b_a, w.params.W_x, w.params.b_x)
    a_t = oracle.decay_log_space(oracle.sigmoid(za), w.params.Lambda)
    d_o = 1.0 - a_t
    b_o = np.sqrt(1.0 - a_t * a_t) * oracle.sigmoid(zx) * f64(u)
    assert rel(d, d_o) <= 1e-2 and rel(b, b_o) <= 1e-2


def test_coeff_stages_equal_forward():
    """rglru_forward (bf16) is exactly conv1d → gate_coeffs → scan_coeffs."""
    B, T, R = 2, 300, 264
    w = _wl(B, T, R, torch.bfloat16)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    h0 = w.h0.to(DEV)
    y_f, h_f, _ = rglru.forward(p, x, h0)
    u = rglru.conv1d(p, x)
    co = rglru.gate_coeffs(p, u.view(B * T, R))
    y_s, h_s = rglru.scan_coeffs(co, B, T, R, h0)
    assert torch.equal(y_f, y_s) and torch.equal(h_f, h_s)


@pytest.mark.parametrize("M,N,K", [(300, 136, 200), (1024, 512, 1024), (128, 256, 64), (129, 264, 72),
                                   (4096, 1024, 4096)])
def test_gemm_bf16_matches_matmul(M, N, K):
    g = torch.Generator("cpu").manual_seed(M + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    Bm = (torch.randn(N, K, generator=g) / math.sqrt(K)).to(torch.bfloat16)
    C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    rglru.gemm_bf16(A.to(DEV), Bm.to(DEV), C=C)
    ref = f64(A) @ f64(Bm).T
    assert rel(C, ref) <= 8e-3
    assert _abi.load().rglru_workspace_status(None, None) == 0


def _scan_reference(w, za, zx, with_state, gate=None):
    """Oracle scan given (rounded) gate pre-activations: the GPU scan's own inputs."""
    u, _ = oracle.conv1d_causal(w.x, w.params.conv_w, w.params.conv_b, w.extra["state0"] if with_state else None)
    B, T, R = w.x.shape
    r = oracle.sigmoid(za.reshape(B, T, R))
    i = oracle.sigmoid(zx.reshape(B, T, R))
    a_t = oracle.decay_direct(r, f64(w.params.Lambda))
    y, h_T = oracle.rglru_recurrence(a_t, i, u, f64(w.h0))
    if gate is not None:
        y = y * oracle.gelu(gate)
    return y, h_T


@pytest.mark.parametrize("dtype,B,T,R", [(torch.bfloat16, 2, 200, 264), (torch.float32, 1, 256, 256),
                                         (torch.float32, 3, 130, 72), (torch.bfloat16, 1, 1000, 128),
                                         (torch.bfloat16, 2, 3, 8)])
@pytest.mark.parametrize("gated", [False, True])
def test_scan_matches_oracle(dtype, B, T, R, gated):
    w = _wl(B, T, R, dtype)
    p = rglru.Params.from_host(w.params)
    u, _ = oracle.conv1d_causal(w.x, w.params.conv_w, w.params.conv_b, w.extra["state0"])
    za, zx = oracle.gate_preactivations(u.reshape(B * T, R), w.params.W_a, w.params.b_a, w.params.W_x, w.params.b_x)
    z = pack_gates(za, zx, R, dtype, DEV)
    za_r, zx_r = unpack_gates(z, R)                 # what the GPU sees after rounding
    gate = None
    if gated:
        gate = torch.randn(B, T, R, generator=torch.Generator("cpu").manual_seed(3)).to(dtype)
    y = torch.full((B, T, R), float("nan"), dtype=dtype, device=DEV)
    h_T = torch.full((B, R), float("nan"), device=DEV)
    rglru.scan(p, w.x.to(DEV), z, w.h0.to(DEV), w.extra["state0"].to(DEV),
               gate.to(DEV) if gated else None, y=y, h_T=h_T)
    y_ref, h_ref = _scan_reference(w, za_r, zx_r, True, gate)
    assert rel(y, y_ref) <= TOL[dtype]
    assert rel(h_T, h_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,B,T,R", [(torch.float32, 1, 256, 256), (torch.bfloat16, 2, 200, 264),
                                         (torch.bfloat16, 1, 65, 8), (torch.bfloat16, 4, 1, 136),
                                         (torch.float32, 2, 190, 136)])
@pytest.mark.parametrize("with_state", [False, True])
def test_forward_matches_oracle(dtype, B, T, R, with_state):
    w = _wl(B, T, R, dtype)
    p = rglru.Params.from_host(w.params)
    h0 = w.h0 if with_state else None
    st0 = w.extra["state0"] if with_state else None
    y = torch.full((B, T, R), float("nan"), dtype=dtype, device=DEV)
    y, h_T, stT = rglru.forward(p, w.x.to(DEV), h0.to(DEV) if with_state else None,
                                st0.to(DEV) if with_state else None, y=y)
    ws_status = rglru.workspace_status(None)
    y_ref, h_ref, st_ref = oracle.rglru_forward(w.x, w.params.conv_w, w.params.conv_b, w.params.W_a,
                                                w.params.b_a, w.params.W_x, w.params.b_x, w.params.Lambda,
                                                h0=h0, conv_state0=st0)
    assert ws_status == 0
    assert rel(y, y_ref) <= TOL[dtype]
    assert rel(h_T, h_ref) <= TOL[dtype]
    assert np.array_equal(f64(stT), st_ref)


@pytest.mark.parametrize("x_scale", [1e5, 1e30, 1e-30])
def test_bf16_forward_keeps_the_input_scale(x_scale):
    """The bf16 forward holds every u-scaled value in a format with float32's exponent range
    (u and y bf16, b_t = √(1−a_t²)·i_t·u_t bf16): inputs far outside fp16's range — |u| around
    1e5 or 1e30, or 1e-30 with the conv bias 0 so that u keeps that scale — give finite outputs
    within the bf16 bound of the oracle. The gate weights are scaled by 1/x_scale so that the
    pre-activations stay O(1) (otherwise every gate saturates and the bf16 rounding of u
    decides r and i, which no bf16 operand avoids)."""
    B, T, R = 2, 200, 264
    w = _wl(B, T, R, torch.bfloat16, seed=11)
    w.x = (w.x.double() * x_scale).to(torch.bfloat16)
    w.params.conv_b = torch.zeros(R)
    w.params.W_a = (w.params.W_a.double() / x_scale).to(torch.bfloat16)
    w.params.W_x = (w.params.W_x.double() / x_scale).to(torch.bfloat16)
    h0 = (w.h0.double() * x_scale).float()
    st0 = (w.extra["state0"].double() * x_scale).to(torch.bfloat16)
    assert torch.isfinite(w.x.float()).all() and torch.isfinite(h0).all()
    p = rglru.Params.from_host(w.params)
    y, h_T, _ = rglru.forward(p, w.x.to(DEV), h0.to(DEV), st0.to(DEV))
    assert rglru.workspace_status(None) == 0
    y_ref, h_ref, _ = oracle.rglru_forward(w.x, w.params.conv_w, w.params.conv_b, w.params.W_a, w.params.b_a,
                                           w.params.W_x, w.params.b_x, w.params.Lambda, h0=h0, conv_state0=st0)
    assert torch.isfinite(y.float()).all() and torch.isfinite(h_T).all()
    assert rel(y, y_ref) <= TOL[torch.bfloat16]
    assert rel(h_T, h_ref) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_forward_on_a_garbage_workspace(dtype):
    """rglru_forward leaves the zeroing of the scan's status word, ticket and chunk carries
    to its Conv1D kernel (no memset): a workspace full of arbitrary bytes — words that read as
    published carries among them — gives the same result as a zeroed one, bit for bit, and
    a clean status."""
    B, T, R = 3, 300, 264
    w = _wl(B, T, R, dtype)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    nbytes = rglru.forward_workspace_bytes(B, T, R, dtype)
    ws0 = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    y0, h0, _ = rglru.forward(p, x, workspace=ws0)
    g = torch.Generator().manual_seed(7)
    ws1 = torch.randint(0, 256, (nbytes,), generator=g, dtype=torch.uint8).to(DEV)
    y1, h1, _ = rglru.forward(p, x, workspace=ws1)
    assert rglru.workspace_status(ws0) == 0 and rglru.workspace_status(ws1) == 0
    assert torch.equal(y0, y1) and torch.equal(h0, h1)


def test_back_to_back_forwards_share_a_workspace():
    """Calls queued back to back on one stream, one workspace, no synchronisation between
    them: the second call's Conv1D kernel zeroes the workspace the first call's scan used,
    and the gate GEMM and scan start early as programmatic dependents — each result must
    equal the same call made alone, bit for bit."""
    B, T, R = 4, 256, 520
    w1 = _wl(B, T, R, torch.bfloat16, seed=1)
    w2 = _wl(B, T, R, torch.bfloat16, seed=2)
    p = rglru.Params.from_host(w1.params)
    x1, x2 = w1.x.to(DEV), w2.x.to(DEV)
    ws = torch.empty(rglru.forward_workspace_bytes(B, T, R, torch.bfloat16), dtype=torch.uint8, device=DEV)
    ya, ha, _ = rglru.forward(p, x1, workspace=ws)
    torch.cuda.synchronize()
    yb, hb, _ = rglru.forward(p, x2, workspace=ws)
    torch.cuda.synchronize()
    outs = [rglru.forward(p, x, workspace=ws, want_conv_state=False) for x in (x1, x2, x1, x2)]
    torch.cuda.synchronize()
    assert rglru.workspace_status(ws) == 0
    for (y, h, _), (yr, hr) in zip(outs, [(ya, ha), (yb, hb), (ya, ha), (yb, hb)]):
        assert torch.equal(y, yr) and torch.equal(h, hr)


@pytest.mark.parametrize("B,T,R", [(2, 256, 264), (1, 128, 128), (3, 384, 136), (1, 640, 8)])
@pytest.mark.parametrize("with_state", [False, True])
def test_fused_gate_scan_matches_oracle(B, T, R, with_state):
    """rglru_gate_scan: the gate GEMM with the scan fused in its epilogue (bf16,
    T % 128 == 0). Shapes cover a partial 128-channel block, an odd number of 128-step
    chunks (the last 2-SM tile half-empty) and a single chunk."""
    w = _wl(B, T, R, torch.bfloat16, seed=T)
    p = rglru.Params.from_host(w.params)
    h0 = w.h0 if with_state else None
    st0 = w.extra["state0"] if with_state else None
    x = w.x.to(DEV)
    u = rglru.conv1d(p, x, st0.to(DEV) if with_state else None)
    y = torch.full((B, T, R), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(rglru.gate_scan_workspace_bytes(B, T, R), dtype=torch.uint8, device=DEV)
    y, h_T = rglru.gate_scan(p, u, h0.to(DEV) if with_state else None, workspace=ws, y=y)
    assert rglru.workspace_status(ws) == 0
    y_ref, h_ref, _ = oracle.rglru_forward(w.x, w.params.conv_w, w.params.conv_b, w.params.W_a, w.params.b_a,
                                           w.params.W_x, w.params.b_x, w.params.Lambda, h0=h0, conv_state0=st0)
    assert rel(y, y_ref) <= TOL[torch.bfloat16]
    assert rel(h_T, h_ref) <= TOL[torch.bfloat16]


def test_forward_takes_the_fused_path_at_large_r_and_matches_oracle():
    """rglru_forward with bf16 IO, T a multiple of 128 and R ≥ 4096 runs Conv1D + the gate
    GEMM with the scan in its epilogue (2 kernels); smaller R or ragged T keep the separate
    path (3). Both against the oracle, with a state and a conv history."""
    assert rglru.forward_kernels(1, 256, 4096, torch.bfloat16) == 2
    assert rglru.forward_kernels(1, 256, 3072, torch.bfloat16) == 3
    assert rglru.forward_kernels(8, 2048, 2048, torch.bfloat16) == 3
    assert rglru.forward_kernels(1, 200, 4096, torch.bfloat16) == 3
    assert rglru.forward_kernels(1, 256, 4096, torch.float32) == 3
    B, T, R = 1, 256, 4096
    w = _wl(B, T, R, torch.bfloat16, seed=21)
    p = rglru.Params.from_host(w.params)
    st0 = w.extra["state0"]
    ws = torch.full((rglru.forward_workspace_bytes(B, T, R, torch.bfloat16),), 0xFF, dtype=torch.uint8, device=DEV)
    y, h_T, cs = rglru.forward(p, w.x.to(DEV), w.h0.to(DEV), st0.to(DEV), workspace=ws)
    assert rglru.workspace_status(ws) == 0
    y_ref, h_ref, cs_ref = oracle.rglru_forward(w.x, w.params.conv_w, w.params.conv_b, w.params.W_a, w.params.b_a,
                                                w.params.W_x, w.params.b_x, w.params.Lambda, h0=w.h0,
                                                conv_state0=st0)
    assert rel(y, y_ref) <= TOL[torch.bfloat16]
    assert rel(h_T, h_ref) <= TOL[torch.bfloat16]
    assert rel(cs, cs_ref) == 0.0
    # the same call again on the now-dirty workspace: the carries are cleared each call
    y2, h2, _ = rglru.forward(p, w.x.to(DEV), w.h0.to(DEV), st0.to(DEV), workspace=ws)
    assert torch.equal(y, y2) and torch.equal(h_T, h2)


# ------------------------------------------------------------------------------------
# invariants on the GPU path
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_zero_recurrence_gate_keeps_state_bitwise(dtype):
    """r ≡ 0 ⇒ a_t = 1 and √(1−a_t²) = 0 exactly, so h_t = h_0 bit for bit."""
    B, T, R = 2, 150, 136
    w = _wl(B, T, R, dtype)
    w.params.W_a = torch.zeros(R, R, dtype=dtype)
    w.params.b_a = torch.full((R,), -1000.0)
    p = rglru.Params.from_host(w.params)
    h0 = w.h0.to(DEV)
    y, h_T, _ = rglru.forward(p, w.x.to(DEV), h0)
    assert torch.equal(h_T, h0)
    assert torch.equal(y.float(), h0.to(dtype).float()[:, None, :].expand(B, T, R))


def test_batch_rows_are_independent():
    """A row's result does not depend on the other rows, bit for bit: the conv and the GEMM
    are per-row, and every scan chunk starts from the exact inclusive state its predecessor
    chunk published, so the float32 chain is the same whatever order the tiles ran in."""
    B, T, R = 3, 300, 264
    w = _wl(B, T, R, torch.bfloat16)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    y, h_T, _ = rglru.forward(p, x)
    y1, h1, _ = rglru.forward(p, x[1:2].contiguous())
    assert torch.equal(h_T[1:2], h1)
    assert torch.equal(y[1:2], y1)
    u = rglru.conv1d(p, x)
    u1 = rglru.conv1d(p, x[1:2].contiguous())
    assert torch.equal(u[1:2], u1)
    z = rglru.gate_proj(p, u.view(B * T, R))
    z1 = rglru.gate_proj(p, u1.view(T, R))
    assert torch.equal(z[T:2 * T], z1)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_nan_in_gate_padding_neither_stalls_nor_leaks(dtype):
    """The packed pre-activations of channels past R are padding: filled with the canonical
    NaN (whose carry encoding would otherwise read as "not published"), they must neither
    stall the chunk chain — a stall costs a full bounded wait and a timeout status — nor
    change any output."""
    import time
    B, T, R = 2, 200, 136
    w = _wl(B, T, R, dtype)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    u = rglru.conv1d(p, x)
    z = rglru.gate_proj(p, u.view(B * T, R))
    y_ref, h_ref = rglru.scan(p, x, z)
    n_pad = 128 * ((R + 127) // 128)
    cols = [256 * (c // 128) + (c % 128) + off for c in range(R, n_pad) for off in (0, 128)]
    nan_bits = torch.tensor([0x7FFFFFFF], dtype=torch.int32).view(torch.float32) if dtype == torch.float32 \
        else torch.tensor([0x7FFF], dtype=torch.int16).view(torch.bfloat16)
    zp = z.clone()
    zp[:, cols] = nan_bits.to(DEV)
    ws = torch.zeros(rglru.scan_workspace_bytes(B, T, R, dtype), dtype=torch.uint8, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    y, h = rglru.scan(p, x, zp, workspace=ws)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert rglru.workspace_status(ws) == 0
    assert dt < 0.5
    assert torch.equal(y, y_ref) and torch.equal(h, h_ref)


def test_forward_host_equals_forward():
    """forward_host pipelines row groups through host copies on three streams; the result is
    bit-identical to one rglru_forward over the whole batch, on every call."""
    B, T, R = 4, 300, 264
    w = inputs.make_forward(B, T, R, torch.bfloat16, seed=5)
    p = rglru.Params.from_host(w.params)
    y_ref, h_ref, _ = rglru.forward(p, w.x.to(DEV), want_conv_state=False)
    plan = rglru.HostForwardPlan(B, T, R, torch.bfloat16, groups=4, slots=3)
    x_host = w.x.pin_memory()
    y_host = torch.empty(B, T, R, dtype=torch.bfloat16).pin_memory()
    h_host = torch.empty(B, R, dtype=torch.float32).pin_memory()
    for _ in range(2):
        y_host.fill_(float("nan"))
        rglru.forward_host(p, x_host, y_host, h_host, plan)
        torch.cuda.synchronize()
        assert plan.status() == 0
        assert torch.equal(y_host, y_ref.cpu())
        assert torch.equal(h_host, h_ref.cpu())


def test_forward_host_in_time_chunks():
    """A single long sequence (B = 1) goes through forward_host in time chunks, each started
    from the state the previous chunk returned: the result equals those chained
    rglru_forward calls bit for bit, and the whole-sequence forward within the split test's
    bound."""
    B, T, R, G = 1, 640, 264, 5
    w = inputs.make_forward(B, T, R, torch.bfloat16, seed=8)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    plan = rglru.HostForwardPlan(B, T, R, torch.bfloat16, groups=G, slots=3)
    assert plan.split == "time"
    x_host = w.x.pin_memory()
    y_host = torch.empty(B, T, R, dtype=torch.bfloat16).pin_memory()
    h_host = torch.empty(B, R, dtype=torch.float32).pin_memory()
    rglru.forward_host(p, x_host, y_host, h_host, plan)
    torch.cuda.synchronize()
    assert plan.status() == 0
    h, st, ys = None, None, []
    for g in range(G):
        yg, h, st = rglru.forward(p, x[:, g * 128:(g + 1) * 128].contiguous(), h, st)
        ys.append(yg)
    assert torch.equal(y_host, torch.cat(ys, 1).cpu()) and torch.equal(h_host, h.cpu())
    y, h_T, _ = rglru.forward(p, x)
    assert rel(y_host, y) <= 8e-3 and rel(h_host, h_T) <= 8e-3


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_split_sequence_equals_whole(dtype):
    """forward(0:T1) → (h, conv state) → forward(T1:T) equals forward(0:T)."""
    B, T, R = 2, 500, 136
    w = _wl(B, T, R, dtype)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    y, h_T, st = rglru.forward(p, x)
    for T1 in (1, 64, 129, 499):
        ya, ha, sa = rglru.forward(p, x[:, :T1].contiguous())
        yb, hb, sb = rglru.forward(p, x[:, T1:].contiguous(), ha, sa)
        tol = 1e-5 if dtype == torch.float32 else 8e-3
        assert rel(torch.cat([ya, yb], 1), y) <= tol, T1
        assert rel(hb, h_T) <= tol
        assert torch.equal(sb, st)


def test_decode_steps_equal_forward():
    """T decode steps from a zero state equal one prefill of length T."""
    B, T, R = 8, 40, 264
    w = _wl(B, T, R, torch.bfloat16)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    y, h_T, st = rglru.forward(p, x)
    ring = torch.zeros(B, 3, R, dtype=torch.bfloat16, device=DEV)
    h = torch.zeros(B, R, device=DEV)
    ys = []
    for t in range(T):
        ys.append(rglru.step(p, x[:, t].contiguous(), ring, h, t).clone())
    assert rglru.workspace_status(None) == 0
    assert rel(torch.stack(ys, 1), y) <= 1e-2
    assert rel(h, h_T) <= 1e-2
    # after T = 40 ≡ 1 (mod 3) steps the ring's oldest slot is T mod 3
    order = [(T + j) % 3 for j in range(3)]
    assert torch.equal(ring[:, order], st)


def test_decode_checkpoint_resume_is_bitwise():
    """The decode state is (h, conv ring, step): saving it and continuing from copies in
    fresh buffers gives bit-identical outputs."""
    B, R, n1, n2 = 16, 264, 5, 7
    w = inputs.make_decode(B, R, torch.bfloat16, seed=4)
    p = rglru.Params.from_host(w.params)
    toks = [inputs.decode_token(k, B, R).to(DEV) for k in range(n1 + n2)]
    ring = torch.zeros(B, 3, R, dtype=torch.bfloat16, device=DEV)
    h = torch.zeros(B, R, device=DEV)
    for k in range(n1):
        rglru.step(p, toks[k], ring, h, k)
    saved = (h.cpu().clone(), ring.cpu().clone())
    ref = [rglru.step(p, toks[k], ring, h, k).clone() for k in range(n1, n1 + n2)]
    h2, ring2 = saved[0].to(DEV), saved[1].to(DEV)
    got = [rglru.step(p, toks[k], ring2, h2, k).clone() for k in range(n1, n1 + n2)]
    assert all(torch.equal(a, b) for a, b in zip(ref, got))
    assert torch.equal(h, h2) and torch.equal(ring, ring2)


# (130, 200): the 1-SM step kernel (R not a multiple of 128); the others run the transposed
# split-K kernel, with a ragged batch (5), one batch half (128) and both halves (130, 256)
@pytest.mark.parametrize("B,R", [(130, 200), (5, 256), (128, 384), (130, 256), (256, 128)])
def test_decode_small_matches_oracle_every_step(B, R):
    steps = 9
    w = inputs.make_decode(B, R, torch.bfloat16, seed=2)
    p = rglru.Params.from_host(w.params)
    hp = host_params64(w.params)
    ring = torch.zeros(B, 3, R, dtype=torch.bfloat16, device=DEV)
    h = torch.zeros(B, R, device=DEV)
    ring_o, h_o = np.zeros((B, 3, R)), np.zeros((B, R))
    for k in range(steps):
        xt = inputs.decode_token(k, B, R)
        y = rglru.step(p, xt.to(DEV), ring, h, k)
        y_o, h_o, ring_o = oracle.rglru_step(xt, ring_o, k, h_o, **hp)
        assert rel(y, y_o) <= TOL[torch.bfloat16], k
        assert rel(h, h_o) <= TOL[torch.bfloat16], k
        assert np.array_equal(f64(ring), ring_o)


def test_block_small_matches_oracle():
    B, T, D, R = 2, 150, 136, 264
    w = inputs.make_block(B, T, D, R, torch.bfloat16, seed=6)
    p = rglru.Params.from_host(w.params)
    out = torch.full((B, T, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    out, h_T = rglru.block_forward(p, w.W_1.to(DEV), w.W_2.to(DEV), w.W_o.to(DEV), w.x.to(DEV), out=out)
    assert rglru.workspace_status(None) == 0
    ref, h_ref = oracle.recurrent_block(w.x, w.W_1, w.W_2, w.W_o, **host_params64(w.params))
    assert rel(out, ref) <= TOL[torch.bfloat16]
    assert rel(h_T, h_ref) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("B,T,D,R,M", [(2, 150, 136, 264, 3)])
def test_hawk_layer_small_matches_oracle(B, T, D, R, M):
    w = inputs.make_layer(B, T, D, R, M, torch.bfloat16, seed=7)
    p = rglru.Params.from_host(w.params)
    lw = rglru.LayerWeights.from_host(w)
    out = torch.full((B, T, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = torch.full((rglru.layer_workspace_bytes(B, T, D, R, M * D),), 0xFF, dtype=torch.uint8, device=DEV)
    out, h_T = rglru.layer_forward(p, lw, w.x.to(DEV), eps=oracle.RMS_EPS, out=out, workspace=ws)
    assert rglru.workspace_status(ws) == 0
    e = w.extra
    ref, h_ref = oracle.hawk_residual_layer(w.x, e["norm1_scale"], w.W_1, w.W_2, w.W_o, e["norm2_scale"],
                                            e["W_gate"], e["W_up"], e["W_down"], **host_params64(w.params))
    assert rel(out, ref) <= TOL_LAYER
    assert rel(h_T, h_ref) <= TOL[torch.bfloat16]


# ------------------------------------------------------------------------------------
# failure detection without a GPU fault: a chunk that never publishes its carry makes
# its successor's bounded wait run out; the status word reports it and the context
# stays usable.
def test_lookback_timeout_is_reported_and_recovered():
    lib = _abi.load()
    B, T, R = 1, 64 * 3, 128
    w = _wl(B, T, R, torch.bfloat16)
    p = rglru.Params.from_host(w.params)
    x = w.x.to(DEV)
    ws = torch.empty(rglru.forward_workspace_bytes(B, T, R, torch.bfloat16), dtype=torch.uint8, device=DEV)
    try:
        lib.rglru_debug_scan_stall(1)        # (b=0, block 0, chunk 1) stays silent
        rglru.forward(p, x, workspace=ws)
        assert rglru.workspace_status(ws) == _abi.STATUS_CODE["RGLRU_ERR_TIMEOUT"]
    finally:
        lib.rglru_debug_scan_stall(-1)
    y, h_T, _ = rglru.forward(p, x, workspace=ws)
    assert rglru.workspace_status(ws) == 0
    y_ref, h_ref, _ = oracle.rglru_forward(w.x, w.params.conv_w, w.params.conv_b, w.params.W_a, w.params.b_a,
                                           w.params.W_x, w.params.b_x, w.params.Lambda)
    assert rel(y, y_ref) <= TOL[torch.bfloat16]
