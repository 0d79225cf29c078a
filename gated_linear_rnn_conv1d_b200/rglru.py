"""Python binding of librglru.so: the same entry points as include/rglru.h, taking torch
tensors. Only argument marshalling happens here — PyTorch provides device memory and
streams; every step of the layer runs in the library's CUDA kernels. There is no CPU or
PyTorch fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import _abi

_DT = {torch.float32: _abi.RGLRU_F32, torch.bfloat16: _abi.RGLRU_BF16}


def _io(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}: use torch.bfloat16 or torch.float32")
    return _DT[t.dtype]


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("librglru takes CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("librglru takes contiguous tensors only")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream: Optional[torch.cuda.Stream]):
    st = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(st.cuda_stream)


@dataclass
class Params:
    """Device-resident layer parameters (see rglru_params in include/rglru.h)."""
    conv_w: torch.Tensor   # [4][R] float32
    conv_b: torch.Tensor   # [R] float32
    W_a: torch.Tensor      # [R][R] io dtype
    b_a: torch.Tensor      # [R] float32
    W_x: torch.Tensor      # [R][R] io dtype
    b_x: torch.Tensor      # [R] float32
    Lambda: torch.Tensor   # [R] float32

    @classmethod
    def from_host(cls, p, device="cuda") -> "Params":
        """Copies an object with the same fields (e.g. inputs.RGLRUParams) to `device`."""
        return cls(*(getattr(p, f).to(device).contiguous() for f in
                     ("conv_w", "conv_b", "W_a", "b_a", "W_x", "b_x", "Lambda")))

    @property
    def R(self) -> int:
        return self.conv_b.numel()

    def struct(self) -> _abi.RGLRUParams:
        return _abi.RGLRUParams(*(t.data_ptr() for t in (self.conv_w, self.conv_b, self.W_a, self.b_a,
                                                          self.W_x, self.b_x, self.Lambda)))


def _workspace(nbytes: int, device, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return ws
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def forward_workspace_bytes(B: int, T: int, R: int, dtype: torch.dtype) -> int:
    return _abi.load().rglru_forward_workspace_bytes(B, T, R, _DT[dtype])


def forward(params: Params, x: torch.Tensor, h0: Optional[torch.Tensor] = None,
            conv_state0: Optional[torch.Tensor] = None, *, workspace: Optional[torch.Tensor] = None,
            y: Optional[torch.Tensor] = None, h_T: Optional[torch.Tensor] = None,
            conv_state_T: Optional[torch.Tensor] = None, want_conv_state: bool = True,
            stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """rglru_forward: x [B][T][R] → (y [B][T][R], h_T [B][R] fp32, conv_state_T [B][3][R])."""
    lib = _abi.load()
    B, T, R = x.shape
    io = _io(x)
    y = torch.empty_like(x) if y is None else y
    h_T = torch.empty(B, R, dtype=torch.float32, device=x.device) if h_T is None else h_T
    if conv_state_T is None and want_conv_state:
        conv_state_T = torch.empty(B, 3, R, dtype=x.dtype, device=x.device)
    ws = _workspace(lib.rglru_forward_workspace_bytes(B, T, R, io), x.device, workspace)
    st = params.struct()
    _abi.check("rglru_forward", lib.rglru_forward(
        ctypes.byref(st), _p(x), _p(h0), _p(conv_state0), _p(y), _p(h_T), _p(conv_state_T), B, T, R, io,
        _p(ws), ws.numel() * ws.element_size(), _s(stream)))
    return y, h_T, conv_state_T


def forward_kernels(B: int, T: int, R: int, dtype: torch.dtype) -> int:
    """How many kernels rglru_forward launches (2: gate GEMM with the fused scan, 3: separate)."""
    return _abi.load().rglru_forward_kernels(B, T, R, _DT[dtype])


def saved_bytes(B: int, T: int, R: int) -> int:
    return _abi.load().rglru_saved_bytes(B, T, R)


def forward_train(params: Params, x: torch.Tensor, h0: Optional[torch.Tensor] = None,
                  conv_state0: Optional[torch.Tensor] = None, *, workspace: Optional[torch.Tensor] = None,
                  saved: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None):
    """rglru_forward_train (bf16 IO): as forward, and the gate pre-activations saved for
    backward(..., saved=...). Returns (y, h_T, conv_state_T, saved)."""
    lib = _abi.load()
    B, T, R = x.shape
    y = torch.empty_like(x)
    h_T = torch.empty(B, R, dtype=torch.float32, device=x.device)
    conv_state_T = torch.empty(B, 3, R, dtype=x.dtype, device=x.device)
    saved = _workspace(lib.rglru_saved_bytes(B, T, R), x.device, saved)
    ws = _workspace(lib.rglru_forward_workspace_bytes(B, T, R, _abi.RGLRU_BF16), x.device, workspace)
    st = params.struct()
    _abi.check("rglru_forward_train", lib.rglru_forward_train(
        ctypes.byref(st), _p(x), _p(h0), _p(conv_state0), _p(y), _p(h_T), _p(conv_state_T), _p(saved), B, T, R,
        _p(ws), ws.numel() * ws.element_size(), _s(stream)))
    return y, h_T, conv_state_T, saved


def backward_workspace_bytes(B: int, T: int, R: int) -> int:
    return _abi.load().rglru_backward_workspace_bytes(B, T, R)


def backward(params: Params, x: torch.Tensor, y: torch.Tensor, dy: torch.Tensor, h0: Optional[torch.Tensor] = None,
             dh_T: Optional[torch.Tensor] = None, conv_state0: Optional[torch.Tensor] = None, *,
             want_dh0: bool = True, want_dconv_state0: bool = True, workspace: Optional[torch.Tensor] = None,
             saved: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> dict:
    """rglru_backward (bf16 IO): gradients of a loss with ∂ℓ/∂y = dy (and ∂ℓ/∂h_T = dh_T)
    for the forward that mapped x (with h0, conv_state0) to y. Returns a dict with dx
    [B][T][R] bf16, dconv_state0 [B][3][R] bf16 (or None), dconv_w [4][R], dconv_b, dW_a,
    db_a, dW_x, db_x, dLambda and dh0 [B][R] (or None), all float32 but dx and dconv_state0.
    With `saved` (from forward_train) the gate pre-activations are read, not recomputed
    (rglru_backward_saved)."""
    lib = _abi.load()
    B, T, R = x.shape
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {
        "dx": torch.empty_like(x),
        "dconv_state0": torch.empty(B, 3, R, dtype=x.dtype, device=dev) if want_dconv_state0 else None,
        "dconv_w": torch.empty(4, R, **f32), "dconv_b": torch.empty(R, **f32),
        "dW_a": torch.empty(R, R, **f32), "db_a": torch.empty(R, **f32),
        "dW_x": torch.empty(R, R, **f32), "db_x": torch.empty(R, **f32),
        "dLambda": torch.empty(R, **f32),
        "dh0": torch.empty(B, R, **f32) if want_dh0 else None,
    }
    g = _abi.RGLRUGrads(*(_p(out[k]) for k in ("dx", "dconv_state0", "dconv_w", "dconv_b", "dW_a", "db_a", "dW_x",
                                                  "db_x", "dLambda", "dh0")))
    ws = _workspace(lib.rglru_backward_workspace_bytes(B, T, R), dev, workspace)
    st = params.struct()
    if saved is None:
        _abi.check("rglru_backward", lib.rglru_backward(
            ctypes.byref(st), _p(x), _p(y), _p(dy), _p(h0), _p(dh_T), _p(conv_state0), ctypes.byref(g), B, T, R,
            _p(ws), ws.numel() * ws.element_size(), _s(stream)))
    else:
        _abi.check("rglru_backward_saved", lib.rglru_backward_saved(
            ctypes.byref(st), _p(x), _p(y), _p(dy), _p(h0), _p(dh_T), _p(conv_state0), _p(saved), ctypes.byref(g),
            B, T, R, _p(ws), ws.numel() * ws.element_size(), _s(stream)))
    return out


class HostForwardPlan:
    """Device buffers and streams for forward_host on inputs of shape [B][T][R].

    The input is cut into `groups` pieces, `slots` of them in flight at once, each slot with
    its own device copy of x and y and a forward workspace. Pieces are row groups of the
    batch when B is a multiple of `groups` (rows are independent); otherwise (a long single
    sequence) they are consecutive time chunks of T / groups steps, a multiple of 64, each
    started from the state (h, Conv1D history) the previous chunk ended in. Made once and
    reused, so forward_host itself allocates nothing.
    """

    def __init__(self, B: int, T: int, R: int, dtype: torch.dtype = torch.bfloat16, *, groups: int = 4,
                 slots: int = 3, device=None):
        self.B, self.T, self.R, self.dtype, self.groups = B, T, R, dtype, groups
        if B % groups == 0:
            self.split, self.rows, self.steps = "rows", B // groups, T
        elif T % groups == 0 and (T // groups) % 64 == 0:
            self.split, self.rows, self.steps = "time", B, T // groups
        else:
            raise ValueError(f"neither B={B} nor T={T} splits into {groups} groups (time chunks: multiples of 64)")
        self.slots = min(slots, groups)
        dev = torch.device("cuda") if device is None else torch.device(device)
        nws = forward_workspace_bytes(self.rows, self.steps, R, dtype)
        shape = (self.rows, self.steps, R)
        self.x = [torch.empty(shape, dtype=dtype, device=dev) for _ in range(self.slots)]
        self.y = [torch.empty(shape, dtype=dtype, device=dev) for _ in range(self.slots)]
        self.h_T = [torch.empty(self.rows, R, dtype=torch.float32, device=dev) for _ in range(self.slots)]
        self.ws = [torch.empty(max(nws, 256), dtype=torch.uint8, device=dev) for _ in range(self.slots)]
        # time chunks hand their final state to the next chunk (ping-pong, never read and
        # written by the same call)
        self.conv_state = [torch.empty(self.rows, 3, R, dtype=dtype, device=dev) for _ in range(2)] \
            if self.split == "time" else None
        self.copy_in = torch.cuda.Stream(dev)
        self.compute = torch.cuda.Stream(dev)
        self.copy_out = torch.cuda.Stream(dev)
        self.device = dev

    def status(self) -> int:
        """The first non-zero status word of the slots' workspaces (0: all calls were clean)."""
        for ws in self.ws:
            st = workspace_status(ws)
            if st != 0:
                return st
        return 0


def forward_host(params: Params, x_host: torch.Tensor, y_host: torch.Tensor, h_T_host: torch.Tensor,
                 plan: HostForwardPlan, stream: Optional[torch.cuda.Stream] = None) -> None:
    """rglru_forward on host tensors (pinned for the copies to overlap): x_host [B][T][R] →
    y_host [B][T][R], h_T_host [B][R] fp32, zero initial state and history.

    The plan's pieces are pipelined: the host→device copy of one piece, rglru_forward on the
    next and the device→host copy of a third run on three streams at once. Row groups are
    independent; time chunks run one after another on the compute stream, each from the
    state its predecessor returned. The work is ordered after `stream` (default: the
    current stream) and `stream` waits for all of it before later work, so events recorded
    on it time the whole transfer. With row groups the results are bit-identical to one
    rglru_forward over the whole batch; with time chunks they equal the sequence split at
    the chunk boundaries.
    """
    if x_host.shape != (plan.B, plan.T, plan.R) or x_host.dtype != plan.dtype:
        raise ValueError("x_host does not match the plan")
    outer = torch.cuda.current_stream(plan.device) if stream is None else stream
    start = torch.cuda.Event()
    start.record(outer)
    freed = [None] * plan.slots  # event: the slot's last device→host copy has finished
    for g in range(plan.groups):
        k = g % plan.slots
        if plan.split == "rows":
            piece = (slice(g * plan.rows, (g + 1) * plan.rows),)
        else:
            piece = (slice(None), slice(g * plan.steps, (g + 1) * plan.steps))
        with torch.cuda.stream(plan.copy_in):
            plan.copy_in.wait_event(start)
            if freed[k] is not None:
                plan.copy_in.wait_event(freed[k])
            plan.x[k].copy_(x_host[piece], non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(plan.copy_in)
        plan.compute.wait_event(loaded)
        if plan.split == "rows":
            forward(params, plan.x[k], workspace=plan.ws[k], y=plan.y[k], h_T=plan.h_T[k], want_conv_state=False,
                    stream=plan.compute)
        else:
            h_in = plan.h_T[(g - 1) % plan.slots] if g > 0 else None
            st_in = plan.conv_state[(g - 1) % 2] if g > 0 else None
            forward(params, plan.x[k], h_in, st_in, workspace=plan.ws[k], y=plan.y[k], h_T=plan.h_T[k],
                    conv_state_T=plan.conv_state[g % 2], stream=plan.compute)
        done = torch.cuda.Event()
        done.record(plan.compute)
        with torch.cuda.stream(plan.copy_out):
            plan.copy_out.wait_event(done)
            y_host[piece].copy_(plan.y[k], non_blocking=True)
            if plan.split == "rows":
                h_T_host[piece[0]].copy_(plan.h_T[k], non_blocking=True)
            elif g == plan.groups - 1:
                h_T_host.copy_(plan.h_T[k], non_blocking=True)
            freed[k] = torch.cuda.Event()
            freed[k].record(plan.copy_out)
    for e in freed:
        if e is not None:
            outer.wait_event(e)


def step_workspace_bytes(B: int, R: int, dtype: torch.dtype = torch.bfloat16) -> int:
    return _abi.load().rglru_step_workspace_bytes(B, R, _DT[dtype])


def step(params: Params, x_t: torch.Tensor, conv_state: torch.Tensor, h: torch.Tensor, step_index: int, *,
         workspace: Optional[torch.Tensor] = None, y_t: Optional[torch.Tensor] = None,
         stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """rglru_step: one decode step; updates conv_state and h in place, returns y_t."""
    lib = _abi.load()
    B, R = x_t.shape
    io = _io(x_t)
    y_t = torch.empty_like(x_t) if y_t is None else y_t
    ws = _workspace(lib.rglru_step_workspace_bytes(B, R, io), x_t.device, workspace)
    st = params.struct()
    _abi.check("rglru_step", lib.rglru_step(
        ctypes.byref(st), _p(x_t), _p(conv_state), _p(h), _p(y_t), B, R, int(step_index), io, _p(ws),
        ws.numel() * ws.element_size(), _s(stream)))
    return y_t


def block_workspace_bytes(B: int, T: int, D: int, R: int) -> int:
    return _abi.load().rglru_block_workspace_bytes(B, T, D, R, _abi.RGLRU_BF16)


def block_forward(params: Params, W_1: torch.Tensor, W_2: torch.Tensor, W_o: torch.Tensor, x: torch.Tensor,
                  h0: Optional[torch.Tensor] = None, *, workspace: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None, h_T: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """rglru_block_forward: x [B][T][D] → (out [B][T][D], h_T [B][R])."""
    lib = _abi.load()
    B, T, D = x.shape
    R = W_1.shape[0]
    io = _io(x)
    out = torch.empty_like(x) if out is None else out
    h_T = torch.empty(B, R, dtype=torch.float32, device=x.device) if h_T is None else h_T
    ws = _workspace(lib.rglru_block_workspace_bytes(B, T, D, R, io), x.device, workspace)
    st = params.struct()
    _abi.check("rglru_block_forward", lib.rglru_block_forward(
        ctypes.byref(st), _p(W_1), _p(W_2), _p(W_o), _p(x), _p(h0), _p(out), _p(h_T), B, T, D, R, io, _p(ws),
        ws.numel() * ws.element_size(), _s(stream)))
    return out, h_T


@dataclass
class LayerWeights:
    """Device-resident weights of one Hawk residual layer besides the RG-LRU parameters
    (see rglru_layer_weights in include/rglru.h). Linears bf16 [out][in]; gains float32."""
    norm1_scale: torch.Tensor  # [D]
    W_1: torch.Tensor          # [R][D]
    W_2: torch.Tensor          # [R][D]
    W_o: torch.Tensor          # [D][R]
    norm2_scale: torch.Tensor  # [D]
    W_gate: torch.Tensor       # [H][D]
    W_up: torch.Tensor         # [H][D]
    W_down: torch.Tensor       # [D][H]

    FIELDS = ("norm1_scale", "W_1", "W_2", "W_o", "norm2_scale", "W_gate", "W_up", "W_down")

    @classmethod
    def from_host(cls, w, device="cuda") -> "LayerWeights":
        """Copies an object with the same fields (e.g. an inputs.Workload of a layer) to `device`."""
        src = w.extra if hasattr(w, "extra") and "W_gate" in w.extra else {}
        return cls(*((src[f] if f in src else getattr(w, f)).to(device).contiguous() for f in cls.FIELDS))

    @property
    def H(self) -> int:
        return self.W_gate.shape[0]

    def struct(self) -> _abi.RGLRULayerWeights:
        return _abi.RGLRULayerWeights(*(getattr(self, f).data_ptr() for f in self.FIELDS))


def layer_workspace_bytes(B: int, T: int, D: int, R: int, H: int) -> int:
    return _abi.load().rglru_layer_workspace_bytes(B, T, D, R, H, _abi.RGLRU_BF16)


def layer_forward(params: Params, weights: LayerWeights, x: torch.Tensor, h0: Optional[torch.Tensor] = None, *,
                  eps: float = 1e-6, workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                  h_T: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """rglru_layer_forward: x [B][T][D] → (out [B][T][D], h_T [B][R])."""
    lib = _abi.load()
    B, T, D = x.shape
    R, H = weights.W_1.shape[0], weights.H
    io = _io(x)
    out = torch.empty_like(x) if out is None else out
    h_T = torch.empty(B, R, dtype=torch.float32, device=x.device) if h_T is None else h_T
    ws = _workspace(lib.rglru_layer_workspace_bytes(B, T, D, R, H, io), x.device, workspace)
    st, wst = params.struct(), weights.struct()
    _abi.check("rglru_layer_forward", lib.rglru_layer_forward(
        ctypes.byref(st), ctypes.byref(wst), _p(x), _p(h0), _p(out), _p(h_T), B, T, D, R, H, float(eps), io, _p(ws),
        ws.numel() * ws.element_size(), _s(stream)))
    return out, h_T


def layer_step_workspace_bytes(B: int, D: int, R: int, H: int) -> int:
    return _abi.load().rglru_layer_step_workspace_bytes(B, D, R, H, _abi.RGLRU_BF16)


def layer_step(params: Params, weights: LayerWeights, x_t: torch.Tensor, conv_state: torch.Tensor,
               h: torch.Tensor, step_index: int, *, eps: float = 1e-6, workspace: Optional[torch.Tensor] = None,
               out_t: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """rglru_layer_step: x_t [B][D] → out_t [B][D]; conv_state [B][3][R] and h [B][R] in place."""
    lib = _abi.load()
    B, D = x_t.shape
    R, H = weights.W_1.shape[0], weights.H
    io = _io(x_t)
    out_t = torch.empty_like(x_t) if out_t is None else out_t
    ws = _workspace(lib.rglru_layer_step_workspace_bytes(B, D, R, H, io), x_t.device, workspace)
    st, wst = params.struct(), weights.struct()
    _abi.check("rglru_layer_step", lib.rglru_layer_step(
        ctypes.byref(st), ctypes.byref(wst), _p(x_t), _p(conv_state), _p(h), _p(out_t), B, D, R, H, int(step_index),
        float(eps), io, _p(ws), ws.numel() * ws.element_size(), _s(stream)))
    return out_t


@dataclass
class AttentionWeights:
    """Device-resident weights of Griffin's local-attention block (see rglru_attention_weights
    in include/rglru.h): W_qkv [(H+2)·128][D] (W_q, then W_k, then W_v rows), W_o [D][H·128],
    bf16. For the residual layer also the two RMSNorm gains (float32) and the gated MLP."""
    W_qkv: torch.Tensor
    W_o: torch.Tensor
    norm1_scale: Optional[torch.Tensor] = None
    norm2_scale: Optional[torch.Tensor] = None
    W_gate: Optional[torch.Tensor] = None
    W_up: Optional[torch.Tensor] = None
    W_down: Optional[torch.Tensor] = None

    @classmethod
    def from_host(cls, w: dict, device="cuda") -> "AttentionWeights":
        """Copies a dict with W_q, W_k, W_v, W_o (and optionally the layer's norm gains and MLP
        weights) to `device`, stacking W_q, W_k, W_v into W_qkv."""
        W_qkv = torch.cat([w["W_q"], w["W_k"], w["W_v"]], 0)
        opt = {k: w[k].to(device).contiguous() for k in ("norm1_scale", "norm2_scale", "W_gate", "W_up", "W_down")
               if k in w}
        return cls(W_qkv.to(device).contiguous(), w["W_o"].to(device).contiguous(), **opt)

    def struct(self) -> _abi.RGLRUAttentionWeights:
        return _abi.RGLRUAttentionWeights(self.W_qkv.data_ptr(), self.W_o.data_ptr())

    def layer_struct(self) -> _abi.RGLRUAttentionLayerWeights:
        return _abi.RGLRUAttentionLayerWeights(*(getattr(self, f).data_ptr() for f in (
            "norm1_scale", "W_qkv", "W_o", "norm2_scale", "W_gate", "W_up", "W_down")))


def attention_rings(B: int, window: int, device="cuda") -> Tuple[torch.Tensor, torch.Tensor]:
    """Empty KV rings of the local attention: keys and values [B][window][128], slot-major."""
    return (torch.empty(B, window, 128, dtype=torch.bfloat16, device=device),
            torch.empty(B, window, 128, dtype=torch.bfloat16, device=device))


def _check_rings(k_ring: torch.Tensor, v_ring: torch.Tensor, B: int) -> int:
    W = k_ring.shape[1]
    for r in (k_ring, v_ring):
        if tuple(r.shape) != (B, W, 128) or not r.is_contiguous():
            raise ValueError(f"KV rings must be contiguous [B][window][128], got {tuple(r.shape)}")
    return W


def attention_step_workspace_bytes(B: int, D: int, window: int) -> int:
    return _abi.load().rglru_attention_step_workspace_bytes(B, D, window)


def attention_step(weights: AttentionWeights, x_t: torch.Tensor, k_ring: torch.Tensor, v_ring: torch.Tensor,
                   pos: int, *, workspace: Optional[torch.Tensor] = None, out_t: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """rglru_attention_step: x_t [B][D] → out_t [B][D] at position pos; the rings in place."""
    lib = _abi.load()
    B, D = x_t.shape
    W = _check_rings(k_ring, v_ring, B)
    out_t = torch.empty_like(x_t) if out_t is None else out_t
    ws = _workspace(lib.rglru_attention_step_workspace_bytes(B, D, W), x_t.device, workspace)
    st = weights.struct()
    _abi.check("rglru_attention_step", lib.rglru_attention_step(
        ctypes.byref(st), _p(x_t), _p(k_ring), _p(v_ring), _p(out_t), B, D, W, int(pos), _p(ws),
        ws.numel() * ws.element_size(), _s(stream)))
    return out_t


def attention_layer_step_workspace_bytes(B: int, D: int, H: int, window: int) -> int:
    return _abi.load().rglru_attention_layer_step_workspace_bytes(B, D, H, window)


def attention_layer_step(weights: AttentionWeights, x_t: torch.Tensor, k_ring: torch.Tensor, v_ring: torch.Tensor,
                         pos: int, *, eps: float = 1e-6, workspace: Optional[torch.Tensor] = None,
                         out_t: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """rglru_attention_layer_step: Griffin's local-attention residual layer, one decode step."""
    lib = _abi.load()
    B, D = x_t.shape
    W = _check_rings(k_ring, v_ring, B)
    H = weights.W_gate.shape[0]
    out_t = torch.empty_like(x_t) if out_t is None else out_t
    ws = _workspace(lib.rglru_attention_layer_step_workspace_bytes(B, D, H, W), x_t.device, workspace)
    st = weights.layer_struct()
    _abi.check("rglru_attention_layer_step", lib.rglru_attention_layer_step(
        ctypes.byref(st), _p(x_t), _p(k_ring), _p(v_ring), _p(out_t), B, D, H, W, int(pos), float(eps), _p(ws),
        ws.numel() * ws.element_size(), _s(stream)))
    return out_t


def conv1d(params: Params, x: torch.Tensor, conv_state0: Optional[torch.Tensor] = None, *,
           u: Optional[torch.Tensor] = None, conv_state_T: Optional[torch.Tensor] = None,
           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    lib = _abi.load()
    B, T, R = x.shape
    u = torch.empty_like(x) if u is None else u
    _abi.check("rglru_conv1d", lib.rglru_conv1d(_p(params.conv_w), _p(params.conv_b), _p(x), _p(conv_state0),
                                                _p(u), _p(conv_state_T), B, T, R, _io(x), _s(stream)))
    return u


def gate_pitch(R: int) -> int:
    return int(_abi.load().rglru_gate_pitch(R))


def gate_proj(params: Params, u: torch.Tensor, *, z: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """rglru_gate_proj: u [N][R] (or [B][T][R]) → packed z [N][gate_pitch(R)]."""
    lib = _abi.load()
    R = u.shape[-1]
    N = u.numel() // R
    z = torch.empty(N, gate_pitch(R), dtype=u.dtype, device=u.device) if z is None else z
    _abi.check("rglru_gate_proj", lib.rglru_gate_proj(_p(u), _p(params.W_a), _p(params.b_a), _p(params.W_x),
                                                      _p(params.b_x), _p(z), N, R, _io(u), _s(stream)))
    return z


def scan_workspace_bytes(B: int, T: int, R: int, dtype: torch.dtype) -> int:
    return _abi.load().rglru_scan_workspace_bytes(B, T, R, _DT[dtype])


def scan(params: Params, x: torch.Tensor, z: torch.Tensor, h0: Optional[torch.Tensor] = None,
         conv_state0: Optional[torch.Tensor] = None, gate_g: Optional[torch.Tensor] = None, *,
         workspace: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
         h_T: Optional[torch.Tensor] = None,
         stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """rglru_scan: (x, packed z) → (y, h_T)."""
    lib = _abi.load()
    B, T, R = x.shape
    io = _io(x)
    y = torch.empty_like(x) if y is None else y
    h_T = torch.empty(B, R, dtype=torch.float32, device=x.device) if h_T is None else h_T
    ws = _workspace(lib.rglru_scan_workspace_bytes(B, T, R, io), x.device, workspace)
    st = params.struct()
    _abi.check("rglru_scan", lib.rglru_scan(
        ctypes.byref(st), _p(x), _p(z), _p(conv_state0), _p(h0), _p(gate_g), _p(y), _p(h_T), B, T, R, io, _p(ws),
        ws.numel() * ws.element_size(), _s(stream)))
    return y, h_T


def gate_coeffs(params: Params, u: torch.Tensor, *, g: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """rglru_gate_coeffs: u [N_tok][R] bf16 → packed recurrence coefficients as raw 16-bit
    words (torch.int16): d = 1 − a_t as fp16 in the recurrence-gate places,
    b_t = √(1−a_t²)·i_t·u_t as bf16 in the input-gate places (see split_coeffs)."""
    lib = _abi.load()
    N, R = u.shape
    g = torch.empty(N, gate_pitch(R), dtype=torch.int16, device=u.device) if g is None else g
    if g.dtype != torch.int16 or g.shape != (N, gate_pitch(R)):
        raise ValueError("g must be int16 [N_tok][gate_pitch(R)]")
    st = params.struct()
    _abi.check("rglru_gate_coeffs", lib.rglru_gate_coeffs(ctypes.byref(st), _p(u), _p(g), N, R, _s(stream)))
    return g


def split_coeffs(g: torch.Tensor, R: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """The packed coefficient words of gate_coeffs as (d [N][R] float16, b [N][R] bfloat16)."""
    N = g.shape[0]
    blocks = g.view(N, -1, 2, 128)
    d = blocks[:, :, 0, :].reshape(N, -1)[:, :R].view(torch.float16)
    b = blocks[:, :, 1, :].reshape(N, -1)[:, :R].view(torch.bfloat16)
    return d, b


def scan_coeffs(g: torch.Tensor, B: int, T: int, R: int, h0: Optional[torch.Tensor] = None,
                gate_g: Optional[torch.Tensor] = None, *, workspace: Optional[torch.Tensor] = None,
                y: Optional[torch.Tensor] = None, h_T: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """rglru_scan_coeffs: packed coefficients of B·T rows (from gate_coeffs) → (y [B][T][R]
    bf16, h_T [B][R] float32); needs neither x nor the parameters."""
    lib = _abi.load()
    if g.shape[0] != B * T or g.dtype != torch.int16:
        raise ValueError("g must be the int16 packed coefficients of B·T rows (from gate_coeffs)")
    y = torch.empty(B, T, R, dtype=torch.bfloat16, device=g.device) if y is None else y
    h_T = torch.empty(B, R, dtype=torch.float32, device=g.device) if h_T is None else h_T
    ws = _workspace(lib.rglru_scan_workspace_bytes(B, T, R, _abi.RGLRU_BF16), g.device, workspace)
    _abi.check("rglru_scan_coeffs", lib.rglru_scan_coeffs(
        _p(g), _p(h0), _p(gate_g), _p(y), _p(h_T), B, T, R, _p(ws), ws.numel() * ws.element_size(), _s(stream)))
    return y, h_T


def gate_scan_workspace_bytes(B: int, T: int, R: int) -> int:
    return _abi.load().rglru_gate_scan_workspace_bytes(B, T, R, _abi.RGLRU_BF16)


def gate_scan(params: Params, u: torch.Tensor, h0: Optional[torch.Tensor] = None, *,
              workspace: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
              h_T: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """rglru_gate_scan: gate GEMM with the scan fused in its epilogue, from u = Conv1D(x)
    (bf16, T % 128 == 0)."""
    lib = _abi.load()
    B, T, R = u.shape
    io = _io(u)
    y = torch.empty_like(u) if y is None else y
    h_T = torch.empty(B, R, dtype=torch.float32, device=u.device) if h_T is None else h_T
    ws = _workspace(lib.rglru_gate_scan_workspace_bytes(B, T, R, io), u.device, workspace)
    st = params.struct()
    _abi.check("rglru_gate_scan", lib.rglru_gate_scan(
        ctypes.byref(st), _p(u), _p(h0), _p(y), _p(h_T), B, T, R, io, _p(ws), ws.numel() * ws.element_size(),
        _s(stream)))
    return y, h_T


def gemm_bf16(A: torch.Tensor, Bm: torch.Tensor, *, C: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """rglru_gemm_bf16: C[M][N] = A[M][K] · B[N][K]ᵀ (bf16 in/out, fp32 accumulate)."""
    lib = _abi.load()
    K = A.shape[-1]
    M = A.numel() // K
    N = Bm.shape[0]
    C = torch.empty(*A.shape[:-1], N, dtype=torch.bfloat16, device=A.device) if C is None else C
    _abi.check("rglru_gemm_bf16", lib.rglru_gemm_bf16(_p(A), _p(Bm), _p(C), M, N, K, _s(stream)))
    return C


def workspace_status(workspace: Optional[torch.Tensor], stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronises the stream and returns (and clears) the status word of `workspace`
    (None: the library-global word used by calls that take no workspace)."""
    lib = _abi.load()
    return lib.rglru_workspace_status(_p(workspace) if workspace is not None else None, _s(stream))
