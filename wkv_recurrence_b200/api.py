"""Python binding of libwkv.so with the same entry points as include/wkv.h.

Argument marshalling only: tensors -> device pointers, the current CUDA stream,
dtype codes. PyTorch provides device memory and streams; every step of the
operator runs in the library's kernels. There is no fallback path: without the
built library or a CUDA device these functions raise.

The names mirror the page's step function ``wkv_step(state, k, v, w, u) ->
(out, state)`` ("Linear attention without writing a CUDA kernel", section "The
recurrence"): ``step`` takes and returns the (num, den, max_e) state, and
``forward`` runs the same recurrence over a [B, T, C] sequence.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _abi
from ._abi import WkvError  # noqa: F401

State = Tuple[torch.Tensor, torch.Tensor, torch.Tensor]

_DT = {torch.float32: _abi.WKV_F32, torch.bfloat16: _abi.WKV_BF16}
_workspaces = {}


def _dtype_code(t: torch.Tensor, name: str) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"{name}: dtype {t.dtype} is not supported (float32 or bfloat16)")
    return _DT[t.dtype]


def _need_cuda(t: torch.Tensor, name: str, dtype=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _options(options: Optional[dict]):
    if not options:
        return None
    o = _abi.wkv_options()
    for key, val in options.items():
        if not hasattr(o, key):
            raise KeyError(f"unknown option {key!r}")
        setattr(o, key, int(val))
    return ctypes.byref(o)


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def workspace_size(B: int, T: int, C: int, options: Optional[dict] = None) -> int:
    """Bytes of workspace ``forward`` needs for this shape (host-only)."""
    n = _abi.lib().wkv_forward_workspace_size(int(B), int(T), int(C), _options(options))
    if n == 0:
        raise ValueError("invalid sizes or options")
    return int(n)


def forward_kernel(B: int, T: int, C: int, kv_dtype: torch.dtype = torch.float32,
                   options: Optional[dict] = None) -> int:
    """The kernel number (as in ``options["kernel"]``) ``forward`` launches for
    this shape with 16-byte aligned inputs (host-only)."""
    if kv_dtype not in _DT:
        raise TypeError(f"dtype {kv_dtype} is not supported (float32 or bfloat16)")
    n = _abi.lib().wkv_forward_kernel(int(B), int(T), int(C), _DT[kv_dtype], _options(options))
    if n == 0:
        raise ValueError("invalid sizes or options")
    return int(n)


def forward_launches(B: int, T: int, C: int, kv_dtype: torch.dtype = torch.float32,
                     options: Optional[dict] = None) -> int:
    """How many kernels one ``forward`` call launches for this shape (host-only)."""
    if kv_dtype not in _DT:
        raise TypeError(f"dtype {kv_dtype} is not supported (float32 or bfloat16)")
    return int(_abi.lib().wkv_forward_launches(int(B), int(T), int(C), _DT[kv_dtype], _options(options)))


def make_workspace(B: int, T: int, C: int, options: Optional[dict] = None, device=None) -> torch.Tensor:
    """A zero-filled workspace for ``forward`` (zero once; the library keeps it ready)."""
    return torch.zeros(workspace_size(B, T, C, options), dtype=torch.uint8,
                       device=device if device is not None else torch.device("cuda"))


def _default_workspace(nbytes: int, device: torch.device) -> torch.Tensor:
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def _ext(w_t: Optional[torch.Tensor], r: Optional[torch.Tensor], shape, kv_dtype):
    """The wkv_ext struct for optional per-token decays and receptance, or None."""
    if w_t is None and r is None:
        return None
    if w_t is not None:
        _need_cuda(w_t, "w_t", torch.float32)
        if tuple(w_t.shape) != tuple(shape):
            raise ValueError(f"w_t must be {tuple(shape)}")
    if r is not None:
        _need_cuda(r, "r", kv_dtype)
        if tuple(r.shape) != tuple(shape):
            raise ValueError(f"r must be {tuple(shape)}")
    return _abi.wkv_ext(None if w_t is None else w_t.data_ptr(), None if r is None else r.data_ptr())


def forward(k: torch.Tensor, v: torch.Tensor, w: Optional[torch.Tensor], u: torch.Tensor,
            state: Optional[State] = None, *, out_dtype: Optional[torch.dtype] = None,
            out: Optional[torch.Tensor] = None, state_out: Optional[State] = None,
            workspace: Optional[torch.Tensor] = None, options: Optional[dict] = None,
            return_state: bool = True, w_t: Optional[torch.Tensor] = None, r: Optional[torch.Tensor] = None):
    """WKV over a sequence. k, v: [B, T, C] (float32 or bfloat16); w, u: [C] float32.

    state: optional (num, den, max_e), each float32 [B, C]. Returns
    (out [B, T, C], (num, den, max_e)) -- the state after the last token.
    w_t: optional float32 [B, T, C] per-token decays in place of w (w may then
    be None). r: optional receptance [B, T, C] (dtype of k): out = sigmoid(r) wkv.
    """
    _need_cuda(k, "k")
    _need_cuda(v, "v", k.dtype)
    if w_t is None or w is not None:
        _need_cuda(w, "w", torch.float32)
    _need_cuda(u, "u", torch.float32)
    if k.dim() != 3 or v.shape != k.shape:
        raise ValueError("k and v must both be [B, T, C]")
    B, T, C = k.shape
    if (w is not None and w.shape != (C,)) or u.shape != (C,):
        raise ValueError("w and u must be [C]")
    ext = _ext(w_t, r, (B, T, C), k.dtype)
    dev = k.device
    out_dtype = out_dtype or k.dtype
    if out is None:
        out = torch.empty((B, T, C), dtype=out_dtype, device=dev)
    _need_cuda(out, "out", out_dtype)
    sin = None
    if state is not None:
        for i, s in enumerate(state):
            _need_cuda(s, f"state[{i}]", torch.float32)
            if s.shape != (B, C):
                raise ValueError("state arrays must be [B, C]")
        sin = _abi.wkv_cstate(*(s.data_ptr() for s in state))
    sout = None
    if return_state or state_out is not None:
        if state_out is None:
            state_out = tuple(torch.empty((B, C), dtype=torch.float32, device=dev) for _ in range(3))
        for i, s in enumerate(state_out):
            _need_cuda(s, f"state_out[{i}]", torch.float32)
        sout = _abi.wkv_state(*(s.data_ptr() for s in state_out))
    opts = _options(options)
    need = _abi.lib().wkv_forward_workspace_size(B, T, C, opts)
    if need == 0:
        raise ValueError("invalid sizes or options")
    if workspace is None:
        workspace = _default_workspace(need, dev)
    _need_cuda(workspace, "workspace")
    code = _abi.lib().wkv_forward_ext(
        B, T, C, _ptr(k), _ptr(v), _dtype_code(k, "k"), _ptr(w), _ptr(u),
        _ptr(out), _dtype_code(out, "out"),
        ctypes.byref(sin) if sin is not None else None,
        ctypes.byref(sout) if sout is not None else None,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(), opts,
        ctypes.byref(ext) if ext is not None else None)
    _abi.check(code, "wkv_forward")
    return out, state_out


_host_buffers = {}


def forward_host(k: torch.Tensor, v: torch.Tensor, w: torch.Tensor, u: torch.Tensor,
                 state: Optional[State] = None, *, out_dtype: Optional[torch.dtype] = None,
                 out: Optional[torch.Tensor] = None, state_out: Optional[State] = None,
                 return_state: bool = True, seg_tokens: int = 0, buffer: Optional[torch.Tensor] = None):
    """WKV over a sequence whose k, v (and out) live in host memory: k, v, out
    are CPU tensors [B, T, C] (page-locked, e.g. ``.pin_memory()``, for the
    copies to overlap the compute); w, u and the states are CUDA tensors as for
    ``forward``. The library streams segments of seg_tokens tokens (0 =
    choose) through the device, copies in, compute and copies back of
    neighbouring segments side by side. Returns (out, state) like ``forward``;
    the work is queued on the current stream (synchronise before reading out).
    """
    for t, name in ((k, "k"), (v, "v")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU tensor")
    if v.dtype != k.dtype or k.dim() != 3 or v.shape != k.shape:
        raise ValueError("k and v must both be [B, T, C] of one dtype")
    _need_cuda(w, "w", torch.float32)
    _need_cuda(u, "u", torch.float32)
    B, T, C = k.shape
    if w.shape != (C,) or u.shape != (C,):
        raise ValueError("w and u must be [C]")
    dev = w.device
    out_dtype = out_dtype or k.dtype
    if out is None:
        out = torch.empty((B, T, C), dtype=out_dtype, pin_memory=True)
    if out.is_cuda or not out.is_contiguous() or out.shape != (B, T, C) or out.dtype != out_dtype:
        raise ValueError("out must be a contiguous CPU tensor [B, T, C] of out_dtype")
    sin = None
    if state is not None:
        for i, x in enumerate(state):
            _need_cuda(x, f"state[{i}]", torch.float32)
            if x.shape != (B, C):
                raise ValueError("state arrays must be [B, C]")
        sin = _abi.wkv_cstate(*(x.data_ptr() for x in state))
    sout = None
    if return_state or state_out is not None:
        if state_out is None:
            state_out = tuple(torch.empty((B, C), dtype=torch.float32, device=dev) for _ in range(3))
        for i, x in enumerate(state_out):
            _need_cuda(x, f"state_out[{i}]", torch.float32)
        sout = _abi.wkv_state(*(x.data_ptr() for x in state_out))
    L = _abi.lib()
    kvc, oc = _dtype_code(k, "k"), _dtype_code(out, "out")
    need = L.wkv_forward_host_buffer_size(B, T, C, kvc, oc, int(seg_tokens))
    if need == 0:
        raise ValueError("invalid sizes")
    if buffer is None:
        key = (dev.index, torch.cuda.current_stream(dev).cuda_stream)
        buffer = _host_buffers.get(key)
        if buffer is None or buffer.numel() < need:
            buffer = torch.zeros(need, dtype=torch.uint8, device=dev)
            _host_buffers[key] = buffer
    _need_cuda(buffer, "buffer")
    code = L.wkv_forward_host(B, T, C, _ptr(k), _ptr(v), kvc, _ptr(w), _ptr(u), _ptr(out), oc,
                              ctypes.byref(sin) if sin is not None else None,
                              ctypes.byref(sout) if sout is not None else None,
                              _ptr(buffer), buffer.numel(), int(seg_tokens), _stream())
    _abi.check(code, "wkv_forward_host")
    return out, state_out


def forward_host_buffer_size(B: int, T: int, C: int, kv_dtype: torch.dtype = torch.float32,
                             out_dtype: Optional[torch.dtype] = None, seg_tokens: int = 0) -> int:
    """Bytes of the device buffer ``forward_host`` needs (host-only)."""
    out_dtype = out_dtype or kv_dtype
    return int(_abi.lib().wkv_forward_host_buffer_size(int(B), int(T), int(C), _DT[kv_dtype], _DT[out_dtype],
                                                       int(seg_tokens)))


def step(state: State, k: torch.Tensor, v: torch.Tensor, w: Optional[torch.Tensor], u: torch.Tensor, *,
         out_dtype: Optional[torch.dtype] = None, out: Optional[torch.Tensor] = None,
         state_out: Optional[State] = None, inplace: bool = False,
         w_t: Optional[torch.Tensor] = None, r: Optional[torch.Tensor] = None):
    """One decode token for S streams. k, v: [S, C]; state: (num, den, max_e) [S, C].

    Returns (out [S, C], new state). With ``inplace=True`` the state tensors
    are updated in place and returned. w_t: optional float32 [S, C] decays of
    this token in place of w; r: optional receptance [S, C] (out = sigmoid(r) wkv).
    """
    _need_cuda(k, "k")
    _need_cuda(v, "v", k.dtype)
    if w_t is None or w is not None:
        _need_cuda(w, "w", torch.float32)
    _need_cuda(u, "u", torch.float32)
    if k.dim() != 2 or v.shape != k.shape:
        raise ValueError("k and v must both be [S, C]")
    S, C = k.shape
    ext = _ext(w_t, r, (S, C), k.dtype)
    for i, s in enumerate(state):
        _need_cuda(s, f"state[{i}]", torch.float32)
        if s.shape != (S, C):
            raise ValueError("state arrays must be [S, C]")
    out_dtype = out_dtype or k.dtype
    if out is None:
        out = torch.empty((S, C), dtype=out_dtype, device=k.device)
    _need_cuda(out, "out", out_dtype)
    if inplace:
        state_out = state
    elif state_out is None:
        state_out = tuple(torch.empty_like(s) for s in state)
    sin = _abi.wkv_cstate(*(s.data_ptr() for s in state))
    sout = _abi.wkv_state(*(s.data_ptr() for s in state_out))
    code = _abi.lib().wkv_step_ext(S, C, _ptr(k), _ptr(v), _dtype_code(k, "k"), _ptr(w), _ptr(u),
                                   _ptr(out), _dtype_code(out, "out"), ctypes.byref(sin),
                                   ctypes.byref(sout), _stream(), ctypes.byref(ext) if ext is not None else None)
    _abi.check(code, "wkv_step")
    return out, state_out


def backward(k: torch.Tensor, v: torch.Tensor, w: torch.Tensor, u: torch.Tensor, gout: torch.Tensor,
             state: Optional[State] = None, *, need_state_grad: bool = True,
             workspace: Optional[torch.Tensor] = None):
    """Gradients of a loss with dL/d wkv = gout [B, T, C] (float32).

    Returns (dk, dv, dw, du, dstate): dk, dv float32 [B, T, C]; dw, du float32
    [C] summed over the batch; dstate the gradients of (num, den, max_e) of
    ``state`` (zeros without one), or None if not needed.
    """
    _need_cuda(k, "k")
    _need_cuda(v, "v", k.dtype)
    _need_cuda(w, "w", torch.float32)
    _need_cuda(u, "u", torch.float32)
    _need_cuda(gout, "gout", torch.float32)
    if k.dim() != 3 or v.shape != k.shape or gout.shape != k.shape:
        raise ValueError("k, v and gout must be [B, T, C]")
    B, T, C = k.shape
    dev = k.device
    dk = torch.empty((B, T, C), dtype=torch.float32, device=dev)
    dv = torch.empty_like(dk)
    dw = torch.empty(C, dtype=torch.float32, device=dev)
    du = torch.empty_like(dw)
    sin = None
    if state is not None:
        for i, s in enumerate(state):
            _need_cuda(s, f"state[{i}]", torch.float32)
        sin = _abi.wkv_cstate(*(s.data_ptr() for s in state))
    dstate = None
    dsout = None
    if need_state_grad:
        dstate = tuple(torch.empty((B, C), dtype=torch.float32, device=dev) for _ in range(3))
        dsout = _abi.wkv_state(*(s.data_ptr() for s in dstate))
    need = _abi.lib().wkv_backward_workspace_size(B, T, C)
    if need == 0:
        raise ValueError("invalid sizes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _need_cuda(workspace, "workspace")
    code = _abi.lib().wkv_backward(
        B, T, C, _ptr(k), _ptr(v), _dtype_code(k, "k"), _ptr(w), _ptr(u),
        ctypes.byref(sin) if sin is not None else None, _ptr(gout), _ptr(dk), _ptr(dv), _ptr(dw), _ptr(du),
        ctypes.byref(dsout) if dsout is not None else None, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream())
    _abi.check(code, "wkv_backward")
    return dk, dv, dw, du, dstate


def v6_forward(r: torch.Tensor, w: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
               state: Optional[torch.Tensor] = None, *, out_dtype: Optional[torch.dtype] = None,
               out: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
               return_state: bool = True, workspace: Optional[torch.Tensor] = None):
    """The RWKV-v6 matrix-valued state over a sequence: r, k, v [B, T, H, D]
    (float32 or bfloat16), w [B, T, H, D] float32 decay factors; state
    [B, H, D, D] float32 or None. Returns (y [B, T, H, D], state after the
    last token or None)."""
    _need_cuda(k, "k")
    _need_cuda(v, "v", k.dtype)
    _need_cuda(r, "r", k.dtype)
    _need_cuda(w, "w", torch.float32)
    if k.dim() != 4 or v.shape != k.shape or r.shape != k.shape or w.shape != k.shape:
        raise ValueError("r, w, k, v must all be [B, T, H, D]")
    B, T, H, D = k.shape
    out_dtype = out_dtype or k.dtype
    if out is None:
        out = torch.empty((B, T, H, D), dtype=out_dtype, device=k.device)
    _need_cuda(out, "out", out_dtype)
    if state is not None:
        _need_cuda(state, "state", torch.float32)
        if state.shape != (B, H, D, D):
            raise ValueError("state must be [B, H, D, D]")
    if return_state and state_out is None:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=k.device)
    if state_out is not None:
        _need_cuda(state_out, "state_out", torch.float32)
    if workspace is None:
        workspace = _default_workspace(256, k.device)
    code = _abi.lib().wkv_v6_forward(B, T, H, D, _ptr(r), _ptr(w), _ptr(k), _ptr(v), _dtype_code(k, "k"), _ptr(out),
                                   _dtype_code(out, "out"), _ptr(state), _ptr(state_out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream())
    _abi.check(code, "wkv_v6_forward")
    return out, state_out


class WKV(torch.autograd.Function):
    """The operator as a torch autograd function: forward through wkv_forward,
    backward through wkv_backward (per-channel w, float32 or bfloat16 k and v,
    gradients in float32). ``WKV.apply(k, v, w, u)`` returns wkv [B, T, C]."""

    @staticmethod
    def forward(ctx, k, v, w, u):
        out, _ = forward(k, v, w, u, return_state=False)
        ctx.save_for_backward(k, v, w, u)
        return out

    @staticmethod
    def backward(ctx, gout):
        k, v, w, u = ctx.saved_tensors
        dk, dv, dw, du, _ = backward(k, v, w, u, gout.float().contiguous(), need_state_grad=False)
        return dk.to(k.dtype), dv.to(v.dtype), dw, du


def query_status(workspace: torch.Tensor) -> int:
    """Synchronise the current stream; return and clear the device-side status of a workspace."""
    return int(_abi.lib().wkv_query_status(_ptr(workspace), _stream()))


def empty_state(B: int, C: int, device=None) -> State:
    """The empty state (0, 0, -inf) as three float32 [B, C] tensors."""
    dev = device if device is not None else torch.device("cuda")
    return (torch.zeros(B, C, device=dev), torch.zeros(B, C, device=dev),
            torch.full((B, C), float("-inf"), device=dev))


class PreparedForward:
    """``forward`` with its arguments checked and marshalled once.

    For loops that call the operator on the same buffers again and again
    (benchmarks, decode loops, CUDA-graph capture): ``__call__`` is a single
    C-ABI call with the stored pointers, on the stream current at preparation
    time unless another is passed.
    """

    def __init__(self, k, v, w, u, state=None, *, out, state_out=None, workspace=None,
                 options: Optional[dict] = None, w_t=None, r=None):
        _need_cuda(k, "k")
        _need_cuda(v, "v", k.dtype)
        if w_t is None or w is not None:
            _need_cuda(w, "w", torch.float32)
        _need_cuda(u, "u", torch.float32)
        B, T, C = k.shape
        if v.shape != k.shape or (w is not None and w.shape != (C,)) or u.shape != (C,) or out.shape != k.shape:
            raise ValueError("shapes must be k, v, out [B, T, C] and w, u [C]")
        _need_cuda(out, "out")
        self._ext = _ext(w_t, r, (B, T, C), k.dtype)
        self._keep = [k, v, w, u, out, w_t, r]
        self._sin = self._sout = None
        if state is not None:
            for i, s in enumerate(state):
                _need_cuda(s, f"state[{i}]", torch.float32)
            self._sin = _abi.wkv_cstate(*(s.data_ptr() for s in state))
            self._keep += list(state)
        if state_out is not None:
            for i, s in enumerate(state_out):
                _need_cuda(s, f"state_out[{i}]", torch.float32)
            self._sout = _abi.wkv_state(*(s.data_ptr() for s in state_out))
            self._keep += list(state_out)
        self._opts_struct = None
        if options:
            self._opts_struct = _abi.wkv_options()
            for key, val in options.items():
                setattr(self._opts_struct, key, int(val))
        opts = ctypes.byref(self._opts_struct) if self._opts_struct is not None else None
        need = _abi.lib().wkv_forward_workspace_size(B, T, C, opts)
        if need == 0:
            raise ValueError("invalid sizes or options")
        if workspace is None:
            workspace = make_workspace(B, T, C, options, device=k.device)
        _need_cuda(workspace, "workspace")
        self.workspace = workspace
        self._keep.append(workspace)
        self._fn = _abi.lib().wkv_forward_ext
        self._args = (B, T, C, _ptr(k), _ptr(v), _dtype_code(k, "k"), _ptr(w), _ptr(u), _ptr(out),
                      _dtype_code(out, "out"),
                      ctypes.byref(self._sin) if self._sin is not None else None,
                      ctypes.byref(self._sout) if self._sout is not None else None,
                      _ptr(workspace), workspace.numel() * workspace.element_size())
        self._stream = _stream()
        self._opts = opts
        self._ext_ref = ctypes.byref(self._ext) if self._ext is not None else None

    def __call__(self, stream=None) -> None:
        code = self._fn(*self._args, self._stream if stream is None else stream, self._opts, self._ext_ref)
        if code:
            _abi.check(code, "wkv_forward")


class PreparedStep:
    """``step`` with its arguments checked and marshalled once (see PreparedForward)."""

    def __init__(self, state, k, v, w, u, *, out, state_out=None):
        _need_cuda(k, "k")
        _need_cuda(v, "v", k.dtype)
        _need_cuda(w, "w", torch.float32)
        _need_cuda(u, "u", torch.float32)
        _need_cuda(out, "out")
        S, C = k.shape
        state_out = state if state_out is None else state_out
        for i, s in enumerate(tuple(state) + tuple(state_out)):
            _need_cuda(s, f"state[{i}]", torch.float32)
            if s.shape != (S, C):
                raise ValueError("state arrays must be [S, C]")
        self._keep = [k, v, w, u, out, *state, *state_out]
        self._sin = _abi.wkv_cstate(*(s.data_ptr() for s in state))
        self._sout = _abi.wkv_state(*(s.data_ptr() for s in state_out))
        self._fn = _abi.lib().wkv_step
        self._args = (S, C, _ptr(k), _ptr(v), _dtype_code(k, "k"), _ptr(w), _ptr(u), _ptr(out),
                      _dtype_code(out, "out"), ctypes.byref(self._sin), ctypes.byref(self._sout))
        self._stream = _stream()

    def __call__(self, stream=None) -> None:
        code = self._fn(*self._args, self._stream if stream is None else stream)
        if code:
            _abi.check(code, "wkv_step")
