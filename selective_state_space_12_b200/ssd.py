"""Python binding of libssd with the C ABI's names (argument marshalling only).

Tensors are PyTorch CUDA tensors; PyTorch supplies device memory and streams.
Every step of the layer runs in libssd's kernels. Outputs that the caller
does not pass are allocated with torch; the forward's workspace is taken from
torch's caching allocator unless the caller passes one, so that repeated calls
do not allocate inside the library.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _lib

_DTYPES = {torch.float32: _lib.SSD_F32, torch.bfloat16: _lib.SSD_BF16}
CHUNKS = (16, 32, 64, 128, 256)


class SSDError(RuntimeError):
    """A non-OK libssd status, with the library's message."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.STATUS_NAMES.get(status, status)}: {_lib.last_error()}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream: Optional[torch.cuda.Stream], device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def make_dims(batch, seqlen, nheads, headdim, dstate, ngroups, dtype) -> _lib.Dims:
    if isinstance(dtype, torch.dtype):
        if dtype not in _DTYPES:
            raise TypeError(f"unsupported I/O dtype {dtype}; use float32 or bfloat16")
        dtype = _DTYPES[dtype]
    return _lib.Dims(int(batch), int(seqlen), int(nheads), int(headdim), int(dstate),
                     int(ngroups), int(dtype), 0)


def _check_tensor(name, t, shape, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def ssd_forward_workspace_size(dims: _lib.Dims, chunk: int) -> int:
    return int(_lib.load().ssd_forward_workspace_size(ctypes.byref(dims), int(chunk)))


def ssd_forward(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                C: torch.Tensor, D: Optional[torch.Tensor] = None,
                h0: Optional[torch.Tensor] = None, chunk: int = 256,
                y: Optional[torch.Tensor] = None, h_final: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, want_final: bool = True,
                stream: Optional[torch.cuda.Stream] = None
                ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """y, h_final = SSD(x, dt, A, B, C, D, h0) by the chunked algorithm.

    x (b,L,H,P), dt (b,L,H), B/C (b,L,G,N) share one dtype (float32 or
    bfloat16); A, D (H,) and h0, h_final (b,H,P,N) are float32."""
    lib = _lib.load()
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev, io = x.device, x.dtype
    _check_tensor("x", x, (batch, L, H, P), io, dev)
    _check_tensor("dt", dt, (batch, L, H), io, dev)
    _check_tensor("A", A, (H,), torch.float32, dev)
    _check_tensor("B", B, (batch, L, G, N), io, dev)
    _check_tensor("C", C, (batch, L, G, N), io, dev)
    if D is not None:
        _check_tensor("D", D, (H,), torch.float32, dev)
    if h0 is not None:
        _check_tensor("h0", h0, (batch, H, P, N), torch.float32, dev)
    dims = make_dims(batch, L, H, P, N, G, io)
    if y is None:
        y = torch.empty_like(x)
    _check_tensor("y", y, (batch, L, H, P), io, dev)
    if h_final is None and want_final:
        h_final = torch.empty((batch, H, P, N), dtype=torch.float32, device=dev)
    if h_final is not None:
        _check_tensor("h_final", h_final, (batch, H, P, N), torch.float32, dev)
    ws_bytes = ssd_forward_workspace_size(dims, chunk)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_given = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib.ssd_forward(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(h0),
                             int(chunk), _ptr(y), _ptr(h_final), ctypes.byref(dims),
                             _ptr(workspace), ws_given, _stream_handle(stream, dev))
    if st != _lib.SSD_OK:
        raise SSDError(st, "ssd_forward")
    return y, h_final


def make_options(dt_bias: Optional[torch.Tensor] = None, dt_softplus: bool = False,
                 dt_limit: Optional[Tuple[float, float]] = None,
                 zoh: bool = False) -> _lib.Options:
    """struct ssd_options: the raw step dt -> dt + dt_bias[h] -> softplus ->
    clamp to dt_limit = (dt_min, dt_max); input weight dt, or with ``zoh`` the
    zero-order hold (exp(dt A) - 1) / A. dt_bias is a float32 (H,) CUDA tensor."""
    o = _lib.Options()
    o.dt_bias = _ptr(dt_bias)
    o.dt_softplus = 1 if dt_softplus else 0
    o.discretization = _lib.SSD_DISC_ZOH if zoh else _lib.SSD_DISC_EULER
    if dt_limit is not None:
        o.dt_min, o.dt_max = float(dt_limit[0]), float(dt_limit[1])
    return o


def ssd_forward_ex(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                   C: torch.Tensor, D: Optional[torch.Tensor] = None,
                   h0: Optional[torch.Tensor] = None, chunk: int = 256,
                   dt_bias: Optional[torch.Tensor] = None, dt_softplus: bool = False,
                   dt_limit: Optional[Tuple[float, float]] = None, zoh: bool = False,
                   y: Optional[torch.Tensor] = None, h_final: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, want_final: bool = True,
                   stream: Optional[torch.cuda.Stream] = None
                   ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """ssd_forward on RAW steps dt, prepared in the kernels by the step options
    (see make_options)."""
    lib = _lib.load()
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev, io = x.device, x.dtype
    _check_tensor("x", x, (batch, L, H, P), io, dev)
    _check_tensor("dt", dt, (batch, L, H), io, dev)
    _check_tensor("A", A, (H,), torch.float32, dev)
    _check_tensor("B", B, (batch, L, G, N), io, dev)
    _check_tensor("C", C, (batch, L, G, N), io, dev)
    if D is not None:
        _check_tensor("D", D, (H,), torch.float32, dev)
    if h0 is not None:
        _check_tensor("h0", h0, (batch, H, P, N), torch.float32, dev)
    if dt_bias is not None:
        _check_tensor("dt_bias", dt_bias, (H,), torch.float32, dev)
    dims = make_dims(batch, L, H, P, N, G, io)
    opts = make_options(dt_bias, dt_softplus, dt_limit, zoh)
    if y is None:
        y = torch.empty_like(x)
    _check_tensor("y", y, (batch, L, H, P), io, dev)
    if h_final is None and want_final:
        h_final = torch.empty((batch, H, P, N), dtype=torch.float32, device=dev)
    if h_final is not None:
        _check_tensor("h_final", h_final, (batch, H, P, N), torch.float32, dev)
    ws_bytes = ssd_forward_workspace_size(dims, chunk)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ws_given = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib.ssd_forward_ex(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(h0), int(chunk), _ptr(y), _ptr(h_final),
                                ctypes.byref(dims), ctypes.byref(opts), _ptr(workspace),
                                ws_given, _stream_handle(stream, dev))
    if st != _lib.SSD_OK:
        raise SSDError(st, "ssd_forward_ex")
    return y, h_final


def ssd_step_ex(h: torch.Tensor, x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor,
                B: torch.Tensor, C: torch.Tensor, D: Optional[torch.Tensor] = None,
                dt_bias: Optional[torch.Tensor] = None, dt_softplus: bool = False,
                dt_limit: Optional[Tuple[float, float]] = None, zoh: bool = False,
                y: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """ssd_step on a RAW step dt (b,H) with the step options (see make_options)."""
    lib = _lib.load()
    batch, H, P, N = h.shape
    G = B.shape[1]
    dev, io = x.device, x.dtype
    _check_tensor("h", h, (batch, H, P, N), torch.float32, dev)
    _check_tensor("x", x, (batch, H, P), io, dev)
    _check_tensor("dt", dt, (batch, H), io, dev)
    _check_tensor("A", A, (H,), torch.float32, dev)
    _check_tensor("B", B, (batch, G, N), io, dev)
    _check_tensor("C", C, (batch, G, N), io, dev)
    if D is not None:
        _check_tensor("D", D, (H,), torch.float32, dev)
    if dt_bias is not None:
        _check_tensor("dt_bias", dt_bias, (H,), torch.float32, dev)
    if y is None:
        y = torch.empty_like(x)
    _check_tensor("y", y, (batch, H, P), io, dev)
    dims = make_dims(batch, 1, H, P, N, G, io)
    opts = make_options(dt_bias, dt_softplus, dt_limit, zoh)
    with torch.cuda.device(dev):
        st = lib.ssd_step_ex(_ptr(h), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                             _ptr(y), ctypes.byref(dims), ctypes.byref(opts),
                             _stream_handle(stream, dev))
    if st != _lib.SSD_OK:
        raise SSDError(st, "ssd_step_ex")
    return y


def ssd_forward_state(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                      chunk: int = 256, dt_bias: Optional[torch.Tensor] = None,
                      dt_softplus: bool = False, dt_limit: Optional[Tuple[float, float]] = None,
                      zoh: bool = False, state_out: Optional[torch.Tensor] = None,
                      decay_out: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None
                      ) -> Tuple[torch.Tensor, torch.Tensor]:
    """(end state (b,H,P,N), total decay (b,H)) of each lane's sequence from a
    zero initial state: the local step of sequence parallelism. dt is raw when
    step options are given (as for ssd_forward_ex)."""
    lib = _lib.load()
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev, io = x.device, x.dtype
    _check_tensor("x", x, (batch, L, H, P), io, dev)
    _check_tensor("dt", dt, (batch, L, H), io, dev)
    _check_tensor("A", A, (H,), torch.float32, dev)
    _check_tensor("B", B, (batch, L, G, N), io, dev)
    if dt_bias is not None:
        _check_tensor("dt_bias", dt_bias, (H,), torch.float32, dev)
    if state_out is None:
        state_out = torch.empty((batch, H, P, N), dtype=torch.float32, device=dev)
    if decay_out is None:
        decay_out = torch.empty((batch, H), dtype=torch.float32, device=dev)
    _check_tensor("state_out", state_out, (batch, H, P, N), torch.float32, dev)
    _check_tensor("decay_out", decay_out, (batch, H), torch.float32, dev)
    dims = make_dims(batch, L, H, P, N, G, io)
    opts = make_options(dt_bias, dt_softplus, dt_limit, zoh)
    need = int(lib.ssd_forward_state_workspace_size(ctypes.byref(dims), int(chunk)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_given = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib.ssd_forward_state(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), int(chunk),
                                   _ptr(state_out), _ptr(decay_out), ctypes.byref(dims),
                                   ctypes.byref(opts), _ptr(workspace), ws_given,
                                   _stream_handle(stream, dev))
    if st != _lib.SSD_OK:
        raise SSDError(st, "ssd_forward_state")
    return state_out, decay_out


def ssd_state_chain(states: torch.Tensor, decays: torch.Tensor, part: int,
                    h0: Optional[torch.Tensor] = None, h_in: Optional[torch.Tensor] = None,
                    want_total: bool = False,
                    stream: Optional[torch.cuda.Stream] = None
                    ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """(h_in, h_total): the state entering piece ``part`` from the pieces' end
    states (R,b,H,P,N) and decays (R,b,H), and (want_total) the chain over all
    pieces."""
    lib = _lib.load()
    R, batch, H, P, N = states.shape
    dev = states.device
    _check_tensor("states", states, (R, batch, H, P, N), torch.float32, dev)
    _check_tensor("decays", decays, (R, batch, H), torch.float32, dev)
    if h0 is not None:
        _check_tensor("h0", h0, (batch, H, P, N), torch.float32, dev)
    if h_in is None:
        h_in = torch.empty((batch, H, P, N), dtype=torch.float32, device=dev)
    _check_tensor("h_in", h_in, (batch, H, P, N), torch.float32, dev)
    h_total = torch.empty_like(h_in) if want_total else None
    dims = make_dims(batch, 0, H, P, N, 1, torch.float32)
    with torch.cuda.device(dev):
        st = lib.ssd_state_chain(_ptr(states), _ptr(decays), int(R), int(part), _ptr(h0),
                                 _ptr(h_in), _ptr(h_total), ctypes.byref(dims),
                                 _stream_handle(stream, dev))
    if st != _lib.SSD_OK:
        raise SSDError(st, "ssd_state_chain")
    return h_in, h_total


def ssd_selective_scan(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                       C: torch.Tensor, Dskip: Optional[torch.Tensor] = None,
                       h0: Optional[torch.Tensor] = None,
                       dt_bias: Optional[torch.Tensor] = None, dt_softplus: bool = False,
                       dt_limit: Optional[Tuple[float, float]] = None, zoh: bool = False,
                       y: Optional[torch.Tensor] = None, h_final: Optional[torch.Tensor] = None,
                       want_final: bool = True, stream: Optional[torch.cuda.Stream] = None
                       ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """The selective scan with a diagonal A per channel: x, dt (b,L,D), A (D,N),
    B/C (b,L,G,N), Dskip (D,), h0/h_final (b,D,N); step options as for
    ssd_forward_ex (dt_bias per channel)."""
    lib = _lib.load()
    batch, L, Dc = x.shape
    N = A.shape[1]
    G = B.shape[2]
    dev, io = x.device, x.dtype
    _check_tensor("x", x, (batch, L, Dc), io, dev)
    _check_tensor("dt", dt, (batch, L, Dc), io, dev)
    _check_tensor("A", A, (Dc, N), torch.float32, dev)
    _check_tensor("B", B, (batch, L, G, N), io, dev)
    _check_tensor("C", C, (batch, L, G, N), io, dev)
    if Dskip is not None:
        _check_tensor("Dskip", Dskip, (Dc,), torch.float32, dev)
    if h0 is not None:
        _check_tensor("h0", h0, (batch, Dc, N), torch.float32, dev)
    if dt_bias is not None:
        _check_tensor("dt_bias", dt_bias, (Dc,), torch.float32, dev)
    if y is None:
        y = torch.empty_like(x)
    _check_tensor("y", y, (batch, L, Dc), io, dev)
    if h_final is None and want_final:
        h_final = torch.empty((batch, Dc, N), dtype=torch.float32, device=dev)
    if h_final is not None:
        _check_tensor("h_final", h_final, (batch, Dc, N), torch.float32, dev)
    dims = make_dims(batch, L, Dc, 1, N, G, io)
    opts = make_options(dt_bias, dt_softplus, dt_limit, zoh)
    with torch.cuda.device(dev):
        st = lib.ssd_selective_scan(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(Dskip),
                                    _ptr(h0), _ptr(y), _ptr(h_final), ctypes.byref(dims),
                                    ctypes.byref(opts), _stream_handle(stream, dev))
    if st != _lib.SSD_OK:
        raise SSDError(st, "ssd_selective_scan")
    return y, h_final


def ssd_backward(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                 C: torch.Tensor, D: Optional[torch.Tensor], h0: Optional[torch.Tensor],
                 dy: torch.Tensor, dh_final: Optional[torch.Tensor] = None,
                 want_dh0: bool = True, workspace: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None) -> dict:
    """Gradients of sum dy . y + sum dh_final . h_final for ssd_forward's
    plain layer: a dict of fp32 tensors dx, ddt, dA, dB, dC, dD, dh0."""
    lib = _lib.load()
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev, io = x.device, x.dtype
    for name, t, shape, dtype in (("x", x, (batch, L, H, P), io), ("dt", dt, (batch, L, H), io),
                                  ("A", A, (H,), torch.float32),
                                  ("B", B, (batch, L, G, N), io), ("C", C, (batch, L, G, N), io),
                                  ("dy", dy, (batch, L, H, P), io)):
        _check_tensor(name, t, shape, dtype, dev)
    if D is not None:
        _check_tensor("D", D, (H,), torch.float32, dev)
    for name, t in (("h0", h0), ("dh_final", dh_final)):
        if t is not None:
            _check_tensor(name, t, (batch, H, P, N), torch.float32, dev)
    f = dict(dtype=torch.float32, device=dev)
    out = dict(dx=torch.empty((batch, L, H, P), **f), ddt=torch.empty((batch, L, H), **f),
               dA=torch.empty((H,), **f), dB=torch.empty((batch, L, G, N), **f),
               dC=torch.empty((batch, L, G, N), **f), dD=torch.empty((H,), **f),
               dh0=torch.empty((batch, H, P, N), **f) if want_dh0 else None)
    dims = make_dims(batch, L, H, P, N, G, io)
    need = int(lib.ssd_backward_workspace_size(ctypes.byref(dims)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_given = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib.ssd_backward(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(h0),
                              _ptr(dy), _ptr(dh_final), _ptr(out["dx"]), _ptr(out["ddt"]),
                              _ptr(out["dA"]), _ptr(out["dB"]), _ptr(out["dC"]),
                              _ptr(out["dD"]), _ptr(out["dh0"]), ctypes.byref(dims),
                              _ptr(workspace), ws_given, _stream_handle(stream, dev))
    if st != _lib.SSD_OK:
        raise SSDError(st, "ssd_backward")
    return out


def ssd_step(h: torch.Tensor, x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor,
             B: torch.Tensor, C: torch.Tensor, D: Optional[torch.Tensor] = None,
             y: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """One decode step: updates h (b,H,P,N) float32 in place, returns y (b,H,P)."""
    lib = _lib.load()
    batch, H, P, N = h.shape
    G = B.shape[1]
    dev, io = x.device, x.dtype
    _check_tensor("h", h, (batch, H, P, N), torch.float32, dev)
    _check_tensor("x", x, (batch, H, P), io, dev)
    _check_tensor("dt", dt, (batch, H), io, dev)
    _check_tensor("A", A, (H,), torch.float32, dev)
    _check_tensor("B", B, (batch, G, N), io, dev)
    _check_tensor("C", C, (batch, G, N), io, dev)
    if D is not None:
        _check_tensor("D", D, (H,), torch.float32, dev)
    if y is None:
        y = torch.empty_like(x)
    _check_tensor("y", y, (batch, H, P), io, dev)
    dims = make_dims(batch, 1, H, P, N, G, io)
    with torch.cuda.device(dev):
        st = lib.ssd_step(_ptr(h), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                          _ptr(y), ctypes.byref(dims), _stream_handle(stream, dev))
    if st != _lib.SSD_OK:
        raise SSDError(st, "ssd_step")
    return y


def ssd_device_status(stream: Optional[torch.cuda.Stream] = None,
                      device: Optional[torch.device] = None) -> int:
    dev = device or torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        return int(_lib.load().ssd_device_status(_stream_handle(stream, dev)))


def ssd_last_error() -> str:
    return _lib.last_error()


def ssd_set_wait_limit(cycles: int) -> None:
    """Bound, in SM clock cycles, on each pipelined wait of the forward
    kernels launched after the call (0 restores the default of about 2 s)."""
    _lib.load().ssd_set_wait_limit(int(cycles))


def ssd_abi_version() -> int:
    return int(_lib.load().ssd_abi_version())


class PreparedCall:
    """A libssd call with its arguments marshalled once (validation included),
    for loops that repeat the same call on the same buffers: each invocation
    is exactly one call of the C entry point on the captured stream."""

    def __init__(self, fn, args, where):
        self._fn, self._args, self._where = fn, args, where

    def __call__(self) -> None:
        st = self._fn(*self._args)
        if st != _lib.SSD_OK:
            raise SSDError(st, self._where)


def prepare_forward(x, dt, A, B, C, D, h0, chunk, y, h_final, workspace,
                    stream: Optional[torch.cuda.Stream] = None,
                    options: Optional[_lib.Options] = None) -> PreparedCall:
    """ssd_forward on fixed buffers (all given), validated and marshalled once;
    with ``options`` (make_options), ssd_forward_ex on raw steps dt."""
    lib = _lib.load()
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev, io = x.device, x.dtype
    for name, t, shape, dtype in (("x", x, (batch, L, H, P), io), ("dt", dt, (batch, L, H), io),
                                  ("A", A, (H,), torch.float32),
                                  ("B", B, (batch, L, G, N), io), ("C", C, (batch, L, G, N), io),
                                  ("y", y, (batch, L, H, P), io)):
        _check_tensor(name, t, shape, dtype, dev)
    if D is not None:
        _check_tensor("D", D, (H,), torch.float32, dev)
    for name, t in (("h0", h0), ("h_final", h_final)):
        if t is not None:
            _check_tensor(name, t, (batch, H, P, N), torch.float32, dev)
    dims = make_dims(batch, L, H, P, N, G, io)
    need = ssd_forward_workspace_size(dims, chunk)
    ws_given = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if need > 0 and (workspace is None or ws_given < need):
        raise ValueError(f"workspace of {ws_given} bytes given, {need} needed")
    head = (_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(h0), int(chunk),
            _ptr(y), _ptr(h_final), ctypes.byref(dims))
    tail = (_ptr(workspace), ws_given, _stream_handle(stream, dev))
    if options is None:
        call = PreparedCall(lib.ssd_forward, head + tail, "ssd_forward")
    else:
        call = PreparedCall(lib.ssd_forward_ex, head + (ctypes.byref(options),) + tail,
                            "ssd_forward_ex")
    call._keep = (dims, options, x, dt, A, B, C, D, h0, y, h_final, workspace)
    return call


def prepare_step(h, x, dt, A, B, C, D, y,
                 stream: Optional[torch.cuda.Stream] = None,
                 options: Optional[_lib.Options] = None) -> PreparedCall:
    """ssd_step on fixed buffers, validated and marshalled once; with
    ``options`` (make_options), ssd_step_ex on a raw step dt."""
    lib = _lib.load()
    batch, H, P, N = h.shape
    G = B.shape[1]
    dev, io = x.device, x.dtype
    for name, t, shape, dtype in (("h", h, (batch, H, P, N), torch.float32),
                                  ("x", x, (batch, H, P), io), ("dt", dt, (batch, H), io),
                                  ("A", A, (H,), torch.float32), ("B", B, (batch, G, N), io),
                                  ("C", C, (batch, G, N), io), ("y", y, (batch, H, P), io)):
        _check_tensor(name, t, shape, dtype, dev)
    if D is not None:
        _check_tensor("D", D, (H,), torch.float32, dev)
    dims = make_dims(batch, 1, H, P, N, G, io)
    head = (_ptr(h), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y),
            ctypes.byref(dims))
    if options is None:
        call = PreparedCall(lib.ssd_step, head + (_stream_handle(stream, dev),), "ssd_step")
    else:
        call = PreparedCall(lib.ssd_step_ex,
                            head + (ctypes.byref(options), _stream_handle(stream, dev)),
                            "ssd_step_ex")
    call._keep = (dims, options, h, x, dt, A, B, C, D, y)
    return call


def launch_count() -> int:
    """Kernels libssd has launched in this process."""
    return int(_lib.load().ssd_launch_count())


def profile_begin() -> None:
    st = _lib.load().ssd_profile_begin()
    if st != _lib.SSD_OK:
        raise SSDError(st, "ssd_profile_begin")


def profile_end(max_entries: int = 64):
    """{kernel name: (launches, total_ms)} for the closed window."""
    arr = (_lib.KernelTime * max_entries)()
    n = _lib.load().ssd_profile_end(arr, max_entries)
    if n < 0:
        raise SSDError(_lib.SSD_ERR_CUDA, "ssd_profile_end")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(n)}


class HostForward:
    """The forward from pinned host buffers to pinned host buffers.

    The batch is cut into ``splits`` slices; each slice's host->device
    copies, its forward (ssd_forward, the library's kernels) and its
    device->host copies go to three streams chained by events, so that the
    upload of slice i + 1 and the download of slice i overlap (both PCIe
    directions busy) and the forward runs between them. Device buffers and
    the workspace are allocated once for the given sizes.

    Call with the host tensors of one step; returns the event that marks the
    last download. The calling stream (``stream``, default: the current one)
    is made to wait for it, so work queued on it afterwards sees the results.
    """

    def __init__(self, batch: int, seqlen: int, nheads: int, headdim: int, dstate: int,
                 ngroups: int, dtype: torch.dtype, chunk: int = 256, splits: int = 4,
                 h0: bool = False, want_final: bool = True, device=None):
        dev = torch.device(device) if device is not None else torch.device("cuda")
        self.dev, self.chunk, self.h0 = dev, int(chunk), bool(h0)
        splits = max(1, min(int(splits), int(batch)))
        bounds = [batch * i // splits for i in range(splits + 1)]
        self.slices = [(a, b) for a, b in zip(bounds, bounds[1:]) if b > a]
        H, P, N, G = nheads, headdim, dstate, ngroups
        e = dict(dtype=dtype, device=dev)
        f = dict(dtype=torch.float32, device=dev)
        self.x = torch.empty((batch, seqlen, H, P), **e)
        self.dt = torch.empty((batch, seqlen, H), **e)
        self.B = torch.empty((batch, seqlen, G, N), **e)
        self.C = torch.empty((batch, seqlen, G, N), **e)
        self.y = torch.empty((batch, seqlen, H, P), **e)
        self.A = torch.empty((H,), **f)
        self.D = torch.empty((H,), **f)
        self.h0_d = torch.empty((batch, H, P, N), **f) if h0 else None
        self.hf = torch.empty((batch, H, P, N), **f) if want_final else None
        ws = max(ssd_forward_workspace_size(make_dims(b - a, seqlen, H, P, N, G, dtype), chunk)
                 for a, b in self.slices)
        self.ws = torch.empty(max(ws, 1), dtype=torch.uint8, device=dev)
        self.s_in = torch.cuda.Stream(dev)
        self.s_comp = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.calls = []
        for a, b in self.slices:
            self.calls.append(prepare_forward(
                self.x[a:b], self.dt[a:b], self.A, self.B[a:b], self.C[a:b], self.D,
                None if self.h0_d is None else self.h0_d[a:b], self.chunk, self.y[a:b],
                None if self.hf is None else self.hf[a:b], self.ws, stream=self.s_comp))

    @property
    def h2d_bytes(self) -> int:
        n = sum(t.numel() * t.element_size() for t in (self.x, self.dt, self.B, self.C, self.A,
                                                        self.D))
        return n + (self.h0_d.numel() * 4 if self.h0_d is not None else 0)

    @property
    def d2h_bytes(self) -> int:
        n = self.y.numel() * self.y.element_size()
        return n + (self.hf.numel() * 4 if self.hf is not None else 0)

    def __call__(self, x, dt, A, B, C, D, y_out, hf_out=None, h0=None,
                 stream: Optional[torch.cuda.Stream] = None) -> torch.cuda.Event:
        caller = stream if stream is not None else torch.cuda.current_stream(self.dev)
        start = torch.cuda.Event()
        start.record(caller)
        for s in (self.s_in, self.s_comp, self.s_out):
            s.wait_event(start)
        last = None
        for i, ((a, b), call) in enumerate(zip(self.slices, self.calls)):
            ev_in, ev_fw = torch.cuda.Event(), torch.cuda.Event()
            with torch.cuda.stream(self.s_in):
                if i == 0:
                    self.A.copy_(A, non_blocking=True)
                    self.D.copy_(D, non_blocking=True)
                self.x[a:b].copy_(x[a:b], non_blocking=True)
                self.dt[a:b].copy_(dt[a:b], non_blocking=True)
                self.B[a:b].copy_(B[a:b], non_blocking=True)
                self.C[a:b].copy_(C[a:b], non_blocking=True)
                if self.h0_d is not None:
                    self.h0_d[a:b].copy_(h0[a:b], non_blocking=True)
                ev_in.record(self.s_in)
            self.s_comp.wait_event(ev_in)
            with torch.cuda.device(self.dev):
                call()
            ev_fw.record(self.s_comp)
            self.s_out.wait_event(ev_fw)
            with torch.cuda.stream(self.s_out):
                y_out[a:b].copy_(self.y[a:b], non_blocking=True)
                if hf_out is not None and self.hf is not None:
                    hf_out[a:b].copy_(self.hf[a:b], non_blocking=True)
                last = torch.cuda.Event()
                last.record(self.s_out)
        caller.wait_event(last)
        return last
