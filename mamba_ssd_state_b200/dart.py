"""Python binding of libdart.so (argument marshalling only).

Every computation runs in the library's CUDA kernels; this module checks
tensor shapes/dtypes, allocates outputs and workspaces with PyTorch (device
memory and streams are PyTorch's), and passes raw pointers plus the current
CUDA stream to the C ABI declared in ``include/dart.h``.  The functions carry
the C names.  Inputs given as CPU tensors are copied to the device first and
the results copied back (the host-buffer path), so the same calls serve
device-resident and host-resident data.

There is no fallback: if the library is missing or no CUDA device is present
the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_HERE, "libdart.so")

DART_OK, DART_ERR_INVALID_ARG, DART_ERR_UNSUPPORTED, DART_ERR_CUDA, DART_ERR_TIMEOUT, DART_ERR_DEVICE = range(6)
DART_F32, DART_BF16 = 0, 1
_STATUS = {0: "DART_OK", 1: "DART_ERR_INVALID_ARG", 2: "DART_ERR_UNSUPPORTED", 3: "DART_ERR_CUDA",
           4: "DART_ERR_TIMEOUT", 5: "DART_ERR_DEVICE"}

# every symbol include/dart.h declares
EXPORTS = ("dart_ssd_chunk_scan_workspace_bytes", "dart_ssd_chunk_scan", "dart_sma_forward",
           "dart_decode_step_workspace_bytes", "dart_decode_step", "dart_supported",
           "dart_sync_status", "dart_last_error", "dart_abi_version", "dart_launch_count",
           "dart_sma_impl", "dart_decode_step_noalloc", "dart_sma_decayed_workspace_bytes",
           "dart_sma_forward_decayed", "dart_decode_step_decayed", "dart_decode_memlog_init",
           "dart_decode_step_e4m3", "dart_cache_quantize_e4m3", "dart_sma_backward_workspace_bytes",
           "dart_sma_backward", "dart_ssd_scan_backward_workspace_bytes", "dart_ssd_scan_backward",
           "dart_selftest_wait_timeout")


class DartError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("batch", "seqlen", "nheads", "headdim", "dstate", "chunk", "ngroups")]


_P = ctypes.c_void_p
_lib = None


def load(path: str = LIBRARY) -> ctypes.CDLL:
    """Load libdart.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"{path} not found: build it with `python -m mamba_ssd_state_b200.build`")
    lib = ctypes.CDLL(path)
    D = ctypes.POINTER(Dims)
    lib.dart_ssd_chunk_scan_workspace_bytes.restype = ctypes.c_size_t
    lib.dart_ssd_chunk_scan_workspace_bytes.argtypes = [D, ctypes.c_int]
    lib.dart_ssd_chunk_scan.restype = ctypes.c_int
    lib.dart_ssd_chunk_scan.argtypes = [D, ctypes.c_int] + [_P] * 10 + [ctypes.c_size_t, _P]
    lib.dart_sma_forward.restype = ctypes.c_int
    lib.dart_sma_forward.argtypes = [D, ctypes.c_int] + [_P] * 4 + [ctypes.c_float, _P, _P, _P]
    lib.dart_decode_step_decayed.restype = ctypes.c_int
    lib.dart_decode_step_decayed.argtypes = ([D, ctypes.c_int] + [_P] * 7 + [ctypes.c_float] + [_P] * 3
                                             + [ctypes.c_int] + [_P] * 5 + [ctypes.c_size_t, _P])
    lib.dart_ssd_scan_backward_workspace_bytes.restype = ctypes.c_size_t
    lib.dart_ssd_scan_backward_workspace_bytes.argtypes = [D]
    lib.dart_ssd_scan_backward.restype = ctypes.c_int
    lib.dart_ssd_scan_backward.argtypes = [D, ctypes.c_int] + [_P] * 17 + [ctypes.c_size_t, _P]
    lib.dart_sma_backward_workspace_bytes.restype = ctypes.c_size_t
    lib.dart_sma_backward_workspace_bytes.argtypes = [D]
    lib.dart_sma_backward.restype = ctypes.c_int
    lib.dart_sma_backward.argtypes = ([D, ctypes.c_int] + [_P] * 4 + [ctypes.c_float] + [_P] * 7
                                      + [ctypes.c_size_t, _P])
    lib.dart_decode_step_e4m3.restype = ctypes.c_int
    lib.dart_decode_step_e4m3.argtypes = ([D, ctypes.c_int] + [_P] * 7 + [ctypes.c_float] + [_P] * 4
                                          + [ctypes.c_int] + [_P] * 5 + [ctypes.c_size_t, _P])
    lib.dart_cache_quantize_e4m3.restype = ctypes.c_int
    lib.dart_cache_quantize_e4m3.argtypes = [D, ctypes.c_int, _P, ctypes.c_int, _P, _P, ctypes.c_int, _P]
    lib.dart_decode_memlog_init.restype = ctypes.c_int
    lib.dart_decode_memlog_init.argtypes = [D, _P, _P, _P, ctypes.c_int, _P]
    lib.dart_sma_decayed_workspace_bytes.restype = ctypes.c_size_t
    lib.dart_sma_decayed_workspace_bytes.argtypes = [D]
    lib.dart_sma_forward_decayed.restype = ctypes.c_int
    lib.dart_sma_forward_decayed.argtypes = ([D, ctypes.c_int] + [_P] * 6 + [ctypes.c_float, _P, _P, _P,
                                             ctypes.c_size_t, _P])
    lib.dart_decode_step_workspace_bytes.restype = ctypes.c_size_t
    lib.dart_decode_step_workspace_bytes.argtypes = [D, ctypes.c_int, ctypes.c_int]
    lib.dart_decode_step.restype = ctypes.c_int
    lib.dart_decode_step.argtypes = ([D, ctypes.c_int] + [_P] * 7 + [ctypes.c_float] + [_P] * 3
                                     + [ctypes.c_int] + [_P] * 4 + [ctypes.c_size_t, _P])
    lib.dart_supported.restype = ctypes.c_int
    lib.dart_supported.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.dart_sync_status.restype = ctypes.c_int
    lib.dart_sync_status.argtypes = [_P]
    lib.dart_selftest_wait_timeout.restype = ctypes.c_int
    lib.dart_selftest_wait_timeout.argtypes = [ctypes.c_uint, _P]
    lib.dart_last_error.restype = ctypes.c_char_p
    lib.dart_last_error.argtypes = []
    lib.dart_abi_version.restype = ctypes.c_int
    lib.dart_abi_version.argtypes = []
    lib.dart_launch_count.restype = ctypes.c_ulonglong
    lib.dart_launch_count.argtypes = []
    lib.dart_sma_impl.restype = ctypes.c_char_p
    lib.dart_sma_impl.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.dart_decode_step_noalloc.restype = ctypes.c_int
    lib.dart_decode_step_noalloc.argtypes = ([D, ctypes.c_int] + [_P] * 7 + [ctypes.c_float] + [_P] * 3
                                             + [ctypes.c_int] + [_P] * 4)
    _lib = lib
    return lib


def _check(rc: int):
    if rc != DART_OK:
        raise DartError(rc, load().dart_last_error().decode())


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return DART_F32
    if t == torch.bfloat16:
        return DART_BF16
    raise TypeError(f"unsupported dtype {t}; use float32 or bfloat16")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t: Optional[torch.Tensor], device, dtype=None) -> Optional[torch.Tensor]:
    """Contiguous tensor on `device` (copying host tensors there)."""
    if t is None:
        return None
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    if t.device != device:
        t = t.to(device, non_blocking=True)
    return t.contiguous()


def _to_host(*ts):
    """Copies device tensors back into page-locked host tensors (torch's
    caching host allocator) with asynchronous copies, then waits for them."""
    out = []
    for t in ts:
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t, non_blocking=True)
        out.append(h)
    if ts:
        torch.cuda.current_stream(ts[0].device).synchronize()
    return out


def _device_of(*ts) -> torch.device:
    for t in ts:
        if isinstance(t, torch.Tensor) and t.is_cuda:
            return t.device
    if not torch.cuda.is_available():
        raise RuntimeError("dart: no CUDA device available (there is no CPU path)")
    return torch.device("cuda", torch.cuda.current_device())


def _shape(name, t, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def _bc_groups(name, t, lead, H) -> int:
    """Number of B/C groups of a B or C tensor: shape lead + (N,) is one group
    shared by all heads, lead + (G, N) is G groups (G divides H, head h reads
    group h // (H // G))."""
    if t.dim() == len(lead) + 1:
        _shape(name, t, (*lead, t.shape[-1]))
        return 1
    if t.dim() == len(lead) + 2:
        G = t.shape[-2]
        _shape(name, t, (*lead, G, t.shape[-1]))
        if G < 1 or H % G:
            raise ValueError(f"{name}: {G} groups do not divide {H} heads")
        return G
    raise ValueError(f"{name}: expected shape {tuple(lead)} + ([G,] N), got {tuple(t.shape)}")


def supported(dstate: int, headdim: int, chunk: int, dtype: torch.dtype) -> bool:
    return bool(load().dart_supported(dstate, headdim, chunk, _dtype_code(dtype)))


def abi_version() -> int:
    return load().dart_abi_version()


def sma_impl(dstate: int, headdim: int, chunk: int, dtype: torch.dtype) -> str:
    """Which SMA kernel the library dispatches to for this shape/dtype."""
    return load().dart_sma_impl(dstate, headdim, chunk, _dtype_code(dtype)).decode()


def launch_count() -> int:
    """Kernels the library has enqueued so far in this process."""
    return int(load().dart_launch_count())


# ---------------------------------------------------------------------------
def dart_ssd_chunk_scan(x, dt, A, Bm, Cm, chunk: int, init_state=None, *, y_ssd=None, dH=None,
                        states=None, workspace=None):
    """SSD chunked scan keeping the chunk memories.

    x[B,L,H,P], Bm/Cm[B,L,N] or [B,L,G,N] with G groups of heads (head h
    reads group h // (H // G)) (float32 or bfloat16), dt[B,L,H] and A[H] float32,
    init_state optional float32 [B,H,N,P].  Returns (y_ssd float32 [B,L,H,P],
    dH [B,H,C,N,P] in x's dtype, states float32 [B,H,C,N,P]).  Optional
    preallocated outputs/workspace avoid allocation in timed loops."""
    lib = load()
    host = not x.is_cuda
    dev = _device_of(x, dt, A, Bm, Cm)
    x, Bm, Cm = (_dev(v, dev, x.dtype) for v in (x, Bm, Cm))
    dt, A = _dev(dt, dev, torch.float32), _dev(A, dev, torch.float32)
    init_state = _dev(init_state, dev, torch.float32)
    Bsz, L, H, P = x.shape
    N = Bm.shape[-1]
    _shape("dt", dt, (Bsz, L, H)); _shape("A", A, (H,))
    G = _bc_groups("Bm", Bm, (Bsz, L), H)
    if _bc_groups("Cm", Cm, (Bsz, L), H) != G or Cm.shape != Bm.shape:
        raise ValueError("Bm and Cm must have the same shape")
    if init_state is not None:
        _shape("init_state", init_state, (Bsz, H, N, P))
    C = -(-L // chunk)   # a partial last chunk counts
    dims = Dims(Bsz, L, H, P, N, chunk, G)
    code = _dtype_code(x.dtype)
    if y_ssd is None:
        y_ssd = torch.empty((Bsz, L, H, P), device=dev, dtype=torch.float32)
    if dH is None:
        dH = torch.empty((Bsz, H, C, N, P), device=dev, dtype=x.dtype)
    if states is None:
        states = torch.empty((Bsz, H, C, N, P), device=dev, dtype=torch.float32)
    wsb = lib.dart_ssd_chunk_scan_workspace_bytes(ctypes.byref(dims), code)
    if workspace is None:
        workspace = torch.empty(max(16, wsb), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        _check(lib.dart_ssd_chunk_scan(ctypes.byref(dims), code, _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm),
                                       _ptr(Cm), _ptr(init_state), _ptr(y_ssd), _ptr(dH), _ptr(states),
                                       _ptr(workspace), workspace.numel(), _stream()))
    if host:
        return tuple(_to_host(y_ssd, dH, states))
    return y_ssd, dH, states


def dart_sma_forward(Q, E, Cm, dH, chunk: int, g: float, y_ssd=None, *, out=None):
    """State-memory attention plus gated residual: returns float32 [B,L,H,P]
    equal to y_ssd + g*o (or o when y_ssd is None)."""
    lib = load()
    host = not Q.is_cuda
    dev = _device_of(Q, E, Cm, dH)
    Q, E, Cm, dH = (_dev(v, dev, Q.dtype) for v in (Q, E, Cm, dH))
    y_ssd = _dev(y_ssd, dev, torch.float32)
    Bsz, L, H, N = Q.shape
    P = E.shape[-1]
    C = -(-L // chunk)   # a partial last chunk counts
    _shape("E", E, (Bsz, L, H, P)); _shape("dH", dH, (Bsz, H, C, N, P))
    G = _bc_groups("Cm", Cm, (Bsz, L), H)
    if y_ssd is not None:
        _shape("y_ssd", y_ssd, (Bsz, L, H, P))
    if out is None:
        out = torch.empty((Bsz, L, H, P), device=dev, dtype=torch.float32)
    dims = Dims(Bsz, L, H, P, N, chunk, G)
    with torch.cuda.device(dev):
        _check(lib.dart_sma_forward(ctypes.byref(dims), _dtype_code(Q.dtype), _ptr(Q), _ptr(E), _ptr(Cm),
                                    _ptr(dH), float(g), _ptr(y_ssd), _ptr(out), _stream()))
    return _to_host(out)[0] if host else out


def dart_sma_forward_decayed(Q, E, Cm, dH, dt, A, chunk: int, g: float, y_ssd=None, *, out=None,
                             workspace=None):
    """The decayed-memory variant of dart_sma_forward: memory c reaches token
    t scaled by exp(A_h sum_{r=e(c)+1..t} dt_r).  dt [B,L,H] and A [H] are
    float32, as given to the scan.  Returns float32 [B,L,H,P]."""
    lib = load()
    host = not Q.is_cuda
    dev = _device_of(Q, E, Cm, dH, dt, A)
    Q, E, Cm, dH = (_dev(v, dev, Q.dtype) for v in (Q, E, Cm, dH))
    dt, A = _dev(dt, dev, torch.float32), _dev(A, dev, torch.float32)
    y_ssd = _dev(y_ssd, dev, torch.float32)
    Bsz, L, H, N = Q.shape
    P = E.shape[-1]
    C = -(-L // chunk)
    _shape("E", E, (Bsz, L, H, P)); _shape("dH", dH, (Bsz, H, C, N, P))
    G = _bc_groups("Cm", Cm, (Bsz, L), H)
    _shape("dt", dt, (Bsz, L, H)); _shape("A", A, (H,))
    if y_ssd is not None:
        _shape("y_ssd", y_ssd, (Bsz, L, H, P))
    if out is None:
        out = torch.empty((Bsz, L, H, P), device=dev, dtype=torch.float32)
    dims = Dims(Bsz, L, H, P, N, chunk, G)
    wsb = lib.dart_sma_decayed_workspace_bytes(ctypes.byref(dims))
    if workspace is None:
        workspace = torch.empty(max(16, wsb), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        _check(lib.dart_sma_forward_decayed(ctypes.byref(dims), _dtype_code(Q.dtype), _ptr(Q), _ptr(E),
                                            _ptr(Cm), _ptr(dH), _ptr(dt), _ptr(A), float(g), _ptr(y_ssd),
                                            _ptr(out), _ptr(workspace), workspace.numel(), _stream()))
    return _to_host(out)[0] if host else out


def dart_sma_backward(Q, E, Cm, dH, chunk: int, g: float, dy, *, workspace=None) -> dict:
    """Gradients of sum(dy * y) for y = y_ssd + g * SMA(Q, E, Cm; dH) (raw
    memories): a dict of float32 device tensors dQ [B,L,H,N], dE [B,L,H,P],
    dCm [B,L,N], ddH [B,H,C,N,P] and dg (shape [1]).  Inputs as for
    dart_sma_forward, on the device; dy float32 [B,L,H,P]."""
    lib = load()
    dev = _device_of(Q, E, Cm, dH, dy)
    Q, E, Cm, dH = (_dev(v, dev, Q.dtype) for v in (Q, E, Cm, dH))
    dy = _dev(dy, dev, torch.float32)
    Bsz, L, H, N = Q.shape
    P = E.shape[-1]
    C = -(-L // chunk)
    _shape("E", E, (Bsz, L, H, P)); _shape("dH", dH, (Bsz, H, C, N, P))
    G = _bc_groups("Cm", Cm, (Bsz, L), H)
    _shape("dy", dy, (Bsz, L, H, P))
    dims = Dims(Bsz, L, H, P, N, chunk, G)
    out = {"dQ": torch.empty((Bsz, L, H, N), device=dev), "dE": torch.empty((Bsz, L, H, P), device=dev),
           "dCm": torch.empty(tuple(Cm.shape), device=dev), "ddH": torch.empty((Bsz, H, C, N, P), device=dev),
           "dg": torch.empty((1,), device=dev)}
    wsb = lib.dart_sma_backward_workspace_bytes(ctypes.byref(dims))
    if workspace is None:
        workspace = torch.empty(max(16, wsb), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        _check(lib.dart_sma_backward(ctypes.byref(dims), _dtype_code(Q.dtype), _ptr(Q), _ptr(E), _ptr(Cm), _ptr(dH),
                                     float(g), _ptr(dy), _ptr(out["dQ"]), _ptr(out["dE"]), _ptr(out["dCm"]),
                                     _ptr(out["ddH"]), _ptr(out["dg"]), _ptr(workspace), workspace.numel(),
                                     _stream()))
    return out


def dart_ssd_scan_backward(x, dt, A, Bm, Cm, chunk: int, states, dy, ddH=None, init_state=None, *,
                           dCm_add=None, workspace=None) -> dict:
    """Gradients of sum(dy * y_ssd) + sum(ddH * dH) through the scan: a dict
    of float32 device tensors dx, ddt, dA, dBm, dCm and, with an initial
    state, dinit_state.  x/Bm/Cm as given to the forward (dtype),
    dt/A/init_state float32, states = the forward's boundary states, dy
    float32 [B,L,H,P], ddH float32 [B,H,C,N,P] or None.  The library adds
    dCm_add (float32 [B,L,N], e.g. dart_sma_backward's dCm) into dCm."""
    lib = load()
    dev = _device_of(x, dt, A, Bm, Cm, states, dy)
    x, Bm, Cm = (_dev(v, dev, x.dtype) for v in (x, Bm, Cm))
    dt, A, states, dy = (_dev(v, dev, torch.float32) for v in (dt, A, states, dy))
    ddH = _dev(ddH, dev, torch.float32)
    dCm_add = _dev(dCm_add, dev, torch.float32)
    init_state = _dev(init_state, dev, torch.float32)
    Bsz, L, H, P = x.shape
    N = Bm.shape[-1]
    C = -(-L // chunk)
    _shape("states", states, (Bsz, H, C, N, P)); _shape("dy", dy, (Bsz, L, H, P))
    if ddH is not None:
        _shape("ddH", ddH, (Bsz, H, C, N, P))
    G = _bc_groups("Bm", Bm, (Bsz, L), H)
    if Cm.shape != Bm.shape:
        raise ValueError("Bm and Cm must have the same shape")
    if dCm_add is not None:
        _shape("dCm_add", dCm_add, tuple(Cm.shape))
    dims = Dims(Bsz, L, H, P, N, chunk, G)
    out = {"dx": torch.empty((Bsz, L, H, P), device=dev), "ddt": torch.empty((Bsz, L, H), device=dev),
           "dA": torch.empty((H,), device=dev), "dBm": torch.empty(tuple(Bm.shape), device=dev),
           "dCm": torch.empty(tuple(Cm.shape), device=dev)}
    if init_state is not None:
        out["dinit_state"] = torch.empty((Bsz, H, N, P), device=dev)
    wsb = lib.dart_ssd_scan_backward_workspace_bytes(ctypes.byref(dims))
    if workspace is None:
        workspace = torch.empty(max(16, wsb), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        _check(lib.dart_ssd_scan_backward(ctypes.byref(dims), _dtype_code(x.dtype), _ptr(x), _ptr(dt), _ptr(A),
                                          _ptr(Bm), _ptr(Cm), _ptr(init_state), _ptr(states), _ptr(dy), _ptr(ddH),
                                          _ptr(dCm_add), _ptr(out["dx"]), _ptr(out["ddt"]), _ptr(out["dA"]), _ptr(out["dBm"]),
                                          _ptr(out["dCm"]), _ptr(out.get("dinit_state")), _ptr(workspace),
                                          workspace.numel(), _stream()))
    return out


def layer_backward(x, dt, A, Bm, Cm, Q, E, chunk: int, g: float, dy, init_state=None) -> dict:
    """Gradients of sum(dy * y) for the DART layer forward (raw memories):
    runs the forward scan for its memories and boundary states, the SMA
    backward, then the scan backward driven by dy and the memory gradients.
    Returns float32 device tensors dx, ddt, dA, dBm, dCm, dQ, dE, dg (and
    dinit_state with an initial state)."""
    y_ssd, dH, states = dart_ssd_chunk_scan(x, dt, A, Bm, Cm, chunk, init_state)
    sm = dart_sma_backward(Q, E, Cm, dH, chunk, g, dy)
    # the scan backward adds the SMA's C gradient into its own (in the library)
    out = dart_ssd_scan_backward(x, dt, A, Bm, Cm, chunk, states, dy, sm["ddH"], init_state, dCm_add=sm["dCm"])
    out.update(dQ=sm["dQ"], dE=sm["dE"], dg=sm["dg"])
    return out


def sma_decayed_workspace_bytes(batch, seqlen, nheads, headdim, dstate, chunk) -> int:
    return int(load().dart_sma_decayed_workspace_bytes(
        ctypes.byref(Dims(batch, seqlen, nheads, headdim, dstate, chunk, 1))))


def layer_forward(x, dt, A, Bm, Cm, Q, E, chunk: int, g: float, init_state=None, *,
                  outputs=("y", "dH", "states"), buffers: Optional[dict] = None,
                  decayed: bool = False):
    """The DART layer forward: scan, then SMA with the gated residual written
    in place over y_ssd.  Returns a dict with the requested `outputs` among
    y, dH, states.  With host (CPU) inputs the inputs are copied to the
    current device and only the requested outputs are copied back.
    `buffers` may hold preallocated device tensors y, dH, states, workspace
    (and sma_workspace for the decayed variant).  ``decayed`` selects the
    decayed-memory SMA."""
    host = not x.is_cuda
    dev = _device_of(x)
    args = [_dev(v, dev) for v in (x, dt, A, Bm, Cm, Q, E)]
    init_state = _dev(init_state, dev)
    b = buffers or {}
    y, dH, states = dart_ssd_chunk_scan(*args[:5], chunk, init_state, y_ssd=b.get("y"), dH=b.get("dH"),
                                        states=b.get("states"), workspace=b.get("workspace"))
    if decayed:
        dart_sma_forward_decayed(args[5], args[6], args[4], dH, args[1], args[2], chunk, g, y, out=y,
                                 workspace=b.get("sma_workspace"))
    else:
        dart_sma_forward(args[5], args[6], args[4], dH, chunk, g, y, out=y)
    res = {"y": y, "dH": dH, "states": states}
    if host:
        return dict(zip(outputs, _to_host(*(res[k] for k in outputs))))
    return {k: res[k] for k in outputs}


def dart_decode_step(x, dt, A, Bm, Cm, Q, E, g: float, state, dH_cur, cache, nchunks, pos,
                     chunk: int, *, y=None, workspace=None, memlog=None, cache_exp=None):
    """One decode step for every sequence.  x[Bs,H,P], Bm/Cm[Bs,N] (or
    [Bs,G,N] with G groups of heads),
    Q[Bs,H,N], E[Bs,H,P] (cache dtype), dt[Bs,H], A[H] float32; state and
    dH_cur float32 [Bs,H,N,P], cache [Bs,H,cmax,N,P], nchunks/pos int32 [Bs]
    are device tensors updated in place.  With ``memlog`` (float32
    [Bs,H,cmax] device tensor, updated in place) the memories are decayed to
    the new token (dart_decode_step_decayed).  A uint8 ``cache`` is an E4M3
    cache with row exponents ``cache_exp`` (int8 [Bs,H,cmax,N], in place);
    the token inputs then keep their own dtype (dart_decode_step_e4m3).
    Returns y float32 [Bs,H,P]."""
    lib = load()
    e4m3 = cache.dtype == torch.uint8
    if e4m3 and (cache_exp is None or cache_exp.dtype != torch.int8):
        raise ValueError("an E4M3 (uint8) cache needs its int8 row exponents cache_exp")
    bufs = [("state", state), ("dH_cur", dH_cur), ("cache", cache), ("nchunks", nchunks), ("pos", pos)]
    if memlog is not None:
        bufs.append(("memlog", memlog))
    if e4m3:
        bufs.append(("cache_exp", cache_exp))
    for name, t in bufs:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor (updated in place)")
    dev = cache.device
    host = not x.is_cuda
    in_dtype = x.dtype if e4m3 else cache.dtype
    x, Bm, Cm, Q, E = (_dev(v, dev, in_dtype) for v in (x, Bm, Cm, Q, E))
    dt, A = _dev(dt, dev, torch.float32), _dev(A, dev, torch.float32)
    Bs, H, P = x.shape
    N = Bm.shape[-1]
    cmax = cache.shape[2]
    _shape("state", state, (Bs, H, N, P)); _shape("dH_cur", dH_cur, (Bs, H, N, P))
    _shape("cache", cache, (Bs, H, cmax, N, P)); _shape("Q", Q, (Bs, H, N)); _shape("E", E, (Bs, H, P))
    _shape("dt", dt, (Bs, H))
    G = _bc_groups("Bm", Bm, (Bs,), H)
    if Cm.shape != Bm.shape:
        raise ValueError("Bm and Cm must have the same shape")
    if state.dtype != torch.float32 or dH_cur.dtype != torch.float32:
        raise TypeError("state and dH_cur must be float32")
    if nchunks.dtype != torch.int32 or pos.dtype != torch.int32:
        raise TypeError("nchunks and pos must be int32")
    if memlog is not None:
        _shape("memlog", memlog, (Bs, H, cmax))
        if memlog.dtype != torch.float32:
            raise TypeError("memlog must be float32")
    if e4m3:
        _shape("cache_exp", cache_exp, (Bs, H, cmax, N))
    dims = Dims(Bs, 0, H, P, N, chunk, G)
    code = _dtype_code(in_dtype)
    if y is None:
        y = torch.empty((Bs, H, P), device=dev, dtype=torch.float32)
    wsb = lib.dart_decode_step_workspace_bytes(ctypes.byref(dims), code, cmax)
    if workspace is None:
        workspace = torch.empty(max(16, wsb), device=dev, dtype=torch.uint8)
    with torch.cuda.device(dev):
        if e4m3:
            _check(lib.dart_decode_step_e4m3(ctypes.byref(dims), code, _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm),
                                             _ptr(Cm), _ptr(Q), _ptr(E), float(g), _ptr(state), _ptr(dH_cur),
                                             _ptr(cache), _ptr(cache_exp), cmax, _ptr(nchunks), _ptr(pos),
                                             _ptr(memlog), _ptr(y), _ptr(workspace), workspace.numel(),
                                             _stream()))
        elif memlog is None:
            _check(lib.dart_decode_step(ctypes.byref(dims), code, _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm),
                                        _ptr(Cm), _ptr(Q), _ptr(E), float(g), _ptr(state), _ptr(dH_cur),
                                        _ptr(cache), cmax, _ptr(nchunks), _ptr(pos), _ptr(y), _ptr(workspace),
                                        workspace.numel(), _stream()))
        else:
            _check(lib.dart_decode_step_decayed(ctypes.byref(dims), code, _ptr(x), _ptr(dt), _ptr(A), _ptr(Bm),
                                                _ptr(Cm), _ptr(Q), _ptr(E), float(g), _ptr(state),
                                                _ptr(dH_cur), _ptr(cache), cmax, _ptr(nchunks), _ptr(pos),
                                                _ptr(memlog), _ptr(y), _ptr(workspace), workspace.numel(),
                                                _stream()))
    return _to_host(y)[0] if host else y


def cache_quantize_e4m3(dH, nmem: int, cache, cache_exp):
    """Quantize memories 0..nmem-1 of a prefill's dH [B,H,C,N,P] (float32 or
    bfloat16, on the device) into slots 0..nmem-1 of an E4M3 cache (uint8
    [B,H,cmax,N,P] codes, int8 [B,H,cmax,N] row exponents), in place."""
    lib = load()
    for name, t in (("dH", dH), ("cache", cache), ("cache_exp", cache_exp)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if cache.dtype != torch.uint8 or cache_exp.dtype != torch.int8:
        raise TypeError("cache must be uint8 and cache_exp int8")
    Bsz, H, C, N, P = dH.shape
    cmax = cache.shape[2]
    _shape("cache", cache, (Bsz, H, cmax, N, P)); _shape("cache_exp", cache_exp, (Bsz, H, cmax, N))
    dims = Dims(Bsz, C, H, P, N, 1, 1)   # C memories: seqlen C at chunk 1
    with torch.cuda.device(dH.device):
        _check(lib.dart_cache_quantize_e4m3(ctypes.byref(dims), _dtype_code(dH.dtype), _ptr(dH), int(nmem),
                                            _ptr(cache), _ptr(cache_exp), cmax, _stream()))
    return cache, cache_exp


def decode_memlog_init(dt, A, chunk: int, memlog):
    """Fill memlog[b,h,c] (float32 [B,H,cmax] device tensor) for decode after
    a prefill whose dt [B,L,H] is given: the log-decay of each of the L //
    chunk completed memories, sum_{r=(c+1)S..L-1} dt A_h."""
    lib = load()
    if not memlog.is_cuda or not memlog.is_contiguous() or memlog.dtype != torch.float32:
        raise ValueError("memlog must be a contiguous float32 CUDA tensor")
    dev = memlog.device
    dt, A = _dev(dt, dev, torch.float32), _dev(A, dev, torch.float32)
    Bsz, L, H = dt.shape
    _shape("A", A, (H,)); _shape("memlog", memlog, (Bsz, H, memlog.shape[2]))
    dims = Dims(Bsz, L, H, 0, 0, chunk, 1)
    with torch.cuda.device(dev):
        _check(lib.dart_decode_memlog_init(ctypes.byref(dims), _ptr(dt), _ptr(A), _ptr(memlog),
                                           memlog.shape[2], _stream()))
    return memlog


def dart_decode_step_noalloc(x, dt, A, Bm, Cm, Q, E, g: float, state, dH_cur, cache, nchunks, pos,
                             chunk: int, *, y=None):
    """dart_decode_step for callers that cannot allocate device memory: the
    library keeps the step's scratch in a fixed 16 MiB static device array
    instead of a caller workspace (see include/dart.h for its limits).  All
    tensors must already be on the device; `y` may be preallocated so that the
    call allocates nothing at all.  Calls overlapping on the GPU race on the
    shared scratch."""
    lib = load()
    for name, t in (("x", x), ("dt", dt), ("A", A), ("Bm", Bm), ("Cm", Cm), ("Q", Q), ("E", E),
                    ("state", state), ("dH_cur", dH_cur), ("cache", cache), ("nchunks", nchunks), ("pos", pos)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    Bs, H, P = x.shape
    N = Bm.shape[-1]
    cmax = cache.shape[2]
    _shape("state", state, (Bs, H, N, P)); _shape("dH_cur", dH_cur, (Bs, H, N, P))
    _shape("cache", cache, (Bs, H, cmax, N, P))
    G = _bc_groups("Bm", Bm, (Bs,), H)
    if Cm.shape != Bm.shape:
        raise ValueError("Bm and Cm must have the same shape")
    if y is None:
        y = torch.empty((Bs, H, P), device=cache.device, dtype=torch.float32)
    dims = Dims(Bs, 0, H, P, N, chunk, G)
    with torch.cuda.device(cache.device):
        _check(lib.dart_decode_step_noalloc(ctypes.byref(dims), _dtype_code(cache.dtype), _ptr(x), _ptr(dt),
                                            _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(Q), _ptr(E), float(g), _ptr(state),
                                            _ptr(dH_cur), _ptr(cache), cmax, _ptr(nchunks), _ptr(pos), _ptr(y),
                                            _stream()))
    return y


def decode_workspace_bytes(nseq, nheads, headdim, dstate, chunk, cmax, dtype) -> int:
    dims = Dims(nseq, 0, nheads, headdim, dstate, chunk, 1)
    return load().dart_decode_step_workspace_bytes(ctypes.byref(dims), _dtype_code(dtype), cmax)


def sma_backward_workspace_bytes(batch, seqlen, nheads, headdim, dstate, chunk) -> int:
    dims = Dims(batch, seqlen, nheads, headdim, dstate, chunk, 1)
    return int(load().dart_sma_backward_workspace_bytes(ctypes.byref(dims)))


def scan_backward_workspace_bytes(batch, seqlen, nheads, headdim, dstate, chunk) -> int:
    dims = Dims(batch, seqlen, nheads, headdim, dstate, chunk, 1)
    return int(load().dart_ssd_scan_backward_workspace_bytes(ctypes.byref(dims)))


def scan_workspace_bytes(batch, seqlen, nheads, headdim, dstate, chunk, dtype) -> int:
    dims = Dims(batch, seqlen, nheads, headdim, dstate, chunk, 1)
    return load().dart_ssd_chunk_scan_workspace_bytes(ctypes.byref(dims), _dtype_code(dtype))


def dart_selftest_wait_timeout(limit_us: int, stream: Optional[torch.cuda.Stream] = None):
    """Launch the failure-detection drill: one bounded wait on an mbarrier
    nothing arrives on, giving up after limit_us; the next dart_sync_status
    raises DartError(DART_ERR_TIMEOUT) and clears the status word."""
    s = stream or torch.cuda.current_stream()
    _check(load().dart_selftest_wait_timeout(int(limit_us), ctypes.c_void_p(s.cuda_stream)))


def dart_sync_status(stream: Optional[torch.cuda.Stream] = None):
    """Synchronise the stream and raise DartError if a kernel latched an error."""
    s = stream or torch.cuda.current_stream()
    _check(load().dart_sync_status(ctypes.c_void_p(s.cuda_stream)))
