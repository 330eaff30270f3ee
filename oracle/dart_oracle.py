"""Python front end of the fp64 CPU oracle (``dart_oracle.c``).

TEST INFRASTRUCTURE ONLY: ``tests/``, the smoke check in ``__graft_entry__``
and the CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA
library never imports this module, and this module imports nothing from the
CUDA library.  Inputs are numpy arrays in the layouts documented in
``dart_oracle.c``; everything is converted to float (inputs) or double
(state-like arrays) and handed to the C code, which does all the arithmetic.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "dart_oracle.c")
LIBRARY = os.path.join(_HERE, "libdart_oracle.so")


class _Dims(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int) for name in
                ("batch", "seqlen", "nheads", "headdim", "dstate", "chunk", "ngroups")]


def _groups(a, ndim_shared: int) -> int:
    """Number of B/C groups of an array: ndim_shared dims means one group
    shared by all heads; one more dim is the group axis (second to last)."""
    return 1 if a.ndim == ndim_shared else a.shape[-2]


def build(source: str = SOURCE, library: str = LIBRARY, extra_flags=()) -> str:
    """Compile the oracle with gcc into a shared library; returns its path."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           *extra_flags, source, "-o", library, "-lm"]
    subprocess.run(cmd, check=True)
    return library


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


_P = ctypes.c_void_p


class Oracle:
    """Handle on one compiled oracle library (the default one, or a test build)."""

    def __init__(self, library: str = LIBRARY, nthreads: Optional[int] = None):
        if library == LIBRARY and (not os.path.exists(LIBRARY)
                                   or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE)):
            build()
        self.lib = ctypes.CDLL(library)
        self.nthreads = nthreads or default_threads()
        self.lib.oracle_ssd_scan.restype = ctypes.c_int
        self.lib.oracle_ssd_scan.argtypes = [ctypes.POINTER(_Dims)] + [_P] * 9 + [ctypes.c_int]
        self.lib.oracle_sma.restype = ctypes.c_int
        self.lib.oracle_sma.argtypes = ([ctypes.POINTER(_Dims)] + [_P] * 6 + [ctypes.c_double]
                                        + [_P] * 5 + [ctypes.c_int, ctypes.c_int])
        self.lib.oracle_decode_step.restype = ctypes.c_int
        self.lib.oracle_decode_step.argtypes = (
            [ctypes.POINTER(_Dims), ctypes.c_int] + [_P] * 7 + [ctypes.c_double]
            + [_P] * 6 + [ctypes.c_int, _P, ctypes.c_int])
        self.lib.oracle_ssd_scan_backward.restype = ctypes.c_int
        self.lib.oracle_ssd_scan_backward.argtypes = [ctypes.POINTER(_Dims)] + [_P] * 14 + [ctypes.c_int]
        self.lib.oracle_quantize_e4m3.restype = ctypes.c_int
        self.lib.oracle_quantize_e4m3.argtypes = [_P, ctypes.c_long, ctypes.c_int, _P, _P, _P]

    # ------------------------------------------------------------------
    @staticmethod
    def _f32(a):
        return np.ascontiguousarray(np.asarray(a, dtype=np.float32))

    @staticmethod
    def _f64(a):
        return np.ascontiguousarray(np.asarray(a, dtype=np.float64))

    @staticmethod
    def _ptr(a):
        return None if a is None else a.ctypes.data_as(_P)

    # ------------------------------------------------------------------
    def ssd_scan(self, x, dt, A, Bm, Cm, chunk: int, init_state=None):
        """Token-by-token recurrence.  Returns (y_ssd[B,L,H,P], dH[B,H,C,N,P],
        states[B,H,C,N,P]) in float64, C = ceil(L / chunk) (a partial last
        chunk closes at token L-1)."""
        x, dt, A, Bm, Cm = (self._f32(v) for v in (x, dt, A, Bm, Cm))
        Bsz, L, H, P = x.shape
        N = Bm.shape[-1]
        C = -(-L // chunk)
        d = _Dims(Bsz, L, H, P, N, chunk, _groups(Bm, 3))
        y = np.empty((Bsz, L, H, P), np.float64)
        dH = np.empty((Bsz, H, C, N, P), np.float64)
        st = np.empty((Bsz, H, C, N, P), np.float64)
        h0 = None if init_state is None else self._f64(init_state)
        rc = self.lib.oracle_ssd_scan(ctypes.byref(d), self._ptr(x), self._ptr(dt), self._ptr(A),
                                      self._ptr(Bm), self._ptr(Cm), self._ptr(h0), self._ptr(y),
                                      self._ptr(dH), self._ptr(st), self.nthreads)
        if rc:
            raise ValueError("oracle_ssd_scan rejected its arguments")
        return y, dH, st

    def scan_backward(self, x, dt, A, Bm, Cm, chunk: int, dy, gD=None, init_state=None):
        """Gradients of sum(dy * y_ssd) + sum(gD * dH) through the token
        recurrence (reverse mode, token by token).  Returns a dict of float64
        arrays dx, ddt, dA, dBm, dCm (shaped like Bm / Cm: summed over the
        heads of each group) and, with an initial state, dinit_state."""
        x, dt, A, Bm, Cm = (self._f32(v) for v in (x, dt, A, Bm, Cm))
        Bsz, L, H, P = x.shape
        N = Bm.shape[-1]
        d = _Dims(Bsz, L, H, P, N, chunk, _groups(Bm, 3))
        dy = self._f64(dy)
        gD = None if gD is None else self._f64(gD)
        h0 = None if init_state is None else self._f64(init_state)
        out = {"dx": np.empty((Bsz, L, H, P), np.float64), "ddt": np.empty((Bsz, L, H), np.float64),
               "dA": np.empty((H,), np.float64), "dBm": np.empty(Bm.shape, np.float64),
               "dCm": np.empty(Cm.shape, np.float64)}
        dinit = None if h0 is None else np.empty((Bsz, H, N, P), np.float64)
        rc = self.lib.oracle_ssd_scan_backward(
            ctypes.byref(d), self._ptr(x), self._ptr(dt), self._ptr(A), self._ptr(Bm), self._ptr(Cm),
            self._ptr(h0), self._ptr(dy), self._ptr(gD), self._ptr(out["dx"]), self._ptr(out["ddt"]),
            self._ptr(out["dA"]), self._ptr(out["dBm"]), self._ptr(out["dCm"]), self._ptr(dinit), self.nthreads)
        if rc:
            raise ValueError("oracle_ssd_scan_backward rejected its arguments")
        if dinit is not None:
            out["dinit_state"] = dinit
        return out

    def sma(self, Q, E, Cm, dH, chunk: int, g: float = 1.0, y_ssd=None,
            tokens=None, want_scores: bool = False, dt=None, A=None):
        """Naive state-memory attention.  Returns dict with 'o' (raw readout),
        'y' (y_ssd + g*o; y_ssd = 0 when not given) and optionally 'scores'
        ([B,H,rows,C], NaN where masked).  With ``tokens`` only those
        positions are computed and rows are compacted to [B,len(tokens),H,P].
        With ``dt`` [B,L,H] and ``A`` [H] every memory is decayed from its
        chunk's last token to t before use (the decayed-memory variant)."""
        if (dt is None) != (A is None):
            raise ValueError("dt and A go together")
        Q, E, Cm = (self._f32(v) for v in (Q, E, Cm))
        dtv = None if dt is None else self._f32(dt)
        Av = None if A is None else self._f32(A)
        dH = self._f64(dH)
        Bsz, L, H, N = Q.shape
        P = E.shape[-1]
        C = -(-L // chunk)
        d = _Dims(Bsz, L, H, P, N, chunk, _groups(Cm, 3))
        tok = None if tokens is None else np.ascontiguousarray(np.asarray(tokens, np.int32))
        rows = L if tok is None else len(tok)
        o = np.empty((Bsz, rows, H, P), np.float64)
        y = np.empty((Bsz, rows, H, P), np.float64)
        ys = None if y_ssd is None else self._f64(y_ssd)
        if ys is not None and ys.shape != o.shape:
            raise ValueError("y_ssd must have the output row shape")
        sc = np.empty((Bsz, H, rows, C), np.float64) if want_scores else None
        rc = self.lib.oracle_sma(ctypes.byref(d), self._ptr(Q), self._ptr(E), self._ptr(Cm),
                                 self._ptr(dH), self._ptr(dtv), self._ptr(Av), float(g),
                                 self._ptr(ys), self._ptr(o),
                                 self._ptr(y), self._ptr(sc), self._ptr(tok),
                                 0 if tok is None else len(tok), self.nthreads)
        if rc:
            raise ValueError("oracle_sma rejected its arguments")
        out = {"o": o, "y": y}
        if want_scores:
            out["scores"] = sc
        return out

    def layer_forward(self, x, dt, A, Bm, Cm, Q, E, chunk: int, g: float, init_state=None,
                      tokens=None, decayed: bool = False):
        """Full DART layer forward: scan, SMA over the scan's own fp64 dH,
        gated residual.  Returns dict(y, y_ssd, o, dH, states).  ``decayed``
        selects the decayed-memory SMA."""
        y_ssd, dH, st = self.ssd_scan(x, dt, A, Bm, Cm, chunk, init_state)
        ys = y_ssd if tokens is None else y_ssd[:, np.asarray(tokens)]
        r = self.sma(Q, E, Cm, dH, chunk, g, ys, tokens,
                     dt=dt if decayed else None, A=A if decayed else None)
        return {"y": r["y"], "o": r["o"], "y_ssd": y_ssd, "dH": dH, "states": st}

    def quantize_e4m3(self, x):
        """E4M3 cache rows: x[..., P] (float64) -> (codes uint8 [..., P],
        exponents int8 [...], dequantized float64 [..., P])."""
        x = self._f64(x)
        P = x.shape[-1]
        rows = x.size // P
        codes = np.empty(x.shape, np.uint8)
        exps = np.empty(x.shape[:-1], np.int8)
        deq = np.empty(x.shape, np.float64)
        if self.lib.oracle_quantize_e4m3(self._ptr(x), rows, P, self._ptr(codes), self._ptr(exps),
                                         self._ptr(deq)):
            raise ValueError("oracle_quantize_e4m3 rejected its arguments")
        return codes, exps, deq

    def decode_step(self, x, dt, A, Bm, Cm, Q, E, g, state, dH_cur, cache, nchunks, pos,
                    chunk: int, memlog=None, cache_e4m3: bool = False):
        """One decode step.  state, dH_cur, cache (float64, C-contiguous) and
        nchunks, pos (int32) are updated in place.  With ``memlog`` (float64
        [Bs,H,cmax], updated in place: the log-decay each cached memory has
        accumulated since its chunk closed) the memories are decayed to the
        new token before use.  With ``cache_e4m3`` the cache holds dequantized
        E4M3 rows and an append stores the quantized memory.  Returns
        y[Bs,H,P]."""
        x, dt, A, Bm, Cm, Q, E = (self._f32(v) for v in (x, dt, A, Bm, Cm, Q, E))
        bufs = [(state, np.float64), (dH_cur, np.float64), (cache, np.float64),
                (nchunks, np.int32), (pos, np.int32)]
        if memlog is not None:
            bufs.append((memlog, np.float64))
        for arr, dtp in bufs:
            if arr.dtype != dtp or not arr.flags.c_contiguous:
                raise ValueError("decode buffers must be contiguous with the documented dtype")
        Bs, H, P = x.shape
        N = Bm.shape[-1]
        cmax = cache.shape[2]
        d = _Dims(Bs, 0, H, P, N, chunk, _groups(Bm, 2))
        y = np.empty((Bs, H, P), np.float64)
        rc = self.lib.oracle_decode_step(ctypes.byref(d), cmax, self._ptr(x), self._ptr(dt),
                                         self._ptr(A), self._ptr(Bm), self._ptr(Cm),
                                         self._ptr(Q), self._ptr(E), float(g), self._ptr(state),
                                         self._ptr(dH_cur), self._ptr(cache), self._ptr(nchunks),
                                         self._ptr(pos), self._ptr(memlog), int(bool(cache_e4m3)),
                                         self._ptr(y), self.nthreads)
        if rc:
            raise ValueError("oracle_decode_step rejected its arguments")
        return y


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle compiled from this directory's source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
