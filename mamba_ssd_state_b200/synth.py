"""Seeded synthetic inputs for the DART layer.

This module draws random tensors and nothing else: it holds none of the
layer's arithmetic, so both the CUDA library's tests/benchmark and the CPU
oracle can be fed from it.  Every tensor comes from its own numpy PCG64 stream,
derived from (seed, tensor name[, index]) so that any one tensor -- or one
sequence of the decode cache -- can be regenerated alone.

Distributions (the pages train on the Pile and evaluate on MQAR/NIAH; none of
that data is needed to exercise the layer, so these shapes and distributions
stand in for it):
  x ~ N(0,1) [B,L,H,P];  B, C ~ N(0,1)/sqrt(N) [B,L,N] (shared by all heads);
  dt = softplus(N(0,1) - 4)  (tiny fp32 case) or log-uniform in [1e-3, 1e-1];
  A = -exp(U(0, ln 16)) per head;  Q ~ N(0,1) [B,L,H,N];  E ~ N(0,1)/sqrt(P);
  decode cache and state ~ N(0,1)/sqrt(N).
bf16 tensors are drawn in float32 and rounded once, to nearest-even.
"""
from __future__ import annotations

import hashlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, asdict

import numpy as np
import torch


@dataclass(frozen=True)
class LayerShape:
    batch: int
    seqlen: int
    nheads: int
    headdim: int   # P
    dstate: int    # N
    chunk: int     # S
    dtype: str     # "f32" or "bf16"
    dt_dist: str   # "softplus" or "loguniform"
    g: float = 0.5

    @property
    def nchunks(self) -> int:
        return -(-self.seqlen // self.chunk)   # a partial last chunk counts

    def asdict(self):
        return asdict(self)


@dataclass(frozen=True)
class DecodeShape:
    nseq: int
    nheads: int
    headdim: int
    dstate: int
    chunk: int
    ncached: int     # chunk memories already in the cache at step 0
    cmax: int        # cache capacity in chunks
    nsteps: int
    dtype: str = "bf16"
    g: float = 0.5


# The five workloads of the method's evaluation at the layer level.
TINY_FP32 = LayerShape(1, 512, 2, 16, 16, 64, "f32", "softplus")
LAYER_L2K = LayerShape(4, 2048, 32, 64, 128, 256, "bf16", "loguniform")
TRAIN_L8K = LayerShape(2, 8192, 32, 64, 128, 256, "bf16", "loguniform")
# the training-length layer with a sequence that ends 100 tokens into its last chunk
TRAIN_L8K_PARTIAL = LayerShape(2, 8192 - 100, 32, 64, 128, 256, "bf16", "loguniform")
LONG_L64K = LayerShape(1, 65536, 32, 64, 128, 256, "bf16", "loguniform")
DECODE_64x32K = DecodeShape(64, 32, 64, 128, 256, 128, 129, 256)

SHAPES = {"tiny_fp32": TINY_FP32, "layer_L2k": LAYER_L2K, "train_L8k": TRAIN_L8K,
          "long_L64k": LONG_L64K}


def _rng(seed: int, *key) -> np.random.Generator:
    """Independent stream for (seed, key...)."""
    h = hashlib.sha256(repr((int(seed),) + tuple(key)).encode()).digest()
    words = [int.from_bytes(h[i:i + 4], "little") for i in range(0, 16, 4)]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(words)))


def _normal(seed, name, shape, scale=1.0):
    a = _rng(seed, name).standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return a


def _dt(seed, name, shape, dist):
    r = _rng(seed, name)
    if dist == "softplus":
        z = r.standard_normal(shape, dtype=np.float64) - 4.0
        return np.log1p(np.exp(z)).astype(np.float32)
    if dist == "loguniform":
        u = r.uniform(np.log(1e-3), np.log(1e-1), size=shape)
        return np.exp(u).astype(np.float32)
    raise ValueError(dist)


def _A(seed, nheads):
    u = _rng(seed, "A").uniform(0.0, np.log(16.0), size=(nheads,))
    return (-np.exp(u)).astype(np.float32)


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _cast(a: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch_dtype(dtype))


def layer_inputs(shape: LayerShape, seed: int = 0, ngroups: int = 1) -> dict:
    """CPU tensors x, dt, A, Bm, Cm, Q, E (x/Bm/Cm/Q/E in the shape's dtype,
    dt and A always float32) and the gate g.  With ngroups > 1, Bm and Cm are
    [B, L, ngroups, N] (one row per group of heads), else [B, L, N]."""
    Bz, L, H, P, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate
    bc = (Bz, L, N) if ngroups == 1 else (Bz, L, ngroups, N)
    out = {
        "A": torch.from_numpy(_A(seed, H)),
        "dt": torch.from_numpy(_dt(seed, "dt", (Bz, L, H), shape.dt_dist)),
        "x": _cast(_normal(seed, "x", (Bz, L, H, P)), shape.dtype),
        "Bm": _cast(_normal(seed, "B", bc, 1.0 / np.sqrt(N)), shape.dtype),
        "Cm": _cast(_normal(seed, "C", bc, 1.0 / np.sqrt(N)), shape.dtype),
        "Q": _cast(_normal(seed, "Q", (Bz, L, H, N)), shape.dtype),
        "E": _cast(_normal(seed, "E", (Bz, L, H, P), 1.0 / np.sqrt(P)), shape.dtype),
    }
    out["g"] = float(shape.g)
    return out


def memory_inputs(batch, nheads, nchunks, dstate, headdim, dtype, seed=0, scale=None):
    """Stand-alone chunk memories dH[B,H,C,N,P] ~ N(0,1)*scale (default
    1/sqrt(N)), for exercising state-memory attention on its own."""
    s = (1.0 / np.sqrt(dstate)) if scale is None else scale
    return _cast(_normal(seed, "dH", (batch, nheads, nchunks, dstate, headdim), s), dtype)


def decode_cache_sequence(shape: DecodeShape, b: int, seed: int = 0) -> np.ndarray:
    """float32 [H, cmax, N, P] cache of sequence b: the first ``ncached``
    slots hold N(0,1)/sqrt(N) memories, the rest are zero."""
    H, N, P = shape.nheads, shape.dstate, shape.headdim
    out = np.zeros((H, shape.cmax, N, P), np.float32)
    out[:, :shape.ncached] = _rng(seed, "cache", b).standard_normal(
        (H, shape.ncached, N, P), dtype=np.float32) * np.float32(1.0 / np.sqrt(N))
    return out


def decode_state_sequence(shape: DecodeShape, b: int, seed: int = 0) -> np.ndarray:
    """float32 [H, N, P] recurrent state of sequence b, N(0,1)/sqrt(N)."""
    H, N, P = shape.nheads, shape.dstate, shape.headdim
    return _rng(seed, "state", b).standard_normal((H, N, P), dtype=np.float32) * np.float32(
        1.0 / np.sqrt(N))


def decode_initial(shape: DecodeShape, seed: int = 0, sequences=None, threads: int = 8) -> dict:
    """CPU tensors for the decode state at step 0: cache [Bs,H,cmax,N,P] in the
    shape's dtype, state and dH_cur [Bs,H,N,P] float32, nchunks/pos int32.
    ``sequences`` selects a subset (they keep their own streams)."""
    seqs = list(range(shape.nseq)) if sequences is None else list(sequences)
    H, N, P = shape.nheads, shape.dstate, shape.headdim
    cache = torch.empty((len(seqs), H, shape.cmax, N, P), dtype=torch_dtype(shape.dtype))

    def fill(i):
        cache[i].copy_(torch.from_numpy(decode_cache_sequence(shape, seqs[i], seed)))

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(fill, range(len(seqs))))
    state = torch.from_numpy(np.stack([decode_state_sequence(shape, b, seed) for b in seqs]))
    return {
        "cache": cache,
        "state": state.contiguous(),
        "dH_cur": torch.zeros((len(seqs), H, N, P), dtype=torch.float32),
        "nchunks": torch.full((len(seqs),), shape.ncached, dtype=torch.int32),
        "pos": torch.zeros((len(seqs),), dtype=torch.int32),
    }


def decode_tokens(shape: DecodeShape, step: int, seed: int = 0, sequences=None, ngroups: int = 1) -> dict:
    """Token inputs of one decode step for every sequence (or a subset):
    x[Bs,H,P], dt[Bs,H], Bm[Bs,N], Cm[Bs,N], Q[Bs,H,N], E[Bs,H,P]; drawn per
    (step, sequence) as in the 370M-shape layer case.  With ngroups > 1, Bm
    and Cm are [Bs, ngroups, N]."""
    seqs = list(range(shape.nseq)) if sequences is None else list(sequences)
    H, N, P = shape.nheads, shape.dstate, shape.headdim
    bc = (N,) if ngroups == 1 else (ngroups, N)
    cols = {k: [] for k in ("x", "dt", "Bm", "Cm", "Q", "E")}
    for b in seqs:
        r = _rng(seed, "token", step, b)
        cols["x"].append(r.standard_normal((H, P), dtype=np.float32))
        cols["dt"].append(np.exp(r.uniform(np.log(1e-3), np.log(1e-1), size=(H,))).astype(np.float32))
        cols["Bm"].append(r.standard_normal(bc, dtype=np.float32) / np.float32(np.sqrt(N)))
        cols["Cm"].append(r.standard_normal(bc, dtype=np.float32) / np.float32(np.sqrt(N)))
        cols["Q"].append(r.standard_normal((H, N), dtype=np.float32))
        cols["E"].append(r.standard_normal((H, P), dtype=np.float32) / np.float32(np.sqrt(P)))
    out = {k: np.stack(v) for k, v in cols.items()}
    res = {k: (torch.from_numpy(v) if k == "dt" else _cast(v, shape.dtype)) for k, v in out.items()}
    return res


def decode_A(shape: DecodeShape, seed: int = 0) -> torch.Tensor:
    return torch.from_numpy(_A(seed, shape.nheads))
