"""fp64 CPU gradients of the DART layer: the reference for its backward pass.

TEST INFRASTRUCTURE ONLY: only ``tests/`` may import this module; the CUDA
library never does, and nothing here touches the CUDA library.

The layer (DART abstract: "DART supports practical training"; Pith review of
DART, "Core claim" and "What carries the argument"; SSD view Eq. (4) cited in
the Pith review's "Axiom & Free-Parameter Ledger") is restated here with
plain PyTorch float64 CPU operations, token by token and memory by memory,
exactly as ``dart_oracle.c`` defines it:

  recurrence   H_t = exp(dt_t A_h) H_{t-1} + dt_t B_t x_t^T,  y_ssd_t = H_t^T C_t
  memory       dH[c] = the part of H at the chunk's last token e(c) that the
               chunk's own tokens contribute (an accumulator restarted at the
               first token of every chunk; C = ceil(L / S) chunks)
  SMA          for c < k(t) = t // S:  v = C_t^T dH[c],  key = dH[c] E_t,
               s = Q_t . key / sqrt(N);  o_t = sum_c softmax_c(s) v  (0 if k = 0)
               decayed variant: dH[c] scaled by exp(A_h sum_{r=e(c)+1}^{t} dt_r)
  output       y_t = y_ssd_t + g o_t

and the gradients of sum(dy * y) with respect to every input (x, dt, A, Bm,
Cm, Q, E, g, and an optional initial state) come from torch.autograd over that
restatement.  Nothing is blocked, fused or reordered beyond the definitions;
it is slow on purpose and meant for sequences of tens of tokens.  The tests
pin the restatement to the C oracle's forward and the gradients to central
finite differences and to closed forms.

Layouts as in ``dart_oracle.c``: x[B,L,H,P] dt[B,L,H] A[H] Bm[B,L,N] Cm[B,L,N]
Q[B,L,H,N] E[B,L,H,P] y[B,L,H,P] dH[B,H,C,N,P] init_state[B,H,N,P].  B and C
may also carry a group axis, Bm/Cm[B,L,G,N] with G dividing H: head h then
reads group h // (H / G) (Mamba-2 ngroups).
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np
import torch

_F64 = torch.float64


def _bc(M, b, t, h, H):
    """Row of B or C that head h reads at token t: [N]."""
    if M.dim() == 3:
        return M[b, t]
    return M[b, t, h // (H // M.shape[2])]


def _t(a, requires_grad=False):
    t = torch.as_tensor(np.asarray(a), dtype=_F64).clone()
    t.requires_grad_(requires_grad)
    return t


def ssd_scan(x, dt, A, Bm, Cm, chunk: int, init_state=None):
    """Token-by-token recurrence on torch tensors (differentiable).
    Returns (y_ssd [B,L,H,P], dH [B,H,C,N,P], states [B,H,C,N,P])."""
    Bz, L, H, P = x.shape
    N = Bm.shape[-1]
    S = chunk
    C = -(-L // S)
    ys, dHs, sts = [], [], []
    for b in range(Bz):
        yb, dHb, stb = [], [], []
        for h in range(H):
            Hs = init_state[b, h] if init_state is not None else torch.zeros(N, P, dtype=_F64)
            D = torch.zeros(N, P, dtype=_F64)
            yh, dHh, sth = [], [], []
            for t in range(L):
                if t % S == 0:
                    D = torch.zeros(N, P, dtype=_F64)   # a new chunk's own contribution
                decay = torch.exp(dt[b, t, h] * A[h])
                inp = dt[b, t, h] * torch.outer(_bc(Bm, b, t, h, H), x[b, t, h])
                Hs = decay * Hs + inp
                D = decay * D + inp
                yh.append(Hs.transpose(0, 1) @ _bc(Cm, b, t, h, H))
                if t % S == S - 1 or t == L - 1:        # the chunk closes at its last token
                    dHh.append(D)
                    sth.append(Hs)
            yb.append(torch.stack(yh))                   # [L, P]
            dHb.append(torch.stack(dHh))                 # [C, N, P]
            stb.append(torch.stack(sth))
        ys.append(torch.stack(yb, 1))                    # [L, H, P]
        dHs.append(torch.stack(dHb))                     # [H, C, N, P]
        sts.append(torch.stack(stb))
    assert all(d.shape[1] == C for d in dHs)
    return torch.stack(ys), torch.stack(dHs), torch.stack(sts)


def sma(Q, E, Cm, dH, chunk: int, dt=None, A=None):
    """Raw readout o [B,L,H,P] of state-memory attention (differentiable);
    with dt and A the memories are decayed from e(c) to t first."""
    Bz, L, H, N = Q.shape
    P = E.shape[-1]
    S = chunk
    inv_sqrt_n = 1.0 / math.sqrt(N)
    out = []
    for b in range(Bz):
        ob = []
        for t in range(L):
            k = t // S
            oh = []
            for h in range(H):
                if k == 0:
                    oh.append(torch.zeros(P, dtype=_F64))
                    continue
                scores, values = [], []
                for c in range(k):
                    M = dH[b, h, c]
                    if dt is not None:
                        M = torch.exp(A[h] * dt[b, c * S + S:t + 1, h].sum()) * M
                    key = M @ E[b, t, h]                  # [N]
                    values.append(_bc(Cm, b, t, h, H) @ M)  # [P]
                    scores.append((Q[b, t, h] @ key) * inv_sqrt_n)
                p = torch.softmax(torch.stack(scores), 0)
                oh.append((p[:, None] * torch.stack(values)).sum(0))
            ob.append(torch.stack(oh))
        out.append(torch.stack(ob))
    return torch.stack(out)


def layer_forward(x, dt, A, Bm, Cm, Q, E, chunk: int, g, init_state=None, decayed: bool = False):
    """y = y_ssd + g o on torch tensors; returns (y, y_ssd, o, dH, states)."""
    y_ssd, dH, st = ssd_scan(x, dt, A, Bm, Cm, chunk, init_state)
    o = sma(Q, E, Cm, dH, chunk, dt if decayed else None, A if decayed else None)
    return y_ssd + g * o, y_ssd, o, dH, st


def layer_grads(x, dt, A, Bm, Cm, Q, E, chunk: int, g: float, dy, init_state=None,
                decayed: bool = False) -> dict:
    """Gradients of sum(dy * y) for the layer forward: a dict with the forward
    outputs (y, y_ssd, o, dH, states as numpy float64) and dx, ddt, dA, dBm,
    dCm, dQ, dE, dg (and dinit_state when an initial state is given)."""
    names = ["x", "dt", "A", "Bm", "Cm", "Q", "E", "g"]
    vals = [x, dt, A, Bm, Cm, Q, E, np.float64(g)]
    ts = {n: _t(v, True) for n, v in zip(names, vals)}
    h0 = None if init_state is None else _t(init_state, True)
    y, y_ssd, o, dH, st = layer_forward(ts["x"], ts["dt"], ts["A"], ts["Bm"], ts["Cm"], ts["Q"], ts["E"],
                                        chunk, ts["g"], h0, decayed)
    loss = (y * _t(dy)).sum()
    want = [ts[n] for n in names] + ([h0] if h0 is not None else [])
    grads = torch.autograd.grad(loss, want, allow_unused=True)
    res = {"y": y.detach().numpy(), "y_ssd": y_ssd.detach().numpy(), "o": o.detach().numpy(),
           "dH": dH.detach().numpy(), "states": st.detach().numpy()}
    for n, gr, src in zip(names + ["init_state"], grads, want):
        res["d" + n] = (gr if gr is not None else torch.zeros_like(src)).detach().numpy()
    return res


def sma_grads(Q, E, Cm, dH, chunk: int, g: float, dy, dt=None, A=None) -> dict:
    """Gradients of sum(dy * g o) for SMA alone over given memories: o and
    dQ, dE, dCm, ddH, dg (and ddt, dA for the decayed variant)."""
    names = ["Q", "E", "Cm", "dH", "g"] + (["dt", "A"] if dt is not None else [])
    vals = [Q, E, Cm, dH, np.float64(g)] + ([dt, A] if dt is not None else [])
    ts = {n: _t(v, True) for n, v in zip(names, vals)}
    o = sma(ts["Q"], ts["E"], ts["Cm"], ts["dH"], chunk, ts.get("dt"), ts.get("A"))
    loss = (ts["g"] * o * _t(dy)).sum()
    grads = torch.autograd.grad(loss, [ts[n] for n in names], allow_unused=True)
    res = {"o": o.detach().numpy()}
    for n, gr in zip(names, grads):
        res["d" + n] = (gr if gr is not None else torch.zeros_like(ts[n])).detach().numpy()
    return res


def scan_grads(x, dt, A, Bm, Cm, chunk: int, dy, gdH, init_state=None) -> dict:
    """Gradients of sum(dy * y_ssd) + sum(gdH * dH) through the scan alone
    (gdH is what the SMA backward hands back for the memories): dx, ddt, dA,
    dBm, dCm (and dinit_state when an initial state is given), plus the
    forward outputs y_ssd, dH, states."""
    names = ["x", "dt", "A", "Bm", "Cm"]
    ts = {n: _t(v, True) for n, v in zip(names, (x, dt, A, Bm, Cm))}
    h0 = None if init_state is None else _t(init_state, True)
    y_ssd, dH, st = ssd_scan(ts["x"], ts["dt"], ts["A"], ts["Bm"], ts["Cm"], chunk, h0)
    loss = (y_ssd * _t(dy)).sum() + (dH * _t(gdH)).sum()
    want = [ts[n] for n in names] + ([h0] if h0 is not None else [])
    grads = torch.autograd.grad(loss, want, allow_unused=True)
    res = {"y_ssd": y_ssd.detach().numpy(), "dH": dH.detach().numpy(), "states": st.detach().numpy()}
    for n, gr, src in zip(names + ["init_state"], grads, want):
        res["d" + n] = (gr if gr is not None else torch.zeros_like(src)).detach().numpy()
    return res
