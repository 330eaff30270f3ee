"""Pins of the fp64 oracle to facts other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.dart_oracle.Oracle`` and raises
AssertionError when the oracle disagrees with a closed form, an identity of
the method, a textbook routine on explicitly materialised keys/values, or the
pages' worked example.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on deliberately broken builds and checks
that every planted mistake trips at least one.

Citations are to the pages' own sections: the Pith review of DART ("Core
claim", "What carries the argument", referee major comment 3 on Eq. (8),
circularity check on Eq. (14)), the DART abstract, and the paper-daily
summary's worked example.
"""
from __future__ import annotations

import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_layer(seed, Bz, L, H, P, N, dt_scale=0.3, a_max=2.0):
    r = np.random.default_rng(seed)
    return dict(
        x=r.standard_normal((Bz, L, H, P)).astype(np.float32),
        dt=(r.uniform(0.05, 1.0, (Bz, L, H)) * dt_scale).astype(np.float32),
        A=(-r.uniform(0.1, a_max, (H,))).astype(np.float32),
        Bm=(r.standard_normal((Bz, L, N)) / np.sqrt(N)).astype(np.float32),
        Cm=(r.standard_normal((Bz, L, N)) / np.sqrt(N)).astype(np.float32),
        Q=r.standard_normal((Bz, L, H, N)).astype(np.float32),
        E=(r.standard_normal((Bz, L, H, P)) / np.sqrt(P)).astype(np.float32),
    )


def _log_decay(dt, A):
    """a[b,t,h] = dt * A_h (the per-token log-decay, as float64)."""
    return dt.astype(np.float64) * A.astype(np.float64)[None, None, :]


def _close(a, b, tol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(np.max(np.abs(b)) if b.size else 0.0, 1e-300)
    assert err <= tol * max(scale, 1.0), f"{what}: max|err| {err:.3e} (scale {scale:.3e})"


# ----------------------------------------------------------------------------
# recurrence
# ----------------------------------------------------------------------------
def pin_closed_form_single_token(orc):
    """A single non-zero input token s: with the recurrence
    H_t = exp(dt_t A) H_{t-1} + dt_t B_t x_t^T, the state for t >= s is
    exp(sum_{r=s+1..t} dt_r A) dt_s B_s x_s^T and y_t = H_t^T C_t; before s
    everything is zero.  The chunk holding s owns the whole contribution."""
    Bz, L, H, P, N, S = 1, 24, 2, 3, 5, 8
    inp = _rand_layer(1, Bz, L, H, P, N)
    s = 10
    x = np.zeros_like(inp["x"])
    x[0, s] = inp["x"][0, s]
    y, dH, st = orc.ssd_scan(x, inp["dt"], inp["A"], inp["Bm"], inp["Cm"], S)
    a = _log_decay(inp["dt"], inp["A"])[0]  # [L,H]
    for h in range(H):
        outer = inp["dt"][0, s, h] * np.outer(inp["Bm"][0, s].astype(np.float64),
                                              x[0, s, h].astype(np.float64))
        for t in range(L):
            if t < s:
                expect_y = np.zeros(P)
            else:
                Ht = np.exp(a[s + 1:t + 1, h].sum()) * outer
                expect_y = Ht.T @ inp["Cm"][0, t].astype(np.float64)
            _close(y[0, t, h], expect_y, 1e-12, f"y[t={t},h={h}]")
        for c in range(L // S):
            e = c * S + S - 1
            exp_dh = np.exp(a[s + 1:e + 1, h].sum()) * outer if c == s // S else np.zeros((N, P))
            _close(dH[0, h, c], exp_dh, 1e-12, f"dH[c={c}]")
            exp_st = np.exp(a[s + 1:e + 1, h].sum()) * outer if e >= s else np.zeros((N, P))
            _close(st[0, h, c], exp_st, 1e-12, f"states[c={c}]")


def pin_quadratic_form(orc):
    """The SSD (structured masked attention) form of Mamba-2 -- Eq. (4) of the
    SSD view the Pith review cites: y_t = sum_{s<=t} (C_t . B_s)
    exp(sum_{r=s+1..t} a_r) dt_s x_s, plus exp(sum_{r<=t} a_r) C_t^T H_init.
    Written here as an explicit double loop over (t, s)."""
    Bz, L, H, P, N, S = 2, 32, 3, 4, 6, 8
    inp = _rand_layer(2, Bz, L, H, P, N)
    r = np.random.default_rng(22)
    h0 = r.standard_normal((Bz, H, N, P))
    y, _, _ = orc.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], S, init_state=h0)
    a = _log_decay(inp["dt"], inp["A"])
    cum = np.cumsum(a, axis=1)  # inclusive prefix sums over t
    Bm, Cm, x, dt = (inp[k].astype(np.float64) for k in ("Bm", "Cm", "x", "dt"))
    expect = np.zeros_like(y)
    for b in range(Bz):
        for h in range(H):
            for t in range(L):
                acc = np.exp(cum[b, t, h]) * (h0[b, h].T @ Cm[b, t])
                for s in range(t + 1):
                    w = (Cm[b, t] @ Bm[b, s]) * np.exp(cum[b, t, h] - cum[b, s, h]) * dt[b, s, h]
                    acc = acc + w * x[b, s, h]
                expect[b, t, h] = acc
    _close(y, expect, 1e-11, "y_ssd vs quadratic form")


def pin_chunk_memory_definition(orc):
    """dH[c] is what chunk c contributes to the state at its own last token
    e(c) (Pith review, "What carries the argument"; referee comment 3 on
    Eq. (8)): sum_{s in c} exp(sum_{r=s+1..e(c)} a_r) dt_s B_s x_s^T.  The
    boundary states obey states[c] = exp(sum_{r in c} a_r) states[c-1] + dH[c]
    and the final state is the decayed sum of all chunk memories."""
    Bz, L, H, P, N, S = 1, 40, 2, 3, 4, 8
    inp = _rand_layer(3, Bz, L, H, P, N)
    _, dH, st = orc.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], S)
    a = _log_decay(inp["dt"], inp["A"])[0]
    Bm, x, dt = inp["Bm"][0].astype(np.float64), inp["x"][0].astype(np.float64), inp["dt"][0]
    C = L // S
    for h in range(H):
        for c in range(C):
            e = c * S + S - 1
            m = np.zeros((N, P))
            for s in range(c * S, e + 1):
                m += np.exp(a[s + 1:e + 1, h].sum()) * dt[s, h] * np.outer(Bm[s], x[s, h])
            _close(dH[0, h, c], m, 1e-12, f"dH[h={h},c={c}]")
            prev = st[0, h, c - 1] if c else np.zeros((N, P))
            _close(st[0, h, c], np.exp(a[c * S:e + 1, h].sum()) * prev + dH[0, h, c], 1e-12,
                   "states recursion")
        final = sum(np.exp(a[c * S + S:, h].sum()) * dH[0, h, c] for c in range(C))
        _close(st[0, h, C - 1], final, 1e-12, "final state = decayed sum of dH")


def pin_init_state_continuation(orc):
    """Running the recurrence over L1 + L2 tokens equals running L1 tokens and
    continuing L2 tokens from the boundary state (the recurrence is Markov in
    H).  Chunk memories of the continued part are unaffected by the carried
    state."""
    Bz, L, H, P, N, S = 1, 32, 2, 4, 4, 8
    inp = _rand_layer(4, Bz, L, H, P, N)
    keys = ("x", "dt", "Bm", "Cm")
    y, dH, st = orc.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], S)
    first = {k: inp[k][:, :16] for k in keys}
    second = {k: inp[k][:, 16:] for k in keys}
    y1, _, st1 = orc.ssd_scan(first["x"], first["dt"], inp["A"], first["Bm"], first["Cm"], S)
    y2, dH2, st2 = orc.ssd_scan(second["x"], second["dt"], inp["A"], second["Bm"], second["Cm"], S,
                                init_state=st1[:, :, -1])
    _close(np.concatenate([y1, y2], 1), y, 1e-12, "continued y")
    _close(dH2, dH[:, :, 2:], 1e-12, "continued dH")
    _close(st2, st[:, :, 2:], 1e-12, "continued states")


# ----------------------------------------------------------------------------
# state-memory attention
# ----------------------------------------------------------------------------
def pin_single_prior_chunk(orc):
    """A token of chunk 1 sees exactly one memory, so its softmax weight is 1
    and o_t = C_t^T dH[0] whatever Q and E are (Pith review, "Core claim":
    value = C_t dH[c]; mask c < chunk(t))."""
    Bz, L, H, P, N, S = 1, 16, 2, 5, 3, 8
    inp = _rand_layer(5, Bz, L, H, P, N)
    dH = np.random.default_rng(55).standard_normal((Bz, H, 2, N, P))
    r = orc.sma(inp["Q"], inp["E"], inp["Cm"], dH, S, g=1.0)
    for h in range(H):
        for t in range(S, 2 * S):
            _close(r["o"][0, t, h], inp["Cm"][0, t].astype(np.float64) @ dH[0, h, 0], 1e-13,
                   f"o[t={t}]")
        assert np.all(r["o"][0, :S, h] == 0.0), "chunk 0 has no memory"


def pin_bruteforce_attention(orc):
    """Materialise, per token, the key matrix K_t[c] = (dH[c] E_t)^T and value
    matrix V_t[c] = C_t^T dH[c] over c < chunk(t), then call torch's
    scaled-dot-product attention (a textbook softmax(q K^T / sqrt(N)) V)."""
    Bz, L, H, P, N, S = 2, 48, 2, 5, 7, 8
    inp = _rand_layer(6, Bz, L, H, P, N)
    dH = np.random.default_rng(66).standard_normal((Bz, H, L // S, N, P))
    g = 0.75
    ys = np.random.default_rng(67).standard_normal((Bz, L, H, P))
    r = orc.sma(inp["Q"], inp["E"], inp["Cm"], dH, S, g=g, y_ssd=ys)
    Q = torch.from_numpy(inp["Q"].astype(np.float64))
    E = torch.from_numpy(inp["E"].astype(np.float64))
    Cm = torch.from_numpy(inp["Cm"].astype(np.float64))
    M = torch.from_numpy(dH)
    for b in range(Bz):
        for h in range(H):
            for t in range(L):
                k = t // S
                if k == 0:
                    expect = torch.zeros(P, dtype=torch.float64)
                else:
                    Kt = torch.einsum("cnp,p->cn", M[b, h, :k], E[b, t, h])       # [k, N]
                    Vt = torch.einsum("n,cnp->cp", Cm[b, t], M[b, h, :k])         # [k, P]
                    expect = torch.nn.functional.scaled_dot_product_attention(
                        Q[b, t, h][None, None, None, :], Kt[None, None], Vt[None, None])[0, 0, 0]
                _close(r["o"][b, t, h], expect.numpy(), 1e-12, f"o[b={b},t={t},h={h}]")
                _close(r["y"][b, t, h], ys[b, t, h] + g * expect.numpy(), 1e-12, "gated y")


def pin_worked_example(orc):
    """The paper-daily summary's L=8, S=4, N=2 example, finished in DART's
    terms (tests/golden/worked_example.txt)."""
    vals = {}
    with open(os.path.join(GOLDEN, "worked_example.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if line:
                vals[line[0]] = [float(v) for v in line[1:]]
    L, S, N, P = (int(vals[k][0]) for k in ("L", "S", "N", "P"))
    g = vals["g"][0]
    q = np.array(vals["q"], np.float32)
    x = np.zeros((1, L, 1, P), np.float32)
    Bm = np.zeros((1, L, N), np.float32)
    x[0, 0, 0, 0] = Bm[0, 0, 0] = 1.0
    x[0, 1, 0, 1] = Bm[0, 1, 1] = 1.0
    Cm = np.zeros((1, L, N), np.float32)
    Cm[0, :, 0] = 1.0
    E = np.zeros((1, L, 1, P), np.float32)
    E[0, :, 0, 0] = 1.0
    Q = np.broadcast_to(q, (1, L, 1, N)).copy()
    dt = np.ones((1, L, 1), np.float32)
    A = np.zeros((1,), np.float32)
    y_ssd, dH, _ = orc.ssd_scan(x, dt, A, Bm, Cm, S)
    np.testing.assert_allclose(dH[0, 0, 0].ravel(), vals["dH_c0"], atol=1e-15)
    r = orc.sma(Q, E, Cm, dH, S, g=g, y_ssd=y_ssd, want_scores=True)
    np.testing.assert_allclose(r["scores"][0, 0, 4, 0], vals["score_t4_c0"][0], rtol=1e-14)
    for t in range(L):
        np.testing.assert_allclose(r["y"][0, t, 0], vals[f"y_t{t}"], atol=1e-14)


def pin_gate_zero(orc):
    """g = 0 removes the SMA branch (Pith review, "If this is right": the
    SMA-removal ablation gives Mamba-2): y equals y_ssd exactly."""
    Bz, L, H, P, N, S = 1, 32, 2, 4, 6, 8
    inp = _rand_layer(7, Bz, L, H, P, N)
    r = orc.layer_forward(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], inp["Q"], inp["E"],
                          S, g=0.0)
    assert np.array_equal(r["y"], r["y_ssd"])
    assert np.any(r["o"] != 0.0)


def pin_one_hot_mask(orc):
    """One-hot memories dH[c] = (c+1) e_0 e_0^T with a query that makes the
    score grow steeply with c: the softmax is a one-hot on the last allowed
    chunk, so o_t[0] = chunk(t) * C_t[0].  An off-by-one in the causal mask
    (c < chunk(t)) moves the value by a whole chunk."""
    Bz, L, H, P, N, S = 1, 48, 1, 3, 4, 8
    C = L // S
    dH = np.zeros((Bz, H, C, N, P))
    for c in range(C):
        dH[0, 0, c, 0, 0] = c + 1.0
    Q = np.zeros((Bz, L, H, N), np.float32)
    Q[..., 0] = 400.0
    E = np.zeros((Bz, L, H, P), np.float32)
    E[..., 0] = 1.0
    Cm = np.random.default_rng(8).uniform(0.5, 1.5, (Bz, L, N)).astype(np.float32)
    r = orc.sma(Q, E, Cm, dH, S, g=1.0)
    for t in range(L):
        k = t // S
        expect = k * float(Cm[0, t, 0]) if k else 0.0
        assert abs(r["o"][0, t, 0, 0] - expect) < 1e-9 * max(1.0, expect), (t, r["o"][0, t, 0, 0], expect)
        assert np.all(r["o"][0, t, 0, 1:] == 0.0)


def pin_sampled_rows(orc):
    """Computing a sample of token positions gives the same rows as the full
    computation (the sample path is what the large-size parity tests use)."""
    Bz, L, H, P, N, S = 2, 40, 2, 3, 5, 8
    inp = _rand_layer(9, Bz, L, H, P, N)
    dH = np.random.default_rng(99).standard_normal((Bz, H, L // S, N, P))
    full = orc.sma(inp["Q"], inp["E"], inp["Cm"], dH, S, g=0.3)
    tok = [0, 7, 8, 15, 16, 39, 22]
    part = orc.sma(inp["Q"], inp["E"], inp["Cm"], dH, S, g=0.3, tokens=tok)
    assert np.array_equal(part["o"], full["o"][:, tok])


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------
def pin_decode_matches_prefill(orc):
    """Forward over L + S tokens equals forward over L tokens followed by S
    single-token decode steps against the cache of chunk memories (DART
    abstract: the inference cache is the chunk state memories), including the
    append when the last token closes its chunk."""
    Bz, L, H, P, N, S = 2, 24, 2, 4, 5, 8
    T = L + S
    inp = _rand_layer(10, Bz, T, H, P, N)
    g = 0.6
    full = orc.layer_forward(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], inp["Q"],
                             inp["E"], S, g)
    pre = orc.layer_forward(*(inp[k][:, :L] if k != "A" else inp[k]
                              for k in ("x", "dt", "A", "Bm", "Cm", "Q", "E")), S, g)
    cmax = L // S + 2
    cache = np.zeros((Bz, H, cmax, N, P))
    cache[:, :, :L // S] = pre["dH"]
    state = np.ascontiguousarray(pre["states"][:, :, -1])
    dcur = np.zeros((Bz, H, N, P))
    nch = np.full((Bz,), L // S, np.int32)
    pos = np.zeros((Bz,), np.int32)
    for t in range(L, T):
        y = orc.decode_step(inp["x"][:, t], inp["dt"][:, t], inp["A"], inp["Bm"][:, t],
                            inp["Cm"][:, t], inp["Q"][:, t], inp["E"][:, t], g, state, dcur,
                            cache, nch, pos, S)
        _close(y, full["y"][:, t], 1e-12, f"decode y at t={t}")
    assert np.all(nch == L // S + 1) and np.all(pos == 0)
    _close(cache[:, :, L // S], full["dH"][:, :, L // S], 1e-12, "appended memory")
    assert np.all(dcur == 0.0)
    _close(state, full["states"][:, :, -1], 1e-12, "decode state")


def pin_partial_last_chunk(orc):
    """A sequence that is not a multiple of S ends in a partial chunk, which
    closes at token L-1: its dH and state follow the same definitions with
    e(C-1) = L-1 (brute force below), the full chunks are those of the
    length-32 prefix, and every output row (y_ssd and the layer output) is
    the same row of a longer sequence with the same leading inputs
    (causality: row t reads only tokens <= t and chunk memories c < k(t))."""
    Bz, L, H, P, N, S = 1, 37, 2, 3, 4, 8
    T = 48
    inp = _rand_layer(21, Bz, T, H, P, N)
    cut = {k: (v[:, :L] if k != "A" else v) for k, v in inp.items()}
    y, dH, st = orc.ssd_scan(cut["x"], cut["dt"], cut["A"], cut["Bm"], cut["Cm"], S)
    C = -(-L // S)
    assert dH.shape[2] == C == 5
    a = _log_decay(cut["dt"], cut["A"])[0]
    Bm, x, dt = cut["Bm"][0].astype(np.float64), cut["x"][0].astype(np.float64), cut["dt"][0]
    c0 = (C - 1) * S
    for h in range(H):
        m = np.zeros((N, P))
        for s_ in range(c0, L):
            m += np.exp(a[s_ + 1:L, h].sum()) * dt[s_, h] * np.outer(Bm[s_], x[s_, h])
        _close(dH[0, h, C - 1], m, 1e-12, f"partial dH[h={h}]")
        _close(st[0, h, C - 1], np.exp(a[c0:L, h].sum()) * st[0, h, C - 2] + m, 1e-12, "partial state")
    y32, dH32, st32 = orc.ssd_scan(*(cut[k][:, :32] if k != "A" else cut[k]
                                     for k in ("x", "dt", "A", "Bm", "Cm")), S)
    _close(dH[:, :, :4], dH32, 1e-12, "full chunks of the ragged scan")
    _close(st[:, :, :4], st32, 1e-12, "full-chunk states of the ragged scan")
    g = 0.7
    ragged = orc.layer_forward(*(cut[k] for k in ("x", "dt", "A", "Bm", "Cm", "Q", "E")), S, g)
    longer = orc.layer_forward(*(inp[k] for k in ("x", "dt", "A", "Bm", "Cm", "Q", "E")), S, g)
    _close(ragged["y_ssd"], longer["y_ssd"][:, :L], 1e-12, "ragged y_ssd = prefix rows")
    _close(ragged["y"], longer["y"][:, :L], 1e-12, "ragged layer output = prefix rows")


def pin_ragged_prefill_then_decode(orc):
    """A prefill that stops inside a chunk hands its partial chunk to decode:
    state = states[C-1], running contribution = dH[C-1], C-1 cached memories,
    position L mod S.  Decoding the remaining tokens of a longer sequence
    reproduces the full forward's outputs, its appended memory and its final
    state (the decode rule and the chunked scan are separate code paths)."""
    Bz, L, H, P, N, S = 2, 21, 2, 3, 5, 8
    T = 40
    inp = _rand_layer(22, Bz, T, H, P, N)
    g = 0.4
    full = orc.layer_forward(*(inp[k] for k in ("x", "dt", "A", "Bm", "Cm", "Q", "E")), S, g)
    pre = orc.layer_forward(*(inp[k][:, :L] if k != "A" else inp[k]
                              for k in ("x", "dt", "A", "Bm", "Cm", "Q", "E")), S, g)
    Cfull = L // S
    cmax = T // S + 1
    cache = np.zeros((Bz, H, cmax, N, P))
    cache[:, :, :Cfull] = pre["dH"][:, :, :Cfull]
    state = np.ascontiguousarray(pre["states"][:, :, -1])
    dcur = np.ascontiguousarray(pre["dH"][:, :, -1])
    nch = np.full((Bz,), Cfull, np.int32)
    pos = np.full((Bz,), L % S, np.int32)
    for t in range(L, T):
        y = orc.decode_step(inp["x"][:, t], inp["dt"][:, t], inp["A"], inp["Bm"][:, t],
                            inp["Cm"][:, t], inp["Q"][:, t], inp["E"][:, t], g, state, dcur,
                            cache, nch, pos, S)
        _close(y, full["y"][:, t], 1e-12, f"decode y at t={t}")
    assert np.all(nch == T // S) and np.all(pos == 0)
    _close(cache[:, :, :T // S], full["dH"], 1e-12, "memories after the handoff")
    _close(state, full["states"][:, :, -1], 1e-12, "decode state")


def pin_cache_ratio(orc):
    """Eq. (14) (Pith review, circularity check): per head the DART cache is
    M N P elements (M = L/S chunk memories) against 2 L P for a token-level
    attention cache, a ratio of N/(2S): 0.25 at S=256, N=128 (the abstract's
    75% saving).  Checked on the shapes of the 128-memory decode cache."""
    del orc
    L, S, N, P = 32768, 256, 128, 64
    dart = (L // S) * N * P
    attn = 2 * L * P
    assert dart / attn == N / (2 * S) == 0.25


# ----------------------------------------------------------------------------
# decayed-memory variant (referee major comment 3 on Eq. (8): the memories
# carried to t by the recurrence's decay, exp(sum_{r=e(c)+1..t} a_r) dH[c])
# ----------------------------------------------------------------------------
def _recurrence_states(inp, b, h, start, stop, reset_at=None):
    """Plain token-by-token recurrence H_t = exp(dt_t A) H_{t-1} + dt_t B_t x_t^T
    for one (b, h) from zero at ``start``; with ``reset_at`` (a set of
    positions) the state restarts from zero before those tokens.  Returns
    {t: H_t}."""
    N = inp["Bm"].shape[-1]
    P = inp["x"].shape[-1]
    Hs = np.zeros((N, P))
    out = {}
    for t in range(start, stop):
        if reset_at is not None and t in reset_at:
            Hs = np.zeros((N, P))
        dtt = float(inp["dt"][b, t, h])
        Hs = np.exp(dtt * float(inp["A"][h])) * Hs + dtt * np.outer(
            inp["Bm"][b, t].astype(np.float64), inp["x"][b, t, h].astype(np.float64))
        out[t] = Hs
    return out


def pin_decayed_memories_sum_to_state(orc):
    """With decayed memories, sum_{c < k(t)} of the carried dH[c] is exactly
    the part of the SSM state H_t that tokens before chunk k(t) left behind:
    H_t minus the state the tokens of chunk k(t) up to t build from zero.
    With Q = 0 every score is 0, the softmax is uniform over the k(t)
    memories and o_t = C_t^T (H_t - H_t^in) / k(t).  Both states come from a
    token-by-token recurrence written here; L is not a multiple of S."""
    Bz, L, H, P, N, S = 2, 44, 2, 3, 4, 8
    inp = _rand_layer(13, Bz, L, H, P, N, dt_scale=0.5)
    Q = np.zeros_like(inp["Q"])
    r = orc.layer_forward(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], Q, inp["E"], S,
                          g=1.0, decayed=True)
    chunk_starts = set(range(0, L, S))
    for b in range(Bz):
        for h in range(H):
            full = _recurrence_states(inp, b, h, 0, L)
            inner = _recurrence_states(inp, b, h, 0, L, reset_at=chunk_starts)
            for t in range(L):
                k = t // S
                if k == 0:
                    assert np.all(r["o"][b, t, h] == 0.0)
                    continue
                expect = inp["Cm"][b, t].astype(np.float64) @ (full[t] - inner[t]) / k
                _close(r["o"][b, t, h], expect, 1e-11, f"decayed o[b={b},t={t},h={h}]")


def pin_decayed_bruteforce_attention(orc):
    """Decayed keys and values materialised per token and fed to torch's
    scaled-dot-product attention.  The factor for memory c at token t is the
    fraction of a unit placed in the state at e(c) that survives to t, taken
    from a scalar run of the recurrence with no further input.  With A = 0
    nothing decays and the variant equals the raw-memory SMA."""
    Bz, L, H, P, N, S = 1, 40, 2, 5, 6, 8
    inp = _rand_layer(14, Bz, L, H, P, N, dt_scale=0.6)
    C = L // S
    dH = np.random.default_rng(144).standard_normal((Bz, H, C, N, P))
    ys = np.random.default_rng(145).standard_normal((Bz, L, H, P))
    g = 0.5
    r = orc.sma(inp["Q"], inp["E"], inp["Cm"], dH, S, g=g, y_ssd=ys, dt=inp["dt"], A=inp["A"])
    Q, E, Cm, M = (torch.from_numpy(v.astype(np.float64)) for v in
                   (inp["Q"], inp["E"], inp["Cm"], dH))
    for h in range(H):
        surv = np.zeros((C, L))   # surv[c, t]: what is left at t of a unit held at e(c)
        for c in range(C):
            z = 1.0
            for t in range(c * S + S, L):
                z = np.exp(float(inp["dt"][0, t, h]) * float(inp["A"][h])) * z
                surv[c, t] = z
        for t in range(L):
            k = t // S
            if k == 0:
                continue
            w = torch.from_numpy(surv[:k, t])[:, None]
            Kt = w * torch.einsum("cnp,p->cn", M[0, h, :k], E[0, t, h])
            Vt = w * torch.einsum("n,cnp->cp", Cm[0, t], M[0, h, :k])
            expect = torch.nn.functional.scaled_dot_product_attention(
                Q[0, t, h][None, None, None, :], Kt[None, None], Vt[None, None])[0, 0, 0].numpy()
            _close(r["o"][0, t, h], expect, 1e-12, f"decayed o[t={t},h={h}]")
            _close(r["y"][0, t, h], ys[0, t, h] + g * expect, 1e-12, "decayed gated y")
    zeroA = np.zeros_like(inp["A"])
    r0 = orc.sma(inp["Q"], inp["E"], inp["Cm"], dH, S, g=g, y_ssd=ys, dt=inp["dt"], A=zeroA)
    raw = orc.sma(inp["Q"], inp["E"], inp["Cm"], dH, S, g=g, y_ssd=ys)
    assert np.array_equal(r0["y"], raw["y"]), "A = 0: decayed and raw memories differ"


def pin_decayed_decode_matches_prefill(orc):
    """Decayed memories in decode: each cached memory carries the log-decay
    accumulated since its chunk closed (the slot of a memory not yet appended
    holds junk until the append sets it).  (1) Decoding a whole sequence from an
    empty cache, and (2) decoding on from a prefill that stops inside a chunk,
    with every cached memory's log-decay set to sum_{r=e(c)+1}^{L-1} dt_r A_h
    (summed here from dt), both reproduce the decayed-memory layer forward
    token by token, which the recurrence pins above."""
    Bz, H, P, N, S = 2, 2, 3, 4, 8
    T = 4 * S + 3
    inp = _rand_layer(23, Bz, T, H, P, N, dt_scale=0.4)
    g = 0.8
    keys = ("x", "dt", "A", "Bm", "Cm", "Q", "E")
    full = orc.layer_forward(*(inp[k] for k in keys), S, g, decayed=True)
    cmax = T // S + 1
    # (1) from an empty cache
    cache = np.zeros((Bz, H, cmax, N, P))
    state = np.zeros((Bz, H, N, P))
    dcur = np.zeros((Bz, H, N, P))
    memlog = np.full((Bz, H, cmax), 7.0)   # slots of memories not yet appended hold junk
    nch = np.zeros((Bz,), np.int32)
    pos = np.zeros((Bz,), np.int32)
    for t in range(T):
        y = orc.decode_step(inp["x"][:, t], inp["dt"][:, t], inp["A"], inp["Bm"][:, t],
                            inp["Cm"][:, t], inp["Q"][:, t], inp["E"][:, t], g, state, dcur,
                            cache, nch, pos, S, memlog=memlog)
        _close(y, full["y"][:, t], 1e-12, f"decayed decode y at t={t}")
    a = _log_decay(inp["dt"], inp["A"])
    for c in range(T // S):
        _close(memlog[:, :, c], a[:, (c + 1) * S:T].sum(1), 1e-12, f"memlog[{c}]")
    # (2) from a ragged prefill
    L = 2 * S + 5
    pre = orc.layer_forward(*(inp[k][:, :L] if k != "A" else inp[k] for k in keys), S, g, decayed=True)
    Cfull = L // S
    cache = np.zeros((Bz, H, cmax, N, P))
    cache[:, :, :Cfull] = pre["dH"][:, :, :Cfull]
    state = np.ascontiguousarray(pre["states"][:, :, -1])
    dcur = np.ascontiguousarray(pre["dH"][:, :, -1])
    memlog = np.full((Bz, H, cmax), 7.0)
    for c in range(Cfull):
        memlog[:, :, c] = a[:, (c + 1) * S:L].sum(1)
    nch = np.full((Bz,), Cfull, np.int32)
    pos = np.full((Bz,), L % S, np.int32)
    for t in range(L, T):
        y = orc.decode_step(inp["x"][:, t], inp["dt"][:, t], inp["A"], inp["Bm"][:, t],
                            inp["Cm"][:, t], inp["Q"][:, t], inp["E"][:, t], g, state, dcur,
                            cache, nch, pos, S, memlog=memlog)
        _close(y, full["y"][:, t], 1e-12, f"decayed decode after prefill, y at t={t}")


# ----------------------------------------------------------------------------
# fp8 (OCP E4M3) decode cache: rows of P values as codes times 2^k
# ----------------------------------------------------------------------------
def _torch_e4m3_codes(v):
    """Library rounding of float32-exact values to float8_e4m3fn codes."""
    t = torch.from_numpy(np.ascontiguousarray(v, np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _torch_e4m3_values(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def pin_e4m3_rows_match_library(orc):
    """Codes equal torch's float8_e4m3fn cast of x 2^-k (round to nearest even)
    for rows of every magnitude, exact ties and subnormals included; the row
    exponent is the smallest k with max|row| 2^-k <= 448 (so the scaled max
    lies in (224, 448]); dequantized values are the library's code values
    times 2^k exactly; every finite code survives a round trip."""
    r = np.random.default_rng(31)
    P = 64
    rows = []
    for amax in np.exp(r.uniform(np.log(1e-7), np.log(1e3), 200)):
        row = (r.standard_normal(P) * amax / 3).astype(np.float32)
        row[r.integers(0, P)] = np.float32(amax) * (1 if r.random() < 0.5 else -1)
        rows.append(row)
    rows.append(np.zeros(P, np.float32))
    one = np.zeros(P, np.float32)
    one[5] = -3.0e-3
    rows.append(one)
    # exact midpoints between neighbouring codes (ties), in a row whose max is 448
    vals = _torch_e4m3_values(np.arange(0, 0x7E, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    for i in range(0, len(mids), P - 1):
        row = np.zeros(P, np.float32)
        chunk = mids[i:i + P - 1]
        row[:len(chunk)] = chunk
        row[-1] = 448.0
        rows.append(row)
    X = np.stack(rows).astype(np.float64)
    codes, exps, deq = orc.quantize_e4m3(X)
    amax = np.abs(X).max(1)
    nz = amax > 0
    scaled_max = amax[nz] * np.exp2(-exps[nz].astype(np.float64))
    assert np.all(scaled_max <= 448.0) and np.all(scaled_max > 224.0), "row exponent"
    want = _torch_e4m3_codes(X * np.exp2(-exps.astype(np.float64))[:, None])
    assert np.array_equal(codes, want), f"{np.count_nonzero(codes != want)} codes differ from the library"
    assert np.array_equal(deq, _torch_e4m3_values(codes) * np.exp2(exps.astype(np.float64))[:, None])
    # round trip of every finite code (0x7F / 0xFF are NaN in E4M3FN)
    fin = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    v = _torch_e4m3_values(fin)
    row = np.zeros((1, 4 * P))
    row[0, :len(v)] = v
    row[0, -1] = 448.0
    c2, e2, _ = orc.quantize_e4m3(row)
    assert e2[0] == 0 and np.array_equal(c2[0, :len(v)], fin)


def pin_e4m3_decode_append(orc):
    """With an E4M3 cache the decode step reads the dequantized memories and
    quantizes the memory it appends: run side by side with the plain-cache
    decode from the same cache, the outputs agree exactly until the append,
    the appended slot is the quantizer's output for the plain slot, and the
    next outputs equal the plain decode run with that slot quantized."""
    Bz, H, P, N, S = 2, 2, 8, 4, 4
    T = 6
    inp = _rand_layer(32, Bz, T, H, P, N)
    cmax = 3
    r = np.random.default_rng(33)
    _, _, cache0 = orc.quantize_e4m3(r.standard_normal((Bz, H, cmax, N, P)) * 0.3)
    st = [dict(cache=cache0.copy(), state=r.standard_normal((Bz, H, N, P)) * 0.1,
               dcur=r.standard_normal((Bz, H, N, P)) * 0.05, nch=np.full((Bz,), 1, np.int32),
               pos=np.full((Bz,), 1, np.int32)) for _ in range(2)]
    st[1] = {k: v.copy() for k, v in st[0].items()}
    g = 0.9

    def step(sd, t, e4m3):
        return orc.decode_step(inp["x"][:, t], inp["dt"][:, t], inp["A"], inp["Bm"][:, t], inp["Cm"][:, t],
                               inp["Q"][:, t], inp["E"][:, t], g, sd["state"], sd["dcur"], sd["cache"],
                               sd["nch"], sd["pos"], S, cache_e4m3=e4m3)
    for t in range(3):   # positions 1, 2, 3: the third step appends memory 1
        ya, yb = step(st[0], t, True), step(st[1], t, False)
        assert np.array_equal(ya, yb), f"step {t}"
    assert np.all(st[0]["nch"] == 2)
    _, _, q = orc.quantize_e4m3(st[1]["cache"][:, :, 1])
    assert np.array_equal(st[0]["cache"][:, :, 1], q), "appended slot = quantized memory"
    assert not np.array_equal(q, st[1]["cache"][:, :, 1])
    st[1]["cache"][:, :, 1] = q
    for t in range(3, T):
        ya, yb = step(st[0], t, True), step(st[1], t, False)
        assert np.array_equal(ya, yb), f"step {t}"


# ----------------------------------------------------------------------------
# B and C shared by groups of heads (Mamba-2 ngroups)
# ----------------------------------------------------------------------------
def pin_ngroups_split_into_independent_problems(orc):
    """With G groups head h reads B and C of group h // (H / G).  A layer with
    H = 4 heads in G = 2 groups (and G = 4: every head its own B, C) equals G
    separate layers of H / G heads each fed its own group's B and C through
    the single-group path pinned above: scan outputs, SMA and layer output,
    and a decode step."""
    Bz, L, H, P, N, S = 2, 20, 4, 3, 4, 8
    r = np.random.default_rng(41)
    for G in (2, 4):
        inp = _rand_layer(41 + G, Bz, L, H, P, N)
        Bg = (r.standard_normal((Bz, L, G, N)) / np.sqrt(N)).astype(np.float32)
        Cg = (r.standard_normal((Bz, L, G, N)) / np.sqrt(N)).astype(np.float32)
        full = orc.layer_forward(inp["x"], inp["dt"], inp["A"], Bg, Cg, inp["Q"], inp["E"], S, 0.6)
        hg = H // G
        for g in range(G):
            hs = slice(g * hg, (g + 1) * hg)
            part = orc.layer_forward(inp["x"][:, :, hs], inp["dt"][:, :, hs], inp["A"][hs], Bg[:, :, g],
                                     Cg[:, :, g], inp["Q"][:, :, hs], inp["E"][:, :, hs], S, 0.6)
            for k in ("y", "y_ssd", "o"):
                assert np.array_equal(full[k][:, :, hs], part[k]), (G, g, k)
            for k in ("dH", "states"):
                assert np.array_equal(full[k][:, hs], part[k]), (G, g, k)
        # one decode step from the prefill's last boundary
        cmax = L // S + 1
        nc = L // S
        t = L - 1
        rr = np.random.default_rng(42)
        cache = np.zeros((Bz, H, cmax, N, P))
        cache[:, :, :nc] = full["dH"][:, :, :nc]
        state = rr.standard_normal((Bz, H, N, P))
        dcur = rr.standard_normal((Bz, H, N, P)) * 0.1
        nch = np.full((Bz,), nc, np.int32)
        pos = np.full((Bz,), 3, np.int32)
        ys = {}
        for g in [None] + list(range(G)):
            hs = slice(None) if g is None else slice(g * hg, (g + 1) * hg)
            Bt = Bg[:, t] if g is None else Bg[:, t, g]
            Ct = Cg[:, t] if g is None else Cg[:, t, g]
            st, dc, ca = (np.array(a[:, hs], copy=True, order="C") for a in (state, dcur, cache))
            ys[g] = orc.decode_step(inp["x"][:, t, hs], inp["dt"][:, t, hs], inp["A"][hs], Bt, Ct,
                                    inp["Q"][:, t, hs], inp["E"][:, t, hs], 0.6, st, dc, ca,
                                    nch.copy(), pos.copy(), S)
        for g in range(G):
            assert np.array_equal(ys[None][:, g * hg:(g + 1) * hg], ys[g]), (G, g, "decode")


# ----------------------------------------------------------------------------
# gradients through the scan (the training pass of the DART abstract)
# ----------------------------------------------------------------------------
def pin_scan_backward_matches_autograd(orc):
    """The C oracle's reverse-mode walk of the token recurrence equals
    autograd over the float64 torch restatement of the same recurrence
    (``oracle/dart_backward.py``, itself pinned to central finite differences
    of the C forward in ``test_oracle_backward.py``), to 1e-10 relative: one
    group and two groups of heads, with and without an initial state and a
    memory gradient, ragged last chunk."""
    from oracle import dart_backward
    for seed, (Bz, L, H, P, N, S, G, init, gmem) in enumerate([
            (1, 3 * 8 + 5, 2, 3, 4, 8, 1, True, True),
            (2, 2 * 4 + 3, 4, 2, 3, 4, 2, False, True),
            (1, 17, 2, 3, 2, 8, 1, True, False)]):
        inp = _rand_layer(60 + seed, Bz, L, H, P, N)
        r = np.random.default_rng(70 + seed)
        if G > 1:
            inp["Bm"] = (r.standard_normal((Bz, L, G, N)) / np.sqrt(N)).astype(np.float32)
            inp["Cm"] = (r.standard_normal((Bz, L, G, N)) / np.sqrt(N)).astype(np.float32)
        C = -(-L // S)
        dy = r.standard_normal((Bz, L, H, P))
        gD = r.standard_normal((Bz, H, C, N, P)) if gmem else None
        h0 = r.standard_normal((Bz, H, N, P)) * 0.3 if init else None
        args = [inp[k].astype(np.float64) for k in ("x", "dt", "A", "Bm", "Cm")]
        got = orc.scan_backward(*args, S, dy, gD, init_state=h0)
        ref = dart_backward.scan_grads(*args, S, dy, np.zeros((Bz, H, C, N, P)) if gD is None else gD,
                                       init_state=h0)
        for k, v in got.items():
            err = np.max(np.abs(v - ref[k])) / max(np.max(np.abs(ref[k])), 1e-300)
            assert err <= 1e-10, (seed, k, err)


ALL_PINS = [
    pin_closed_form_single_token,
    pin_quadratic_form,
    pin_chunk_memory_definition,
    pin_init_state_continuation,
    pin_single_prior_chunk,
    pin_bruteforce_attention,
    pin_worked_example,
    pin_gate_zero,
    pin_one_hot_mask,
    pin_sampled_rows,
    pin_decode_matches_prefill,
    pin_partial_last_chunk,
    pin_ragged_prefill_then_decode,
    pin_cache_ratio,
    pin_decayed_memories_sum_to_state,
    pin_decayed_bruteforce_attention,
    pin_decayed_decode_matches_prefill,
    pin_e4m3_rows_match_library,
    pin_e4m3_decode_append,
    pin_ngroups_split_into_independent_problems,
    pin_scan_backward_matches_autograd,
]
