"""The chunk-parallel form of the scan backward, checked on the CPU.

The scan backward kernels do not walk the token recurrence; they use its
exact decomposition per chunk (the adjoint carried in from later chunks,
Gin[c-1] = exp(Ae(c)) Gin[c] + dS[c]; the quadratic intra-chunk products for
dx, dB, dC; the decay gradient split into exp(Acum_t) sum(Gl_t o h_in), the
crossing sum Rect_t = sum_{r<t<=s} W_{s,r} and the running sums of u and v).
This test writes that decomposition out in float64 numpy and compares it with
the C oracle's reverse-mode walk of the token recurrence: the two must agree
to rounding (1e-10), on grouped B and C, a ragged last chunk, an initial
state and a memory gradient.  A second test checks the scalar kernel's
warp-scan form of the decay-gradient recursions against the recursions.  It
uses only the seeded input generator and the oracle; no compiled library is
loaded."""
import numpy as np
import pytest

from mamba_ssd_state_b200 import synth
from oracle import dart_oracle


def _chunked_backward(x, dt, A, Bm, Cm, S, dy, gD, h0, states):
    Bz, L, H, P = x.shape
    N = Bm.shape[-1]
    G = 1 if Bm.ndim == 3 else Bm.shape[2]
    C = -(-L // S)
    out = {"dx": np.zeros_like(x), "ddt": np.zeros_like(dt), "dA": np.zeros(H),
           "dBh": np.zeros((Bz, L, H, N)), "dCh": np.zeros((Bz, L, H, N)), "dinit_state": np.zeros((Bz, H, N, P))}
    for b in range(Bz):
        for h in range(H):
            g_ = h // (H // G)
            Bb = Bm[b] if G == 1 else Bm[b, :, g_]
            Cb = Cm[b] if G == 1 else Cm[b, :, g_]
            # adjoint entering each chunk from the later chunks
            Gin = np.zeros((C, N, P))
            carry = np.zeros((N, P))
            for c in range(C - 1, -1, -1):
                Gin[c] = carry
                s0, e = c * S, min(L, c * S + S)
                acum = np.cumsum(dt[b, s0:e, h] * A[h])
                dS = (np.exp(acum)[:, None] * Cb[s0:e]).T @ dy[b, s0:e, h]
                carry = np.exp(acum[-1]) * carry + dS
            out["dinit_state"][b, h] = carry
            for c in range(C):
                s0, e = c * S, min(L, c * S + S)
                n = e - s0
                l = dt[b, s0:e, h] * A[h]
                acum = np.cumsum(l)
                Ae = acum[-1]
                hin = states[b, h, c - 1] if c > 0 else (h0[b, h] if h0 is not None else np.zeros((N, P)))
                R = Gin[c] + (gD[b, h, c] if gD is not None else 0.0)
                Bc, Cc, xc, dyc, dtc = Bb[s0:e], Cb[s0:e], x[b, s0:e, h], dy[b, s0:e, h], dt[b, s0:e, h]
                f = np.exp(Ae - acum)
                dec = np.exp(np.minimum(acum[None, :] - acum[:, None], 0.0))   # [t, s] = exp(Acum_s - Acum_t), s >= t
                up = np.triu(np.ones((n, n)))
                Mx = up * dec * (Bc @ Cc.T)                     # [t, s] (B_t . C_s)
                Mb = up * dec * (xc @ dyc.T)                    # [t, s] (x_t . dy_s)
                Mc = up.T * dec.T * dtc[None, :] * (dyc @ xc.T)  # [t, r] exp(Acum_t - Acum_r) dt_r (dy_t . x_r)
                dxraw = Mx @ dyc + f[:, None] * (Bc @ R)
                dBraw = Mb @ Cc + f[:, None] * (xc @ R.T)
                dCt = Mc @ Bc + np.exp(acum)[:, None] * (dyc @ hin.T)
                out["dx"][b, s0:e, h] = dtc[:, None] * dxraw
                out["dBh"][b, s0:e, h] = dtc[:, None] * dBraw
                out["dCh"][b, s0:e, h] = dCt
                q1 = (xc * dxraw).sum(1)
                u = (xc * (Bc @ R)).sum(1)
                v = (dyc * (Cc @ hin)).sum(1)
                W = np.triu(dtc[:, None] * Mx * (xc @ dyc.T), 1)   # [t, s] = W_{s,t}, s > t
                cols, rows = W.sum(1), W.sum(0)
                c0 = (Gin[c] * hin).sum()
                gh, rect = np.zeros(n), np.zeros(n)
                gg = rc = 0.0
                for t in range(n - 1, -1, -1):
                    gg = v[t] + (np.exp(l[t + 1]) * gg if t + 1 < n else 0.0)
                    rc += rows[t] - cols[t]
                    gh[t], rect[t] = gg, rc
                E = 0.0
                for t in range(n):
                    am1 = acum[t - 1] if t > 0 else 0.0
                    dl = np.exp(acum[t]) * gh[t] + rect[t] + np.exp(Ae) * c0 + np.exp(Ae - am1) * E
                    out["ddt"][b, s0 + t, h] = q1[t] + A[h] * dl
                    out["dA"][h] += dtc[t] * dl
                    E = np.exp(l[t]) * E + dtc[t] * u[t]
    # dB, dC summed over the heads of each group
    hg = H // G
    shp = (Bz, L, N) if G == 1 else (Bz, L, G, N)
    out["dBm"] = out.pop("dBh").reshape(Bz, L, G, hg, N).sum(3).reshape(shp)
    out["dCm"] = out.pop("dCh").reshape(Bz, L, G, hg, N).sum(3).reshape(shp)
    return out


@pytest.mark.parametrize("Bz,L,H,P,N,S,G,init,mem", [
    (1, 3 * 16 + 5, 2, 4, 8, 16, 1, True, True),
    (2, 2 * 8 + 3, 4, 3, 4, 8, 2, False, True),
    (1, 40, 4, 4, 4, 8, 4, True, False),
])
def test_chunked_scan_backward_equals_token_walk(Bz, L, H, P, N, S, G, init, mem):
    orc = dart_oracle.get()
    inp = synth.layer_inputs(synth.LayerShape(Bz, L, H, P, N, S, "f32", "loguniform"), seed=L + G, ngroups=G)
    x, dt, A, Bm, Cm = (inp[k].double().numpy() for k in ("x", "dt", "A", "Bm", "Cm"))
    r = np.random.default_rng(L)
    C = -(-L // S)
    dy = r.standard_normal((Bz, L, H, P))
    gD = r.standard_normal((Bz, H, C, N, P)) if mem else None
    h0 = r.standard_normal((Bz, H, N, P)) * 0.3 if init else None
    _, _, states = orc.ssd_scan(x, dt, A, Bm, Cm, S, init_state=h0)
    ref = orc.scan_backward(x, dt, A, Bm, Cm, S, dy, gD, init_state=h0)
    got = _chunked_backward(x, dt, A, Bm, Cm, S, dy, gD, h0, states)
    for k in ("dx", "ddt", "dA", "dBm", "dCm") + (("dinit_state",) if init else ()):
        err = np.max(np.abs(got[k] - ref[k])) / max(np.max(np.abs(ref[k])), 1e-300)
        assert err <= 1e-10, (k, err)


# ---------------------------------------------------------------------------
# The per-chunk decay-gradient recursions, sequential and as warp scans.
# The scalar kernel of the scan backward runs these recursions over a chunk's
# tokens, eight per lane of one warp:
#   Rect_t = Rect_{t+1} + rowsum_t - colsum_t,
#   gh_t = v_t + a_{t+1} gh_{t+1},
#   E_t = a_t E_{t-1} + dt_t u_t,
# each as a scan of per-lane sums or affine maps.  The two functions below
# are that decomposition, written out lane by lane with Hillis-Steele steps,
# and the recursions themselves; they must agree to rounding for any chunk
# length.
# ---------------------------------------------------------------------------
def _recursions_sequential(dt, A, u, v, q, rw, cl, c0):
    n = len(dt)
    acum = np.cumsum(dt * A)
    Ae = acum[-1]
    gh, rect = np.zeros(n), np.zeros(n)
    g = r = 0.0
    for t in range(n - 1, -1, -1):
        g = v[t] + (np.exp(dt[t + 1] * A) * g if t + 1 < n else 0.0)
        r += rw[t] - cl[t]
        gh[t], rect[t] = g, r
    E = dA = 0.0
    ddt = np.zeros(n)
    for t in range(n):
        am1 = acum[t - 1] if t > 0 else 0.0
        dl = np.exp(acum[t]) * gh[t] + rect[t] + np.exp(Ae) * c0 + np.exp(Ae - am1) * E
        ddt[t] = q[t] + A * dl
        dA += dt[t] * dl
        E = np.exp(dt[t] * A) * E + dt[t] * u[t]
    return ddt, dA


def _scan(vals, combine, reverse):
    """Inclusive Hillis-Steele scan over 32 lanes (toward lower lanes when
    reverse), combine(mine, other) with `other` the farther lanes' partial."""
    vals = list(vals)
    d = 1
    while d < 32:
        nxt = list(vals)
        for l in range(32):
            o = l + d if reverse else l - d
            if 0 <= o < 32:
                nxt[l] = combine(vals[l], vals[o])
        vals, d = nxt, 2 * d
    return vals


def _recursions_warp(dt, A, u, v, q, rw, cl, c0, K=8):
    n = len(dt)
    tok = [[t for t in range(K * l, K * l + K) if t < n] for l in range(32)]
    a = lambda t: np.exp(dt[t] * A) if t < n else 0.0   # nothing follows the chunk
    # prefix of dt A
    tot = [sum(dt[t] * A for t in ts) for ts in tok]
    incl = _scan(tot, lambda m, o: m + o, reverse=False)
    acum = np.zeros(n)
    for l, ts in enumerate(tok):
        run = incl[l - 1] if l > 0 else 0.0
        for t in ts:
            run += dt[t] * A
            acum[t] = run
    Ae = incl[31]
    # gh: map x -> K + M x from gh after the lane to gh at its first token
    maps = []
    for ts in tok:
        M, Kc = 1.0, 0.0
        for t in reversed(ts):
            Kc, M = v[t] + a(t + 1) * Kc, a(t + 1) * M
        maps.append((M, Kc))
    suf = _scan(maps, lambda m, o: (m[0] * o[0], m[1] + m[0] * o[1]), reverse=True)
    gh = np.zeros(n)
    for l, ts in enumerate(tok):
        x = suf[l + 1][1] if l < 31 else 0.0
        for t in reversed(ts):
            x = v[t] + a(t + 1) * x
            gh[t] = x
    # Rect: suffix sums
    seg = [sum(rw[t] - cl[t] for t in ts) for ts in tok]
    ssum = _scan(seg, lambda m, o: m + o, reverse=True)
    rect = np.zeros(n)
    for l, ts in enumerate(tok):
        r = ssum[l + 1] if l < 31 else 0.0
        for t in reversed(ts):
            r += rw[t] - cl[t]
            rect[t] = r
    # E: map y -> P + N y from E before the lane to E after it
    maps = []
    for ts in tok:
        N_, P_ = 1.0, 0.0
        for t in ts:
            P_, N_ = a(t) * P_ + dt[t] * u[t], a(t) * N_
        maps.append((N_, P_))
    pre = _scan(maps, lambda m, o: (m[0] * o[0], m[1] + m[0] * o[1]), reverse=False)
    ddt, dA = np.zeros(n), 0.0
    for l, ts in enumerate(tok):
        E = pre[l - 1][1] if l > 0 else 0.0
        for t in ts:
            am1 = acum[t - 1] if t > 0 else 0.0
            dl = np.exp(acum[t]) * gh[t] + rect[t] + np.exp(Ae) * c0 + np.exp(Ae - am1) * E
            ddt[t] = q[t] + A * dl
            dA += dt[t] * dl
            E = a(t) * E + dt[t] * u[t]
    return ddt, dA


@pytest.mark.parametrize("n", [1, 8, 9, 33, 128, 129, 255, 256])
@pytest.mark.parametrize("heavy", [False, True])
def test_decay_gradient_recursions_as_warp_scans(n, heavy):
    r = np.random.default_rng(n + 7 * heavy)
    A = -16.0 if heavy else -1.0
    dt = np.full(n, 0.1) if heavy else np.exp(r.uniform(np.log(1e-3), np.log(1e-1), n))
    u, v, q, rw, cl = (r.standard_normal(n) for _ in range(5))
    c0 = r.standard_normal()
    d1, a1 = _recursions_sequential(dt, A, u, v, q, rw, cl, c0)
    d2, a2 = _recursions_warp(dt, A, u, v, q, rw, cl, c0)
    assert np.max(np.abs(d1 - d2)) <= 1e-12 * np.max(np.abs(d1))
    assert abs(a1 - a2) <= 1e-12 * abs(a1)
