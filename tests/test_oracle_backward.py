"""Pins of the fp64 backward oracle (``oracle/dart_backward.py``), CPU only.

* Its forward restatement equals the C oracle's forward (itself pinned in
  ``oracle_pins.py``) on ragged lengths, an initial state and decayed
  memories.
* Every gradient equals a central finite difference of the C oracle's
  forward, sum(dy * y), on sampled coordinates.  The C oracle reads its
  inputs as float32, so each step is a power of two on the coordinate's
  float32 grid and both perturbed inputs are exact.
* Closed forms: dg = sum(dy * o); a token with a single visible memory has
  o_t = C_t^T dH[0], so dQ_t = dE_t = 0 there and the memory gradient is
  sum_t C_t (g dy_t)^T over those tokens.
"""
import numpy as np
import pytest

from oracle import dart_backward, dart_oracle

KEYS = ("x", "dt", "A", "Bm", "Cm", "Q", "E")


@pytest.fixture(scope="module")
def orc():
    return dart_oracle.get()


def _inputs(seed, Bz, L, H, P, N, a_max=1.5):
    r = np.random.default_rng(seed)
    f = lambda a: np.asarray(a, np.float32).astype(np.float64)   # float32 values held in float64
    return dict(
        x=f(r.standard_normal((Bz, L, H, P))),
        dt=f(r.uniform(0.05, 0.5, (Bz, L, H))),
        A=f(-r.uniform(0.1, a_max, (H,))),
        Bm=f(r.standard_normal((Bz, L, N)) / np.sqrt(N)),
        Cm=f(r.standard_normal((Bz, L, N)) / np.sqrt(N)),
        Q=f(r.standard_normal((Bz, L, H, N))),
        E=f(r.standard_normal((Bz, L, H, P)) / np.sqrt(P)),
    )


def _c_loss(orc, inp, S, g, dy, h0=None, decayed=False):
    r = orc.layer_forward(*(inp[k] for k in KEYS), S, g, init_state=h0, decayed=decayed)
    return float(np.sum(dy * r["y"]))


def _step(v):
    """A power-of-two step about 2^-12 of |v|, a multiple of v's float32 ulp."""
    e = np.frexp(max(abs(v), 1e-3))[1]
    return float(np.ldexp(1.0, e - 13))


@pytest.mark.parametrize("decayed", [False, True])
def test_forward_restatement_matches_c_oracle(orc, decayed):
    Bz, L, H, P, N, S = 2, 21, 2, 3, 4, 8
    inp = _inputs(1, Bz, L, H, P, N)
    h0 = np.random.default_rng(2).standard_normal((Bz, H, N, P)) * 0.3
    ref = orc.layer_forward(*(inp[k] for k in KEYS), S, 0.7, init_state=h0, decayed=decayed)
    ts = {k: dart_backward._t(v) for k, v in inp.items()}
    y, y_ssd, o, dH, st = dart_backward.layer_forward(*(ts[k] for k in KEYS), S, 0.7,
                                                      dart_backward._t(h0), decayed)
    for name, got in (("y", y), ("y_ssd", y_ssd), ("o", o), ("dH", dH), ("states", st)):
        np.testing.assert_allclose(got.detach().numpy(), ref[name], rtol=1e-12, atol=1e-12, err_msg=name)


@pytest.mark.parametrize("decayed", [False, True])
def test_layer_gradients_match_finite_differences(orc, decayed):
    """Ragged length (3 chunks, the last partial), initial state, g != 1."""
    Bz, L, H, P, N, S = 1, 19, 2, 3, 4, 8
    g = 0.8
    inp = _inputs(3, Bz, L, H, P, N)
    h0 = np.random.default_rng(4).standard_normal((Bz, H, N, P)) * 0.3
    dy = np.random.default_rng(5).standard_normal((Bz, L, H, 3))
    gr = dart_backward.layer_grads(*(inp[k] for k in KEYS), S, g, dy, init_state=h0, decayed=decayed)
    r = np.random.default_rng(6)
    for name in KEYS:
        a = inp[name]
        for idx in [tuple(r.integers(0, s) for s in a.shape) for _ in range(4)]:
            hstep = _step(a[idx])
            plus, minus = {k: v.copy() for k, v in inp.items()}, {k: v.copy() for k, v in inp.items()}
            plus[name][idx] += hstep
            minus[name][idx] -= hstep
            fd = (_c_loss(orc, plus, S, g, dy, h0, decayed) - _c_loss(orc, minus, S, g, dy, h0, decayed)) / (2 * hstep)
            got = gr["d" + name][idx]
            assert abs(got - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, got, fd)
    # g and the initial state (double inputs of the C oracle)
    fd = (_c_loss(orc, inp, S, g + 1e-4, dy, h0, decayed) - _c_loss(orc, inp, S, g - 1e-4, dy, h0, decayed)) / 2e-4
    assert abs(gr["dg"] - fd) <= 1e-7 * max(1.0, abs(fd))
    for idx in [(0, 1, 2, 1), (0, 0, 3, 0)]:
        hp, hm = h0.copy(), h0.copy()
        hp[idx] += 1e-4
        hm[idx] -= 1e-4
        fd = (_c_loss(orc, inp, S, g, dy, hp, decayed) - _c_loss(orc, inp, S, g, dy, hm, decayed)) / 2e-4
        assert abs(gr["dinit_state"][idx] - fd) <= 1e-7 * max(1.0, abs(fd))


def test_gate_gradient_closed_form():
    Bz, L, H, P, N, S = 1, 24, 2, 3, 4, 8
    inp = _inputs(7, Bz, L, H, P, N)
    dy = np.random.default_rng(8).standard_normal((Bz, L, H, P))
    gr = dart_backward.layer_grads(*(inp[k] for k in KEYS), S, 0.3, dy)
    assert abs(gr["dg"] - np.sum(dy * gr["o"])) <= 1e-12 * max(1.0, abs(gr["dg"]))


def test_single_visible_memory_closed_form():
    """Tokens of chunk 1 see memory 0 only: o_t = C_t^T dH[0], the softmax has
    one entry, so Q and E get no gradient there, dCm_t = dH[0] (g dy_t) and
    ddH[0] = sum over those tokens of C_t (g dy_t)^T; chunk-0 tokens give
    nothing."""
    Bz, L, H, P, N, S = 1, 16, 2, 3, 4, 8
    inp = _inputs(9, Bz, L, H, P, N)
    dH = np.random.default_rng(10).standard_normal((Bz, H, 2, N, P))
    dy = np.random.default_rng(11).standard_normal((Bz, L, H, P))
    g = 1.3
    gr = dart_backward.sma_grads(inp["Q"], inp["E"], inp["Cm"], dH, S, g, dy)
    assert np.all(gr["dQ"] == 0.0) and np.allclose(gr["dE"], 0.0, atol=1e-14)
    for t in range(S, 2 * S):
        want = sum(dH[0, h, 0] @ (g * dy[0, t, h]) for h in range(H))
        np.testing.assert_allclose(gr["dCm"][0, t], want, rtol=1e-12, atol=1e-13)
    assert np.all(gr["dCm"][0, :S] == 0.0)
    for h in range(H):
        want = sum(np.outer(inp["Cm"][0, t], g * dy[0, t, h]) for t in range(S, 2 * S))
        np.testing.assert_allclose(gr["ddH"][0, h, 0], want, rtol=1e-12, atol=1e-13)
    assert np.all(gr["ddH"][:, :, 1] == 0.0), "no token attends to the last memory"


@pytest.mark.parametrize("decayed", [False, True])
def test_sma_gradients_match_finite_differences(orc, decayed):
    """SMA alone over given memories (the memory gradient is what the scan's
    backward consumes), against finite differences of the C oracle's SMA."""
    Bz, L, H, P, N, S = 1, 26, 2, 3, 4, 8
    inp = _inputs(12, Bz, L, H, P, N)
    C = -(-L // S)
    dH = np.random.default_rng(13).standard_normal((Bz, H, C, N, P)) * 0.5
    dy = np.random.default_rng(14).standard_normal((Bz, L, H, P))
    g = 0.9
    extra = dict(dt=inp["dt"], A=inp["A"]) if decayed else {}
    gr = dart_backward.sma_grads(inp["Q"], inp["E"], inp["Cm"], dH, S, g, dy, **extra)

    def loss(Q, E, Cm, M, dt=None, A=None):
        r = orc.sma(Q, E, Cm, M, S, g, dt=dt, A=A)
        return float(np.sum(dy * r["y"]))
    args = dict(Q=inp["Q"], E=inp["E"], Cm=inp["Cm"], M=dH, **extra)
    r = np.random.default_rng(15)
    for name, key in (("Q", "dQ"), ("E", "dE"), ("Cm", "dCm"), ("M", "ddH")) + \
            ((("dt", "ddt"), ("A", "dA")) if decayed else ()):
        a = args[name]
        for idx in [tuple(r.integers(0, s) for s in a.shape) for _ in range(5)]:
            hstep = _step(a[idx]) if name != "M" else 1e-5
            p_, m_ = dict(args), dict(args)
            p_[name], m_[name] = a.copy(), a.copy()
            p_[name][idx] += hstep
            m_[name][idx] -= hstep
            fd = (loss(**p_) - loss(**m_)) / (2 * hstep)
            assert abs(gr[key][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, gr[key][idx], fd)


def test_layer_gradients_compose_from_scan_and_sma():
    """The chain rule across the two steps: layer gradients = the scan's
    gradients driven by (dy, ddH from the SMA backward) plus the SMA's own
    gradients of Q, E and C (B and C of the scan and of SMA are one tensor)."""
    Bz, L, H, P, N, S = 1, 21, 2, 3, 4, 8
    g = 0.6
    inp = _inputs(21, Bz, L, H, P, N)
    h0 = np.random.default_rng(22).standard_normal((Bz, H, N, P)) * 0.2
    dy = np.random.default_rng(23).standard_normal((Bz, L, H, P))
    full = dart_backward.layer_grads(*(inp[k] for k in KEYS), S, g, dy, init_state=h0)
    sm = dart_backward.sma_grads(inp["Q"], inp["E"], inp["Cm"], full["dH"], S, g, dy)
    sc = dart_backward.scan_grads(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], S, dy, sm["ddH"],
                                  init_state=h0)
    for k in ("dx", "ddt", "dA", "dBm", "dinit_state"):
        np.testing.assert_allclose(sc[k], full[k], rtol=1e-11, atol=1e-12, err_msg=k)
    np.testing.assert_allclose(sc["dCm"] + sm["dCm"], full["dCm"], rtol=1e-11, atol=1e-12)
    for k in ("dQ", "dE"):
        np.testing.assert_allclose(sm[k], full[k], rtol=1e-11, atol=1e-12, err_msg=k)


def test_scan_gradients_match_finite_differences(orc):
    """dx, ddt, dA, dB, dC of sum(dy * y_ssd) + sum(gdH * dH) against central
    differences of the C oracle's scan (ragged length, initial state)."""
    Bz, L, H, P, N, S = 1, 19, 2, 3, 4, 8
    inp = _inputs(24, Bz, L, H, P, N)
    C = -(-L // S)
    r = np.random.default_rng(25)
    h0 = r.standard_normal((Bz, H, N, P)) * 0.3
    dy = r.standard_normal((Bz, L, H, P))
    gdH = r.standard_normal((Bz, H, C, N, P))
    gr = dart_backward.scan_grads(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], S, dy, gdH, init_state=h0)

    def loss(d):
        y, dH, _ = orc.ssd_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S, init_state=h0)
        return float(np.sum(dy * y) + np.sum(gdH * dH))
    for name in ("x", "dt", "A", "Bm", "Cm"):
        a = inp[name]
        for idx in [tuple(r.integers(0, s_) for s_ in a.shape) for _ in range(4)]:
            hstep = _step(a[idx])
            plus, minus = dict(inp), dict(inp)
            plus[name], minus[name] = a.copy(), a.copy()
            plus[name][idx] += hstep
            minus[name][idx] -= hstep
            fd = (loss(plus) - loss(minus)) / (2 * hstep)
            assert abs(gr["d" + name][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, gr["d" + name][idx], fd)


def test_grouped_B_C_restatement_and_split(orc):
    """B and C per group of heads (H = 4, G = 2): the restatement equals the C
    oracle's grouped forward, and the layer gradients equal those of two
    single-group problems (heads of group g with group g's B and C), with dB
    and dC landing on the group's slice."""
    Bz, L, H, P, N, S, G = 1, 18, 4, 3, 4, 8, 2
    inp = _inputs(41, Bz, L, H, P, N)
    r = np.random.default_rng(42)
    f = lambda a: np.asarray(a, np.float32).astype(np.float64)
    Bg = f(r.standard_normal((Bz, L, G, N)) / np.sqrt(N))
    Cg = f(r.standard_normal((Bz, L, G, N)) / np.sqrt(N))
    dy = r.standard_normal((Bz, L, H, P))
    g = 0.7
    grouped = dict(inp, Bm=Bg, Cm=Cg)
    ref = orc.layer_forward(*(grouped[k] for k in KEYS), S, g)
    full = dart_backward.layer_grads(*(grouped[k] for k in KEYS), S, g, dy)
    np.testing.assert_allclose(full["y"], ref["y"], rtol=1e-12, atol=1e-12)
    hg = H // G
    for gi in range(G):
        hs = slice(gi * hg, (gi + 1) * hg)
        part_in = dict(x=inp["x"][:, :, hs], dt=inp["dt"][:, :, hs], A=inp["A"][hs], Bm=Bg[:, :, gi],
                       Cm=Cg[:, :, gi], Q=inp["Q"][:, :, hs], E=inp["E"][:, :, hs])
        part = dart_backward.layer_grads(*(part_in[k] for k in KEYS), S, g, dy[:, :, hs])
        for k in ("dx", "ddt", "dQ", "dE"):
            np.testing.assert_allclose(full[k][:, :, hs], part[k], rtol=1e-11, atol=1e-12, err_msg=k)
        np.testing.assert_allclose(full["dA"][hs], part["dA"], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(full["dBm"][:, :, gi], part["dBm"], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(full["dCm"][:, :, gi], part["dCm"], rtol=1e-11, atol=1e-12)
