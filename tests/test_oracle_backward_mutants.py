"""Plant plausible mistakes in copies of ``oracle/dart_backward.py`` and check
that the backward oracle's pins catch every one.  Each mutant is loaded as
its own module from a temporary file; the real module is never touched.
The checks are those of ``test_oracle_backward.py``: the forward restatement
against the C oracle, and the gradients against finite differences of the C
oracle (plus the gate's closed form)."""
import importlib.util
import os

import numpy as np
import pytest

from oracle import dart_oracle
from tests.test_oracle_backward import KEYS, _inputs, _step

SOURCE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "dart_backward.py")

# (name, text to find, replacement)
MUTATIONS = [
    ("no_chunk_restart", "                    D = torch.zeros(N, P, dtype=_F64)   # a new chunk's own contribution\n",
     "                    pass\n"),
    ("decay_after_input", "                Hs = decay * Hs + inp\n", "                Hs = decay * (Hs + inp)\n"),
    ("memory_not_decayed", "                D = decay * D + inp\n", "                D = D + inp\n"),
    ("readout_before_update", "                yh.append(Hs.transpose(0, 1) @ _bc(Cm, b, t, h, H))\n",
     "                yh.append((Hs - inp).transpose(0, 1) @ _bc(Cm, b, t, h, H))\n"),
    ("group_by_modulo", "    return M[b, t, h // (H // M.shape[2])]\n", "    return M[b, t, h % M.shape[2]]\n"),
    ("scale_by_P", "    inv_sqrt_n = 1.0 / math.sqrt(N)\n", "    inv_sqrt_n = 1.0 / math.sqrt(P)\n"),
    ("mask_off_by_one", "            k = t // S\n", "            k = (t + 1) // S\n"),
    ("value_read_with_Q", "                    values.append(_bc(Cm, b, t, h, H) @ M)  # [P]\n",
     "                    values.append(Q[b, t, h] @ M)  # [P]\n"),
    ("decay_window_from_e", "dt[b, c * S + S:t + 1, h].sum()", "dt[b, c * S + S - 1:t + 1, h].sum()"),
    ("gate_ignored", "    return y_ssd + g * o, y_ssd, o, dH, st\n", "    return y_ssd + o, y_ssd, o, dH, st\n"),
    ("scan_loss_drops_memories", "    loss = (y_ssd * _t(dy)).sum() + (dH * _t(gdH)).sum()\n",
     "    loss = (y_ssd * _t(dy)).sum()\n"),
    ("sma_loss_drops_gate", "    loss = (ts[\"g\"] * o * _t(dy)).sum()\n", "    loss = (o * _t(dy)).sum()\n"),
]


def _load(tmp_path, name, old, new):
    src = open(SOURCE).read()
    assert src.count(old) == 1, f"pattern for {name} not found exactly once"
    path = tmp_path / f"dart_backward_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"dart_backward_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _pins_hold(mod, orc) -> bool:
    """True when the module passes every check; False at the first failure."""
    Bz, L, H, P, N, S = 1, 19, 2, 3, 4, 8
    g = 0.8
    inp = _inputs(31, Bz, L, H, P, N)
    r = np.random.default_rng(32)
    h0 = r.standard_normal((Bz, H, N, P)) * 0.3
    dy = r.standard_normal((Bz, L, H, P))
    C = -(-L // S)
    gdH = r.standard_normal((Bz, H, C, N, P))
    try:
        # forward restatement against the C oracle (raw and decayed memories)
        for decayed in (False, True):
            ref = orc.layer_forward(*(inp[k] for k in KEYS), S, g, init_state=h0, decayed=decayed)
            ts = {k: mod._t(v) for k, v in inp.items()}
            out = mod.layer_forward(*(ts[k] for k in KEYS), S, g, mod._t(h0), decayed)
            for name, got in zip(("y", "y_ssd", "o", "dH", "states"), out):
                if not np.allclose(got.detach().numpy(), ref[name], rtol=1e-10, atol=1e-10):
                    return False
        # B and C per group of heads (H = 4, G = 2) against the C oracle
        gin = _inputs(33, 1, 17, 4, 3, 4)
        rg = np.random.default_rng(34)
        gin["Bm"] = np.asarray(rg.standard_normal((1, 17, 2, 4)) / 2, np.float32).astype(np.float64)
        gin["Cm"] = np.asarray(rg.standard_normal((1, 17, 2, 4)) / 2, np.float32).astype(np.float64)
        gref = orc.layer_forward(*(gin[k] for k in KEYS), S, g)
        gts = {k: mod._t(v) for k, v in gin.items()}
        gout = mod.layer_forward(*(gts[k] for k in KEYS), S, g)
        if not np.allclose(gout[0].detach().numpy(), gref["y"], rtol=1e-10, atol=1e-10):
            return False
        # layer gradients against finite differences of the C oracle
        gr = mod.layer_grads(*(inp[k] for k in KEYS), S, g, dy, init_state=h0)

        def c_loss(d, gg=g):
            y = orc.layer_forward(*(d[k] for k in KEYS), S, gg, init_state=h0)["y"]
            return float(np.sum(dy * y))
        for name in KEYS:
            a = inp[name]
            for idx in [tuple(r.integers(0, s) for s in a.shape) for _ in range(2)]:
                hs = _step(a[idx])
                p_, m_ = dict(inp), dict(inp)
                p_[name], m_[name] = a.copy(), a.copy()
                p_[name][idx] += hs
                m_[name][idx] -= hs
                fd = (c_loss(p_) - c_loss(m_)) / (2 * hs)
                if abs(gr["d" + name][idx] - fd) > 1e-6 * max(1.0, abs(fd)):
                    return False
        fd = (c_loss(inp, g + 1e-4) - c_loss(inp, g - 1e-4)) / 2e-4
        if abs(gr["dg"] - fd) > 1e-7 * max(1.0, abs(fd)):
            return False
        # SMA-only gradients: the gate's closed form
        sm = mod.sma_grads(inp["Q"], inp["E"], inp["Cm"], gr["dH"], S, g, dy)
        if abs(sm["dg"] - np.sum(dy * gr["o"])) > 1e-10 * max(1.0, abs(sm["dg"])):
            return False
        # scan-only gradients against finite differences of the C oracle's scan
        sc = mod.scan_grads(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], S, dy, gdH, init_state=h0)

        def s_loss(d):
            y, dH, _ = orc.ssd_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S, init_state=h0)
            return float(np.sum(dy * y) + np.sum(gdH * dH))
        for name in ("x", "dt", "Bm"):
            a = inp[name]
            for idx in [tuple(r.integers(0, s) for s in a.shape) for _ in range(2)]:
                hs = _step(a[idx])
                p_, m_ = dict(inp), dict(inp)
                p_[name], m_[name] = a.copy(), a.copy()
                p_[name][idx] += hs
                m_[name][idx] -= hs
                fd = (s_loss(p_) - s_loss(m_)) / (2 * hs)
                if abs(sc["d" + name][idx] - fd) > 1e-6 * max(1.0, abs(fd)):
                    return False
    except (AssertionError, RuntimeError, IndexError, ValueError):
        return False
    return True


@pytest.fixture(scope="module")
def orc():
    return dart_oracle.get()


def test_unmutated_backward_oracle_passes(orc, tmp_path):
    mod = _load(tmp_path, "identity", "import math\n", "import math\n")
    assert _pins_hold(mod, orc)


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_backward_mutant_is_caught(orc, tmp_path, name, old, new):
    mod = _load(tmp_path, name, old, new)
    assert not _pins_hold(mod, orc), f"mutant {name} passed every pin"
