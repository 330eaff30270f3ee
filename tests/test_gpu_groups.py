"""GPU parity with B and C shared by groups of heads (Mamba-2's ngroups):
B and C are [B, L, G, N] and head h reads group h // (H // G).  Every
kernel family (tensor-core scan and attention at S = 256 and 128, the
CUDA-core float32 kernels, decode, both backwards) against the fp64 oracle
on the same seeded inputs; tolerances as in the ungrouped tests.  A grouped
run with every group holding the same rows must equal the ungrouped run bit
for bit, which pins the head-to-group map from the other side."""
import numpy as np
import pytest
import torch

from mamba_ssd_state_b200 import build, dart, synth
from mamba_ssd_state_b200.synth import DecodeShape, LayerShape
from oracle import dart_backward, dart_oracle
from tests.parity import TOL, assert_close, oracle_inputs, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return dart_oracle.get()


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return dart.load()


def _gpu_layer(inp, chunk):
    d = to_device(inp)
    y_ssd, dH, st = dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], chunk)
    o = dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, chunk, d["g"])
    y = dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, chunk, d["g"], y_ssd.clone())
    dart.dart_sync_status()
    return {"y_ssd": y_ssd, "dH": dH, "states": st, "o": o, "y": y}


@pytest.mark.parametrize("shape,G", [
    (LayerShape(1, 3 * 256 + 77, 32, 64, 128, 256, "bf16", "loguniform"), 2),
    (LayerShape(1, 3 * 256 + 77, 32, 64, 128, 256, "bf16", "loguniform"), 8),
    (LayerShape(2, 4 * 128 + 60, 8, 64, 128, 128, "bf16", "loguniform"), 4),
    (LayerShape(2, 3 * 64 + 17, 4, 16, 16, 64, "f32", "softplus"), 2),
    (LayerShape(1, 5 * 64, 4, 64, 64, 64, "f32", "softplus"), 4),
], ids=["bf16_S256_H32_G2", "bf16_S256_H32_G8", "bf16_S128_H8_G4", "f32_N16_G2", "f32_N64_G_eq_H"])
def test_grouped_layer_forward(orc, shape, G):
    inp = synth.layer_inputs(shape, seed=100 + G, ngroups=G)
    assert tuple(inp["Bm"].shape) == (shape.batch, shape.seqlen, G, shape.dstate)
    got = _gpu_layer(inp, shape.chunk)
    o = oracle_inputs(inp)
    ref = orc.layer_forward(o["x"], o["dt"], o["A"], o["Bm"], o["Cm"], o["Q"], o["E"], shape.chunk, inp["g"])
    tol = TOL[synth.torch_dtype(shape.dtype)]
    for k in ("y_ssd", "dH", "states", "o", "y"):
        assert_close(k, got[k], ref[k], tol)


def test_grouped_equal_rows_match_ungrouped_bit_for_bit():
    """G = 4 groups that all carry the ungrouped rows: every output is the
    ungrouped run's, exactly (same kernels, same operands per head)."""
    shape = LayerShape(1, 2 * 256 + 40, 8, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=7)
    grp = dict(inp)
    for k in ("Bm", "Cm"):
        grp[k] = inp[k][:, :, None, :].expand(-1, -1, 4, -1).contiguous()
    a, b = _gpu_layer(inp, shape.chunk), _gpu_layer(grp, shape.chunk)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_grouped_decayed_sma(orc):
    shape = LayerShape(1, 4 * 256 + 30, 8, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=11, ngroups=2)
    inp["A"] = torch.full_like(inp["A"], -0.05)
    d = to_device(inp)
    y_ssd, dH, _ = dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], shape.chunk)
    o = dart.dart_sma_forward_decayed(d["Q"], d["E"], d["Cm"], dH, d["dt"], d["A"], shape.chunk, d["g"])
    dart.dart_sync_status()
    oi = oracle_inputs(inp)
    ref = orc.layer_forward(oi["x"], oi["dt"], oi["A"], oi["Bm"], oi["Cm"], oi["Q"], oi["E"], shape.chunk,
                            inp["g"], decayed=True)
    assert_close("o", o, ref["o"], TOL[torch.bfloat16])


def test_grouped_rejects_groups_not_dividing_heads():
    shape = LayerShape(1, 256, 4, 64, 128, 256, "bf16", "loguniform")
    inp = to_device(synth.layer_inputs(shape, seed=1, ngroups=3))
    with pytest.raises(ValueError):
        dart.dart_ssd_chunk_scan(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], 256)


@pytest.mark.parametrize("dtype,G", [("bf16", 2), ("bf16", 8), ("f32", 4)])
def test_grouped_decode(orc, dtype, G):
    """Four sequences at different counters, chunk 4 so appends happen inside
    the run; y compared every step, then state, running contribution, cache
    and counters."""
    shape = DecodeShape(4, 8, 64, 128, 4, 6, 9, 9, dtype)
    tol = TOL[synth.torch_dtype(dtype)]
    init = synth.decode_initial(shape, seed=G)
    init["nchunks"] = torch.tensor([6, 0, 3, 2], dtype=torch.int32)
    init["pos"] = torch.tensor([0, 1, 3, 2], dtype=torch.int32)
    for b, n in enumerate(init["nchunks"].tolist()):
        init["cache"][b, :, n:] = 1e4     # never read
    dev = {k: v.cuda() for k, v in init.items()}
    ref = {"cache": init["cache"].double().numpy().copy(), "state": init["state"].double().numpy().copy(),
           "dH_cur": init["dH_cur"].double().numpy().copy(), "nchunks": init["nchunks"].numpy().copy(),
           "pos": init["pos"].numpy().copy()}
    A = synth.decode_A(shape, G)
    for step in range(shape.nsteps):
        tok = synth.decode_tokens(shape, step, seed=G, ngroups=G)
        assert tuple(tok["Bm"].shape) == (shape.nseq, G, shape.dstate)
        y = dart.dart_decode_step(tok["x"].cuda(), tok["dt"].cuda(), A.cuda(), tok["Bm"].cuda(),
                                  tok["Cm"].cuda(), tok["Q"].cuda(), tok["E"].cuda(), shape.g, dev["state"],
                                  dev["dH_cur"], dev["cache"], dev["nchunks"], dev["pos"], shape.chunk)
        t = oracle_inputs(tok)
        yr = orc.decode_step(t["x"], t["dt"], A.numpy(), t["Bm"], t["Cm"], t["Q"], t["E"], shape.g, ref["state"],
                             ref["dH_cur"], ref["cache"], ref["nchunks"], ref["pos"], shape.chunk)
        assert_close(f"y step {step}", y, yr, tol)
    dart.dart_sync_status()
    assert np.array_equal(dev["nchunks"].cpu().numpy(), ref["nchunks"])
    assert np.array_equal(dev["pos"].cpu().numpy(), ref["pos"])
    assert_close("state", dev["state"], ref["state"], tol)
    assert_close("dH_cur", dev["dH_cur"], ref["dH_cur"], tol)
    for b in range(shape.nseq):
        n = int(ref["nchunks"][b])
        assert_close(f"cache {b}", dev["cache"][b, :, :n], ref["cache"][b, :, :n], tol)


@pytest.mark.parametrize("shape,dt_name,G", [
    ((1, 2 * 64 + 17, 4, 16, 16, 64), "f32", 2),
    ((1, 2 * 256 + 77, 4, 64, 128, 256), "bf16", 2),
], ids=["f32_N16_G2", "bf16_N128_G2"])
def test_grouped_layer_backward(shape, dt_name, G):
    """dart.layer_backward with grouped B and C against autograd over the
    whole grouped layer: dBm and dCm sum over the heads of each group."""
    Bz, L, H, P, N, S = shape
    inp = synth.layer_inputs(synth.LayerShape(Bz, L, H, P, N, S, dt_name, "loguniform"), seed=L, ngroups=G)
    dy = torch.from_numpy(np.random.default_rng(L).standard_normal((Bz, L, H, P)).astype(np.float32))
    keys = ("x", "dt", "A", "Bm", "Cm", "Q", "E")
    g = 0.6
    got = dart.layer_backward(*(inp[k].cuda() for k in keys), S, g, dy.cuda())
    dart.dart_sync_status()
    ref = dart_backward.layer_grads(*(inp[k].double().numpy() for k in keys), S, g, dy.double().numpy())
    tol = {"f32": 1e-4, "bf16": 2e-2}[dt_name]
    assert tuple(got["dBm"].shape) == (Bz, L, G, N) and tuple(got["dCm"].shape) == (Bz, L, G, N)
    for k in ("dx", "ddt", "dA", "dBm", "dCm", "dQ", "dE"):
        assert_close(k, got[k], ref[k], tol)
