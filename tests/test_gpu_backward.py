"""GPU parity of the SMA backward (dart_sma_backward) against the fp64
backward oracle (``oracle/dart_backward.py``, autograd over the pinned
forward restatement), on the same seeded inputs.  Both sides read the same
float32-exact inputs, so the only differences are fp32 accumulation:
max|err| / max|ref| <= 1e-4 for float32 inputs (CUDA cores, fp32 throughout)
and <= 1e-2 for bf16 inputs: the tensor-core path rounds the scaled operand
rows (ds / sqrt(N)) E and p do to bf16 (2^-9 relative) before its products,
which accumulate in fp32, as the forward's bf16 memories do."""
import numpy as np
import pytest
import torch

from mamba_ssd_state_b200 import build, dart, synth
from oracle import dart_backward, dart_oracle
from tests.parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return dart.load()


def _case(Bz, L, H, P, N, S, dtype, seed):
    r = np.random.default_rng(seed)
    C = -(-L // S)
    f = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(dtype)
    inp = dict(Q=f(r.standard_normal((Bz, L, H, N))), E=f(r.standard_normal((Bz, L, H, P)) / np.sqrt(P)),
               Cm=f(r.standard_normal((Bz, L, N)) / np.sqrt(N)),
               dH=f(r.standard_normal((Bz, H, C, N, P)) * 0.3))
    dy = torch.from_numpy(r.standard_normal((Bz, L, H, P)).astype(np.float32))
    return inp, dy


@pytest.mark.parametrize("shape,dtype,tol", [
    ((1, 3 * 64 + 17, 2, 16, 16, 64), torch.float32, 1e-4),
    ((2, 3 * 128 + 40, 2, 64, 64, 128), torch.float32, 1e-4),
    ((1, 3 * 256, 2, 64, 128, 256), torch.bfloat16, 1e-2),
    ((1, 2 * 256 + 77, 3, 64, 128, 256), torch.bfloat16, 1e-2),
    ((2, 3 * 128 + 50, 2, 64, 128, 128), torch.bfloat16, 1e-2),
    ((1, 100, 2, 64, 128, 256), torch.bfloat16, 1e-2),
], ids=["f32_N16_ragged", "f32_N64_B2_ragged", "bf16_N128", "bf16_N128_ragged", "bf16_S128_B2_ragged",
        "bf16_single_partial_chunk"])
def test_sma_backward_matches_oracle(shape, dtype, tol):
    Bz, L, H, P, N, S = shape
    g = 0.7
    inp, dy = _case(Bz, L, H, P, N, S, dtype, seed=L)
    got = dart.dart_sma_backward(*(inp[k].cuda() for k in ("Q", "E", "Cm", "dH")), S, g, dy.cuda())
    dart.dart_sync_status()
    ref = dart_backward.sma_grads(*(inp[k].double().numpy() for k in ("Q", "E", "Cm", "dH")), S, g,
                                  dy.double().numpy())
    for k in ("dQ", "dE", "dCm", "ddH"):
        print(k, assert_close(k, got[k], ref[k], tol))
    assert abs(float(got["dg"][0]) - float(ref["dg"])) <= tol * max(1.0, abs(float(ref["dg"])))


def test_sma_backward_deterministic():
    inp, dy = _case(1, 3 * 256, 2, 64, 128, 256, torch.bfloat16, seed=3)
    args = [inp[k].cuda() for k in ("Q", "E", "Cm", "dH")]
    a = dart.dart_sma_backward(*args, 256, 0.5, dy.cuda())
    b = dart.dart_sma_backward(*args, 256, 0.5, dy.cuda())
    for k in a:
        assert torch.equal(a[k], b[k]), k


# ---------------------------------------------------------------------------
# scan backward and the whole layer backward
# ---------------------------------------------------------------------------
SCAN_CASES = [
    ((1, 3 * 64 + 17, 2, 16, 16, 64), "f32", True),
    ((2, 3 * 128 + 40, 2, 64, 64, 128), "f32", False),
    ((1, 3 * 256, 2, 64, 128, 256), "bf16", False),
    ((1, 2 * 256 + 77, 3, 64, 128, 256), "bf16", True),
    ((2, 3 * 128 + 50, 2, 64, 128, 128), "bf16", True),
    ((1, 256 + 100, 2, 64, 128, 256), "bf16", False),
]
SCAN_IDS = ["f32_N16_ragged_init", "f32_N64_B2_ragged", "bf16_N128", "bf16_N128_ragged_init", "bf16_S128_B2_ragged_init",
            "bf16_second_block_past_the_end"]
TOL_FWD_INPUTS = {"f32": 1e-4, "bf16": 2e-2}   # bf16: the tensor-core forward's states carry bf16 rounding


def _layer_case(shape, dt_name, seed):
    Bz, L, H, P, N, S = shape
    inp = synth.layer_inputs(synth.LayerShape(Bz, L, H, P, N, S, dt_name, "loguniform"), seed=seed)
    r = np.random.default_rng(seed)
    C = -(-L // S)
    dy = torch.from_numpy(r.standard_normal((Bz, L, H, P)).astype(np.float32))
    gdH = torch.from_numpy((r.standard_normal((Bz, H, C, N, P)) * 0.5).astype(np.float32))
    h0 = torch.from_numpy((r.standard_normal((Bz, H, N, P)) * 0.2).astype(np.float32))
    return inp, dy, gdH, h0


@pytest.mark.parametrize("shape,dt_name,with_init", SCAN_CASES, ids=SCAN_IDS)
def test_scan_backward_matches_oracle(shape, dt_name, with_init):
    Bz, L, H, P, N, S = shape
    inp, dy, gdH, h0 = _layer_case(shape, dt_name, seed=L + 1)
    h0 = h0 if with_init else None
    d = {k: inp[k].cuda() for k in ("x", "dt", "A", "Bm", "Cm")}
    _, _, states = dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S,
                                            None if h0 is None else h0.cuda())
    got = dart.dart_ssd_scan_backward(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S, states, dy.cuda(), gdH.cuda(),
                                      None if h0 is None else h0.cuda())
    dart.dart_sync_status()
    ref = dart_backward.scan_grads(*(inp[k].double().numpy() for k in ("x", "dt", "A", "Bm", "Cm")), S,
                                   dy.double().numpy(), gdH.double().numpy(),
                                   init_state=None if h0 is None else h0.double().numpy())
    tol = TOL_FWD_INPUTS[dt_name]
    for k in ("dx", "ddt", "dA", "dBm", "dCm") + (("dinit_state",) if h0 is not None else ()):
        assert_close(k, got[k], ref[k], tol)
    # dCm_add is added into dCm inside the library: the same float sum as
    # adding it afterwards, so the two agree bit for bit
    add = torch.from_numpy(np.random.default_rng(L + 3).standard_normal((Bz, L, N)).astype(np.float32)).cuda()
    got2 = dart.dart_ssd_scan_backward(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S, states, dy.cuda(),
                                       gdH.cuda(), None if h0 is None else h0.cuda(), dCm_add=add)
    dart.dart_sync_status()
    assert torch.equal(got2["dCm"], got["dCm"] + add)
    assert torch.equal(got2["dx"], got["dx"])


@pytest.mark.parametrize("shape,dt_name,with_init", [SCAN_CASES[0], SCAN_CASES[3]], ids=[SCAN_IDS[0], SCAN_IDS[3]])
def test_layer_backward_matches_oracle(shape, dt_name, with_init):
    """dart.layer_backward (forward scan, SMA backward, scan backward driven
    by dy and the memory gradients) against autograd over the whole layer."""
    Bz, L, H, P, N, S = shape
    inp, dy, _, h0 = _layer_case(shape, dt_name, seed=L + 2)
    h0 = h0 if with_init else None
    g = 0.6
    keys = ("x", "dt", "A", "Bm", "Cm", "Q", "E")
    got = dart.layer_backward(*(inp[k].cuda() for k in keys), S, g, dy.cuda(),
                              None if h0 is None else h0.cuda())
    dart.dart_sync_status()
    ref = dart_backward.layer_grads(*(inp[k].double().numpy() for k in keys), S, g, dy.double().numpy(),
                                    init_state=None if h0 is None else h0.double().numpy())
    tol = TOL_FWD_INPUTS[dt_name]
    for k in ("dx", "ddt", "dA", "dBm", "dCm", "dQ", "dE") + (("dinit_state",) if h0 is not None else ()):
        assert_close(k, got[k], ref[k], tol)
    assert abs(float(got["dg"][0]) - float(ref["dg"])) <= tol * max(1.0, abs(float(ref["dg"])))


def test_scan_backward_train_L8k_every_output():
    """The training-length layer (B=2, L=8192, H=32, P=64, N=128, S=256,
    bf16): the chunk-parallel scan backward against the C oracle's
    token-by-token reverse-mode walk on every output element, driven by
    random dy and memory gradients and an initial state."""
    shape = synth.TRAIN_L8K
    S = shape.chunk
    inp = synth.layer_inputs(shape, seed=9)
    r = np.random.default_rng(9)
    Bz, L, H, P, N = shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.dstate
    C = L // S
    dy = torch.from_numpy(r.standard_normal((Bz, L, H, P)).astype(np.float32))
    gdH = torch.from_numpy((r.standard_normal((Bz, H, C, N, P)) * 0.5).astype(np.float32))
    h0 = torch.from_numpy((r.standard_normal((Bz, H, N, P)) * 0.2).astype(np.float32))
    d = {k: inp[k].cuda() for k in ("x", "dt", "A", "Bm", "Cm")}
    _, _, states = dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S, h0.cuda())
    got = dart.dart_ssd_scan_backward(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], S, states, dy.cuda(),
                                      gdH.cuda(), h0.cuda())
    dart.dart_sync_status()
    ref = dart_oracle.get().scan_backward(*(inp[k].float().numpy() for k in ("x", "dt", "A", "Bm", "Cm")), S,
                                          dy.numpy(), gdH.numpy(), init_state=h0.numpy())
    for k in ("dx", "ddt", "dA", "dBm", "dCm", "dinit_state"):
        assert_close(k, got[k], ref[k], TOL_FWD_INPUTS["bf16"])
