"""GPU parity of the decayed-memory SMA variant (referee major comment 3 on SMA
Eq. (8), Pith review of DART: memories carried to the query token by the
recurrence's decay) against the fp64 oracle on the same seeded inputs.
Tolerances as in test_gpu_parity: max|err|/max|ref| <= 1e-4 (float32) and
<= 2e-2 (bf16 inputs, float32 accumulation)."""
import numpy as np
import pytest
import torch

from mamba_ssd_state_b200 import build, dart, synth
from mamba_ssd_state_b200.synth import LayerShape
from oracle import dart_oracle
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


def _layer(orc, shape, inp, tol, tokens=None):
    """Scan on the GPU, then decayed SMA on the GPU (raw o and gated y); the
    oracle runs the same layer with decayed memories over its own fp64 dH."""
    d = to_device(inp)
    y_ssd, dH, _ = dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], shape.chunk)
    o = dart.dart_sma_forward_decayed(d["Q"], d["E"], d["Cm"], dH, d["dt"], d["A"], shape.chunk, d["g"])
    y = dart.dart_sma_forward_decayed(d["Q"], d["E"], d["Cm"], dH, d["dt"], d["A"], shape.chunk, d["g"],
                                      y_ssd.clone())
    dart.dart_sync_status()
    oi = oracle_inputs(inp)
    ref = orc.layer_forward(oi["x"], oi["dt"], oi["A"], oi["Bm"], oi["Cm"], oi["Q"], oi["E"], shape.chunk,
                            inp["g"], tokens=tokens, decayed=True)
    if tokens is not None:
        o, y = o[:, tokens], y[:, tokens]
    assert_close("o", o, ref["o"], tol)
    assert_close("y", y, ref["y"], tol)
    return o, y, ref


def _mild(inp, a=-0.05):
    """A small |A| so that several memories survive to the end of a chunk."""
    inp = dict(inp)
    inp["A"] = torch.full_like(inp["A"], a)
    return inp


def test_decayed_bf16_pair_kernel_default_decay(orc):
    """S = 256 (CTA-pair tensor-core kernel), 7 chunks, 3 heads, the synthetic
    dt / A distribution (strong decay: mostly the latest memory counts)."""
    shape = LayerShape(1, 7 * 256, 3, 64, 128, 256, "bf16", "loguniform")
    _layer(orc, shape, synth.layer_inputs(shape, seed=31), TOL[torch.bfloat16])


def test_decayed_bf16_pair_kernel_mild_decay(orc):
    """A = -0.05: every memory keeps a weight between about e^-2 and 1, so the
    softmax mixes many of them; 10 chunks exercise several memory batches."""
    shape = LayerShape(2, 10 * 256, 2, 64, 128, 256, "bf16", "loguniform")
    _layer(orc, shape, _mild(synth.layer_inputs(shape, seed=32)), TOL[torch.bfloat16])


def test_decayed_bf16_single_cta_S128(orc):
    shape = LayerShape(1, 9 * 128, 3, 64, 128, 128, "bf16", "loguniform")
    _layer(orc, shape, _mild(synth.layer_inputs(shape, seed=33), -0.1), TOL[torch.bfloat16])


@pytest.mark.parametrize("tail", [200, 37])
def test_decayed_bf16_partial_last_chunk(orc, tail):
    shape = LayerShape(1, 6 * 256 + tail, 2, 64, 128, 256, "bf16", "loguniform")
    _layer(orc, shape, _mild(synth.layer_inputs(shape, seed=34 + tail)), TOL[torch.bfloat16])


def test_decayed_fp32_cuda_core_path(orc):
    """float32 throughout (CUDA-core SMA), N = P = 16, S = 64, with a partial
    last chunk."""
    shape = LayerShape(1, 9 * 64 + 21, 2, 16, 16, 64, "f32", "softplus")
    _layer(orc, shape, _mild(synth.layer_inputs(shape, seed=35), -0.2), TOL[torch.float32])


def test_decayed_bf16_N64_cuda_core_path(orc):
    shape = LayerShape(1, 5 * 128, 2, 64, 64, 128, "bf16", "loguniform")
    assert dart.sma_impl(64, 64, 128, torch.bfloat16) == "sma_simt"
    _layer(orc, shape, _mild(synth.layer_inputs(shape, seed=36)), TOL[torch.bfloat16])


@pytest.mark.parametrize("chunk", [256, 128])
def test_decayed_with_A_zero_equals_raw(orc, chunk):
    """A = 0: nothing decays, so the decayed variant reproduces the raw SMA."""
    shape = LayerShape(1, 6 * chunk, 2, 64, 128, chunk, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=37)
    d = to_device(inp)
    dH = synth.memory_inputs(1, 2, 6, 128, 64, "bf16", seed=37).cuda()
    zero = torch.zeros_like(d["A"])
    dec = dart.dart_sma_forward_decayed(d["Q"], d["E"], d["Cm"], dH, d["dt"], zero, chunk, 0.5)
    raw = dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, chunk, 0.5)
    dart.dart_sync_status()
    assert_close("decayed(A=0) vs raw", dec, raw.double().cpu().numpy(), 1e-6)


def test_decayed_train_L8k_sampled(orc):
    """The B=2, L=8192, H=32, S=256 training shape, in the launch form the
    benchmark times (output in place over y_ssd), checked on sampled tokens
    (every chunk's first and last token plus random ones) of two heads."""
    shape = synth.TRAIN_L8K
    inp = synth.layer_inputs(shape, seed=0)
    d = to_device(inp)
    y_ssd, dH, _ = dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], shape.chunk)
    y = y_ssd.clone()
    dart.dart_sma_forward_decayed(d["Q"], d["E"], d["Cm"], dH, d["dt"], d["A"], shape.chunk, d["g"], y, out=y)
    dart.dart_sync_status()
    heads = [5, 27]
    sub = dict(inp)
    for k in ("x", "dt", "Q", "E"):
        sub[k] = inp[k][:, :, heads]
    sub["A"] = inp["A"][heads]
    oi = oracle_inputs(sub)
    r = np.random.default_rng(8)
    tok = sorted(set([c * 256 for c in range(32)] + [c * 256 + 255 for c in range(32)]
                     + r.integers(0, shape.seqlen, 48).tolist()))
    ref = orc.layer_forward(oi["x"], oi["dt"], oi["A"], oi["Bm"], oi["Cm"], oi["Q"], oi["E"], shape.chunk,
                            inp["g"], tokens=tok, decayed=True)
    assert_close("y (sampled)", y[:, tok][:, :, heads], ref["y"], TOL[torch.bfloat16])
    # the o part alone, relative to its own scale
    o_gpu = (y[:, tok][:, :, heads] - y_ssd[:, tok][:, :, heads]) / inp["g"]
    assert_close("o (sampled)", o_gpu, ref["o"], TOL[torch.bfloat16])


def test_decayed_layer_forward_binding(orc):
    """dart.layer_forward(decayed=True) from host tensors equals the two-call
    device path."""
    shape = LayerShape(1, 4 * 256, 2, 64, 128, 256, "bf16", "loguniform")
    inp = _mild(synth.layer_inputs(shape, seed=38))
    host = dart.layer_forward(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], inp["Q"], inp["E"],
                              shape.chunk, inp["g"], outputs=("y",), decayed=True)["y"]
    _, y, _ = _layer(orc, shape, inp, TOL[torch.bfloat16])
    assert torch.equal(host, y.cpu())
