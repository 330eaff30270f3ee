"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on
the same seeded inputs.  Tolerance: max|err|/max|ref| <= 1e-4 (float32 runs)
and <= 2e-2 (bf16 inputs, float32 accumulation), per output tensor."""
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


def gpu_layer(inp, shape, init_state=None):
    d = to_device(inp)
    y_ssd, dH, st = dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], shape.chunk,
                                             None if init_state is None else init_state.cuda())
    o = dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, shape.chunk, d["g"])
    y = dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, shape.chunk, d["g"], y_ssd)
    dart.dart_sync_status()
    return {"y_ssd": y_ssd, "dH": dH, "states": st, "o": o, "y": y}


def heads_slice(inp, heads):
    """Inputs restricted to a subset of heads (heads are independent problems)."""
    out = dict(inp)
    for k in ("x", "dt", "Q", "E"):
        out[k] = inp[k][:, :, heads]
    out["A"] = inp["A"][heads]
    return out


def check_full(orc, shape, inp, tol, init_state=None, outputs=("y_ssd", "dH", "states", "o", "y")):
    got = gpu_layer(inp, shape, init_state)
    o = oracle_inputs(inp)
    ref = orc.layer_forward(o["x"], o["dt"], o["A"], o["Bm"], o["Cm"], o["Q"], o["E"], shape.chunk,
                            inp["g"], init_state=None if init_state is None else init_state.numpy())
    errs = {k: assert_close(k, got[k], ref[k], tol) for k in outputs}
    return got, ref, errs


# ---------------------------------------------------------------------------
# full-size comparisons at sizes the oracle finishes in seconds
# ---------------------------------------------------------------------------
def test_tiny_fp32_config(orc):
    """B=1, L=512, H=2, P=16, N=16, S=64, float32 throughout."""
    inp = synth.layer_inputs(synth.TINY_FP32, seed=0)
    check_full(orc, synth.TINY_FP32, inp, TOL[torch.float32])


def test_bf16_ragged_chunks_several_tiles(orc):
    """7 chunks of 256 (an odd number of memories, several query tiles per
    chunk, a ragged last group) with 3 heads."""
    shape = LayerShape(1, 7 * 256, 3, 64, 128, 256, "bf16", "loguniform")
    check_full(orc, shape, synth.layer_inputs(shape, seed=1), TOL[torch.bfloat16])


def test_bf16_many_heads_per_group(orc):
    """16 and 32 heads: the scan kernels walk many heads per CTA, so every
    double-buffered stage is reused several times; every head is compared."""
    for H, seed in ((16, 41), (32, 42)):
        shape = LayerShape(1, 3 * 256, H, 64, 128, 256, "bf16", "loguniform")
        check_full(orc, shape, synth.layer_inputs(shape, seed=seed), TOL[torch.bfloat16])


def test_bf16_two_batches_S128(orc):
    shape = LayerShape(2, 5 * 128, 2, 64, 128, 128, "bf16", "loguniform")
    check_full(orc, shape, synth.layer_inputs(shape, seed=2), TOL[torch.bfloat16])


def test_fp32_N64_P64_S64(orc):
    shape = LayerShape(1, 6 * 64, 2, 64, 64, 64, "f32", "softplus")
    check_full(orc, shape, synth.layer_inputs(shape, seed=3), TOL[torch.float32])


def test_bf16_N64_P64_cuda_core_path(orc):
    """bf16 at a shape the tensor-core kernel does not cover (N=64) runs the
    CUDA-core SMA kernel; same tolerance."""
    assert dart.sma_impl(64, 64, 128, torch.bfloat16) == "sma_simt"
    shape = LayerShape(2, 5 * 128, 2, 64, 64, 128, "bf16", "loguniform")
    check_full(orc, shape, synth.layer_inputs(shape, seed=31), TOL[torch.bfloat16])


# ---------------------------------------------------------------------------
# sequences that end inside a chunk (C = ceil(L / S), the last chunk partial)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("tail", [200, 100, 37])
def test_bf16_partial_last_chunk(orc, tail):
    """3 full chunks of 256 and a partial one: 200 tokens (its second 128-row
    half partly past the end), 100 (second half entirely past the end) and 37;
    two sequences, so a box past the end of the first must not reach the
    second."""
    shape = LayerShape(2, 3 * 256 + tail, 3, 64, 128, 256, "bf16", "loguniform")
    check_full(orc, shape, synth.layer_inputs(shape, seed=50 + tail), TOL[torch.bfloat16])


def test_bf16_partial_last_chunk_S128(orc):
    """S = 128 (one-CTA attention kernel), 4 full chunks and 60 tokens."""
    shape = LayerShape(2, 4 * 128 + 60, 2, 64, 128, 128, "bf16", "loguniform")
    check_full(orc, shape, synth.layer_inputs(shape, seed=53), TOL[torch.bfloat16])


def test_fp32_partial_last_chunk(orc):
    """The CUDA-core kernels: fp32, S = 64, 7 full chunks and 27 tokens."""
    shape = LayerShape(2, 7 * 64 + 27, 2, 16, 16, 64, "f32", "softplus")
    check_full(orc, shape, synth.layer_inputs(shape, seed=54), TOL[torch.float32])


def test_dispatch_uses_tensor_cores_for_the_layer_shape():
    assert dart.sma_impl(128, 64, 256, torch.bfloat16) == "sma_tcgen05"
    assert dart.sma_impl(128, 64, 128, torch.bfloat16) == "sma_tcgen05"
    assert dart.sma_impl(128, 64, 256, torch.float32) == "sma_simt"


def test_layer_L2k_config_full(orc):
    """B=4, L=2048, H=32, P=64, N=128, S=256 (the Mamba-2-370M layer shape)."""
    inp = synth.layer_inputs(synth.LAYER_L2K, seed=0)
    check_full(orc, synth.LAYER_L2K, inp, TOL[torch.bfloat16])


# ---------------------------------------------------------------------------
# the two large configurations: every output of a head subset for the scan,
# and sampled token rows (first/last of every chunk plus random) for SMA
# ---------------------------------------------------------------------------
def _sample_tokens(L, S, n_random, seed):
    r = np.random.default_rng(seed)
    t = set()
    for c in range(L // S):
        t.update((c * S, c * S + S - 1))
    t.update(r.integers(0, L, n_random).tolist())
    return sorted(t)


def test_train_L8k_config_full(orc):
    """B=2, L=8192, H=32, P=64, N=128, S=256: every output element."""
    inp = synth.layer_inputs(synth.TRAIN_L8K, seed=0)
    check_full(orc, synth.TRAIN_L8K, inp, TOL[torch.bfloat16])


@pytest.mark.parametrize("shape,heads,nrand", [(synth.LONG_L64K, [0, 3, 9, 15, 16, 22, 30, 31], 64)],
                         ids=["long_L64k"])
def test_large_config_sampled(orc, shape, heads, nrand):
    """L = 65536 (256 chunks, 32 heads): the scan compared on every head and
    every element, so every persistent CTA's first and last work item is
    checked whatever the split; SMA on sampled token rows (first and last of
    every chunk plus random ones) of eight heads spread over the range."""
    inp = synth.layer_inputs(shape, seed=0)
    got = gpu_layer(inp, shape)
    o = oracle_inputs(inp)
    y_ssd, dH, st = orc.ssd_scan(o["x"], o["dt"], o["A"], o["Bm"], o["Cm"], shape.chunk)
    tol = TOL[torch.bfloat16]
    for h0 in range(0, shape.nheads, 8):    # per head block, so a bad head is named
        hs = slice(h0, h0 + 8)
        assert_close(f"y_ssd heads {h0}..", got["y_ssd"][:, :, hs], y_ssd[:, :, hs], tol)
        assert_close(f"dH heads {h0}..", got["dH"][:, hs], dH[:, hs], tol)
        assert_close(f"states heads {h0}..", got["states"][:, hs], st[:, hs], tol)
    o = oracle_inputs(heads_slice(inp, heads))
    y_ssd, dH = y_ssd[:, :, heads], dH[:, heads]
    tok = _sample_tokens(shape.seqlen, shape.chunk, nrand, seed=5)
    r = orc.sma(o["Q"], o["E"], o["Cm"], dH, shape.chunk, inp["g"], y_ssd[:, tok], tokens=tok)
    assert_close("o (sampled)", got["o"][:, tok][:, :, heads], r["o"], tol)
    assert_close("y (sampled)", got["y"][:, tok][:, :, heads], r["y"], tol)


# ---------------------------------------------------------------------------
# edge cases of the method
# ---------------------------------------------------------------------------
def test_single_chunk_has_no_memory(orc):
    """L = S: no chunk memory exists, so o = 0 and y = y_ssd."""
    shape = LayerShape(2, 256, 4, 64, 128, 256, "bf16", "loguniform")
    got, _, _ = check_full(orc, shape, synth.layer_inputs(shape, seed=4), TOL[torch.bfloat16])
    assert torch.count_nonzero(got["o"]) == 0
    assert torch.equal(got["y"], got["y_ssd"])


def test_two_chunks(orc):
    shape = LayerShape(1, 512, 2, 64, 128, 256, "bf16", "loguniform")
    check_full(orc, shape, synth.layer_inputs(shape, seed=5), TOL[torch.bfloat16])


def test_peaked_softmax(orc):
    """Queries scaled by 30 make the softmax nearly one-hot, so score errors
    would surface directly in the output."""
    shape = LayerShape(1, 6 * 256, 2, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=6)
    inp["Q"] = (inp["Q"].float() * 30).to(torch.bfloat16)
    check_full(orc, shape, inp, TOL[torch.bfloat16])


def test_heavy_decay(orc):
    """A = -16 on every head: memories are dominated by the last few tokens
    of their chunk and the inter-chunk term nearly vanishes."""
    shape = LayerShape(1, 4 * 256, 2, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=7)
    inp["A"] = torch.full_like(inp["A"], -16.0)
    check_full(orc, shape, inp, TOL[torch.bfloat16])


def test_gate_zero_is_mamba2(orc):
    shape = LayerShape(1, 3 * 256, 2, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=8)
    inp["g"] = 0.0
    got, _, _ = check_full(orc, shape, inp, TOL[torch.bfloat16])
    assert torch.equal(got["y"], got["y_ssd"])


def test_init_state(orc):
    shape = LayerShape(1, 3 * 256, 2, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=9)
    h0 = torch.from_numpy(np.random.default_rng(9).standard_normal((1, 2, 128, 64)).astype(np.float32) * 0.1)
    check_full(orc, shape, inp, TOL[torch.bfloat16], init_state=h0)


def test_init_state_fp32(orc):
    shape = LayerShape(1, 4 * 64, 2, 16, 16, 64, "f32", "softplus")
    inp = synth.layer_inputs(shape, seed=10)
    h0 = torch.from_numpy(np.random.default_rng(10).standard_normal((1, 2, 16, 16)).astype(np.float32))
    check_full(orc, shape, inp, TOL[torch.float32], init_state=h0)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_one_hot_memories_pin_the_mask(orc, dtype):
    """dH[c] = (c+1) e0 e0^T and a large query: the softmax is one-hot on the
    last allowed chunk, so o_t[0] = chunk(t) * C_t[0] exactly up to rounding;
    an off-by-one in the causal mask moves it by a whole chunk."""
    Bz, L, H, N, P, S = 1, 8 * 256, 2, 128, 64, 256
    C = L // S
    dH = torch.zeros(Bz, H, C, N, P)
    for c in range(C):
        dH[:, :, c, 0, 0] = c + 1.0
    Q = torch.zeros(Bz, L, H, N)
    Q[..., 0] = 400.0
    E = torch.zeros(Bz, L, H, P)
    E[..., 0] = 1.0
    Cm = torch.from_numpy(np.random.default_rng(11).uniform(0.5, 1.5, (Bz, L, N)).astype(np.float32))
    Q, E, Cm, dHd = (t.to(dtype) for t in (Q, E, Cm, dH))
    o = dart.dart_sma_forward(Q.cuda(), E.cuda(), Cm.cuda(), dHd.cuda(), S, 1.0).cpu()
    k = (torch.arange(L) // S).float()
    expect = k[None, :, None] * Cm.float()[:, :, None, 0]
    tol = 1e-6 if dtype == torch.float32 else 1e-2
    assert torch.allclose(o[..., 0], expect.expand(Bz, L, H), rtol=tol, atol=0)
    assert torch.count_nonzero(o[..., 1:]) == 0
    ref = orc.sma(Q.float().numpy(), E.float().numpy(), Cm.float().numpy(), dHd.float().numpy(), S, 1.0)
    assert_close("o", o, ref["o"], TOL[dtype])


def test_sma_on_shared_memories(orc):
    """SMA alone, both sides fed the same generated bf16 chunk memories."""
    shape = LayerShape(2, 9 * 256, 3, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=12)
    dH = synth.memory_inputs(2, 3, 9, 128, 64, "bf16", seed=12)
    o = dart.dart_sma_forward(inp["Q"].cuda(), inp["E"].cuda(), inp["Cm"].cuda(), dH.cuda(), 256, 0.5)
    oi = oracle_inputs(inp)
    ref = orc.sma(oi["Q"], oi["E"], oi["Cm"], dH.float().numpy(), 256, 0.5)
    assert_close("o", o, ref["o"], TOL[torch.bfloat16])


def test_sma_output_modes(orc):
    """out = y_ssd + g o written three ways: in place over y_ssd, into a
    separate buffer (y_ssd left untouched), and o alone without y_ssd."""
    shape = LayerShape(2, 6 * 256, 3, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=21)
    dH = synth.memory_inputs(2, 3, 6, 128, 64, "bf16", seed=21).cuda()
    d = to_device(inp)
    y_ssd = torch.randn(2, 6 * 256, 3, 64, generator=torch.Generator().manual_seed(21)).cuda()
    oi = oracle_inputs(inp)
    ref = orc.sma(oi["Q"], oi["E"], oi["Cm"], dH.float().cpu().numpy(), 256, 0.5, y_ssd.cpu().double().numpy())
    keep = y_ssd.clone()
    sep = dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, 256, 0.5, y_ssd)
    assert torch.equal(y_ssd, keep)
    inplace = y_ssd.clone()
    dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, 256, 0.5, inplace, out=inplace)
    o = dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, 256, 0.5)
    dart.dart_sync_status()
    assert_close("y (separate out)", sep, ref["y"], TOL[torch.bfloat16])
    assert_close("y (in place)", inplace, ref["y"], TOL[torch.bfloat16])
    assert_close("o", o, ref["o"], TOL[torch.bfloat16])
    assert torch.equal(sep, inplace)


def test_deterministic():
    shape = LayerShape(1, 4 * 256, 4, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=13)
    a = gpu_layer(inp, shape)
    b = gpu_layer(inp, shape)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_host_buffer_path_matches_device_path():
    shape = LayerShape(1, 3 * 256, 2, 64, 128, 256, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=14)
    host = dart.layer_forward(inp["x"], inp["dt"], inp["A"], inp["Bm"], inp["Cm"], inp["Q"], inp["E"],
                              256, inp["g"])
    d = to_device(inp)
    dev = dart.layer_forward(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], d["Q"], d["E"], 256, d["g"])
    assert not host["y"].is_cuda
    assert torch.equal(host["y"], dev["y"].cpu())
