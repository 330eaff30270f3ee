"""GPU parity of the fp8 (OCP E4M3) decode cache against the fp64 oracle.

Quantization is byte work: the codes and row exponents the library writes
for a given memory must equal the oracle's bit for bit.  The decode step
reads dequantized memories, so its outputs are compared like the bf16
decode (max|err|/max|ref| <= 2e-2 for bf16 token inputs, 1e-4 for float32).
A memory appended during decode is quantized from the running fp32
contribution on the GPU and from fp64 in the oracle, so a code may flip to
its neighbour where the two land on either side of a rounding boundary;
those flips are counted and bounded instead of required to be absent."""
import numpy as np
import pytest
import torch

from mamba_ssd_state_b200 import build, dart, synth
from mamba_ssd_state_b200.synth import DecodeShape, LayerShape
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


def _gpu_quantize(dH, nmem, cmax):
    """E4M3 cache (device tensors) holding memories 0..nmem-1 of dH."""
    B, H, C, N, P = dH.shape
    cache = torch.full((B, H, cmax, N, P), 0xAB, dtype=torch.uint8, device="cuda")
    cexp = torch.full((B, H, cmax, N), 99, dtype=torch.int8, device="cuda")
    dart.cache_quantize_e4m3(dH.cuda().contiguous(), nmem, cache, cexp)
    dart.dart_sync_status()
    return cache, cexp


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_cache_quantize_is_bit_exact(orc, dtype):
    """Memories whose rows span 1e-7 .. 1e3 in magnitude (subnormal codes,
    exponents from about -30 to 2, all-zero rows): codes and exponents equal
    the oracle's; slots past nmem are left untouched."""
    r = np.random.default_rng(51)
    B, H, C, N, P = 2, 3, 5, 128, 64
    x = r.standard_normal((B, H, C, N, P)) * np.exp(r.uniform(np.log(1e-7), np.log(1e3), (B, H, C, N, 1)))
    x[0, 1, 2, 7] = 0.0
    x[1, 0, 3, 9, :] = 0.0
    x[1, 0, 3, 9, 5] = -2.5e-6
    dH = torch.from_numpy(x.astype(np.float32)).to(dtype)
    cache, cexp = (t.cpu() for t in _gpu_quantize(dH, 4, 6))
    codes, exps, _ = orc.quantize_e4m3(dH[:, :, :4].double().numpy())
    assert np.array_equal(cexp[:, :, :4].numpy(), exps), "row exponents"
    diff = cache[:, :, :4].numpy() != codes
    assert not diff.any(), f"{int(diff.sum())} of {diff.size} codes differ"
    assert torch.all(cache[:, :, 4:] == 0xAB) and torch.all(cexp[:, :, 4:] == 99)


def _e4m3_init(orc, shape, init, seqs):
    """E4M3 cache of the initial memories on both sides: the GPU quantizes the
    shape's memories, the oracle quantizes the same values of the sequences
    it follows (bit-exact, see above) and keeps them dequantized as its cache."""
    cache, cexp = _gpu_quantize(init["cache"], shape.cmax, shape.cmax)
    _, _, deq = orc.quantize_e4m3(init["cache"][seqs].double().numpy())
    return cache, cexp, deq


def _run(orc, shape, init, steps, seqs, seed=0, check_every=1, memlog=None):
    tol = TOL[synth.torch_dtype(shape.dtype)]
    A = synth.decode_A(shape, seed)
    cache, cexp, deq = _e4m3_init(orc, shape, init, seqs)
    dev = {k: v.cuda() for k, v in init.items() if k != "cache"}
    dev["cache"], dev["cache_exp"] = cache, cexp
    ref = {"cache": np.ascontiguousarray(deq), "state": init["state"][seqs].double().numpy().copy(),
           "dH_cur": init["dH_cur"][seqs].double().numpy().copy(), "nchunks": init["nchunks"][seqs].numpy().copy(),
           "pos": init["pos"][seqs].numpy().copy()}
    ml_dev = None if memlog is None else memlog.cuda().contiguous()
    ml_ref = None if memlog is None else memlog[seqs].double().numpy().copy()
    for step in range(steps):
        tok = synth.decode_tokens(shape, step, seed)
        y = dart.dart_decode_step(tok["x"].cuda(), tok["dt"].cuda(), A.cuda(), tok["Bm"].cuda(), tok["Cm"].cuda(),
                                  tok["Q"].cuda(), tok["E"].cuda(), shape.g, dev["state"], dev["dH_cur"],
                                  dev["cache"], dev["nchunks"], dev["pos"], shape.chunk, memlog=ml_dev,
                                  cache_exp=dev["cache_exp"])
        t = oracle_inputs({k: v[seqs] for k, v in tok.items()})
        yr = orc.decode_step(t["x"], t["dt"], A.numpy(), t["Bm"], t["Cm"], t["Q"], t["E"], shape.g, ref["state"],
                             ref["dH_cur"], ref["cache"], ref["nchunks"], ref["pos"], shape.chunk,
                             memlog=ml_ref, cache_e4m3=True)
        if step % check_every == 0 or step == steps - 1:
            assert_close(f"y step {step}", y[seqs], yr, tol)
    dart.dart_sync_status()
    assert np.array_equal(dev["nchunks"].cpu().numpy()[seqs], ref["nchunks"])
    assert np.array_equal(dev["pos"].cpu().numpy()[seqs], ref["pos"])
    assert_close("state", dev["state"][seqs], ref["state"], tol)
    assert_close("dH_cur", dev["dH_cur"][seqs], ref["dH_cur"], tol)
    # every cached memory, dequantized: the initial ones exactly, appended ones up to neighbour flips
    codes = dev["cache"][seqs].cpu()
    ex = dev["cache_exp"][seqs].cpu()
    vals = codes.view(torch.float8_e4m3fn).double() * torch.exp2(ex.double())[..., None]
    for i, b in enumerate(seqs):
        n0, n = int(init["nchunks"][b]), int(ref["nchunks"][i])
        got, want = vals[i, :, :n].numpy(), ref["cache"][i, :, :n]
        assert np.array_equal(got[:, :n0], want[:, :n0]), "initial memories"
        if n > n0:
            flips = got[:, n0:] != want[:, n0:]
            assert flips.mean() <= 1e-3, f"{int(flips.sum())} appended codes differ"
            rel = np.abs(got[:, n0:] - want[:, n0:]) / np.maximum(np.abs(want[:, n0:]), 1e-30)
            assert np.all(rel[flips] <= 0.126), "a differing code is more than one step away"
    return dev, ref


def _small(shape, nchunks, pos, seed):
    init = synth.decode_initial(shape, seed)
    init["nchunks"] = torch.tensor(nchunks, dtype=torch.int32)
    init["pos"] = torch.tensor(pos, dtype=torch.int32)
    r = np.random.default_rng(seed)
    for b, p in enumerate(pos):
        if p > 0:
            init["dH_cur"][b] = torch.from_numpy(r.standard_normal(init["dH_cur"][b].shape).astype(np.float32) * 0.05)
    return init


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_e4m3_decode_small_with_appends(orc, dtype):
    """Three sequences at different counters with chunk size 4: several
    appends quantized on the fly; one sequence starts from an empty cache."""
    shape = DecodeShape(3, 2, 64, 128, 4, 7, 7, 9, dtype)
    _run(orc, shape, _small(shape, [2, 0, 3], [0, 2, 3], seed=5), shape.nsteps, [0, 1, 2])


def test_e4m3_decode_N64(orc):
    shape = DecodeShape(2, 3, 64, 64, 8, 5, 6, 11, "bf16")
    _run(orc, shape, _small(shape, [1, 4], [6, 0], seed=6), shape.nsteps, [0, 1])


def test_e4m3_decayed_decode(orc):
    """The fp8 cache with decayed memories (mem_logdecay given)."""
    shape = DecodeShape(3, 2, 64, 128, 4, 7, 7, 9, "bf16")
    init = _small(shape, [2, 0, 3], [0, 2, 3], seed=7)
    r = np.random.default_rng(7)
    ml = -r.uniform(0, 3, (3, 2, 7)).astype(np.float32)
    _run(orc, shape, init, shape.nsteps, [0, 1, 2], memlog=torch.from_numpy(ml))


def test_e4m3_decode_config_sampled(orc):
    """The 64-sequence, 128-memory decode batch from an E4M3 cache, 256 steps
    with the append on the last; the oracle follows sequences 0 and 63."""
    shape = synth.DECODE_64x32K
    init = synth.decode_initial(shape, seed=0)
    dev, ref = _run(orc, shape, init, shape.nsteps, [0, 63], check_every=15)
    assert int(dev["nchunks"].min()) == 129


def test_e4m3_prefill_handoff_tracks_bf16_decode():
    """Prefill of 2 S + 100 tokens, its complete memories quantized into an
    E4M3 cache, then decode to 4 S: outputs stay within the E4M3 rounding
    (2^-4 relative per element) of the same decode from the bf16 cache."""
    S = 256
    shape = LayerShape(2, 4 * S, 3, 64, 128, S, "bf16", "loguniform")
    d = to_device(synth.layer_inputs(shape, seed=25))
    L = 2 * S + 100
    keys = ("x", "dt", "A", "Bm", "Cm", "Q", "E")
    pre = dart.layer_forward(*(d[k][:, :L] if k != "A" else d[k] for k in keys), S, d["g"])
    B, H, N, P, cmax = 2, 3, 128, 64, 5
    runs = []
    for e4m3 in (False, True):
        if e4m3:
            cache = torch.zeros(B, H, cmax, N, P, dtype=torch.uint8, device="cuda")
            cexp = torch.zeros(B, H, cmax, N, dtype=torch.int8, device="cuda")
            dart.cache_quantize_e4m3(pre["dH"], 2, cache, cexp)
        else:
            cache = torch.zeros(B, H, cmax, N, P, dtype=torch.bfloat16, device="cuda")
            cache[:, :, :2] = pre["dH"][:, :, :2]
            cexp = None
        state = pre["states"][:, :, -1].contiguous()
        dcur = pre["dH"][:, :, -1].float().contiguous()
        nch = torch.full((B,), 2, dtype=torch.int32, device="cuda")
        pos = torch.full((B,), L % S, dtype=torch.int32, device="cuda")
        ys = [dart.dart_decode_step(d["x"][:, t], d["dt"][:, t], d["A"], d["Bm"][:, t], d["Cm"][:, t],
                                    d["Q"][:, t], d["E"][:, t], d["g"], state, dcur, cache, nch, pos, S,
                                    cache_exp=cexp) for t in range(L, 4 * S)]
        dart.dart_sync_status()
        runs.append(torch.stack(ys, 1))
        assert torch.all(nch == 4) and torch.all(pos == 0)
    assert_close("E4M3 vs bf16 cache decode", runs[1], runs[0].double().cpu().numpy(), 0.07)
