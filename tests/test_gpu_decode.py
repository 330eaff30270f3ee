"""GPU parity of the decode step against the oracle, prefill/decode
consistency on the GPU, and the device-side error path."""
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


def _oracle_state(init):
    return {"cache": init["cache"].double().numpy().copy(), "state": init["state"].double().numpy().copy(),
            "dH_cur": init["dH_cur"].double().numpy().copy(), "nchunks": init["nchunks"].numpy().copy(),
            "pos": init["pos"].numpy().copy()}


def _run_decode(orc, shape, init, steps, seqs_for_oracle, seed=0, check_every=1, memlog=None):
    """Run `steps` decode steps on the GPU for every sequence and in the
    oracle for `seqs_for_oracle`; compare y each checked step and the final
    state, running contribution, cache and counters.  With `memlog` (float32
    [B,H,cmax]) both sides run the decayed-memory step from it."""
    tol = TOL[synth.torch_dtype(shape.dtype)]
    A = synth.decode_A(shape, seed)
    g = shape.g
    dev = {k: v.cuda() for k, v in init.items()}
    sub = {k: v[seqs_for_oracle] for k, v in init.items()}
    ref = _oracle_state(sub)
    ml_dev = None if memlog is None else memlog.cuda().contiguous()
    ml_ref = None if memlog is None else memlog[seqs_for_oracle].double().numpy().copy()
    worst = 0.0
    for step in range(steps):
        tok = synth.decode_tokens(shape, step, seed)
        y = dart.dart_decode_step(tok["x"].cuda(), tok["dt"].cuda(), A.cuda(), tok["Bm"].cuda(), tok["Cm"].cuda(),
                                  tok["Q"].cuda(), tok["E"].cuda(), g, dev["state"], dev["dH_cur"],
                                  dev["cache"], dev["nchunks"], dev["pos"], shape.chunk, memlog=ml_dev)
        t = oracle_inputs({k: v[seqs_for_oracle] for k, v in tok.items()})
        yr = orc.decode_step(t["x"], t["dt"], A.numpy(), t["Bm"], t["Cm"], t["Q"], t["E"], g, ref["state"],
                             ref["dH_cur"], ref["cache"], ref["nchunks"], ref["pos"], shape.chunk,
                             memlog=ml_ref)
        if step % check_every == 0 or step == steps - 1:
            worst = max(worst, assert_close(f"y step {step}", y[seqs_for_oracle], yr, tol))
    dart.dart_sync_status()
    assert np.array_equal(dev["nchunks"].cpu().numpy()[seqs_for_oracle], ref["nchunks"])
    assert np.array_equal(dev["pos"].cpu().numpy()[seqs_for_oracle], ref["pos"])
    assert_close("state", dev["state"][seqs_for_oracle], ref["state"], tol)
    assert_close("dH_cur", dev["dH_cur"][seqs_for_oracle], ref["dH_cur"], tol)
    got_cache = dev["cache"][seqs_for_oracle]
    for i in range(len(seqs_for_oracle)):
        n = int(ref["nchunks"][i])
        assert_close(f"cache of sequence {seqs_for_oracle[i]}", got_cache[i, :, :n], ref["cache"][i, :, :n], tol)
        if memlog is not None:
            got = ml_dev[seqs_for_oracle[i], :, :n].double().cpu().numpy()
            assert np.allclose(got, ml_ref[i, :, :n], rtol=1e-5, atol=1e-5), "memory log-decays"
    if memlog is not None:
        dev["memlog"] = ml_dev
    return dev, ref, worst


def _memlog(shape, nchunks, seed, junk=50.0):
    """Log-decays of the cached memories, -U(0, 3); slots past nchunks hold
    junk that must be ignored (exp(50) would swamp any read of it)."""
    r = np.random.default_rng(seed)
    ml = -r.uniform(0.0, 3.0, (shape.nseq, shape.nheads, shape.cmax)).astype(np.float32)
    for b in range(shape.nseq):
        ml[b, :, int(nchunks[b]):] = junk
    return torch.from_numpy(ml)


def _small_init(shape, nchunks, pos, seed):
    init = synth.decode_initial(shape, seed)
    init["nchunks"] = torch.tensor(nchunks, dtype=torch.int32)
    init["pos"] = torch.tensor(pos, dtype=torch.int32)
    # a non-zero running contribution for sequences that start mid-chunk
    r = np.random.default_rng(seed)
    for b, p in enumerate(pos):
        if p > 0:
            init["dH_cur"][b] = torch.from_numpy(r.standard_normal(init["dH_cur"][b].shape).astype(np.float32) * 0.05)
    # slots past nchunks hold garbage that must never be read
    for b, n in enumerate(nchunks):
        init["cache"][b, :, n:] = 1e4
    return init


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_small_with_appends(orc, dtype):
    """Three sequences at different counters, chunk size 4: appends happen at
    different steps, one sequence starts with an empty cache."""
    shape = DecodeShape(3, 2, 64, 128, 4, 7, 7, 9, dtype)
    init = _small_init(shape, [2, 0, 3], [0, 2, 3], seed=1)
    _run_decode(orc, shape, init, shape.nsteps, [0, 1, 2])


def test_decode_tiny_fp32_dims(orc):
    shape = DecodeShape(2, 2, 16, 16, 8, 5, 5, 12, "f32")
    init = _small_init(shape, [1, 3], [5, 0], seed=2)
    _run_decode(orc, shape, init, shape.nsteps, [0, 1])


def test_decode_config_sampled(orc):
    """64 sequences with 128 cached memories each (context 32768 at S=256),
    256 steps with the append on the last one; the oracle follows eight
    sequences spread over the batch (every ninth) and y is compared on every
    step."""
    shape = synth.DECODE_64x32K
    init = synth.decode_initial(shape, seed=0)
    dev, ref, _ = _run_decode(orc, shape, init, shape.nsteps, [0, 9, 18, 27, 36, 45, 54, 63])
    assert np.all(ref["nchunks"] == 129) and np.all(ref["pos"] == 0)
    assert int(dev["nchunks"].min()) == 129


def test_prefill_then_decode_matches_longer_prefill():
    """forward(L + S) on the GPU equals forward(L) followed by S decode steps
    fed from its dH and final boundary state, including the append."""
    S = 256
    shape = LayerShape(2, 4 * S, 3, 64, 128, S, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=20)
    d = to_device(inp)
    L = 3 * S
    full = dart.layer_forward(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], d["Q"], d["E"], S, d["g"])
    pre = dart.layer_forward(*(d[k][:, :L] if k != "A" else d[k] for k in ("x", "dt", "A", "Bm", "Cm", "Q", "E")),
                             S, d["g"])
    B, H, N, P = 2, 3, 128, 64
    cmax = 5
    cache = torch.zeros(B, H, cmax, N, P, dtype=torch.bfloat16, device="cuda")
    cache[:, :, :3] = pre["dH"]
    state = pre["states"][:, :, -1].contiguous()
    dcur = torch.zeros_like(state)
    nch = torch.full((B,), 3, dtype=torch.int32, device="cuda")
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    ys = []
    for t in range(L, L + S):
        ys.append(dart.dart_decode_step(d["x"][:, t], d["dt"][:, t], d["A"], d["Bm"][:, t], d["Cm"][:, t],
                                        d["Q"][:, t], d["E"][:, t], d["g"], state, dcur, cache, nch, pos, S))
    dart.dart_sync_status()
    y_dec = torch.stack(ys, 1)
    assert_close("decode vs prefill y", y_dec, full["y"][:, L:].cpu().numpy(), 2e-2)
    assert torch.all(nch == 4) and torch.all(pos == 0)
    assert_close("appended memory", cache[:, :, 3].float(), full["dH"][:, :, 3].float().cpu().numpy(), 2e-2)
    assert_close("state", state, full["states"][:, :, -1].cpu().numpy(), 2e-2)


def test_ragged_prefill_then_decode_matches_longer_prefill():
    """A prefill that ends inside a chunk (L = 2 S + 100) hands its partial
    chunk to decode (dH_cur = dH[C-1], state = states[C-1], C-1 memories,
    position L mod S); decoding to 4 S reproduces the longer prefill."""
    S = 256
    shape = LayerShape(2, 4 * S, 3, 64, 128, S, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=23)
    d = to_device(inp)
    L = 2 * S + 100
    full = dart.layer_forward(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], d["Q"], d["E"], S, d["g"])
    pre = dart.layer_forward(*(d[k][:, :L] if k != "A" else d[k] for k in ("x", "dt", "A", "Bm", "Cm", "Q", "E")),
                             S, d["g"])
    assert pre["dH"].shape[2] == 3
    B, H, N, P = 2, 3, 128, 64
    cmax = 5
    cache = torch.zeros(B, H, cmax, N, P, dtype=torch.bfloat16, device="cuda")
    cache[:, :, :2] = pre["dH"][:, :, :2]
    state = pre["states"][:, :, -1].contiguous()
    dcur = pre["dH"][:, :, -1].float().contiguous()
    nch = torch.full((B,), 2, dtype=torch.int32, device="cuda")
    pos = torch.full((B,), L % S, dtype=torch.int32, device="cuda")
    ys = []
    for t in range(L, 4 * S):
        ys.append(dart.dart_decode_step(d["x"][:, t], d["dt"][:, t], d["A"], d["Bm"][:, t], d["Cm"][:, t],
                                        d["Q"][:, t], d["E"][:, t], d["g"], state, dcur, cache, nch, pos, S))
    dart.dart_sync_status()
    y_dec = torch.stack(ys, 1)
    assert_close("decode vs prefill y", y_dec, full["y"][:, L:].cpu().numpy(), 2e-2)
    assert torch.all(nch == 4) and torch.all(pos == 0)
    assert_close("memories", cache[:, :, :4].float(), full["dH"].float().cpu().numpy(), 2e-2)
    assert_close("state", state, full["states"][:, :, -1].cpu().numpy(), 2e-2)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decayed_decode_small_with_appends(orc, dtype):
    """Decayed memories (dart_decode_step_decayed): three sequences, appends
    at different steps, one starting from an empty cache."""
    shape = DecodeShape(3, 2, 64, 128, 4, 7, 7, 9, dtype)
    init = _small_init(shape, [2, 0, 3], [0, 2, 3], seed=1)
    _run_decode(orc, shape, init, shape.nsteps, [0, 1, 2], memlog=_memlog(shape, [2, 0, 3], 1))


def test_decayed_decode_tiny_fp32_dims(orc):
    shape = DecodeShape(2, 2, 16, 16, 8, 5, 5, 12, "f32")
    init = _small_init(shape, [1, 3], [5, 0], seed=2)
    _run_decode(orc, shape, init, shape.nsteps, [0, 1], memlog=_memlog(shape, [1, 3], 2))


def test_decayed_decode_config_sampled(orc):
    """The 64-sequence, 128-memory decode batch with decayed memories, 256
    steps (append on the last); the oracle follows sequences 0 and 63."""
    shape = synth.DECODE_64x32K
    init = synth.decode_initial(shape, seed=0)
    ml = _memlog(shape, init["nchunks"].tolist(), 3)
    dev, ref, _ = _run_decode(orc, shape, init, shape.nsteps, [0, 63], check_every=15, memlog=ml)
    assert np.all(ref["nchunks"] == 129)
    assert torch.all(dev["memlog"][:, :, 128] == 0.0)   # appended by the last step, nothing added yet


@pytest.mark.parametrize("L_extra", [100, 0])
def test_decayed_prefill_then_decode_matches_longer_prefill(L_extra):
    """Prefill of L = 2 S + L_extra tokens with decayed memories, memory
    log-decays from dart_decode_memlog_init (checked against fp64 suffix sums
    of dt A), then decayed decode to 4 S: the outputs match the decayed
    prefill of the longer sequence."""
    S = 256
    shape = LayerShape(2, 4 * S, 3, 64, 128, S, "bf16", "loguniform")
    inp = synth.layer_inputs(shape, seed=24)
    inp["A"] = torch.full_like(inp["A"], -0.3)   # several memories stay visible
    d = to_device(inp)
    L = 2 * S + L_extra
    keys = ("x", "dt", "A", "Bm", "Cm", "Q", "E")
    full = dart.layer_forward(*(d[k] for k in keys), S, d["g"], decayed=True)
    pre = dart.layer_forward(*(d[k][:, :L] if k != "A" else d[k] for k in keys), S, d["g"], decayed=True)
    B, H, N, P = 2, 3, 128, 64
    cmax = 5
    nc = L // S
    memlog = torch.full((B, H, cmax), 50.0, device="cuda")
    dart.decode_memlog_init(d["dt"][:, :L], d["A"], S, memlog)
    a = inp["dt"][:, :L].double() * inp["A"].double()[None, None, :]
    for c in range(nc):
        want = a[:, (c + 1) * S:L].sum(1)                        # [B, H]
        assert torch.allclose(memlog[:, :, c].double().cpu(), want, rtol=1e-5, atol=1e-5), c
    assert torch.all(memlog[:, :, nc:] == 50.0)
    cache = torch.zeros(B, H, cmax, N, P, dtype=torch.bfloat16, device="cuda")
    cache[:, :, :nc] = pre["dH"][:, :, :nc]
    state = pre["states"][:, :, -1].contiguous()
    if L % S:
        dcur = pre["dH"][:, :, -1].float().contiguous()
    else:
        dcur = torch.zeros(B, H, N, P, device="cuda")
    nch = torch.full((B,), nc, dtype=torch.int32, device="cuda")
    pos = torch.full((B,), L % S, dtype=torch.int32, device="cuda")
    ys = []
    for t in range(L, 4 * S):
        ys.append(dart.dart_decode_step(d["x"][:, t], d["dt"][:, t], d["A"], d["Bm"][:, t], d["Cm"][:, t],
                                        d["Q"][:, t], d["E"][:, t], d["g"], state, dcur, cache, nch, pos, S,
                                        memlog=memlog))
    dart.dart_sync_status()
    y_dec = torch.stack(ys, 1)
    assert_close("decayed decode vs decayed prefill y", y_dec, full["y"][:, L:].cpu().numpy(), 2e-2)
    assert torch.all(nch == 4) and torch.all(pos == 0)


def test_decode_bad_counters_are_flagged():
    """A sequence with pos outside [0, S) or a full cache is skipped and the
    device status reports DART_ERR_DEVICE; the other sequences advance."""
    shape = DecodeShape(3, 2, 64, 128, 4, 2, 3, 1, "bf16")
    init = synth.decode_initial(shape, seed=3)
    init["pos"] = torch.tensor([0, 7, 3], dtype=torch.int32)      # seq 1: pos out of range
    init["nchunks"] = torch.tensor([2, 2, 3], dtype=torch.int32)  # seq 2: append into a full cache
    dev = {k: v.cuda() for k, v in init.items()}
    st0 = dev["state"].clone()
    tok = synth.decode_tokens(shape, 0, 3)
    A = synth.decode_A(shape, 3)
    dart.dart_decode_step(tok["x"].cuda(), tok["dt"].cuda(), A.cuda(), tok["Bm"].cuda(), tok["Cm"].cuda(),
                          tok["Q"].cuda(), tok["E"].cuda(), 0.5, dev["state"], dev["dH_cur"], dev["cache"],
                          dev["nchunks"], dev["pos"], shape.chunk)
    with pytest.raises(dart.DartError) as ei:
        dart.dart_sync_status()
    assert ei.value.status == dart.DART_ERR_DEVICE
    assert torch.equal(dev["state"][1:], st0[1:])
    assert not torch.equal(dev["state"][0], st0[0])
    assert dev["pos"].tolist() == [1, 7, 3] and dev["nchunks"].tolist() == [2, 2, 3]
    dart.dart_sync_status()  # the status word was cleared by the read
