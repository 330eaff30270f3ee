"""The benchmark's algorithmic work counts (CPU): the FLOP and byte figures
that `roofline.achieved` divides by the measured kernel time.

* SMA: 4 N P flop per valid (token, earlier memory) pair per head; the pair
  count is checked against an explicit loop, ragged lengths included.
* Decode: the bytes a step must move grow by exactly one memory per (seq,
  head) per cached chunk, the append adds one memory, and an E4M3 memory is
  (P + 1) / (2 P) of a bf16 one.
* The workload figures quoted in the design notes (266.29 and 26.07 GFLOP,
  4.565 GB per decode step on average) are what the functions return.
* Both arms (kernels and oracle) name the headline workload with one config.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mamba_ssd_state_b200 import synth  # noqa: E402


@pytest.mark.parametrize("L,S", [(8192, 256), (8092, 256), (1000, 128), (64, 64), (65, 64)])
def test_sma_pairs_match_explicit_count(L, S):
    shape = synth.LayerShape(2, L, 3, 64, 128, S, "bf16", "loguniform")
    pairs = sum(t // S for t in range(L))          # memories c < k(t) for each token
    assert bench.sma_flops(shape) == 4.0 * 128 * 64 * pairs * 2 * 3


def test_quoted_forward_work():
    assert bench.sma_flops(synth.TRAIN_L8K) == pytest.approx(266.287972352e9, rel=1e-12)
    assert bench.ssd_flops(synth.TRAIN_L8K) == pytest.approx(26.073890816e9, rel=1e-12)


def test_decode_bytes_structure():
    d = synth.DECODE_64x32K
    mem_bf16 = d.dstate * d.headdim * 2
    mem_e4 = d.dstate * (d.headdim + 1)
    for e4m3, mem in ((False, mem_bf16), (True, mem_e4)):
        base = bench.decode_bytes(d, 128, False, e4m3)
        assert bench.decode_bytes(d, 129, False, e4m3) - base == d.nseq * d.nheads * mem
        assert bench.decode_bytes(d, 128, True, e4m3) - base == d.nseq * d.nheads * mem
    assert mem_e4 / mem_bf16 == (d.headdim + 1) / (2 * d.headdim)
    # the average over the 256 timed steps (the last one appends), as quoted
    steps = [bench.decode_bytes(d, d.ncached + s // d.chunk, s % d.chunk == d.chunk - 1) for s in range(256)]
    assert sum(steps) / 256 == pytest.approx(4.565147648e9, rel=1e-12)


def test_both_arms_share_the_headline_config():
    """The reference arm and the kernel arm report the same `config` object,
    so a driver comparing them sees the same workload."""
    import inspect
    cfg = bench.fwd_config(4)
    assert cfg["workload"] == "dart_layer_fwd_L8k" and cfg["parallelism"] == "dp4" and cfg["ngroups"] == 1
    assert (cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"], cfg["chunk"]) == \
        (2, 8192, 32, 64, 128, 256)
    assert "fwd_config(args.gpus)" in inspect.getsource(bench.run_reference)
    assert "fwd_config(dist.world)" in inspect.getsource(bench.main)
