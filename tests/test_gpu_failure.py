"""Failure detection on the GPU without a fault: the drill kernel makes one
bounded wait run out (an mbarrier nothing arrives on), the status word
reports DART_ERR_TIMEOUT with the drill's kernel id and wait site, the word
is cleared by that read, and the tensor-core kernels that run next produce
the same bits as before the drill."""
import pytest
import torch

from mamba_ssd_state_b200 import build, dart, synth
from mamba_ssd_state_b200.synth import LayerShape
from tests.parity import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    return dart.load()


def _layer(d, chunk):
    y_ssd, dH, st = dart.dart_ssd_chunk_scan(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], chunk)
    y = dart.dart_sma_forward(d["Q"], d["E"], d["Cm"], dH, chunk, d["g"], y_ssd.clone())
    return y_ssd, dH, st, y


def test_bounded_wait_times_out_and_the_next_call_runs_clean():
    shape = LayerShape(1, 3 * 128 + 40, 2, 64, 128, 128, "bf16", "loguniform")
    d = to_device(synth.layer_inputs(shape, seed=5))
    before = _layer(d, shape.chunk)
    dart.dart_sync_status()
    dart.dart_selftest_wait_timeout(2000)          # gives up after 2 ms
    with pytest.raises(dart.DartError) as err:
        dart.dart_sync_status()
    assert err.value.status == dart.DART_ERR_TIMEOUT
    assert "kernel 9, wait site 1" in str(err.value)
    dart.dart_sync_status()                         # the read cleared the word
    after = _layer(d, shape.chunk)
    dart.dart_sync_status()
    for a, b in zip(before, after):
        assert torch.equal(a, b)
