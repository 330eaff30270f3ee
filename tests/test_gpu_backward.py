"""GPU parity of the SMA backward (dart_sma_backward) against the fp64
backward oracle (``oracle/dart_backward.py``, autograd over the pinned
forward restatement), on the same seeded inputs.  Both sides read the same
float32-exact inputs, so the only differences are fp32 accumulation:
max|err| / max|ref| <= 1e-4 for float32 inputs and <= 1e-3 for bf16 inputs
(each value exactly representable; the kernels accumulate in fp32 over up to
N * P terms per output, twice as deep as the forward)."""
import numpy as np
import pytest
import torch

from mamba_ssd_state_b200 import build, dart, synth
from oracle import dart_backward
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
    ((1, 3 * 256, 2, 64, 128, 256), torch.bfloat16, 1e-3),
    ((1, 2 * 256 + 77, 3, 64, 128, 256), torch.bfloat16, 1e-3),
], ids=["f32_N16_ragged", "f32_N64_B2_ragged", "bf16_N128", "bf16_N128_ragged"])
def test_sma_backward_matches_oracle(shape, dtype, tol):
    Bz, L, H, P, N, S = shape
    g = 0.7
    inp, dy = _case(Bz, L, H, P, N, S, dtype, seed=L)
    got = dart.dart_sma_backward(*(inp[k].cuda() for k in ("Q", "E", "Cm", "dH")), S, g, dy.cuda())
    dart.dart_sync_status()
    ref = dart_backward.sma_grads(*(inp[k].double().numpy() for k in ("Q", "E", "Cm", "dH")), S, g,
                                  dy.double().numpy())
    for k in ("dQ", "dE", "dCm", "ddH"):
        assert_close(k, got[k], ref[k], tol)
    assert abs(float(got["dg"][0]) - float(ref["dg"])) <= tol * max(1.0, abs(float(ref["dg"])))


def test_sma_backward_deterministic():
    inp, dy = _case(1, 3 * 256, 2, 64, 128, 256, torch.bfloat16, seed=3)
    args = [inp[k].cuda() for k in ("Q", "E", "Cm", "dH")]
    a = dart.dart_sma_backward(*args, 256, 0.5, dy.cuda())
    b = dart.dart_sma_backward(*args, 256, 0.5, dy.cuda())
    for k in a:
        assert torch.equal(a[k], b[k]), k
