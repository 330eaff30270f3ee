"""dart_decode_step_noalloc: the decode step for callers that cannot allocate
device memory (for example a host runtime that hands out only preallocated
tensors, or a serving loop that must not call the allocator between steps).
It keeps its scratch in a fixed static device array instead of a caller
workspace.  The GPU test checks it against dart_decode_step, through the C
ABI, on two calls in a row; the limit test needs no GPU.

This file is named to be collected last, so that a run stopping at the
first failure has already run every other test."""
import ctypes

import pytest
import torch

from mamba_ssd_state_b200 import build, dart, synth
from tests.parity import TOL, assert_close

FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced on the host


def test_noalloc_rejects_batches_beyond_the_fixed_scratch():
    build.build()
    lib = dart.load()
    # 64 sequences x 32 heads x 129 chunks of memory fit; 4096 sequences do not
    ok = dart.Dims(64, 0, 32, 64, 128, 256, 1)
    assert lib.dart_decode_step_workspace_bytes(ctypes.byref(ok), dart.DART_BF16, 129) <= 16 << 20
    big = dart.Dims(4096, 0, 32, 64, 128, 256, 1)
    assert lib.dart_decode_step_workspace_bytes(ctypes.byref(big), dart.DART_BF16, 129) > 16 << 20
    rc = lib.dart_decode_step_noalloc(ctypes.byref(big), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                      0.5, FAKE, FAKE, FAKE, 129, FAKE, FAKE, FAKE, None)
    assert rc == dart.DART_ERR_UNSUPPORTED
    assert b"16777216" in lib.dart_last_error()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    dart.load()
    # chunk size 2: the second call closes a chunk and appends a memory
    shape = synth.DecodeShape(6, 4, 64, 128, 2, 5, 7, 2, "bf16")
    init = synth.decode_initial(shape, seed=7)
    init["pos"] = torch.tensor([0, 1, 0, 1, 0, 1], dtype=torch.int32)
    A = synth.decode_A(shape, seed=7).cuda()
    ref = {k: v.clone().cuda() for k, v in init.items()}
    got = {k: v.clone().cuda() for k, v in init.items()}
    y_got = torch.empty((shape.nseq, shape.nheads, shape.headdim), device="cuda", dtype=torch.float32)
    tol = TOL[torch.bfloat16]
    for step in range(2):
        t = {k: v.cuda() for k, v in synth.decode_tokens(shape, step, seed=7).items()}
        args = (t["x"], t["dt"], A, t["Bm"], t["Cm"], t["Q"], t["E"], shape.g)
        y_ref = dart.dart_decode_step(*args, ref["state"], ref["dH_cur"], ref["cache"], ref["nchunks"], ref["pos"],
                                      shape.chunk)
        dart.dart_decode_step_noalloc(*args, got["state"], got["dH_cur"], got["cache"], got["nchunks"], got["pos"],
                                      shape.chunk, y=y_got)
        dart.dart_sync_status()
        assert_close(f"y, call {step + 1}", y_got, y_ref.cpu().numpy(), tol)
        assert_close(f"state, call {step + 1}", got["state"], ref["state"].cpu().numpy(), tol)
        assert_close(f"dH_cur, call {step + 1}", got["dH_cur"], ref["dH_cur"].cpu().numpy(), tol)
        assert torch.equal(got["nchunks"], ref["nchunks"]) and torch.equal(got["pos"], ref["pos"])
    assert_close("cache", got["cache"].float(), ref["cache"].float().cpu().numpy(), tol)
    assert got["nchunks"].tolist() == [6, 6, 6, 6, 6, 6]
