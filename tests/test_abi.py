"""The C-ABI library builds, loads and exports every symbol include/dart.h
declares; host-side validation rejects bad arguments before touching the GPU.
CPU only: no call here reaches a kernel launch."""
import ctypes
import os
import re

import pytest
import torch

from mamba_ssd_state_b200 import build, dart

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dart.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return dart.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dart_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("dart_ssd_chunk_scan", "dart_sma_forward", "dart_decode_step", "dart_sync_status"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), f"{name} declared in dart.h but not exported"
    assert set(dart.EXPORTS) <= set(_declared())


def test_abi_version(lib):
    assert lib.dart_abi_version() == 4


def test_wait_drill_rejects_limits_out_of_range(lib):
    """Host-side validation only: no launch happens for these."""
    assert lib.dart_selftest_wait_timeout(0, None) == dart.DART_ERR_INVALID_ARG
    assert lib.dart_selftest_wait_timeout(2000001, None) == dart.DART_ERR_INVALID_ARG


def test_supported_set(lib):
    assert dart.supported(128, 64, 256, torch.bfloat16)
    assert dart.supported(16, 16, 64, torch.float32)
    assert not dart.supported(96, 64, 256, torch.bfloat16)
    assert not dart.supported(128, 64, 100, torch.bfloat16)


FAKE = ctypes.c_void_p(0x10000)       # 16-byte aligned, never dereferenced on the host
MISALIGNED = ctypes.c_void_p(0x10004)


def _scan(lib, dims, dtype=dart.DART_BF16, x=FAKE, ws_bytes=1 << 20):
    return lib.dart_ssd_chunk_scan(ctypes.byref(dims), dtype, x, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE,
                                   FAKE, FAKE, ws_bytes, None)


def test_ragged_seqlen_counts_the_partial_chunk(lib):
    """L = 300, S = 256: two chunks, the second one partial.  The workspace
    is sized for ceil(L / S) chunks and a smaller one is rejected before any
    launch."""
    d = dart.Dims(1, 300, 2, 64, 128, 256, 1)
    need = lib.dart_ssd_chunk_scan_workspace_bytes(ctypes.byref(d), dart.DART_BF16)
    bhc = 1 * 2 * 2
    assert need == 256 + bhc * 128 * 64 * 2 + 3 * bhc * 256 * 4
    assert _scan(lib, d, ws_bytes=need - 16) == dart.DART_ERR_INVALID_ARG


def test_scan_rejects_ngroups_not_dividing_heads(lib):
    """B and C come in ngroups groups, head h reading group h / (nheads /
    ngroups); a count that does not divide nheads, or is below 1, is rejected
    before any launch."""
    assert _scan(lib, dart.Dims(1, 256, 4, 64, 128, 256, 3)) == dart.DART_ERR_INVALID_ARG
    assert _scan(lib, dart.Dims(1, 256, 4, 64, 128, 256, 0)) == dart.DART_ERR_INVALID_ARG
    assert _scan(lib, dart.Dims(1, 256, 4, 64, 128, 256, 8)) == dart.DART_ERR_INVALID_ARG


def test_scan_rejects_uncompiled_shape(lib):
    assert _scan(lib, dart.Dims(1, 256, 2, 64, 96, 256, 1)) == dart.DART_ERR_UNSUPPORTED


def test_scan_rejects_null_and_misaligned(lib):
    d = dart.Dims(1, 256, 2, 64, 128, 256, 1)
    assert _scan(lib, d, x=None) == dart.DART_ERR_INVALID_ARG
    assert b"null" in lib.dart_last_error()
    assert _scan(lib, d, x=MISALIGNED) == dart.DART_ERR_INVALID_ARG
    assert b"aligned" in lib.dart_last_error()


def test_scan_rejects_small_workspace(lib):
    d = dart.Dims(2, 512, 4, 64, 128, 256, 1)
    need = lib.dart_ssd_chunk_scan_workspace_bytes(ctypes.byref(d), dart.DART_BF16)
    bhc = 2 * 4 * 2
    # per-chunk decay sums padded to 256 bytes + the bf16 state entering each
    # chunk + three fp32 per-token decay terms
    assert need == 256 + bhc * 128 * 64 * 2 + 3 * bhc * 256 * 4
    assert lib.dart_ssd_chunk_scan_workspace_bytes(ctypes.byref(d), dart.DART_F32) == 256
    assert _scan(lib, d, ws_bytes=need - 1) == dart.DART_ERR_INVALID_ARG


def test_scan_rejects_bad_dtype_and_dims(lib):
    assert _scan(lib, dart.Dims(1, 256, 2, 64, 128, 256, 1), dtype=7) == dart.DART_ERR_INVALID_ARG
    assert _scan(lib, dart.Dims(0, 256, 2, 64, 128, 256, 1)) == dart.DART_ERR_INVALID_ARG
    assert lib.dart_ssd_chunk_scan(None, 1, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE,
                                   16, None) == dart.DART_ERR_INVALID_ARG


def test_sma_rejects_bad_args(lib):
    d = dart.Dims(1, 512, 2, 64, 128, 256, 1)
    rc = lib.dart_sma_forward(ctypes.byref(d), dart.DART_BF16, FAKE, None, FAKE, FAKE, 0.5, None, FAKE, None)
    assert rc == dart.DART_ERR_INVALID_ARG
    d.chunk = 96   # not a compiled chunk length (a seqlen that is not a multiple of chunk is accepted)
    rc = lib.dart_sma_forward(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, 0.5, None, FAKE, None)
    assert rc == dart.DART_ERR_UNSUPPORTED


def test_sma_rejects_partially_overlapping_out(lib):
    """out must be y_ssd itself or disjoint from it."""
    d = dart.Dims(1, 512, 2, 64, 128, 256, 1)
    base = 1 << 32
    y = ctypes.c_void_p(base)
    rc = lib.dart_sma_forward(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, 0.5, y,
                              ctypes.c_void_p(base + 4096), None)
    assert rc == dart.DART_ERR_INVALID_ARG
    assert b"overlaps" in lib.dart_last_error()


def test_sma_decayed_workspace_and_validation(lib):
    """Workspace = B*H*C*S floats (padded to 256 bytes) + B*H*C doubles, C =
    ceil(L/S); missing dt/A, a small or misaligned workspace and uncompiled
    shapes are rejected on the host."""
    d = dart.Dims(2, 500, 3, 64, 128, 256, 1)
    C = 2
    la2 = (2 * 3 * C * 256 * 4 + 255) // 256 * 256
    assert lib.dart_sma_decayed_workspace_bytes(ctypes.byref(d)) == la2 + 2 * 3 * C * 8
    assert lib.dart_sma_decayed_workspace_bytes(None) == 0
    ws = lib.dart_sma_decayed_workspace_bytes(ctypes.byref(d))
    f = lib.dart_sma_forward_decayed
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, None, FAKE, 0.5, None, FAKE,
             FAKE, ws, None) == dart.DART_ERR_INVALID_ARG
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.5, None, FAKE,
             FAKE, ws, None) == dart.DART_ERR_INVALID_ARG
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.5, None, FAKE,
             FAKE, ws - 1, None) == dart.DART_ERR_INVALID_ARG
    assert b"workspace" in lib.dart_last_error()
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.5, None, FAKE,
             ctypes.c_void_p((1 << 32) + 8), ws, None) == dart.DART_ERR_INVALID_ARG
    base = 1 << 32
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.5,
             ctypes.c_void_p(base), ctypes.c_void_p(base + 4096), FAKE, ws, None) == dart.DART_ERR_INVALID_ARG
    d.chunk = 96
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.5, None, FAKE,
             FAKE, 1 << 30, None) == dart.DART_ERR_UNSUPPORTED


def test_decayed_decode_validation(lib):
    """The decayed decode step needs mem_logdecay on top of dart_decode_step's
    arguments; the memlog initialiser rejects prefills that overflow cmax."""
    d = dart.Dims(4, 0, 2, 64, 128, 256, 1)
    ws = lib.dart_decode_step_workspace_bytes(ctypes.byref(d), dart.DART_BF16, 9)
    args = [FAKE] * 7 + [0.5] + [FAKE] * 3 + [9] + [FAKE, FAKE, None, FAKE, FAKE, ws, None]
    assert lib.dart_decode_step_decayed(ctypes.byref(d), dart.DART_BF16, *args) == dart.DART_ERR_INVALID_ARG
    assert b"mem_logdecay" in lib.dart_last_error()
    p = dart.Dims(2, 10 * 256 + 7, 2, 64, 128, 256, 1)
    assert lib.dart_decode_memlog_init(ctypes.byref(p), FAKE, FAKE, FAKE, 9, None) == dart.DART_ERR_INVALID_ARG
    assert lib.dart_decode_memlog_init(ctypes.byref(p), FAKE, None, FAKE, 16, None) == dart.DART_ERR_INVALID_ARG
    assert lib.dart_decode_memlog_init(None, FAKE, FAKE, FAKE, 16, None) == dart.DART_ERR_INVALID_ARG


def test_e4m3_decode_validation(lib):
    """The fp8-cache decode needs the code cache and the row exponents; only
    P = 64 (N = 64 or 128) is compiled; the handoff quantizer checks nmem."""
    d = dart.Dims(4, 0, 2, 64, 128, 256, 1)
    ws = lib.dart_decode_step_workspace_bytes(ctypes.byref(d), dart.DART_BF16, 9)
    f = lib.dart_decode_step_e4m3
    args = [FAKE] * 7 + [0.5] + [FAKE, FAKE, FAKE, None] + [9] + [FAKE, FAKE, None, FAKE, FAKE, ws, None]
    assert f(ctypes.byref(d), dart.DART_BF16, *args) == dart.DART_ERR_INVALID_ARG
    assert b"cache_exp" in lib.dart_last_error()
    d16 = dart.Dims(4, 0, 2, 16, 16, 64, 1)
    args[3 + 8] = FAKE
    assert f(ctypes.byref(d16), dart.DART_F32, *args) == dart.DART_ERR_UNSUPPORTED
    p = dart.Dims(2, 5 * 256, 2, 64, 128, 256, 1)
    q = lib.dart_cache_quantize_e4m3
    assert q(ctypes.byref(p), dart.DART_BF16, FAKE, 6, FAKE, FAKE, 9, None) == dart.DART_ERR_INVALID_ARG
    assert q(ctypes.byref(p), dart.DART_BF16, FAKE, 5, FAKE, FAKE, 4, None) == dart.DART_ERR_INVALID_ARG
    assert q(ctypes.byref(p), dart.DART_BF16, FAKE, 2, FAKE, None, 4, None) == dart.DART_ERR_INVALID_ARG


def test_sma_backward_workspace_and_validation(lib):
    d = dart.Dims(2, 500, 3, 64, 128, 256, 1)
    C, tiles = 2, 16
    pad = lambda b: (b + 255) // 256 * 256
    want = 2 * pad(4 * 2 * 3 * 500 * C) + pad(4 * 2 * 500 * 3 * 128) + pad(4 * 2 * 3 * tiles)
    assert lib.dart_sma_backward_workspace_bytes(ctypes.byref(d)) == want
    ws = want
    f = lib.dart_sma_backward
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, 0.5, None, FAKE, FAKE, FAKE, FAKE, FAKE,
             FAKE, ws, None) == dart.DART_ERR_INVALID_ARG
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, 0.5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
             FAKE, ws - 1, None) == dart.DART_ERR_INVALID_ARG
    d.chunk = 96
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, 0.5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
             FAKE, 1 << 30, None) == dart.DART_ERR_UNSUPPORTED


def test_scan_backward_workspace_and_validation(lib):
    d = dart.Dims(2, 500, 3, 64, 128, 256, 1)
    pad = lambda b: (b + 255) // 256 * 256
    C = 2   # ceil(500 / 256)
    # chunk adjoints, chunk decay sums, five per-token scalars, one scalar per chunk,
    # per-head dB and dC, per-chunk dA
    want = (pad(4 * 2 * 3 * C * 128 * 64) + pad(4 * 2 * 3 * C) + pad(4 * 6 * 2 * 3 * C * 256) + pad(4 * 2 * 3 * C)
            + 2 * pad(4 * 2 * 500 * 3 * 128) + pad(4 * 2 * 3 * C))
    assert lib.dart_ssd_scan_backward_workspace_bytes(ctypes.byref(d)) == want
    f = lib.dart_ssd_scan_backward
    ok = [FAKE] * 5 + [None, FAKE, FAKE, None, None] + [FAKE] * 5 + [None, FAKE]
    assert f(ctypes.byref(d), dart.DART_BF16, *ok[:6], None, *ok[7:], want, None) == dart.DART_ERR_INVALID_ARG
    assert b"states" in lib.dart_last_error()
    assert f(ctypes.byref(d), dart.DART_BF16, *ok, want - 1, None) == dart.DART_ERR_INVALID_ARG
    d.chunk = 512
    assert f(ctypes.byref(d), dart.DART_BF16, *ok, 1 << 40, None) == dart.DART_ERR_UNSUPPORTED
    d.chunk = 256
    d.headdim, d.dstate = 32, 32
    assert f(ctypes.byref(d), dart.DART_BF16, *ok, 1 << 40, None) == dart.DART_ERR_UNSUPPORTED


def test_decode_rejects_bad_args(lib):
    d = dart.Dims(4, 0, 2, 64, 128, 256, 1)
    ws = lib.dart_decode_step_workspace_bytes(ctypes.byref(d), dart.DART_BF16, 9)
    assert ws > 0

    def call(cmax=9, state=FAKE, ws_bytes=ws):
        return lib.dart_decode_step(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                    0.5, state, FAKE, FAKE, cmax, FAKE, FAKE, FAKE, FAKE, ws_bytes, None)

    assert call(cmax=0) == dart.DART_ERR_INVALID_ARG
    assert call(state=None) == dart.DART_ERR_INVALID_ARG
    assert call(ws_bytes=ws - 4) == dart.DART_ERR_INVALID_ARG


def test_decode_cmax_bound(lib):
    """Every decode entry takes 1 <= cmax <= 2^20; a cmax near INT_MAX (whose
    split count would overflow 32-bit arithmetic) is rejected on the host,
    and the workspace query answers 0 for it instead of a one-split size."""
    d = dart.Dims(4, 0, 2, 64, 128, 256, 1)
    big = (1 << 31) - 10
    assert lib.dart_decode_step_workspace_bytes(ctypes.byref(d), dart.DART_BF16, big) == 0
    assert lib.dart_decode_step_workspace_bytes(ctypes.byref(d), dart.DART_BF16, (1 << 20) + 1) == 0
    assert lib.dart_decode_step_workspace_bytes(ctypes.byref(d), dart.DART_BF16, 1 << 20) > 0
    tok = [FAKE] * 7 + [0.5]          # x, dt, A, B, C, Q, E and g
    mem = [FAKE] * 3                  # state, dH_cur, cache
    for cmax in ((1 << 20) + 1, big):
        assert lib.dart_decode_step(ctypes.byref(d), dart.DART_BF16, *tok, *mem, cmax, *[FAKE] * 4, 1 << 40,
                                    None) == dart.DART_ERR_INVALID_ARG
        assert b"cmax" in lib.dart_last_error()
        assert lib.dart_decode_step_decayed(ctypes.byref(d), dart.DART_BF16, *tok, *mem, cmax, *[FAKE] * 5,
                                            1 << 40, None) == dart.DART_ERR_INVALID_ARG
        assert lib.dart_decode_step_e4m3(ctypes.byref(d), dart.DART_BF16, *tok, *mem, FAKE, cmax, FAKE, FAKE,
                                         None, FAKE, FAKE, 1 << 40, None) == dart.DART_ERR_INVALID_ARG
        assert lib.dart_decode_step_noalloc(ctypes.byref(d), dart.DART_BF16, *tok, *mem, cmax, FAKE, FAKE, FAKE,
                                            None) == dart.DART_ERR_INVALID_ARG
        assert b"cmax" in lib.dart_last_error()


def test_binding_fails_loudly_without_cuda(lib):
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    x = torch.zeros(1, 256, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        dart.dart_ssd_chunk_scan(x, torch.zeros(1, 256, 1), torch.zeros(1),
                                 torch.zeros(1, 256, 128, dtype=torch.bfloat16),
                                 torch.zeros(1, 256, 128, dtype=torch.bfloat16), 256)


def test_backward_rejects_groups_that_do_not_divide_heads(lib):
    """ngroups must divide nheads in the backward calls too (B, C and their
    gradients are [B, L, G, N], head h reading group h / (H / G))."""
    d = dart.Dims(2, 500, 3, 64, 128, 256, 2)
    f = lib.dart_sma_backward
    assert f(ctypes.byref(d), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, 0.5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
             FAKE, 1 << 40, None) == dart.DART_ERR_INVALID_ARG
    assert b"ngroups" in lib.dart_last_error()
    ok = [FAKE] * 5 + [None, FAKE, FAKE, None, None] + [FAKE] * 5 + [None, FAKE]
    assert lib.dart_ssd_scan_backward(ctypes.byref(d), dart.DART_BF16, *ok, 1 << 40, None) == \
        dart.DART_ERR_INVALID_ARG
    assert b"ngroups" in lib.dart_last_error()
