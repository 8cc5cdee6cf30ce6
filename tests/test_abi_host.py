"""Host-side tests of the C ABI: the library loads without a GPU, exports every
symbol include/twell.h declares, and rejects bad arguments before any launch.

Bad-argument calls pass fake (never dereferenced) device addresses: the
library validates every argument on the host and returns before touching the
device, so these tests run on a machine without a GPU.
"""
import ctypes
import os
import re

import pytest

from activation_sparse_transformer_tma_b200 import build as tw_build
from activation_sparse_transformer_tma_b200 import twell

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "twell.h")

OK, INVALID, UNSUPPORTED, ALIGN, CUDA = 0, 1, 2, 3, 4
FAKE = 0x10000  # 16-byte aligned, never dereferenced on the host


@pytest.fixture(scope="module")
def L():
    tw_build.build()
    return twell.lib()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"TW_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ("twell_gate_gemm", "twell_fused_updown", "twell_to_hybrid", "hybrid_ffn_backward"):
        assert n in names
    assert sorted(names) == sorted(twell.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for n in declared_symbols():
        assert hasattr(L, n), n
        assert ctypes.cast(getattr(L, n), ctypes.c_void_p).value


def test_nm_shows_only_the_abi_as_dynamic_text_symbols(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", twell.LIB_PATH], capture_output=True,
                         text=True).stdout
    text_syms = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(declared_symbols()) <= text_syms


def test_status_strings_and_version(L):
    for code, name in enumerate(twell.STATUS):
        assert L.tw_status_string(code).decode() == name
    assert L.twell_version() >= 100


def _tw(T=256, F=1024, W=128, C=8, dtype=twell.TW_BF16, spill_cap=64, base=FAKE):
    return twell.TwTwellC(T, F, W, C, dtype, base, base, base, base, spill_cap, base, base, base)


def _gate(L, tw, x=FAKE, w=FAKE, T=256, d=512, F=1024, dtype=twell.TW_BF16):
    return L.twell_gate_gemm(x, w, T, d, F, dtype, ctypes.byref(tw), None, None, None)


def test_gate_validation(L):
    assert _gate(L, _tw(), x=None) == INVALID
    assert _gate(L, _tw(), x=FAKE + 8) == ALIGN
    assert _gate(L, _tw(W=32)) == UNSUPPORTED            # tile widths: 64, 128, 256
    assert _gate(L, _tw(W=192)) == UNSUPPORTED
    assert _gate(L, _tw(W=64, C=65)) == UNSUPPORTED      # capacity above the tile width
    assert _gate(L, _tw(C=129)) == UNSUPPORTED           # capacity above the tile width
    assert _gate(L, _tw(F=1000), F=1000) == UNSUPPORTED  # F not a multiple of W
    assert _gate(L, _tw(T=255)) == INVALID               # out->T != T
    assert _gate(L, _tw(), d=500) == UNSUPPORTED         # d % 8 != 0
    assert _gate(L, _tw(), d=32) == UNSUPPORTED          # tensor-core path needs d >= 64
    assert _gate(L, _tw(dtype=twell.TW_F32)) == INVALID  # dtype mismatch
    assert _gate(L, _tw(C=-1)) == INVALID
    bad = _tw()
    bad.cnt = None
    assert _gate(L, bad) == INVALID


def test_fused_validation(L):
    tw = _tw()
    f = L.twell_fused_updown
    ws = L.twell_fused_updown_workspace_size(256, 512)
    assert ws > 0
    args = lambda d, wu=FAKE, yd=twell.TW_BF16, n=ws, w=FAKE: (
        FAKE, ctypes.byref(tw), wu, FAKE, d, FAKE, yd, w, n, None, None)
    assert f(*args(4096)) == UNSUPPORTED
    assert f(*args(100)) == UNSUPPORTED
    assert f(*args(512, wu=FAKE + 4)) == ALIGN
    assert f(*args(512, wu=None)) == INVALID
    assert f(*args(512, yd=7)) == INVALID
    assert f(*args(512, n=ws - 1)) == 8        # TW_ERR_WORKSPACE
    assert f(*args(512, w=None)) == INVALID
    # fp32 rows: one warp's ring of 1024-column fp32 slices is the shared-memory limit
    tw32 = _tw(dtype=twell.TW_F32)
    ws32 = L.twell_fused_updown_workspace_size(256, 2048)
    assert f(FAKE, ctypes.byref(tw32), FAKE, FAKE, 2048, FAKE, twell.TW_F32, FAKE, ws32,
             None, None) == UNSUPPORTED


def test_empty_batch_needs_no_token_buffers(L):
    # T == 0: the arrays sized by T may be NULL; the fused call returns before any launch
    tw0 = twell.TwTwellC(0, 1024, 128, 8, twell.TW_BF16, None, None, None, None, 0, None, None,
                         FAKE)
    assert L.twell_fused_updown(None, ctypes.byref(tw0), FAKE, FAKE, 512, None, twell.TW_F32,
                                None, 0, None, None) == 0
    # with tokens the same NULL buffers are rejected
    tw1 = twell.TwTwellC(1, 1024, 128, 8, twell.TW_BF16, None, None, None, None, 0, None, None,
                         FAKE)
    assert L.twell_fused_updown(None, ctypes.byref(tw1), FAKE, FAKE, 512, None, twell.TW_F32,
                                None, 0, None, None) == INVALID


def _hy(T=256, F=1024, C_h=64, cap=32, dtype=twell.TW_BF16, base=FAKE):
    return twell.TwHybridC(T, F, C_h, dtype, base, base, base, base, base, cap, base, base, base, base)


def test_hybrid_validation(L):
    tw, hy = _tw(), _hy()
    assert L.twell_to_hybrid(ctypes.byref(tw), ctypes.byref(_hy(T=128)), None, None) == INVALID
    assert L.twell_to_hybrid(ctypes.byref(tw), ctypes.byref(_hy(C_h=2000)), None, None) == INVALID
    assert L.twell_to_hybrid(ctypes.byref(tw), ctypes.byref(_hy(F=65536 + 128)), None, None) in (INVALID, UNSUPPORTED)
    ws = L.hybrid_ffn_backward_workspace_size(256, 512, 1024, 64, 32)
    assert ws > 0
    args = [FAKE, FAKE, ctypes.byref(hy), FAKE, FAKE, FAKE, 512, 2e-5, FAKE, twell.TW_BF16,
            FAKE, FAKE, FAKE, FAKE]
    assert L.hybrid_ffn_backward(*args, ws - 1, None, None) == 8       # TW_ERR_WORKSPACE
    args2 = list(args)
    args2[0] = FAKE + 2
    assert L.hybrid_ffn_backward(*args2, ws, None, None) == ALIGN
    # dense backup rows are read 16 bytes at a time: F must be a multiple of 8
    odd = _hy(F=1020)
    fws = L.hybrid_ffn_forward_workspace_size(256, 512)
    assert L.hybrid_ffn_forward(FAKE, ctypes.byref(odd), FAKE, FAKE, 512, FAKE, twell.TW_F32, FAKE,
                                fws, None, None) == UNSUPPORTED


def test_workspace_size_grows_with_capacity(L):
    a = L.hybrid_ffn_backward_workspace_size(8192, 2048, 8192, 64, 64)
    b = L.hybrid_ffn_backward_workspace_size(8192, 2048, 8192, 64, 1024)
    assert b > a > 0
    assert L.hybrid_ffn_backward_workspace_size(-1, 2048, 8192, 64, 64) == 0


def test_dense_validation(L):
    f = L.dense_ffn_forward
    assert f(FAKE, FAKE, FAKE, FAKE, 256, 100, 1024, FAKE, FAKE, None, None) == UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, 256, 512, 1000, FAKE, FAKE, None, None) == UNSUPPORTED
    assert f(None, FAKE, FAKE, FAKE, 256, 512, 1024, FAKE, FAKE, None, None) == INVALID


def test_small_batch_validation(L):
    f = L.twell_ffn_small_batch
    ws = L.twell_ffn_small_batch_workspace_size(8, 512, 1024)
    assert ws > 0

    def call(T=8, d=512, F=1024, W=128, dtype=twell.TW_BF16, n=ws, y=FAKE):
        tw = _tw(T=T, F=F, W=W, dtype=dtype)
        return f(FAKE, FAKE, FAKE, FAKE, T, d, F, ctypes.byref(tw), None, y, twell.TW_F32, FAKE,
                 n, None, None)

    assert call(T=65) == UNSUPPORTED                 # up to 64 tokens in one launch
    assert call(W=64) == UNSUPPORTED                 # tile width 128 only
    assert call(dtype=twell.TW_F32) == UNSUPPORTED   # bf16 only
    assert call(d=4096) == UNSUPPORTED               # x of 16 tokens staged in shared memory
    assert call(d=500) == UNSUPPORTED
    assert call(n=ws - 1) == 8                       # TW_ERR_WORKSPACE
    assert call(y=None) == INVALID
    assert call(y=FAKE + 4) == ALIGN


def test_dense_training_validation(L):
    ws = L.dense_ffn_train_workspace_size(256, 1024)
    assert ws == 5 * 256 * 1024 * 2
    assert L.dense_ffn_train_saved_bytes(256, 1024) == 3 * 256 * 1024 * 2
    fwd = L.dense_ffn_train_forward
    assert fwd(FAKE, FAKE, FAKE, FAKE, 256, 500, 1024, FAKE, ws, FAKE, None, None) == UNSUPPORTED
    assert fwd(FAKE, FAKE, FAKE, FAKE, 256, 512, 1000, FAKE, ws, FAKE, None, None) == UNSUPPORTED
    assert fwd(FAKE, FAKE, FAKE, FAKE, 256, 512, 1024, FAKE, ws - 1, FAKE, None, None) == 8
    assert fwd(FAKE, FAKE, FAKE, FAKE, 256, 512, 1024, None, ws, FAKE, None, None) == INVALID
    bwd = L.dense_ffn_train_backward
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 256, 512, 1024, 2e-5, FAKE, ws, FAKE, FAKE, FAKE]
    assert bwd(*args, None, None, None) == INVALID    # dWd missing
    args2 = list(args)
    args2[1] = FAKE + 8
    assert bwd(*args2, FAKE, None, None) == ALIGN


def test_row_gather_validation(L):
    """The measurement entry points reject bad sizes and a misaligned buffer
    before any launch, and launch nothing for zero gathers or zero bytes."""
    ok = twell.STATUS.index("TW_OK")
    bad = twell.STATUS.index("TW_ERR_INVALID_ARG")
    align = twell.STATUS.index("TW_ERR_ALIGNMENT")
    g = L.tw_measure_row_gather
    assert g(FAKE, 0, 2048, 10, 1, FAKE, None) == bad       # no rows
    assert g(FAKE, 10, 2056, 10, 1, FAKE, None) == bad      # d > 2048
    assert g(FAKE, 10, 100, 10, 1, FAKE, None) == bad       # d % 8 != 0
    assert g(FAKE, 10, 2048, -1, 1, FAKE, None) == bad      # negative count
    assert g(None, 10, 2048, 10, 1, FAKE, None) == bad
    assert g(FAKE, 10, 2048, 10, 1, None, None) == bad
    assert g(FAKE + 8, 10, 2048, 10, 1, FAKE, None) == align
    assert g(FAKE, 10, 2048, 0, 1, FAKE, None) == ok         # nothing to launch
    r = L.tw_measure_stream_read
    assert r(FAKE, -16, FAKE, None) == bad                    # negative size
    assert r(FAKE, 24, FAKE, None) == bad                     # not whole 16-byte chunks
    assert r(None, 16, FAKE, None) == bad
    assert r(FAKE, 16, None, None) == bad
    assert r(FAKE + 8, 16, FAKE, None) == align
    assert r(FAKE, 0, FAKE, None) == ok                       # nothing to launch
