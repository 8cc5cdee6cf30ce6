"""twell_fused_updown_noalloc: the fused up+down projection for callers that
cannot allocate device memory (no workspace argument; the library keeps its
work plan in a fixed 16 MiB device array of its own).

The GPU tests call it through the C ABI twice in a row and check both results
against the workspace entry point twell_fused_updown and against the fp64 CPU
oracle on a seeded sample of rows, within the parity bar used for y
everywhere (1e-2 * rms).  One case has far more heavy tokens than the array
has partial rows for, so most of them run unsplit, the path in which this
entry point differs from the workspace one.  This file is named so that
pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from activation_sparse_transformer_tma_b200 import synth
from activation_sparse_transformer_tma_b200 import twell as tw


def _noalloc_rc(x, g, Wu, Wd, y):
    s = g.struct()
    return tw.lib().twell_fused_updown_noalloc(
        x.data_ptr(), ctypes.byref(s), Wu.data_ptr(), Wd.data_ptr(), x.shape[1], y.data_ptr(),
        tw.TW_F32 if y.dtype == torch.float32 else tw.TW_BF16, None,
        torch.cuda.current_stream().cuda_stream)


SCRATCH_BYTES = 16 << 20


def _oracle_rows(w, rows):
    dt = w["dtype"]
    x, Wg, Wu, Wd = (synth.widen(w[k], dt) for k in ("x", "Wg_t", "Wu_t", "Wd"))
    return oracle.dense_ffn(x[rows], Wg, Wu, Wd, g_round="bf16")["y"]


@pytest.mark.gpu
@pytest.mark.parametrize("name,T,mean_active", [("ffn_0p5b", 2048, 29.0),
                                                ("ffn_2b", 16384, 29.0),
                                                ("ffn_2b", 4096, 300.0)])
def test_noalloc_matches_workspace_entry_point_and_oracle(name, T, mean_active):
    w = synth.make_workload(name, T=T, mean_active=mean_active)
    dev = {k: torch.from_numpy(w[k].view(np.int16)).cuda().view(torch.bfloat16)
           for k in ("x", "Wg_t", "Wu_t", "Wd")}
    d, F, C = w["d"], w["F"], w["C"]
    g = tw.Twell(T, F, C, dtype=torch.bfloat16, spill_cap=(F // 128) * T)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tw.twell_gate_gemm(dev["x"], dev["Wg_t"], g, None, st)

    y_ws = torch.empty((T, d), dtype=torch.float32, device="cuda")
    tw.twell_fused_updown(dev["x"], g, dev["Wu_t"], dev["Wd"], y_ws, tw.fused_workspace(T, d), st)
    outs = []
    for _ in range(2):  # two calls in a row share the library's array
        y = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_rc(dev["x"], g, dev["Wu_t"], dev["Wd"], y) == 0
        outs.append(y)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, tw.status_bits(st)
    if mean_active > 100:
        # Split parts of 64 entries that the heavy tokens would need, against
        # the most partial rows of d fp32 values the whole array could hold:
        # the array's split capacity binds, so heavy tokens run unsplit.
        n = g.cnt.to(torch.int64).sum(0)
        parts = int(((n + 63) // 64 * (n > 64)).sum().item())
        assert parts > SCRATCH_BYTES // (4 * d)
    ref = y_ws.double().cpu().numpy()
    scale = np.sqrt(np.mean(ref ** 2))
    rows = synth.subsample_rows(T, 64, seed=3)
    y_or = _oracle_rows(w, rows)
    s_or = np.sqrt(np.mean(y_or ** 2))
    for y in outs:
        got = y.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref)) <= 1e-2 * scale
        assert np.max(np.abs(got[rows] - y_or)) <= 1e-2 * s_or
    # the same plan twice: identical bits
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("T,d", [(2_000_000, 1024), (697_185, 8), (696_849, 2048)])
def test_noalloc_rejects_a_plan_larger_than_its_array(T, d):
    # Host-side check, before any device work: fake, never dereferenced
    # addresses.  The plan takes about 24 bytes per token, so the 16 MiB array
    # holds T <= 696,848 tokens at every supported d; one token more (at the
    # widest d), or more than the narrowest d allows, is rejected.
    fake = 0x10000
    s = tw.TwTwellC(T, 1024, 128, 8, tw.TW_BF16, fake, fake, fake, fake, 64, fake, fake, fake)
    rc = tw.lib().twell_fused_updown_noalloc(fake, ctypes.byref(s), fake, fake, d, fake,
                                             tw.TW_F32, None, None)
    assert rc == 2  # TW_ERR_UNSUPPORTED


def test_noalloc_empty_batch_needs_no_token_buffers():
    # T == 0: as for twell_fused_updown, x, y and the per-token TwELL arrays
    # may be NULL; the call returns TW_OK before any device work.
    fake = 0x10000
    s0 = tw.TwTwellC(0, 1024, 128, 8, tw.TW_BF16, None, None, None, None, 0, None, None, fake)
    assert tw.lib().twell_fused_updown_noalloc(None, ctypes.byref(s0), fake, fake, 512, None,
                                               tw.TW_F32, None, None) == 0
    # with tokens the same NULL buffers are rejected
    s1 = tw.TwTwellC(1, 1024, 128, 8, tw.TW_BF16, None, None, None, None, 0, None, None, fake)
    assert tw.lib().twell_fused_updown_noalloc(None, ctypes.byref(s1), fake, fake, 512, None,
                                               tw.TW_F32, None, None) == 1  # TW_ERR_INVALID_ARG
