"""twell_fused_updown_noalloc: the fused up+down projection for callers that
cannot allocate device memory (no workspace argument; the library keeps its
work plan in a fixed 16 MiB device array of its own).

The GPU test calls it through the C ABI twice in a row and checks both
results against the workspace entry point twell_fused_updown, within the
parity bar used for y everywhere (1e-2 * rms).  This file is named so that
pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from activation_sparse_transformer_tma_b200 import synth
from activation_sparse_transformer_tma_b200 import twell as tw


def _noalloc_rc(x, g, Wu, Wd, y):
    s = g.struct()
    return tw.lib().twell_fused_updown_noalloc(
        x.data_ptr(), ctypes.byref(s), Wu.data_ptr(), Wd.data_ptr(), x.shape[1], y.data_ptr(),
        tw.TW_F32 if y.dtype == torch.float32 else tw.TW_BF16, None,
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
@pytest.mark.parametrize("name,T", [("ffn_0p5b", 2048), ("ffn_2b", 16384)])
def test_noalloc_matches_workspace_entry_point(name, T):
    w = synth.make_workload(name, T=T)
    dev = {k: torch.from_numpy(w[k].view(np.int16)).cuda().view(torch.bfloat16)
           for k in ("x", "Wg_t", "Wu_t", "Wd")}
    d, F, C = w["d"], w["F"], w["C"]
    g = tw.Twell(T, F, C, dtype=torch.bfloat16, spill_cap=(F // 128) * T // 4)
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
    ref = y_ws.double().cpu().numpy()
    scale = np.sqrt(np.mean(ref ** 2))
    for y in outs:
        got = y.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref)) <= 1e-2 * scale
    # the same plan twice: identical bits
    assert torch.equal(outs[0], outs[1])


def test_noalloc_rejects_a_plan_larger_than_its_array():
    # Host-side check, before any device work: fake, never dereferenced
    # addresses; T far beyond what 16 MiB of plan can describe.
    fake = 0x10000
    T = 2_000_000
    s = tw.TwTwellC(T, 1024, 128, 8, tw.TW_BF16, fake, fake, fake, fake, 64, fake, fake, fake)
    rc = tw.lib().twell_fused_updown_noalloc(fake, ctypes.byref(s), fake, fake, 1024, fake,
                                             tw.TW_F32, None, None)
    assert rc == 2  # TW_ERR_UNSUPPORTED
