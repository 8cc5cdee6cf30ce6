"""Helpers for the GPU parity tests: move seeded inputs to the device, bring
results back as exact fp64, and compare TwELL / hybrid encodings bit for bit
against the CPU oracle run on the GPU's own dumped gate tensor."""
import numpy as np
import torch

import oracle
from activation_sparse_transformer_tma_b200 import synth


def to_dev(a, dtype):
    """Stored synth tensor (uint16 bf16 bits or float32) -> CUDA tensor."""
    if dtype == synth.BF16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def raw(t):
    """CUDA tensor -> numpy storage (uint16 bits for bf16)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def f64(t):
    """CUDA tensor -> exact fp64 numpy values."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return synth.bf16_to_f64(t.view(torch.int16).numpy().view(np.uint16))
    return t.numpy().astype(np.float64)


def inputs(w):
    dt = w["dtype"]
    return {k: to_dev(w[k], dt) for k in ("x", "Wg_t", "Wu_t", "Wd", "dy") if k in w}


def widened(w):
    dt = w["dtype"]
    return {k: synth.widen(w[k], dt) for k in ("x", "Wg_t", "Wu_t", "Wd", "dy") if k in w}


def rms(a):
    return float(np.sqrt(np.mean(np.square(a)))) if a.size else 0.0


def assert_twell_matches_oracle(tw_gpu, g_dump64, rows=None):
    """The GPU's TwELL must equal the oracle's encoding of the GPU's own dense g.

    rows: optional sorted token subset (the oracle encodes g_dump64 = g[rows]).
    Values, indices and counts bit for bit; spill entries as a set keyed by (t, k).
    """
    W, C = tw_gpu.W, tw_gpu.C
    ref = oracle.twell_encode(g_dump64, W, C)
    T = tw_gpu.T
    rows = np.arange(T) if rows is None else np.asarray(rows)
    cnt = raw(tw_gpu.cnt)[:, rows]
    assert np.array_equal(cnt, ref["cnt"]), "cnt differs"
    if C:
        val = f64(tw_gpu.val)[:, rows]
        idx = raw(tw_gpu.idx)[:, rows]
        assert np.array_equal(val.view(np.uint64), ref["val"].view(np.uint64)), "val differs"
        assert np.array_equal(idx, ref["idx"]), "idx differs"
    # spills: compare as sets keyed by (t, k)
    n_gpu = int(tw_gpu.spill_n.item())
    assert n_gpu <= tw_gpu.spill_cap
    sref = raw(tw_gpu.spill_ref)
    stk = raw(tw_gpu.spill_tk)[:n_gpu]
    sval = f64(tw_gpu.spill_val)[:n_gpu]
    gpu_sp = {}
    for r, (t, k) in enumerate(stk):
        gpu_sp[(int(t), int(k))] = r
    row_pos = {int(t): i for i, t in enumerate(rows)}
    if rows.size == T:
        assert n_gpu == ref["n_spill"]
    for (t_local, k), sv in zip(ref["spill_tk"], ref["spill_val"]):
        t = int(rows[t_local])
        assert (t, int(k)) in gpu_sp, f"missing spill ({t},{k})"
        r = gpu_sp[(t, int(k))]
        assert sref[k, t] == r
        assert np.array_equal(sval[r].view(np.uint64), sv.view(np.uint64))
    # every GPU spill of a checked row is expected by the oracle
    ref_keys = {(int(rows[t]), int(k)) for t, k in ref["spill_tk"]}
    for key in gpu_sp:
        if key[0] in row_pos:
            assert key in ref_keys
    return ref
