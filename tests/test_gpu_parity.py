"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bars (written per check below):
* TwELL values / indices / counts and the hybrid split: bit-exact against the
  oracle's encoding of the GPU's own dumped gate tensor (spills as sets).
* End-to-end y: max|y_gpu - y_ref| <= 1e-2 * rms(y_ref) for bf16 and
  <= 1e-5 * rms(y_ref) for fp32, y_ref the fp64 oracle from the same inputs
  with g rounded to its storage dtype (TwELL stores g in the model dtype), and
  y stored in fp32 (the accumulator precision).  A bf16-stored y adds its own
  rounding, up to 2^-9 |y| per element, which for heavy-tailed y exceeds the
  first bar; it is checked elementwise against 1e-2 rms + 2^-8 |y_ref|.
* Gradients: the oracle's backward conditioned on the GPU's saved hybrid g and
  u; max|d_gpu - d_ref| <= 1e-2 * rms(d_ref) per tensor (bf16).
"""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_transformer_tma_b200 import synth
from activation_sparse_transformer_tma_b200 import twell as tw
from gpu_helpers import assert_twell_matches_oracle, f64, inputs, raw, rms, widened

pytestmark = pytest.mark.gpu

TOL = {synth.BF16: 1e-2, synth.F32: 1e-5}
TDT = {synth.BF16: torch.bfloat16, synth.F32: torch.float32}


def run_forward(w, C=None, spill_cap=None, dump=True, y_dtype=torch.float32):
    dev = inputs(w)
    T, d, F = w["T"], w["d"], w["F"]
    C = w["C"] if C is None else C
    dt = TDT[w["dtype"]]
    W = w.get("W", 128)
    if spill_cap is None:
        spill_cap = (F // W) * T  # room for every (t, k) to spill
    g = tw.Twell(T, F, C, dtype=dt, spill_cap=spill_cap, W=W)
    gd = torch.empty((T, F), dtype=dt, device="cuda") if dump else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tw.twell_gate_gemm(dev["x"], dev["Wg_t"], g, gd, st)
    y = torch.empty((T, d), dtype=y_dtype, device="cuda")
    tw.twell_fused_updown(dev["x"], g, dev["Wu_t"], dev["Wd"], y, tw.fused_workspace(T, d), st)
    torch.cuda.synchronize()
    return dev, g, gd, y, st


def check_gate_values(g_dump64, x64, wg64, rows, g_round="bf16"):
    """Dumped g against the oracle's rounded fp64 gate: the fp32-accumulated z
    may land on the other side of a rounding boundary (one bf16 ulp, 2^-7
    relative) or of zero (|z| at the level of the fp32 accumulation error)."""
    ref = oracle.gate_rows(x64, wg64, rows, g_round=g_round)
    err = np.abs(g_dump64[rows] - ref)
    assert np.all(err <= 2.0 ** -7 * np.abs(ref) + 1e-4), float(err.max())


def check_y(y64, w64, rows, tol, g_round="bf16", elem_rel=0.0):
    out = oracle.dense_ffn(w64["x"][rows], w64["Wg_t"], w64["Wu_t"], w64["Wd"], g_round=g_round)
    ref = out["y"]
    s = rms(ref)
    err = np.abs(y64[rows] - ref)
    assert np.all(err <= tol * s + elem_rel * np.abs(ref)), (float(err.max()), s)
    return float(err.max()) / s


SMALL = [
    # T, d, F, C, kind, mean_active
    (300, 320, 640, 8, "dead20", 29.0),      # ragged T and F, spills
    (300, 320, 640, 8, "dead20", 120.0),     # spill-heavy
    (1, 256, 1024, 8, "zipf", 29.0),         # one token
    (129, 64, 256, 0, "dead20", 29.0),       # C = 0: every non-empty tile spills
    (257, 2048, 1280, 32, "zipf", 40.0),     # full-width rows, largest C
    (128, 512, 2048, 16, "uniform4", 29.0),
    (40, 512, 640, 2, "dead20", 60.0),       # small batch: x box narrower than the tile, spills
    (64, 1024, 1024, 8, "zipf", 29.0),
    (65, 256, 1024, 8, "zipf", 29.0),
    # C = 8 with full-width rows (d is exactly a team's slices): TwELL data
    # staged one item ahead when T % 4 == 0, read directly otherwise
    (301, 2048, 1280, 8, "zipf", 29.0),      # direct
    (1001, 512, 1024, 8, "dead20", 29.0),    # direct, many items
    (300, 512, 640, 8, "dead20", 120.0),     # staged, spill-heavy
]


@pytest.mark.parametrize("T,d,F,C,kind,ma", SMALL)
def test_bf16_gate_and_fused_small(T, d, F, C, kind, ma):
    w = synth.make_workload(T=T, d=d, F=F, W=128, C=C, dtype=synth.BF16, kind=kind,
                            mean_active=ma, seed=T + d)
    dev, g, gd, y, st = run_forward(w)
    assert int(st.item()) == 0
    w64 = widened(w)
    g64 = f64(gd)
    rows = np.arange(T, dtype=np.int32)
    check_gate_values(g64, w64["x"], w64["Wg_t"], rows)
    assert_twell_matches_oracle(g, g64)
    check_y(f64(y), w64, rows, TOL[synth.BF16])


# planned gather engine with both slice widths (and 12 tokens), and the
# one-CTA-per-token small-batch kernel (T <= 8)
@pytest.mark.parametrize("d,T", [(320, 300), (256, 300), (256, 12), (256, 6)])
def test_bf16_output_y(d, T):
    w = synth.make_workload(T=T, d=d, F=640, W=128, C=8, dtype=synth.BF16, kind="dead20",
                            mean_active=29.0, seed=620)
    _, g, gd, y, st = run_forward(w, y_dtype=torch.bfloat16)
    _, _, _, y32, _ = run_forward(w)
    _, _, _, y32b, _ = run_forward(w)
    # both paths are deterministic, and the bf16 output is the fp32 result rounded once
    assert torch.equal(y32, y32b)
    assert torch.equal(y, y32.to(torch.bfloat16))
    check_y(f64(y), widened(w), np.arange(T, dtype=np.int32), TOL[synth.BF16],
            elem_rel=2.0 ** -8)


@pytest.mark.parametrize("C,T", [(16, None), (2, None), (2, 10)])  # T=10: small-batch kernel
def test_fp32_tiny_config(C, T):
    w = synth.make_workload("tiny_fp32") if T is None else synth.make_workload("tiny_fp32", T=T)
    dev, g, gd, y, st = run_forward(w, C=C)
    assert int(st.item()) == 0
    w64 = widened(w)
    g64 = f64(gd)
    rows = np.arange(w["T"], dtype=np.int32)
    ref = oracle.gate_rows(w64["x"], w64["Wg_t"], rows, g_round="f32")
    # fp32 recursive summation of d products: |err| <= d * 2^-24 * sum_i |x_i w_i|
    # (plus one rounding of the result)
    bound = w["d"] * 2.0 ** -24 * (np.abs(w64["x"]) @ np.abs(w64["Wg_t"]).T) + 2.0 ** -23 * np.abs(ref)
    assert np.all(np.abs(g64 - ref) <= bound)
    assert_twell_matches_oracle(g, g64)
    if C == 2:
        assert int(g.spill_n.item()) > 0
    check_y(f64(y), w64, rows, TOL[synth.F32], g_round="f32")


# Capacities above 32 up to the tile width.  Half the units of a tile are
# active on average (mean_active = 300 of 512 live units), so at C = 64 many
# tiles spill and the slots past 32 are written straight from the epilogue;
# at C = W = 128 the TwELL holds every tile whole and nothing spills.  T = 300
# runs the tile GEMM, T <= 64 the small-batch gate, and fp32 its own kernel.
WIDE_C = [
    # T, C, dtype
    (300, 64, synth.BF16),
    (300, 128, synth.BF16),
    (300, 40, synth.BF16),     # not a multiple of 8: scalar stores of the staged slots
    (40, 64, synth.BF16),
    (40, 128, synth.BF16),
    (1, 128, synth.BF16),
    (130, 64, synth.F32),
    (130, 128, synth.F32),
]


@pytest.mark.parametrize("T,C,dt", WIDE_C)
def test_capacity_up_to_tile_width(T, C, dt):
    d = 256 if dt == synth.F32 else 320
    w = synth.make_workload(T=T, d=d, F=640, W=128, C=C, dtype=dt, kind="dead20",
                            mean_active=300.0, seed=T + C)
    dev, g, gd, y, st = run_forward(w)
    assert int(st.item()) == 0
    w64 = widened(w)
    g64 = f64(gd)
    ref = assert_twell_matches_oracle(g, g64)
    cnt = raw(g.cnt)
    assert cnt.max() > 32  # the rows past the staged slots are exercised
    if C == 128:
        assert int(g.spill_n.item()) == 0 and ref["n_spill"] == 0
    else:
        assert int(g.spill_n.item()) > 0
    rows = np.arange(T, dtype=np.int32)
    check_y(f64(y), w64, rows, TOL[dt], g_round="bf16" if dt == synth.BF16 else "f32")


# Tile widths other than 128: the tile GEMM packs BN / W TwELL tiles per
# accumulator tile (W = 256 always on the 256-wide accumulator), also for
# small batches; the fp32 gate sizes its tile by W; the fused kernel and the
# hybrid conversion read W from the TwELL descriptor.
TILE_W = [
    # W, T, C, dtype
    (64, 300, 8, synth.BF16),
    (256, 300, 8, synth.BF16),
    (256, 300, 64, synth.BF16),
    (64, 40, 4, synth.BF16),
    (256, 33, 16, synth.BF16),
    (64, 130, 8, synth.F32),
    (256, 130, 8, synth.F32),
]


@pytest.mark.parametrize("W,T,C,dt", TILE_W)
def test_tile_widths(W, T, C, dt):
    d = 256 if dt == synth.F32 else 320
    w = synth.make_workload(T=T, d=d, F=1024, W=W, C=C, dtype=dt, kind="dead20",
                            mean_active=60.0, seed=W + T + C)
    dev, g, gd, y, st = run_forward(w)
    assert int(st.item()) == 0
    w64 = widened(w)
    g64 = f64(gd)
    assert_twell_matches_oracle(g, g64)
    assert int(g.spill_n.item()) > 0 or C >= 64
    check_y(f64(y), w64, np.arange(T, dtype=np.int32), TOL[dt],
            g_round="bf16" if dt == synth.BF16 else "f32")


@pytest.mark.parametrize("W", [64, 256])
def test_hybrid_from_other_tile_widths(W):
    w = synth.make_workload(T=300, d=256, F=1024, W=W, C=8, C_h=64, dtype=synth.BF16,
                            kind="pareto", lam=2e-5, seed=W, mean_active=30.0, with_dy=True)
    got = check_hybrid_all(w, run_hybrid(w, backup_cap=300))
    assert 0 < got["n_backup"] < 300


def test_hybrid_weight_gradients_of_a_unit_with_thousands_of_entries():
    """Zipf units without the permutation: the hottest units are active for
    half of 5000 tokens, so their records exceed the 2048 a CTA sorts in
    shared memory and take the sorted-runs path of the weight gradients."""
    w = synth.make_workload(T=5000, d=256, F=1024, W=128, C=8, C_h=64, dtype=synth.BF16,
                            kind="zipf", lam=2e-5, seed=31, mean_active=29.0, permute=False,
                            with_dy=True)
    res = run_hybrid(w, backup_cap=5000)
    hy = res[5]
    got = check_hybrid_all(w, res)
    cols = got["ell_idx"][got["ell_g"] != 0]
    bcols = np.nonzero(got["backup_g"])[1]
    per_unit = np.bincount(np.concatenate([cols, bcols]).astype(np.int64), minlength=1024)
    assert per_unit.max() > 2048


def test_hybrid_from_wide_capacity_twell():
    """TwELL -> hybrid with C = 64: tiles with more than 32 slots feed ELL rows."""
    w = synth.make_workload(T=300, d=256, F=640, W=128, C=64, C_h=155, dtype=synth.BF16,
                            kind="dead20", lam=2e-5, seed=77, mean_active=150.0, with_dy=True)
    got = check_hybrid_all(w, run_hybrid(w, backup_cap=300))
    assert 0 < got["n_backup"] < 300


def test_ffn_0p5b_full_size():
    w = synth.make_workload("ffn_0p5b")
    dev, g, gd, y, st = run_forward(w)
    assert int(st.item()) == 0
    w64 = widened(w)
    g64 = f64(gd)
    assert_twell_matches_oracle(g, g64)
    rows = synth.subsample_rows(w["T"], 192)
    check_gate_values(g64, w64["x"], w64["Wg_t"], rows)
    check_y(f64(y), w64, rows, TOL[synth.BF16])


def test_zipf_hot_units_in_one_tile():
    """Zipf units without the seeded permutation of their ranks: the 128 hottest
    units are tile 0, so nearly every token overflows that tile and most of
    the entries come from spill segments.  TwELL on every token, y on a
    sample of rows."""
    w = synth.make_workload(T=4096, d=1024, F=4096, W=128, C=8, dtype=synth.BF16, kind="zipf",
                            mean_active=29.0, seed=3, permute=False)
    dev, g, gd, y, st = run_forward(w)
    assert int(st.item()) == 0
    assert int(g.spill_n.item()) > w["T"] // 2
    g64 = f64(gd)
    assert_twell_matches_oracle(g, g64)
    w64 = widened(w)
    rows = synth.subsample_rows(w["T"], 192)
    check_gate_values(g64, w64["x"], w64["Wg_t"], rows)
    check_y(f64(y), w64, rows, TOL[synth.BF16])


@pytest.mark.parametrize("T", [16, 64])
def test_small_batch_hot_units_in_one_tile(T):
    """The single-launch small batch with every token's hottest units in tile 0
    (one heavy tile per token): T = 16 takes the packing-with-dots path, T = 64
    the balanced one."""
    w = synth.make_workload(T=T, d=2048, F=8192, W=128, C=8, dtype=synth.BF16, kind="zipf",
                            mean_active=29.0, seed=9, permute=False)
    dev = inputs(w)
    d, F = w["d"], w["F"]
    g = tw.Twell(T, F, 8, dtype=torch.bfloat16, spill_cap=(F // 128) * T)
    gd = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tw.twell_ffn_small_batch(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"], g, y,
                             tw.small_batch_workspace(T, d, F), gd, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, tw.status_bits(st)
    g64 = f64(gd)
    assert_twell_matches_oracle(g, g64)
    check_y(f64(y), widened(w), np.arange(T, dtype=np.int32), TOL[synth.BF16])


def test_ffn_2b_full_size():
    """The bench workload, same launch configuration: TwELL compared on every
    token (in chunks), y on a seeded sample of rows."""
    w = synth.make_workload("ffn_2b")
    dev, g, gd, y, st = run_forward(w)
    assert int(st.item()) == 0
    T = w["T"]
    for r0 in range(0, T, 2048):
        rows = np.arange(r0, min(T, r0 + 2048))
        assert_twell_matches_oracle(g, f64(gd[r0:r0 + len(rows)]), rows=rows)
    w64 = widened(w)
    rows = synth.subsample_rows(T, 96)
    check_gate_values(f64(gd), w64["x"], w64["Wg_t"], rows)
    check_y(f64(y), w64, rows, TOL[synth.BF16])


def test_weight_rows_16_byte_aligned():
    """Weights 16-byte aligned but not 32 (the ABI asks for 16) give the same
    parity as aligned ones on the full-width kernel."""
    T, d, F = 300, 2048, 640
    w = synth.make_workload(T=T, d=d, F=F, W=128, C=8, dtype=synth.BF16, kind="zipf",
                            mean_active=29.0, seed=77)
    dv = inputs(w)
    shifted = {}
    for k in ("Wu_t", "Wd"):
        buf = torch.empty(F * d + 8, dtype=torch.bfloat16, device="cuda")
        v = buf[8:].view(F, d)  # 16 bytes past a 32-byte boundary
        v.copy_(dv[k])
        assert v.data_ptr() % 32 == 16
        shifted[k] = v
    g = tw.Twell(T, F, 8, dtype=torch.bfloat16, spill_cap=(F // 128) * T)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tw.twell_gate_gemm(dv["x"], dv["Wg_t"], g, None, st)
    ys = []
    for Wu, Wd in ((dv["Wu_t"], dv["Wd"]), (shifted["Wu_t"], shifted["Wd"])):
        y = torch.empty((T, d), dtype=torch.float32, device="cuda")
        tw.twell_fused_updown(dv["x"], g, Wu, Wd, y, tw.fused_workspace(T, d), st)
        ys.append(y)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, tw.status_bits(st)
    w64 = widened(w)
    rows = synth.subsample_rows(T, 64)
    for y in ys:
        check_y(f64(y), w64, rows, TOL[synth.BF16])


def test_back_to_back_calls_share_one_workspace():
    """Gate and fused calls of two different batches queued back to back on one
    stream, sharing the TwELL buffers and the fused workspace, with no host
    synchronisation between them: each launch waits for the previous one's
    results (programmatic dependent launches) and the planner clears the
    engine's counters itself.  Both outputs equal those of separate,
    synchronised calls, bit for bit."""
    T, d, F = 3000, 1024, 2048
    wa = synth.make_workload(T=T, d=d, F=F, W=128, C=8, dtype=synth.BF16, kind="zipf",
                             mean_active=29.0, seed=101)
    wb = synth.make_workload(T=T, d=d, F=F, W=128, C=8, dtype=synth.BF16, kind="zipf",
                             mean_active=60.0, seed=202)
    da, db = inputs(wa), inputs(wb)
    g = tw.Twell(T, F, 8, dtype=torch.bfloat16, spill_cap=(F // 128) * T)
    ws = tw.fused_workspace(T, d)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    refs = []
    for dv in (da, db):  # separate calls, synchronised
        y = torch.empty((T, d), dtype=torch.float32, device="cuda")
        tw.twell_gate_gemm(dv["x"], dv["Wg_t"], g, None, st)
        tw.twell_fused_updown(dv["x"], g, dv["Wu_t"], dv["Wd"], y, ws, st)
        torch.cuda.synchronize()
        refs.append(y)
    ys = [torch.empty((T, d), dtype=torch.float32, device="cuda") for _ in range(4)]
    for i, dv in enumerate((da, db, da, db)):  # queued back to back
        tw.twell_gate_gemm(dv["x"], dv["Wg_t"], g, None, st)
        tw.twell_fused_updown(dv["x"], g, dv["Wu_t"], dv["Wd"], ys[i], ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, tw.status_bits(st)
    for i in range(4):
        assert torch.equal(ys[i], refs[i % 2]), i
    check_y(f64(refs[1]), widened(wb), synth.subsample_rows(T, 48), TOL[synth.BF16])


# Small batches (T <= 64) take the cluster split-K gate; the cases cover
# cluster sizes 8, 8 with uneven k-block shares (d = 520), 2 (partials of
# 48 tokens), 1 (more tiles than SMs), C = 0 and the largest C.  The last
# case splits every token into tens of parts of the fused kernel.
FEW = [
    # T, d, F, C, kind, mean_active
    (1, 1024, 1024, 8, "zipf", 29.0),
    (5, 520, 2048, 2, "dead20", 60.0),
    (33, 2048, 4096, 8, "zipf", 29.0),
    (17, 256, 19200, 8, "zipf", 29.0),
    (64, 128, 640, 0, "dead20", 29.0),
    (16, 2048, 1280, 32, "zipf", 40.0),
    (20, 512, 8192, 8, "zipf", 400.0),  # dozens of parts per token: deep sum trees
]


@pytest.mark.parametrize("T,d,F,C,kind,ma", FEW)
def test_small_batch_gate(T, d, F, C, kind, ma):
    w = synth.make_workload(T=T, d=d, F=F, W=128, C=C, dtype=synth.BF16, kind=kind,
                            mean_active=ma, seed=T * 7 + d)
    dev, g, gd, y, st = run_forward(w)
    assert int(st.item()) == 0
    w64 = widened(w)
    g64 = f64(gd)
    rows = np.arange(T, dtype=np.int32)
    check_gate_values(g64, w64["x"], w64["Wg_t"], rows)
    assert_twell_matches_oracle(g, g64)
    check_y(f64(y), w64, rows, TOL[synth.BF16])
    # the same launch without the dense dump writes the same TwELL
    _, g2, _, _, _ = run_forward(w, dump=False)
    assert torch.equal(g.cnt, g2.cnt) and torch.equal(g.spill_n, g2.spill_n)
    if C > 0:
        assert torch.equal(g.val, g2.val) and torch.equal(g.idx, g2.idx)


def test_small_batch_spill_capacity_overflow_is_flagged():
    w = synth.make_workload(T=40, d=256, F=512, W=128, C=2, dtype=synth.BF16, kind="dead20",
                            mean_active=60.0, seed=41)
    _, g, gd, y, st = run_forward(w, spill_cap=4)
    assert int(g.spill_n.item()) > 4
    assert "TW_ERR_SPILL_CAPACITY" in tw.status_bits(st)
    ref = oracle.twell_encode(f64(gd), 128, 2)
    assert np.array_equal(raw(g.cnt), ref["cnt"])
    assert int(g.spill_n.item()) == ref["n_spill"]


@pytest.mark.parametrize("T", [1, 8, 64])
def test_decode_sizes(T):
    w = synth.make_workload("decode_2b", T=T)
    dev, g, gd, y, st = run_forward(w)
    assert int(st.item()) == 0
    w64 = widened(w)
    rows = np.arange(T, dtype=np.int32)
    check_gate_values(f64(gd), w64["x"], w64["Wg_t"], rows)
    assert_twell_matches_oracle(g, f64(gd))
    check_y(f64(y), w64, rows, TOL[synth.BF16])


# One cooperative launch for the whole small-batch FFN: gate partial sums on
# mma.sync over every SM, TwELL packing, dot products, updates (per chunk of
# a token's entries, with partial rows for the long tokens).  T crosses the
# 8-token MMA column tiles and the 16-token switch to balanced dot products
# and updates; d and F are ragged against the 32-column steps and 256-column
# slices.
SMALL_STEP = [
    # T, d, F, C, kind, mean_active
    (1, 2048, 8192, 8, "zipf", 29.0),
    (5, 320, 640, 2, "dead20", 60.0),
    (8, 512, 1024, 8, "zipf", 29.0),
    (9, 256, 1280, 0, "dead20", 29.0),
    (16, 2048, 4096, 8, "zipf", 29.0),
    (16, 1024, 1024, 64, "dead20", 300.0),
    (3, 64, 256, 128, "dead20", 100.0),
    (4, 72, 384, 8, "dead20", 29.0),      # d not a multiple of 32
    (12, 1000, 1280, 8, "zipf", 29.0),
    (17, 320, 640, 8, "dead20", 60.0),   # balanced dot products and updates from here on
    (32, 512, 1024, 8, "zipf", 100.0),
    (33, 2048, 2048, 8, "zipf", 29.0),
    (64, 512, 1280, 16, "zipf", 200.0),  # heavy tokens: many entries per tile
    # about 6 chunks of 128 entries per token: the chunk rows of the workspace
    # run out, and the tokens past them are added up unsplit
    (48, 256, 2048, 8, "dead20", 700.0),
]


@pytest.mark.parametrize("T,d,F,C,kind,ma", SMALL_STEP)
def test_small_batch_single_launch(T, d, F, C, kind, ma):
    w = synth.make_workload(T=T, d=d, F=F, W=128, C=C, dtype=synth.BF16, kind=kind,
                            mean_active=ma, seed=T * 13 + d)
    dev = inputs(w)
    g = tw.Twell(T, F, C, dtype=torch.bfloat16, spill_cap=(F // 128) * T)
    gd = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
    ws = tw.small_batch_workspace(T, d, F)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ys = []
    for _ in range(3):  # the barrier counters reset themselves between calls
        y = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
        tw.twell_ffn_small_batch(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"], g, y, ws, gd, st)
        ys.append(y)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, tw.status_bits(st)
    assert int(ws[:8].view(torch.int32).abs().sum().item()) == 0
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])
    w64 = widened(w)
    g64 = f64(gd)
    rows = np.arange(T, dtype=np.int32)
    check_gate_values(g64, w64["x"], w64["Wg_t"], rows)
    assert_twell_matches_oracle(g, g64)
    check_y(f64(ys[0]), w64, rows, TOL[synth.BF16])
    # bf16 y: the fp32 result rounded once
    yb = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    tw.twell_ffn_small_batch(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"], g, yb, ws, None, st)
    torch.cuda.synchronize()
    assert torch.equal(yb, ys[0].to(torch.bfloat16))


@pytest.mark.parametrize("T", [1, 8, 16, 64])
def test_small_batch_single_launch_decode_2b(T):
    """The decoding workload (the 2B weights, the first T tokens) in the launch
    configuration the benchmark times."""
    w = synth.make_workload("decode_2b", T=T)
    dev = inputs(w)
    d, F, C = w["d"], w["F"], w["C"]
    g = tw.Twell(T, F, C, dtype=torch.bfloat16, spill_cap=4096)
    gd = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tw.twell_ffn_small_batch(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"], g, y,
                             tw.small_batch_workspace(T, d, F), gd, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, tw.status_bits(st)
    w64 = widened(w)
    g64 = f64(gd)
    assert_twell_matches_oracle(g, g64)
    check_y(f64(y), w64, np.arange(T, dtype=np.int32), TOL[synth.BF16])


def test_bounded_wait_runs_out_and_the_next_call_is_correct():
    """The tile GEMM's waits are bounded.  With its loads withheld (a test aid),
    the MMA issuer waits on a barrier that no copy will complete; after the
    20 ms limit every CTA flags TW_ERR_TIMEOUT, frees its tensor memory and
    returns.  A normal call right after it, on the same stream, packs the
    TwELL bit-exactly."""
    import time
    w = synth.make_workload(T=300, d=256, F=640, W=128, C=8, dtype=synth.BF16, kind="dead20",
                            mean_active=29.0, seed=5)
    dev = inputs(w)
    g = tw.Twell(300, 640, 8, dtype=torch.bfloat16, spill_cap=5 * 300)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    tw.lib().tw_test_withhold_next_gate_loads(20_000_000)
    t0 = time.perf_counter()
    tw.twell_gate_gemm(dev["x"], dev["Wg_t"], g, None, st)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 2.0
    assert "TW_ERR_TIMEOUT" in tw.status_bits(st)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    gd = torch.empty((300, 640), dtype=torch.bfloat16, device="cuda")
    tw.twell_gate_gemm(dev["x"], dev["Wg_t"], g, gd, st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0, tw.status_bits(st2)
    g64 = f64(gd)
    check_gate_values(g64, widened(w)["x"], widened(w)["Wg_t"], np.arange(300, dtype=np.int32))
    assert_twell_matches_oracle(g, g64)


def test_fused_without_dump_matches_dump_run():
    w = synth.make_workload(T=200, d=256, F=512, W=128, C=8, dtype=synth.BF16, kind="dead20",
                            mean_active=29.0, seed=3)
    _, g1, _, y1, _ = run_forward(w, dump=True)
    _, g2, _, y2, _ = run_forward(w, dump=False)
    assert torch.equal(g1.cnt, g2.cnt) and torch.equal(g1.val, g2.val)
    assert torch.equal(y1, y2)


def test_all_inactive_gives_zero():
    # x >= 0 and every gate weight < 0: every pre-activation is negative.
    rng = np.random.default_rng(4)
    w = dict(T=130, d=256, F=512, W=128, C=8, dtype=synth.BF16)
    w["x"] = synth.to_storage(np.abs(rng.standard_normal((130, 256))), synth.BF16)
    w["Wg_t"] = synth.to_storage(-np.abs(rng.standard_normal((512, 256))) / 16 - 1e-3, synth.BF16)
    w["Wu_t"] = synth.to_storage(rng.standard_normal((512, 256)) / 16, synth.BF16)
    w["Wd"] = synth.to_storage(rng.standard_normal((512, 256)) / 16, synth.BF16)
    _, g, gd, y, st = run_forward(w)
    assert int(g.cnt.max().item()) == 0 and int(g.spill_n.item()) == 0
    assert float(y.float().abs().max().item()) == 0.0


def test_spill_capacity_overflow_is_flagged_not_faulted():
    w = synth.make_workload(T=256, d=256, F=512, W=128, C=2, dtype=synth.BF16, kind="dead20",
                            mean_active=60.0, seed=6)
    _, g, gd, y, st = run_forward(w, spill_cap=4)
    need = int(g.spill_n.item())
    assert need > 4
    assert "TW_ERR_SPILL_CAPACITY" in tw.status_bits(st)
    # counts and slots stay exact; the stored spills are a subset of the oracle's
    ref = oracle.twell_encode(f64(gd), 128, 2)
    assert np.array_equal(raw(g.cnt), ref["cnt"])
    assert need == ref["n_spill"]
    assert torch.isfinite(y.float()).all()


def test_oracle_encoded_twell_drives_the_fused_kernel():
    """Consumer-side check of the format contract: TwELL built by the oracle,
    uploaded, and consumed by the fused kernel."""
    w = synth.make_workload(T=150, d=512, F=1024, W=128, C=4, dtype=synth.BF16, kind="dead20",
                            mean_active=40.0, seed=7)
    w64 = widened(w)
    dense = oracle.dense_ffn(w64["x"], w64["Wg_t"], w64["Wu_t"], w64["Wd"])
    g_b = synth.round_bf16(dense["g"])
    enc = oracle.twell_encode(g_b, 128, 4)
    assert enc["n_spill"] > 0
    g = tw.Twell(150, 1024, 4, dtype=torch.bfloat16, spill_cap=enc["n_spill"] + 1)
    bits = lambda a: torch.from_numpy(synth.bf16_bits(a).view(np.int16)).cuda().view(torch.bfloat16)
    g.val.copy_(bits(enc["val"]))
    g.idx.copy_(torch.from_numpy(enc["idx"]))
    g.cnt.copy_(torch.from_numpy(enc["cnt"]))
    g.spill_ref.copy_(torch.from_numpy(enc["spill_ref"]))
    g.spill_val[:enc["n_spill"]].copy_(bits(enc["spill_val"]))
    dev = inputs(w)
    y = torch.empty((150, 512), dtype=torch.float32, device="cuda")
    tw.twell_fused_updown(dev["x"], g, dev["Wu_t"], dev["Wd"], y, tw.fused_workspace(150, 512))
    torch.cuda.synchronize()
    ref = oracle.twell_ffn(w64["x"], enc, w64["Wu_t"], w64["Wd"])
    assert np.max(np.abs(f64(y) - ref)) <= 1e-4 * rms(ref)


@pytest.mark.parametrize("T", [300, 1, 8, 64])  # 1..64: the decode-sized comparator
def test_dense_comparator(T):
    w = synth.make_workload(T=T, d=512, F=1024, W=128, C=8, dtype=synth.BF16, kind="dead20",
                            mean_active=29.0, seed=8)
    dev = inputs(w)
    Wd_dense = dev["Wd"].t().contiguous()
    h = torch.empty((T, 1024), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((T, 512), dtype=torch.bfloat16, device="cuda")
    tw.dense_ffn_forward(dev["x"], dev["Wg_t"], dev["Wu_t"], Wd_dense, h, y)
    torch.cuda.synchronize()
    w64 = widened(w)
    # the comparator stores h and y in bf16, as a dense bf16 FFN does
    dense = oracle.dense_ffn(w64["x"], w64["Wg_t"], w64["Wu_t"], w64["Wd"])
    hr = dense["g"] * dense["u"]
    # h is stored in bf16 (a relative error of at most 2^-9 per element, plus
    # a flip of g near 0); y = h Wd is then stored in bf16
    assert np.all(np.abs(f64(h) - hr) <= 2.0 ** -8 * np.abs(hr) + 1e-4 * rms(hr))
    bound = 2.0 ** -8 * (np.abs(hr) @ np.abs(w64["Wd"])) + 2.0 ** -8 * np.abs(dense["y"])
    assert np.all(np.abs(f64(y) - dense["y"]) <= bound + 1e-2 * rms(dense["y"]))


def test_dense_comparator_2b_shape_sampled():
    w = synth.make_workload("ffn_2b")
    dev = inputs(w)
    T, d, F = w["T"], w["d"], w["F"]
    h = torch.empty((T, F), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    tw.dense_ffn_forward(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"].t().contiguous(), h, y)
    torch.cuda.synchronize()
    rows = synth.subsample_rows(T, 48)
    w64 = widened(w)
    dense = oracle.dense_ffn(w64["x"][rows], w64["Wg_t"], w64["Wu_t"], w64["Wd"])
    hr = dense["g"] * dense["u"]
    bound = 2.0 ** -8 * (np.abs(hr) @ np.abs(w64["Wd"])) + 2.0 ** -8 * np.abs(dense["y"])
    assert np.all(np.abs(f64(y)[rows] - dense["y"]) <= bound + 1e-2 * rms(dense["y"]))


# ----------------------------------------------------- dense training FFN ---
def run_dense_training(w):
    dev = inputs(w)
    T, d, F = w["T"], w["d"], w["F"]
    ws = tw.dense_train_workspace(T, F)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.empty((T, d), dtype=torch.float32, device="cuda")
    dx = torch.empty((T, d), dtype=torch.float32, device="cuda")
    dW = [torch.empty((F, d), dtype=torch.float32, device="cuda") for _ in range(3)]
    tw.dense_ffn_train_forward(dev["x"], dev["Wg_t"], dev["Wu_t"], dev["Wd"], ws, y, st)
    tw.dense_ffn_train_backward(dev["x"], dev["dy"], dev["Wg_t"], dev["Wu_t"], dev["Wd"],
                                w["lam"], ws, dx, dW[0], dW[1], dW[2], st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, tw.status_bits(st)
    g, u, h = tw.dense_train_saved(ws, T, F)
    return f64(g), f64(u), f64(h), f64(y), f64(dx), [f64(a) for a in dW]


def dense_grad_bounds(w64, g64, u64, lam, rows=None, units=None):
    """Elementwise error bounds of the dense training comparator's gradients
    from its own arithmetic: du and dz enter the dx and weight-gradient
    matmuls rounded to bf16 (at most 2^-9 relative each), h enters dWd as
    bf16(g u) with u unrounded, while the conditioned oracle uses g times the
    stored u (two bf16 roundings apart); the fp32 accumulation adds far less.
    Each bound is twice the first-order sum of those roundings, sum |a| |b|
    over the matmul, so (dx, dWg_t, dWu_t, dWd) on the rows / units given."""
    x, dy, Wg, Wu, Wd = (w64[k] for k in ("x", "dy", "Wg_t", "Wu_t", "Wd"))
    if rows is not None:
        x, dy, g64, u64 = x[rows], dy[rows], g64[rows], u64[rows]
    dh = dy @ (Wd if units is None else Wd[units]).T
    if units is not None:
        g64, u64 = g64[:, units], u64[:, units]
    du = np.abs(dh * g64)
    dz = np.abs(np.where(g64 > 0, dh * u64 + lam, 0.0))
    hh = np.abs(g64 * u64)
    if units is None:
        bdx = 2.0 ** -8 * (du @ np.abs(Wu) + dz @ np.abs(Wg))
    else:
        bdx = None
    ax, ady = np.abs(x), np.abs(dy)
    return bdx, 2.0 ** -8 * (dz.T @ ax), 2.0 ** -8 * (du.T @ ax), 2.0 ** -7 * (hh.T @ ady)


def dense_grads_oracle(w64, g64, u64, lam, rows=None, units=None):
    """The oracle's backward conditioned on the GPU's saved g and u: every
    token row with a non-zero g is a dense backup row of a hybrid split with
    C_h = 0, u is kept on the pattern; optionally restricted to token rows
    (exact for dx of those rows) or to units (exact for their weight rows)."""
    x, dy, Wg, Wu, Wd = (w64[k] for k in ("x", "dy", "Wg_t", "Wu_t", "Wd"))
    if rows is not None:
        x, dy, g64, u64 = x[rows], dy[rows], g64[rows], u64[rows]
    if units is not None:
        Wg, Wu, Wd, g64, u64 = Wg[units], Wu[units], Wd[units], g64[:, units], u64[:, units]
    hy = oracle.hybrid_split(g64, 0)
    bu = (u64 * (g64 != 0))[hy["backup_rows"]]
    return oracle.hybrid_backward(x, dy, hy, np.zeros((len(x), 0)), bu, Wg, Wu, Wd, lam)


@pytest.mark.parametrize("T,d,F", [(300, 256, 640), (260, 320, 1024), (128, 64, 128)])
def test_dense_training_comparator(T, d, F):
    """Ragged T (partial 128-row tiles and 64-row k-blocks of the weight
    gradients), F not a multiple of 256, d not a multiple of 256."""
    w = synth.make_workload(T=T, d=d, F=F, W=128, C=8, C_h=64, dtype=synth.BF16, kind="pareto",
                            lam=2e-5, seed=T + F, mean_active=40.0, with_dy=True)
    g, u, h, y, dx, dW = run_dense_training(w)
    w64 = widened(w)
    rows = np.arange(T, dtype=np.int32)
    check_gate_values(g, w64["x"], w64["Wg_t"], rows)
    # u = x Wu rounded once to bf16; h = g u (fp32 u) rounded once to bf16, so
    # against g times the stored u it is off by at most two bf16 roundings
    u_ref = w64["x"] @ w64["Wu_t"].T
    assert np.all(np.abs(u - u_ref) <= 2.0 ** -8 * np.abs(u_ref) + 1e-4 * rms(u_ref))
    assert np.all(np.abs(h - g * u) <= 2.0 ** -7 * np.abs(g * u))
    # y against the fp64 FFN: each term of y rounds h once to bf16 (2^-9 relative)
    out = oracle.dense_ffn(w64["x"], w64["Wg_t"], w64["Wu_t"], w64["Wd"], g_round="bf16")
    bound = 2.0 ** -8 * (np.abs(out["g"] * out["u"]) @ np.abs(w64["Wd"]))
    assert np.all(np.abs(y - out["y"]) <= bound + 1e-2 * rms(out["y"]))
    # gradients: oracle conditioned on the GPU's saved g and u, elementwise
    # within the bf16-operand bound plus 1e-2 rms
    ref = dense_grads_oracle(w64, g, u, w["lam"])
    bnd = dense_grad_bounds(w64, g, u, w["lam"])
    for name, a, b, e in zip(("dx", "dWg_t", "dWu_t", "dWd"), [dx] + dW, ref, bnd):
        viol = np.abs(a - b) - (e + 1e-2 * rms(b))
        assert np.all(viol <= 0), (name, float(np.max(np.abs(a - b))), rms(b), float(viol.max()))


def test_dense_training_comparator_train_2b_sampled():
    """The training workload's full shape (T=8192, d=2048, F=8192): dx on a
    seeded sample of token rows, the weight gradients on a seeded sample of
    units, each exact for the rows / units it covers."""
    w = synth.make_workload("train_2b")
    g, u, h, y, dx, dW = run_dense_training(w)
    w64 = widened(w)
    T, F = w["T"], w["F"]
    rows = synth.subsample_rows(T, 48, seed=11)
    units = synth.subsample_rows(F, 48, seed=12)
    check_gate_values(g, w64["x"], w64["Wg_t"], rows)
    ref_r = dense_grads_oracle(w64, g, u, w["lam"], rows=rows)
    bdx = dense_grad_bounds(w64, g, u, w["lam"], rows=rows)[0]
    assert np.all(np.abs(dx[rows] - ref_r[0]) <= bdx + 1e-2 * rms(ref_r[0]))
    ref_u = dense_grads_oracle(w64, g, u, w["lam"], units=units)
    bnd_u = dense_grad_bounds(w64, g, u, w["lam"], units=units)[1:]
    for name, a, b, e in zip(("dWg_t", "dWu_t", "dWd"), dW, ref_u[1:], bnd_u):
        err = np.abs(a[units] - b)
        assert np.all(err <= e + 1e-2 * rms(b)), (name, float(err.max()), rms(b))
    out = oracle.dense_ffn(w64["x"][rows], w64["Wg_t"], w64["Wu_t"], w64["Wd"], g_round="bf16")
    bound = 2.0 ** -8 * (np.abs(out["g"] * out["u"]) @ np.abs(w64["Wd"]))
    assert np.all(np.abs(y[rows] - out["y"]) <= bound + 1e-2 * rms(out["y"]))


# ----------------------------------------------------------------- hybrid ---
def run_hybrid(w, backup_cap=None):
    T, d, F = w["T"], w["d"], w["F"]
    dev, g, gd, y, st = run_forward(w)
    hy = tw.Hybrid(T, F, w["C_h"], dtype=TDT[w["dtype"]], backup_cap=backup_cap)
    tw.twell_to_hybrid(g, hy, st)
    yh = torch.empty((T, d), dtype=torch.float32, device="cuda")
    tw.hybrid_ffn_forward(dev["x"], hy, dev["Wu_t"], dev["Wd"], yh, dev_status=st)
    hy.ell_u_after_forward = hy.ell_u.clone()  # diagnostics: u before the backward runs
    ws = torch.empty(tw.hybrid_ffn_backward_workspace_size(T, d, F, w["C_h"], hy.backup_cap),
                     dtype=torch.uint8, device="cuda")
    dx = torch.empty((T, d), dtype=torch.float32, device="cuda")  # fp32, like y
    dW = [torch.empty((F, d), dtype=torch.float32, device="cuda") for _ in range(3)]
    tw.hybrid_ffn_backward(dev["x"], dev["dy"], hy, dev["Wg_t"], dev["Wu_t"], dev["Wd"],
                           w["lam"], dx, dW[0], dW[1], dW[2], ws, st)
    torch.cuda.synchronize()
    return dev, g, gd, y, st, hy, yh, dx, dW


def test_hybrid_steps_back_to_back():
    """Whole training steps of two batches (gate, TwELL -> hybrid, forward,
    backward) queued back to back on one stream with shared buffers and
    workspaces: every output equals that of separate, synchronised steps, bit
    for bit (the launches wait for their predecessors' results, and the
    counters and u arrays are cleared by the library's own kernels)."""
    ws_ = [synth.make_workload(T=900, d=256, F=1024, W=128, C=8, C_h=16, dtype=synth.BF16,
                               kind="pareto", lam=2e-5, seed=s_, mean_active=14.0)
           for s_ in (31, 32)]
    T, d, F, C_h = 900, 256, 1024, 16
    devs = [inputs(w) for w in ws_]
    g = tw.Twell(T, F, 8, dtype=torch.bfloat16, spill_cap=(F // 128) * T)
    hy = tw.Hybrid(T, F, C_h, dtype=torch.bfloat16, backup_cap=T)
    bws = torch.empty(tw.hybrid_ffn_backward_workspace_size(T, d, F, C_h, T), dtype=torch.uint8,
                      device="cuda")
    fws = torch.empty(tw.hybrid_ffn_forward_workspace_size(T, d), dtype=torch.uint8,
                      device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(dv, w, outs):
        tw.twell_gate_gemm(dv["x"], dv["Wg_t"], g, None, st)
        tw.twell_to_hybrid(g, hy, st)
        tw.hybrid_ffn_forward(dv["x"], hy, dv["Wu_t"], dv["Wd"], outs[0], fws, st)
        tw.hybrid_ffn_backward(dv["x"], dv["dy"], hy, dv["Wg_t"], dv["Wu_t"], dv["Wd"], w["lam"],
                               outs[1], outs[2], outs[3], outs[4], bws, st)

    def fresh():
        return [torch.empty((T, d), dtype=torch.float32, device="cuda") for _ in range(2)] + \
               [torch.empty((F, d), dtype=torch.float32, device="cuda") for _ in range(3)]

    refs = []
    for dv, w in zip(devs, ws_):  # separate, synchronised steps
        outs = fresh()
        step(dv, w, outs)
        torch.cuda.synchronize()
        refs.append(outs)
    runs = [fresh() for _ in range(4)]
    for i in range(4):  # queued back to back
        step(devs[i % 2], ws_[i % 2], runs[i])
    torch.cuda.synchronize()
    assert int(st.item()) == 0, tw.status_bits(st)
    for i in range(4):
        for a, b in zip(runs[i], refs[i % 2]):
            assert torch.equal(a, b), i


def hybrid_to_np(hy):
    nb = min(int(hy.n_backup.item()), hy.backup_cap)
    return {"T": hy.T, "F": hy.F, "C_h": hy.C_h, "ell_g": f64(hy.ell_g),
            "ell_idx": raw(hy.ell_idx).view(np.uint16), "row_nnz": raw(hy.row_nnz),
            "row_slot": raw(hy.row_slot), "backup_rows": raw(hy.backup_rows)[:nb],
            "backup_g": f64(hy.backup_g)[:nb], "n_backup": int(hy.n_backup.item())}


def check_hybrid_all(w, res):
    dev, g, gd, y, st, hy, yh, dx, dW = res
    assert int(st.item()) == 0, tw.status_bits(st)
    g64 = f64(gd)
    # split: bit-exact against the oracle's split of the GPU's own gate
    ref = oracle.hybrid_split(g64, w["C_h"])
    got = hybrid_to_np(hy)
    assert got["n_backup"] == ref["n_backup"]
    for k in ("row_nnz", "row_slot", "backup_rows"):
        assert np.array_equal(got[k], ref[k]), k
    assert np.array_equal(got["ell_idx"], ref["ell_idx"])
    assert np.array_equal(got["ell_g"].view(np.uint64), ref["ell_g"].view(np.uint64))
    assert np.array_equal(got["backup_g"].view(np.uint64), ref["backup_g"].view(np.uint64))
    # forward: u on the pattern and y, against the oracle on the GPU's pattern
    w64 = widened(w)
    ell_u, backup_u, y_ref = oracle.hybrid_forward(w64["x"], got, w64["Wu_t"], w64["Wd"])
    nb = len(got["backup_g"])
    ug = np.concatenate([f64(hy.ell_u).ravel(), f64(hy.backup_u)[:nb].ravel()])
    ur = np.concatenate([ell_u.ravel(), backup_u.ravel()])
    on = np.concatenate([got["ell_g"].ravel(), got["backup_g"].ravel()]) != 0
    assert np.all(ug[~on] == 0)                       # +0 off the pattern
    viol = np.abs(ug - ur) - (2.0 ** -8 * np.abs(ur) + 1e-3 * rms(ur[on]))
    if np.any(viol > 0):
        i = int(np.argmax(viol))
        n_ell = f64(hy.ell_u).size
        where = (("ell", divmod(i, w["C_h"])) if i < n_ell else ("backup", divmod(i - n_ell, w["F"])))
        bad = np.nonzero(viol[:n_ell] > 0)[0]
        rows_bad = np.unique(bad // w["C_h"])
        u_fwd = f64(hy.ell_u_after_forward).ravel()
        info = [(int(r), int(got["row_nnz"][r]), int(got["row_slot"][r])) for r in rows_bad[:8]]
        yerr = [float(np.max(np.abs(f64(yh)[r] - y_ref[r]))) for r in rows_bad[:8]]
        raise AssertionError(
            f"u mismatch at {where}: gpu {ug[i]} oracle {ur[i]}, {int((viol > 0).sum())} "
            f"violations; rows (t, nnz, slot) {info}; u right after the forward "
            f"{u_fwd[i]}; y row errors {yerr} (rms {rms(y_ref)})")
    tol = TOL[w["dtype"]]
    assert np.max(np.abs(f64(yh) - y_ref)) <= tol * rms(y_ref)
    # the hybrid forward y equals the inference y up to rounding
    assert np.max(np.abs(f64(yh) - f64(y))) <= tol * rms(y_ref)
    # backward, conditioned on the GPU's saved g and u
    got_u = dict(got)
    grads = oracle.hybrid_backward(w64["x"], w64["dy"], got, f64(hy.ell_u),
                                   f64(hy.backup_u)[:nb], w64["Wg_t"], w64["Wu_t"], w64["Wd"],
                                   w["lam"])
    for name, a, b in zip(("dx", "dWg_t", "dWu_t", "dWd"), (dx, dW[0], dW[1], dW[2]), grads):
        err = np.max(np.abs(f64(a) - b))
        assert err <= tol * rms(b), (name, err, rms(b))
    return got_u


def test_hybrid_small_ragged():
    w = synth.make_workload(T=700, d=256, F=1024, W=128, C=8, C_h=16, dtype=synth.BF16,
                            kind="pareto", lam=2e-5, seed=9, mean_active=12.0)
    got = check_hybrid_all(w, run_hybrid(w))
    assert 0 < got["n_backup"] < 700


def test_hybrid_wide_rows():
    # 4 * F bytes of per-warp histograms plus 4 * F bytes of list positions
    # exceed the transposition's shared-memory budget at F = 26624, so the
    # fill reads the positions from global memory instead
    w = synth.make_workload(T=96, d=128, F=26624, W=128, C=8, C_h=16, dtype=synth.BF16,
                            kind="pareto", lam=2e-5, seed=12, mean_active=12.0)
    got = check_hybrid_all(w, run_hybrid(w))
    assert got["n_backup"] > 0


@pytest.mark.parametrize("C_h", [0, 1024])
def test_hybrid_extreme_caps(C_h):
    w = synth.make_workload(T=130, d=128, F=1024, W=128, C=8, C_h=C_h, dtype=synth.BF16,
                            kind="pareto", lam=2e-5, seed=10, mean_active=10.0)
    got = check_hybrid_all(w, run_hybrid(w, backup_cap=130))
    if C_h == 0:
        assert got["n_backup"] == int((got["row_nnz"] > 0).sum())
    else:
        assert got["n_backup"] == 0


def test_hybrid_fp32_small():
    # fp32 activations: fp32 gate on the CUDA cores, fp32 gather engine (FMA dot products)
    w = synth.make_workload(T=150, d=128, F=512, W=128, C=4, C_h=8, dtype=synth.F32,
                            kind="pareto", lam=2e-5, seed=12, mean_active=10.0)
    got = check_hybrid_all(w, run_hybrid(w, backup_cap=150))
    assert 0 < got["n_backup"] < 150


def test_hybrid_bf16_outputs_are_the_fp32_results_rounded():
    w = synth.make_workload(T=300, d=256, F=640, W=128, C=8, C_h=16, dtype=synth.BF16,
                            kind="pareto", lam=2e-5, seed=13, mean_active=14.0)
    T, d, F = w["T"], w["d"], w["F"]
    dev, g, gd, y, st = run_forward(w)
    hy = tw.Hybrid(T, F, w["C_h"], dtype=torch.bfloat16, backup_cap=T)
    tw.twell_to_hybrid(g, hy, st)
    ws = torch.empty(tw.hybrid_ffn_backward_workspace_size(T, d, F, w["C_h"], T),
                     dtype=torch.uint8, device="cuda")
    outs = {}
    for dt in (torch.float32, torch.bfloat16):
        yh = torch.empty((T, d), dtype=dt, device="cuda")
        tw.hybrid_ffn_forward(dev["x"], hy, dev["Wu_t"], dev["Wd"], yh, dev_status=st)
        dx = torch.empty((T, d), dtype=dt, device="cuda")
        dW = [torch.empty((F, d), dtype=torch.float32, device="cuda") for _ in range(3)]
        tw.hybrid_ffn_backward(dev["x"], dev["dy"], hy, dev["Wg_t"], dev["Wu_t"], dev["Wd"],
                               w["lam"], dx, dW[0], dW[1], dW[2], ws, st)
        torch.cuda.synchronize()
        outs[dt] = (yh, dx, dW)
    assert int(st.item()) == 0, tw.status_bits(st)
    y32, dx32, dW32 = outs[torch.float32]
    y16, dx16, dW16 = outs[torch.bfloat16]
    assert torch.equal(y16, y32.to(torch.bfloat16))
    assert torch.equal(dx16, dx32.to(torch.bfloat16))
    for a, b in zip(dW16, dW32):  # the weight gradients do not depend on the dx dtype
        assert torch.equal(a, b)


def test_empty_batch_through_every_entry_point():
    d, F, C, C_h = 256, 512, 8, 16
    rng = np.random.default_rng(14)
    bf = lambda a: torch.from_numpy(synth.to_storage(a, synth.BF16).view(np.int16)).cuda().view(
        torch.bfloat16)
    x = torch.empty((0, d), dtype=torch.bfloat16, device="cuda")
    Wg, Wu, Wd = (bf(rng.standard_normal((F, d)) / 16) for _ in range(3))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = tw.Twell(0, F, C, dtype=torch.bfloat16)
    tw.twell_gate_gemm(x, Wg, g, None, st)
    y = torch.empty((0, d), dtype=torch.float32, device="cuda")
    tw.twell_fused_updown(x, g, Wu, Wd, y, tw.fused_workspace(0, d), st)
    hy = tw.Hybrid(0, F, C_h, dtype=torch.bfloat16, backup_cap=4)
    tw.twell_to_hybrid(g, hy, st)
    tw.hybrid_ffn_forward(x, hy, Wu, Wd, y, dev_status=st)
    ws = torch.empty(max(1, tw.hybrid_ffn_backward_workspace_size(0, d, F, C_h, 4)),
                     dtype=torch.uint8, device="cuda")
    dW = [torch.full((F, d), 7.0, dtype=torch.float32, device="cuda") for _ in range(3)]
    tw.hybrid_ffn_backward(x, x, hy, Wg, Wu, Wd, 2e-5, y, dW[0], dW[1], dW[2], ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert int(g.spill_n.item()) == 0 and int(hy.n_backup.item()) == 0
    for a in dW:  # no tokens: the weight gradients are zero, not left unwritten
        assert float(a.abs().max().item()) == 0.0


def test_hybrid_backup_capacity_overflow_is_flagged():
    w = synth.make_workload(T=256, d=128, F=512, W=128, C=8, C_h=2, dtype=synth.BF16,
                            kind="pareto", lam=2e-5, seed=11, mean_active=10.0)
    dev, g, gd, y, st = run_forward(w)
    hy = tw.Hybrid(256, 512, 2, dtype=torch.bfloat16, backup_cap=3)
    tw.twell_to_hybrid(g, hy, st)
    torch.cuda.synchronize()
    assert int(hy.n_backup.item()) > 3
    assert "TW_ERR_BACKUP_CAPACITY" in tw.status_bits(st)
    # the forward still runs on what was stored: u is cleared in the 3 stored
    # backup rows (and no further) and is +0 wherever g is
    hy.backup_u.view(torch.int16).fill_(0x3F80)  # bf16 1.0 everywhere beforehand
    yh = torch.empty((256, 128), dtype=torch.float32, device="cuda")
    tw.hybrid_ffn_forward(dev["x"], hy, dev["Wu_t"], dev["Wd"], yh, dev_status=st)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(yh).all())
    bg, bu = f64(hy.backup_g), f64(hy.backup_u)
    assert np.all(bu[:3][bg[:3] == 0] == 0)


def test_training_config_full_size():
    w = synth.make_workload("train_2b")
    res = run_hybrid(w, backup_cap=2048)
    got = check_hybrid_all(w, res)
    assert got["n_backup"] > 0


def _splitmix64(x):
    """splitmix64 (Steele, Lea and Flood, 2014) on uint64 arrays, mod 2^64."""
    with np.errstate(over="ignore"):
        z = x + np.uint64(0x9E3779B97F4A7C15)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


@pytest.mark.parametrize("rows,d,n", [(1000, 2048, 3001), (77, 520, 500), (5, 8, 1)])
def test_row_gather_measurement_reads_the_rows_it_names(rows, d, n):
    """The roofline's row-gather measurement reads row splitmix64((seed << 32)
    ^ i) mod rows in full for every i < n: the XOR of all words read equals the
    host's, for ragged d (chunks past the last lane round) and an odd n."""
    rng = np.random.default_rng(rows + d)
    bits = rng.integers(-32768, 32767, size=(rows, d), dtype=np.int16)
    mat = torch.from_numpy(bits).cuda().view(torch.bfloat16)
    chk = torch.zeros(1, dtype=torch.int32, device="cuda")
    seed = 7
    tw.measure_row_gather(mat, n, seed, chk)
    torch.cuda.synchronize()
    idx = np.arange(n, dtype=np.uint64) ^ (np.uint64(seed) << np.uint64(32))
    sel = (_splitmix64(idx) % np.uint64(rows)).astype(np.int64)
    words = bits.view(np.uint32)[sel]
    want = np.bitwise_xor.reduce(words.ravel()) if words.size else np.uint32(0)
    assert int(chk.item()) & 0xFFFFFFFF == int(want)


@pytest.mark.parametrize("nbytes", [16, 4096 + 48, 33554432 + 1024 * 16 + 16])
def test_stream_read_measurement_reads_every_word(nbytes):
    """The stream-read floor reads every 16-byte chunk once: the XOR of all words
    equals the host's, for sizes below one grid pass, with a ragged tail after
    the eight-deep rounds, and at the gate's 33.5 MB plus a tail."""
    rng = np.random.default_rng(nbytes)
    words = rng.integers(0, 2**32, size=nbytes // 4, dtype=np.uint64).astype(np.uint32)
    buf = torch.from_numpy(words.view(np.int32)).cuda()
    chk = torch.zeros(1, dtype=torch.int32, device="cuda")
    tw.measure_stream_read(buf, chk)
    torch.cuda.synchronize()
    assert int(chk.item()) & 0xFFFFFFFF == int(np.bitwise_xor.reduce(words))
