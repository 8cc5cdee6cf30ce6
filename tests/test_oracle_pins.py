"""Pins of the CPU oracle against facts fixed independently of its own code.

The pages print no worked example, so each function is pinned by at least one
of: a hand-worked fixture (tests/golden/), an exact round trip, an invariant
(counts sum to nnz), a closed form (one active unit), a special case that
reduces to a library routine (dense fp64 matmuls), central finite differences
of the loss, and torch fp64 autograd.  All of these run on the CPU.
"""
import numpy as np
import pytest

import oracle
from golden_io import matrix, read, scalar

RNG = np.random.default_rng(12345)


def sparse_gate(T, F, density, rng=RNG, scale=1.0):
    """A random non-negative g with about `density` non-zeros (no -0)."""
    g = np.abs(rng.standard_normal((T, F))) * scale + 0.01
    mask = rng.random((T, F)) < density
    return np.where(mask, g, 0.0)


def bits(a):
    return np.ascontiguousarray(a, dtype=np.float64).view(np.uint64)


# ------------------------------------------------------------------ TwELL ---
def test_twell_golden_hand_worked():
    fx = read("twell_w4_c2.txt")
    W, C = int(scalar(fx, "W")), int(scalar(fx, "C"))
    g = matrix(fx, "g")
    tw = oracle.twell_encode(g, W, C)
    for k, t, cnt, v0, v1, i0, i1 in fx["tw"]:
        k, t = int(k), int(t)
        assert tw["cnt"][k, t] == cnt
        assert list(tw["val"][k, t]) == [v0, v1]
        assert list(tw["idx"][k, t]) == [i0, i1]
    assert tw["n_spill"] == len(fx["spill"])
    for (t, k, *seg), tk, sv in zip(fx["spill"], tw["spill_tk"], tw["spill_val"]):
        assert (tk[0], tk[1]) == (int(t), int(k))
        assert list(sv) == seg
        assert tw["spill_ref"][int(k), int(t)] >= 0
    assert np.array_equal(oracle.twell_decode(tw), g)


@pytest.mark.parametrize("W,C", [(4, 0), (4, 1), (4, 2), (4, 4), (8, 3), (128, 8), (128, 16),
                                 (128, 128)])
@pytest.mark.parametrize("density", [0.0, 0.05, 0.3, 1.0])
def test_twell_round_trip_and_invariants(W, C, density):
    T, F = 7, 4 * W
    g = sparse_gate(T, F, density)
    tw = oracle.twell_encode(g, W, C)
    # decode(encode(g)) == g, bit for bit
    assert np.array_equal(bits(oracle.twell_decode(tw)), bits(g))
    # per-tile counts sum to the number of non-zeros
    assert int(tw["cnt"].astype(np.int64).sum()) == int((g != 0).sum())
    K = F // W
    seg = g.reshape(T, K, W)
    n_spill = 0
    for k in range(K):
        for t in range(T):
            nz = np.nonzero(seg[t, k])[0]
            assert tw["cnt"][k, t] == len(nz)
            m = min(len(nz), C)
            # first min(cnt, C) non-zeros in ascending column order
            assert list(tw["idx"][k, t, :m]) == list(nz[:m])
            assert np.array_equal(tw["val"][k, t, :m], seg[t, k, nz[:m]])
            # padding is (+0, 0)
            assert np.all(bits(tw["val"][k, t, m:]) == 0)
            assert np.all(tw["idx"][k, t, m:] == 0)
            if len(nz) > C:
                r = tw["spill_ref"][k, t]
                assert tuple(tw["spill_tk"][r]) == (t, k)
                assert np.array_equal(tw["spill_val"][r], seg[t, k])
                n_spill += 1
            else:
                assert tw["spill_ref"][k, t] == -1
    assert tw["n_spill"] == n_spill


def test_twell_capacity_special_cases():
    T, W = 5, 16
    g = sparse_gate(T, 4 * W, 0.4)
    # C >= W: slots hold the whole tile's non-zeros, nothing spills
    full = oracle.twell_encode(g, W, W)
    assert full["n_spill"] == 0
    # C = 0: every non-empty (t,k) spills
    none = oracle.twell_encode(g, W, 0)
    assert none["n_spill"] == int((full["cnt"] > 0).sum())
    # all-zero gate: all counts zero, nothing spills, decode is zero
    z = oracle.twell_encode(np.zeros((T, 4 * W)), W, 3)
    assert z["cnt"].max() == 0 and z["n_spill"] == 0
    # spill capacity smaller than needed: the true need is still reported
    part = oracle.twell_encode(g, W, 0, spill_cap=2)
    assert part["n_spill"] == none["n_spill"] and len(part["spill_tk"]) == 2


# -------------------------------------------------------------- dense FFN ---
def _one_unit():
    fx = read("ffn_one_unit.txt")
    return (fx, matrix(fx, "x"), matrix(fx, "Wg_t"), matrix(fx, "Wu_t"),
            matrix(fx, "Wd"))


def test_dense_ffn_one_active_unit_closed_form():
    fx, x, Wg_t, Wu_t, Wd = _one_unit()
    out = oracle.dense_ffn(x, Wg_t, Wu_t, Wd)
    assert np.array_equal(out["y"], matrix(fx, "y"))
    assert np.array_equal(out["g"][0], [1.0, 0.0, 0.0, 0.0])
    assert out["u"][0, 0] == 3.0


def test_dense_backward_one_active_unit_closed_form():
    fx, x, Wg_t, Wu_t, Wd = _one_unit()
    dy = matrix(fx, "dy")
    lam = scalar(fx, "lambda")
    dx, dWg, dWu, dWd = oracle.dense_ffn_backward(x, Wg_t, Wu_t, Wd, dy, lam)
    assert np.array_equal(dx, matrix(fx, "dx"))
    assert np.array_equal(dWd[0], matrix(fx, "dWd0")[0])
    assert np.array_equal(dWu[0], matrix(fx, "dWu_t0")[0])
    assert np.array_equal(dWg[0], matrix(fx, "dWg_t0")[0])
    for a in (dWd, dWu, dWg):
        assert np.all(a[1:] == 0.0)


def _rand_problem(T, d, F, rng, bias=0.0):
    x = rng.standard_normal((T, d))
    Wg_t = rng.standard_normal((F, d)) / np.sqrt(d)
    Wu_t = rng.standard_normal((F, d)) / np.sqrt(d)
    Wd = rng.standard_normal((F, d)) / np.sqrt(F)
    x[:, 0] = 1.0
    Wg_t[:, 0] = -bias
    return x, Wg_t, Wu_t, Wd


def test_dense_ffn_matches_numpy_matmuls():
    rng = np.random.default_rng(7)
    x, Wg_t, Wu_t, Wd = _rand_problem(9, 24, 40, rng, bias=0.5)
    out = oracle.dense_ffn(x, Wg_t, Wu_t, Wd)
    z = x @ Wg_t.T
    assert np.allclose(out["z"], z, rtol=1e-13, atol=1e-13)
    assert np.allclose(out["u"], x @ Wu_t.T, rtol=1e-13, atol=1e-13)
    assert np.allclose(out["y"], (np.maximum(z, 0) * (x @ Wu_t.T)) @ Wd, rtol=1e-12, atol=1e-13)
    assert np.all(out["g"] >= 0) and np.all((out["g"] == 0) == (z <= 0))


def test_gate_rows_matches_dense():
    rng = np.random.default_rng(8)
    x, Wg_t, Wu_t, Wd = _rand_problem(12, 16, 32, rng, bias=0.3)
    rows = np.array([0, 5, 11], np.int32)
    g = oracle.gate_rows(x, Wg_t, rows)
    assert np.array_equal(g, oracle.dense_ffn(x, Wg_t, Wu_t, Wd)["g"][rows])


@pytest.mark.parametrize("W,C", [(4, 1), (8, 2), (16, 16)])
def test_twell_ffn_equals_dense_ffn(W, C):
    rng = np.random.default_rng(W * 100 + C)
    x, Wg_t, Wu_t, Wd = _rand_problem(11, 20, 4 * W, rng, bias=1.0)
    dense = oracle.dense_ffn(x, Wg_t, Wu_t, Wd)
    tw = oracle.twell_encode(dense["g"], W, C)
    y = oracle.twell_ffn(x, tw, Wu_t, Wd)
    scale = np.sqrt(np.mean(dense["y"] ** 2))
    assert np.max(np.abs(y - dense["y"])) <= 1e-12 * scale


# ------------------------------------------------------------------ hybrid ---
def test_hybrid_golden_hand_worked():
    fx = read("twell_w4_c2.txt")
    C_h = int(scalar(fx, "C_h"))
    g = matrix(fx, "g")
    hy = oracle.hybrid_split(g, C_h)
    for t, nnz, slot, v0, v1, i0, i1 in fx["row"]:
        t = int(t)
        assert hy["row_nnz"][t] == nnz and hy["row_slot"][t] == slot
        assert list(hy["ell_g"][t]) == [v0, v1] and list(hy["ell_idx"][t]) == [i0, i1]
    assert hy["n_backup"] == len(fx["backup"])
    for slot, t in fx["backup"]:
        assert hy["backup_rows"][int(slot)] == t
        assert np.array_equal(hy["backup_g"][int(slot)], g[int(t)])
    assert np.array_equal(oracle.hybrid_decode(hy), g)


@pytest.mark.parametrize("C_h", [0, 1, 3, 8, 64])
def test_hybrid_split_invariants(C_h):
    T, F = 13, 64
    g = sparse_gate(T, F, 0.08)
    g[3] = 0.0                       # an empty row
    g[4, :20] = 1.25                 # a crowded row
    hy = oracle.hybrid_split(g, C_h)
    nnz = (g != 0).sum(1)
    assert np.array_equal(hy["row_nnz"], nnz)
    backup = np.nonzero(nnz > C_h)[0]
    assert np.array_equal(hy["backup_rows"], backup)            # ascending token order
    assert np.array_equal(hy["row_slot"][backup], np.arange(len(backup)))
    assert np.all(hy["row_slot"][nnz <= C_h] == -1)
    for t in np.nonzero(nnz <= C_h)[0]:
        nz = np.nonzero(g[t])[0]
        assert list(hy["ell_idx"][t, :len(nz)]) == list(nz)
        assert np.all(bits(hy["ell_g"][t, len(nz):]) == 0) and np.all(hy["ell_idx"][t, len(nz):] == 0)
    assert np.array_equal(bits(oracle.hybrid_decode(hy)), bits(g))
    if C_h == 0:
        assert hy["n_backup"] == int((nnz > 0).sum())
    if C_h >= F:
        assert hy["n_backup"] == 0


def test_hybrid_split_no_backup_when_cap_is_F():
    g = sparse_gate(6, 32, 0.9)
    assert oracle.hybrid_split(g, 32)["n_backup"] == 0


def test_hybrid_forward_equals_dense():
    rng = np.random.default_rng(21)
    x, Wg_t, Wu_t, Wd = _rand_problem(10, 16, 48, rng, bias=0.6)
    dense = oracle.dense_ffn(x, Wg_t, Wu_t, Wd)
    C_h = int(np.median((dense["g"] != 0).sum(1)))
    hy = oracle.hybrid_split(dense["g"], C_h)
    assert 0 < hy["n_backup"] < 10
    ell_u, backup_u, y = oracle.hybrid_forward(x, hy, Wu_t, Wd)
    scale = np.sqrt(np.mean(dense["y"] ** 2))
    assert np.max(np.abs(y - dense["y"])) <= 1e-12 * scale
    for t in range(10):
        on = dense["g"][t] != 0
        if hy["row_slot"][t] < 0:
            n = on.sum()
            assert np.allclose(ell_u[t, :n], dense["u"][t, on], rtol=1e-13, atol=1e-14)
            assert np.all(ell_u[t, n:] == 0)
        else:
            b = backup_u[hy["row_slot"][t]]
            assert np.allclose(b[on], dense["u"][t, on], rtol=1e-13, atol=1e-14)
            assert np.all(b[~on] == 0)
            # a backup row has no ELL entries: its ELL u slots are +0
            assert np.all(ell_u[t].view(np.uint64) == 0)


# ---------------------------------------------------------------- backward ---
def _loss(x, Wg_t, Wu_t, Wd, dy, lam):
    out = oracle.dense_ffn(x, Wg_t, Wu_t, Wd)
    return float(np.sum(out["y"] * dy) + lam * np.sum(out["g"]))


def test_dense_backward_matches_central_differences():
    rng = np.random.default_rng(3)
    T, d, F, lam = 3, 5, 12, 0.3
    for _ in range(50):               # keep every pre-activation away from the kink
        x, Wg_t, Wu_t, Wd = _rand_problem(T, d, F, rng, bias=0.2)
        if np.min(np.abs(oracle.dense_ffn(x, Wg_t, Wu_t, Wd)["z"])) > 2e-2:
            break
    dy = rng.standard_normal((T, d))
    grads = oracle.dense_ffn_backward(x, Wg_t, Wu_t, Wd, dy, lam)
    params = [x, Wg_t, Wu_t, Wd]
    h = 1e-6
    for p_i, (p, gr) in enumerate(zip(params, grads)):
        fd = np.empty_like(p)
        for idx in np.ndindex(p.shape):
            old = p[idx]
            p[idx] = old + h
            lp = _loss(*params, dy, lam)
            p[idx] = old - h
            lm = _loss(*params, dy, lam)
            p[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        assert np.allclose(gr, fd, rtol=1e-6, atol=1e-7), p_i


def test_dense_backward_matches_torch_autograd():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(4)
    x, Wg_t, Wu_t, Wd = _rand_problem(6, 8, 24, rng, bias=0.4)
    dy = rng.standard_normal((6, 8))
    lam = 2e-2
    # exact zeros in z exercise the ReLU'(0) = 0 and sign(0) = 0 conventions
    Wg_t[5, 1:] = 0.0
    Wg_t[5, 0] = 0.0
    tx, tg, tu, td = (torch.tensor(a, requires_grad=True) for a in (x, Wg_t, Wu_t, Wd))
    z = tx @ tg.T
    g = torch.relu(z)
    y = (g * (tx @ tu.T)) @ td
    L = (y * torch.tensor(dy)).sum() + lam * g.abs().sum()
    L.backward()
    ours = oracle.dense_ffn_backward(x, Wg_t, Wu_t, Wd, dy, lam)
    for a, b in zip(ours, (tx.grad, tg.grad, tu.grad, td.grad)):
        assert np.allclose(a, b.numpy(), rtol=1e-12, atol=1e-13)


def test_hybrid_backward_equals_dense_backward():
    rng = np.random.default_rng(5)
    x, Wg_t, Wu_t, Wd = _rand_problem(12, 16, 40, rng, bias=0.7)
    dy = rng.standard_normal((12, 16))
    lam = 2e-5
    dense = oracle.dense_ffn(x, Wg_t, Wu_t, Wd)
    C_h = int(np.median((dense["g"] != 0).sum(1)))
    hy = oracle.hybrid_split(dense["g"], C_h)
    assert 0 < hy["n_backup"] < 12
    ell_u, backup_u, _ = oracle.hybrid_forward(x, hy, Wu_t, Wd)
    ours = oracle.hybrid_backward(x, dy, hy, ell_u, backup_u, Wg_t, Wu_t, Wd, lam)
    ref = oracle.dense_ffn_backward(x, Wg_t, Wu_t, Wd, dy, lam)
    for a, b in zip(ours, ref):
        s = np.sqrt(np.mean(b ** 2))
        assert np.max(np.abs(a - b)) <= 1e-12 * s


def test_all_inactive_gives_zero_output_and_only_zero_grads():
    rng = np.random.default_rng(6)
    x, Wg_t, Wu_t, Wd = _rand_problem(4, 8, 16, rng, bias=1e4)
    out = oracle.dense_ffn(x, Wg_t, Wu_t, Wd)
    assert np.all(out["g"] == 0) and np.all(out["y"] == 0)
    tw = oracle.twell_encode(out["g"], 8, 2)
    assert tw["cnt"].max() == 0
    dy = rng.standard_normal((4, 8))
    for a in oracle.dense_ffn_backward(x, Wg_t, Wu_t, Wd, dy, 0.1):
        assert np.all(a == 0)


# ------------------------------------------------------------ rounding -----
def test_storage_rounding_bf16_hand_worked_ties():
    # bf16 keeps 8 significant bits: the spacing just above 1 is 2^-7.
    cases = [
        (1.0, 1.0),
        (1.0 + 2.0 ** -8, 1.0),                        # halfway, ties to even (down)
        (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),        # halfway, ties to even (up)
        (1.0 + 2.0 ** -8 + 2.0 ** -30, 1.0 + 2.0 ** -7),  # just above halfway
        (-(1.0 + 2.0 ** -8 - 2.0 ** -30), -1.0),       # just below halfway, negative
        (3.14159, 3.140625),                           # 3.140625 = 201 * 2^-6
        (0.0, 0.0),
        (2.0 ** -100 * 1.5, 2.0 ** -100 * 1.5),        # exactly representable
    ]
    for v, r in cases:
        assert oracle.round_storage(v, "bf16") == r, v
    assert oracle.round_storage(1.0 + 2.0 ** -30, "f32") == 1.0
    assert oracle.round_storage(1.0 + 2.0 ** -23, "f32") == 1.0 + 2.0 ** -23


def test_storage_rounding_matches_independent_generator_rounding():
    from activation_sparse_transformer_tma_b200 import synth
    v = np.random.default_rng(0).standard_normal(2000) * 10.0 ** np.random.default_rng(1).uniform(-6, 6, 2000)
    ours = np.array([oracle.round_storage(a, "bf16") for a in v])
    assert np.array_equal(ours, synth.round_bf16(v))


def test_dense_ffn_rounds_only_g():
    rng = np.random.default_rng(9)
    x, Wg_t, Wu_t, Wd = _rand_problem(5, 16, 24, rng, bias=0.3)
    exact = oracle.dense_ffn(x, Wg_t, Wu_t, Wd)
    rounded = oracle.dense_ffn(x, Wg_t, Wu_t, Wd, g_round="bf16")
    gb = np.vectorize(lambda a: oracle.round_storage(a, "bf16"))(exact["g"])
    assert np.array_equal(rounded["g"], gb)
    assert np.array_equal(rounded["u"], exact["u"]) and np.array_equal(rounded["z"], exact["z"])
    assert np.allclose(rounded["y"], (gb * exact["u"]) @ Wd, rtol=1e-12, atol=1e-14)
    g_rows = oracle.gate_rows(x, Wg_t, np.array([1, 3], np.int32), g_round="bf16")
    assert np.array_equal(g_rows, gb[[1, 3]])
