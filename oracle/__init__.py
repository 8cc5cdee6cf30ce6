"""CPU oracle for the activation-sparse gated FFN and the TwELL / hybrid formats.

TEST INFRASTRUCTURE ONLY.  This package is imported by the tests, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py`` and by
nothing else.  It shares no code with the CUDA library: the arithmetic lives in
``twell_oracle.c`` (plain single-threaded fp64 C); this file only marshals
numpy arrays through ctypes.

Method source: technical summary page of "Sparser, Faster, Lighter Transformer
Language Models" (arXiv 2603.23198), sections 2.1 (TwELL), 2.2 (fused
inference), 2.3 (hybrid format), 2.4 (training kernels, L1 term).

Every function here is pinned by ``tests/test_oracle_pins.py`` against facts
fixed independently of this code (round trips, invariants, closed forms,
finite differences, torch fp64 autograd, a hand-worked golden example).  The
pages print no worked example, so no pin comes from values printed there.
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        D = ctypes.POINTER(ctypes.c_double)
        U8 = ctypes.POINTER(ctypes.c_uint8)
        U16 = ctypes.POINTER(ctypes.c_uint16)
        I32 = ctypes.POINTER(ctypes.c_int32)
        i = ctypes.c_int
        lib.orc_round_storage.argtypes = [ctypes.c_double, i]
        lib.orc_round_storage.restype = ctypes.c_double
        lib.orc_dense_ffn.argtypes = [i, i, i, D, D, D, D, i, D, D, D, D]
        lib.orc_dense_ffn.restype = None
        lib.orc_gate_rows.argtypes = [i, I32, i, i, D, D, i, D]
        lib.orc_gate_rows.restype = None
        lib.orc_twell_encode.argtypes = [i, i, i, i, D, D, U8, U8, I32,
                                         ctypes.c_int32, I32, D]
        lib.orc_twell_encode.restype = ctypes.c_int32
        lib.orc_twell_decode.argtypes = [i, i, i, i, D, U8, U8, I32, D, D]
        lib.orc_twell_decode.restype = None
        lib.orc_twell_ffn.argtypes = [i, i, i, i, i, D, D, U8, U8, I32, D, D, D, D]
        lib.orc_twell_ffn.restype = None
        lib.orc_hybrid_split.argtypes = [i, i, i, D, D, U16, I32, I32,
                                         ctypes.c_int32, I32, D]
        lib.orc_hybrid_split.restype = ctypes.c_int32
        lib.orc_hybrid_decode.argtypes = [i, i, i, D, U16, I32, D, D]
        lib.orc_hybrid_decode.restype = None
        lib.orc_hybrid_forward.argtypes = [i, i, i, i, D, D, U16, I32, D, D, D,
                                           D, D, D]
        lib.orc_hybrid_forward.restype = None
        lib.orc_hybrid_backward.argtypes = [i, i, i, i, D, D, D, D, U16, I32, D,
                                            D, D, D, D, ctypes.c_double, D, D, D, D]
        lib.orc_hybrid_backward.restype = None
        lib.orc_dense_ffn_backward.argtypes = [i, i, i, D, D, D, D, D,
                                               ctypes.c_double, D, D, D, D]
        lib.orc_dense_ffn_backward.restype = None
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a, ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _pd(a):
    return _p(a, ctypes.c_double)


ROUND = {None: 0, "f64": 0, "bf16": 1, "f32": 2}


def round_storage(v, dtype):
    """Round one fp64 value to the storage dtype ('bf16', 'f32' or None)."""
    return _load().orc_round_storage(float(v), ROUND[dtype])


def dense_ffn(x, Wg_t, Wu_t, Wd, g_round=None):
    """Plain dense FFN in fp64 with g rounded to its storage dtype g_round
    (None, 'bf16' or 'f32').  Returns dict z, g, u (all [T,F]) and y [T,d]."""
    x, Wg_t, Wu_t, Wd = map(_f64, (x, Wg_t, Wu_t, Wd))
    T, d = x.shape
    F = Wg_t.shape[0]
    assert Wg_t.shape == (F, d) and Wu_t.shape == (F, d) and Wd.shape == (F, d)
    z = np.empty((T, F)); g = np.empty((T, F)); u = np.empty((T, F)); y = np.empty((T, d))
    _load().orc_dense_ffn(T, d, F, _pd(x), _pd(Wg_t), _pd(Wu_t), _pd(Wd), ROUND[g_round],
                          _pd(z), _pd(g), _pd(u), _pd(y))
    return {"z": z, "g": g, "u": u, "y": y}


def gate_rows(x, Wg_t, rows, g_round=None):
    """g = relu(x[rows] Wg) in fp64, rounded to g_round, [len(rows), F]."""
    x, Wg_t = _f64(x), _f64(Wg_t)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    d = x.shape[1]
    F = Wg_t.shape[0]
    g = np.empty((len(rows), F))
    _load().orc_gate_rows(len(rows), _p(rows, ctypes.c_int32), d, F, _pd(x),
                          _pd(Wg_t), ROUND[g_round], _pd(g))
    return g


def twell_encode(g, W, C, spill_cap=None):
    """TwELL encoding of a dense [T,F] g.  Arrays are tile-major ([K,T,...]).

    spill_ref holds -1 where (t,k) did not overflow.  n_spill is the number of
    spill entries the input needs (entries past spill_cap are not stored).
    """
    g = _f64(g)
    T, F = g.shape
    assert F % W == 0
    K = F // W
    if spill_cap is None:
        spill_cap = K * T
    val = np.empty((K, T, C)); idx = np.empty((K, T, C), np.uint8)
    cnt = np.empty((K, T), np.uint8); spill_ref = np.full((K, T), -1, np.int32)
    spill_tk = np.zeros((max(spill_cap, 1), 2), np.int32)
    spill_val = np.zeros((max(spill_cap, 1), W))
    n = _load().orc_twell_encode(T, F, W, C, _pd(g), _pd(val), _p(idx, ctypes.c_uint8),
                                 _p(cnt, ctypes.c_uint8), _p(spill_ref, ctypes.c_int32),
                                 spill_cap, _p(spill_tk, ctypes.c_int32), _pd(spill_val))
    m = min(n, spill_cap)
    return {"T": T, "F": F, "W": W, "C": C, "val": val, "idx": idx, "cnt": cnt,
            "spill_ref": spill_ref, "spill_tk": spill_tk[:m].copy(),
            "spill_val": spill_val[:m].copy(), "n_spill": int(n)}


def twell_decode(tw):
    T, F, W, C = tw["T"], tw["F"], tw["W"], tw["C"]
    val = _f64(tw["val"]); idx = np.ascontiguousarray(tw["idx"], np.uint8)
    cnt = np.ascontiguousarray(tw["cnt"], np.uint8)
    sref = np.ascontiguousarray(tw["spill_ref"], np.int32)
    sval = _f64(tw["spill_val"]) if len(tw["spill_val"]) else np.zeros((1, W))
    g = np.empty((T, F))
    _load().orc_twell_decode(T, F, W, C, _pd(val), _p(idx, ctypes.c_uint8),
                             _p(cnt, ctypes.c_uint8), _p(sref, ctypes.c_int32),
                             _pd(sval), _pd(g))
    return g


def twell_ffn(x, tw, Wu_t, Wd):
    """y from the TwELL gate by iterating over the active units only."""
    x, Wu_t, Wd = map(_f64, (x, Wu_t, Wd))
    T, F, W, C = tw["T"], tw["F"], tw["W"], tw["C"]
    d = x.shape[1]
    assert x.shape[0] == T
    val = _f64(tw["val"]); idx = np.ascontiguousarray(tw["idx"], np.uint8)
    cnt = np.ascontiguousarray(tw["cnt"], np.uint8)
    sref = np.ascontiguousarray(tw["spill_ref"], np.int32)
    sval = _f64(tw["spill_val"]) if len(tw["spill_val"]) else np.zeros((1, W))
    y = np.empty((T, d))
    _load().orc_twell_ffn(T, d, F, W, C, _pd(x), _pd(val), _p(idx, ctypes.c_uint8),
                          _p(cnt, ctypes.c_uint8), _p(sref, ctypes.c_int32), _pd(sval),
                          _pd(Wu_t), _pd(Wd), _pd(y))
    return y


def hybrid_split(g, C_h, backup_cap=None):
    """Hybrid split of a dense [T,F] g: ELL rows (nnz <= C_h) and backup rows."""
    g = _f64(g)
    T, F = g.shape
    if backup_cap is None:
        backup_cap = T
    ell_g = np.empty((T, max(C_h, 0))); ell_idx = np.empty((T, max(C_h, 0)), np.uint16)
    row_nnz = np.empty(T, np.int32); row_slot = np.empty(T, np.int32)
    backup_rows = np.zeros(max(backup_cap, 1), np.int32)
    backup_g = np.zeros((max(backup_cap, 1), F))
    n = _load().orc_hybrid_split(T, F, C_h, _pd(g), _pd(ell_g), _p(ell_idx, ctypes.c_uint16),
                                 _p(row_nnz, ctypes.c_int32), _p(row_slot, ctypes.c_int32),
                                 backup_cap, _p(backup_rows, ctypes.c_int32), _pd(backup_g))
    m = min(n, backup_cap)
    return {"T": T, "F": F, "C_h": C_h, "ell_g": ell_g, "ell_idx": ell_idx,
            "row_nnz": row_nnz, "row_slot": row_slot,
            "backup_rows": backup_rows[:m].copy(), "backup_g": backup_g[:m].copy(),
            "n_backup": int(n)}


def hybrid_decode(hy):
    T, F, C_h = hy["T"], hy["F"], hy["C_h"]
    bg = _f64(hy["backup_g"]) if len(hy["backup_g"]) else np.zeros((1, F))
    g = np.empty((T, F))
    _load().orc_hybrid_decode(T, F, C_h, _pd(_f64(hy["ell_g"])),
                              _p(np.ascontiguousarray(hy["ell_idx"], np.uint16), ctypes.c_uint16),
                              _p(np.ascontiguousarray(hy["row_slot"], np.int32), ctypes.c_int32),
                              _pd(bg), _pd(g))
    return g


def hybrid_forward(x, hy, Wu_t, Wd):
    """u sampled on the hybrid pattern and y = (g*u) Wd.  Returns (ell_u, backup_u, y)."""
    x, Wu_t, Wd = map(_f64, (x, Wu_t, Wd))
    T, F, C_h = hy["T"], hy["F"], hy["C_h"]
    d = x.shape[1]
    nb = max(len(hy["backup_g"]), 1)
    bg = _f64(hy["backup_g"]) if len(hy["backup_g"]) else np.zeros((1, F))
    ell_u = np.empty((T, C_h)); backup_u = np.zeros((nb, F)); y = np.empty((T, d))
    _load().orc_hybrid_forward(T, d, F, C_h, _pd(x), _pd(_f64(hy["ell_g"])),
                               _p(np.ascontiguousarray(hy["ell_idx"], np.uint16), ctypes.c_uint16),
                               _p(np.ascontiguousarray(hy["row_slot"], np.int32), ctypes.c_int32),
                               _pd(bg), _pd(Wu_t), _pd(Wd), _pd(ell_u), _pd(backup_u), _pd(y))
    return ell_u, backup_u[:len(hy["backup_g"])].copy(), y


def hybrid_backward(x, dy, hy, ell_u, backup_u, Wg_t, Wu_t, Wd, lam):
    """Gradients from the saved hybrid g and u.  Returns (dx, dWg_t, dWu_t, dWd)."""
    x, dy, Wg_t, Wu_t, Wd = map(_f64, (x, dy, Wg_t, Wu_t, Wd))
    T, F, C_h = hy["T"], hy["F"], hy["C_h"]
    d = x.shape[1]
    bg = _f64(hy["backup_g"]) if len(hy["backup_g"]) else np.zeros((1, F))
    bu = _f64(backup_u) if len(backup_u) else np.zeros((1, F))
    dx = np.empty((T, d)); dWg = np.empty((F, d)); dWu = np.empty((F, d)); dWd = np.empty((F, d))
    _load().orc_hybrid_backward(T, d, F, C_h, _pd(x), _pd(dy), _pd(_f64(hy["ell_g"])),
                                _pd(_f64(ell_u)),
                                _p(np.ascontiguousarray(hy["ell_idx"], np.uint16), ctypes.c_uint16),
                                _p(np.ascontiguousarray(hy["row_slot"], np.int32), ctypes.c_int32),
                                _pd(bg), _pd(bu), _pd(Wg_t), _pd(Wu_t), _pd(Wd), float(lam),
                                _pd(dx), _pd(dWg), _pd(dWu), _pd(dWd))
    return dx, dWg, dWu, dWd


def dense_ffn_backward(x, Wg_t, Wu_t, Wd, dy, lam):
    """Textbook chain-rule gradients of sum(y*dy) + lam*sum(g).  (dx, dWg_t, dWu_t, dWd)."""
    x, Wg_t, Wu_t, Wd, dy = map(_f64, (x, Wg_t, Wu_t, Wd, dy))
    T, d = x.shape
    F = Wg_t.shape[0]
    dx = np.empty((T, d)); dWg = np.empty((F, d)); dWu = np.empty((F, d)); dWd = np.empty((F, d))
    _load().orc_dense_ffn_backward(T, d, F, _pd(x), _pd(Wg_t), _pd(Wu_t), _pd(Wd), _pd(dy),
                                   float(lam), _pd(dx), _pd(dWg), _pd(dWu), _pd(dWd))
    return dx, dWg, dWu, dWd
