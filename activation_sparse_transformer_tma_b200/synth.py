"""Seeded synthetic workloads for the activation-sparse gated FFN.

This module only draws inputs: it holds none of the FFN's arithmetic.  It is
the one module shared by the CPU oracle's tests and the CUDA path's tests and
bench.  The recipe, per workload (there are no trained weights or datasets
here; the shapes stand in for the 0.5B and 2B models' FFN layers):

* x ~ N(0, 1) of shape [T, d]; column 0 is overwritten with a per-token scale
  s_t (a constant channel).
* Wg_t, Wu_t ~ N(0, 1/d) of shape [F, d]; Wd ~ N(0, 1/F) of shape [F, d].
  Wg_t[:, 0] is overwritten with -theta_j, so the gate pre-activation is
  z_tj = -s_t * theta_j + eps with eps ~ N(0, (d-1)/d), and
  P(unit j active for token t) = Phi(-s_t * theta_j / sigma), sigma = sqrt((d-1)/d).
* theta and s are set per workload to give the stated activation statistics
  (about 29 active units per token, i.e. >99% sparsity, for the bf16 ones).
* Everything is drawn in fp64 from NumPy PCG64 streams spawned from one seed
  (one stream per tensor, in the order x, Wg, Wu, Wd, structure draws, dy) and
  rounded once, round-to-nearest-even, to the workload dtype.

bf16 tensors are carried as uint16 bit patterns; fp32 as float32.
"""
from __future__ import annotations

import numpy as np
from scipy.special import ndtr, ndtri

BF16 = "bf16"
F32 = "f32"

# name -> (T, d, F, W, C, dtype, kind)
PRESETS = {
    "tiny_fp32": dict(T=64, d=256, F=1024, W=128, C=16, dtype=F32, kind="uniform4"),
    "ffn_0p5b": dict(T=4096, d=1024, F=4096, W=128, C=8, dtype=BF16, kind="dead20"),
    "ffn_2b": dict(T=16384, d=2048, F=8192, W=128, C=8, dtype=BF16, kind="zipf"),
    "decode_2b": dict(T=64, d=2048, F=8192, W=128, C=8, dtype=BF16, kind="zipf"),
    "train_2b": dict(T=8192, d=2048, F=8192, W=128, C=8, C_h=64, dtype=BF16,
                     kind="pareto", lam=2e-5),
}

MEAN_ACTIVE = 29.0


# ---------------------------------------------------------------- rounding ---
def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp64 values once, to nearest even, onto the bf16 grid (as fp64)."""
    a = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(a)                       # a = m * 2**e, 0.5 <= |m| < 1
    q = np.rint(m * 256.0)                   # 8 significant bits, ties to even
    out = np.ldexp(q, e - 8)
    # bf16 has fp32's exponent range; inputs here are far from its limits.
    assert np.all(np.abs(out[out != 0]) >= 2.0 ** -126)
    return out


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of values already on the bf16 grid."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def to_storage(a64: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == BF16:
        return bf16_bits(round_bf16(a64))
    if dtype == F32:
        return np.asarray(a64, dtype=np.float64).astype(np.float32)
    raise ValueError(dtype)


def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 value of a stored tensor."""
    if dtype == BF16:
        return bf16_to_f64(a)
    if dtype == F32:
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    raise ValueError(dtype)


# ------------------------------------------------------------- calibration ---
def _bisect(f, lo, hi, target, iters=100):
    """Solve f(v) = target for increasing f on [lo, hi]."""
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if f(mid) < target:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def _zipf_probs(F, ranks, mean_active, alpha=1.1, pmax=0.5):
    r = ranks.astype(np.float64) + 1.0
    base = r ** -alpha
    A = _bisect(lambda a: np.minimum(pmax, a * base).sum(), 0.0, 1e6, mean_active)
    return np.minimum(pmax, A * base)


def _lognormal_scale(theta, sigma, mean_active, ln_sigma=0.5, nodes=48):
    """c such that E_L[sum_j Phi(-c*L*theta_j/sigma)] = mean_active, L ~ LogNormal(0, ln_sigma).

    The expectation over L is taken by Gauss-Hermite quadrature.
    """
    xs, ws = np.polynomial.hermite_e.hermegauss(nodes)
    ws = ws / ws.sum()
    L = np.exp(ln_sigma * xs)

    def expected(c):
        return float(sum(w * ndtr(-c * l * theta / sigma).sum() for l, w in zip(L, ws)))

    # expected() decreases in c (theta >= 0); bisect on its negative.
    return _bisect(lambda c: -expected(c), 1e-3, 1e3, -mean_active)


# --------------------------------------------------------------- workloads ---
def make_workload(name: str | None = None, *, seed: int = 0, T=None, d=None, F=None,
                  W=None, C=None, C_h=None, dtype=None, kind=None, lam=None,
                  mean_active=MEAN_ACTIVE, permute=True, with_dy=None):
    """Draw one workload.  ``name`` picks a preset; keyword arguments override it.

    Returned dict: shapes and parameters, the stored tensors x [T,d], Wg_t, Wu_t,
    Wd [F,d] (and dy [T,d] for training workloads), plus ``stats`` describing
    the drawn structure.
    """
    cfg = dict(PRESETS[name]) if name else {}
    for k, v in dict(T=T, d=d, F=F, W=W, C=C, C_h=C_h, dtype=dtype, kind=kind,
                     lam=lam).items():
        if v is not None:
            cfg[k] = v
    cfg.setdefault("C_h", 64)
    cfg.setdefault("lam", 2e-5)
    T, d, F, kind, dt = cfg["T"], cfg["d"], cfg["F"], cfg["kind"], cfg["dtype"]
    full_T = PRESETS[name]["T"] if name else T
    gen_T = max(T, full_T)           # decode draws x as a prefix of the 2B stream

    ss = np.random.SeedSequence(seed)
    r_x, r_wg, r_wu, r_wd, r_st, r_dy = [np.random.Generator(np.random.PCG64(s))
                                         for s in ss.spawn(6)]
    x = r_x.standard_normal((gen_T, d))[:T]
    Wg_t = r_wg.standard_normal((F, d)) / np.sqrt(d)
    Wu_t = r_wu.standard_normal((F, d)) / np.sqrt(d)
    Wd = r_wd.standard_normal((F, d)) / np.sqrt(F)
    sigma = np.sqrt((d - 1) / d)
    stats = {"kind": kind, "sigma": sigma}

    if kind == "uniform4":                  # 4% per-unit activation probability
        theta = np.full(F, ndtri(0.96) * sigma)
        s = np.ones(T)
    elif kind == "dead20":                  # 20% dead units, mean 29 active
        dead = r_st.choice(F, size=int(round(0.2 * F)), replace=False)
        alive = F - len(dead)
        theta = np.full(F, ndtri(1.0 - mean_active / alive) * sigma)
        theta[dead] = 1e4
        s = np.ones(T)
        stats["dead_units"] = np.sort(dead)
    elif kind == "zipf":                    # Zipf(1.1) units, lognormal token skew
        ranks = r_st.permutation(F) if permute else np.arange(F)
        p = _zipf_probs(F, ranks, mean_active)
        theta = ndtri(1.0 - p) * sigma
        c = _lognormal_scale(theta, sigma, mean_active)
        s = c * r_st.lognormal(0.0, 0.5, size=gen_T)[:T]
        stats.update(p=p, c=c)
    elif kind == "pareto":                  # heavy-tailed per-token active counts
        theta = np.ones(F)
        alpha, xm = 1.5, mean_active * (1.5 - 1.0) / 1.5
        n = xm * (1.0 + r_st.pareto(alpha, size=gen_T)[:T])
        n = np.minimum(n, F / 2)
        s = sigma * ndtri(1.0 - n / F)       # x[t,0] = tau_t, theta_j = 1
        stats["target_active"] = n
    else:
        raise ValueError(kind)

    x[:, 0] = s
    Wg_t[:, 0] = -theta
    stats["theta"] = theta
    stats["s"] = s
    stats["expected_active"] = ndtr(-np.outer(s[: min(T, 4096)], theta) / sigma).sum(1).mean() \
        if kind != "pareto" else float(np.mean(stats["target_active"]))

    out = dict(cfg)
    out["name"] = name or "custom"
    out["x"] = to_storage(x, dt)
    out["Wg_t"] = to_storage(Wg_t, dt)
    out["Wu_t"] = to_storage(Wu_t, dt)
    out["Wd"] = to_storage(Wd, dt)
    if with_dy or (with_dy is None and kind == "pareto"):
        out["dy"] = to_storage(r_dy.standard_normal((T, d)), dt)
    out["stats"] = stats
    return out


def subsample_rows(T: int, n: int, seed: int = 1) -> np.ndarray:
    """A seeded, sorted sample of n distinct token rows out of T."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    n = min(n, T)
    return np.sort(rng.choice(T, size=n, replace=False)).astype(np.int32)
