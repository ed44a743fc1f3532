"""Tolerance checks shared by the parity tests.

Tolerances (stated for this operation): bf16 inputs with fp32 accumulation
  |out - ref| <= 1e-2 + 1e-2 |ref|,  |lse - ref| <= 2e-3,
  dq / dk / dv / dsink relative L2 error <= 2e-2;
fp16 inputs: out 2.5e-3 + 2.5e-3 |ref|, lse 1e-3, gradients 5e-3: the tensor cores see P
  and dS rounded to fp16 (unit roundoff 2^-11 = 4.9e-4) and the outputs are rounded once
  more, so about five unit roundoffs per output with room for fp32 accumulation order;
fp32 inputs: the same checks with 1e-4 in place of each bf16 bound.
A row with no visible key must have lse = -inf on both sides.
"""
import numpy as np

TOL = {
    "bf16": {"out_abs": 1e-2, "out_rel": 1e-2, "lse": 2e-3, "grad": 2e-2},
    "fp16": {"out_abs": 2.5e-3, "out_rel": 2.5e-3, "lse": 1e-3, "grad": 5e-3},
    "fp32": {"out_abs": 1e-4, "out_rel": 1e-4, "lse": 1e-4, "grad": 1e-4},
}


def to_np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_out(got, ref, dtype: str, what: str = "out"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    t = TOL[dtype]
    err = np.abs(got - ref)
    bound = t["out_abs"] + t["out_rel"] * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                             f"max err {err.max():.3e}; first bad {idx.tolist()} "
                             f"got {got[tuple(idx[0])]:.6f} ref {ref[tuple(idx[0])]:.6f}")
    return float(err.max()) if err.size else 0.0


def check_lse(got, ref, dtype: str, what: str = "lse"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    ninf_ref = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), ninf_ref), f"{what}: -inf rows differ"
    fin = ~ninf_ref
    assert np.all(np.isfinite(got[fin])), f"{what}: non-finite values"
    err = np.abs(got[fin] - ref[fin])
    e = float(err.max()) if err.size else 0.0
    assert e <= TOL[dtype]["lse"], f"{what}: max err {e:.3e}"
    return e


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))


def check_grad(got, ref, dtype: str, what: str):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    r = rel_l2(got, ref)
    assert r <= TOL[dtype]["grad"], f"{what}: relative L2 error {r:.3e}"
    return r
