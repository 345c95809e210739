"""Comparison of GPU log-mel output with the float64 oracle.

Tolerance (from the accuracy target for the path): |GPU - oracle| <= 2e-3
wherever the oracle mel energy M > 1e-8; where M == 0 (silent frames, empty
filters) the GPU value must be exactly ln(1e-10) rounded to fp32; where
0 < M <= 1e-8 the GPU value must lie in [fp32 ln(1e-10), ln(1e-8) + 2e-3].
"""
import numpy as np

TOL = 2e-3
FLOOR32 = np.float32(np.log(1e-10))


def check_against_oracle(gpu, L, M, tol=TOL):
    g = np.asarray(gpu, np.float32)
    assert g.shape == L.shape == M.shape, (g.shape, L.shape, M.shape)
    if g.size == 0:
        return {"cells": 0}
    big = M > 1e-8
    zero = M == 0
    small = ~big & ~zero
    assert np.all(np.isfinite(g))
    err = np.abs(g.astype(np.float64) - L)
    max_err = float(err[big].max()) if big.any() else 0.0
    if big.any() and max_err > tol:
        r, c = np.unravel_index(np.argmax(np.where(big, err, 0)), err.shape)
        raise AssertionError(f"max |d| {max_err:.3e} > {tol} at row {r} band {c}: gpu {g[r, c]} oracle "
                             f"{L[r, c]} energy {M[r, c]:.3e}")
    bad_floor = zero & (g != FLOOR32)
    assert not bad_floor.any(), f"{int(bad_floor.sum())} zero-energy cells differ from the fp32 floor"
    if small.any():
        gs = g[small]
        assert np.all((gs >= FLOOR32) & (gs <= np.log(1e-8) + tol)), "tiny-energy cells out of band"
    return {"cells": int(g.size), "max_err": max_err, "zero_cells": int(zero.sum()),
            "tiny_cells": int(small.sum())}
