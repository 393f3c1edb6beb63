"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on the same
seeded inputs and compare element by element at the tolerance the target states,
|gpu - oracle| <= 2e-3 * (1 + |oracle|), on out and lse."""
import numpy as np

RTOL_ABS = 2e-3


def assert_close(gpu, ref, what, tol=RTOL_ABS):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    inf_ref = np.isinf(ref)
    # -inf (empty sequence) must be reproduced exactly
    assert np.array_equal(np.isinf(gpu), inf_ref), f"{what}: inf pattern differs"
    assert np.all(gpu[inf_ref] == ref[inf_ref]), f"{what}: inf sign differs"
    g, r = gpu[~inf_ref], ref[~inf_ref]
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    err = np.abs(g - r)
    bound = tol * (1.0 + np.abs(r))
    worst = float((err / bound).max()) if err.size else 0.0
    assert np.all(err <= bound), (
        f"{what}: {int((err > bound).sum())} of {err.size} elements outside "
        f"|gpu-oracle| <= {tol}*(1+|oracle|); worst ratio {worst:.3f}, max abs err {err.max():.3e}")
    return worst
