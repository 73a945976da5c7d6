"""Shared helpers of the GPU parity tests: tolerances, input staging, and the
element-wise comparison against the float64 oracle."""
import numpy as np
import torch

# Tolerances of the MoDA path: bf16 inputs max-abs 2e-2 and mean-abs 2e-3 on
# outputs and gradients, 1e-2 relative on lse; fp32 inputs 1e-5.
TOL = {
    "bf16": dict(max_abs=2e-2, mean_abs=2e-3, lse_rel=1e-2),
    "f32": dict(max_abs=1e-5, mean_abs=1e-5, lse_rel=1e-5),
}


def to_cuda(x: dict) -> dict:
    return {k: (None if v is None else v.cuda()) for k, v in x.items()}


def f64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype != torch.float64 else t.cpu().numpy()


def compare(name, got, want, dtype, what="out", grad=False):
    """Element-wise comparison with the path's tolerance; returns the errors.

    ``grad=True`` (gradients stored in bf16): the max-abs bound is the stated
    one plus one bf16 ulp of the reference, 2^-8 * |want|, because storing a
    gradient of magnitude |g| in bf16 alone costs up to 2^-9 * |g| — more than
    2e-2 once |g| > 10, which dK / dV (sums over G*T rows) and dQ under large
    depth keys reach. The mean-abs bound is unchanged."""
    tol = TOL[dtype]
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    if what == "lse":
        rel = np.abs(got - want) / np.maximum(np.abs(want), 1e-6)
        # a relative bound is meaningless where lse crosses 0: also accept
        # the absolute bound there
        bad = (rel > tol["lse_rel"]) & (np.abs(got - want) > tol["lse_rel"])
        assert not bad.any(), f"{name}: lse rel err max {rel.max():.3e}"
        return float(rel.max())
    err = np.abs(got - want)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    if grad and dtype == "bf16":
        allowed = tol["max_abs"] + np.abs(want) * 2.0 ** -8
        worst = float((err / allowed).max()) if err.size else 0.0
        # how many elements needed the relative term (error above the plain
        # stated bound), reported with every gradient comparison
        n_rel = int(np.count_nonzero(err > tol["max_abs"]))
        print(f"{name}: {n_rel} of {err.size} elements above {tol['max_abs']} "
              f"(within 2^-8 |g| of it), max-abs {mx:.3e}")
        assert worst <= 1.0, f"{name}: max-abs {mx:.3e}, {worst:.2f}x the bf16-scaled bound"
    else:
        assert mx <= tol["max_abs"], f"{name}: max-abs {mx:.3e} > {tol['max_abs']}"
    assert mean <= tol["mean_abs"], f"{name}: mean-abs {mean:.3e} > {tol['mean_abs']}"
    return mx, mean
