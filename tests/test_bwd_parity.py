"""GPU parity of the MoDA backward (dq, dk, dv, dkd, dvd) against the float64
oracle's derivative of the forward, element by element."""
import numpy as np
import pytest
import torch

import oracle
from moda_inputs import WORKLOADS, Workload, make_inputs
from parity_util import compare, f64, to_cuda

pytestmark = pytest.mark.gpu

moda = pytest.importorskip("depth_kv_attention_b200")


def impls_for(w):
    out = ["simt"]
    if w.dtype == "bf16" and w.d == 128 and 128 % w.G == 0:
        out.append("tc")
    return out


_ORACLE = {}  # the last workload's oracle gradients, shared by its impl variants
_LAST_GRADS = [None]


def check_bwd(w, impl, x=None):
    """Backward of kernel family ``impl`` against the oracle's exact
    derivative. The forward output and lse it consumes come from the same
    family's forward, as in training."""
    x = make_inputs(w, with_dout=True) if x is None else x
    xc = to_cuda(x)
    out, lse = moda.moda_fwd(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], w.scale, impl=impl)
    grads = moda.moda_bwd(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], out, lse, xc["dout"],
                          w.scale, impl=impl)
    torch.cuda.synchronize()
    assert moda.moda_device_status() == 0
    _LAST_GRADS[0] = grads
    if w.name not in _ORACLE:
        _ORACLE.clear()
        _ORACLE[w.name] = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"],
                                          w.scale)
    want = _ORACLE[w.name]
    errs = {}
    for name, g, r in zip(["dq", "dk", "dv", "dkd", "dvd"], grads, want[:5]):
        if w.Ld == 0 and name in ("dkd", "dvd"):
            continue
        errs[name] = compare(f"{w.name}/{impl} {name}", f64(g), r, w.dtype, grad=True)
        # report error relative to the gradient's rms as well
        rms = float(np.sqrt(np.mean(r ** 2))) or 1.0
        print(f"{w.name}/{impl} {name}: max-abs {errs[name][0]:.2e} rms {rms:.2e}")
    return errs


SMALL = [
    Workload("bwd_f32", 2, 70, 4, 2, 64, 3, "f32", 31),
    Workload("bwd_f32_odd", 1, 33, 3, 1, 40, 2, "f32", 32),
    Workload("bwd_ragged_g8", 2, 300, 16, 2, 128, 5, "bf16", 33),
    Workload("bwd_g32", 1, 200, 32, 1, 128, 28, "bf16", 34),
    Workload("bwd_ld0", 1, 150, 8, 2, 128, 0, "bf16", 35),
    Workload("bwd_depth_stress", 1, 129, 16, 2, 128, 7, "bf16", 36, depth_std=4.0),
    Workload("bwd_g1", 1, 140, 4, 4, 128, 2, "bf16", 37),
]


CASES = [(w, impl) for w in SMALL for impl in impls_for(w)]


@pytest.mark.parametrize("w,impl", CASES, ids=[f"{w.name}-{i}" for w, i in CASES])
def test_bwd_small(w, impl):
    """Forward then backward of one kernel family, against the exact
    derivative. The depth-stress case (kd ~ N(0, 4^2)) is the one where the
    rounding of the stored output would show: D taken from it would move dq
    by |kd| times that rounding; the backward forms D from its own P, dP."""
    check_bwd(w, impl)


@pytest.mark.parametrize("impl", ["tc", "simt"])
def test_bwd_g32_workload_full(impl):
    """The wide-GQA forward+backward workload (T=8192, G=32, Ld=28), full,
    forward and backward of one kernel family against the exact derivative."""
    w = WORKLOADS["g32_fwdbwd"]
    if impl not in impls_for(w):
        pytest.skip("shape not on this path")
    check_bwd(w, impl, make_inputs(w, with_dout=True))


def test_bwd_depth_stress_wide_gqa_tc():
    """Depth-dominated rows at G = 32 and Ld = 28 (kd ~ N(0, 4^2)), several
    query tiles and a ragged tail: the tensor-core chain against the exact
    derivative."""
    check_bwd(Workload("bwd_stress_g32", 1, 333, 32, 1, 128, 28, "bf16", 38, depth_std=4.0), "tc")
