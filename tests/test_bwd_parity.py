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


def check_bwd(w, impl, x=None, fwd_impl=None):
    """Backward of kernel family ``impl`` against the oracle.

    The forward output and lse it consumes come from the library's own
    forward (family ``fwd_impl``, default the same as ``impl``), as in
    training."""
    x = make_inputs(w, with_dout=True) if x is None else x
    xc = to_cuda(x)
    out, lse = moda.moda_fwd(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], w.scale,
                             impl=fwd_impl or impl)
    grads = moda.moda_bwd(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], out, lse, xc["dout"],
                          w.scale, impl=impl)
    torch.cuda.synchronize()
    assert moda.moda_device_status() == 0
    _LAST_GRADS[0] = grads
    if w.name not in _ORACLE:
        _ORACLE.clear()
        # moda_bwd forms D = <dout, out> from the output it is given, which the
        # forward stored in the input dtype: the oracle forms D the same way,
        # from its own forward output rounded to that dtype.
        ro, _ = oracle.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale)
        stored = torch.from_numpy(ro).to(x["q"].dtype)
        _ORACLE[w.name] = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"],
                                          w.scale, out_for_D=stored)
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
    # Under depth keys ~ N(0, 4^2) the backward amplifies any error of the
    # stored forward output through D = <dout, out> by |kd| (4 sigma here).
    # The tensor-core forward's output, with P rounded to bf16, is within the
    # forward tolerance but not within that amplified margin, so this case
    # feeds every backward the SIMT forward's output (fp32 P) and measures
    # the backward's own arithmetic; the tensor-core forward -> backward chain
    # is checked end to end on all unit-variance cases.
    check_bwd(w, impl, fwd_impl="simt" if w.depth_std > 1.0 else None)


@pytest.mark.parametrize("impl", ["tc", "simt"])
def test_bwd_g32_workload_full(impl):
    """The wide-GQA forward+backward workload (T=8192, G=32, Ld=28), full,
    against the oracle of the stored-output definition and, end to end,
    against the exact derivative (D from the exact forward output)."""
    w = WORKLOADS["g32_fwdbwd"]
    if impl not in impls_for(w):
        pytest.skip("shape not on this path")
    x = make_inputs(w, with_dout=True)
    check_bwd(w, impl, x)
    grads = _LAST_GRADS[0]
    exact = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], w.scale)
    for name, g, r in zip(["dq", "dk", "dv", "dkd", "dvd"], grads, exact[:5]):
        compare(f"{w.name}/{impl} {name} vs exact derivative", f64(g), r, w.dtype, grad=True)
