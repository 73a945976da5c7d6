"""GPU parity of the per-token depth-slot selection (moda_fwd_sel,
moda_bwd_sel) against the float64 oracle's ``depth_sel``.

Depth keys are drawn wider than the sequence keys (depth_std 2) so that the
depth slots carry a large share of each softmax and a selection mistake
moves the result well past the tolerance."""
import numpy as np
import pytest
import torch

import oracle
from moda_inputs import WORKLOADS, Workload, make_depth_sel, make_inputs, pack_depth_sel, sample_rows
from parity_util import compare, f64, to_cuda

pytestmark = pytest.mark.gpu

moda = pytest.importorskip("depth_kv_attention_b200")


def impls_for(w):
    out = ["simt"]
    if w.dtype == "bf16" and w.d == 128 and 128 % w.G == 0:
        out.append("tc")
    return out


FWD = [
    (Workload("sel_g8_random", 2, 300, 16, 2, 128, 5, "bf16", 41, depth_std=2.0), "random"),
    (Workload("sel_g32_window", 1, 150, 32, 1, 128, 28, "bf16", 42, depth_std=2.0), "window"),
    (Workload("sel_g4_ld64", 1, 97, 8, 2, 128, 64, "bf16", 43, depth_std=2.0), "random"),
    (Workload("sel_g1_ld33", 1, 70, 4, 4, 128, 33, "bf16", 44, depth_std=2.0), "window"),
    (Workload("sel_none", 1, 130, 8, 1, 128, 7, "bf16", 45, depth_std=2.0), "none"),
    (Workload("sel_t1", 1, 1, 8, 1, 128, 4, "bf16", 46, depth_std=2.0), "random"),
    (Workload("sel_f32", 2, 70, 4, 2, 64, 3, "f32", 47, depth_std=2.0), "random"),
]
FWD_CASES = [(w, kind, impl) for w, kind in FWD for impl in impls_for(w)]


def run_sel(w, x, bits, impl):
    xc = to_cuda(x)
    out, lse = moda.moda_fwd_sel(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], bits.cuda(),
                                 w.scale, impl=impl)
    torch.cuda.synchronize()
    assert moda.moda_device_status() == 0
    return xc, out, lse


@pytest.mark.parametrize("w,kind,impl", FWD_CASES, ids=[f"{w.name}-{i}" for w, _, i in FWD_CASES])
def test_sel_fwd_small(w, kind, impl):
    x = make_inputs(w)
    sel = make_depth_sel(w, kind)
    _, out, lse = run_sel(w, x, pack_depth_sel(sel), impl)
    ro, rl = oracle.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale, depth_sel=sel.numpy())
    compare(f"{w.name}/{impl} out", f64(out), ro, w.dtype)
    compare(f"{w.name}/{impl} lse", f64(lse), rl, w.dtype, what="lse")


@pytest.mark.parametrize("impl", ["simt", "tc"])
def test_sel_all_slots_is_unselected_forward(impl):
    """A mask with every slot set (and bits above Ld set too, which are
    ignored) gives exactly moda_fwd's output."""
    w = Workload("sel_all", 2, 211, 16, 2, 128, 6, "bf16", 48, depth_std=2.0)
    x = make_inputs(w)
    bits = torch.full((w.B, w.T), -1, dtype=torch.int64)
    xc, out, lse = run_sel(w, x, bits, impl)
    o0, l0 = moda.moda_fwd(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], w.scale, impl=impl)
    torch.cuda.synchronize()
    assert torch.equal(out, o0) and torch.equal(lse, l0)


def test_sel_t4k_window_full():
    """The 4K workload (G=8, Ld=16) with a per-token window of recent slots,
    whole output, on the tensor-core path."""
    w = WORKLOADS["t4k"]
    x = make_inputs(w)
    sel = make_depth_sel(w, "window")
    _, out, lse = run_sel(w, x, pack_depth_sel(sel), "tc")
    ro, rl = oracle.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale, depth_sel=sel.numpy())
    compare("t4k window out", f64(out), ro, w.dtype)
    compare("t4k window lse", f64(lse), rl, w.dtype, what="lse")


def test_sel_t16k_sampled():
    """2x16K, Ld=24, random half of the slots, on 256 sampled rows of every
    head."""
    w = WORKLOADS["t16k_b2"].with_(depth_std=2.0)
    x = make_inputs(w)
    sel = make_depth_sel(w, "random")
    _, out, lse = run_sel(w, x, pack_depth_sel(sel), "tc")
    out, lse = out.cpu(), lse.cpu()
    rows = sample_rows(w, 256)
    for b in range(w.B):
        for h in range(w.Hq):
            ro, rl = oracle.forward_rows(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale, b, h, rows,
                                         depth_sel=sel.numpy())
            compare(f"t16k sel b{b} h{h} out", f64(out[b, rows, h]), ro, w.dtype)
            compare(f"t16k sel b{b} h{h} lse", f64(lse[b, h, rows]), rl, w.dtype, what="lse")


BWD = [
    (Workload("selb_g8", 2, 300, 16, 2, 128, 5, "bf16", 51, depth_std=2.0), "random"),
    (Workload("selb_g32", 1, 200, 32, 1, 128, 28, "bf16", 52, depth_std=2.0), "window"),
    (Workload("selb_ld64", 1, 97, 8, 2, 128, 64, "bf16", 53, depth_std=2.0), "random"),
    (Workload("selb_f32", 2, 70, 4, 2, 64, 3, "f32", 54, depth_std=2.0), "random"),
]
BWD_CASES = [(w, kind, impl) for w, kind in BWD for impl in impls_for(w)]


@pytest.mark.parametrize("w,kind,impl", BWD_CASES, ids=[f"{w.name}-{i}" for w, _, i in BWD_CASES])
def test_sel_bwd_small(w, kind, impl):
    """Forward then backward of one kernel family under a selection, against
    the exact derivative; unselected depth slots get exactly zero."""
    x = make_inputs(w, with_dout=True)
    sel = make_depth_sel(w, kind)
    bits = pack_depth_sel(sel).cuda()
    xc = to_cuda(x)
    out, lse = moda.moda_fwd_sel(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], bits, w.scale,
                                 impl=impl)
    grads = moda.moda_bwd_sel(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], bits, out, lse,
                              xc["dout"], w.scale, impl=impl)
    torch.cuda.synchronize()
    assert moda.moda_device_status() == 0
    want = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], w.scale,
                           depth_sel=sel.numpy())
    for name, g, r in zip(["dq", "dk", "dv", "dkd", "dvd"], grads, want[:5]):
        compare(f"{w.name}/{impl} {name}", f64(g), r, w.dtype, grad=True)
    unsel = ~sel
    for g in grads[3:5]:
        assert torch.all(g.cpu()[unsel] == 0)
