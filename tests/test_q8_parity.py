"""GPU parity of the 8-bit depth KV path against the float64 oracle.

The quantiser (moda_depth_quantize_q8, moda_depth_write_q8) is integer work
decided in float32 on both sides: codes and scales are compared bit for bit.
The forward over the 8-bit cache (moda_fwd_q8) is compared with the oracle's
forward over the dequantised depth keys and values (fl32(scale * code) in the
cache's storage dtype), at the path's tolerance."""
import numpy as np
import pytest
import torch

import oracle
from moda_inputs import WORKLOADS, Workload, make_inputs, sample_rows
from parity_util import compare, f64, to_cuda

pytestmark = pytest.mark.gpu

moda = pytest.importorskip("depth_kv_attention_b200")


def impls_for(w):
    out = ["simt"]
    if w.dtype == "bf16" and w.d == 128 and 128 % w.G == 0:
        out.append("tc")
    return out


QUANT = [
    Workload("q_bf16", 2, 37, 8, 2, 128, 5, "bf16", 81, depth_std=3.0),
    Workload("q_f32_odd_d", 1, 19, 4, 1, 40, 3, "f32", 82),
    Workload("q_d64", 1, 64, 8, 4, 64, 2, "bf16", 83),
]


@pytest.mark.parametrize("w", QUANT, ids=[w.name for w in QUANT])
def test_quantize_bit_exact(w):
    x = make_inputs(w)
    kd8, vd8, ks, vs = moda.moda_depth_quantize_q8(x["kd"].cuda(), x["vd"].cuda())
    torch.cuda.synchronize()
    for got_c, got_s, src in ((kd8, ks, x["kd"]), (vd8, vs, x["vd"])):
        want_c, want_s = oracle.quantize_q8(src)
        np.testing.assert_array_equal(got_c.cpu().numpy(), want_c)
        np.testing.assert_array_equal(got_s.cpu().numpy(), want_s)


def test_quantize_zero_rows_and_ties():
    """A zero row (scale 0, codes 0) and rows whose x / scale has exact
    half-way values (amax 127: ties go to the even code)."""
    kd = torch.zeros(1, 2, 1, 1, 128, dtype=torch.float32)
    kd[0, 1, 0, 0, :8] = torch.tensor([127.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -127.0])
    kd8, _, ks, _ = moda.moda_depth_quantize_q8(kd.cuda(), kd.cuda())
    torch.cuda.synchronize()
    assert ks.cpu().tolist() == [[[[0.0]], [[1.0]]]]
    assert kd8[0, 0].abs().sum().item() == 0
    assert kd8[0, 1, 0, 0, :8].cpu().tolist() == [127, 2, 4, -2, -4, 0, 2, -127]


def test_write_q8_touches_one_slot():
    w = Workload("wq8", 2, 45, 8, 2, 128, 4, "bf16", 84)
    x = make_inputs(w)
    g = torch.Generator("cpu")
    g.manual_seed(3)
    k = torch.randn(w.B, w.T, w.Hkv, w.d, generator=g).to(torch.bfloat16)
    v = torch.randn(w.B, w.T, w.Hkv, w.d, generator=g).to(torch.bfloat16)
    ck, sk = oracle.quantize_q8(x["kd"])
    cv, sv = oracle.quantize_q8(x["vd"])
    dev = [torch.from_numpy(a.copy()).cuda() for a in (ck, cv, sk, sv)]
    moda.moda_depth_write_q8(k.cuda(), v.cuda(), *dev, slot=2)
    torch.cuda.synchronize()
    want = oracle.depth_write_q8(ck, cv, sk, sv, k, v, 2)
    for got, exp in zip(dev, want):
        np.testing.assert_array_equal(got.cpu().numpy(), exp)


FWD = [
    Workload("q8_ragged_g8", 2, 300, 16, 2, 128, 5, "bf16", 85),
    Workload("q8_g32_ld28", 1, 150, 32, 1, 128, 28, "bf16", 86),
    Workload("q8_g1", 1, 200, 4, 4, 128, 3, "bf16", 87),
    Workload("q8_depth_stress", 2, 257, 16, 2, 128, 9, "bf16", 88, depth_std=4.0),
    Workload("q8_t1", 1, 1, 8, 1, 128, 4, "bf16", 89),
    Workload("q8_f32", 2, 77, 6, 2, 72, 3, "f32", 90),
]
FWD_CASES = [(w, impl) for w in FWD for impl in impls_for(w)]


def run_q8(w, x, impl):
    xc = to_cuda(x)
    kd8, vd8, ks, vs = moda.moda_depth_quantize_q8(xc["kd"], xc["vd"])
    out, lse = moda.moda_fwd_q8(xc["q"], xc["k"], xc["v"], kd8, vd8, ks, vs, w.scale, impl=impl)
    torch.cuda.synchronize()
    assert moda.moda_device_status() == 0
    return out, lse


def dequantised(x, dtype="bf16"):
    ck, sk = oracle.quantize_q8(x["kd"])
    cv, sv = oracle.quantize_q8(x["vd"])
    return oracle.dequantize_q8(ck, sk, dtype), oracle.dequantize_q8(cv, sv, dtype)


@pytest.mark.parametrize("w,impl", FWD_CASES, ids=[f"{w.name}-{i}" for w, i in FWD_CASES])
def test_fwd_q8_small(w, impl):
    x = make_inputs(w)
    out, lse = run_q8(w, x, impl)
    kdq, vdq = dequantised(x, w.dtype)
    ro, rl = oracle.forward(x["q"], x["k"], x["v"], kdq, vdq, w.scale)
    compare(f"{w.name}/{impl} out", f64(out), ro, w.dtype)
    compare(f"{w.name}/{impl} lse", f64(lse), rl, w.dtype, what="lse")


def test_fwd_q8_t4k_full_and_t16k_sampled():
    """The 4K workload in full and the 2x16K workload (Ld = 24) on 256
    sampled rows of 8 heads, tensor-core path."""
    w = WORKLOADS["t4k"]
    x = make_inputs(w)
    out, lse = run_q8(w, x, "tc")
    kdq, vdq = dequantised(x)
    ro, rl = oracle.forward(x["q"], x["k"], x["v"], kdq, vdq, w.scale)
    compare("t4k q8 out", f64(out), ro, w.dtype)
    compare("t4k q8 lse", f64(lse), rl, w.dtype, what="lse")
    w = WORKLOADS["t16k_b2"]
    x = make_inputs(w)
    out, lse = run_q8(w, x, "tc")
    out, lse = out.cpu(), lse.cpu()
    kdq, vdq = dequantised(x)
    rows = sample_rows(w, 256)
    for b in range(w.B):
        for h in (0, 5, 11, 17, 20, 26, 30, 31):
            ro, rl = oracle.forward_rows(x["q"], x["k"], x["v"], kdq, vdq, w.scale, b, h, rows)
            compare(f"t16k q8 b{b} h{h} out", f64(out[b, rows, h]), ro, w.dtype)
            compare(f"t16k q8 b{b} h{h} lse", f64(lse[b, h, rows]), rl, w.dtype, what="lse")


def test_fwd_q8_ld0_is_plain_forward():
    w = Workload("q8_ld0", 1, 130, 8, 1, 128, 0, "bf16", 91)
    xc = to_cuda(make_inputs(w))
    o1, l1 = moda.moda_fwd_q8(xc["q"], xc["k"], xc["v"], None, None, None, None, w.scale)
    o2, l2 = moda.moda_fwd(xc["q"], xc["k"], xc["v"], None, None, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
