"""moda_bwd_noalloc: the backward for callers that cannot allocate device
memory (a host program that only hands over its input and output buffers, or
a runtime whose memory pool owns the whole device, so the library cannot get
a workspace from it). The entry point keeps its scratch in a fixed array
compiled into the library.

Checks, through the C ABI: two calls in a row (the second sees the array as
the first left it) agree with the existing moda_bwd entry point within the
tolerance the parity tests use, and bit for bit with moda_bwd_ex on the
scalar kernels it shares; a problem whose scratch exceeds the array is
rejected. This file runs last, and passes alone in a fresh process too."""
import pytest
import torch

from moda_inputs import Workload, make_inputs
from parity_util import compare, f64, to_cuda

pytestmark = pytest.mark.gpu

moda = pytest.importorskip("depth_kv_attention_b200")

NAMES = ["dq", "dk", "dv", "dkd", "dvd"]


def _grads(w):
    x = to_cuda(make_inputs(w, with_dout=True))
    out, lse = moda.moda_fwd(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale)
    ref = moda.moda_bwd(x["q"], x["k"], x["v"], x["kd"], x["vd"], out, lse, x["dout"], w.scale)
    same_kernels = moda.moda_bwd(x["q"], x["k"], x["v"], x["kd"], x["vd"], out, lse, x["dout"],
                                 w.scale, impl="simt")
    got = moda.moda_bwd_noalloc(x["q"], x["k"], x["v"], x["kd"], x["vd"], out, lse, x["dout"],
                                w.scale)
    torch.cuda.synchronize()
    return ref, same_kernels, got


def test_noalloc_backward_matches_moda_bwd_on_two_calls_in_a_row():
    calls = [Workload("noalloc_a", 2, 300, 16, 2, 128, 5, "bf16", 61),
             Workload("noalloc_b", 1, 200, 32, 1, 128, 28, "bf16", 62)]
    for w in calls:
        ref, same, got = _grads(w)
        for n, r, s, g in zip(NAMES, ref, same, got):
            compare(f"{w.name} {n} vs moda_bwd", f64(g), f64(r), "bf16", grad=True)
            assert torch.equal(g, s), f"{w.name} {n}: differs from moda_bwd_ex on the same kernels"


def test_noalloc_fp32_matches_scalar_backward_and_oracle():
    """fp32 inputs (the tiny fp32 workload's shape: T=128, G=4, d=64, Ld=4):
    the float row statistics in the shared array and the fp32 kernels, bit
    for bit against moda_bwd on the same kernels and within 1e-5 of the
    float64 oracle's exact derivative, on two calls in a row."""
    import oracle
    w = Workload("noalloc_f32", 1, 128, 4, 1, 64, 4, "f32", 63)
    x = make_inputs(w, with_dout=True)
    want = oracle.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], w.scale)
    for _ in range(2):
        ref, same, got = _grads(w)
        for n, s, g, r in zip(NAMES, same, got, want):
            assert torch.equal(g, s), f"{w.name} {n}: differs from moda_bwd_ex on the same kernels"
            compare(f"{w.name} {n} vs oracle", f64(g), r, "f32")


def test_noalloc_rejects_problems_beyond_its_scratch():
    limit = 16 * 1024 * 1024
    B, T, Hq = 1, limit // (4 * 32) + 1, 32  # B*Hq*T*4 bytes just over the array
    P = 0x10000  # never dereferenced: the call is rejected before any launch
    code = moda._c_bwd_noalloc(P, P, P, P, P, P, P, P, B, T, Hq, 1, 128, 2, 0, 0.088,
                               P, P, P, P, P, None)
    assert code == 4  # MODA_ERR_WORKSPACE
