"""Failure detection without a GPU fault: every on-chip wait of the
tensor-core kernel is bounded. A poll cap of one try makes the waits run out;
the kernel must record MODA_ERR_DEVICE_TIMEOUT in the device status word,
drain its own copies and MMAs, free TMEM and return, leaving the context
usable for a normal call afterwards."""
import pytest
import torch

import oracle
from moda_inputs import Workload, make_inputs
from parity_util import compare, f64, to_cuda

pytestmark = pytest.mark.gpu

moda = pytest.importorskip("depth_kv_attention_b200")

TIMEOUT = 6  # MODA_ERR_DEVICE_TIMEOUT


@pytest.mark.parametrize("impl", ["tc", "tc2"])
def test_bounded_wait_reports_timeout_and_context_survives(impl):
    """Both tensor-core forwards: the single-CTA kernel and the CTA-pair
    kernel (whose expired waits also raise the peer CTA's abort flag and
    still meet at the final cluster barrier)."""
    w = Workload("fault", 1, 640, 16, 2, 128, 5, "bf16", 41)
    x = make_inputs(w)
    xc = to_cuda(x)
    assert moda.moda_device_status() == 0
    moda.moda_debug_set_wait_limit(1)
    try:
        moda.moda_fwd(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], w.scale, impl=impl)
        st = moda.moda_device_status()
    finally:
        moda.moda_debug_set_wait_limit(0)
    assert st == TIMEOUT, moda.moda_status_string(st)
    # the status word is cleared by the read
    assert moda.moda_device_status() == 0
    # the context is intact: a normal call after the expired waits is correct
    out, lse = moda.moda_fwd(xc["q"], xc["k"], xc["v"], xc["kd"], xc["vd"], w.scale, impl=impl)
    torch.cuda.synchronize()
    assert moda.moda_device_status() == 0
    ro, rl = oracle.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale)
    compare("after-timeout out", f64(out), ro, "bf16")
    compare("after-timeout lse", f64(lse), rl, "bf16", what="lse")
