"""GPU parity of the write step (moda_depth_write) against the oracle's
depth_write: a bit-exact copy into one slot of the depth cache, the other
slots untouched; then the forward over a cache filled layer by layer."""
import numpy as np
import pytest
import torch

import oracle
from moda_inputs import Workload, make_inputs
from parity_util import compare, f64

pytestmark = pytest.mark.gpu

moda = pytest.importorskip("depth_kv_attention_b200")


@pytest.mark.parametrize("B,T,Hkv,d,Ld,slot,dtype", [
    (2, 77, 3, 128, 5, 0, torch.bfloat16),
    (1, 300, 4, 128, 28, 27, torch.bfloat16),
    (3, 9, 1, 64, 2, 1, torch.bfloat16),
    (2, 33, 2, 72, 4, 2, torch.float32),
])
def test_depth_write_bit_exact(B, T, Hkv, d, Ld, slot, dtype):
    g = torch.Generator("cpu")
    g.manual_seed(7000 + T)
    k = torch.randn((B, T, Hkv, d), generator=g).to(dtype)
    v = torch.randn((B, T, Hkv, d), generator=g).to(dtype)
    kd = torch.randn((B, T, Ld, Hkv, d), generator=g).to(dtype)
    vd = torch.randn((B, T, Ld, Hkv, d), generator=g).to(dtype)
    want_k, want_v = oracle.depth_write(kd.numpy() if dtype == torch.float32 else kd.float().numpy(),
                                        vd.numpy() if dtype == torch.float32 else vd.float().numpy(),
                                        k.float().numpy(), v.float().numpy(), slot)
    kd_c, vd_c = kd.cuda(), vd.cuda()
    moda.moda_depth_write(k.cuda(), v.cuda(), kd_c, vd_c, slot)
    torch.cuda.synchronize()
    # every element equal, bit for bit (the values are exact in float32)
    assert np.array_equal(kd_c.float().cpu().numpy(), want_k)
    assert np.array_equal(vd_c.float().cpu().numpy(), want_v)
    assert torch.equal(kd_c.cpu()[:, :, slot], k) and torch.equal(vd_c.cpu()[:, :, slot], v)


def test_depth_written_layer_by_layer_then_forward():
    """Fill an empty depth cache slot by slot with the write step, then run
    the forward on it; the result matches the oracle on the same cache."""
    w = Workload("write_then_read", 1, 257, 16, 2, 128, 6, "bf16", 71)
    x = make_inputs(w)
    g = torch.Generator("cpu")
    g.manual_seed(72)
    kd = torch.zeros_like(x["kd"]).cuda()
    vd = torch.zeros_like(x["vd"]).cuda()
    layers = [(torch.randn(x["k"].shape, generator=g).to(torch.bfloat16),
               torch.randn(x["v"].shape, generator=g).to(torch.bfloat16)) for _ in range(w.Ld)]
    for slot, (kl, vl) in enumerate(layers):
        moda.moda_depth_write(kl.cuda(), vl.cuda(), kd, vd, slot)
    out, lse = moda.moda_fwd(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), kd, vd, w.scale)
    torch.cuda.synchronize()
    assert moda.moda_device_status() == 0
    sk = torch.stack([kl for kl, _ in layers], dim=2)
    sv = torch.stack([vl for _, vl in layers], dim=2)
    assert torch.equal(kd.cpu(), sk) and torch.equal(vd.cpu(), sv)
    ro, rl = oracle.forward(x["q"], x["k"], x["v"], sk, sv, w.scale)
    compare("write-then-read out", f64(out), ro, "bf16")
    compare("write-then-read lse", f64(lse), rl, "bf16", what="lse")
