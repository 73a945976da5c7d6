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


def test_producer_writes_straight_into_depth_slots():
    """The write step fused with its producer: each earlier layer's key and
    value projections (GEMMs x_l @ W) write their [B*T, Hkv*d] output directly
    into slot l of the native depth cache through the slot view (leading
    dimension Ld*Hkv*d). No copy or elementwise kernel runs while the cache is
    filled, the slots hold the projections, and the forward over the cache
    matches the oracle."""
    B, T, Hq, Hkv, d, Ld, Dm = 2, 300, 16, 2, 128, 3, 256
    g = torch.Generator("cpu")
    g.manual_seed(23)
    dt = torch.bfloat16
    xs = [torch.randn(B * T, Dm, generator=g).to(dt).cuda() for _ in range(Ld)]
    wk = [(torch.randn(Dm, Hkv * d, generator=g) / 16).to(dt).cuda() for _ in range(Ld)]
    wv = [(torch.randn(Dm, Hkv * d, generator=g) / 16).to(dt).cuda() for _ in range(Ld)]
    q = torch.randn(B, T, Hq, d, generator=g).to(dt).cuda()
    k = torch.randn(B, T, Hkv, d, generator=g).to(dt).cuda()
    v = torch.randn(B, T, Hkv, d, generator=g).to(dt).cuda()
    kd = torch.zeros(B, T, Ld, Hkv, d, dtype=dt, device="cuda")
    vd = torch.zeros_like(kd)
    torch.cuda.synchronize()
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for layer in range(Ld):
            for cache, w in ((kd, wk[layer]), (vd, wv[layer])):
                view = moda.depth_slot_view(cache, layer).view(B * T, Hkv * d)  # stride (Ld*Hkv*d, 1)
                torch.mm(xs[layer], w, out=view)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type.name == "CUDA"]
    assert names, "no kernel recorded"
    bad = [n for n in names if any(s in n.lower() for s in ("copy", "elementwise", "memcpy", "fill"))]
    assert not bad, bad
    for layer in range(Ld):
        want_k = (xs[layer] @ wk[layer]).view(B, T, Hkv, d)
        want_v = (xs[layer] @ wv[layer]).view(B, T, Hkv, d)
        torch.testing.assert_close(kd[:, :, layer], want_k, rtol=1e-2, atol=1e-2)
        torch.testing.assert_close(vd[:, :, layer], want_v, rtol=1e-2, atol=1e-2)
    out, lse = moda.moda_fwd(q, k, v, kd, vd)
    torch.cuda.synchronize()
    ro, rl = oracle.forward(q.cpu(), k.cpu(), v.cpu(), kd.cpu(), vd.cpu(), 1.0 / d ** 0.5)
    compare("strided-producer cache out", f64(out), ro, "bf16")
    compare("strided-producer cache lse", f64(lse), rl, "bf16", what="lse")
