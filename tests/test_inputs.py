"""Host-side input generators used by the tests and the bench: seeded, and
the depth-selection masks pack bit i = slot i."""
import torch

from moda_inputs import WORKLOADS, Workload, make_depth_sel, make_inputs, pack_depth_sel


def test_inputs_are_seeded_and_shaped():
    w = Workload("gen", 2, 9, 4, 2, 16, 3, "bf16", 5, depth_std=2.0)
    a, b = make_inputs(w, with_dout=True), make_inputs(w, with_dout=True)
    for name in ("q", "k", "v", "kd", "vd", "dout"):
        assert torch.equal(a[name], b[name]), name
    assert a["q"].shape == (2, 9, 4, 16) and a["k"].shape == (2, 9, 2, 16)
    assert a["kd"].shape == (2, 9, 3, 2, 16) and a["q"].dtype == torch.bfloat16
    assert WORKLOADS["t64k"].T == 65536 and WORKLOADS["t64k"].Ld == 28


def test_depth_selection_kinds_and_packing():
    w = Workload("sel", 2, 40, 4, 1, 16, 64, "bf16", 6)
    allsel, nonesel = make_depth_sel(w, "all"), make_depth_sel(w, "none")
    assert bool(allsel.all()) and not bool(nonesel.any())
    win = make_depth_sel(w, "window")
    # a window keeps the most recent slots: once a slot is kept, every later one is
    for row in win.reshape(-1, w.Ld):
        kept = row.nonzero().flatten()
        if len(kept):
            assert kept.tolist() == list(range(int(kept[0]), w.Ld))
    rnd = make_depth_sel(w, "random", density=0.5)
    assert 0.3 < rnd.float().mean().item() < 0.7
    assert torch.equal(rnd, make_depth_sel(w, "random", density=0.5))
    bits = pack_depth_sel(rnd)
    assert bits.dtype == torch.int64 and bits.shape == (2, 40)
    for i in range(w.Ld):
        got = ((bits >> i) & 1).bool()
        assert torch.equal(got, rnd[:, :, i]), i
    assert int(pack_depth_sel(allsel)[0, 0]) == -1  # all 64 bits set
