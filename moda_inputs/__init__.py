"""Seeded synthetic inputs for the MoDA attention path.

This module is shared by the oracle (``oracle/``), the tests and the bench. It
holds NO arithmetic of the method: it only draws Gaussian tensors in a fixed
order from a seeded CPU generator, rounds them to the storage dtype, and picks
seeded query-row samples. Everything that computes attention lives elsewhere.

Recipe (the same for every workload):
  * one ``torch.Generator('cpu')`` per workload, seeded with ``seed``;
  * ``randn`` in fp32, drawn in the order q, k, v, kd, vd, dout;
  * kd is multiplied by ``depth_std`` (1.0 for the timed workloads; the
    depth-stress cases use 4.0 so that depth keys dominate the softmax);
  * cast to the storage dtype (bf16 rounds to nearest even);
  * ``scale = 1/sqrt(d)``.

Tensor layouts (row-major, contiguous):
  q    [B, T, Hq, d]        k, v   [B, T, Hkv, d]
  kd   [B, T, Ld, Hkv, d]   vd     [B, T, Ld, Hkv, d]
  dout [B, T, Hq, d]
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "sample_rows", "workload", "make_depth_sel",
           "pack_depth_sel"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    d: int
    Ld: int
    dtype: str  # "bf16" or "f32"
    seed: int
    backward: bool = False
    depth_std: float = 1.0
    note: str = ""

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self) -> torch.dtype:
        return {"bf16": torch.bfloat16, "f32": torch.float32}[self.dtype]

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five synthetic workloads of the MoDA attention path (tiny fp32, 4K, 2x16K,
# 64K long context, and the wide-GQA forward+backward case).  Seeds are
# 1000 + workload index.
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 128, 4, 1, 64, 4, "f32", 1000,
                         note="tiny fp32 forward, G=4, d=64, Ld=4"),
    "t4k": Workload("t4k", 1, 4096, 32, 4, 128, 16, "bf16", 1001,
                    note="bf16 forward T=4096 G=8 Ld=16"),
    "t16k_b2": Workload("t16k_b2", 2, 16384, 32, 4, 128, 24, "bf16", 1002,
                        note="bf16 forward B=2 T=16384 G=8 Ld=24 (and Ld=0)"),
    "t64k": Workload("t64k", 1, 65536, 32, 4, 128, 28, "bf16", 1003,
                     note="bf16 forward long context T=65536 G=8 Ld=28"),
    "g32_fwdbwd": Workload("g32_fwdbwd", 1, 8192, 32, 1, 128, 28, "bf16", 1004,
                           backward=True,
                           note="bf16 forward+backward T=8192 G=32 Ld=28"),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def make_inputs(w: Workload, with_dout: bool | None = None) -> dict:
    """Draw the inputs of workload ``w`` on the CPU.

    Returns a dict with q, k, v, kd, vd (and dout when ``with_dout`` or
    ``w.backward``) as contiguous CPU tensors of ``w.torch_dtype``. ``kd`` and
    ``vd`` have a zero-length depth axis when ``w.Ld == 0``; the draw order is
    unchanged by ``Ld`` for q, k, v.
    """
    if with_dout is None:
        with_dout = w.backward
    g = torch.Generator("cpu")
    g.manual_seed(w.seed)
    dt = w.torch_dtype
    shapes = [
        ("q", (w.B, w.T, w.Hq, w.d)),
        ("k", (w.B, w.T, w.Hkv, w.d)),
        ("v", (w.B, w.T, w.Hkv, w.d)),
        ("kd", (w.B, w.T, w.Ld, w.Hkv, w.d)),
        ("vd", (w.B, w.T, w.Ld, w.Hkv, w.d)),
    ]
    if with_dout:
        shapes.append(("dout", (w.B, w.T, w.Hq, w.d)))
    out = {}
    for name, shp in shapes:
        x = torch.randn(shp, generator=g, dtype=torch.float32)
        if name == "kd" and w.depth_std != 1.0:
            x.mul_(w.depth_std)
        out[name] = x.to(dt).contiguous()
    return out


def sample_rows(w: Workload, n_rows: int = 256, n_head: int = 16) -> list[int]:
    """Seeded query-row sample used for long sequences.

    Rows ``0..n_head-1`` and ``T-1`` always appear (the first rows are where
    the depth keys carry the most weight); the rest are uniform draws without
    replacement from ``[n_head, T-1)`` with a generator seeded at ``seed+1``.
    Returns a sorted list of distinct positions.
    """
    T = w.T
    if T <= n_rows:
        return list(range(T))
    head = list(range(min(n_head, T)))
    rest_n = n_rows - len(head) - 1
    g = torch.Generator("cpu")
    g.manual_seed(w.seed + 1)
    pool = torch.arange(n_head, T - 1)
    pick = pool[torch.randperm(pool.numel(), generator=g)[:rest_n]].tolist()
    return sorted(set(head + pick + [T - 1]))


def make_depth_sel(w: Workload, kind: str = "random", density: float = 0.5, seed_offset: int = 2):
    """Seeded per-token depth selection [B, T, Ld] (bool).

    kind "random": each depth entry kept with probability ``density``;
    "window": each token keeps a contiguous window of its most recent
    entries (the last W of Ld, W uniform in [0, Ld]); "all"; "none".
    """
    g = torch.Generator("cpu")
    g.manual_seed(w.seed + seed_offset)
    shape = (w.B, w.T, w.Ld)
    if kind == "all":
        return torch.ones(shape, dtype=torch.bool)
    if kind == "none":
        return torch.zeros(shape, dtype=torch.bool)
    if kind == "random":
        return torch.rand(shape, generator=g) < density
    if kind == "window":
        width = torch.randint(0, w.Ld + 1, (w.B, w.T, 1), generator=g)
        i = torch.arange(w.Ld).view(1, 1, -1)
        return i >= (w.Ld - width)
    raise ValueError(kind)


def pack_depth_sel(sel) -> torch.Tensor:
    """[B, T, Ld] bool -> [B, T] int64 bit masks (bit i = entry i), Ld <= 64."""
    B, T, Ld = sel.shape
    if Ld > 64:
        raise ValueError("bit masks hold at most 64 depth entries")
    bits = torch.zeros((B, T), dtype=torch.int64)
    for i in range(Ld):
        bits |= sel[:, :, i].to(torch.int64) << i
    return bits
