"""C-ABI checks that need no GPU: the library loads, exports every function
that include/moda.h declares, and rejects bad arguments synchronously with
the documented status codes before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moda.h")

moda = pytest.importorskip("depth_kv_attention_b200",
                           reason="libmoda.so not built (python depth_kv_attention_b200/csrc/build.py)")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(moda_[a-z0-9_]+)\s*\(",
                                 src, flags=re.M)))


def test_header_declares_the_abi():
    fns = declared_functions()
    for name in ["moda_fwd", "moda_fwd_sel", "moda_bwd", "moda_bwd_sel", "moda_bwd_workspace_bytes", "moda_pack_depth",
                 "moda_fwd_packed", "moda_device_status", "moda_status_string"]:
        assert name in fns


def test_every_declared_symbol_is_exported():
    lib = ctypes.CDLL(moda.LIB_PATH)
    missing = [f for f in declared_functions() if not hasattr(lib, f)]
    assert not missing, missing


def test_version_and_status_strings():
    assert moda.moda_abi_version() == 3
    assert moda.moda_status_string(0) == "MODA_OK"
    assert moda.moda_status_string(6) == "MODA_ERR_DEVICE_TIMEOUT"
    assert moda.moda_status_string(99) == "MODA_ERR_UNKNOWN"


# Fake, 16-byte aligned "device" addresses: validation rejects the call before
# any CUDA call or dereference, so they are never used.
P = 0x10000


def fwd(q=P, k=P, v=P, kd=P, vd=P, B=1, T=8, Hq=4, Hkv=2, d=64, Ld=2, dt=0, scale=0.125,
        out=P, lse=P, impl=0):
    return moda._c_fwd_ex(q, k, v, kd, vd, B, T, Hq, Hkv, d, Ld, dt, scale, out, lse, None, impl)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(kd=None), 1), (dict(vd=None), 1),
    (dict(B=0), 1), (dict(T=0), 1), (dict(Hq=3, Hkv=2), 1), (dict(Ld=-1), 1), (dict(d=0), 1),
    (dict(dt=7), 1), (dict(scale=float("nan")), 1), (dict(impl=9), 1),
    (dict(d=256), 2),
    (dict(q=P + 2), 3), (dict(kd=P + 8), 3), (dict(lse=P + 4), 3), (dict(out=P + 1), 3),
])
def test_fwd_validation(kw, code):
    assert fwd(**kw) == code


def bwd(ws=P, ws_bytes=1 << 30, dq=P, dkd=P, Ld=2, **kw):
    dims = dict(B=1, T=8, Hq=4, Hkv=2, d=64)
    dims.update(kw)
    return moda._c_bwd_ex(P, P, P, P, P, P, P, P, dims["B"], dims["T"], dims["Hq"], dims["Hkv"],
                          dims["d"], Ld, 0, 0.125, dq, P, P, dkd, P, ws, ws_bytes, None, 0)


def test_bwd_validation():
    assert bwd(ws=None) == 4
    assert bwd(ws_bytes=16) == 4
    assert bwd(dq=None) == 1
    assert bwd(dkd=None) == 1
    assert bwd(dq=P + 4) == 3
    assert bwd(ws=P + 8) == 3


def test_workspace_and_pack_sizes():
    # fp32 row statistics [B,Hq,T] (256-byte rounded) + fp32 dk, dv accumulators for bf16
    assert moda._c_bwd_ws(1, 8, 4, 2, 64, 2, 0) == 256 + 8 * (2 * 2) * 64 * 4
    assert moda._c_bwd_ws(1, 8, 4, 2, 64, 2, 1) == 256
    assert moda._c_bwd_ws(1, 8, 3, 2, 64, 2, 0) == 0
    assert moda._c_pack_bytes(2, 5, 3, 128, 7, 0) == 2 * 2 * 5 * 7 * 3 * 128 * 2
    assert moda._c_pack(P, P, 1, 4, 1, 128, 2, 0, P + 8, None) == 3
    assert moda._c_pack(P, P, 1, 4, 1, 6, 2, 0, P, None) == 2


def fwd_sel(sel=P, Ld=2, d=64, q=P):
    return moda._c_fwd_sel(q, P, P, P, P, sel, 1, 8, 4, 2, d, Ld, 0, 0.125, P, P, None, 0)


def bwd_sel(sel=P, Ld=2, dq=P):
    return moda._c_bwd_sel(P, P, P, P, P, sel, P, P, P, 1, 8, 4, 2, 64, Ld, 0, 0.125, dq, P, P, P, P,
                           P, 1 << 30, None, 0)


def test_selection_validation():
    """Depth-slot masks: 8-byte aligned, at most 64 slots; the checks of the
    unselected entry points still apply."""
    assert fwd_sel(sel=P + 4) == 3
    assert fwd_sel(Ld=65) == 2
    assert fwd_sel(d=0) == 1
    assert fwd_sel(q=P + 2) == 3
    assert bwd_sel(sel=P + 4) == 3
    assert bwd_sel(Ld=65) == 2
    assert bwd_sel(dq=None) == 1


def depth_write(slot=1, Ld=3, d=64, dt=0, k=P, kd=P):
    return moda._c_depth_write(k, P, 2, 5, 2, d, Ld, slot, dt, kd, P, None)


def test_depth_write_validation():
    """The write step rejects a slot outside [0, Ld), NULL or misaligned
    buffers, and rows that are not whole 16-byte vectors."""
    assert depth_write(slot=3) == 1
    assert depth_write(slot=-1) == 1
    assert depth_write(Ld=0, slot=0) == 1
    assert depth_write(k=None) == 1
    assert depth_write(kd=P + 8) == 3
    assert depth_write(d=12) == 2          # 24 bytes per bf16 row


def fwd_host(staging=P, staging_bytes=1 << 30, q=P, B=1, T=8, Hq=4, Hkv=2, d=64, Ld=2, dt=0):
    return moda._c_fwd_host(q, P, P, P, P, B, T, Hq, Hkv, d, Ld, dt, 0.125, P, P, staging,
                            staging_bytes, None)


def test_fwd_host_staging_size_and_validation():
    """moda_fwd_host stages q, k, v, kd, vd, out and lse at 256-byte-aligned
    offsets of the caller's device buffer; a missing, short or misaligned
    staging buffer and bad shapes are rejected before any copy."""
    B, T, Hq, Hkv, d, Ld = 1, 8, 4, 2, 64, 2
    r = lambda n: (n + 255) // 256 * 256  # noqa: E731
    want = (2 * r(B * T * Hq * d * 2) + 2 * r(B * T * Hkv * d * 2) + 2 * r(B * T * Ld * Hkv * d * 2)
            + r(B * Hq * T * 4))
    assert moda._c_host_bytes(B, T, Hq, Hkv, d, Ld, 0) == want
    assert moda._c_host_bytes(B, T, 3, Hkv, d, Ld, 0) == 0
    assert fwd_host(staging=None) == 4
    assert fwd_host(staging_bytes=want - 1) == 4
    assert fwd_host(staging=P + 16) == 3
    assert fwd_host(q=None) == 1
    assert fwd_host(Hq=3) == 1
    assert fwd_host(d=256) == 2


def test_q8_validation():
    """8-bit depth entry points: NULL / misaligned scales and codes, slots
    outside [0, Ld), unsupported d."""
    fq = lambda ks=P, kd8=P, Ld=2: moda._c_fwd_q8(P, P, P, kd8, P, ks, P, 1, 8, 4, 2, 64, Ld, 0, 0.125,  # noqa: E731
                                                   P, P, None, 0)
    assert fq(ks=None) == 1
    assert fq(ks=P + 2) == 3
    assert fq(kd8=P + 8) == 3
    assert fq(kd8=None) == 1
    qz = lambda kd8=P, ks=P, d=64: moda._c_quant_q8(P, P, 1, 4, 2, d, 2, 0, kd8, P, ks, P, None)  # noqa: E731
    assert qz(kd8=None) == 1
    assert qz(ks=P + 1) == 3
    assert qz(d=256) == 2
    wq = lambda slot=0, Ld=2: moda._c_write_q8(P, P, 1, 4, 2, 64, Ld, slot, 0, P, P, P, P, None)  # noqa: E731
    assert wq(slot=2) == 1
    assert wq(slot=-1) == 1
    assert wq(Ld=0) == 1


def test_slot_layout_is_the_native_slot():
    import torch
    """moda_depth_slot_layout's offset and strides address exactly
    kd[:, :, slot] of the native cache (CPU: a view on a host tensor)."""
    kd = torch.arange(2 * 5 * 3 * 2 * 4).reshape(2, 5, 3, 2, 4)
    for slot in range(3):
        assert torch.equal(moda.depth_slot_view(kd, slot), kd[:, :, slot])
    assert moda.moda_depth_slot_layout(2, 5, 2, 4, 3, 1) == (8, (120, 24, 4, 1))
    with pytest.raises(moda.ModaError):
        moda.moda_depth_slot_layout(2, 5, 2, 4, 3, 3)



def test_header_is_plain_c_and_links():
    """include/moda.h compiles as C99 and a C program links against
    libmoda.so and runs the argument checks (no GPU needed)."""
    import shutil
    import subprocess
    import tempfile
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = os.path.join(ROOT, "tests", "c", "abi_client.c")
    libdir = os.path.dirname(moda.LIB_PATH)
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "abi_client")
        r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                            "-o", exe, os.path.join(libdir, "libmoda.so"), f"-Wl,-rpath,{libdir}"],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
        assert r.returncode == 0, (r.stdout, r.stderr)
        assert r.stdout.split() == ["MODA_ERR_WORKSPACE", "0"]
