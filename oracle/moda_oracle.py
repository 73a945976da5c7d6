"""Float64 CPU oracle for Mixture-of-Depths Attention (MoDA).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` may import or call this module. The
product path (``depth_kv_attention_b200``) never touches it, and this module
imports nothing from the product.

What it computes (the "read" step of MoDA):

  For every batch b, query head h, position t, with kv-head g = h // G
  (G = Hq / Hkv, contiguous head groups):

    s_j   = scale * <q[b,t,h], k[b,j,g]>          j = 0..t      (causal)
    s'_i  = scale * <q[b,t,h], kd[b,t,i,g]>       i = 0..Ld-1   (same token)
    one softmax over the concatenation [s || s']
    out[b,t,h] = sum_j p_j v[b,j,g] + sum_i p'_i vd[b,t,i,g]
    lse[b,h,t] = log( sum_j e^{s_j} + sum_i e^{s'_i} )     (natural log)

Sources:
  * "动态混合深度注意力机制MoDA技术解析" (mhpn.cn blog), §1.2: the MoDA attention
    formula, a single softmax over the concatenated logits of the current
    layer's keys and the keys of the preceding layers, divided by sqrt(d),
    times the concatenated values.
  * same page, §2.2 "dual mask": the sequence mask lets a token see itself and
    earlier positions; the depth mask lets a query see only the depth entries
    of its own position.
  * "Mixture-of-Depths Attention" (gist.science, German technical summary),
    §2 "Methodik", Read-Step and Unified Softmax: a query at position t reads
    the depth keys/values of the same position t from layers 0..l-1, and both
    score sets are normalised by one softmax.
  * "Mixture-of-Depths Attention" (gist.science, French technical summary),
    §2 "Méthodologie", Opération: one unified softmax over sequence and depth.

Selected depth (the pages' future-work item, "Mixture-of-Depths Attention",
gist.science German summary §5: bounded depth-KV slots, e.g. a sliding window
over layers or a dynamic selection): an optional ``depth_sel`` [B, T, Ld] of
booleans keeps depth entry i of token t only where depth_sel[b,t,i] is true;
the other depth logits leave the softmax (as if that slot were absent).

Readings where the pages are silent:
  * the depth logits take the same ``scale`` as the sequence logits (the §1.2
    formula divides the whole concatenation by sqrt(d));
  * GQA maps query head h to kv-head h // G;
  * ``lse`` is the natural log of the softmax denominator of the scaled logits;
  * the backward pass is the derivative of the forward above (the pages give
    none); it is pinned by central finite differences in the tests.

All arithmetic is float64. Inputs may be numpy arrays or torch tensors of any
float dtype; they are upcast exactly (bf16 -> float32 -> float64 is exact).
The concatenated logit row is materialised explicitly, in blocks of at most
``row_block`` query rows per (b, h), and normalised with a two-pass softmax.
"""
from __future__ import annotations

import numpy as np

__all__ = ["to_f64", "forward", "forward_rows", "backward", "depth_write", "quantize_q8",
           "dequantize_q8", "depth_write_q8", "round_to_bf16"]


def to_f64(x) -> np.ndarray:
    """Exact upcast of a numpy array or torch tensor to a float64 array."""
    if hasattr(x, "detach"):  # torch tensor, without importing torch here
        x = x.detach().to("cpu")
        if str(x.dtype) in ("torch.bfloat16", "torch.float16"):
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _dims(q, k, kd):
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    Ld = kd.shape[2]
    return B, T, Hq, Hkv, Hq // Hkv, d, Ld


def _concat_logits(qr, kseq, kdep, scale, ts, sel=None):
    """Concatenated logit rows [sequence || depth] for query rows ``qr``.

    qr   [R, d]   query vectors of positions ``ts`` (one head)
    kseq [J, d]   sequence keys 0..J-1 of the head's kv-head
    kdep [R, Ld, d] depth keys of the SAME positions ``ts``
    sel  [R, Ld] booleans or None: depth entries kept for each row's position
    Returns s [R, J + Ld] with -inf where the causal mask hides a key or a
    depth entry is not selected.
    """
    s_seq = scale * (qr @ kseq.T)                            # [R, J]
    j = np.arange(kseq.shape[0])
    s_seq = np.where(j[None, :] <= np.asarray(ts)[:, None], s_seq, -np.inf)
    s_dep = scale * np.einsum("rc,ric->ri", qr, kdep)        # [R, Ld]
    if sel is not None:
        s_dep = np.where(sel, s_dep, -np.inf)
    return np.concatenate([s_seq, s_dep], axis=1)


def _sel(depth_sel, b, t0, t1):
    return None if depth_sel is None else np.asarray(depth_sel[b, t0:t1], dtype=bool)


def _softmax_rows(s):
    """Two-pass softmax of each row; returns (p, lse)."""
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=1, keepdims=True)
    return e / z, (m + np.log(z))[:, 0]


def forward(q, k, v, kd, vd, scale: float, row_block: int = 256, depth_sel=None):
    """Full MoDA forward. Returns (out [B,T,Hq,d], lse [B,Hq,T]) in float64.

    ``depth_sel`` (optional, [B,T,Ld] bool): depth entries each position keeps."""
    q, k, v, kd, vd = (to_f64(x) for x in (q, k, v, kd, vd))
    B, T, Hq, Hkv, G, d, Ld = _dims(q, k, kd)
    out = np.empty((B, T, Hq, d))
    lse = np.empty((B, Hq, T))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for t0 in range(0, T, row_block):
                t1 = min(T, t0 + row_block)
                ts = np.arange(t0, t1)
                s = _concat_logits(q[b, t0:t1, h], k[b, :t1, g],
                                   kd[b, t0:t1, :, g], scale, ts, _sel(depth_sel, b, t0, t1))
                p, l = _softmax_rows(s)
                vals = p[:, :t1] @ v[b, :t1, g]
                vals += np.einsum("ri,ric->rc", p[:, t1:], vd[b, t0:t1, :, g])
                out[b, t0:t1, h] = vals
                lse[b, h, t0:t1] = l
    return out, lse


def forward_rows(q, k, v, kd, vd, scale: float, b: int, h: int, ts, depth_sel=None):
    """MoDA forward for selected positions ``ts`` of one (b, h).

    Same definition as ``forward``; used to check long sequences on sampled
    rows. Returns (out [R, d], lse [R]).
    """
    ts = np.asarray(sorted(int(t) for t in ts))
    idx = [int(t) for t in ts]
    Hq, Hkv = q.shape[2], k.shape[2]
    g = h // (Hq // Hkv)
    jmax = int(ts.max()) + 1
    qr = to_f64(q[b][idx])[:, h]
    kseq = to_f64(k[b, :jmax, g])
    vseq = to_f64(v[b, :jmax, g])
    kdep = to_f64(kd[b][idx])[:, :, g]
    vdep = to_f64(vd[b][idx])[:, :, g]
    sel = None if depth_sel is None else np.asarray(depth_sel[b][idx], dtype=bool)
    s = _concat_logits(qr, kseq, kdep, scale, ts, sel)
    p, l = _softmax_rows(s)
    vals = p[:, :jmax] @ vseq + np.einsum("ri,ric->rc", p[:, jmax:], vdep)
    return vals, l


def backward(q, k, v, kd, vd, dout, scale: float, row_block: int = 256, out_for_D=None,
             depth_sel=None):
    """Gradients of the MoDA forward for upstream gradient ``dout``.

    ``depth_sel`` (optional, [B,T,Ld] bool): as in ``forward``; unselected
    depth entries get zero gradients.

    ``out_for_D`` (optional, [B,T,Hq,d]): the forward output to form
    D = <dout, out> from. By default D uses the exact float64 forward output,
    which makes the result the exact derivative. A backward that receives the
    forward output as stored (e.g. rounded to bf16) forms D from that stored
    output instead; passing it here gives the oracle of that definition.

    The pages describe no backward pass; this is the derivative of the
    forward definition above (softmax Jacobian), written per row block:

      P   = exp(s - lse)                  (the forward's probabilities)
      D   = <dout, out>                   per row
      dP  = [dout . v_j  ||  dout . vd_i]
      dS  = P * (dP - D)
      dq  = scale * (sum_j dS_j k_j + sum_i dS'_i kd_i)
      dk_j  += scale * dS_j q      dv_j  += P_j dout      (summed over rows)
      dkd_i += scale * dS'_i q     dvd_i += P'_i dout     (same position)

    Returns (dq, dk, dv, dkd, dvd, out, lse), all float64.
    """
    q, k, v, kd, vd, dout = (to_f64(x) for x in (q, k, v, kd, vd, dout))
    B, T, Hq, Hkv, G, d, Ld = _dims(q, k, kd)
    out, lse = forward(q, k, v, kd, vd, scale, row_block, depth_sel)
    outD = out if out_for_D is None else to_f64(out_for_D)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dkd = np.zeros_like(kd)
    dvd = np.zeros_like(vd)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for t0 in range(0, T, row_block):
                t1 = min(T, t0 + row_block)
                ts = np.arange(t0, t1)
                qr = q[b, t0:t1, h]
                dor = dout[b, t0:t1, h]
                s = _concat_logits(qr, k[b, :t1, g], kd[b, t0:t1, :, g], scale, ts,
                                   _sel(depth_sel, b, t0, t1))
                P = np.exp(s - lse[b, h, t0:t1][:, None])
                D = np.sum(dor * outD[b, t0:t1, h], axis=1)
                dP_seq = dor @ v[b, :t1, g].T
                dP_dep = np.einsum("rc,ric->ri", dor, vd[b, t0:t1, :, g])
                dP = np.concatenate([dP_seq, dP_dep], axis=1)
                dS = P * (dP - D[:, None])
                dS_seq, dS_dep = dS[:, :t1], dS[:, t1:]
                P_seq, P_dep = P[:, :t1], P[:, t1:]
                dq[b, t0:t1, h] = scale * (dS_seq @ k[b, :t1, g]
                                           + np.einsum("ri,ric->rc", dS_dep, kd[b, t0:t1, :, g]))
                dk[b, :t1, g] += scale * (dS_seq.T @ qr)
                dv[b, :t1, g] += P_seq.T @ dor
                dkd[b, t0:t1, :, g] += scale * dS_dep[:, :, None] * qr[:, None, :]
                dvd[b, t0:t1, :, g] += P_dep[:, :, None] * dor[:, None, :]
    return dq, dk, dv, dkd, dvd, out, lse


def depth_write(kd, vd, k, v, slot: int):
    """The write step ("Mixture-of-Depths Attention", gist.science German
    summary §2, Write-Step): the layer's keys / values k, v [B,T,Hkv,d] are
    appended to the depth stream as slot ``slot`` of every token's depth
    entries. Returns new arrays kd', vd' [B,T,Ld,Hkv,d] equal to kd, vd except
    kd'[:, :, slot] = k and vd'[:, :, slot] = v (values unchanged: a copy)."""
    kd2 = np.array(kd, copy=True)
    vd2 = np.array(vd, copy=True)
    kd2[:, :, slot] = np.asarray(k)
    vd2[:, :, slot] = np.asarray(v)
    return kd2, vd2


# ------------------------------------------------------------ 8-bit depth KV
#
# "动态混合深度注意力机制MoDA技术解析" (mhpn.cn) §4.2 (memory tips): where device
# memory is short, the depth KV of models beyond 32 layers can be stored with
# 8-bit quantisation. The page names no format. Reading used here: symmetric
# per-row absmax int8, one float32 scale per (b, t, slot, kv-head) row of d
# values:
#
#   amax   = max_c |x_c|                     (x: the row in float32)
#   sigma  = fl32(amax / 127)                (0 for an all-zero row)
#   code_c = clamp(round_half_even(fl32(x_c / sigma)), -127, 127)
#   x^_c   = the cache's storage dtype of fl32(sigma * code_c)
#            (bf16, round to nearest even, for a bf16 cache; float32 itself
#             for a float32 cache): the 8-bit cache decompresses into the
#             same type the unquantised depth cache holds
#
# fl32 is one IEEE float32 operation, rounded to nearest even: both sides of
# a comparison take every decision that fixes a code or a value in float32.
# The attention itself is the unchanged MoDA read step over the dequantised
# depth keys and values x^.


def quantize_q8(x):
    """Symmetric per-row int8 quantisation of the last axis of ``x`` (a float
    array or tensor; bf16 is upcast exactly). Returns (codes int8 [..., d],
    scales float32 [...])."""
    xf = np.asarray(to_f64(x), dtype=np.float64).astype(np.float32)  # exact for bf16 / f32 inputs
    amax = np.max(np.abs(xf), axis=-1)
    sigma = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(sigma > 0, sigma, np.float32(1.0)).astype(np.float32)
    r = (xf / safe[..., None]).astype(np.float32)
    codes = np.clip(np.rint(r), -127, 127)                       # rint: ties to even
    codes = np.where(sigma[..., None] > 0, codes, 0).astype(np.int8)
    return codes, sigma


def round_to_bf16(x32):
    """float32 -> the nearest bf16 value (ties to even mantissa), returned as
    float32: keep the upper 16 bits of the float32 pattern after adding half
    of the dropped range plus the parity of the kept bit (finite inputs)."""
    b = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def dequantize_q8(codes, scales, dtype: str = "bf16"):
    """x^ = fl32(scale * code) in the cache's storage dtype ("bf16" or
    "f32"), returned exactly as float64 [..., d]."""
    prod = (np.asarray(codes, dtype=np.float32)
            * np.asarray(scales, dtype=np.float32)[..., None]).astype(np.float32)
    if dtype == "bf16":
        prod = round_to_bf16(prod)
    elif dtype != "f32":
        raise ValueError(dtype)
    return prod.astype(np.float64)


def depth_write_q8(kd8, vd8, kd_scale, vd_scale, k, v, slot: int):
    """The write step into an 8-bit depth cache: k, v [B,T,Hkv,d] quantised
    row by row (``quantize_q8``) into slot ``slot`` of the codes kd8, vd8
    [B,T,Ld,Hkv,d] and scales kd_scale, vd_scale [B,T,Ld,Hkv]. Returns new
    arrays (kd8', vd8', kd_scale', vd_scale'); other slots unchanged."""
    out = [np.array(a, copy=True) for a in (kd8, vd8, kd_scale, vd_scale)]
    ck, sk = quantize_q8(k)
    cv, sv = quantize_q8(v)
    out[0][:, :, slot] = ck
    out[1][:, :, slot] = cv
    out[2][:, :, slot] = sk
    out[3][:, :, slot] = sv
    return tuple(out)
