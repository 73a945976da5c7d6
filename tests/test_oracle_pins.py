"""Pins for the float64 oracle, none of which reuses the oracle's own code.

Each test ties the oracle to something fixed outside it: a hand-worked
example, a library routine that computes a special case (scaled dot-product
attention), the pages' flash-compatible flattened view of the depth keys,
closed forms, invariants, and brute-force scalar loops.  A final group plants
plausible mistakes in the oracle (monkeypatched, CPU only) and checks that the
pins catch them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.moda_oracle as om
from moda_inputs import Workload, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(B, T, Hq, Hkv, d, Ld, seed, depth_std=1.0):
    w = Workload("pin", B, T, Hq, Hkv, d, Ld, "f32", seed, depth_std=depth_std)
    x = make_inputs(w, with_dout=True)
    return {k: om.to_f64(v) for k, v in x.items()}, w.scale


def sdpa_f64(q, k, v, mask_or_bias):
    """torch scaled_dot_product_attention in float64 on CPU, per head.

    q [Tq, d], k/v [Tk, d]; ``mask_or_bias`` is a bool mask (True = attend)
    or an additive float bias [Tq, Tk]."""
    qt = torch.from_numpy(q)[None, None]
    kt = torch.from_numpy(k)[None, None]
    vt = torch.from_numpy(v)[None, None]
    m = torch.from_numpy(mask_or_bias)[None, None]
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=1.0)[0, 0].numpy()


# ----------------------------------------------------------------- golden
def test_hand_worked_example():
    """A T=2, G=2, Ld=1 example worked by hand with exact fractions."""
    with open(os.path.join(GOLDEN, "hand_worked_t2_d2.json")) as f:
        g = json.load(f)
    x = {k: np.array(v, dtype=np.float64) for k, v in g["inputs"].items() if k != "scale"}
    out, lse = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], g["inputs"]["scale"])
    exp_out = np.vectorize(lambda s: float(Fraction(s)))(np.array(g["expected"]["out_fractions"]))
    exp_lse = np.log(np.array(g["expected"]["lse_of"], dtype=np.float64))
    np.testing.assert_allclose(out, exp_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, exp_lse, rtol=0, atol=1e-12)


# ------------------------------------------------------- library special cases
@pytest.mark.parametrize("B,T,Hq,Hkv,d", [(1, 37, 4, 2, 16), (2, 19, 6, 3, 8), (1, 24, 8, 1, 32)])
def test_ld0_is_causal_attention(B, T, Hq, Hkv, d):
    """Ld=0 reduces to causal softmax attention (GQA group h // G)."""
    x, scale = rand_case(B, T, Hq, Hkv, d, 0, seed=11)
    out, lse = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale)
    G = Hq // Hkv
    causal = np.tril(np.ones((T, T), dtype=bool))
    for b in range(B):
        for h in range(Hq):
            ref = sdpa_f64(x["q"][b, :, h] * scale, x["k"][b, :, h // G], x["v"][b, :, h // G], causal)
            np.testing.assert_allclose(out[b, :, h], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("B,T,Hq,Hkv,d,Ld", [(1, 9, 4, 2, 8, 3), (2, 6, 2, 1, 5, 4), (1, 13, 3, 3, 4, 1)])
def test_flash_compatible_flattened_view(B, T, Hq, Hkv, d, Ld):
    """The pages' flash-compatible view: depth keys flattened along one T*Ld
    axis appended to the sequence keys, with an explicit mask (causal on the
    first T columns; column T + t'*Ld + i visible to row t iff t' == t)."""
    x, scale = rand_case(B, T, Hq, Hkv, d, Ld, seed=12)
    out, _ = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale)
    G = Hq // Hkv
    mask = np.zeros((T, T + T * Ld), dtype=bool)
    mask[:, :T] = np.tril(np.ones((T, T), dtype=bool))
    for t in range(T):
        mask[t, T + t * Ld: T + (t + 1) * Ld] = True
    for b in range(B):
        for h in range(Hq):
            g = h // G
            kk = np.concatenate([x["k"][b, :, g], x["kd"][b, :, :, g].reshape(T * Ld, d)])
            vv = np.concatenate([x["v"][b, :, g], x["vd"][b, :, :, g].reshape(T * Ld, d)])
            ref = sdpa_f64(x["q"][b, :, h] * scale, kk, vv, mask)
            np.testing.assert_allclose(out[b, :, h], ref, rtol=0, atol=1e-12)


def test_depth_copies_of_own_key_add_log_bias():
    """kd[t,i]=k[t], vd[t,i]=v[t] for all i equals causal attention with
    ln(1+Ld) added to the diagonal logit."""
    T, d, Ld = 21, 8, 5
    x, scale = rand_case(1, T, 2, 1, d, Ld, seed=13)
    kd = np.repeat(x["k"][:, :, None], Ld, axis=2)
    vd = np.repeat(x["v"][:, :, None], Ld, axis=2)
    out, lse = om.forward(x["q"], x["k"], x["v"], kd, vd, scale)
    bias = np.where(np.tril(np.ones((T, T), dtype=bool)), 0.0, -np.inf)
    bias[np.arange(T), np.arange(T)] = math.log(1 + Ld)
    for h in range(2):
        ref = sdpa_f64(x["q"][0, :, h] * scale, x["k"][0, :, 0], x["v"][0, :, 0], bias)
        np.testing.assert_allclose(out[0, :, h], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------ closed forms
def test_t1_closed_form():
    """T=1, Ld=1: softmax over {self, one depth entry} by hand."""
    rng = np.random.default_rng(5)
    q, k, v, kd, vd = (rng.standard_normal(s) for s in
                       [(1, 1, 1, 7), (1, 1, 1, 7), (1, 1, 1, 7), (1, 1, 1, 1, 7), (1, 1, 1, 1, 7)])
    scale = 0.37
    a = scale * sum(q[0, 0, 0, c] * k[0, 0, 0, c] for c in range(7))
    bb = scale * sum(q[0, 0, 0, c] * kd[0, 0, 0, 0, c] for c in range(7))
    ea, eb = math.exp(a), math.exp(bb)
    want = (ea * v[0, 0, 0] + eb * vd[0, 0, 0, 0]) / (ea + eb)
    out, lse = om.forward(q, k, v, kd, vd, scale)
    np.testing.assert_allclose(out[0, 0, 0], want, rtol=0, atol=1e-13)
    assert abs(lse[0, 0, 0] - math.log(ea + eb)) < 1e-13


def test_zero_depth_keys_closed_form():
    """kd = 0 gives every depth logit the value 0: Z = sum_j e^{s_j} + Ld."""
    T, d, Ld = 11, 6, 3
    x, scale = rand_case(1, T, 2, 2, d, Ld, seed=14)
    kd = np.zeros_like(x["kd"])
    out, lse = om.forward(x["q"], x["k"], x["v"], kd, x["vd"], scale)
    for h in range(2):
        for t in range(T):
            es = [math.exp(scale * float(np.dot(x["q"][0, t, h], x["k"][0, j, h]))) for j in range(t + 1)]
            Z = sum(es) + Ld
            num = sum(e * x["v"][0, j, h] for j, e in enumerate(es)) + x["vd"][0, t, :, h].sum(axis=0)
            np.testing.assert_allclose(out[0, t, h], num / Z, rtol=0, atol=1e-12)
            assert abs(lse[0, h, t] - math.log(Z)) < 1e-12


# --------------------------------------------------------------- brute force
def brute_force(q, k, v, kd, vd, scale):
    """Scalar loops with an online (single-pass, running max) softmax, the
    depth entries visited FIRST: a different order and algorithm from the
    oracle's materialised two-pass softmax."""
    B, T, Hq, d = q.shape
    Hkv, Ld = k.shape[2], kd.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, T, Hq, d))
    lse = np.zeros((B, Hq, T))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for t in range(T):
                keys = [(kd[b, t, i, g], vd[b, t, i, g]) for i in range(Ld)]
                keys += [(k[b, j, g], v[b, j, g]) for j in range(t, -1, -1)]
                m, l, acc = -math.inf, 0.0, [0.0] * d
                for kk, vv in keys:
                    s = scale * sum(float(q[b, t, h, c]) * float(kk[c]) for c in range(d))
                    mn = max(m, s)
                    corr = math.exp(m - mn) if m != -math.inf else 0.0
                    p = math.exp(s - mn)
                    l = l * corr + p
                    acc = [a * corr + p * float(vv[c]) for c, a in enumerate(acc)]
                    m = mn
                out[b, t, h] = [a / l for a in acc]
                lse[b, h, t] = m + math.log(l)
    return out, lse


@pytest.mark.parametrize("B,T,Hq,Hkv,d,Ld,std", [(1, 6, 4, 2, 3, 2, 1.0), (2, 5, 2, 1, 4, 3, 4.0),
                                                  (1, 7, 3, 1, 2, 1, 2.0)])
def test_brute_force_scalar_loops(B, T, Hq, Hkv, d, Ld, std):
    x, scale = rand_case(B, T, Hq, Hkv, d, Ld, seed=15, depth_std=std)
    out, lse = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale)
    bo, bl = brute_force(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- invariants
def test_depth_permutation_invariance():
    x, scale = rand_case(2, 17, 4, 2, 8, 6, seed=16, depth_std=3.0)
    out, lse = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale)
    perm = np.random.default_rng(0).permutation(6)
    out2, lse2 = om.forward(x["q"], x["k"], x["v"], x["kd"][:, :, perm], x["vd"][:, :, perm], scale)
    np.testing.assert_allclose(out, out2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)


def test_lse_difference_and_convexity():
    """lse(Ld) - lse(0) = ln(1 + sum_i e^{s'_i} / sum_j e^{s_j}) >= 0, and
    every output coordinate lies in the hull of the attended values."""
    T, d, Ld = 15, 4, 3
    x, scale = rand_case(1, T, 2, 1, d, Ld, seed=17, depth_std=2.0)
    out, lse = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale)
    _, lse0 = om.forward(x["q"], x["k"], x["v"], x["kd"][:, :, :0], x["vd"][:, :, :0], scale)
    for h in range(2):
        for t in range(T):
            qv = x["q"][0, t, h]
            seq = sum(math.exp(scale * float(qv @ x["k"][0, j, 0])) for j in range(t + 1))
            dep = sum(math.exp(scale * float(qv @ x["kd"][0, t, i, 0])) for i in range(Ld))
            assert abs((lse[0, h, t] - lse0[0, h, t]) - math.log1p(dep / seq)) < 1e-12
            vals = np.concatenate([x["v"][0, :t + 1, 0], x["vd"][0, t, :, 0]])
            assert np.all(out[0, t, h] <= vals.max(axis=0) + 1e-12)
            assert np.all(out[0, t, h] >= vals.min(axis=0) - 1e-12)


def test_row_sampling_and_blocking_agree():
    x, scale = rand_case(2, 40, 4, 2, 8, 3, seed=18)
    out, lse = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, row_block=256)
    out3, lse3 = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, row_block=7)
    np.testing.assert_allclose(out, out3, rtol=0, atol=1e-13)
    ts = [0, 3, 17, 39]
    ro, rl = om.forward_rows(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, 1, 3, ts)
    np.testing.assert_allclose(ro, out[1, ts, 3], rtol=0, atol=1e-13)
    np.testing.assert_allclose(rl, lse[1, 3, ts], rtol=0, atol=1e-13)


# ------------------------------------------------------------------ backward
def _loss(x, dout, scale):
    out, _ = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale)
    return float(np.sum(out * dout))


@pytest.mark.parametrize("B,T,Hq,Hkv,d,Ld", [(1, 5, 4, 2, 3, 2), (2, 4, 2, 1, 2, 3)])
def test_backward_central_differences(B, T, Hq, Hkv, d, Ld):
    x, scale = rand_case(B, T, Hq, Hkv, d, Ld, seed=19, depth_std=2.0)
    dout = x.pop("dout")
    dq, dk, dv, dkd, dvd, _, _ = om.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], dout, scale)
    grads = {"q": dq, "k": dk, "v": dv, "kd": dkd, "vd": dvd}
    eps = 1e-6
    for name, gr in grads.items():
        base = x[name]
        num = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = base[idx]
            base[idx] = old + eps
            lp = _loss(x, dout, scale)
            base[idx] = old - eps
            lm = _loss(x, dout, scale)
            base[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(num - gr)) / max(1e-12, np.max(np.abs(gr)))
        assert err < 1e-6, (name, err)


def test_backward_sum_identities():
    """Shifting every value (sequence and depth) of a kv group by c shifts each
    output of the group by c, so sum(dv)+sum(dvd) = sum over the group's rows
    of dout; shifting every key by c adds the same amount to every logit of a
    row, so sum(dk)+sum(dkd) = 0."""
    x, scale = rand_case(2, 23, 6, 2, 5, 4, seed=20, depth_std=2.0)
    dq, dk, dv, dkd, dvd, _, _ = om.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale)
    G = 3
    for b in range(2):
        for g in range(2):
            sdo = x["dout"][b, :, g * G:(g + 1) * G].sum(axis=(0, 1))
            np.testing.assert_allclose(dv[b, :, g].sum(0) + dvd[b, :, :, g].sum((0, 1)), sdo, atol=1e-11)
            np.testing.assert_allclose(dk[b, :, g].sum(0) + dkd[b, :, :, g].sum((0, 1)), 0, atol=1e-11)


# ----------------------------------------------------- planted mistakes caught
def _pins_pass():
    try:
        test_hand_worked_example()
        test_brute_force_scalar_loops(1, 6, 4, 2, 3, 2, 1.0)
        test_flash_compatible_flattened_view(1, 9, 4, 2, 8, 3)
        return True
    except AssertionError:
        return False


def test_planted_mistakes_are_caught(monkeypatch):
    assert _pins_pass()
    orig = om._concat_logits

    mutants = {
        # causal mask dropped (token sees the future)
        "no_causal": lambda qr, ks, kdp, sc, ts, sel=None: np.concatenate(
            [sc * (qr @ ks.T), sc * np.einsum("rc,ric->ri", qr, kdp)], axis=1),
        # strict causal mask (self excluded)
        "strict_causal": lambda qr, ks, kdp, sc, ts, sel=None: np.concatenate(
            [np.where(np.arange(ks.shape[0])[None] < np.asarray(ts)[:, None], sc * (qr @ ks.T), -np.inf),
             sc * np.einsum("rc,ric->ri", qr, kdp)], axis=1),
        # depth logits without the scale
        "unscaled_depth": lambda qr, ks, kdp, sc, ts, sel=None: np.concatenate(
            [orig(qr, ks, kdp[:, :0], sc, ts), np.einsum("rc,ric->ri", qr, kdp)], axis=1),
        # depth logits with a flipped sign
        "neg_depth": lambda qr, ks, kdp, sc, ts, sel=None: np.concatenate(
            [orig(qr, ks, kdp[:, :0], sc, ts), -sc * np.einsum("rc,ric->ri", qr, kdp)], axis=1),
    }
    for name, fn in mutants.items():
        monkeypatch.setattr(om, "_concat_logits", fn)
        assert not _pins_pass(), name
        monkeypatch.setattr(om, "_concat_logits", orig)

    # softmax without the max shift but with the lse dropping m
    orig_sm = om._softmax_rows

    def bad_softmax(s):
        p, l = orig_sm(s)
        return p, l - np.max(s, axis=1)
    monkeypatch.setattr(om, "_softmax_rows", bad_softmax)
    assert not _pins_pass()
    monkeypatch.setattr(om, "_softmax_rows", orig_sm)
    assert _pins_pass()


def test_backward_with_stored_output_shifts_by_the_D_error():
    """With D formed from a perturbed forward output out + delta, every row's
    dS changes by -P * <dout, delta>, so dq changes by
    -scale * <dout, delta> * (sum_j P_j k_j + sum_i P'_i kd_i) (P from the
    exact forward), dv and dvd do not change at all."""
    x, scale = rand_case(1, 6, 2, 1, 4, 3, seed=21, depth_std=2.0)
    base = om.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale)
    delta = np.random.default_rng(3).standard_normal(x["q"].shape) * 1e-2
    pert = om.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale,
                       out_for_D=base[5] + delta)
    np.testing.assert_allclose(pert[2], base[2], rtol=0, atol=1e-14)
    np.testing.assert_allclose(pert[4], base[4], rtol=0, atol=1e-14)
    lse = base[6]
    for h in range(2):
        for t in range(6):
            qv = x["q"][0, t, h]
            dD = float(np.dot(x["dout"][0, t, h], delta[0, t, h]))
            acc = np.zeros(4)
            for j in range(t + 1):
                acc += math.exp(scale * float(qv @ x["k"][0, j, 0]) - lse[0, h, t]) * x["k"][0, j, 0]
            for i in range(3):
                acc += math.exp(scale * float(qv @ x["kd"][0, t, i, 0]) - lse[0, h, t]) * x["kd"][0, t, i, 0]
            np.testing.assert_allclose(pert[0][0, t, h] - base[0][0, t, h], -scale * dD * acc,
                                       rtol=0, atol=1e-12)


# ---------------------------------------------------------- selected depth
def test_selected_depth_reduces_to_slicing_and_special_cases():
    """Selection of all entries = no selection; a selection of the first L'
    entries of every token = the forward with kd, vd sliced to L'; an empty
    selection = Ld = 0 (plain causal attention)."""
    x, scale = rand_case(2, 13, 4, 2, 8, 6, seed=31, depth_std=2.0)
    B, T, Ld = 2, 13, 6
    base = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale)
    allsel = np.ones((B, T, Ld), dtype=bool)
    o, l = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, depth_sel=allsel)
    np.testing.assert_array_equal(o, base[0])
    first = np.zeros((B, T, Ld), dtype=bool)
    first[:, :, :4] = True
    o, l = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, depth_sel=first)
    o2, l2 = om.forward(x["q"], x["k"], x["v"], x["kd"][:, :, :4], x["vd"][:, :, :4], scale)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l, l2, rtol=0, atol=1e-13)
    o, l = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, depth_sel=np.zeros_like(first))
    o3, l3 = om.forward(x["q"], x["k"], x["v"], x["kd"][:, :, :0], x["vd"][:, :, :0], scale)
    np.testing.assert_allclose(o, o3, rtol=0, atol=1e-13)


def _selected_depth_case():
    x, scale = rand_case(1, 6, 4, 2, 3, 4, seed=32, depth_std=2.0)
    rng = np.random.default_rng(7)
    sel = rng.random((1, 6, 4)) < 0.5
    return x, scale, sel


def _check_selected_depth_brute_force():
    x, scale, sel = _selected_depth_case()
    o, l = om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, depth_sel=sel)
    for t in range(6):
        keep = np.flatnonzero(sel[0, t])
        sub = {n: x[n][:, :t + 1] for n in ("q", "k", "v")}
        kd = np.zeros((1, t + 1, len(keep), 2, 3))
        vd = np.zeros_like(kd)
        kd[0, t] = x["kd"][0, t, keep]
        vd[0, t] = x["vd"][0, t, keep]
        bo, bl = brute_force(sub["q"], sub["k"], sub["v"], kd, vd, scale)
        np.testing.assert_allclose(o[0, t], bo[0, t], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[0, :, t], bl[0, :, t], rtol=0, atol=1e-12)


def test_selected_depth_brute_force_and_gradients():
    """Per-token random selection against the scalar brute force run on each
    token's gathered depth entries; backward against central differences, and
    unselected depth entries get exactly zero gradient."""
    _check_selected_depth_brute_force()
    x, scale, sel = _selected_depth_case()
    g = om.backward(x["q"], x["k"], x["v"], x["kd"], x["vd"], x["dout"], scale, depth_sel=sel)
    assert np.all(g[3][~sel] == 0) and np.all(g[4][~sel] == 0)
    eps = 1e-6
    for name, gi in (("q", 0), ("kd", 3), ("vd", 4), ("k", 1)):
        base = x[name]
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = base[idx]
            base[idx] = old + eps
            lp = float(np.sum(om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, depth_sel=sel)[0] * x["dout"]))
            base[idx] = old - eps
            lm = float(np.sum(om.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, depth_sel=sel)[0] * x["dout"]))
            base[idx] = old
            assert abs((lp - lm) / (2 * eps) - g[gi][idx]) < 1e-6 * max(1.0, abs(g[gi][idx])), (name, idx)


def test_planted_selection_mistakes_are_caught(monkeypatch):
    """A selection ignored, inverted or taken from the neighbouring token
    fails the selection pins."""
    def sel_pins_pass():
        try:
            test_selected_depth_reduces_to_slicing_and_special_cases()
            _check_selected_depth_brute_force()
            return True
        except AssertionError:
            return False

    assert sel_pins_pass()
    orig_sel = om._sel
    mutants = {
        "ignored": lambda ds, b, t0, t1: None,
        "inverted": lambda ds, b, t0, t1: None if ds is None else ~np.asarray(ds[b, t0:t1], dtype=bool),
        "shifted": lambda ds, b, t0, t1: None if ds is None else np.roll(np.asarray(ds[b], dtype=bool), 1, axis=0)[t0:t1],
    }
    for name, fn in mutants.items():
        monkeypatch.setattr(om, "_sel", fn)
        assert not sel_pins_pass(), name
        monkeypatch.setattr(om, "_sel", orig_sel)


# ---------------------------------------------------------------- write step
def test_depth_write_against_loops_and_forward():
    """The write step against scalar loops (only slot `slot` of every token
    changes), and a depth cache filled layer by layer equals one whose depth
    axis holds the layers' keys / values in order, as the forward reads it."""
    rng = np.random.default_rng(41)
    B, T, Ld, Hkv, d = 2, 5, 3, 2, 4
    kd = rng.standard_normal((B, T, Ld, Hkv, d))
    vd = rng.standard_normal((B, T, Ld, Hkv, d))
    k = rng.standard_normal((B, T, Hkv, d))
    v = rng.standard_normal((B, T, Hkv, d))
    kd_before = kd.copy()
    kd2, vd2 = om.depth_write(kd, vd, k, v, 1)
    for b in range(B):
        for t in range(T):
            for i in range(Ld):
                for h in range(Hkv):
                    for c in range(d):
                        ek = k[b, t, h, c] if i == 1 else kd[b, t, i, h, c]
                        ev = v[b, t, h, c] if i == 1 else vd[b, t, i, h, c]
                        assert kd2[b, t, i, h, c] == ek and vd2[b, t, i, h, c] == ev
    assert np.array_equal(kd, kd_before)  # the inputs are not modified
    # layer by layer into an empty cache, then the forward of the next layer
    Hq = 4
    layers = [(rng.standard_normal((B, T, Hkv, d)), rng.standard_normal((B, T, Hkv, d))) for _ in range(Ld)]
    ckd = np.zeros((B, T, Ld, Hkv, d))
    cvd = np.zeros((B, T, Ld, Hkv, d))
    for slot, (kl, vl) in enumerate(layers):
        ckd, cvd = om.depth_write(ckd, cvd, kl, vl, slot)
    q = rng.standard_normal((B, T, Hq, d))
    ks, vs = rng.standard_normal((B, T, Hkv, d)), rng.standard_normal((B, T, Hkv, d))
    o1, l1 = om.forward(q, ks, vs, ckd, cvd, 0.5)
    stacked_k = np.stack([kl for kl, _ in layers], axis=2)
    stacked_v = np.stack([vl for _, vl in layers], axis=2)
    o2, l2 = brute_force(q, ks, vs, stacked_k, stacked_v, 0.5)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


# ------------------------------------------------------------ 8-bit depth KV
def test_q8_hand_worked_rows_and_ties():
    """Rows whose scale is exact (amax 127 -> sigma 1, amax 254 -> sigma 2):
    the codes are the nearest integers of x / sigma with ties to even, the
    amax element maps to +-127, an all-zero row has scale 0 and codes 0."""
    rows = np.array([[127.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -127.0],
                     [254.0, 5.0, 7.0, -5.0, 1.0, 3.0, -254.0, 0.0],
                     [0.0] * 8], dtype=np.float32)
    codes, sigma = om.quantize_q8(rows)
    assert sigma.tolist() == [1.0, 2.0, 0.0]
    assert codes.tolist() == [[127, 2, 4, -2, -4, 0, 2, -127],
                              [127, 2, 4, -2, 0, 2, -127, 0],
                              [0] * 8]
    assert codes.dtype == np.int8 and sigma.dtype == np.float32


def test_q8_nearest_code_and_error_bound():
    """On random bf16 rows: every code is the nearest multiple of sigma (no
    neighbour code is closer), |x - sigma*code| <= sigma/2 up to the float32
    rounding of x / sigma, codes lie in [-127, 127], and each row's largest
    |x| maps to |code| = 127."""
    g = torch.Generator("cpu")
    g.manual_seed(5)
    x = (torch.randn(64, 7, 128, generator=g) * torch.rand(64, 7, 1, generator=g) * 10).to(torch.bfloat16)
    xf = om.to_f64(x)
    codes, sigma = om.quantize_q8(x)
    c = codes.astype(np.float64)
    s = sigma.astype(np.float64)[..., None]
    err = np.abs(xf - s * c)
    assert np.all(np.abs(c) <= 127)
    # x / sigma is rounded to float32 before the integer rounding: half an
    # ulp of a quotient below 128 is at most 2^-18, so a code may sit up to
    # sigma * 2^-18 beyond the exact half-way point
    assert np.all(err <= s * (0.5 + 2.0 ** -17) + 1e-30)
    for dc in (-1, 1):
        nb = np.clip(c + dc, -127, 127)
        assert np.all(err <= np.abs(xf - s * nb) + s * 2.0 ** -16)
    amax_idx = np.argmax(np.abs(xf), axis=-1)[..., None]
    assert np.all(np.abs(np.take_along_axis(c, amax_idx, -1)) == 127)
    # the scale is amax / 127 in float32
    np.testing.assert_array_equal(sigma, (np.max(np.abs(xf), -1).astype(np.float32) / np.float32(127)))


def test_q8_dequantise_is_exact_and_write_step_touches_one_slot():
    g = torch.Generator("cpu")
    g.manual_seed(6)
    B, T, Ld, Hkv, d = 2, 5, 3, 2, 16
    kd = torch.randn(B, T, Ld, Hkv, d, generator=g).to(torch.bfloat16)
    vd = torch.randn(B, T, Ld, Hkv, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, T, Hkv, d, generator=g).to(torch.bfloat16)
    ck, sk = om.quantize_q8(kd)
    cv, sv = om.quantize_q8(vd)
    # float32 cache: one float32 product; bf16 cache: that product rounded to
    # bf16 exactly as torch rounds float32 to bfloat16 (a library routine)
    deq32 = om.dequantize_q8(ck, sk, "f32")
    deq16 = om.dequantize_q8(ck, sk, "bf16")
    for idx in [(0, 0, 0, 0, 3), (1, 4, 2, 1, 15), (1, 2, 1, 0, 0)]:
        assert deq32[idx] == float(np.float32(ck[idx]) * np.float32(sk[idx[:-1]]))
    prod = torch.from_numpy(deq32.astype(np.float32))
    np.testing.assert_array_equal(deq16, prod.to(torch.bfloat16).to(torch.float64).numpy())
    # ties: 1 + 2^-8 lies half-way between bf16 neighbours 1 and 1 + 2^-7
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 3.0], dtype=np.float32)
    assert om.round_to_bf16(ties).tolist() == [1.0, 1 + 2.0 ** -6, -1.0, 3.0]
    kd8, vd8, sk2, sv2 = om.depth_write_q8(ck, cv, sk, sv, k, v, 1)
    for slot in (0, 2):
        np.testing.assert_array_equal(kd8[:, :, slot], ck[:, :, slot])
        np.testing.assert_array_equal(sv2[:, :, slot], sv[:, :, slot])
    c1, s1 = om.quantize_q8(k)
    np.testing.assert_array_equal(kd8[:, :, 1], c1)
    np.testing.assert_array_equal(sk2[:, :, 1], s1)
    c2, s2 = om.quantize_q8(v)
    np.testing.assert_array_equal(vd8[:, :, 1], c2)
    np.testing.assert_array_equal(sv2[:, :, 1], s2)


def test_planted_q8_mistakes_are_caught(monkeypatch):
    """Truncation instead of rounding, ties away from zero, and a scale of
    amax / 128 each fail the hand-worked or the nearest-code pin."""
    real = om.quantize_q8

    def trunc(x):
        xf = np.asarray(om.to_f64(x)).astype(np.float32)
        sigma = (np.max(np.abs(xf), -1) / np.float32(127)).astype(np.float32)
        safe = np.where(sigma > 0, sigma, 1).astype(np.float32)
        return np.trunc(xf / safe[..., None]).astype(np.int8), sigma

    def away(x):
        xf = np.asarray(om.to_f64(x)).astype(np.float32)
        sigma = (np.max(np.abs(xf), -1) / np.float32(127)).astype(np.float32)
        safe = np.where(sigma > 0, sigma, 1).astype(np.float32)
        r = xf / safe[..., None]
        return (np.sign(r) * np.floor(np.abs(r) + 0.5)).astype(np.int8), sigma

    def scale128(x):
        xf = np.asarray(om.to_f64(x)).astype(np.float32)
        sigma = (np.max(np.abs(xf), -1) / np.float32(128)).astype(np.float32)
        safe = np.where(sigma > 0, sigma, 1).astype(np.float32)
        return np.clip(np.rint(xf / safe[..., None]), -127, 127).astype(np.int8), sigma

    for bad in (trunc, away, scale128):
        monkeypatch.setattr(om, "quantize_q8", bad)
        with pytest.raises(AssertionError):
            test_q8_hand_worked_rows_and_ties()
        monkeypatch.setattr(om, "quantize_q8", real)
