"""Checks that pin the CPU oracle to what the pages and the mathematics fix.

Each ``check_*`` takes a loaded oracle (``oracle.pq_oracle.Oracle``) and
raises AssertionError when the oracle disagrees with the pin. They are run on
the real oracle by ``test_oracle_pins.py`` and on deliberately broken copies
of it by ``test_oracle_mutants.py`` (every plausible mistake must fail at
least one of them).

What each pin compares against is independent of the oracle's code:
printed level sets and bins (golden files), the worked overflow example,
nearest-level brute force, the LSQ and XNOR-Net textbook forms, torch's own
bf16 conversion, fp64 finite differences, a closed form for fully clipped
rows, and hand-computed packed bytes.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

from oracle.pq_oracle import (BINARY, LSQ2, LSQ3, LSQ4, SEQ2, SEQ2_B,
                              TERNARY, ALL_QUANTIZERS)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
NAMES = {"seq2": SEQ2, "ternary": TERNARY, "lsq4": LSQ4, "lsq3": LSQ3,
         "lsq2": LSQ2, "binary": BINARY, "seq2_b": SEQ2_B}


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f32(v):
    return float(np.float32(v))


def frac_f32(nd):
    return f32(Fraction(nd[0], nd[1]))


def printed_levels():
    """Level sets in alpha units as fp32 values, keyed by quantizer."""
    g = golden("level_sets.json")
    out = {SEQ2: sorted(frac_f32(v) for v in g["seq2_levels"]["values"]),
           TERNARY: sorted(frac_f32(v) for v in g["ternary_levels"]["values"])}
    for b, q in (("2", LSQ2), ("3", LSQ3), ("4", LSQ4)):
        out[q] = [float(v) for v in g["lsq_levels"]["values"][b]]
    # the divisor-1.5 reading of the 2-bit SEQ formula: {-1.5,-0.5,0.5,1.5}/1.5
    out[SEQ2_B] = sorted(f32(Fraction(v).limit_denominator(4) / Fraction(3, 2))
                         for v in g["seq2_code_domain"]["values"])
    out[BINARY] = [-1.0, 1.0]
    return out


def lsq_bounds(q):
    b = {LSQ2: 2, LSQ3: 3, LSQ4: 4}[q]
    return -(2 ** (b - 1)), 2 ** (b - 1) - 1


def clip_range(q):
    if q in (LSQ2, LSQ3, LSQ4):
        lo, hi = lsq_bounds(q)
        return float(lo), float(hi)
    if q == BINARY:
        return -1.0, 1.0
    return -f32(0.99), f32(0.99)


def _sweep(q):
    lo, hi = clip_range(q)
    span = max(abs(lo), abs(hi)) * 1.3
    return np.linspace(-span, span, 20001, dtype=np.float32)


# ----------------------------------------------------------------- levels
def check_level_sets(O):
    """Sweeping x over and past the clip range (alpha = 1) yields exactly the
    printed level set."""
    lev = printed_levels()
    for q in ALL_QUANTIZERS:
        x = _sweep(q)
        wq, codes, _ = O.fwd(q, x.reshape(1, -1), np.ones(1, np.float32))
        got = sorted(set((wq.astype(np.uint32) << 16).view(np.float32).ravel().tolist()))
        want = sorted(set(float(np.float32(
            torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).float()))
            for v in lev[q]))
        assert got == want, (q, got, want)


def check_seq_code_domain(O):
    """SEQ2 codes c satisfy c + 0.5 in the printed code domain."""
    dom = golden("level_sets.json")["seq2_code_domain"]["values"]
    x = _sweep(SEQ2)
    _, codes, _ = O.fwd(SEQ2, x.reshape(1, -1), np.ones(1, np.float32))
    got = sorted(set((codes.astype(np.float64) + 0.5).ravel().tolist()))
    assert got == sorted(dom), got


def check_ternary_bins(O):
    """Ternary: in the 1.5-scaled domain the bins are the printed
    equal-width intervals (tested well inside each bin)."""
    for lo, hi, code in golden("level_sets.json")["ternary_bins_scaled"]["bins"]:
        s = np.linspace(lo + 1e-3, hi - 1e-3, 501)
        x = (s / 1.5).astype(np.float32)
        x = np.clip(x, -0.98, 0.98)
        _, codes, _ = O.fwd(TERNARY, x.reshape(1, -1), np.ones(1, np.float32))
        assert np.all(codes == code), (lo, hi, code, np.unique(codes))


def check_nearest_level(O):
    """Brute force: away from bin edges, the code selects the printed level
    nearest to clip(x) (alpha random, w = x*alpha)."""
    rng = np.random.default_rng(7)
    lev = printed_levels()
    for q in (SEQ2, SEQ2_B, TERNARY, LSQ2, LSQ3, LSQ4):
        lo, hi = clip_range(q)
        L = np.array(lev[q], np.float64)
        alpha = np.float32(rng.uniform(0.01, 3.0))
        w = (rng.uniform(lo * 1.3, hi * 1.3, 4000) * alpha).astype(np.float32)
        x = (w / alpha).astype(np.float64)
        xc = np.clip(x, lo, hi)
        d = np.abs(xc[:, None] - L[None, :])
        srt = np.sort(d, axis=1)
        keep = (srt[:, 1] - srt[:, 0]) > 1e-4  # not near a bin edge
        want = L[np.argmin(d, axis=1)]
        # a zero level carries the sign of x (IEEE rounding of a negative
        # argument to zero gives -0.0)
        want = np.where(want == 0, np.copysign(0.0, x), want)
        wq, _, _ = O.fwd(q, w.reshape(1, -1), np.array([alpha]))
        # compare in alpha units through bf16(level*alpha)
        want_bits = torch.tensor((want * float(alpha)).astype(np.float32)).to(
            torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        got_bits = wq.ravel()
        # the printed levels are fp32 values, so level*alpha is exact in fp64
        # and the cast above rounds it to fp32 once, as the quantizer does
        assert np.array_equal(got_bits[keep], want_bits[keep]), q


def check_binary_sign(O):
    """Binary reduces to sign(w)*alpha (XNOR-Net), with sign(+-0) = +1."""
    rng = np.random.default_rng(3)
    w = rng.normal(0, 0.02, (4, 64)).astype(np.float32)
    w[0, :4] = [0.0, -0.0, 1e-38, -1e-38]
    alpha = np.abs(w).mean(axis=1).astype(np.float32)
    wq, codes, _ = O.fwd(BINARY, w, alpha)
    sign = np.where(np.signbit(w) & (w != 0), -1, 1)
    assert np.array_equal(codes, sign)
    want = torch.tensor((sign * alpha[:, None]).astype(np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wq, want)


def check_lsq_textbook(O):
    """LSQ: clamp(rint(w/alpha), -Qn, Qp)*alpha in numpy fp32 (the textbook
    quantizer of the LSQ paper), and integers come back unchanged at
    alpha = 1."""
    rng = np.random.default_rng(11)
    for q in (LSQ2, LSQ3, LSQ4):
        lo, hi = lsq_bounds(q)
        w = rng.normal(0, 0.02, (8, 256)).astype(np.float32)
        alpha = (2 * np.abs(w).mean(axis=1) / math.sqrt(hi)).astype(np.float32)
        v = np.clip(np.rint(w / alpha[:, None]), lo, hi).astype(np.float32)
        want = torch.tensor(v * alpha[:, None]).to(torch.bfloat16).view(
            torch.int16).numpy().view(np.uint16)
        wq, codes, _ = O.fwd(q, w, alpha)
        assert np.array_equal(codes, v.astype(np.int8)), q
        assert np.array_equal(wq, want), q
        ints = np.arange(lo, hi + 1, dtype=np.float32).reshape(1, -1)
        wq, codes, _ = O.fwd(q, ints, np.ones(1, np.float32))
        assert np.array_equal(codes.ravel(), ints.ravel().astype(np.int8))


# --------------------------------------------------------- worked examples
def check_overflow_example(O):
    """The published clip at 1 with round-half-even gives a fifth level
    +1.25 at x = +1; the code's 0.99 clip caps the level at 0.75."""
    g = golden("boundary_overflow.json")
    r = O.quantize_scalar(SEQ2, g["x"], 1.0, clip_hi=g["literal_clip"])
    assert r["code"] == g["literal_code"] and r["level"] == g["literal_level"], r
    r = O.quantize_scalar(SEQ2, g["x"], 1.0)
    assert r["level"] == g["code_max_level"], r
    x = np.linspace(-10, 10, 4001, dtype=np.float32).reshape(1, -1)
    _, codes, _ = O.fwd(SEQ2, x, np.ones(1, np.float32))
    assert codes.max() == 1 and codes.min() == -2


def check_ties_half_even(O):
    """Exact ties of the rounding argument go to the even integer."""
    # SEQ2: t = 2x - 0.5
    assert O.quantize_scalar(SEQ2, 0.5, 1.0)["code"] == 0     # t = 0.5
    assert O.quantize_scalar(SEQ2, -0.5, 1.0)["code"] == -2   # t = -1.5
    assert O.quantize_scalar(SEQ2, 0.0, 1.0)["code"] == 0     # t = -0.5
    # ternary: t = 1.5x; x = fl(1/3) gives fl(1.5x) = 0.5 exactly
    third = f32(1.0 / 3.0)
    assert np.float32(np.float32(third) * np.float32(1.5)) == np.float32(0.5)
    assert O.quantize_scalar(TERNARY, third, 1.0)["code"] == 0
    assert O.quantize_scalar(TERNARY, -third, 1.0)["code"] == 0
    # LSQ: t = x
    assert O.quantize_scalar(LSQ4, 2.5, 1.0)["code"] == 2
    assert O.quantize_scalar(LSQ4, -2.5, 1.0)["code"] == -2
    assert O.quantize_scalar(LSQ4, 3.5, 1.0)["code"] == 4


def check_idempotence(O):
    """Quantizing the dequantized weights again (fp32 pre-cast value and the
    bf16 output, same alpha) returns the same codes and bf16 weights."""
    rng = np.random.default_rng(5)
    for q in ALL_QUANTIZERS:
        w = rng.normal(0, 0.02, (4, 128)).astype(np.float32)
        if q in (LSQ2, LSQ3, LSQ4):
            hi = lsq_bounds(q)[1]
            alpha = (2 * np.abs(w).mean(axis=1) / math.sqrt(hi)).astype(np.float32)
        elif q == BINARY:
            alpha = np.abs(w).mean(axis=1).astype(np.float32)
        else:
            alpha = np.abs(w).max(axis=1).astype(np.float32)
        wq, codes, _ = O.fwd(q, w, alpha)
        wq_f = (wq.astype(np.uint32) << 16).view(np.float32)
        wq2, codes2, _ = O.fwd(q, wq_f, alpha)
        assert np.array_equal(codes, codes2), q
        assert np.array_equal(wq, wq2), q
        pre = np.array([[O.quantize_scalar(q, float(w[r, j]), float(alpha[r]))
                         ["wq32"] for j in range(w.shape[1])]
                        for r in range(w.shape[0])], np.float32)
        wq3, codes3, _ = O.fwd(q, pre, alpha)
        assert np.array_equal(codes, codes3), q


def check_bf16_rne(O):
    """The oracle's fp32 -> bf16 equals torch's round-to-nearest-even
    conversion, including exact ties of both parities and subnormals."""
    rng = np.random.default_rng(9)
    bits = rng.integers(0, 2 ** 32, 3000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2 ** 16, 400, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    special = np.array([0x00000000, 0x80000000, 0x00008000, 0x00018000,
                        0x3F808000, 0x3F818000, 0x7F7FFFFF, 0x7F7F8000,
                        0x00000001, 0x807FFFFF], np.uint32)
    allb = np.concatenate([bits, ties, special])
    f = allb.view(np.float32)
    f = f[np.isfinite(f)]
    got = O.bf16_rne(f)
    want = torch.tensor(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- backward
def check_ste(O):
    """dW is exactly 0 outside [lo, hi] and exactly float(g) inside; the
    interval is closed (x == 0.99f passes)."""
    rng = np.random.default_rng(2)
    for q in ALL_QUANTIZERS:
        lo, hi = clip_range(q)
        alpha = np.float32(0.7)
        x = rng.uniform(lo * 1.5, hi * 1.5, 512).astype(np.float32)
        w = (x * alpha).astype(np.float32)
        xs = (w / alpha).astype(np.float32)
        g = torch.randn(512).mul(1e-3).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        gf = (g.astype(np.uint32) << 16).view(np.float32)
        dw, _, _ = O.bwd(q, w.reshape(1, -1), np.array([alpha]), g.reshape(1, -1), 1.0)
        inside = (xs >= np.float32(lo)) & (xs <= np.float32(hi))
        assert np.all(dw.ravel()[~inside] == 0.0), q
        assert np.array_equal(dw.ravel()[inside], gf[inside]), q
        # closed interval: x exactly on either bound passes the gradient
        edge = np.array([[hi, lo, np.nextafter(np.float32(hi), np.float32(9)),
                          np.nextafter(np.float32(lo), np.float32(-9))]],
                        np.float32)
        ge = np.full((1, 4), 0x3F80, np.uint16)  # g = 1.0
        dw, _, _ = O.bwd(q, edge, np.ones(1, np.float32), ge, 1.0)
        assert dw.ravel().tolist() == [1.0, 1.0, 0.0, 0.0], (q, dw)


def _level_of_code(q, codes):
    lev = printed_levels()[q]
    if q == BINARY:
        return codes.astype(np.float64)
    cmin = {SEQ2: -2, SEQ2_B: -2, TERNARY: -1}.get(q)
    if cmin is None:
        cmin = lsq_bounds(q)[0]
    return np.array(lev, np.float64)[codes.astype(np.int64) - cmin]


def check_dalpha_fd(O):
    """Finite differences in fp64 on 8x16 matrices. With the rounding
    residual frozen at alpha0, S(a) = sum g*a*(L0 + clip(w/a) - clip(w/a0))
    has dS/da at a0 equal to sum g*(L0 - inside*x), the quantity the
    backward reduces per row (grad_scale = 1)."""
    rng = np.random.default_rng(13)
    for q in ALL_QUANTIZERS:
        lo, hi = clip_range(q)
        w = rng.normal(0, 0.02, (8, 16)).astype(np.float32)
        a0 = (np.abs(w).max(axis=1) * rng.uniform(0.6, 1.1, 8)).astype(np.float32)
        if q in (LSQ2, LSQ3, LSQ4):
            a0 = (a0 / hi * 1.2).astype(np.float32)
        g = (rng.normal(0, 1e-3, (8, 16))).astype(np.float32)
        gb = torch.tensor(g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        gf = (gb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        _, codes, _ = O.fwd(q, w, a0)
        _, da, _ = O.bwd(q, w, a0, gb, 1.0)
        L0 = _level_of_code(q, codes)
        wd = w.astype(np.float64)

        def clipf(x):
            return np.clip(x, lo, hi)
        for r in range(8):
            a = float(a0[r])
            x0 = wd[r] / a
            # no element may cross a clip bound within +-h
            h = a * 1e-7
            for s in (a - h, a + h):
                xs = wd[r] / s
                assert np.array_equal((xs >= lo) & (xs <= hi), (x0 >= lo) & (x0 <= hi))

            def S(s):
                return np.sum(gf[r] * s * (L0[r] + clipf(wd[r] / s) - clipf(x0)))
            fd = (S(a + h) - S(a - h)) / (2 * h)
            scale = np.sum(np.abs(gf[r]) * (np.abs(L0[r]) + np.abs(x0)))
            assert abs(float(da[r]) - fd) <= 2e-6 * scale, (q, r, da[r], fd)


def check_dalpha_all_clipped(O):
    """Closed form: when every weight of a row is clipped, d(alpha) =
    grad_scale * sum g * L (the boundary-value gradient)."""
    rng = np.random.default_rng(17)
    for q in ALL_QUANTIZERS:
        lo, hi = clip_range(q)
        sgn = rng.choice([-1.0, 1.0], (3, 40))
        alpha = np.array([0.5, 1.0, 2.0], np.float32)
        w = (sgn * (max(abs(lo), abs(hi)) * 3.0) * alpha[:, None]).astype(np.float32)
        gb = torch.randn(3, 40).mul(1e-3).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        gf = (gb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        gs = 0.125
        dw, da, _ = O.bwd(q, w, alpha, gb, gs)
        assert np.all(dw == 0.0)
        lev = printed_levels()[q]
        L = np.where(sgn > 0, lev[-1], lev[0])
        want = gs * np.sum(gf * L, axis=1)
        assert np.allclose(da, want, rtol=1e-6, atol=1e-12), (q, da, want)


def check_grad_scale(O):
    """Default gradient scale is 1/sqrt(n*Qp), n = weights per alpha, Qp the
    positive bound of the LSQ grid (1 at 2 bits, 3 at 3 bits, 7 at 4 bits)."""
    for q, qp in ((LSQ2, 1), (LSQ3, 3), (LSQ4, 7)):
        assert math.isclose(O.default_grad_scale(q, 4096),
                            1 / math.sqrt(4096 * qp), rel_tol=1e-6)
    rng = np.random.default_rng(19)
    w = rng.normal(0, 0.02, (4, 64)).astype(np.float32)
    alpha = np.abs(w).max(axis=1).astype(np.float32)
    gb = torch.randn(4, 64).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    _, d1, _ = O.bwd(SEQ2, w, alpha, gb, 1.0)
    _, d2, _ = O.bwd(SEQ2, w, alpha, gb, 0.25)
    assert np.array_equal(d1 * np.float32(0.25), d2)


# ------------------------------------------------------------------ packing
def check_pack_golden(O):
    """Hand-computed packed bytes for one row per format."""
    for row in golden("pack_rows.json")["rows"]:
        q = NAMES[row["q"]]
        x = np.array(row["x"], np.float32).reshape(1, -1)
        wq, codes, packed = O.fwd(q, x, np.ones(1, np.float32), pack=True)
        assert codes.ravel().tolist() == row["codes"], (row["q"], codes)
        assert packed.ravel().tolist() == row["bytes"], (row["q"], packed)
        assert O.pack(q, x, np.ones(1, np.float32)).ravel().tolist() == row["bytes"]


def check_pack_roundtrip(O):
    """Unpacking (sign extension of each field) returns the int8 codes."""
    rng = np.random.default_rng(23)
    for q in ALL_QUANTIZERS:
        w = rng.normal(0, 0.02, (5, 48)).astype(np.float32)
        alpha = (np.abs(w).max(axis=1) * 0.5).astype(np.float32)
        _, codes, packed = O.fwd(q, w, alpha, pack=True)
        bits = O.code_bits(q)
        per = 8 // bits
        fields = [(packed >> (bits * i)) & ((1 << bits) - 1) for i in range(per)]
        un = np.stack(fields, axis=-1).reshape(5, -1).astype(np.int16)
        un = np.where(un >= (1 << (bits - 1)), un - (1 << bits), un)
        assert np.array_equal(un.astype(np.int8), codes), q


def check_dequant_golden(O):
    """Stored codes decode to the printed levels (golden rows, alpha = 1)."""
    for row in golden("pack_rows.json")["rows"]:
        q = NAMES[row["q"]]
        packed = np.array(row["bytes"], np.uint8).reshape(1, -1)
        got = (O.dequant(q, packed, np.ones(1, np.float32), len(row["codes"]))
               .astype(np.uint32) << 16).view(np.float32).ravel()
        want = [frac_f32(v) if isinstance(v, list) else float(v) for v in row["levels"]]
        want = torch.tensor(want, dtype=torch.float32).to(torch.bfloat16).float().numpy()
        assert np.array_equal(np.abs(got), np.abs(want)) and np.array_equal(got, want), (row["q"], got)


def check_dequant_inverts_pack(O):
    """Decoding the packed codes reproduces the forward's bf16 weights, up
    to the sign of a zero (codes do not store it)."""
    rng = np.random.default_rng(29)
    for q in ALL_QUANTIZERS:
        w = rng.normal(0, 0.02, (6, 64)).astype(np.float32)
        alpha = (np.abs(w).max(axis=1) * rng.uniform(0.3, 1.0, 6)).astype(np.float32)
        wq, _, packed = O.fwd(q, w, alpha, pack=True)
        dq = O.dequant(q, packed, alpha, 64)
        zero = (wq & 0x7FFF) == 0
        assert np.array_equal(dq[~zero], wq[~zero]), q
        assert np.all(dq[zero] == 0), q


def check_adamw_vs_torch(O):
    """One AdamW step matches torch.optim.AdamW (fp32, CPU) over five steps,
    with and without decoupled weight decay, to within fp32 rounding."""
    from oracle.pq_oracle import AdamW
    rng = np.random.default_rng(43)
    for wd in (0.0, 0.05):
        p0 = rng.normal(0, 0.02, 4096).astype(np.float32)
        t_p = torch.nn.Parameter(torch.from_numpy(p0.copy()))
        opt = torch.optim.AdamW([t_p], lr=2e-3, betas=(0.9, 0.999), eps=1e-8,
                                weight_decay=wd, foreach=False, fused=False)
        p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
        for t in range(1, 6):
            g = rng.normal(0, 1e-3, 4096).astype(np.float32)
            t_p.grad = torch.from_numpy(g.copy())
            opt.step()
            prev = p
            p, m, v = O.adamw_step(p, g, m, v, AdamW.at_step(t, 2e-3, weight_decay=wd))
            st = opt.state[t_p]
            # tolerances against the scale of the quantity (torch forms the
            # first moment as a lerp: same value up to a few ulps)
            gs = float(np.abs(g).max())
            assert np.allclose(m, st["exp_avg"].numpy(), rtol=1e-5, atol=1e-6 * gs), (wd, t)
            assert np.allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-5, atol=1e-6 * gs * gs), (wd, t)
            upd, t_upd = p - prev, t_p.detach().numpy() - prev
            assert np.allclose(upd, t_upd, rtol=1e-4, atol=1e-5 * 2e-3), (wd, t)
            p = t_p.detach().numpy().copy()  # stay on torch's trajectory


def check_adamw_first_step(O):
    """Closed form of Adam's first step from zero moments: the bias-corrected
    moments are g and g^2, so the update is lr * g / (|g| + eps)."""
    from oracle.pq_oracle import AdamW
    g = np.array([1e-3, -2e-2, 5e-1, -7.0, 1e-6], np.float32)
    p0 = np.zeros_like(g)
    p, m, v = O.adamw_step(p0, g, np.zeros_like(g), np.zeros_like(g),
                           AdamW.at_step(1, 1e-2))
    want = -1e-2 * g.astype(np.float64) / (np.abs(g.astype(np.float64)) + 1e-8)
    assert np.allclose(p, want, rtol=1e-5), (p, want)
    assert np.allclose(m, 0.1 * g, rtol=1e-6) and np.allclose(v, 0.001 * g * g, rtol=1e-5)


def check_bwd_adamw_composes(O):
    """The fused backward + AdamW equals the backward followed by AdamW
    steps on W (gradient dW) and alpha (gradient d(alpha)), bit for bit."""
    from oracle.pq_oracle import AdamW
    rng = np.random.default_rng(47)
    for q in ALL_QUANTIZERS:
        w = rng.normal(0, 0.02, (5, 48)).astype(np.float32)
        a = (np.abs(w).max(axis=1) * 0.8).astype(np.float32)
        gb = torch.randn(5, 48).mul(1e-3).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        mw, vw = rng.normal(0, 1e-4, (5, 48)).astype(np.float32), np.abs(rng.normal(0, 1e-7, (5, 48))).astype(np.float32)
        ma, va = rng.normal(0, 1e-4, 5).astype(np.float32), np.abs(rng.normal(0, 1e-7, 5)).astype(np.float32)
        hw, ha = AdamW.at_step(3, 2e-5, weight_decay=0.01), AdamW.at_step(3, 1e-4)
        fw, fa, fmw, fvw, fma, fva, fda = O.bwd_adamw(q, w, a, gb, mw, vw, ma, va, 0.5, hw, ha)
        dw, da, _ = O.bwd(q, w, a, gb, 0.5)
        pw, pmw, pvw = O.adamw_step(w, dw, mw, vw, hw)
        pa, pma, pva = O.adamw_step(a, da, ma, va, ha)
        for x, y in ((fw.ravel(), pw), (fmw.ravel(), pmw), (fvw.ravel(), pvw),
                     (fa, pa), (fma, pma), (fva, pva), (fda, da)):
            assert np.array_equal(x.view(np.uint32), y.view(np.uint32)), q


def check_reduce_equals_single_source(O):
    """The multi-source backward + AdamW reduces to the single-source one:
    one source with multiplier 1, and n identical sources with multiplier
    1/n (n a power of two, so the mean is exact), give the same bits."""
    from oracle.pq_oracle import AdamW
    rng = np.random.default_rng(53)
    for q in ALL_QUANTIZERS:
        w = rng.normal(0, 0.02, (4, 40)).astype(np.float32)
        a = (np.abs(w).max(axis=1) * 0.7).astype(np.float32)
        gb = torch.randn(4, 40).mul(1e-3).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        st = [rng.normal(0, 1e-4, (4, 40)).astype(np.float32),
              np.abs(rng.normal(0, 1e-7, (4, 40))).astype(np.float32),
              rng.normal(0, 1e-4, 4).astype(np.float32),
              np.abs(rng.normal(0, 1e-7, 4)).astype(np.float32)]
        hw, ha = AdamW.at_step(2, 2e-5), AdamW.at_step(2, 1e-4)
        ref = O.bwd_adamw(q, w, a, gb, *st, 0.5, hw, ha)
        # the per-row sum of |terms| of the plain backward (a diagnostic
        # output: the tolerance floor of rows whose sum cancels)
        _, _, ref_abs = O.bwd(q, w, a, gb, 0.5)
        for n, mult in ((1, 1.0), (2, 0.5), (4, 0.25)):
            got = O.reduce_bwd_adamw(q, w, a, [gb] * n, mult, *st, 0.5, hw, ha)
            for x, y in zip(got[:7], ref):
                assert np.array_equal(np.asarray(x).view(np.uint32),
                                      np.asarray(y).view(np.uint32)), (q, n)
            assert np.array_equal(got[7], ref_abs), (q, n)


def check_reduce_sums_in_fp32(O):
    """With two different sources the gradient is their fp32 sum: the
    weights inside the clip range move as Adam's first step moves them for
    g = g0 + g1 (computed here with numpy), outside they do not move."""
    from oracle.pq_oracle import AdamW
    rng = np.random.default_rng(59)
    w = rng.normal(0, 0.02, (3, 64)).astype(np.float32)
    a = (np.abs(w).max(axis=1) * 0.6).astype(np.float32)  # some clipped
    g0 = torch.randn(3, 64).mul(1e-3).to(torch.bfloat16)
    g1 = torch.randn(3, 64).mul(1e-3).to(torch.bfloat16)
    gsum = (g0.float() + g1.float()).numpy()
    z = np.zeros_like(w)
    hw = AdamW.at_step(1, 1e-3)
    nw, *_ = O.reduce_bwd_adamw(SEQ2, w, a, [g0.view(torch.int16).numpy(), g1.view(torch.int16).numpy()],
                                1.0, z, z, np.zeros(3, np.float32), np.zeros(3, np.float32),
                                0.5, hw, AdamW.at_step(1, 1e-4))
    inside = np.abs(w / a[:, None]) <= np.float32(0.99)
    step = -1e-3 * gsum / (np.abs(gsum) + 1e-8)
    assert np.allclose((nw - w)[inside], step[inside], rtol=1e-4, atol=1e-9)
    assert np.array_equal(nw[~inside], w[~inside])


def check_wq_matmul_vs_numpy(O):
    """The low-bit matmul equals numpy's fp64 matmul of X with weights
    decoded from the printed level sets (codes drawn from those a forward
    writes), for every quantizer."""
    rng = np.random.default_rng(61)
    for q in ALL_QUANTIZERS:
        bits = O.code_bits(q)
        m, n, k = 3, 5, 32
        exact = {SEQ2: {-2: -0.75, -1: -0.25, 0: 0.25, 1: 0.75},
                 SEQ2_B: {-2: -1.0, -1: -1 / 3, 0: 1 / 3, 1: 1.0},
                 TERNARY: {-1: -2 / 3, 0: 0.0, 1: 2 / 3},
                 BINARY: {-1: -1.0, 1: 1.0}}.get(q)
        if exact is None:  # LSQ integer grid
            lo, hi = lsq_bounds(q)
            exact = {c: float(c) for c in range(lo, hi + 1)}
        codes = rng.choice(sorted(exact), (n, k))
        L = np.vectorize(exact.get)(codes).astype(np.float64)
        per = 8 // bits
        fields = (codes & ((1 << bits) - 1)).astype(np.uint8).reshape(n, k // per, per)
        packed = np.zeros((n, k // per), np.uint8)
        for i in range(per):
            packed |= fields[:, :, i] << (bits * i)
        alpha = rng.uniform(0.01, 2.0, n).astype(np.float32)
        xb = torch.randn(m, k).to(torch.bfloat16)
        x = xb.float().numpy().astype(np.float64)
        want = x @ (L * alpha[:, None].astype(np.float64)).T
        got = O.wq_matmul(q, xb.view(torch.int16).numpy(), packed, alpha, k)
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12), q


ALL_CHECKS = [check_level_sets, check_seq_code_domain, check_ternary_bins,
              check_nearest_level, check_binary_sign, check_lsq_textbook,
              check_overflow_example, check_ties_half_even, check_idempotence,
              check_bf16_rne, check_ste, check_dalpha_fd,
              check_dalpha_all_clipped, check_grad_scale, check_pack_golden,
              check_pack_roundtrip, check_dequant_golden,
              check_dequant_inverts_pack, check_adamw_vs_torch,
              check_adamw_first_step, check_bwd_adamw_composes,
              check_reduce_equals_single_source, check_reduce_sums_in_fp32,
              check_wq_matmul_vs_numpy]
