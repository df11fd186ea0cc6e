"""Pins for the oracle's operator arithmetic, against facts other than the
oracle itself: hand-worked rows (tests/golden), closed forms, a library
routine for a special case (torch rms_norm), the aclnnRmsNormDynamicQuant page
as a sub-case, invariants of the quantizer, and an independent 50-digit
evaluation on tiny random rows.

A plausible mistake anywhere in the oracle -- dropped epsilon, sum instead of
mean, missing beta, smooth scale applied to the wrong output, /127 vs /7,
round-half-away instead of half-even, swapped nibbles, normalising the
unrounded sum, wrong output selection -- fails at least one of these.
"""
import decimal
from decimal import Decimal
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from int4_quant_b200 import workloads as wl
from tests._util import codes, f32_of_fraction, golden, unpack_int4, unpack_int4_words


def bits(values, dtype="bf16"):
    return wl.to_bits(np.asarray(values, np.float32), dtype)


def f64(bits_, dtype="bf16"):
    return wl.bits_to_float(bits_, dtype).astype(np.float64)


# ---------------------------------------------------------------- hand-worked rows

@pytest.mark.parametrize("case", golden("tie_rows.json")["cases"], ids=lambda c: c["name"])
def test_hand_worked_rows(case):
    dt = case["dtype"]
    x1 = bits([case["x1"]], dt)
    x2 = bits([case["x2"]], dt)
    g = bits(case["gamma"], dt)
    b = bits(case["beta"], dt) if "beta" in case else None
    r = oracle.add_rms_norm_dynamic_quant_v2(x1, x2, g, b, eps=case["eps"], mask=case["mask"],
                                             qdtype=case["qdtype"], dtype=dt)
    assert r["status"] == oracle.ORC_OK
    assert np.array_equal(r["x_out"][0], bits(case["expect_x_out"], dt))
    if "expect_scale1" in case:
        assert r["scale1"][0] == np.float32(case["expect_scale1"])
    if "expect_scale1_rational" in case:
        assert r["scale1"][0] == f32_of_fraction(Fraction(*case["expect_scale1_rational"]))
    if "expect_y1" in case:
        assert r["y1"][0].tolist() == case["expect_y1"]
    if "expect_y1_packed" in case:
        assert r["y1"][0].tolist() == case["expect_y1_packed"]
        assert unpack_int4(r["y1"])[0].tolist() == case["expect_y1_codes"]
    if "expect_y1_words" in case:
        assert r["y1"].dtype == np.uint32
        assert r["y1"][0].tolist() == case["expect_y1_words"]
        assert unpack_int4_words(r["y1"])[0].tolist() == case["expect_y1_codes"]
    assert r["clamp_hits"] == 0


# ---------------------------------------------------------------- output selection

def test_mask_truth_table():
    t = golden("mask_truth_table.json")
    for mask, s1, s2, ok, y1, y2 in t["rows"]:
        st, on1, on2 = oracle.selected_outputs(None if mask is None else tuple(mask), s1, s2)
        assert (st == oracle.ORC_OK) == ok, (mask, s1, s2)
        if ok:
            assert (on1, on2) == (y1, y2), (mask, s1, s2)


def test_mask_truth_table_drives_the_outputs():
    w = wl.random_case(3, 16, seed=5, beta=True)
    s1, s2 = bits(np.linspace(0.5, 2.0, 16)), bits(np.linspace(3.0, 0.25, 16))
    for mask, h1, h2, ok, y1, y2 in golden("mask_truth_table.json")["rows"]:
        r = oracle.add_rms_norm_dynamic_quant_v2(
            w.x1, w.x2, w.gamma, w.beta, s1 if h1 else None, s2 if h2 else None, eps=1e-6,
            mask=None if mask is None else tuple(mask))
        assert (r["status"] == oracle.ORC_OK) == ok
        if ok:
            assert (r["y1"] is not None, r["y2"] is not None) == (y1, y2)
        else:
            assert r["status"] == oracle.ORC_BAD_MASK


def test_int4_containers_hold_the_same_codes():
    # the same row quantized into both INT4 containers: identical codes,
    # identical scales; the word container needs n % 8 == 0
    w = wl.random_case(5, 48, seed=9, beta=True, smooth1=True)
    a = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, w.beta, w.smooth1, eps=1e-6,
                                             qdtype="int4")
    b = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, w.beta, w.smooth1, eps=1e-6,
                                             qdtype="int4_int32")
    assert a["status"] == b["status"] == oracle.ORC_OK
    assert np.array_equal(a["scale1"], b["scale1"])
    assert np.array_equal(unpack_int4(a["y1"]), unpack_int4_words(b["y1"]))
    x = bits(np.ones((2, 12)))
    r = oracle.add_rms_norm_dynamic_quant_v2(x, x, bits(np.ones(12)), eps=1e-6,
                                             qdtype="int4_int32")
    assert r["status"] == oracle.ORC_BAD_SHAPE


def test_rejects_empty_and_odd_int4():
    g = bits(np.ones(8))
    e = np.zeros((0, 8), np.uint16)
    assert oracle.add_rms_norm_dynamic_quant_v2(e, e, g, eps=1e-6)["status"] == oracle.ORC_EMPTY
    x = bits(np.ones((2, 7)))
    r = oracle.add_rms_norm_dynamic_quant_v2(x, x, bits(np.ones(7)), eps=1e-6, qdtype="int4")
    assert r["status"] == oracle.ORC_BAD_SHAPE
    x = bits(np.ones((2, 8)))
    assert oracle.add_rms_norm_dynamic_quant_v2(x, x, g, eps=-1.0)["status"] == oracle.ORC_BAD_ARG


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("c,gam,eps", [(1.0, 1.0, 1e-6), (0.75, 2.0, 0.0), (-3.0, 0.5, 1e-6),
                                       (2.0 ** -10, 1.0, 1e-6), (2.0 ** -10, 1.25, 1e-5)])
@pytest.mark.parametrize("qdtype", ["int8", "int4"])
def test_constant_row(c, gam, eps, qdtype):
    """x = c everywhere, gamma = gam everywhere, no beta:
    y_j = c*gam/sqrt(c^2 + eps) for every j, so every code is sign(c*gam)*Q and
    scale = |c|*gam / (Q*sqrt(c^2 + eps))."""
    n = 64
    Q = oracle.QMAX[qdtype]
    x1 = bits(np.full((2, n), c))
    x2 = bits(np.zeros((2, n)))
    r = oracle.add_rms_norm_dynamic_quant_v2(x1, x2, bits(np.full(n, gam)), eps=eps,
                                             qdtype=qdtype)
    cq, eq = float(np.float32(c)), float(np.float32(eps))
    decimal.getcontext().prec = 50
    exact = Decimal(abs(cq)) * Decimal(gam) / (Q * (Decimal(cq) ** 2 + Decimal(eq)).sqrt())
    want = np.float32(float(exact))
    assert np.all(r["scale1"] == want), (r["scale1"], want)
    assert np.all(codes(r["y1"], qdtype) == np.sign(c * gam) * Q)


def test_constant_row_with_beta():
    """Constant x = c, gamma = 1, per-channel beta b_j: y_j = c/sqrt(c^2+eps) + b_j."""
    n = 16
    c, eps = 0.5, 1e-6
    b = np.linspace(-0.75, 0.75, n).astype(np.float32)
    r = oracle.add_rms_norm_dynamic_quant_v2(bits(np.full((1, n), c)), bits(np.zeros((1, n))),
                                             bits(np.ones(n)), bits(b), eps=eps, debug=True)
    beta64 = f64(bits(b))
    y = c / np.sqrt(c * c + float(np.float32(eps))) + beta64
    np.testing.assert_allclose(r["in1"][0], y, rtol=1e-15, atol=1e-15)
    j = int(np.argmax(np.abs(y)))
    assert codes(r["y1"], "int8")[0, j] == 127 * np.sign(y[j])


def test_single_nonzero_element():
    """One nonzero a at index k (others 0), gamma = 1, no beta:
    Rms = sqrt(a^2/n + eps), y_k = a/Rms, all other y = 0; so code_k = sign(a)*127,
    other codes 0, scale = |a|/(127*sqrt(a^2/n + eps)).  For n = 1024, a = 3,
    eps = 1e-6 this is 0.25195417..., close to the eps -> 0 limit sqrt(n)/127."""
    n, a, k = 1024, 3.0, 517
    x1 = np.zeros((1, n), np.float32)
    x1[0, k] = a
    r = oracle.add_rms_norm_dynamic_quant_v2(bits(x1), bits(np.zeros((1, n))), bits(np.ones(n)),
                                             eps=1e-6)
    decimal.getcontext().prec = 50
    e = Decimal(float(np.float32(1e-6)))
    exact = Decimal(a) / (127 * (Decimal(a) ** 2 / n + e).sqrt())
    assert r["scale1"][0] == np.float32(float(exact))
    assert abs(float(r["scale1"][0]) - 0.25195417) < 1e-7
    q = codes(r["y1"], "int8")[0]
    assert q[k] == 127 and np.count_nonzero(q) == 1


def test_sum_of_squares_uses_the_mean():
    """Two rows that differ only in n: with x = 1 at one index, Rms = sqrt(1/n + eps),
    so scale = 1/(127*Rms) grows like sqrt(n)."""
    out = []
    for n in (64, 256):
        x1 = np.zeros((1, n), np.float32)
        x1[0, 0] = 1.0
        r = oracle.add_rms_norm_dynamic_quant_v2(bits(x1), bits(np.zeros((1, n))),
                                                 bits(np.ones(n)), eps=0.0)
        out.append(float(r["scale1"][0]))
    assert out[0] == pytest.approx(np.sqrt(64) / 127, rel=1e-7)
    assert out[1] == pytest.approx(np.sqrt(256) / 127, rel=1e-7)


def test_dual_output_uses_its_own_smooth_scale():
    """Constant row, gamma = 1, eps = 0 -> y = 1.  input1 = s1, input2 = s2, so
    scale_k = max|s_k|/127 and the codes follow each smooth vector on its own."""
    n = 8
    s1 = np.array([1, 2, 3, 4, 5, 6, 7, 8], np.float32)
    s2 = np.array([8, -4, 2, 1, 0.5, 0.25, 0.125, 0], np.float32)
    r = oracle.add_rms_norm_dynamic_quant_v2(
        bits(np.ones((1, n))), bits(np.zeros((1, n))), bits(np.ones(n)), None, bits(s1),
        bits(s2), eps=0.0, mask=(True, True))
    assert r["scale1"][0] == f32_of_fraction(Fraction(8, 127))
    assert r["scale2"][0] == f32_of_fraction(Fraction(8, 127))
    q1 = codes(r["y1"], "int8")[0]
    q2 = codes(r["y2"], "int8")[0]
    # s/ (8/127) = s * 15.875
    assert q1.tolist() == [16, 32, 48, 64, 79, 95, 111, 127]
    assert q2.tolist() == [127, -64, 32, 16, 8, 4, 2, 0]


# ---------------------------------------------------------------- library special cases

@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_matches_torch_rms_norm_in_fp64(dtype):
    """With no smooth scale, input1 - beta equals torch's rms_norm of x (= xOut)."""
    w = wl.random_case(6, 640, dtype=dtype, seed=21, beta=True)
    r = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, w.beta, eps=1e-5, dtype=dtype,
                                             debug=True)
    x = torch.from_numpy(f64(r["x_out"], dtype))
    g = torch.from_numpy(f64(w.gamma, dtype))
    ref = torch.nn.functional.rms_norm(x, (w.n,), g, eps=float(np.float32(1e-5)))
    np.testing.assert_allclose(r["in1"] - f64(w.beta, dtype), ref.numpy(), rtol=1e-12, atol=1e-13)


def test_x_out_is_the_rounded_sum():
    w = wl.random_case(5, 300, seed=2)
    r = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, eps=1e-6)
    s = torch.from_numpy(wl.bits_to_float(w.x1, "bf16")) + torch.from_numpy(
        wl.bits_to_float(w.x2, "bf16"))
    ref = s.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(r["x_out"], ref)


def test_page5_operator_is_the_no_add_case():
    """outputMask [True, False] with smoothScale1 equals aclnnRmsNormDynamicQuant
    run on x = xOut with the same smooth scale."""
    w = wl.random_case(7, 512, seed=3, beta=True, smooth1=True)
    r = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, w.beta, w.smooth1, eps=1e-6,
                                             mask=(True, False))
    p = oracle.rms_norm_dynamic_quant(r["x_out"], w.gamma, w.beta, w.smooth1, eps=1e-6)
    assert np.array_equal(r["y1"], p["y"]) and np.array_equal(r["scale1"], p["scale"])
    assert r["y2"] is None


@pytest.mark.parametrize("qdtype", ["int8", "int4"])
def test_equivalences(qdtype):
    w = wl.random_case(4, 256, seed=9, beta=True)
    ones = bits(np.ones(256))
    zeros = bits(np.zeros(256))
    base = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, eps=1e-6, qdtype=qdtype)
    # smooth = 1 is no smooth; beta = 0 is no beta
    r = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, zeros, ones, eps=1e-6,
                                             qdtype=qdtype)
    assert np.array_equal(r["y1"], base["y1"]) and np.array_equal(r["scale1"], base["scale1"])
    # identical smooth scales give identical outputs
    s = bits(np.linspace(0.5, 2.0, 256))
    r = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, None, s, s, eps=1e-6,
                                             qdtype=qdtype)
    assert np.array_equal(r["y1"], r["y2"]) and np.array_equal(r["scale1"], r["scale2"])
    # x1 and x2 swap freely (binary32 addition commutes)
    r = oracle.add_rms_norm_dynamic_quant_v2(w.x2, w.x1, w.gamma, eps=1e-6, qdtype=qdtype)
    assert np.array_equal(r["y1"], base["y1"]) and np.array_equal(r["x_out"], base["x_out"])


def test_zero_row_gives_zero_scale_and_codes():
    x1 = bits(np.array([[1.5, -2.0, 0.25, 3.0]]))
    x2 = bits(np.array([[-1.5, 2.0, -0.25, -3.0]]))
    r = oracle.add_rms_norm_dynamic_quant_v2(x1, x2, bits(np.ones(4)), eps=1e-6)
    assert r["scale1"][0] == 0.0 and not r["y1"].any()


def test_sign_flip_symmetry():
    """Negating x1 and x2 (no beta) negates every code and keeps every scale."""
    w = wl.random_case(4, 128, seed=4)
    r = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, eps=1e-6)
    n = oracle.add_rms_norm_dynamic_quant_v2(w.x1 ^ 0x8000, w.x2 ^ 0x8000, w.gamma, eps=1e-6)
    assert np.array_equal(r["scale1"], n["scale1"])
    assert np.array_equal(codes(r["y1"], "int8"), -codes(n["y1"], "int8"))


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("qdtype,dtype", [("int8", "bf16"), ("int4", "bf16"), ("int8", "fp16"),
                                          ("int4", "fp16")])
def test_quantizer_invariants(qdtype, dtype):
    w = wl.random_case(64, 1000, seed=13, dtype=dtype, qdtype=qdtype, beta=True, smooth1=True,
                       smooth2=True, outlier_frac=0.01)
    r = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, w.beta, w.smooth1, w.smooth2,
                                             eps=1e-6, mask=(True, True), qdtype=qdtype,
                                             dtype=dtype, debug=True)
    Q = oracle.QMAX[qdtype]
    assert r["clamp_hits"] == 0
    for k in ("1", "2"):
        q = codes(r["y" + k], qdtype).astype(np.float64)
        s = r["scale" + k].astype(np.float64)[:, None]
        x = r["in" + k]
        assert np.all(np.abs(q) <= Q)
        assert np.all(np.max(np.abs(q), axis=1) == Q)
        assert np.all((np.sign(q) == np.sign(x)) | (q == 0))
        assert np.all(np.abs(s * q - x) <= s / 2 * (1 + 1e-6))
        assert np.all(s >= 0)
        # scale is row_max|input| / Q rounded once to binary32
        amax = np.max(np.abs(x), axis=1)
        assert np.array_equal(r["scale" + k], (amax / Q).astype(np.float32))


# ---------------------------------------------------------------- 50-digit evaluation

def _exact_codes(x1b, x2b, gb, bb, sb, eps, Q, dtype):
    """Evaluates the definition with 50-digit decimals on one row; returns the
    binary32 scale and the codes (None where the quotient is within 1e-9 of a
    tie, which fp64 cannot decide)."""
    decimal.getcontext().prec = 50
    xo = oracle.add_round(x1b, x2b, dtype)  # pinned above against torch
    x = [Decimal(float(v)) for v in f64(xo, dtype)]
    g = [Decimal(float(v)) for v in f64(gb, dtype)]
    b = [Decimal(float(v)) for v in f64(bb, dtype)] if bb is not None else None
    s = [Decimal(float(v)) for v in f64(sb, dtype)] if sb is not None else None
    n = len(x)
    rms = (sum(v * v for v in x) / n + Decimal(float(np.float32(eps)))).sqrt()
    inp = []
    for j in range(n):
        y = x[j] / rms * g[j] + (b[j] if b else 0)
        inp.append(y * s[j] if s else y)
    amax = max(abs(v) for v in inp)
    scale = f32_of_fraction(Fraction(amax / Q))
    out = []
    for v in inp:
        t = v / Decimal(float(scale))
        fl = t.to_integral_value(rounding=decimal.ROUND_FLOOR)
        if abs((t - fl) - Decimal("0.5")) < Decimal("1e-9"):
            out.append(None)
        else:
            out.append(int(t.to_integral_value(rounding=decimal.ROUND_HALF_EVEN)))
    return scale, out


@pytest.mark.parametrize("seed", range(6))
def test_fp64_oracle_agrees_with_50_digit_evaluation(seed):
    dtype = "bf16" if seed % 2 == 0 else "fp16"
    qdtype = "int8" if seed < 3 else "int4"
    w = wl.random_case(3, 48, seed=100 + seed, dtype=dtype, qdtype=qdtype, beta=True,
                       smooth1=True)
    r = oracle.add_rms_norm_dynamic_quant_v2(w.x1, w.x2, w.gamma, w.beta, w.smooth1, eps=1e-6,
                                             qdtype=qdtype, dtype=dtype)
    got = codes(r["y1"], qdtype)
    for i in range(w.rows):
        scale, ex = _exact_codes(w.x1[i], w.x2[i], w.gamma, w.beta, w.smooth1, 1e-6,
                                 oracle.QMAX[qdtype], dtype)
        assert r["scale1"][i] == scale
        for j, e in enumerate(ex):
            if e is not None:
                assert got[i, j] == e, (i, j)
