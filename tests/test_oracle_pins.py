"""Pins of the CPU oracle to facts fixed by the pages and by mathematics.

No CUDA here: these tests make the oracle trustworthy before anything is
compared against it. Which pin catches which plausible mistake:

* hand-computed rows (tests/golden/dynamic_quant_hand.txt, derived from the
  aclnnDynamicQuantV2 "Formula" section): wrong constants, wrong tie rule,
  wrong offset sign, wrong nibble order, wrong expert lookup;
* exact rational arithmetic (tests/exact_fp32.py): any binary32 operation
  done in another precision, fused, replaced by a reciprocal, or rounded with
  another tie rule;
* brute force over every finite fp16 value: the same, exhaustively over the
  input type, plus the fp16 widening;
* invariants of the formulas (absmax element to +-127, asymmetric max to
  offset_opt and min to offset_opt - scale_opt, dequantization error at most
  half a step, monotonicity, sign symmetry, power-of-two scale invariance):
  dropped terms, swapped max/min, transposed operands;
* library routines: bf16/fp16 widening against torch/numpy casts,
  expert lookup against numpy.searchsorted, LayerNorm against
  torch.nn.functional.layer_norm in float64 (aclnnAdaLayerNormQuant step 1);
* closed forms of the AdaLayerNorm path: scale = -1 leaves shift * smooth,
  a constant row leaves bias * (1 + scale) + shift.
"""

from fractions import Fraction
import os

import numpy as np
import pytest
import torch

import exact_fp32 as ex

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dynamic_quant_hand.txt")


def _rows(field, dtype=float):
    return [[dtype(t) for t in r.split()] for r in field.split(";")]


def _load_golden():
    records = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.strip() for p in line.split(" | ")]
            assert len(parts) == 9, line
            mode, y_dtype, xs, sm, gi, codes, packed, scales, offsets = parts
            records.append(dict(
                mode=mode, y_dtype=y_dtype, x=np.array(_rows(xs), np.float32),
                smooth=None if sm == "-" else np.array(_rows(sm), np.float32),
                group_index=None if gi == "-" else np.array([int(t) for t in gi.split()], np.int32),
                codes=np.array(_rows(codes, int), np.int64),
                packed=None if packed == "-" else packed.split(),
                scales=[Fraction(t) for t in scales.split()],
                offsets=None if offsets == "-" else [Fraction(t) for t in offsets.split()],
                line=line))
    return records


GOLDEN_RECORDS = _load_golden()


def _codes_of(y, y_dtype, cols, oracle):
    if y_dtype == "int8":
        return y.astype(np.int64)
    if y_dtype == "int4":
        return oracle.unpack_int4(y, cols).astype(np.int64)
    # int32 words -> bytes (little endian) -> nibbles
    return oracle.unpack_int4(y.view(np.uint8).reshape(y.shape[0], -1), cols).astype(np.int64)


@pytest.mark.parametrize("rec", GOLDEN_RECORDS, ids=[f"golden{i + 1}" for i in range(len(GOLDEN_RECORDS))])
def test_hand_computed_rows(oracle_mod, rec):
    smooth = rec["smooth"]
    if smooth is not None and rec["group_index"] is None:
        smooth = smooth[0]
    y, scale, offset = oracle_mod.dynamic_quant(rec["x"], smooth=smooth, group_index=rec["group_index"],
                                                mode=rec["mode"], y_dtype=rec["y_dtype"])
    cols = rec["x"].shape[1]
    np.testing.assert_array_equal(_codes_of(y, rec["y_dtype"], cols, oracle_mod), rec["codes"])
    if rec["packed"] is not None:
        if rec["y_dtype"] == "int4":
            assert [int(b) for b in y.reshape(-1)] == [int(t) for t in rec["packed"]]
        else:
            assert [int(w) for w in y.reshape(-1)] == [int(t, 16) for t in rec["packed"]]
    expected_scales = [ex.rn32(s) for s in rec["scales"]]
    assert [Fraction(float(s)) for s in scale] == expected_scales
    if rec["offsets"] is not None:
        assert [Fraction(float(o)) for o in offset] == [ex.rn32(o) for o in rec["offsets"]]


# ---------------------------------------------------------------- exact arithmetic

@pytest.mark.parametrize("mode,y_dtype", [("symmetric", "int8"), ("asymmetric", "int8"),
                                          ("symmetric", "int4"), ("asymmetric", "int4")])
def test_exact_rational_chain(oracle_mod, mode, y_dtype):
    rng = np.random.default_rng(11)
    rows, cols = 24, 40
    x = (rng.standard_normal((rows, cols)) * rng.uniform(0.01, 50.0, (rows, 1)) + rng.uniform(-3, 3, (rows, 1)))
    x = x.astype(np.float16)  # the inputs are fp16 values
    y, scale, offset = oracle_mod.dynamic_quant(x, mode=mode, y_dtype=y_dtype)
    codes = _codes_of(y, y_dtype, cols, oracle_mod)
    for r in range(rows):
        want, s, o = ex.exact_codes_row(x[r].astype(np.float32), mode, y_dtype != "int8")
        assert list(codes[r]) == want, f"row {r}"
        assert Fraction(float(scale[r])) == s
        if mode == "asymmetric":
            assert Fraction(float(offset[r])) == o


def test_exact_chain_with_smooth_product(oracle_mod):
    """input = x * smooth is one binary32 multiply (aclnnDynamicQuantV2, Formula)."""
    rng = np.random.default_rng(12)
    rows, cols = 8, 33
    x = rng.standard_normal((rows, cols)).astype(np.float16)
    smooth = rng.uniform(0.5, 2.0, cols).astype(np.float32)
    for mode in ("symmetric", "asymmetric"):
        y, scale, offset = oracle_mod.dynamic_quant(x, smooth=smooth, mode=mode)
        for r in range(rows):
            prod = [ex.f32(ex.rn32(Fraction(float(a)) * Fraction(float(b)))) for a, b in zip(x[r], smooth)]
            want, s, o = ex.exact_codes_row(prod, mode, False)
            assert list(y[r].astype(int)) == want
            assert Fraction(float(scale[r])) == s


def _finite_fp16_values():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    return vals[np.isfinite(vals)]


def test_brute_force_every_fp16_value_symmetric(oracle_mod):
    """Every finite fp16 value in one row (absmax 65504): each code is the exactly
    rounded quotient, rounded half to even."""
    vals = _finite_fp16_values()
    x = vals.reshape(1, -1)
    y, scale, _ = oracle_mod.dynamic_quant(x, mode="symmetric")
    s = ex.rn32(Fraction(65504) / 127)
    assert Fraction(float(scale[0])) == s
    got = y[0].astype(int)
    for v, q in zip(vals.astype(np.float64), got):
        assert q == ex.rne_int(ex.rn32(Fraction(v) / s)), v


def test_brute_force_every_fp16_value_asymmetric(oracle_mod):
    vals = _finite_fp16_values()
    x = vals.reshape(1, -1)
    y, scale, offset = oracle_mod.dynamic_quant(x, mode="asymmetric")
    s = ex.rn32(ex.rn32(Fraction(65504) - Fraction(-65504)) / 255)
    o = ex.rn32(127 - ex.rn32(Fraction(65504) / s))
    assert Fraction(float(scale[0])) == s
    assert Fraction(float(offset[0])) == o
    got = y[0].astype(int)
    for v, q in zip(vals.astype(np.float64), got):
        want = min(127, max(-128, ex.rne_int(ex.rn32(ex.rn32(Fraction(v) / s) + o))))
        assert q == want, v


# ---------------------------------------------------------------- widening (library casts)

def test_fp16_widening_matches_numpy_cast(oracle_mod):
    vals = _finite_fp16_values()
    rng = np.random.default_rng(1)
    rng.shuffle(vals)
    x16 = vals[: 256 * 240].reshape(256, 240)
    for mode in ("symmetric", "asymmetric"):
        a = oracle_mod.dynamic_quant(x16, mode=mode)
        b = oracle_mod.dynamic_quant(x16.astype(np.float32), mode=mode)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


def test_bf16_widening_matches_torch_cast(oracle_mod):
    g = torch.Generator().manual_seed(5)
    bits = torch.randint(-(1 << 15), 1 << 15, (300, 128), generator=g, dtype=torch.int32).to(torch.int16)
    xb = bits.view(torch.bfloat16)
    xb = torch.where(torch.isfinite(xb), xb, torch.zeros_like(xb))
    for mode in ("symmetric", "asymmetric"):
        a = oracle_mod.dynamic_quant(xb, mode=mode)
        b = oracle_mod.dynamic_quant(xb.float(), mode=mode)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


# ---------------------------------------------------------------- invariants

def _random_rows(seed, rows=64, cols=257, dtype=np.float16):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)) * rng.uniform(0.05, 30, (rows, 1)) + rng.uniform(-5, 5, (rows, 1))
    return x.astype(dtype)


def test_symmetric_invariants(oracle_mod):
    x = _random_rows(21)
    xf = x.astype(np.float64)
    for y_dtype, top in (("int8", 127), ("int4", 7)):
        cols = x.shape[1] - (x.shape[1] % 2)
        xx = x[:, :cols]
        y, scale, _ = oracle_mod.dynamic_quant(xx, mode="symmetric", y_dtype=y_dtype)
        q = _codes_of(y, y_dtype, cols, oracle_mod)
        v = xf[:, :cols]
        assert np.abs(q).max() <= top
        arg = np.abs(v).argmax(axis=1)
        rows = np.arange(v.shape[0])
        np.testing.assert_array_equal(q[rows, arg], np.sign(v[rows, arg]) * top)
        # sign preserved, and zero only for small elements
        assert np.all(np.sign(q) * np.sign(v) >= 0)
        # dequantization error at most half a step (plus binary32 quotient error)
        s = scale.astype(np.float64)[:, None]
        assert np.all(np.abs(v - q * s) <= s * (0.5 + 1e-5))
        # the scale is absmax / top up to one binary32 rounding
        np.testing.assert_allclose(scale, np.abs(v).max(axis=1) / top, rtol=2 ** -23)


def test_asymmetric_invariants(oracle_mod):
    x = _random_rows(22)
    xf = x.astype(np.float64)
    rows = np.arange(x.shape[0])
    for y_dtype, (scale_opt, offset_opt) in (("int8", (255, 127)), ("int4", (15, 7))):
        cols = x.shape[1] - (x.shape[1] % 2)
        v = xf[:, :cols]
        y, scale, offset = oracle_mod.dynamic_quant(x[:, :cols], mode="asymmetric", y_dtype=y_dtype)
        q = _codes_of(y, y_dtype, cols, oracle_mod)
        lo, hi = offset_opt - scale_opt, offset_opt
        assert q.min() >= lo and q.max() <= hi
        # the row max lands on offset_opt, the row min on offset_opt - scale_opt
        np.testing.assert_array_equal(q[rows, v.argmax(axis=1)], hi)
        np.testing.assert_array_equal(q[rows, v.argmin(axis=1)], lo)
        # dequantization: x ~ (q - offset) * scale within half a step
        s = scale.astype(np.float64)[:, None]
        o = offset.astype(np.float64)[:, None]
        assert np.all(np.abs(v - (q - o) * s) <= s * (0.5 + 1e-4))
        np.testing.assert_allclose(scale, (v.max(axis=1) - v.min(axis=1)) / scale_opt, rtol=2 ** -22)


@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
def test_monotone(oracle_mod, mode):
    x = _random_rows(23, rows=16, cols=300)
    y, _, _ = oracle_mod.dynamic_quant(x, mode=mode)
    for r in range(x.shape[0]):
        order = np.argsort(x[r].astype(np.float64), kind="stable")
        assert np.all(np.diff(y[r].astype(int)[order]) >= 0)


def test_symmetric_negation(oracle_mod):
    x = _random_rows(24)
    a = oracle_mod.dynamic_quant(x)
    b = oracle_mod.dynamic_quant(-x)
    np.testing.assert_array_equal(a[0].astype(int), -b[0].astype(int))
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
def test_power_of_two_scaling(oracle_mod, mode):
    """Multiplying a row by 2^k multiplies the scale by 2^k and leaves codes and offset."""
    x = _random_rows(25).astype(np.float32)
    a = oracle_mod.dynamic_quant(x, mode=mode)
    b = oracle_mod.dynamic_quant(x * np.float32(8.0), mode=mode)
    c = oracle_mod.dynamic_quant(x, smooth=np.full(x.shape[1], 0.25, np.float32), mode=mode)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1] * 8, b[1])
    np.testing.assert_array_equal(a[0], c[0])
    np.testing.assert_array_equal(a[1] / 4, c[1])
    if mode == "asymmetric":
        np.testing.assert_array_equal(a[2], b[2])
        np.testing.assert_array_equal(a[2], c[2])


# ---------------------------------------------------------------- smooth scales and MoE

@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
def test_unit_smooth_is_identity(oracle_mod, mode):
    x = _random_rows(26)
    a = oracle_mod.dynamic_quant(x, mode=mode)
    b = oracle_mod.dynamic_quant(x, smooth=np.ones(x.shape[1], np.float32), mode=mode)
    for u, v in zip(a, b):
        if u is not None:
            np.testing.assert_array_equal(u, v)


def test_single_expert_equals_dense_smooth(oracle_mod):
    x = _random_rows(27, rows=40, cols=96)
    sm = np.random.default_rng(3).uniform(0.5, 2.0, (1, 96)).astype(np.float32)
    a = oracle_mod.dynamic_quant(x, smooth=sm[0])
    b = oracle_mod.dynamic_quant(x, smooth=sm, group_index=[40])
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_moe_rows_use_their_expert(oracle_mod):
    """Each row equals a dense-smooth call with the smooth row that
    numpy.searchsorted(group_index, r, 'right') selects (the cumulative
    end-row reading of groupIndexOptional), including empty experts."""
    rows, cols, experts = 50, 64, 7
    x = _random_rows(28, rows=rows, cols=cols)
    sm = np.random.default_rng(4).uniform(0.5, 2.0, (experts, cols)).astype(np.float32)
    gi = np.array([3, 3, 20, 21, 21, 45, 50], np.int32)  # experts 1 and 4 are empty
    for mode in ("symmetric", "asymmetric"):
        y, scale, offset = oracle_mod.dynamic_quant(x, smooth=sm, group_index=gi, mode=mode)
        expert = np.searchsorted(gi, np.arange(rows), side="right")
        for r in range(rows):
            yr, sr, orr = oracle_mod.dynamic_quant(x[r:r + 1], smooth=sm[expert[r]], mode=mode)
            np.testing.assert_array_equal(y[r], yr[0])
            assert scale[r] == sr[0]
            if mode == "asymmetric":
                assert offset[r] == orr[0]


def test_moe_rows_past_last_group_rejected(oracle_mod):
    x = _random_rows(29, rows=10, cols=16)
    sm = np.ones((2, 16), np.float32)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.dynamic_quant(x, smooth=sm, group_index=[4, 9])
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.dynamic_quant(x, smooth=sm, group_index=[6, 4])


def test_int32_container_is_int4_bytes(oracle_mod):
    """INT32 output holds the same nibbles as packed INT4, eight per word."""
    x = _random_rows(30, rows=12, cols=64)
    for mode in ("symmetric", "asymmetric"):
        a = oracle_mod.dynamic_quant(x, mode=mode, y_dtype="int4")
        b = oracle_mod.dynamic_quant(x, mode=mode, y_dtype="int32")
        np.testing.assert_array_equal(a[0], b[0].view(np.uint8).reshape(a[0].shape))


def test_shape_errors(oracle_mod):
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.dynamic_quant(np.zeros((2, 3), np.float32), y_dtype="int4")
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.dynamic_quant(np.zeros((2, 12), np.float32), y_dtype="int32")


# ---------------------------------------------------------------- AdaLayerNorm

def _ada_inputs(seed, b=2, s=5, h=48, x_scale=1.0, x_mean=0.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(b, s, h, generator=g) * x_scale + x_mean).to(torch.bfloat16)
    sc = (torch.randn(b, h, generator=g) * 0.1).to(torch.bfloat16)
    sh = (torch.randn(b, h, generator=g) * 0.1).to(torch.bfloat16)
    w = (1 + torch.randn(h, generator=g) * 0.05).to(torch.bfloat16)
    bias = (torch.randn(h, generator=g) * 0.05).to(torch.bfloat16)
    sm = (torch.rand(h, generator=g) * 1.5 + 0.5).to(torch.bfloat16)
    return x, sc, sh, w, bias, sm


@pytest.mark.parametrize("x_scale,x_mean,eps", [(1.0, 0.0, 1e-6), (3.0, 2.0, 1e-5), (1e-3, 1.0, 1e-6)])
def test_layernorm_matches_torch_float64(oracle_mod, x_scale, x_mean, eps):
    """Step 1 against torch.nn.functional.layer_norm (biased variance, epsilon
    inside the square root); steps 2-3 follow the printed affine form."""
    x, sc, sh, w, bias, sm = _ada_inputs(31, x_scale=x_scale, x_mean=x_mean)
    y, mean, std = oracle_mod.ada_layernorm_pre(x, sc, sh, w, bias, sm, epsilon=eps)
    xd = x.double()
    ln = torch.nn.functional.layer_norm(xd, (x.shape[-1],), w.double(), bias.double(), eps)
    want = (ln * (1 + sc.double()[:, None, :]) + sh.double()[:, None, :]) * sm.double()
    # binary32 evaluation: rounding E(x) to fp32 moves x - E(x) by up to u*|E(x)|,
    # which the division by sigma magnifies; the affine factors are below 4 here.
    u = 2.0 ** -24
    sigma = torch.sqrt(xd.var(-1, unbiased=False, keepdim=True) + eps)
    atol = 4 * (u * xd.mean(-1, keepdim=True).abs() / sigma) * 4 + 1e-6
    err = (torch.from_numpy(y).double() - want).abs()
    assert torch.all(err <= atol + 1e-5 * want.abs()), float((err - atol - 1e-5 * want.abs()).max())
    np.testing.assert_allclose(mean, xd.mean(-1).reshape(-1).numpy(), rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(std, torch.sqrt(xd.var(-1, unbiased=False) + eps).reshape(-1).numpy(),
                               rtol=1e-6)
    # plain LayerNorm: no weight/bias, zero adaptive parameters, no smooth
    z = torch.zeros_like(sc)
    y0, _, _ = oracle_mod.ada_layernorm_pre(x, z, z, epsilon=eps)
    ln0 = torch.nn.functional.layer_norm(xd, (x.shape[-1],), None, None, eps)
    err0 = (torch.from_numpy(y0).double() - ln0).abs()
    assert torch.all(err0 <= atol + 1e-5 * ln0.abs())


def test_ada_scale_minus_one_leaves_shift(oracle_mod):
    """y = LN * (1 + (-1)) + shift = shift exactly; with smooth, shift * smooth."""
    x, sc, sh, w, bias, sm = _ada_inputs(32)
    minus_one = torch.full_like(sc, -1.0)
    y, _, _ = oracle_mod.ada_layernorm_pre(x, minus_one, sh, w, bias, sm)
    want = (sh.float() * sm.float())[:, None, :].expand(*y.shape)
    np.testing.assert_array_equal(y, want.numpy())
    out, qs = oracle_mod.ada_layernorm_quant(x, minus_one, sh, w, bias, sm)
    ref_y, ref_s, _ = oracle_mod.dynamic_quant((sh.float() * sm.float()).numpy())
    for b in range(x.shape[0]):
        np.testing.assert_array_equal(out[b], np.broadcast_to(ref_y[b], out[b].shape))
        np.testing.assert_array_equal(qs[b], ref_s[b])


def test_ada_constant_row(oracle_mod):
    """A constant row has Var = 0, so LN = bias and y = bias * (1 + scale) + shift."""
    x, sc, sh, w, bias, sm = _ada_inputs(33)
    x = torch.full_like(x, 0.75)
    y, mean, std = oracle_mod.ada_layernorm_pre(x, sc, sh, w, bias, None, epsilon=1e-6)
    want = bias.float() * (1 + sc.float()) + sh.float()
    for s in range(x.shape[1]):
        np.testing.assert_array_equal(y[:, s, :], want.numpy())
    assert np.all(mean == np.float32(0.75))


def test_ada_quant_is_dynamic_quant_of_prologue(oracle_mod):
    """Steps 4-5 are the symmetric INT8 DynamicQuant of the step-3 value."""
    x, sc, sh, w, bias, sm = _ada_inputs(34, b=3, s=7, h=80)
    y, _, _ = oracle_mod.ada_layernorm_pre(x, sc, sh, w, bias, sm)
    out, qs = oracle_mod.ada_layernorm_quant(x, sc, sh, w, bias, sm)
    ry, rs, _ = oracle_mod.dynamic_quant(y.reshape(-1, y.shape[-1]))
    np.testing.assert_array_equal(out.reshape(ry.shape), ry)
    np.testing.assert_array_equal(qs.reshape(-1), rs)
    assert np.abs(out).max() == 127


def _preimages_of_half_integers(halves, scale, shift=Fraction(0), steps=3):
    """binary32 values v with v/scale + shift within a few ulps of a half-integer."""
    out = []
    for h in halves:
        v0 = np.float32(float((Fraction(h) - shift) * scale))
        v = v0
        for _ in range(steps):
            v = np.nextafter(v, np.float32(-np.inf), dtype=np.float32)
        for _ in range(2 * steps + 1):
            out.append(np.float32(v))
            v = np.nextafter(v, np.float32(np.inf), dtype=np.float32)
    return out


def test_asymmetric_rounding_order_near_ties(oracle_mod):
    """x/scale and + offset are two binary32 roundings (aclnnDynamicQuantV2,
    Formula, asymmetric). Elements sit next to rounding ties, where that
    differs from one rounding of x/scale + offset or from a reciprocal-multiply
    fused with the addition, so a fused or reordered evaluation fails."""
    mn, mx = np.float32(0.0), np.float32(3.0)
    s = ex.rn32(Fraction(float(mx)) / 255)
    o = ex.rn32(127 - ex.rn32(Fraction(float(mx)) / s))
    halves = [Fraction(2 * k + 1, 2) for k in range(-128, 127)]
    picked = [v for v in _preimages_of_half_integers(halves, s, o) if mn <= v <= mx]
    discriminating = 0
    for v in picked:
        fv = Fraction(float(v))
        two_step = ex.rne_int(ex.rn32(ex.rn32(fv / s) + o))
        one_step = ex.rne_int(ex.rn32(fv / s + o))
        fused_recip = ex.rne_int(ex.rn32(fv * ex.rn32(1 / s) + o))
        discriminating += (two_step != one_step) or (two_step != fused_recip)
    assert discriminating >= 3, discriminating
    row = np.array([[mn, mx] + picked], np.float32)
    y, scale, offset = oracle_mod.dynamic_quant(row, mode="asymmetric")
    assert Fraction(float(scale[0])) == s and Fraction(float(offset[0])) == o
    want, _, _ = ex.exact_codes_row(row[0], "asymmetric", False)
    assert list(y[0].astype(int)) == want


def test_symmetric_quotient_near_ties(oracle_mod):
    """x/scale is one binary32 division; a reciprocal multiply differs near ties."""
    amax = np.float32(3.0)
    s = ex.rn32(Fraction(float(amax)) / 127)
    halves = [Fraction(2 * k + 1, 2) for k in range(-127, 127)]
    picked = [v for v in _preimages_of_half_integers(halves, s) if abs(v) <= amax]
    discriminating = 0
    for v in picked:
        fv = Fraction(float(v))
        discriminating += ex.rne_int(ex.rn32(fv / s)) != ex.rne_int(ex.rn32(fv * ex.rn32(1 / s)))
    assert discriminating >= 3, discriminating
    row = np.array([[amax] + picked], np.float32)
    y, scale, _ = oracle_mod.dynamic_quant(row)
    want, _, _ = ex.exact_codes_row(row[0], "symmetric", False)
    assert list(y[0].astype(int)) == want


# ---------------------------------------------------------------- PER_TOKEN dequantization (AntiQuantize)

def _load_antiquant_golden():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "antiquant_per_token.txt")
    recs = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        y_dtype, codes, scale, offset, out_dtype, want = (f.strip() for f in line.split("|"))
        rows = lambda t, conv=float: [[conv(v) for v in r.split()] for r in t.split(";")]
        recs.append(dict(y_dtype=y_dtype, codes=np.array(rows(codes, int), np.int64),
                         scale=[float(v) for v in scale.split()],
                         offset=None if offset == "-" else [float(v) for v in offset.split()],
                         out_dtype=out_dtype, want=np.array(rows(want), np.float64)))
    return recs


def _pack_int4(codes):
    c = (np.asarray(codes, np.int64) & 0xF).astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def _as_float64(out, out_dtype):
    if out_dtype == "bf16":
        return (out.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return out.astype(np.float64)


ANTIQUANT_RECORDS = _load_antiquant_golden()


@pytest.mark.parametrize("rec", ANTIQUANT_RECORDS, ids=[f"antiquant{i + 1}" for i in range(len(ANTIQUANT_RECORDS))])
def test_antiquant_worked_examples(oracle_mod, rec):
    codes = rec["codes"]
    y = codes.astype(np.int8) if rec["y_dtype"] == "int8" else _pack_int4(codes)
    sdt = np.float16 if rec["out_dtype"] == "f16" else np.float32
    scale = np.array(rec["scale"], sdt)
    offset = None if rec["offset"] is None else np.array(rec["offset"], sdt)
    out = oracle_mod.dequant_per_token(y, scale, offset, y_dtype=rec["y_dtype"], cols=codes.shape[1],
                                       out_dtype=rec["out_dtype"])
    np.testing.assert_array_equal(_as_float64(out, rec["out_dtype"]), rec["want"])


def test_narrowing_matches_library_conversions(oracle_mod):
    """binary32 -> binary16 (numpy) and -> bfloat16 (torch), round to nearest even:
    random bit patterns plus ties, subnormals, overflow and specials. The values
    go through the dequantizer as code 1 times a per-row scale (exact)."""
    import torch

    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    ties_h = (np.arange(-3000, 3000, dtype=np.float64) + 0.5) * 2.0 ** -24       # subnormal half ties
    ties_h2 = (np.arange(1024, 2048, dtype=np.float64) + 0.5) * 2.0 ** -10      # normal half ties in [1, 2)
    ties_b = (np.arange(128, 256, dtype=np.float64) + 0.5) * 2.0 ** -7          # bfloat16 ties in [1, 2)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 65504.0, 65519.99, 65520.0, 65536.0, 6e-8, 3e-8,
                        2.0 ** -149, 3.4e38, -3.4e38, 1e-40], np.float64)
    v = np.concatenate([v, ties_h.astype(np.float32), ties_h2.astype(np.float32), ties_b.astype(np.float32),
                        special.astype(np.float32)])
    v = v[np.isfinite(v) | np.isinf(v)]
    ones = np.ones((v.size, 1), np.int8)
    got_h = oracle_mod.dequant_per_token(ones, v, out_dtype="f16")[:, 0]
    with np.errstate(over="ignore"):
        want_h = v.astype(np.float16)
    assert np.array_equal(got_h.view(np.uint16), want_h.view(np.uint16))
    got_b = oracle_mod.dequant_per_token(ones, v, out_dtype="bf16")[:, 0]
    want_b = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got_b, want_b)
    nan = oracle_mod.dequant_per_token(np.ones((1, 1), np.int8), np.array([np.nan], np.float32), out_dtype="bf16")
    assert (int(nan[0, 0]) & 0x7F80) == 0x7F80 and (int(nan[0, 0]) & 0x7F) != 0


@pytest.mark.parametrize("mode,y_dtype", [("symmetric", "int8"), ("asymmetric", "int8"), ("symmetric", "int4"),
                                          ("asymmetric", "int4"), ("asymmetric", "int32")])
def test_dequant_inverts_the_quantizer(oracle_mod, mode, y_dtype):
    """quant then dequant returns every element to within half a quantization
    step (plus fp32 rounding): |x - (q - offset) * scale| <= scale / 2 * (1 + 2^-10).
    Read with the other offset sign, asymmetric rows miss by ~2 * offset * scale."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((64, 96)) * rng.uniform(0.01, 50, size=(64, 1)) + rng.uniform(-5, 5, size=(64, 1)))
    x = x.astype(np.float32)
    y, scale, offset = oracle_mod.dynamic_quant(x, mode=mode, y_dtype=y_dtype)
    back = oracle_mod.dequant_per_token(y, scale, offset, y_dtype=y_dtype, cols=96, out_dtype="f32")
    err = np.abs(back.astype(np.float64) - x.astype(np.float64))
    # half a step, plus the binary32 roundings of x / scale (+ offset) and of
    # (code - offset) * scale: each below 2^-24 of a value under 2^8 steps
    bound = scale.astype(np.float64)[:, None] / 2 * (1 + 2.0 ** -10) + 1e-30
    assert np.all(err <= bound)
    if offset is not None:
        # the other sign moves every element of a row by 2 * offset * scale
        wrong = ((_codes_signed(oracle_mod, y, y_dtype, 96) + offset[:, None]) * scale[:, None]).astype(np.float32)
        far = np.abs(offset) >= 1
        assert far.sum() > 10
        miss = np.abs(wrong - x).max(axis=1)
        assert np.all(miss[far] >= 1.5 * scale[far])


def _codes_signed(oracle_mod, y, y_dtype, cols):
    if y_dtype == "int8":
        return y.astype(np.float64)
    if y_dtype == "int4":
        return oracle_mod.unpack_int4(y, cols).astype(np.float64)
    return oracle_mod.unpack_int4(y.view(np.uint8).reshape(y.shape[0], -1), cols).astype(np.float64)


def test_dequant_power_of_two_scales_are_exact(oracle_mod):
    """scale 2^k and integer offsets: (q - o) * 2^k is exact in binary32."""
    rng = np.random.default_rng(3)
    codes = rng.integers(-128, 128, size=(40, 64)).astype(np.int8)
    k = rng.integers(-20, 20, size=40)
    scale = np.ldexp(np.ones(40), k).astype(np.float32)
    off = rng.integers(-128, 128, size=40).astype(np.float32)
    out = oracle_mod.dequant_per_token(codes, scale, off, out_dtype="f32")
    want = (codes.astype(np.float64) - off[:, None]) * np.ldexp(1.0, k)[:, None]
    np.testing.assert_array_equal(out.astype(np.float64), want)


def test_dequant_int32_container_matches_int4(oracle_mod):
    rng = np.random.default_rng(4)
    codes = rng.integers(-8, 8, size=(5, 32))
    packed = _pack_int4(codes)
    scale = rng.uniform(0.1, 2, 5).astype(np.float32)
    a = oracle_mod.dequant_per_token(packed, scale, y_dtype="int4", cols=32)
    b = oracle_mod.dequant_per_token(packed.view(np.uint32), scale, y_dtype="int32", cols=32)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(a, (codes.astype(np.float32) * scale[:, None]).astype(np.float32))


def test_dequant_shape_errors(oracle_mod):
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.dequant_per_token(np.zeros((2, 3), np.uint8), np.ones(2, np.float32), y_dtype="int4", cols=5)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.dequant_per_token(np.zeros((2, 1), np.uint32), np.ones(2, np.float32), y_dtype="int32", cols=4)


# ---------------------------------------------------------------- PER_GROUP dequantization (AntiQuantize)

def _load_group_golden():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "antiquant_per_group.txt")
    recs = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k_dim, g, codes, scale, offset, want = (f.strip() for f in line.split("|"))
        rows = lambda t, conv=float: np.array([[conv(v) for v in r.split()] for r in t.split(";")])
        recs.append(dict(k_dim=int(k_dim), g=int(g), codes=rows(codes, int).astype(np.int8),
                         scale=rows(scale).astype(np.float32), offset=rows(offset).astype(np.float32),
                         want=rows(want)))
    return recs


GROUP_RECORDS = _load_group_golden()


@pytest.mark.parametrize("rec", GROUP_RECORDS, ids=[f"group{i + 1}" for i in range(len(GROUP_RECORDS))])
def test_per_group_worked_examples(oracle_mod, rec):
    out = oracle_mod.dequant_per_group(rec["codes"], rec["scale"], rec["offset"], group_size=rec["g"],
                                       k_dim=rec["k_dim"], out_dtype="f32")
    np.testing.assert_array_equal(out.astype(np.float64), rec["want"])


def _group_case(rows, cols, g, k_dim, seed, sdt=np.float32):
    rng = np.random.default_rng(seed)
    codes = rng.integers(-128, 128, size=(rows, cols)).astype(np.int8)
    shape = (rows, -(-cols // g)) if k_dim == 1 else (-(-rows // g), cols)
    scale = rng.uniform(1e-3, 0.1, size=shape).astype(sdt)
    offset = rng.normal(0, 10, size=shape).astype(sdt)
    return codes, scale, offset


@pytest.mark.parametrize("out_dtype", ["f32", "f16", "bf16"])
def test_per_group_row_groups_are_per_token_on_the_reshaped_rows(oracle_mod, out_dtype):
    """kDim 1 with g | cols: each row splits into cols/g independent groups, which
    is the PER_TOKEN dequantizer on the [rows*cols/g, g] view."""
    rows, cols, g = 6, 256, 64
    codes, scale, offset = _group_case(rows, cols, g, 1, seed=1)
    got = oracle_mod.dequant_per_group(codes, scale, offset, group_size=g, k_dim=1, out_dtype=out_dtype)
    want = oracle_mod.dequant_per_token(codes.reshape(-1, g), scale.reshape(-1), offset.reshape(-1),
                                        out_dtype=out_dtype).reshape(rows, cols)
    np.testing.assert_array_equal(got.view(np.uint16) if out_dtype != "f32" else got,
                                  want.view(np.uint16) if out_dtype != "f32" else want)


def test_per_group_one_group_per_row_is_per_token(oracle_mod):
    codes, scale, offset = _group_case(5, 100, 128, 1, seed=2)
    got = oracle_mod.dequant_per_group(codes, scale, offset, group_size=128, k_dim=1)
    np.testing.assert_array_equal(got, oracle_mod.dequant_per_token(codes, scale[:, 0], offset[:, 0]))


@pytest.mark.parametrize("rows,g", [(96, 32), (70, 32), (40, 64)])
def test_per_group_column_groups_are_row_groups_of_the_transpose(oracle_mod, rows, g):
    """kDim 0 on [m, n] equals kDim 1 on the transpose [n, m] with the transposed
    table; with g >= m it is per-channel (one scale per column)."""
    cols = 48
    codes, scale, offset = _group_case(rows, cols, g, 0, seed=rows)
    got = oracle_mod.dequant_per_group(codes, scale, offset, group_size=g, k_dim=0, out_dtype="bf16")
    want = oracle_mod.dequant_per_group(np.ascontiguousarray(codes.T), np.ascontiguousarray(scale.T),
                                        np.ascontiguousarray(offset.T), group_size=g, k_dim=1, out_dtype="bf16").T
    np.testing.assert_array_equal(got, want)
    if g >= rows:
        per_channel = oracle_mod.dequant_per_token(np.ascontiguousarray(codes.T), scale[0], offset[0],
                                                   out_dtype="bf16").T
        np.testing.assert_array_equal(got, per_channel)


def test_per_group_argument_errors(oracle_mod):
    codes, scale, offset = _group_case(4, 64, 32, 1, seed=3)
    for kw in (dict(group_size=16), dict(group_size=0), dict(group_size=48), dict(k_dim=2)):
        args = dict(group_size=32, k_dim=1)
        args.update(kw)
        with pytest.raises(oracle_mod.OracleError):
            oracle_mod.dequant_per_group(codes, scale, offset, **args)


# ---------------------------------------------------------------- W8A8 product (aclnnQuantBatchMatmulInplaceAdd)

def _int8(rng, shape):
    return rng.integers(-128, 128, size=shape).astype(np.int8)


def test_w8a8_unit_scales_are_the_integer_product(oracle_mod):
    """With scales 1 the value is the exact integer sum (below 2^24 it is
    exact in binary32), checked against numpy's int64 matmul."""
    rng = np.random.default_rng(21)
    a, b = _int8(rng, (40, 512)), _int8(rng, (24, 512))
    got = oracle_mod.w8a8_gemm(a, b, np.ones(40), np.ones(24))
    want = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.abs(want).max() < 2 ** 24
    np.testing.assert_array_equal(got.astype(np.int64), want)


def test_w8a8_power_of_two_scales_are_exact(oracle_mod):
    rng = np.random.default_rng(22)
    a, b = _int8(rng, (16, 256)), _int8(rng, (12, 256))
    ka, kb = rng.integers(-10, 10, 16), rng.integers(-10, 10, 12)
    got = oracle_mod.w8a8_gemm(a, b, np.ldexp(1.0, ka), np.ldexp(1.0, kb))
    want = (a.astype(np.int64) @ b.astype(np.int64).T) * np.ldexp(1.0, ka[:, None] + kb[None, :])
    np.testing.assert_array_equal(got.astype(np.float64), want)


def test_w8a8_operand_roles_transpose(oracle_mod):
    """Swapping the operands (and their scales) transposes the product: catches
    an index mix-up between a[m,k] and b[n,k]."""
    rng = np.random.default_rng(23)
    a, b = _int8(rng, (9, 96)), _int8(rng, (13, 96))
    sa, sb = rng.uniform(0.01, 2, 9).astype(np.float32), rng.uniform(0.01, 2, 13).astype(np.float32)
    x = oracle_mod.w8a8_gemm(a, b, sa, sb)
    y = oracle_mod.w8a8_gemm(b, a, sb, sa)
    np.testing.assert_array_equal(x, y.T)


def test_w8a8_largest_k_fits_int32_and_2_pow_17_is_rejected(oracle_mod):
    """|sum| <= k * 128 * 128, so k < 2^17 keeps every int32 sum exact: at the
    largest accepted multiple of 16, all codes -128 give 2^31 - 2^18 (exact in
    binary32); at k = 2^17 that sum would be 2^31, one past INT32_MAX."""
    k = (1 << 17) - 16
    a = np.full((1, k), -128, dtype=np.int8)
    out = oracle_mod.w8a8_gemm(a, a, np.ones(1, np.float32), np.ones(1, np.float32), out_dtype="f32")
    assert out[0, 0] == float(k * 128 * 128) == 2.0 ** 31 - 2.0 ** 18
    big = np.full((1, 1 << 17), -128, dtype=np.int8)
    with pytest.raises(Exception):
        oracle_mod.w8a8_gemm(big, big, np.ones(1, np.float32), np.ones(1, np.float32), out_dtype="f32")


def test_w8a8_scale_product_is_taken_first(oracle_mod):
    """The formula multiplies the sum by (scale1 * scale2): rounded products in
    that order. Cases where (acc * s1) * s2 would round differently pin it."""
    rng = np.random.default_rng(24)
    found = 0
    for _ in range(200):
        a = _int8(rng, (1, 64))
        b = _int8(rng, (1, 64))
        s1 = np.float32(rng.uniform(0.001, 1))
        s2 = np.float32(rng.uniform(0.001, 1))
        acc = np.float32(int((a.astype(np.int64) @ b.astype(np.int64).T)[0, 0]))
        page = np.float32(acc * np.float32(s1 * s2))
        other = np.float32(np.float32(acc * s1) * s2)
        if page == other:
            continue
        found += 1
        got = oracle_mod.w8a8_gemm(a, b, np.array([s1]), np.array([s2]))[0, 0]
        assert got == page and got != other
    assert found >= 10


def test_w8a8_accumulate_and_narrow(oracle_mod):
    rng = np.random.default_rng(25)
    a, b = _int8(rng, (8, 128)), _int8(rng, (8, 128))
    sa, sb = rng.uniform(0.01, 0.1, 8).astype(np.float32), rng.uniform(0.01, 0.1, 8).astype(np.float32)
    base = oracle_mod.w8a8_gemm(a, b, sa, sb)  # |values| well inside the binary16 range
    y = rng.standard_normal((8, 8)).astype(np.float32)
    np.testing.assert_array_equal(oracle_mod.w8a8_gemm(a, b, sa, sb, accumulate_into=y), (base + y).astype(np.float32))
    np.testing.assert_array_equal(oracle_mod.w8a8_gemm(a, b, sa, sb, out_dtype="f16"), base.astype(np.float16))
    bf = oracle_mod.w8a8_gemm(a, b, sa, sb, out_dtype="bf16")
    np.testing.assert_array_equal(bf, torch.from_numpy(base).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


# ---------------------------------------------------------------- W8A8 golden records

def _load_w8a8_golden():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "quant_matmul_w8a8.txt")
    recs = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b, sa, sb, y, out_dtype, want = (f.strip() for f in line.split("|"))
        rows = lambda t, conv=float: [[conv(v) for v in r.split()] for r in t.split(";")]
        recs.append(dict(a=np.array(rows(a, int), np.int8), b=np.array(rows(b, int), np.int8),
                         sa=np.array(sa.split(), np.float32), sb=np.array(sb.split(), np.float32),
                         y=None if y == "-" else np.array(rows(y), np.float32), out_dtype=out_dtype,
                         want=np.array(rows(want), np.float64)))
    return recs


@pytest.mark.parametrize("rec", _load_w8a8_golden(), ids=lambda r: f"{r['a'].shape}x{r['b'].shape[0]}-{r['out_dtype']}")
def test_w8a8_golden_records(oracle_mod, rec):
    got = oracle_mod.w8a8_gemm(rec["a"], rec["b"], rec["sa"], rec["sb"], out_dtype=rec["out_dtype"],
                               accumulate_into=None if rec["y"] is None else rec["y"].copy())
    if rec["out_dtype"] == "f16":
        got = got.view(np.float16).astype(np.float64)
    else:
        got = _as_float64(got, rec["out_dtype"])
    np.testing.assert_array_equal(got, rec["want"])
