"""GPU parity: the CUDA kernels (through the C ABI) against the CPU oracle.

DynamicQuant (aclnnDynamicQuantV2, Formula): codes, scales and offsets must be
bit-identical to the oracle. AdaLayerNormQuant (aclnnAdaLayerNormQuant,
Formula): quant_scale within relative 1e-5 and codes within +-1 on at most
0.01 % of the elements, because the row statistics are reduced in another
order and x - E(x) is scaled by 1/sqrt(Var+eps) rather than divided.
"""

import numpy as np
import pytest
import torch

import oracle
from token_dynamic_quantization_b200 import workloads

pytestmark = pytest.mark.gpu

ADA_SCALE_RTOL = 1e-5
ADA_CODE_FRACTION = 1e-4  # 0.01 %


@pytest.fixture(scope="module")
def dq(dq_lib, cuda_device):
    return dq_lib


def _bits(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint32) if a.dtype in (np.float32, np.int32, np.uint32) else a.view(np.uint8)


def run_gpu(dq, x, smooth=None, group_index=None, mode="symmetric", y_dtype="int8", misalign_x=False,
            misalign_y=False, stream=None):
    dev = torch.device("cuda:0")
    if misalign_x:
        flat = torch.empty(x.numel() + 1, dtype=x.dtype, device=dev)
        xg = flat[1:].view(x.shape)
        xg.copy_(x)
    else:
        xg = x.to(dev)
    sg = smooth.to(dev) if smooth is not None else None
    gg = group_index.to(dev) if group_index is not None else None
    out = None
    if misalign_y:
        rows, cols = x.shape
        assert y_dtype == "int8"
        ybuf = torch.empty(rows * cols + 1, dtype=torch.int8, device=dev)
        y = ybuf[1:].view(rows, cols)
        scale = torch.empty(rows, dtype=torch.float32, device=dev)
        off = torch.empty(rows, dtype=torch.float32, device=dev) if mode == "asymmetric" else None
        ws = torch.zeros(1, dtype=torch.int32, device=dev) if group_index is not None else None
        out = (y, scale, off, ws)
    y, s, o, ws = dq.dynamic_quant(xg, sg, gg, mode=mode, y_dtype=y_dtype, out=out, stream=stream)
    torch.cuda.synchronize()
    return (y.cpu().numpy(), s.cpu().numpy(), None if o is None else o.cpu().numpy(),
            None if ws is None else int(ws[0].item()))


def assert_dq_equal(got, want, y_dtype):
    gy, gs, go = got[:3]
    wy, ws_, wo = want
    np.testing.assert_array_equal(_bits(gy).reshape(-1), _bits(wy).reshape(-1))
    np.testing.assert_array_equal(_bits(gs), _bits(ws_))
    if wo is not None:
        np.testing.assert_array_equal(_bits(go), _bits(wo))


def rows_mix(rows, cols, dtype, seed):
    """Rows with varied magnitude, offset and a few special rows."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g)
    x = x * torch.exp(torch.randn(rows, 1, generator=g) * 2) + torch.randn(rows, 1, generator=g) * 3
    if rows > 3:
        x[1] = 0.0                     # all-zero row
        x[2] = 1.5                     # constant row
        x[3, :] = x[3, :] * 5.0 + 1000.0    # large offset, small range (asymmetric guard)
    if rows > 5:
        x[5] *= 1e-4                   # small values
    return x.to(dtype)


SHAPES = [(1, 8), (3, 16), (5, 24), (37, 1000), (64, 1024), (130, 4096), (17, 7168), (5, 8192), (9, 16384),
          (11, 3072), (7, 1792), (6, 3584), (4, 5376),
          (3, 16392), (2, 32768), (7, 40), (6, 2), (11, 520), (300, 64)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"{r}x{c}" for r, c in SHAPES])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["f16", "bf16"])
@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
def test_dynamic_quant_shapes(dq, shape, dtype, mode):
    rows, cols = shape
    x = rows_mix(rows, cols, dtype, seed=rows * 7919 + cols)
    for y_dtype in ("int8", "int4", "int32"):
        if (y_dtype == "int4" and cols % 2) or (y_dtype == "int32" and cols % 8):
            continue
        want = oracle.dynamic_quant(x, mode=mode, y_dtype=y_dtype)
        got = run_gpu(dq, x, mode=mode, y_dtype=y_dtype)
        assert_dq_equal(got, want, y_dtype)


@pytest.mark.parametrize("shape", [(9, 1), (4, 3), (33, 1001), (5, 4097), (3, 20001)])
@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
def test_dynamic_quant_ragged_cols(dq, shape, mode):
    rows, cols = shape
    x = rows_mix(rows, cols, torch.bfloat16, seed=cols)
    want = oracle.dynamic_quant(x, mode=mode)
    assert_dq_equal(run_gpu(dq, x, mode=mode), want, "int8")


@pytest.mark.parametrize("smooth_dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
@pytest.mark.parametrize("cols", [64, 4096, 1001])
def test_dynamic_quant_smooth(dq, smooth_dtype, mode, cols):
    rows = 70
    x = rows_mix(rows, cols, torch.bfloat16, seed=3)
    g = torch.Generator().manual_seed(4)
    smooth = (torch.rand(cols, generator=g) * 1.5 + 0.5).to(smooth_dtype)
    want = oracle.dynamic_quant(x, smooth=smooth, mode=mode)
    assert_dq_equal(run_gpu(dq, x, smooth=smooth, mode=mode), want, "int8")


# Row counts around the dispatch limits: the one-warp-per-row kernel serves at
# most 2 rows per SM of one-warp rows (296 on 148 SMs); beyond that the ring
# kernel runs with one CTA per SM, and its ring of at most 32 row slots is
# reused when a CTA owns more rows than slots (5920 rows: 40 per CTA).
RING_SHAPES = [(296, 1024), (297, 1024), (5920, 1024), (4500, 4096), (1200, 7168), (601, 16384)]


@pytest.mark.parametrize("shape", RING_SHAPES, ids=[f"{r}x{c}" for r, c in RING_SHAPES])
@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
@pytest.mark.parametrize("smooth_dtype", [None, torch.float32, torch.bfloat16], ids=["plain", "f32", "bf16"])
def test_ring_slot_reuse_and_dispatch_limits(dq, shape, mode, smooth_dtype):
    rows, cols = shape
    x = rows_mix(rows, cols, torch.bfloat16, seed=rows + 3 * cols)
    sm = None
    if smooth_dtype is not None:
        sm = (torch.rand(cols, generator=torch.Generator().manual_seed(cols)) * 1.5 + 0.5).to(smooth_dtype)
    for y_dtype in ("int8", "int4"):
        want = oracle.dynamic_quant(x, smooth=sm, mode=mode, y_dtype=y_dtype)
        got = run_gpu(dq, x, smooth=sm, mode=mode, y_dtype=y_dtype)
        assert_dq_equal(got, want, y_dtype)


def test_ring_repeated_calls_stay_exact(dq):
    """Many calls of a shape whose rows cycle through every ring slot many
    times, with fewer row groups than slots and slots not a multiple of the
    groups (16384 rows of 8192 fp16 values, asymmetric INT4: 110 rows per CTA,
    14 slots, 4 groups). A group reaching a slot's next fill round before that
    round was issued must wait for it; every call is checked for NaN scales
    (a wait that ran out) and on sampled rows against the oracle."""
    rows, cols = 16384, 8192
    x = workloads.normal((rows, cols), torch.float16, 71, mean=0.5, std=2.0)
    xg = x.cuda()
    pick = torch.randperm(rows, generator=torch.Generator().manual_seed(72))[:48].sort().values
    want = oracle.dynamic_quant(x[pick], mode="asymmetric", y_dtype="int4")
    out = None
    for call in range(40):
        out = dq.dynamic_quant(xg, mode="asymmetric", y_dtype="int4", out=out)
        if call % 8 == 7:
            torch.cuda.synchronize()
            y, s, o = (t.cpu().numpy() for t in out[:3])
            assert not np.isnan(s).any(), f"call {call}: a row's wait ran out"
            assert_dq_equal((y[pick.numpy()], s[pick.numpy()], o[pick.numpy()]), want, "int4")


@pytest.mark.parametrize("rows,cols,experts", [(5920, 1024, 16), (3000, 4096, 64), (296, 1024, 8)])
def test_ring_moe_many_rows_per_cta(dq, rows, cols, experts):
    g = torch.Generator().manual_seed(rows)
    x = rows_mix(rows, cols, torch.bfloat16, seed=rows + cols)
    sm = torch.rand(experts, cols, generator=g) * 1.5 + 0.5
    counts = torch.bincount(torch.randint(0, experts, (rows,), generator=g), minlength=experts)
    gi = torch.cumsum(counts, 0).to(torch.int32)
    want = oracle.dynamic_quant(x, smooth=sm, group_index=gi.numpy())
    got = run_gpu(dq, x, smooth=sm, group_index=gi)
    assert_dq_equal(got, want, "int8")
    assert got[3] == 0


def _mixed_expert_sizes(rows, seed):
    """Cumulative group index whose experts alternate between runs of large
    experts and runs of tiny or empty ones, ending before the last row: on
    148 CTAs some CTAs' rows belong to one expert, some to two (the ring
    kernel stages those experts' smooth rows) and some to three or more (the
    rest are read through L1), and the last CTA has rows past the last group."""
    g = torch.Generator().manual_seed(seed)
    sizes = []
    while sum(sizes) < rows - 120:
        if torch.rand(1, generator=g).item() < 0.5:
            sizes.append(int(torch.randint(150, 400, (1,), generator=g)))
        else:
            sizes += [int(v) for v in torch.randint(0, 3, (int(torch.randint(3, 9, (1,), generator=g)),), generator=g)]
    end = rows - 60  # rows past the last group
    gi, acc = [], 0
    for sz in sizes:
        acc = min(acc + sz, end)
        gi.append(acc)
    return np.asarray(gi, dtype=np.int32)


@pytest.mark.parametrize("smooth_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
def test_moe_staged_and_unstaged_expert_rows(dq, smooth_dtype, mode):
    rows, cols = 12000, 2048
    gi = _mixed_expert_sizes(rows, 17)
    experts = len(gi)
    x, smooth, gi_t = _moe_inputs(rows, cols, experts, 18, gi)
    smooth = smooth.to(smooth_dtype)
    want = oracle.dynamic_quant(x[: gi[-1]], smooth=smooth, group_index=gi, mode=mode)
    got = run_gpu(dq, x, smooth=smooth, group_index=gi_t, mode=mode)
    end = int(gi[-1])
    np.testing.assert_array_equal(got[0][:end], want[0])
    np.testing.assert_array_equal(_bits(got[1][:end]), _bits(want[1]))
    if mode == "asymmetric":
        np.testing.assert_array_equal(_bits(got[2][:end]), _bits(want[2]))
    assert np.all(got[1][end:] == 0)
    assert got[3] == dq.DQ_WS_ROWS_PAST_LAST_GROUP


@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
@pytest.mark.parametrize("y_dtype", ["int8", "int4"])
def test_misaligned_pointers_take_the_scalar_path(dq, mode, y_dtype):
    x = rows_mix(40, 512, torch.float16, seed=9)
    want = oracle.dynamic_quant(x, mode=mode, y_dtype=y_dtype)
    assert_dq_equal(run_gpu(dq, x, mode=mode, y_dtype=y_dtype, misalign_x=True), want, y_dtype)
    if y_dtype == "int8":
        assert_dq_equal(run_gpu(dq, x, mode=mode, y_dtype=y_dtype, misalign_y=True), want, y_dtype)


def _moe_inputs(rows, cols, experts, seed, gi=None):
    g = torch.Generator().manual_seed(seed)
    x = rows_mix(rows, cols, torch.bfloat16, seed)
    smooth = torch.rand(experts, cols, generator=g) * 1.5 + 0.5
    if gi is None:
        gi = workloads.moe_group_index(rows, experts, seed)
    return x, smooth, torch.as_tensor(gi, dtype=torch.int32)


@pytest.mark.parametrize("cols", [264, 4096, 1000, 77])
@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
def test_moe_group_index(dq, cols, mode):
    rows, experts = 300, 9
    gi = [0, 40, 40, 100, 180, 180, 181, 260, 300]  # empty experts 0, 2, 5
    x, smooth, gi = _moe_inputs(rows, cols, experts, 5, gi)
    want = oracle.dynamic_quant(x, smooth=smooth, group_index=gi.numpy(), mode=mode)
    got = run_gpu(dq, x, smooth=smooth, group_index=gi, mode=mode)
    assert_dq_equal(got, want, "int8")
    assert got[3] == 0  # status word: nothing to report


def test_moe_rows_past_last_group(dq):
    rows, cols, experts = 64, 128, 4
    x, smooth, gi = _moe_inputs(rows, cols, experts, 6, [10, 20, 20, 50])
    got = run_gpu(dq, x, smooth=smooth, group_index=gi)
    want = oracle.dynamic_quant(x[:50], smooth=smooth, group_index=gi.numpy())
    np.testing.assert_array_equal(got[0][:50], want[0])
    np.testing.assert_array_equal(_bits(got[1][:50]), _bits(want[1]))
    assert np.all(got[0][50:] == 0) and np.all(got[1][50:] == 0)
    assert got[3] == dq.DQ_WS_ROWS_PAST_LAST_GROUP


def test_moe_decreasing_group_index_is_flagged(dq):
    x, smooth, gi = _moe_inputs(32, 64, 3, 7, [20, 10, 32])
    got = run_gpu(dq, x, smooth=smooth, group_index=gi)
    assert got[3] & dq.DQ_WS_GROUP_INDEX_INVALID


def test_moe_single_expert_equals_dense(dq):
    x, smooth, gi = _moe_inputs(50, 256, 1, 8, [50])
    a = run_gpu(dq, x, smooth=smooth, group_index=gi)
    b = run_gpu(dq, x, smooth=smooth[0])
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(_bits(a[1]), _bits(b[1]))


def _tie_rows(mode):
    """Rows whose elements sit on or next to rounding ties of the quantizer."""
    rng = np.random.default_rng(77)
    rows = []
    if mode == "symmetric":
        # amax 127: scale 1, so k + 0.5 are exact ties
        r = np.concatenate([[127.0], np.arange(-126.5, 127.0, 1.0)])
        rows.append(r[:256])
        amax = 3.0
        s = np.float32(np.float32(amax) / np.float32(127))
        base = (np.arange(-126, 127) + 0.5) * np.float64(s)
        cand = np.concatenate([np.nextafter(base.astype(np.float32), np.float32(d)) for d in (-np.inf, np.inf)]
                              + [base.astype(np.float32)])
        rows.append(np.concatenate([[amax], cand[:255]]))
    else:
        r = np.concatenate([[0.0, 255.0], np.arange(0.5, 254.0, 1.0)])
        rows.append(r[:256])
        rows.append(np.concatenate([[0.0, 3.0], rng.uniform(0, 3, 254)]))
    return torch.tensor(np.array([np.resize(r, 256) for r in rows]), dtype=torch.float32)


@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
def test_rounding_ties(dq, mode):
    # fp16 holds k + 0.5 exactly for |k| < 1024; near-tie neighbours are rounded to fp16
    x = _tie_rows(mode).to(torch.float16)
    want = oracle.dynamic_quant(x, mode=mode)
    assert_dq_equal(run_gpu(dq, x, mode=mode), want, "int8")


def _preimages(halves, scale, shift, steps=2):
    """fp32 values v with v/scale + shift within a few ulps of each half-integer."""
    out = []
    for h in halves:
        v = np.float32((h - shift) * np.float64(scale))
        for _ in range(steps):
            v = np.nextafter(v, np.float32(-np.inf), dtype=np.float32)
        for _ in range(2 * steps + 1):
            out.append(v)
            v = np.nextafter(v, np.float32(np.inf), dtype=np.float32)
    return np.array(out, np.float32)


@pytest.mark.parametrize("mode", ["symmetric", "asymmetric"])
def test_near_tie_inputs_via_fp32_smooth(dq, mode):
    """x = 1 makes input = x * smooth equal the fp32 smooth value, which is placed
    a few ulps from every rounding tie of the quantizer: the reciprocal fast
    path must hand all of these to the exact division."""
    amax = np.float32(3.0)
    if mode == "symmetric":
        s = np.float32(amax / np.float32(127.0))
        vals = _preimages(np.arange(-126, 127) + 0.5, s, 0.0)
        vals = vals[np.abs(vals) <= amax]
        row = np.concatenate([[amax], vals])
    else:
        s = np.float32(amax / np.float32(255.0))
        off = np.float32(np.float32(127.0) - np.float32(amax / s))
        vals = _preimages(np.arange(-128, 127) + 0.5, s, float(off))
        vals = vals[(vals >= 0) & (vals <= amax)]
        row = np.concatenate([[0.0, amax], vals])
    cols = (len(row) + 7) // 8 * 8
    smooth = torch.from_numpy(np.resize(row, cols).astype(np.float32))
    x = torch.ones(3, cols, dtype=torch.bfloat16)
    x[1] = -1.0
    want = oracle.dynamic_quant(x, smooth=smooth, mode=mode)
    assert_dq_equal(run_gpu(dq, x, smooth=smooth, mode=mode), want, "int8")


def test_asymmetric_huge_offset_rows(dq):
    """Rows whose range is tiny next to their max give |offset| > 2^20; the guard
    band would exceed 1/4 and the whole row takes the exact path."""
    cols = 256
    x = torch.full((4, cols), 1000.0, dtype=torch.float16)
    x[1] = -1000.0
    x[2] = 7.0
    k = torch.arange(cols, dtype=torch.float64) % 4
    smooth = (1.0 + k * 2.0 ** -23).to(torch.float32)
    for y_dtype in ("int8", "int4"):
        want = oracle.dynamic_quant(x, smooth=smooth, mode="asymmetric", y_dtype=y_dtype)
        assert np.abs(want[2]).max() > 2 ** 20
        assert_dq_equal(run_gpu(dq, x, smooth=smooth, mode="asymmetric", y_dtype=y_dtype), want, y_dtype)


def test_determinism_and_streams(dq):
    x = rows_mix(257, 4096, torch.bfloat16, seed=13)
    smooth = torch.rand(4096) + 0.5
    a = run_gpu(dq, x, smooth=smooth)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = run_gpu(dq, x, smooth=smooth, stream=s.cuda_stream)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(_bits(a[1]), _bits(b[1]))


def test_outputs_stay_in_bounds(dq):
    """Canary bytes right after y, scale and offset are left untouched."""
    dev = torch.device("cuda:0")
    rows, cols = 77, 1032
    x = rows_mix(rows, cols, torch.float16, seed=14).to(dev)
    for mode, y_dtype in (("symmetric", "int8"), ("asymmetric", "int4")):
        ycols = cols if y_dtype == "int8" else cols // 2
        ydt = torch.int8 if y_dtype == "int8" else torch.uint8
        ybuf = torch.full((rows * ycols + 64,), 0x5A, dtype=ydt, device=dev)
        sbuf = torch.full((rows + 16,), -7.0, device=dev)
        obuf = torch.full((rows + 16,), -9.0, device=dev)
        out = (ybuf[: rows * ycols].view(rows, ycols), sbuf[:rows], obuf[:rows] if mode == "asymmetric" else None,
               None)
        dq.dynamic_quant(x, mode=mode, y_dtype=y_dtype, out=out)
        torch.cuda.synchronize()
        assert torch.all(ybuf[rows * ycols:] == 0x5A)
        assert torch.all(sbuf[rows:] == -7.0)
        assert torch.all(obuf[rows:] == -9.0)
        if mode == "symmetric":
            assert torch.all(obuf == -9.0)


def test_empty_input_is_a_noop(dq):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda:0")
    y, s, o, _ = dq.dynamic_quant(x)
    torch.cuda.synchronize()
    assert y.shape == (0, 64) and s.shape == (0,)


# ---------------------------------------------------------------- full-size workloads

DQ_WORKLOADS = [w for w in workloads.WORKLOADS if not w.startswith(("ada_", "dequant", "w8a8"))]


@pytest.mark.slow
@pytest.mark.parametrize("name", DQ_WORKLOADS)
def test_workload_parity_full_size(dq, name):
    wl = workloads.make(name)
    t = wl.tensors
    gi = t.get("group_index")
    want = oracle.dynamic_quant(t["x"], smooth=t.get("smooth"), group_index=None if gi is None else gi.numpy(),
                                mode=wl.mode, y_dtype=wl.y_dtype)
    got = run_gpu(dq, t["x"], smooth=t.get("smooth"), group_index=gi, mode=wl.mode, y_dtype=wl.y_dtype)
    assert_dq_equal(got, want, wl.y_dtype)
    if gi is not None:
        assert got[3] == 0


# ---------------------------------------------------------------- AdaLayerNormQuant

def assert_ada_close(got, want):
    go, gs = got
    wo, ws = want
    gs = gs.reshape(-1).astype(np.float64)
    ws = ws.reshape(-1).astype(np.float64)
    rel = np.abs(gs - ws) / np.maximum(np.abs(ws), 1e-30)
    assert rel.max() <= ADA_SCALE_RTOL, rel.max()
    diff = go.astype(np.int16) - wo.astype(np.int16)
    assert np.abs(diff).max() <= 1
    frac = np.count_nonzero(diff) / diff.size
    assert frac <= ADA_CODE_FRACTION, frac
    return rel.max(), frac


def run_ada_gpu(dq, x, sc, sh, w, b, sm, eps, misalign=False):
    dev = torch.device("cuda:0")
    if misalign:
        flat = torch.empty(x.numel() + 1, dtype=x.dtype, device=dev)
        xg = flat[1:].view(x.shape)
        xg.copy_(x)
    else:
        xg = x.to(dev)
    c = lambda t: None if t is None else t.to(dev)
    o, q = dq.ada_layernorm_quant(xg, c(sc), c(sh), c(w), c(b), c(sm), epsilon=eps)
    torch.cuda.synchronize()
    return o.cpu().numpy(), q.cpu().numpy()


def _ada_inputs(b, s, h, dtype, pdtype, seed, x_mean=0.0, x_std=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(b, s, h, generator=g) * x_std + x_mean).to(dtype)
    sc = (torch.randn(b, h, generator=g) * 0.1).to(pdtype)
    sh = (torch.randn(b, h, generator=g) * 0.1).to(pdtype)
    w = (1 + torch.randn(h, generator=g) * 0.05).to(pdtype)
    bias = (torch.randn(h, generator=g) * 0.05).to(pdtype)
    sm = (torch.rand(h, generator=g) * 1.5 + 0.5).to(pdtype)
    return x, sc, sh, w, bias, sm


ADA_SHAPES = [(1, 1, 8), (2, 3, 64), (1, 3, 256), (1, 3, 512), (2, 7, 1024), (3, 11, 2048), (3, 17, 1000),
              (2, 9, 3072), (1, 5, 4096), (2, 3, 4104), (1, 2, 8192), (2, 3, 77)]


@pytest.mark.parametrize("shape", ADA_SHAPES, ids=[f"{b}x{s}x{h}" for b, s, h in ADA_SHAPES])
@pytest.mark.parametrize("dtype,pdtype", [(torch.bfloat16, torch.bfloat16), (torch.float16, torch.float32),
                                          (torch.bfloat16, torch.float16)])
def test_ada_layernorm_quant_shapes(dq, shape, dtype, pdtype):
    b, s, h = shape
    x, sc, sh, w, bias, sm = _ada_inputs(b, s, h, dtype, pdtype, seed=h + s)
    want = oracle.ada_layernorm_quant(x, sc, sh, w, bias, sm, epsilon=1e-6)
    got = run_ada_gpu(dq, x, sc, sh, w, bias, sm, 1e-6)
    assert_ada_close(got, want)


# Many rows per CTA (ring slots reused), batch boundaries inside a CTA's rows,
# and many small batches per CTA (the staged table holds several batches).
ADA_RING_SHAPES = [(3, 1000, 1024), (64, 7, 1024), (2, 2500, 3072), (5, 1111, 2048), (300, 3, 256)]


@pytest.mark.parametrize("shape", ADA_RING_SHAPES, ids=[f"{b}x{s}x{h}" for b, s, h in ADA_RING_SHAPES])
def test_ada_ring_batches_across_ctas(dq, shape):
    b, s, h = shape
    x, sc, sh, w, bias, sm = _ada_inputs(b, s, h, torch.bfloat16, torch.bfloat16, seed=b * 31 + s + h)
    want = oracle.ada_layernorm_quant(x, sc, sh, w, bias, sm, epsilon=1e-6)
    got = run_ada_gpu(dq, x, sc, sh, w, bias, sm, 1e-6)
    assert_ada_close(got, want)


@pytest.mark.parametrize("opt", ["none", "weight", "bias", "smooth", "misaligned"])
def test_ada_optional_parameters(dq, opt):
    x, sc, sh, w, bias, sm = _ada_inputs(2, 33, 512, torch.bfloat16, torch.bfloat16, seed=21, x_mean=0.5,
                                         x_std=2.0)
    kw = dict(w=None, b=None, sm=None)
    if opt == "weight":
        kw["w"] = w
    elif opt == "bias":
        kw["b"] = bias
    elif opt in ("smooth", "misaligned"):
        kw["sm"] = sm
    want = oracle.ada_layernorm_quant(x, sc, sh, kw["w"], kw["b"], kw["sm"], epsilon=1e-5)
    got = run_ada_gpu(dq, x, sc, sh, kw["w"], kw["b"], kw["sm"], 1e-5, misalign=opt == "misaligned")
    assert_ada_close(got, want)


@pytest.mark.parametrize("h", [3072, 1000, 1024])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_ada_large_mean_rows(dq, h, dtype):
    """Rows with mean far above their spread (1000 +- 3): E(x) must be accurate
    to well below the spread, or most codes move."""
    x, sc, sh, w, bias, sm = _ada_inputs(3, 13, h, dtype, torch.bfloat16, seed=h + 5, x_mean=1000.0, x_std=3.0)
    want = oracle.ada_layernorm_quant(x, sc, sh, w, bias, sm, epsilon=1e-6)
    got = run_ada_gpu(dq, x, sc, sh, w, bias, sm, 1e-6)
    assert_ada_close(got, want)


@pytest.mark.parametrize("h", [3072, 1000])
def test_ada_rows_with_outlying_first_elements(dq, h):
    """Rows whose first 8 elements sit far from the row mean: the one-reduction
    moments about those elements would cancel, so these rows take the centred
    second pass."""
    x, sc, sh, w, bias, sm = _ada_inputs(2, 9, h, torch.bfloat16, torch.bfloat16, seed=h + 9)
    x[:, ::2, :8] = 40.0
    x[:, 1::4, :8] = -25.0
    want = oracle.ada_layernorm_quant(x, sc, sh, w, bias, sm, epsilon=1e-6)
    got = run_ada_gpu(dq, x, sc, sh, w, bias, sm, 1e-6)
    assert_ada_close(got, want)


def test_ada_constant_rows_and_scale_minus_one(dq):
    x, sc, sh, w, bias, sm = _ada_inputs(2, 8, 256, torch.bfloat16, torch.bfloat16, seed=22)
    x[0, :4] = 0.75  # constant rows: variance 0
    sc[1] = -1.0     # y = shift * smooth exactly
    want = oracle.ada_layernorm_quant(x, sc, sh, w, bias, sm, epsilon=1e-6)
    got = run_ada_gpu(dq, x, sc, sh, w, bias, sm, 1e-6)
    assert_ada_close(got, want)
    np.testing.assert_array_equal(got[0][1], want[0][1])  # exact where no statistics enter


@pytest.mark.slow
def test_ada_workload_parity_full_size(dq):
    wl = workloads.make("ada_layernorm_quant_bf16_4x4096x3072")
    t = wl.tensors
    want = oracle.ada_layernorm_quant(t["x"], t["ada_scale"], t["ada_shift"], t["weight"], t["bias"], t["smooth"],
                                      epsilon=wl.epsilon)
    got = run_ada_gpu(dq, t["x"], t["ada_scale"], t["ada_shift"], t["weight"], t["bias"], t["smooth"], wl.epsilon)
    rel, frac = assert_ada_close(got, want)
    print(f"\nAdaLayerNormQuant full size: max quant_scale rel err {rel:.3g}, code mismatch fraction {frac:.3g}")


@pytest.mark.parametrize("pdtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("which", [0, 2])
def test_ada_misaligned_parameters_fold_the_same_table(dq, pdtype, which):
    """The ring kernel folds its affine table from 16-byte parameter loads when
    every parameter is 16-byte aligned, one column at a time otherwise: the
    same parameters one element past a 16-byte boundary give the same bits."""
    dev = torch.device("cuda:0")
    x, sc, sh, w, bias, sm = _ada_inputs(2, 300, 3072, torch.bfloat16, pdtype, seed=77 + which)
    aligned = run_ada_gpu(dq, x, sc, sh, w, bias, sm, 1e-6)
    params = [t.to(dev) for t in (sc, sh, w, bias, sm)]
    buf = torch.empty(params[which].numel() + 1, dtype=pdtype, device=dev)
    shifted = buf[1:].view(params[which].shape)
    shifted.copy_(params[which])
    assert shifted.data_ptr() % 16 != 0
    params[which] = shifted
    got = run_ada_gpu(dq, x, *params, 1e-6)
    np.testing.assert_array_equal(got[0], aligned[0])
    np.testing.assert_array_equal(got[1].view(np.uint32), aligned[1].view(np.uint32))
    assert_ada_close(got, oracle.ada_layernorm_quant(x, sc, sh, w, bias, sm, epsilon=1e-6))
