"""The kernels' bounded waits, made to run out on purpose (GPU).

Every wait in the quantizers' and the W8A8 product's pipelines gives up after
a time limit, so that a copy that never completes ends the kernel with an
error mark (NaN scales or a NaN tile) instead of hanging the GPU. These tests
run that path without any fault: they load a test build of the same sources
(libdq_waittest.so, built by token_dynamic_quantization_b200.build with a
2 ms limit) in which the producer leaves out exactly one copy:

* the quantizers' ring kernels skip the row copy of global row 777, so the
  consumer of that row times out: its group marks its remaining rows with NaN
  scales and raises the CTA's abort flag, the other groups of that CTA stop at
  their next row that has not landed, and every other CTA is untouched;
* the W8A8 product skips the operand stage of k-tile 2 of the tile in tile
  row 1, column 0: the MMA lane times out and raises the CTA's abort flag,
  and the epilogue writes that 128-row tile as NaN while every other tile
  (the only tile of its CTA at this size) is exact.

Each test checks that the skipped row or tile is marked, that every other
output is either marked (only inside the CTA that owned the skipped row) or
equal to the oracle's, and that the next call on the same context, which
does not reach the skipped row or tile, is exact again. Nothing faults, traps
or waits forever; the product library has none of the test flags.
"""

import ctypes

import numpy as np
import pytest
import torch

from token_dynamic_quantization_b200 import build as dq_build
from token_dynamic_quantization_b200 import workloads

pytestmark = pytest.mark.gpu

SKIP_ROW = 777
SKIP_TILE_M, SKIP_KTILE = 1, 2


@pytest.fixture(scope="module")
def waitlib(cuda_device):
    path = dq_build.build_wait_test()
    lib = ctypes.CDLL(path)
    vp, i64, i32, ci, sz, f32 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int, ctypes.c_size_t,
                                 ctypes.c_float)
    lib.dq_dynamic_quant.argtypes = [vp, ci, i64, i64, vp, ci, vp, i32, ci, ci, vp, vp, vp, vp, sz, vp]
    lib.dq_dynamic_quant.restype = ci
    lib.dq_ada_layernorm_quant.argtypes = [vp, ci, i64, i64, i64, vp, vp, vp, vp, vp, ci, f32, vp, vp, vp, sz, vp]
    lib.dq_ada_layernorm_quant.restype = ci
    lib.dq_w8a8_gemm.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, ci, i32, vp]
    lib.dq_w8a8_gemm.restype = ci
    return lib


def _p(t):
    return None if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _cta_rows(rows, row):
    """Rows of the ring kernel's CTA that owns `row` (one CTA per SM, fewer
    for few rows; CTA b owns [b * rows / grid, (b + 1) * rows / grid))."""
    grid = min(rows, torch.cuda.get_device_properties(0).multi_processor_count)
    for b in range(grid):
        lo, hi = b * rows // grid, (b + 1) * rows // grid
        if lo <= row < hi:
            return lo, hi
    raise AssertionError("row outside the grid")


def _quantize(lib, x, smooth):
    rows, cols = x.shape
    y = torch.empty((rows, cols), dtype=torch.int8, device=x.device)
    scale = torch.empty(rows, dtype=torch.float32, device=x.device)
    st = lib.dq_dynamic_quant(_p(x), 2, rows, cols, _p(smooth), 0, None, 0, 0, 3, _p(y), _p(scale), None, None, 0,
                              _stream())
    torch.cuda.synchronize()
    return st, y.cpu().numpy(), scale.cpu().numpy()


def test_dynamic_quant_row_copy_timeout(waitlib, oracle_mod):
    rows, cols = 2048, 4096  # bf16 with fp32 smooth scales: the ring kernel
    x = workloads.normal((rows, cols), torch.bfloat16, 41)
    smooth = workloads.uniform((cols,), torch.float32, 42, 0.5, 2.0)
    st, y, scale = _quantize(waitlib, x.cuda(), smooth.cuda())
    assert st == 0
    want_y, want_s, _ = oracle_mod.dynamic_quant(x, smooth=smooth)
    marked = np.isnan(scale)
    assert marked[SKIP_ROW], "the row whose copy was left out must carry a NaN scale"
    lo, hi = _cta_rows(rows, SKIP_ROW)
    assert not marked[:lo].any() and not marked[hi:].any(), "only the failing CTA may mark rows"
    ok = ~marked
    assert np.array_equal(scale[ok].view(np.uint32), want_s[ok].view(np.uint32))
    assert np.array_equal(y[ok], want_y[ok])
    # the same context, a call that does not reach row 777: exact again
    small = x[:512].contiguous()
    st, y2, s2 = _quantize(waitlib, small.cuda(), smooth.cuda())
    assert st == 0
    assert np.array_equal(s2.view(np.uint32), want_s[:512].view(np.uint32))
    assert np.array_equal(y2, want_y[:512])


def _ada(lib, t, batch, seq, hidden):
    dev = torch.device("cuda:0")
    d = {k: (v.to(dev) if v is not None else None) for k, v in t.items()}
    out = torch.empty((batch, seq, hidden), dtype=torch.int8, device=dev)
    qs = torch.empty((batch, seq), dtype=torch.float32, device=dev)
    ws = torch.empty(batch * hidden * 2, dtype=torch.float32, device=dev)
    st = lib.dq_ada_layernorm_quant(_p(d["x"]), 2, batch, seq, hidden, _p(d["ada_scale"]), _p(d["ada_shift"]),
                                    _p(d["weight"]), _p(d["bias"]), _p(d["smooth"]), 2, 1e-6, _p(out), _p(qs), _p(ws),
                                    batch * hidden * 8, _stream())
    torch.cuda.synchronize()
    return st, out.cpu().numpy(), qs.cpu().numpy()


def _ada_inputs(batch, seq, hidden):
    return {
        "x": workloads.normal((batch, seq, hidden), torch.bfloat16, 51),
        "ada_scale": workloads.normal((batch, hidden), torch.bfloat16, 52, std=0.1),
        "ada_shift": workloads.normal((batch, hidden), torch.bfloat16, 53, std=0.1),
        "weight": workloads.normal((hidden,), torch.bfloat16, 54, mean=1.0, std=0.05),
        "bias": workloads.normal((hidden,), torch.bfloat16, 55, std=0.05),
        "smooth": workloads.uniform((hidden,), torch.bfloat16, 56, 0.5, 2.0),
    }


def _ada_close(out, qs, want_o, want_q):
    """The fused path's tolerance: quant_scale within 1e-5 relative, codes
    within 1 on at most 0.01 % of the elements."""
    assert np.all(np.abs(qs.astype(np.float64) - want_q) <= 1e-5 * np.abs(want_q))
    diff = np.abs(out.astype(np.int16) - want_o.astype(np.int16))
    assert diff.max(initial=0) <= 1 and np.count_nonzero(diff) <= max(1, diff.size // 10000)


def test_ada_layernorm_row_copy_timeout(waitlib, oracle_mod):
    batch, seq, hidden = 1, 2048, 3072
    t = _ada_inputs(batch, seq, hidden)
    st, out, qs = _ada(waitlib, t, batch, seq, hidden)
    assert st == 0
    want_o, want_q = oracle_mod.ada_layernorm_quant(t["x"], t["ada_scale"], t["ada_shift"], t["weight"], t["bias"],
                                                    t["smooth"], epsilon=1e-6)
    qs, out, want_q, want_o = qs[0], out[0], want_q[0], want_o[0]
    marked = np.isnan(qs)
    assert marked[SKIP_ROW]
    lo, hi = _cta_rows(seq, SKIP_ROW)
    assert not marked[:lo].any() and not marked[hi:].any()
    ok = ~marked
    _ada_close(out[ok], qs[ok], want_o[ok], want_q[ok])
    # a call that does not reach row 777
    t2 = {k: (v[:, :512].contiguous() if k == "x" else v) for k, v in t.items()}
    st, out2, qs2 = _ada(waitlib, t2, batch, 512, hidden)
    assert st == 0
    _ada_close(out2[0], qs2[0], want_o[:512], want_q[:512])


def _w8a8(lib, a, b, sa, sb):
    m, k = a.shape
    n = b.shape[0]
    out = torch.empty((m, n), dtype=torch.float32, device=a.device)
    st = lib.dq_w8a8_gemm(_p(a), _p(b), m, n, k, _p(sa), _p(sb), _p(out), 0, 0, _stream())
    torch.cuda.synchronize()
    return st, out.cpu().numpy()


def test_w8a8_stage_timeout(waitlib, oracle_mod):
    m, n, k = 512, 512, 1024  # 4 x 2 tiles of 128 x 256, 8 k-tiles: the tensor-core path
    a = workloads.uniform((m, k), torch.float32, 61, -127.0, 127.0).round().to(torch.int8)
    b = workloads.uniform((n, k), torch.float32, 62, -127.0, 127.0).round().to(torch.int8)
    sa = workloads.uniform((m,), torch.float32, 63, 0.001, 0.02)
    sb = workloads.uniform((n,), torch.float32, 64, 0.001, 0.02)
    st, out = _w8a8(waitlib, a.cuda(), b.cuda(), sa.cuda(), sb.cuda())
    assert st == 0
    want = oracle_mod.w8a8_gemm(a.numpy(), b.numpy(), sa.numpy(), sb.numpy(), out_dtype="f32")
    # the tile at tile row 1, column 0 is 128 wide (this shape has fewer tiles
    # than SMs, so the persistent schedule halves every tile) or 256 wide
    nan = np.isnan(out)
    width = 128 if not nan[128 * SKIP_TILE_M, 128] else 256
    tile = np.zeros((m, n), dtype=bool)
    tile[128 * SKIP_TILE_M:128 * (SKIP_TILE_M + 1), 0:width] = True
    assert nan[tile].all(), "the tile whose stage was left out must be NaN"
    assert not nan[~tile].any(), "no other tile may be marked"
    assert np.array_equal(out[~tile].view(np.uint32), want[~tile].view(np.uint32))
    # one tile row only (tile row 1 does not exist): exact again
    st, out2 = _w8a8(waitlib, a[:128].contiguous().cuda(), b.cuda(), sa[:128].contiguous().cuda(), sb.cuda())
    assert st == 0
    assert np.array_equal(out2.view(np.uint32), want[:128].view(np.uint32))
