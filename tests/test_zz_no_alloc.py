"""dq_ada_layernorm_quant_noalloc against dq_ada_layernorm_quant (GPU).

The no-allocation entry point keeps the AdaLayerNorm affine table in the
library's fixed device array instead of a caller workspace; it runs the same
kernels, so its codes and scales must equal the regular entry point's. Two
calls in a row with different shapes check that nothing from one call leaks
into the next. This file is collected last and must also pass on its own in a
fresh process (the first call does the per-device set-up).
"""

import pytest
import torch

from token_dynamic_quantization_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dq(dq_lib, cuda_device):
    return dq_lib


def _inputs(batch, seq, hidden, seed, smooth=True):
    dev = torch.device("cuda:0")
    t = {
        "x": workloads.normal((batch, seq, hidden), torch.bfloat16, seed),
        "ada_scale": workloads.normal((batch, hidden), torch.bfloat16, seed + 1, std=0.1),
        "ada_shift": workloads.normal((batch, hidden), torch.bfloat16, seed + 2, std=0.1),
        "weight": workloads.normal((hidden,), torch.bfloat16, seed + 3, mean=1.0, std=0.05),
        "bias": workloads.normal((hidden,), torch.bfloat16, seed + 4, std=0.05),
        "smooth": workloads.uniform((hidden,), torch.bfloat16, seed + 5, 0.5, 2.0) if smooth else None,
    }
    return {k: (v.to(dev) if v is not None else None) for k, v in t.items()}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _noalloc(dq, t, eps=1e-6):
    x = t["x"]
    batch, seq, hidden = x.shape
    out = torch.empty((batch, seq, hidden), dtype=torch.int8, device=x.device)
    qs = torch.empty((batch, seq), dtype=torch.float32, device=x.device)
    stream = torch.cuda.current_stream().cuda_stream
    st = dq.dq_ada_layernorm_quant_noalloc(_ptr(x), dq.DQ_BF16, batch, seq, hidden, _ptr(t["ada_scale"]),
                                           _ptr(t["ada_shift"]), _ptr(t["weight"]), _ptr(t["bias"]),
                                           _ptr(t["smooth"]), dq.DQ_BF16, eps, _ptr(out), _ptr(qs), stream)
    return st, out, qs


def _regular(dq, t, eps=1e-6):
    return dq.ada_layernorm_quant(t["x"], t["ada_scale"], t["ada_shift"], t["weight"], t["bias"], t["smooth"],
                                  epsilon=eps)


def _assert_same(dq, t):
    st, out, qs = _noalloc(dq, t)
    assert st == dq.DQ_OK, dq.dq_status_string(st)
    ref_out, ref_qs = _regular(dq, t)
    torch.cuda.synchronize()
    # same kernels and table arithmetic: the tolerance of the fused path is not
    # needed, the results are identical
    assert torch.equal(qs.view(torch.int32), ref_qs.view(torch.int32))
    assert torch.equal(out, ref_out)


def test_two_calls_in_a_row_match_the_workspace_entry_point(dq):
    first = _inputs(4, 257, 3072, 10)               # vector path, several rows per CTA
    second = _inputs(3, 129, 1000, 20, smooth=False)  # hidden % 8 != 0: generic path, smaller table
    _assert_same(dq, first)
    _assert_same(dq, second)
    _assert_same(dq, first)


def test_largest_table_is_accepted_and_larger_is_rejected(dq):
    limit = dq.DQ_ADA_NOALLOC_MAX_TABLE
    t = _inputs(limit // 4096, 2, 4096, 30)         # batch * hidden == the limit
    _assert_same(dq, t)
    x = t["x"]
    out = torch.empty((33, 1, 4096), dtype=torch.int8, device=x.device)
    qs = torch.empty((33, 1), dtype=torch.float32, device=x.device)
    # 33 * 4096 > limit: rejected on the host before anything is launched (the
    # pointers are valid but too small for the shape; nothing reads them)
    st = dq.dq_ada_layernorm_quant_noalloc(_ptr(x), dq.DQ_BF16, 33, 1, 4096, _ptr(t["ada_scale"]),
                                           _ptr(t["ada_shift"]), None, None, None, dq.DQ_BF16, 1e-6, _ptr(out),
                                           _ptr(qs), torch.cuda.current_stream().cuda_stream)
    assert st == dq.DQ_ERR_UNSUPPORTED
    empty = dq.dq_ada_layernorm_quant_noalloc(None, dq.DQ_BF16, 0, 5, 4096, None, None, None, None, None,
                                              dq.DQ_BF16, 1e-6, None, None, None)
    assert empty == dq.DQ_OK
