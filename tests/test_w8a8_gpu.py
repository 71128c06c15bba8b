"""GPU parity of the W8A8 product with per-token x per-channel scales.

dq_w8a8_gemm through the C ABI against the CPU oracle, bit for bit: the
integer sum is exact on both sides, and the scale product, the multiply, the
optional accumulation and the narrowing are single binary32 roundings in the
same order. Shapes with K a multiple of 16 run on the tcgen05 tensor cores
(ragged M and N included); others on the CUDA-core kernel.
"""

import numpy as np
import pytest
import torch

import oracle
from token_dynamic_quantization_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dq(dq_lib, cuda_device):
    return dq_lib


def _case(m, n, k, seed):
    g = torch.Generator().manual_seed(seed)
    a = torch.randint(-128, 128, (m, k), generator=g, dtype=torch.int32).to(torch.int8)
    b = torch.randint(-128, 128, (n, k), generator=g, dtype=torch.int32).to(torch.int8)
    sa = (torch.rand(m, generator=g) * 0.02 + 1e-4).float()
    sb = (torch.rand(n, generator=g) * 0.02 + 1e-4).float()
    return a, b, sa, sb


def _run(dq, a, b, sa, sb, out_dtype=torch.float32, accumulate_into=None):
    dev = torch.device("cuda:0")
    out = None if accumulate_into is None else accumulate_into.to(dev)
    o = dq.w8a8_gemm(a.to(dev), b.to(dev), sa.to(dev), sb.to(dev), out_dtype=out_dtype, out=out,
                     accumulate=accumulate_into is not None)
    torch.cuda.synchronize()
    return o.cpu()


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype != torch.float32 else t.numpy().view(np.uint32)


TC_SHAPES = [(128, 128, 128), (256, 384, 512), (128, 256, 1024), (384, 128, 2048), (256, 768, 384), (128, 512, 4096)]


@pytest.mark.parametrize("shape", TC_SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in TC_SHAPES])
def test_tensor_core_path_matches_oracle(dq, shape):
    m, n, k = shape
    a, b, sa, sb = _case(m, n, k, seed=m + n + k)
    want = oracle.w8a8_gemm(a.numpy(), b.numpy(), sa.numpy(), sb.numpy())
    got = _run(dq, a, b, sa, sb)
    np.testing.assert_array_equal(got.numpy().view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("out_dtype,name", [(torch.bfloat16, "bf16"), (torch.float16, "f16")])
def test_tensor_core_narrow_outputs(dq, out_dtype, name):
    a, b, sa, sb = _case(256, 256, 256, seed=3)
    want = oracle.w8a8_gemm(a.numpy(), b.numpy(), sa.numpy(), sb.numpy(), out_dtype=name)
    got = _run(dq, a, b, sa, sb, out_dtype=out_dtype)
    np.testing.assert_array_equal(_bits(got), want.view(np.uint16))


def test_tensor_core_accumulate(dq):
    a, b, sa, sb = _case(128, 256, 384, seed=4)
    y = torch.randn(128, 256, generator=torch.Generator().manual_seed(5))
    want = oracle.w8a8_gemm(a.numpy(), b.numpy(), sa.numpy(), sb.numpy(), accumulate_into=y.numpy())
    got = _run(dq, a, b, sa, sb, accumulate_into=y)
    np.testing.assert_array_equal(got.numpy().view(np.uint32), want.view(np.uint32))


def test_extreme_codes_large_k(dq):
    """All codes -128: |sum| = 16384 k, beyond 2^24 at k = 2048 (the int32 ->
    float conversion rounds)."""
    m, n, k = 128, 128, 2048
    a = torch.full((m, k), -128, dtype=torch.int8)
    b = torch.full((n, k), -128, dtype=torch.int8)
    b[::2] = 127
    sa, sb = torch.ones(m), torch.ones(n) * 0.5
    want = oracle.w8a8_gemm(a.numpy(), b.numpy(), sa.numpy(), sb.numpy())
    got = _run(dq, a, b, sa, sb)
    np.testing.assert_array_equal(got.numpy().view(np.uint32), want.view(np.uint32))


RAGGED_TC_SHAPES = [(130, 128, 128), (128, 128, 96), (64, 200, 256), (1, 256, 16), (200, 300, 272),
                    (77, 520, 1040), (129, 385, 4112), (300, 640, 128), (5, 7, 48)]


@pytest.mark.parametrize("shape", RAGGED_TC_SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in RAGGED_TC_SHAPES])
@pytest.mark.parametrize("out_dtype,name", [(torch.float32, "f32"), (torch.bfloat16, "bf16")])
def test_ragged_tensor_core_path_matches_oracle(dq, shape, out_dtype, name):
    """m, n, k not multiples of the tile (k a multiple of 16): zero-filled
    loads and masked stores on the tensor-core path, bit for bit."""
    m, n, k = shape
    a, b, sa, sb = _case(m, n, k, seed=m + n + k)
    want = oracle.w8a8_gemm(a.numpy(), b.numpy(), sa.numpy(), sb.numpy(), out_dtype=name)
    got = _run(dq, a, b, sa, sb, out_dtype=out_dtype)
    np.testing.assert_array_equal(_bits(got), want.view(np.uint32 if name == "f32" else np.uint16))


def test_ragged_accumulate(dq):
    a, b, sa, sb = _case(150, 330, 208, seed=12)
    base = torch.randn(150, 330, generator=torch.Generator().manual_seed(13))
    want = oracle.w8a8_gemm(a.numpy(), b.numpy(), sa.numpy(), sb.numpy(), out_dtype="f32",
                            accumulate_into=base.numpy().copy())
    got = _run(dq, a, b, sa, sb, accumulate_into=base.clone())
    np.testing.assert_array_equal(_bits(got), want.view(np.uint32))


@pytest.mark.parametrize("shape", [(5, 7, 33), (3, 40, 40), (64, 130, 200)])
def test_cuda_core_path_matches_oracle(dq, shape):
    m, n, k = shape
    a, b, sa, sb = _case(m, n, k, seed=m * n + k)
    want = oracle.w8a8_gemm(a.numpy(), b.numpy(), sa.numpy(), sb.numpy())
    got = _run(dq, a, b, sa, sb)
    np.testing.assert_array_equal(got.numpy().view(np.uint32), want.view(np.uint32))


def test_quantize_then_multiply(dq):
    """The quantizer's codes and per-token scales feed the product directly."""
    g = torch.Generator().manual_seed(6)
    x = torch.randn(256, 512, generator=g).to(torch.bfloat16)
    w = torch.randint(-127, 128, (128, 512), generator=g, dtype=torch.int32).to(torch.int8)
    ws = torch.rand(128, generator=g) * 0.01 + 1e-3
    dev = torch.device("cuda:0")
    y, s, _, _ = dq.dynamic_quant(x.to(dev))
    got = dq.w8a8_gemm(y, w.to(dev), s, ws.to(dev), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    yo, so, _ = oracle.dynamic_quant(x)
    want = oracle.w8a8_gemm(yo, w.numpy(), so, ws.numpy(), out_dtype="bf16")
    np.testing.assert_array_equal(_bits(got.cpu()), want.view(np.uint16))


def test_empty_product(dq):
    dev = torch.device("cuda:0")
    a = torch.empty(0, 256, dtype=torch.int8, device=dev)
    b = torch.randint(-128, 128, (128, 256), dtype=torch.int32).to(torch.int8).to(dev)
    o = dq.w8a8_gemm(a, b, torch.empty(0, device=dev), torch.ones(128, device=dev), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert tuple(o.shape) == (0, 128)


@pytest.mark.slow
def test_w8a8_workload_full_size(dq):
    """The benchmark's 4096^3 product, bf16 out, on sampled rows: one at random
    in each 128-row tile band, plus the first and last rows of the matrix."""
    wl = workloads.make("w8a8_gemm_int8_bf16_4096x4096x4096")
    t = wl.tensors
    dev = torch.device("cuda:0")
    got = dq.w8a8_gemm(t["a"].to(dev), t["b"].to(dev), t["a_scale"].to(dev), t["b_scale"].to(dev),
                       out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    got = _bits(got.cpu())
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([np.arange(0, 4096, 128) + rng.integers(0, 128, 32), [0, 4095]]))
    want = oracle.w8a8_gemm(t["a"][rows].numpy(), t["b"].numpy(), t["a_scale"][rows].numpy(),
                            t["b_scale"].numpy(), out_dtype="bf16")
    np.testing.assert_array_equal(got[rows], want.view(np.uint16))
