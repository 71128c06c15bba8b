"""GPU parity of dequantization (AntiQuantize, PER_TOKEN and PER_GROUP policies).

dq_dequant_per_token through the C ABI against the CPU oracle, bit for bit:
out = (code - offset) * scale in binary32, rounded once to the output type.
Covers int8 / packed int4 / int32 containers, f32 / f16 / bf16 scales and
outputs, with and without offsets, shapes that take the vectorised path and
ragged or misaligned ones that take the scalar path, plus the quantize ->
dequantize round trip on the GPU.
"""

import numpy as np
import pytest
import torch

import oracle
from token_dynamic_quantization_b200 import workloads

pytestmark = pytest.mark.gpu

_TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def dq(dq_lib, cuda_device):
    return dq_lib


def _codes(rows, cols, y_dtype, seed):
    g = torch.Generator().manual_seed(seed)
    if y_dtype == "int8":
        return torch.randint(-128, 128, (rows, cols), generator=g, dtype=torch.int32).to(torch.int8)
    nib = torch.randint(0, 16, (rows, cols), generator=g, dtype=torch.int32)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).to(torch.uint8)
    return packed if y_dtype == "int4" else packed.view(torch.int32)


def _row_params(rows, dtype, seed, offset):
    g = torch.Generator().manual_seed(seed)
    scale = (torch.rand(rows, generator=g) * 0.05 + 1e-3).to(dtype)
    off = (torch.randn(rows, generator=g) * 20).to(dtype) if offset else None
    return scale, off


def _oracle(y, cols, y_dtype, scale, off, out_dtype):
    out = oracle.dequant_per_token(y.numpy() if y_dtype != "int32" else y.numpy().view(np.uint32), scale, off,
                                   y_dtype=y_dtype, cols=cols, out_dtype=out_dtype)
    return out.view(np.uint16) if out_dtype in ("f16", "bf16") else out.view(np.uint32)


def _gpu(dq, y, cols, y_dtype, scale, off, out_dtype, misalign=False):
    dev = torch.device("cuda:0")
    yg = y.to(dev)
    rows = y.shape[0]
    out = None
    if misalign:
        buf = torch.empty(rows * cols + 1, dtype=_TORCH_DT[out_dtype], device=dev)
        out = buf[1:].view(rows, cols)
    o = dq.dequant_per_token(yg, scale.to(dev), None if off is None else off.to(dev), y_dtype=y_dtype, cols=cols,
                             out_dtype=_TORCH_DT[out_dtype], out=out)
    torch.cuda.synchronize()
    o = o.cpu()
    return o.view(torch.int16).numpy().view(np.uint16) if out_dtype != "f32" else o.numpy().view(np.uint32)


SHAPES = [(1, 32), (7, 64), (33, 4096), (5, 1000), (3, 48), (64, 512), (2, 8192)]


@pytest.mark.parametrize("shape", SHAPES, ids=[f"{r}x{c}" for r, c in SHAPES])
@pytest.mark.parametrize("y_dtype", ["int8", "int4", "int32"])
@pytest.mark.parametrize("out_dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("offset", [False, True])
def test_dequant_matches_oracle(dq, shape, y_dtype, out_dtype, offset):
    rows, cols = shape
    if y_dtype == "int32" and cols % 8:
        pytest.skip("INT32 containers need cols % 8 == 0")
    y = _codes(rows, cols, y_dtype, seed=rows * 131 + cols)
    scale, off = _row_params(rows, torch.float32, seed=cols, offset=offset)
    want = _oracle(y, cols, y_dtype, scale, off, out_dtype)
    got = _gpu(dq, y, cols, y_dtype, scale, off, out_dtype)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("sdt", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("out_dtype", ["f16", "bf16", "f32"])
def test_dequant_half_scales(dq, sdt, out_dtype):
    y = _codes(9, 256, "int8", seed=5)
    scale, off = _row_params(9, sdt, seed=6, offset=True)
    want = _oracle(y, 256, "int8", scale, off, out_dtype)
    got = _gpu(dq, y, 256, "int8", scale, off, out_dtype)
    np.testing.assert_array_equal(got, want)


def test_dequant_misaligned_output_takes_the_scalar_path(dq):
    y = _codes(6, 256, "int8", seed=7)
    scale, off = _row_params(6, torch.float32, seed=8, offset=True)
    want = _oracle(y, 256, "int8", scale, off, "bf16")
    got = _gpu(dq, y, 256, "int8", scale, off, "bf16", misalign=True)
    np.testing.assert_array_equal(got, want)


def test_dequant_extreme_scales(dq):
    """Overflow to infinity and underflow to subnormals/zero in the narrow types."""
    y = _codes(4, 64, "int8", seed=9)
    scale = torch.tensor([3e36, 1e-38, 7e-42, 1.0], dtype=torch.float32)
    for out_dtype in ("f16", "bf16", "f32"):
        want = _oracle(y, 64, "int8", scale, None, out_dtype)
        got = _gpu(dq, y, 64, "int8", scale, None, out_dtype)
        np.testing.assert_array_equal(got, want)


def test_dequant_empty(dq):
    dev = torch.device("cuda:0")
    out = dq.dequant_per_token(torch.empty((0, 64), dtype=torch.int8, device=dev),
                               torch.empty(0, device=dev), out_dtype=torch.bfloat16)
    assert out.shape == (0, 64)


@pytest.mark.parametrize("mode,y_dtype", [("symmetric", "int8"), ("asymmetric", "int8"), ("asymmetric", "int4")])
def test_gpu_round_trip(dq, mode, y_dtype):
    """dq_dynamic_quant then dq_dequant_per_token on the GPU equals the
    oracle's dequantization of the oracle's codes, and lands within half a
    step of x."""
    x = workloads.normal((48, 1024), torch.bfloat16, 12, std=3.0)
    dev = torch.device("cuda:0")
    y, s, o, _ = dq.dynamic_quant(x.to(dev), mode=mode, y_dtype=y_dtype)
    back = dq.dequant_per_token(y, s, o, y_dtype=y_dtype, cols=1024, out_dtype=torch.float32)
    torch.cuda.synchronize()
    yo, so, oo = oracle.dynamic_quant(x, mode=mode, y_dtype=y_dtype)
    want = oracle.dequant_per_token(yo, so, oo, y_dtype=y_dtype, cols=1024, out_dtype="f32")
    np.testing.assert_array_equal(back.cpu().numpy(), want)
    err = np.abs(want.astype(np.float64) - x.float().numpy())
    # half a step, plus the binary32 roundings of x / scale (+ offset) and of
    # (code - offset) * scale: each below 2^-24 of a value under 2^8 steps
    assert np.all(err <= so[:, None].astype(np.float64) / 2 * (1 + 2.0 ** -10))


@pytest.mark.slow
def test_dequant_workload_full_size(dq):
    wl = workloads.make("dequant_per_token_int8_bf16_8192x4096")
    t = wl.tensors
    dev = torch.device("cuda:0")
    got = dq.dequant_per_token(t["y"].to(dev), t["scale"].to(dev), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    got = got.cpu().view(torch.int16).numpy().view(np.uint16)
    rows = np.random.default_rng(0).choice(t["y"].shape[0], size=64, replace=False)
    want = oracle.dequant_per_token(t["y"][rows].numpy(), t["scale"][rows], out_dtype="bf16")
    np.testing.assert_array_equal(got[rows], want)


# ---------------------------------------------------------------- PER_GROUP

def _group_tables(rows, cols, g, k_dim, dtype, seed, offset):
    gen = torch.Generator().manual_seed(seed)
    shape = (rows, -(-cols // g)) if k_dim == 1 else (-(-rows // g), cols)
    scale = (torch.rand(shape, generator=gen) * 0.05 + 1e-3).to(dtype)
    off = (torch.randn(shape, generator=gen) * 10).to(dtype) if offset else None
    return scale, off


def _group_gpu(dq, y, cols, y_dtype, scale, off, g, k_dim, out_dtype, misalign_table=False):
    dev = torch.device("cuda:0")
    sg = scale.to(dev)
    if misalign_table:  # a table that is element-aligned but not 16-byte aligned
        buf = torch.empty(scale.numel() + 1, dtype=scale.dtype, device=dev)
        sg = buf[1:].view(scale.shape)
        sg.copy_(scale.to(dev))
    o = dq.dequant_per_group(y.to(dev), sg, None if off is None else off.to(dev), group_size=g, k_dim=k_dim,
                             y_dtype=y_dtype, cols=cols, out_dtype=_TORCH_DT[out_dtype])
    torch.cuda.synchronize()
    o = o.cpu()
    return o.view(torch.int16).numpy().view(np.uint16) if out_dtype != "f32" else o.numpy().view(np.uint32)


def _group_oracle(y, cols, y_dtype, scale, off, g, k_dim, out_dtype):
    out = oracle.dequant_per_group(y.numpy() if y_dtype != "int32" else y.numpy().view(np.uint32), scale, off,
                                   group_size=g, k_dim=k_dim, y_dtype=y_dtype, cols=cols, out_dtype=out_dtype)
    return out.view(np.uint16) if out_dtype in ("f16", "bf16") else out.view(np.uint32)


GROUP_SHAPES = [(8, 256, 32), (33, 4096, 128), (70, 96, 64), (5, 1000, 32), (100, 512, 96)]


@pytest.mark.parametrize("shape", GROUP_SHAPES, ids=[f"{r}x{c}g{g}" for r, c, g in GROUP_SHAPES])
@pytest.mark.parametrize("k_dim", [1, 0])
@pytest.mark.parametrize("y_dtype", ["int8", "int4"])
@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("offset", [False, True])
def test_dequant_per_group_matches_oracle(dq, shape, k_dim, y_dtype, out_dtype, offset):
    rows, cols, g = shape
    y = _codes(rows, cols, y_dtype, seed=rows + cols + g)
    scale, off = _group_tables(rows, cols, g, k_dim, torch.float32, seed=g + k_dim, offset=offset)
    want = _group_oracle(y, cols, y_dtype, scale, off, g, k_dim, out_dtype)
    got = _group_gpu(dq, y, cols, y_dtype, scale, off, g, k_dim, out_dtype)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("sdt", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("k_dim", [1, 0])
def test_dequant_per_group_half_tables(dq, sdt, k_dim):
    y = _codes(40, 512, "int8", seed=13)
    scale, off = _group_tables(40, 512, 32, k_dim, sdt, seed=14, offset=True)
    want = _group_oracle(y, 512, "int8", scale, off, 32, k_dim, "f16")
    got = _group_gpu(dq, y, 512, "int8", scale, off, 32, k_dim, "f16")
    np.testing.assert_array_equal(got, want)


def test_dequant_per_group_unaligned_column_table(dq):
    y = _codes(64, 256, "int8", seed=15)
    scale, _ = _group_tables(64, 256, 32, 0, torch.float32, seed=16, offset=False)
    want = _group_oracle(y, 256, "int8", scale, None, 32, 0, "bf16")
    got = _group_gpu(dq, y, 256, "int8", scale, None, 32, 0, "bf16", misalign_table=True)
    np.testing.assert_array_equal(got, want)


@pytest.mark.slow
def test_dequant_per_group_workload_full_size(dq):
    wl = workloads.make("dequant_per_group_int8_bf16_8192x4096_g128")
    t = wl.tensors
    dev = torch.device("cuda:0")
    got = dq.dequant_per_group(t["y"].to(dev), t["scale"].to(dev), t["offset"].to(dev), group_size=wl.group_size,
                               k_dim=wl.k_dim, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    got = got.cpu().view(torch.int16).numpy().view(np.uint16)
    rows = np.random.default_rng(1).choice(t["y"].shape[0], size=64, replace=False)
    want = oracle.dequant_per_group(t["y"][rows].numpy(), t["scale"][rows], t["offset"][rows],
                                    group_size=wl.group_size, k_dim=wl.k_dim, out_dtype="bf16")
    np.testing.assert_array_equal(got[rows], want)
