"""Host-side checks of the benchmark's arithmetic (no GPU).

The algorithmic bytes per call are the numerator of every roofline figure;
they are pinned here to the per-configuration totals worked out separately
from the shapes (x read, codes and per-row floats written, side tables read
once), and the source hash that guards profile traffic is checked to ignore
comments only.
"""

import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from token_dynamic_quantization_b200 import workloads  # noqa: E402

# read + write bytes per call, by configuration
EXPECTED_BYTES = {
    "sym_int8_f16_64x1024": 131_072 + 65_792,
    "sym_int8_smooth_bf16_8192x4096": 67_125_248 + 33_587_200,
    "moe_sym_int8_bf16_32768x7168_e64": 471_597_312 + 235_012_096,
    "asym_int4_f16_16384x8192": 268_435_456 + 67_239_936,
    "ada_layernorm_quant_bf16_4x4096x3072": 100_730_880 + 50_397_184,
    # codes 8192 x 4096 int8 + fp32 scale [8192] read; bf16 [8192, 4096] written
    "dequant_per_token_int8_bf16_8192x4096": 33_554_432 + 32_768 + 67_108_864,
    # codes + fp32 scale and offset tables [8192, 32] read; bf16 written
    "dequant_per_group_int8_bf16_8192x4096_g128": 33_554_432 + 2 * 1_048_576 + 67_108_864,
    # a and b int8 [4096, 4096], both fp32 scale vectors read; bf16 [4096, 4096] written
    "w8a8_gemm_int8_bf16_4096x4096x4096": 2 * 16_777_216 + 2 * 16_384 + 33_554_432,
}


@pytest.mark.parametrize("name", sorted(EXPECTED_BYTES))
def test_algorithmic_bytes(name):
    assert set(EXPECTED_BYTES) == set(workloads.WORKLOADS)
    assert bench.algorithmic_bytes(workloads.make(name)) == EXPECTED_BYTES[name]


def test_w8a8_work_is_two_m_n_k():
    wl = workloads.make("w8a8_gemm_int8_bf16_4096x4096x4096", rows=256)
    units, divisor, unit, _ = bench.work(wl)
    assert units == 2 * 256 * 4096 * 4096 and divisor == 1e12 and unit == "TFLOP/s"


def test_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    csrc = tmp_path / "token_dynamic_quantization_b200" / "csrc"
    csrc.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "probe", ("k.cuh",))
    src = csrc / "k.cuh"
    src.write_text("int f(int x) {\n  return x + 1;  // one\n}\n")
    h0 = bench.source_hash("probe")
    src.write_text("/* a block\n   comment */\nint f(int x) {\n\n  return x + 1;  // two\n}\n")
    assert bench.source_hash("probe") == h0
    src.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.source_hash("probe") != h0


def test_launch_counts_and_timed_kernels():
    """The bench's claim of kernel launches per call and of the kernel it
    times follow the library's dispatch: the ring kernel for long rows, the
    one-warp kernel for few short rows, one AdaLayerNormQuant launch while the
    CTA's affine table rows fit in 64 KB of shared memory (two otherwise)."""
    small = workloads.make("sym_int8_f16_64x1024")
    large = workloads.make("sym_int8_smooth_bf16_8192x4096")
    ada = workloads.make("ada_layernorm_quant_bf16_4x4096x3072")
    gemm = workloads.make("w8a8_gemm_int8_bf16_4096x4096x4096")
    assert bench.timed_kernel(small) == "dynamic_quant_warp_kernel"
    assert bench.timed_kernel(large) == "dynamic_quant_ring_kernel"
    assert bench.timed_kernel(gemm) == "w8a8_gemm_persistent_kernel"
    assert bench.timed_kernel(ada).startswith("ada_layernorm_quant_ring_kernel")
    for wl in (small, large, gemm, ada):
        assert bench.launches_per_call(wl) == 1
    # 2 batches of 3072 columns per CTA: 48 KB of table rows, folded in the kernel
    assert bench.ada_table_staged(ada)

    class Wide:  # 2 batches of 8192 columns per CTA: 128 KB, the table kernel runs first
        kind = "ada_layernorm_quant"
        primary = torch.empty((4, 4096, 8192), dtype=torch.bfloat16, device="meta")

    assert not bench.ada_table_staged(Wide)
    assert bench.launches_per_call(Wide) == 2


def test_rotation_sets_cover_twelve_l2_capacities():
    """The timed steps rotate over buffer sets of at least 12 x the L2 (input
    lines survived a rotation of 3 x), at least two sets, at most 1024."""
    l2 = bench.L2_BYTES
    for per_set in (168_000_000, 250_000_000, 83_000_000, 1_180_000_000, 3 * l2):
        sets = bench.rotation_sets(per_set)
        assert sets >= 2
        assert sets * per_set >= 12 * l2 or sets == 2
    assert bench.rotation_sets(1_180_000_000) == 2
    assert bench.rotation_sets(168_000_000) == 10
    assert bench.rotation_sets(330_000) == bench.MAX_SETS == 1024
    assert bench.MAX_SETS * 330_000 > l2
