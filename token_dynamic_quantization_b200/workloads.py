"""Seeded synthetic inputs for per-token dynamic quantization.

This module only draws random numbers; it holds none of the quantization
arithmetic. The CUDA path, the CPU oracle (in the tests) and the benchmark
all take their inputs from here, so every side sees identical bytes. All
draws use a CPU ``torch.Generator`` with the seed stated next to each tensor.

Workloads (shapes and distributions of the operators' documented use: the
aclnnDynamicQuantV2 page for per-token quantization with optional smooth
scales and MoE group index, the aclnnAdaLayerNormQuant page for the fused
LayerNorm path):

* ``sym_int8_f16_64x1024``: x fp16 [64, 1024] ~ N(0, 1) (seed 0); symmetric
  INT8, no smooth scales.
* ``sym_int8_smooth_bf16_8192x4096``: x bf16 [8192, 4096] ~ N(0, 1) (seed 0)
  with 41 columns (1 % of 4096, chosen by randperm with seed 1) multiplied by
  20 as activation outliers; smooth fp32 [4096] ~ U(0.5, 2.0) (seed 2);
  symmetric INT8.
* ``moe_sym_int8_bf16_32768x7168_e64``: x bf16 [32768, 7168] ~ N(0, 1)
  (seed 0); rows sorted by expert over 64 experts, per-expert counts from
  32768 uniform multinomial draws (seed 3), group_index = int32 cumulative
  end rows; smooth fp32 [64, 7168] ~ U(0.5, 2.0) (seed 2); symmetric INT8.
* ``asym_int4_f16_16384x8192``: x fp16 [16384, 8192] ~ N(0.5, 2.0) (mean
  0.5, std 2.0, seed 0); asymmetric packed INT4.
* ``ada_layernorm_quant_bf16_4x4096x3072``: x bf16 [4, 4096, 3072] ~ N(0, 1)
  (seed 0); adaptive scale and shift bf16 [4, 3072] ~ N(0, 0.1) (seeds 4, 5);
  LayerNorm weight bf16 [3072] ~ N(1, 0.05) (seed 6), bias ~ N(0, 0.05)
  (seed 7); smooth bf16 [3072] ~ U(0.5, 2.0) (seed 2); epsilon 1e-6.
* ``dequant_per_token_int8_bf16_8192x4096`` (AntiQuantize page, PER_TOKEN
  policy; the inverse of the 8192 x 4096 quantization workload): codes int8
  [8192, 4096] uniform in [-127, 127] (seed 8), per-row scale fp32 [8192]
  ~ U(0.001, 0.05) (seed 9), no offset, bfloat16 output.
* ``dequant_per_group_int8_bf16_8192x4096_g128`` (AntiQuantize page,
  PER_GROUP policy, kDim 1): codes int8 [8192, 4096] uniform in [-127, 127]
  (seed 8), groups of 128 along each row with fp32 scale [8192, 32]
  ~ U(0.001, 0.05) (seed 9) and offset [8192, 32] ~ N(0, 8) (seed 10),
  bfloat16 output.
* ``w8a8_gemm_int8_bf16_4096x4096x4096`` (aclnnQuantBatchMatmulInplaceAdd,
  the consumer of the codes): a int8 [4096, 4096] and b int8 [4096, 4096]
  uniform in [-127, 127] (seeds 11, 12), per-token scale fp32 [4096]
  ~ U(0.001, 0.02) (seed 13), per-channel scale fp32 [4096] ~ U(0.001, 0.02)
  (seed 14), bfloat16 output.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def normal(shape, dtype, seed: int, mean: float = 0.0, std: float = 1.0) -> torch.Tensor:
    """N(mean, std) drawn in fp32 on the CPU, then stored as ``dtype``."""
    t = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(dtype)


def uniform(shape, dtype, seed: int, lo: float, hi: float) -> torch.Tensor:
    """U(lo, hi) drawn in fp32 on the CPU, then stored as ``dtype``."""
    t = torch.rand(*shape, generator=_gen(seed), dtype=torch.float32)
    return (t * (hi - lo) + lo).to(dtype)


def with_outlier_columns(x: torch.Tensor, fraction: float, factor: float, seed: int) -> torch.Tensor:
    """Multiply round(fraction * cols) columns (a seeded randperm choice) by ``factor``."""
    cols = x.shape[-1]
    n = int(round(fraction * cols))
    idx = torch.randperm(cols, generator=_gen(seed))[:n]
    y = x.to(torch.float32)
    y[..., idx] *= factor
    return y.to(x.dtype)


def moe_group_index(rows: int, experts: int, seed: int) -> torch.Tensor:
    """int32 [experts] cumulative end rows of a uniform multinomial split of ``rows``."""
    probs = torch.full((experts,), 1.0 / experts)
    draws = torch.multinomial(probs, rows, replacement=True, generator=_gen(seed))
    counts = torch.bincount(draws, minlength=experts)
    return torch.cumsum(counts, 0).to(torch.int32)


@dataclass
class Workload:
    """One synthetic workload: named tensors on the CPU plus the call's options."""

    name: str
    kind: str                    # "dynamic_quant" | "ada_layernorm_quant" | "dequant_per_token" | "dequant_per_group" | "w8a8_gemm"
    tensors: dict = field(default_factory=dict)
    mode: str = "symmetric"      # dynamic_quant only
    y_dtype: str = "int8"        # code container (dynamic_quant output, dequant_per_token input)
    epsilon: float = 1e-6        # ada_layernorm_quant only
    out_dtype: str = "bf16"      # dequantization only
    group_size: int = 0          # dequant_per_group only
    k_dim: int = 1               # dequant_per_group only

    @property
    def primary(self):
        """The per-row input: x, or the codes of a dequantization."""
        if self.kind == "w8a8_gemm":
            return self.tensors["a"]
        return self.tensors["y"] if self.kind.startswith("dequant") else self.tensors["x"]

    @property
    def rows(self) -> int:
        t = self.primary
        return int(t.numel() // t.shape[-1])

    @property
    def cols(self) -> int:
        if self.kind == "w8a8_gemm":
            return int(self.tensors["a"].shape[-1])
        if self.kind.startswith("dequant"):
            return int(self.tensors["y"].shape[-1]) * {"int8": 1, "int4": 2, "int32": 8}[self.y_dtype]
        return int(self.tensors["x"].shape[-1])


WORKLOADS = (
    "sym_int8_f16_64x1024",
    "sym_int8_smooth_bf16_8192x4096",
    "moe_sym_int8_bf16_32768x7168_e64",
    "asym_int4_f16_16384x8192",
    "ada_layernorm_quant_bf16_4x4096x3072",
    "dequant_per_token_int8_bf16_8192x4096",
    "dequant_per_group_int8_bf16_8192x4096_g128",
    "w8a8_gemm_int8_bf16_4096x4096x4096",
)


def make(name: str, rows: int | None = None) -> Workload:
    """Build one of the named workloads (CPU tensors).

    ``rows``: optional smaller row count drawn the same way (for quick
    captures of the same kernel configuration); the MoE group index is drawn
    for that row count, and for the AdaLayerNorm workload the sequence length
    shrinks (rows = batch * seq).
    """
    if name == "sym_int8_f16_64x1024":
        return Workload(name, "dynamic_quant", {"x": normal((rows or 64, 1024), torch.float16, 0)})
    if name == "sym_int8_smooth_bf16_8192x4096":
        r = rows or 8192
        x = with_outlier_columns(normal((r, 4096), torch.bfloat16, 0), 0.01, 20.0, 1)
        smooth = uniform((4096,), torch.float32, 2, 0.5, 2.0)
        return Workload(name, "dynamic_quant", {"x": x, "smooth": smooth})
    if name == "moe_sym_int8_bf16_32768x7168_e64":
        r = rows or 32768
        x = normal((r, 7168), torch.bfloat16, 0)
        smooth = uniform((64, 7168), torch.float32, 2, 0.5, 2.0)
        gi = moe_group_index(r, 64, 3)
        return Workload(name, "dynamic_quant", {"x": x, "smooth": smooth, "group_index": gi})
    if name == "asym_int4_f16_16384x8192":
        x = normal((rows or 16384, 8192), torch.float16, 0, mean=0.5, std=2.0)
        return Workload(name, "dynamic_quant", {"x": x}, mode="asymmetric", y_dtype="int4")
    if name == "ada_layernorm_quant_bf16_4x4096x3072":
        b, h = 4, 3072
        s = max(1, (rows or 4 * 4096) // b)
        t = {
            "x": normal((b, s, h), torch.bfloat16, 0),
            "ada_scale": normal((b, h), torch.bfloat16, 4, std=0.1),
            "ada_shift": normal((b, h), torch.bfloat16, 5, std=0.1),
            "weight": normal((h,), torch.bfloat16, 6, mean=1.0, std=0.05),
            "bias": normal((h,), torch.bfloat16, 7, std=0.05),
            "smooth": uniform((h,), torch.bfloat16, 2, 0.5, 2.0),
        }
        return Workload(name, "ada_layernorm_quant", t, epsilon=1e-6)
    if name == "dequant_per_token_int8_bf16_8192x4096":
        r = rows or 8192
        g = _gen(8)
        y = torch.randint(-127, 128, (r, 4096), generator=g, dtype=torch.int32).to(torch.int8)
        scale = uniform((r,), torch.float32, 9, 0.001, 0.05)
        return Workload(name, "dequant_per_token", {"y": y, "scale": scale}, y_dtype="int8", out_dtype="bf16")
    if name == "dequant_per_group_int8_bf16_8192x4096_g128":
        r = rows or 8192
        g = _gen(8)
        y = torch.randint(-127, 128, (r, 4096), generator=g, dtype=torch.int32).to(torch.int8)
        scale = uniform((r, 32), torch.float32, 9, 0.001, 0.05)
        offset = normal((r, 32), torch.float32, 10, std=8.0)
        return Workload(name, "dequant_per_group", {"y": y, "scale": scale, "offset": offset}, y_dtype="int8",
                        out_dtype="bf16", group_size=128, k_dim=1)
    if name == "w8a8_gemm_int8_bf16_4096x4096x4096":
        m = rows or 4096
        a = torch.randint(-127, 128, (m, 4096), generator=_gen(11), dtype=torch.int32).to(torch.int8)
        b = torch.randint(-127, 128, (4096, 4096), generator=_gen(12), dtype=torch.int32).to(torch.int8)
        return Workload(name, "w8a8_gemm", {"a": a, "b": b, "a_scale": uniform((m,), torch.float32, 13, 0.001, 0.02),
                                            "b_scale": uniform((4096,), torch.float32, 14, 0.001, 0.02)},
                        out_dtype="bf16")
    raise KeyError(f"unknown workload {name!r}; known: {', '.join(WORKLOADS)}")
