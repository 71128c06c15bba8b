"""CPU oracle for per-token dynamic quantization — TEST INFRASTRUCTURE ONLY.

A plain, single-threaded C++ implementation (``dq_oracle.cpp``) of the
formulas on the aclnnDynamicQuantV2 page ("Formula": symmetric and
asymmetric quantization, with and without smooth scales; MoE smooth-scale
selection from "Description") and the aclnnAdaLayerNormQuant page
("Formula", steps 1-5), the PER_TOKEN and PER_GROUP dequantizers of the
AntiQuantize page and the per-token x per-channel scaled W8A8 product of the
aclnnQuantBatchMatmulInplaceAdd page, wrapped here with ctypes + numpy.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. It shares nothing with the CUDA library: no
header, constant, table or helper, and it never imports the product package.

Every function here is pinned by ``tests/test_oracle_pins.py`` against
hand-computed rows, closed forms, exact rational arithmetic and library
routines (see that file for which pin covers which step).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dq_oracle.cpp")
_HDR = os.path.join(_HERE, "dq_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

# The oracle's own codes (mirroring dq_oracle.h; unrelated to the CUDA ABI).
F32, F16, BF16 = 0, 1, 2
Y_INT8, Y_INT4X2, Y_INT32 = 0, 1, 2
SYMMETRIC, ASYMMETRIC = 0, 1
ERRORS = {0: "ok", -1: "shape", -2: "dtype", -3: "argument", -4: "group_index"}

_lock = threading.Lock()
_lib = None


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile liboracle.so with g++ (IEEE fp32, no contraction)."""
    stale = (not os.path.exists(_LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB) for p in (_SRC, _HDR)
    )
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = [
            "g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math",
            "-shared", "-fPIC", "-o", tmp, _SRC,
        ]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
            ci = ctypes.c_int
            lib.oracle_dynamic_quant.argtypes = [vp, ci, i64, i64, vp, ci, vp, i32, ci, ci, vp, vp, vp]
            lib.oracle_dynamic_quant.restype = ci
            lib.oracle_ada_layernorm_pre.argtypes = [vp, ci, i64, i64, i64, vp, vp, vp, vp, vp, ci, f32,
                                                     vp, vp, vp]
            lib.oracle_ada_layernorm_pre.restype = ci
            lib.oracle_ada_layernorm_quant.argtypes = [vp, ci, i64, i64, i64, vp, vp, vp, vp, vp, ci, f32,
                                                       vp, vp]
            lib.oracle_ada_layernorm_quant.restype = ci
            lib.oracle_dequant_per_token.argtypes = [vp, ci, i64, i64, vp, vp, ci, ci, vp]
            lib.oracle_dequant_per_token.restype = ci
            lib.oracle_dequant_per_group.argtypes = [vp, ci, i64, i64, vp, vp, ci, i64, ci, ci, vp]
            lib.oracle_dequant_per_group.restype = ci
            lib.oracle_w8a8_gemm.argtypes = [vp, vp, i64, i64, i64, vp, vp, ci, ci, vp]
            lib.oracle_w8a8_gemm.restype = ci
            lib.oracle_float_to_half_bits.argtypes = [f32]
            lib.oracle_float_to_half_bits.restype = ctypes.c_uint16
            lib.oracle_float_to_bfloat16_bits.argtypes = [f32]
            lib.oracle_float_to_bfloat16_bits.restype = ctypes.c_uint16
            _lib = lib
    return _lib


def _float_buffer(a, dtype: str | None = None):
    """Return (contiguous numpy array, oracle dtype code) for a float tensor.

    Accepts numpy float32/float16 arrays, torch CPU tensors (float32, float16,
    bfloat16), or raw uint16 bit patterns with ``dtype`` = "f16" / "bf16".
    """
    if a is None:
        return None, F32
    if hasattr(a, "detach"):  # torch tensor: marshal through its bit pattern
        import torch

        t = a.detach().contiguous().cpu()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16), BF16
        if t.dtype == torch.float16:
            return t.view(torch.int16).numpy().view(np.uint16), F16
        if t.dtype == torch.float32:
            return t.numpy(), F32
        raise TypeError(f"oracle: unsupported tensor dtype {t.dtype}")
    arr = np.ascontiguousarray(a)
    if dtype == "bf16":
        return arr.view(np.uint16), BF16
    if dtype == "f16" or arr.dtype == np.float16:
        return arr.view(np.uint16), F16
    if arr.dtype == np.float32:
        return arr, F32
    raise TypeError(f"oracle: unsupported array dtype {arr.dtype}")


def _ptr(arr):
    return None if arr is None else arr.ctypes.data


def _check(status: int):
    if status != 0:
        raise OracleError(f"oracle status {status} ({ERRORS.get(status, '?')})")


def dynamic_quant(x, smooth=None, group_index=None, mode: str = "symmetric", y_dtype: str = "int8",
                  x_dtype: str | None = None, smooth_dtype: str | None = None):
    """Per-token dynamic quantization of a 2-D ``x`` [rows, cols].

    aclnnDynamicQuantV2, Formula. ``smooth``: None, [cols] or [E, cols];
    ``group_index``: None or int32 [E] cumulative end rows (Description, MoE);
    ``mode``: "symmetric" | "asymmetric"; ``y_dtype``: "int8" | "int4" (packed
    two per byte, low nibble first) | "int32" (eight int4 codes per word).
    Returns (y, scale, offset-or-None) as numpy arrays.
    """
    lib = _load()
    xb, xc = _float_buffer(x, x_dtype)
    if xb.ndim != 2:
        raise ValueError("oracle.dynamic_quant expects a 2-D x")
    rows, cols = xb.shape
    sb, sc = _float_buffer(smooth, smooth_dtype)
    gi = None
    num_groups = 0
    if group_index is not None:
        gi = np.ascontiguousarray(np.asarray(group_index, dtype=np.int32))
        num_groups = int(gi.shape[0])
    m = {"symmetric": SYMMETRIC, "asymmetric": ASYMMETRIC}[mode]
    yc = {"int8": Y_INT8, "int4": Y_INT4X2, "int32": Y_INT32}[y_dtype]
    if yc == Y_INT8:
        y = np.zeros((rows, cols), dtype=np.int8)
    elif yc == Y_INT4X2:
        y = np.zeros((rows, cols // 2), dtype=np.uint8)
    else:
        y = np.zeros((rows, cols // 8), dtype=np.uint32)
    scale = np.zeros(rows, dtype=np.float32)
    offset = np.zeros(rows, dtype=np.float32) if m == ASYMMETRIC else None
    _check(lib.oracle_dynamic_quant(_ptr(xb), xc, rows, cols, _ptr(sb), sc, _ptr(gi), num_groups,
                                    m, yc, _ptr(y), _ptr(scale), _ptr(offset)))
    return y, scale, offset


def _ada_args(x, ada_scale, ada_shift, weight, bias, smooth, x_dtype, param_dtype):
    xb, xc = _float_buffer(x, x_dtype)
    if xb.ndim != 3:
        raise ValueError("oracle AdaLayerNorm expects x of shape [batch, seq, hidden]")
    batch, seq, hidden = xb.shape
    params = [_float_buffer(p, param_dtype) for p in (ada_scale, ada_shift, weight, bias, smooth)]
    codes = {c for (arr, c) in params if arr is not None}
    if len(codes) > 1:
        raise TypeError("oracle AdaLayerNorm: all parameters must share one dtype")
    pc = codes.pop() if codes else F32
    return xb, xc, batch, seq, hidden, [arr for (arr, _) in params], pc


def ada_layernorm_pre(x, ada_scale, ada_shift, weight=None, bias=None, smooth=None, epsilon: float = 1e-6,
                      x_dtype: str | None = None, param_dtype: str | None = None):
    """aclnnAdaLayerNormQuant Formula steps 1-3: the fp32 value that gets quantized.

    Returns (y [batch, seq, hidden] float32, mean [batch*seq], std [batch*seq]) where
    std = sqrt(Var(x) + epsilon).
    """
    lib = _load()
    xb, xc, batch, seq, hidden, (a, s, w, b, sm), pc = _ada_args(
        x, ada_scale, ada_shift, weight, bias, smooth, x_dtype, param_dtype)
    y = np.zeros((batch, seq, hidden), dtype=np.float32)
    mean = np.zeros(batch * seq, dtype=np.float32)
    std = np.zeros(batch * seq, dtype=np.float32)
    _check(lib.oracle_ada_layernorm_pre(_ptr(xb), xc, batch, seq, hidden, _ptr(a), _ptr(s), _ptr(w), _ptr(b),
                                        _ptr(sm), pc, ctypes.c_float(epsilon), _ptr(y), _ptr(mean), _ptr(std)))
    return y, mean, std


def ada_layernorm_quant(x, ada_scale, ada_shift, weight=None, bias=None, smooth=None, epsilon: float = 1e-6,
                        x_dtype: str | None = None, param_dtype: str | None = None):
    """aclnnAdaLayerNormQuant Formula steps 1-5. Returns (out int8, quant_scale float32 [batch, seq])."""
    lib = _load()
    xb, xc, batch, seq, hidden, (a, s, w, b, sm), pc = _ada_args(
        x, ada_scale, ada_shift, weight, bias, smooth, x_dtype, param_dtype)
    out = np.zeros((batch, seq, hidden), dtype=np.int8)
    qs = np.zeros((batch, seq), dtype=np.float32)
    _check(lib.oracle_ada_layernorm_quant(_ptr(xb), xc, batch, seq, hidden, _ptr(a), _ptr(s), _ptr(w), _ptr(b),
                                          _ptr(sm), pc, ctypes.c_float(epsilon), _ptr(out), _ptr(qs)))
    return out, qs


def _need_entries(buf, n: int, what: str):
    if buf is not None and np.asarray(buf).size != n:
        raise ValueError(f"oracle: {what} must have {n} entries, got {np.asarray(buf).size}")


def dequant_per_token(codes, scale, offset=None, y_dtype: str = "int8", cols: int | None = None,
                      out_dtype: str = "f32", scale_dtype: str | None = None):
    """Per-token dequantization (AntiQuantize, PER_TOKEN policy), read as the
    inverse of the quantizer: out = (code - offset) * scale in binary32, then
    rounded to ``out_dtype`` ("f32" | "f16" | "bf16").

    ``codes``: int8 [rows, cols], packed uint8 [rows, cols/2] ("int4") or
    uint32 [rows, cols/8] ("int32"); ``scale``, ``offset``: [rows] floats.
    Returns float32 for "f32", float16 for "f16" and the uint16 bit patterns
    for "bf16".
    """
    lib = _load()
    yc = {"int8": Y_INT8, "int4": Y_INT4X2, "int32": Y_INT32}[y_dtype]
    cb = np.ascontiguousarray(codes)
    rows = int(cb.shape[0])
    if cols is None:
        cols = int(cb.shape[1]) * {Y_INT8: 1, Y_INT4X2: 2, Y_INT32: 8}[yc]
    sb, sc = _float_buffer(scale, scale_dtype)
    ob = None
    if offset is not None:
        ob, oc = _float_buffer(offset, scale_dtype)
        if oc != sc:
            raise TypeError("oracle: offset must have the dtype of scale")
    _need_entries(sb, rows, "scale")
    if ob is not None:
        _need_entries(ob, rows, "offset")
    oc_out = {"f32": F32, "f16": F16, "bf16": BF16}[out_dtype]
    out = np.zeros((rows, cols), dtype=np.float32 if oc_out == F32 else np.uint16)
    _check(lib.oracle_dequant_per_token(_ptr(cb), yc, rows, cols, _ptr(sb), _ptr(ob), sc, oc_out, _ptr(out)))
    return out.view(np.float16) if oc_out == F16 else out


def dequant_per_group(codes, scale, offset=None, group_size: int = 32, k_dim: int = 1, y_dtype: str = "int8",
                      cols: int | None = None, out_dtype: str = "f32", scale_dtype: str | None = None):
    """Per-group dequantization (AntiQuantize, PER_GROUP policy): element (i, j)
    uses scale/offset entry (i, j // g) when ``k_dim`` = 1 (table
    [rows, ceil(cols/g)]) or (i // g, j) when ``k_dim`` = 0 (table
    [ceil(rows/g), cols]); value as in ``dequant_per_token``."""
    lib = _load()
    yc = {"int8": Y_INT8, "int4": Y_INT4X2, "int32": Y_INT32}[y_dtype]
    cb = np.ascontiguousarray(codes)
    rows = int(cb.shape[0])
    if cols is None:
        cols = int(cb.shape[1]) * {Y_INT8: 1, Y_INT4X2: 2, Y_INT32: 8}[yc]
    sb, sc = _float_buffer(scale, scale_dtype)
    ob = None
    if offset is not None:
        ob, oc = _float_buffer(offset, scale_dtype)
        if oc != sc:
            raise TypeError("oracle: offset must have the dtype of scale")
    if int(group_size) > 0 and int(group_size) % 32 == 0 and int(k_dim) in (0, 1):  # else the oracle rejects it
        g = int(group_size)
        entries = rows * -(-cols // g) if int(k_dim) == 1 else -(-rows // g) * cols
        _need_entries(sb, entries, "scale")
        if ob is not None:
            _need_entries(ob, entries, "offset")
    oc_out = {"f32": F32, "f16": F16, "bf16": BF16}[out_dtype]
    out = np.zeros((rows, cols), dtype=np.float32 if oc_out == F32 else np.uint16)
    _check(lib.oracle_dequant_per_group(_ptr(cb), yc, rows, cols, _ptr(sb), _ptr(ob), sc, int(group_size),
                                        int(k_dim), oc_out, _ptr(out)))
    return out.view(np.float16) if oc_out == F16 else out


def w8a8_gemm(a, b, a_scale, b_scale, out_dtype: str = "f32", accumulate_into=None):
    """out[m, n] = float(sum_k a[m,k] b[n,k]) * (a_scale[m] * b_scale[n])
    (+ accumulate_into[m, n]), binary32, rounded once per operation in that
    order, then narrowed to ``out_dtype``. a: int8 [M, K]; b: int8 [N, K]."""
    lib = _load()
    ab = np.ascontiguousarray(a, dtype=np.int8)
    bb = np.ascontiguousarray(b, dtype=np.int8)
    m, k = ab.shape
    n = bb.shape[0]
    if bb.shape[1] != k:
        raise ValueError("oracle.w8a8_gemm: K mismatch")
    sa = np.ascontiguousarray(a_scale, dtype=np.float32).reshape(-1)
    sb = np.ascontiguousarray(b_scale, dtype=np.float32).reshape(-1)
    if sa.size != m or sb.size != n:
        raise ValueError(f"oracle.w8a8_gemm: scales must have {m} and {n} entries, got {sa.size} and {sb.size}")
    oc = {"f32": F32, "f16": F16, "bf16": BF16}[out_dtype]
    if accumulate_into is not None:
        if oc != F32:
            raise ValueError("accumulation needs float32 output")
        out = np.array(accumulate_into, dtype=np.float32, copy=True)
        if out.shape != (m, n):
            raise ValueError(f"oracle.w8a8_gemm: accumulate_into must be [{m}, {n}]")
    else:
        out = np.zeros((m, n), dtype=np.float32 if oc == F32 else np.uint16)
    _check(lib.oracle_w8a8_gemm(_ptr(ab), _ptr(bb), m, n, k, _ptr(sa), _ptr(sb), oc,
                                1 if accumulate_into is not None else 0, _ptr(out)))
    return out.view(np.float16) if oc == F16 else out


def float_to_half_bits(v: float) -> int:
    """binary32 -> binary16 bit pattern, round to nearest even."""
    return int(_load().oracle_float_to_half_bits(ctypes.c_float(v)))


def float_to_bfloat16_bits(v: float) -> int:
    """binary32 -> bfloat16 bit pattern, round to nearest even."""
    return int(_load().oracle_float_to_bfloat16_bits(ctypes.c_float(v)))


def unpack_int4(packed: np.ndarray, cols: int) -> np.ndarray:
    """Signed codes from the packed INT4 layout (element 2j low nibble of byte j)."""
    p = np.asarray(packed).astype(np.uint8)
    lo = (p & 0xF).astype(np.int8)
    hi = (p >> 4).astype(np.int8)
    lo = np.where(lo >= 8, lo - 16, lo).astype(np.int8)
    hi = np.where(hi >= 8, hi - 16, hi).astype(np.int8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out[..., :cols]
