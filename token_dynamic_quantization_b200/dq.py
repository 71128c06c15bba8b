"""ctypes binding of libdq.so (C ABI in include/dq.h) — argument marshalling only.

The functions named like the C entry points (``dq_get_workspace_size``,
``dq_dynamic_quant``, ``dq_ada_layernorm_quant``, ``dq_status_string``) take
raw integers (device pointers, sizes, enum values, a ``cudaStream_t``) exactly
as the C ABI does. ``dynamic_quant`` and ``ada_layernorm_quant`` are
tensor-level conveniences: they allocate the outputs with torch (device
memory is torch's job here), pass pointers and the current stream, and return
the tensors. Every step of the computation runs in the CUDA kernels.

Importing this module loads the library and raises ImportError if it is
missing; there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdq.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is not built; run `python -m token_dynamic_quantization_b200.build` "
        "(the CUDA library is required: there is no CPU fallback)")

_lib = ctypes.CDLL(_LIB_PATH)

# ---- enums (values fixed by include/dq.h)
DQ_OK = 0
DQ_ERR_NULL_POINTER = 1
DQ_ERR_BAD_SHAPE = 2
DQ_ERR_BAD_DTYPE = 3
DQ_ERR_UNSUPPORTED = 4
DQ_ERR_MISALIGNED = 5
DQ_ERR_WORKSPACE_TOO_SMALL = 6
DQ_ERR_CUDA = 7
DQ_ERR_BAD_ARGUMENT = 8

DQ_F32, DQ_F16, DQ_BF16, DQ_INT8, DQ_INT4X2, DQ_INT32 = 0, 1, 2, 3, 4, 5
DQ_SYMMETRIC, DQ_ASYMMETRIC = 0, 1
DQ_WS_ROWS_PAST_LAST_GROUP = 0x1
DQ_WS_GROUP_INDEX_INVALID = 0x2
DQ_MAX_GROUPS = 1024
DQ_ADA_NOALLOC_MAX_TABLE = 131072

_vp, _i64, _i32, _f32, _sz, _ci = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                                   ctypes.c_size_t, ctypes.c_int)

_lib.dq_status_string.argtypes = [_ci]
_lib.dq_status_string.restype = ctypes.c_char_p
_lib.dq_get_workspace_size.argtypes = [_i64, _i64, _ci, _ci, _ci, _i32, ctypes.POINTER(_sz)]
_lib.dq_get_workspace_size.restype = _ci
_lib.dq_dynamic_quant.argtypes = [_vp, _ci, _i64, _i64, _vp, _ci, _vp, _i32, _ci, _ci, _vp, _vp, _vp, _vp, _sz,
                                  _vp]
_lib.dq_dynamic_quant.restype = _ci
_lib.dq_ada_layernorm_quant_get_workspace_size.argtypes = [_i64, _i64, _i64, _ci, _ci, ctypes.POINTER(_sz)]
_lib.dq_ada_layernorm_quant_get_workspace_size.restype = _ci
_lib.dq_ada_layernorm_quant.argtypes = [_vp, _ci, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _ci, _f32, _vp, _vp,
                                        _vp, _sz, _vp]
_lib.dq_ada_layernorm_quant.restype = _ci
_lib.dq_dequant_per_token.argtypes = [_vp, _ci, _i64, _i64, _vp, _vp, _ci, _vp, _ci, _vp]
_lib.dq_dequant_per_token.restype = _ci
_lib.dq_dequant_per_group.argtypes = [_vp, _ci, _i64, _i64, _vp, _vp, _ci, _i64, _i32, _vp, _ci, _vp]
_lib.dq_dequant_per_group.restype = _ci
_lib.dq_w8a8_gemm.argtypes = [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _ci, _i32, _vp]
_lib.dq_w8a8_gemm.restype = _ci
_lib.dq_ada_layernorm_quant_noalloc.argtypes = [_vp, _ci, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _ci, _f32, _vp,
                                                _vp, _vp]
_lib.dq_ada_layernorm_quant_noalloc.restype = _ci

LIBRARY_PATH = _LIB_PATH


class DQError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        super().__init__(dq_status_string(status))


# ---------------------------------------------------------------- C-ABI mirrors

def dq_status_string(status: int) -> str:
    return _lib.dq_status_string(status).decode()


def dq_get_workspace_size(rows: int, cols: int, x_dtype: int, mode: int, y_dtype: int, num_groups: int) -> int:
    out = _sz(0)
    st = _lib.dq_get_workspace_size(rows, cols, x_dtype, mode, y_dtype, num_groups, ctypes.byref(out))
    if st != DQ_OK:
        raise DQError(st)
    return int(out.value)


def dq_ada_layernorm_quant_get_workspace_size(batch: int, seq: int, hidden: int, x_dtype: int,
                                              param_dtype: int) -> int:
    out = _sz(0)
    st = _lib.dq_ada_layernorm_quant_get_workspace_size(batch, seq, hidden, x_dtype, param_dtype, ctypes.byref(out))
    if st != DQ_OK:
        raise DQError(st)
    return int(out.value)


def dq_dynamic_quant(x, x_dtype, rows, cols, smooth, smooth_dtype, group_index, num_groups, mode, y_dtype, y,
                     scale, offset, workspace, workspace_bytes, stream) -> int:
    """Raw call: pointers are ints (0/None for NULL). Returns the dq_status."""
    return _lib.dq_dynamic_quant(x, x_dtype, rows, cols, smooth, smooth_dtype, group_index, num_groups, mode,
                                 y_dtype, y, scale, offset, workspace, workspace_bytes, stream)


def dq_ada_layernorm_quant(x, x_dtype, batch, seq, hidden, ada_scale, ada_shift, weight, bias, smooth,
                           param_dtype, epsilon, out, quant_scale, workspace, workspace_bytes, stream) -> int:
    """Raw call: pointers are ints (0/None for NULL). Returns the dq_status."""
    return _lib.dq_ada_layernorm_quant(x, x_dtype, batch, seq, hidden, ada_scale, ada_shift, weight, bias,
                                       smooth, param_dtype, epsilon, out, quant_scale, workspace,
                                       workspace_bytes, stream)


def dq_dequant_per_token(y, y_dtype, rows, cols, scale, offset, scale_dtype, out, out_dtype, stream) -> int:
    """Raw call: pointers are ints (0/None for NULL). Returns the dq_status."""
    return _lib.dq_dequant_per_token(y, y_dtype, rows, cols, scale, offset, scale_dtype, out, out_dtype, stream)


def dq_dequant_per_group(y, y_dtype, rows, cols, scale, offset, scale_dtype, group_size, k_dim, out, out_dtype,
                         stream) -> int:
    """Raw call: pointers are ints (0/None for NULL). Returns the dq_status."""
    return _lib.dq_dequant_per_group(y, y_dtype, rows, cols, scale, offset, scale_dtype, group_size, k_dim, out,
                                     out_dtype, stream)


def dq_w8a8_gemm(a, b, m, n, k, a_scale, b_scale, out, out_dtype, accumulate, stream) -> int:
    """Raw call: pointers are ints (0/None for NULL). Returns the dq_status."""
    return _lib.dq_w8a8_gemm(a, b, m, n, k, a_scale, b_scale, out, out_dtype, accumulate, stream)


def dq_ada_layernorm_quant_noalloc(x, x_dtype, batch, seq, hidden, ada_scale, ada_shift, weight, bias, smooth,
                                   param_dtype, epsilon, out, quant_scale, stream) -> int:
    """Raw call (no workspace: the library's fixed table). Returns the dq_status."""
    return _lib.dq_ada_layernorm_quant_noalloc(x, x_dtype, batch, seq, hidden, ada_scale, ada_shift, weight, bias,
                                               smooth, param_dtype, epsilon, out, quant_scale, stream)


# ---------------------------------------------------------------- tensor-level helpers

def _torch():
    import torch

    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    m = {torch.float32: DQ_F32, torch.float16: DQ_F16, torch.bfloat16: DQ_BF16}
    if t.dtype not in m:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return m[t.dtype]


def _dev_ptr(t, name: str) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


_MODES = {"symmetric": DQ_SYMMETRIC, "asymmetric": DQ_ASYMMETRIC}
_YTYPES = {"int8": DQ_INT8, "int4": DQ_INT4X2, "int32": DQ_INT32}


def output_shapes(rows: int, cols: int, y_dtype: str):
    if y_dtype == "int8":
        return (rows, cols)
    if y_dtype == "int4":
        return (rows, cols // 2)
    return (rows, cols // 8)


def dynamic_quant(x, smooth=None, group_index=None, mode: str = "symmetric", y_dtype: str = "int8",
                  out=None, stream=None, check: bool = True):
    """Per-token dynamic quantization of CUDA tensor ``x`` (last dim = row).

    Returns ``(y, scale, offset, workspace)``: y int8 / uint8 (packed int4) /
    int32 (eight int4 per word) shaped like x with its last dim scaled;
    scale float32 (leading dims of x); offset float32 or None (symmetric);
    workspace (int32 tensor holding the status word) or None.
    ``out`` may pass preallocated ``(y, scale, offset, workspace)``.
    """
    torch = _torch()
    cols = int(x.shape[-1])
    rows = int(x.numel() // cols) if cols else 0
    lead = tuple(x.shape[:-1])
    m, yc = _MODES[mode], _YTYPES[y_dtype]
    ngroups = int(group_index.numel()) if group_index is not None else 0
    ws_bytes = dq_get_workspace_size(rows, cols, _dtype_code(x), m, yc, ngroups)
    if out is None:
        ydt = {"int8": torch.int8, "int4": torch.uint8, "int32": torch.int32}[y_dtype]
        y = torch.empty(lead + output_shapes(1, cols, y_dtype)[1:], dtype=ydt, device=x.device)
        scale = torch.empty(lead, dtype=torch.float32, device=x.device)
        offset = torch.empty(lead, dtype=torch.float32, device=x.device) if m == DQ_ASYMMETRIC else None
        ws = torch.empty((max(ws_bytes, 4) // 4,), dtype=torch.int32, device=x.device) if ws_bytes else None
    else:
        y, scale, offset, ws = out
    if stream is None:
        stream = torch.cuda.current_stream(x.device).cuda_stream
    st = dq_dynamic_quant(_dev_ptr(x, "x"), _dtype_code(x), rows, cols,
                          _dev_ptr(smooth, "smooth"), _dtype_code(smooth) if smooth is not None else DQ_F32,
                          _dev_ptr(group_index, "group_index"), ngroups, m, yc,
                          _dev_ptr(y, "y"), _dev_ptr(scale, "scale"), _dev_ptr(offset, "offset"),
                          _dev_ptr(ws, "workspace"), ws_bytes, stream)
    if check and st != DQ_OK:
        raise DQError(st)
    return y, scale, offset, ws


def ada_layernorm_quant(x, ada_scale, ada_shift, weight=None, bias=None, smooth=None, epsilon: float = 1e-6,
                        out=None, workspace=None, stream=None, check: bool = True):
    """Fused AdaLayerNorm + symmetric INT8 quantization of CUDA tensor ``x`` [batch, seq, hidden].

    Returns ``(out int8 [batch, seq, hidden], quant_scale float32 [batch, seq])``.
    ``workspace``: optional preallocated CUDA tensor of at least
    ``dq_ada_layernorm_quant_get_workspace_size`` bytes (16-byte aligned).
    """
    torch = _torch()
    if x.dim() != 3:
        raise ValueError("x must be [batch, seq, hidden]")
    batch, seq, hidden = (int(d) for d in x.shape)
    pdt = _dtype_code(ada_scale)
    for name, p in (("ada_shift", ada_shift), ("weight", weight), ("bias", bias), ("smooth", smooth)):
        if p is not None and _dtype_code(p) != pdt:
            raise TypeError(f"{name} must have the dtype of ada_scale")
    ws_bytes = dq_ada_layernorm_quant_get_workspace_size(batch, seq, hidden, _dtype_code(x), pdt)
    if out is None:
        o = torch.empty((batch, seq, hidden), dtype=torch.int8, device=x.device)
        qs = torch.empty((batch, seq), dtype=torch.float32, device=x.device)
    else:
        o, qs = out
    if workspace is None and ws_bytes:
        workspace = torch.empty((ws_bytes + 15) // 16 * 4, dtype=torch.float32, device=x.device)
    if stream is None:
        stream = torch.cuda.current_stream(x.device).cuda_stream
    st = dq_ada_layernorm_quant(_dev_ptr(x, "x"), _dtype_code(x), batch, seq, hidden,
                                _dev_ptr(ada_scale, "ada_scale"), _dev_ptr(ada_shift, "ada_shift"),
                                _dev_ptr(weight, "weight"), _dev_ptr(bias, "bias"), _dev_ptr(smooth, "smooth"),
                                pdt, float(epsilon), _dev_ptr(o, "out"), _dev_ptr(qs, "quant_scale"),
                                _dev_ptr(workspace, "workspace"),
                                ws_bytes if workspace is not None else 0, stream)
    if check and st != DQ_OK:
        raise DQError(st)
    return o, qs


def dequant_per_token(y, scale, offset=None, y_dtype: str = "int8", cols: int | None = None,
                      out_dtype=None, out=None, stream=None, check: bool = True):
    """Per-token dequantization of CUDA codes ``y`` (AntiQuantize, PER_TOKEN).

    ``y``: int8 [rows, cols], uint8 [rows, cols/2] ("int4") or int32
    [rows, cols/8] ("int32"); ``scale`` / ``offset``: CUDA [rows] float
    tensors of one dtype; ``out_dtype``: torch.float32 / float16 / bfloat16
    (default: the scale's dtype). Returns the [rows, cols] output tensor.
    """
    torch = _torch()
    yc = _YTYPES[{"int8": "int8", "int4": "int4", "int32": "int32"}[y_dtype]]
    rows = int(y.shape[0]) if y.dim() else 0
    if cols is None:
        cols = int(y.shape[-1]) * {DQ_INT8: 1, DQ_INT4X2: 2, DQ_INT32: 8}[yc]
    sdt = _dtype_code(scale)
    if offset is not None and _dtype_code(offset) != sdt:
        raise TypeError("offset must have the dtype of scale")
    if out_dtype is None:
        out_dtype = scale.dtype
    if out is None:
        out = torch.empty((rows, cols), dtype=out_dtype, device=y.device)
    if stream is None:
        stream = torch.cuda.current_stream(y.device).cuda_stream
    st = dq_dequant_per_token(_dev_ptr(y, "y"), yc, rows, cols, _dev_ptr(scale, "scale"), _dev_ptr(offset, "offset"),
                              sdt, _dev_ptr(out, "out"), _dtype_code(out), stream)
    if check and st != DQ_OK:
        raise DQError(st)
    return out


def dequant_per_group(y, scale, offset=None, group_size: int = 32, k_dim: int = 1, y_dtype: str = "int8",
                      cols: int | None = None, out_dtype=None, out=None, stream=None, check: bool = True):
    """Per-group dequantization of CUDA codes ``y`` (AntiQuantize, PER_GROUP).

    ``scale`` / ``offset``: CUDA tables [rows, ceil(cols/g)] (``k_dim`` 1) or
    [ceil(rows/g), cols] (``k_dim`` 0) of one float dtype. Returns the
    [rows, cols] output tensor (``out_dtype`` defaults to the scale's dtype).
    """
    torch = _torch()
    yc = _YTYPES[y_dtype]
    rows = int(y.shape[0]) if y.dim() else 0
    if cols is None:
        cols = int(y.shape[-1]) * {DQ_INT8: 1, DQ_INT4X2: 2, DQ_INT32: 8}[yc]
    sdt = _dtype_code(scale)
    if offset is not None and _dtype_code(offset) != sdt:
        raise TypeError("offset must have the dtype of scale")
    if out is None:
        out = torch.empty((rows, cols), dtype=out_dtype or scale.dtype, device=y.device)
    if stream is None:
        stream = torch.cuda.current_stream(y.device).cuda_stream
    st = dq_dequant_per_group(_dev_ptr(y, "y"), yc, rows, cols, _dev_ptr(scale, "scale"), _dev_ptr(offset, "offset"),
                              sdt, int(group_size), int(k_dim), _dev_ptr(out, "out"), _dtype_code(out), stream)
    if check and st != DQ_OK:
        raise DQError(st)
    return out


def w8a8_gemm(a, b, a_scale, b_scale, out_dtype=None, out=None, accumulate: bool = False, stream=None,
              check: bool = True):
    """out = float(a @ b.T) * (a_scale[:, None] * b_scale[None, :]) (+ out).

    ``a``: CUDA int8 [M, K]; ``b``: CUDA int8 [N, K]; scales float32 [M], [N].
    Returns the [M, N] output (``out_dtype`` default float32).
    """
    torch = _torch()
    if a.dim() != 2 or b.dim() != 2 or a.dtype != torch.int8 or b.dtype != torch.int8:
        raise TypeError("a and b must be 2-D int8 tensors")
    m, k = (int(v) for v in a.shape)
    n = int(b.shape[0])
    if int(b.shape[1]) != k:
        raise ValueError(f"b must be [N, K] with the K of a ({k}), got {tuple(b.shape)}")
    for name, t, length in (("a_scale", a_scale, m), ("b_scale", b_scale, n)):
        if t.dtype != torch.float32 or t.numel() != length:
            raise TypeError(f"{name} must be float32 with {length} elements")
    if out is None:
        out = torch.empty((m, n), dtype=out_dtype or torch.float32, device=a.device)
    elif tuple(out.shape) != (m, n):
        raise ValueError(f"out must be [{m}, {n}], got {tuple(out.shape)}")
    if stream is None:
        stream = torch.cuda.current_stream(a.device).cuda_stream
    st = dq_w8a8_gemm(_dev_ptr(a, "a"), _dev_ptr(b, "b"), m, n, k, _dev_ptr(a_scale, "a_scale"),
                      _dev_ptr(b_scale, "b_scale"), _dev_ptr(out, "out"), _dtype_code(out), 1 if accumulate else 0,
                      stream)
    if check and st != DQ_OK:
        raise DQError(st)
    return out
