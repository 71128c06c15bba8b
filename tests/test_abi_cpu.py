"""C-ABI checks that need no GPU: exports and host-side validation.

Every call here is rejected by the host validation before anything is
launched, so the fake pointers below are never dereferenced (on any machine).
"""

import os
import re
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]

FAKE = 0x10000  # 64 KiB-aligned fake device address (never dereferenced)


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w]*\s*\*?\s*(dq_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("dq_get_workspace_size", "dq_dynamic_quant", "dq_ada_layernorm_quant_get_workspace_size",
              "dq_ada_layernorm_quant", "dq_dequant_per_token", "dq_dequant_per_group", "dq_w8a8_gemm",
              "dq_ada_layernorm_quant_noalloc", "dq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(dq_lib):
    import ctypes

    lib = ctypes.CDLL(dq_lib.LIBRARY_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), f"libdq.so does not export {n}"


def test_status_strings(dq_lib):
    for s in range(0, 9):
        text = dq_lib.dq_status_string(s)
        assert text.startswith("DQ_")
    assert "unknown" in dq_lib.dq_status_string(99)


def test_workspace_size(dq_lib):
    d = dq_lib
    assert d.dq_get_workspace_size(8192, 4096, d.DQ_BF16, d.DQ_SYMMETRIC, d.DQ_INT8, 0) == 0
    assert d.dq_get_workspace_size(32768, 7168, d.DQ_BF16, d.DQ_SYMMETRIC, d.DQ_INT8, 64) == 4
    assert d.dq_get_workspace_size(0, 2, d.DQ_F16, d.DQ_ASYMMETRIC, d.DQ_INT4X2, 0) == 0
    bad = [
        ((-1, 8, d.DQ_F16, 0, d.DQ_INT8, 0), d.DQ_ERR_BAD_SHAPE),
        ((4, 0, d.DQ_F16, 0, d.DQ_INT8, 0), d.DQ_ERR_BAD_SHAPE),
        ((4, 7, d.DQ_F16, 0, d.DQ_INT4X2, 0), d.DQ_ERR_BAD_SHAPE),
        ((4, 12, d.DQ_F16, 0, d.DQ_INT32, 0), d.DQ_ERR_BAD_SHAPE),
        ((4, 8, d.DQ_F32, 0, d.DQ_INT8, 0), d.DQ_ERR_BAD_DTYPE),
        ((4, 8, d.DQ_F16, 0, d.DQ_F16, 0), d.DQ_ERR_BAD_DTYPE),
        ((4, 8, d.DQ_F16, 2, d.DQ_INT8, 0), d.DQ_ERR_BAD_ARGUMENT),
        ((4, 8, d.DQ_F16, 0, d.DQ_INT8, -1), d.DQ_ERR_BAD_ARGUMENT),
        ((4, 8, d.DQ_F16, 0, d.DQ_INT8, d.DQ_MAX_GROUPS + 1), d.DQ_ERR_UNSUPPORTED),
    ]
    for args, want in bad:
        with pytest.raises(d.DQError) as ei:
            d.dq_get_workspace_size(*args)
        assert ei.value.status == want, args


def _dq(d, **kw):
    a = dict(x=FAKE, x_dtype=d.DQ_BF16, rows=4, cols=64, smooth=None, smooth_dtype=d.DQ_F32, group_index=None,
             num_groups=0, mode=d.DQ_SYMMETRIC, y_dtype=d.DQ_INT8, y=FAKE, scale=FAKE, offset=None,
             workspace=None, workspace_bytes=0, stream=None)
    a.update(kw)
    return d.dq_dynamic_quant(**a)


def test_dynamic_quant_validation(dq_lib):
    d = dq_lib
    assert _dq(d, rows=0, x=None, y=None, scale=None) == d.DQ_OK  # empty input: no-op, no launch
    cases = [
        (dict(x=None), d.DQ_ERR_NULL_POINTER),
        (dict(y=None), d.DQ_ERR_NULL_POINTER),
        (dict(scale=None), d.DQ_ERR_NULL_POINTER),
        (dict(mode=d.DQ_ASYMMETRIC), d.DQ_ERR_NULL_POINTER),           # offset missing
        (dict(rows=-3), d.DQ_ERR_BAD_SHAPE),
        (dict(cols=0), d.DQ_ERR_BAD_SHAPE),
        (dict(cols=63, y_dtype=d.DQ_INT4X2), d.DQ_ERR_BAD_SHAPE),
        (dict(cols=60, y_dtype=d.DQ_INT32), d.DQ_ERR_BAD_SHAPE),
        (dict(x_dtype=d.DQ_INT8), d.DQ_ERR_BAD_DTYPE),
        (dict(y_dtype=d.DQ_BF16), d.DQ_ERR_BAD_DTYPE),
        (dict(smooth=FAKE, smooth_dtype=d.DQ_INT8), d.DQ_ERR_BAD_DTYPE),
        (dict(mode=7), d.DQ_ERR_BAD_ARGUMENT),
        (dict(group_index=FAKE, num_groups=0, smooth=FAKE), d.DQ_ERR_BAD_ARGUMENT),
        (dict(group_index=None, num_groups=3, smooth=FAKE), d.DQ_ERR_BAD_ARGUMENT),
        (dict(group_index=FAKE, num_groups=3), d.DQ_ERR_BAD_ARGUMENT),  # MoE needs smooth scales
        (dict(group_index=FAKE, num_groups=3, smooth=FAKE), d.DQ_ERR_WORKSPACE_TOO_SMALL),
        (dict(group_index=FAKE, num_groups=3, smooth=FAKE, workspace=FAKE, workspace_bytes=2),
         d.DQ_ERR_WORKSPACE_TOO_SMALL),
        (dict(group_index=FAKE, num_groups=d.DQ_MAX_GROUPS + 1, smooth=FAKE, workspace=FAKE, workspace_bytes=4),
         d.DQ_ERR_UNSUPPORTED),
        (dict(x=FAKE + 1), d.DQ_ERR_MISALIGNED),
        (dict(scale=FAKE + 2), d.DQ_ERR_MISALIGNED),
        (dict(mode=d.DQ_ASYMMETRIC, offset=FAKE + 1), d.DQ_ERR_MISALIGNED),
        (dict(smooth=FAKE + 2, smooth_dtype=d.DQ_F32), d.DQ_ERR_MISALIGNED),
        (dict(y=FAKE + 2, y_dtype=d.DQ_INT32), d.DQ_ERR_MISALIGNED),
        (dict(group_index=FAKE + 2, num_groups=3, smooth=FAKE, workspace=FAKE, workspace_bytes=4),
         d.DQ_ERR_MISALIGNED),
        (dict(group_index=FAKE, num_groups=3, smooth=FAKE, workspace=FAKE + 2, workspace_bytes=4),
         d.DQ_ERR_MISALIGNED),
    ]
    for kw, want in cases:
        assert _dq(d, **kw) == want, kw


def test_ada_workspace_size(dq_lib):
    d = dq_lib
    assert d.dq_ada_layernorm_quant_get_workspace_size(4, 4096, 3072, d.DQ_BF16, d.DQ_BF16) == 4 * 3072 * 8
    assert d.dq_ada_layernorm_quant_get_workspace_size(0, 4096, 3072, d.DQ_BF16, d.DQ_BF16) == 0
    for args, want in [((-1, 2, 8, d.DQ_BF16, d.DQ_BF16), d.DQ_ERR_BAD_SHAPE),
                       ((1, 2, 0, d.DQ_BF16, d.DQ_BF16), d.DQ_ERR_BAD_SHAPE),
                       ((1, 2, 8, d.DQ_F32, d.DQ_BF16), d.DQ_ERR_BAD_DTYPE),
                       ((1, 2, 8, d.DQ_F16, d.DQ_INT8), d.DQ_ERR_BAD_DTYPE)]:
        with pytest.raises(d.DQError) as ei:
            d.dq_ada_layernorm_quant_get_workspace_size(*args)
        assert ei.value.status == want


def _ada(d, **kw):
    a = dict(x=FAKE, x_dtype=d.DQ_BF16, batch=2, seq=3, hidden=64, ada_scale=FAKE, ada_shift=FAKE, weight=None,
             bias=None, smooth=None, param_dtype=d.DQ_BF16, epsilon=1e-6, out=FAKE, quant_scale=FAKE,
             workspace=FAKE, workspace_bytes=2 * 64 * 8, stream=None)
    a.update(kw)
    return d.dq_ada_layernorm_quant(**a)


def test_ada_layernorm_quant_validation(dq_lib):
    d = dq_lib
    assert _ada(d, batch=0, x=None, out=None) == d.DQ_OK
    assert _ada(d, seq=0, x=None, out=None) == d.DQ_OK
    cases = [
        (dict(x=None), d.DQ_ERR_NULL_POINTER),
        (dict(ada_scale=None), d.DQ_ERR_NULL_POINTER),
        (dict(ada_shift=None), d.DQ_ERR_NULL_POINTER),
        (dict(out=None), d.DQ_ERR_NULL_POINTER),
        (dict(quant_scale=None), d.DQ_ERR_NULL_POINTER),
        (dict(batch=-1), d.DQ_ERR_BAD_SHAPE),
        (dict(hidden=0), d.DQ_ERR_BAD_SHAPE),
        (dict(x_dtype=d.DQ_F32), d.DQ_ERR_BAD_DTYPE),
        (dict(param_dtype=d.DQ_INT8), d.DQ_ERR_BAD_DTYPE),
        (dict(epsilon=float("nan")), d.DQ_ERR_BAD_ARGUMENT),
        (dict(epsilon=-1.0), d.DQ_ERR_BAD_ARGUMENT),
        (dict(epsilon=float("inf")), d.DQ_ERR_BAD_ARGUMENT),
        (dict(x=FAKE + 1), d.DQ_ERR_MISALIGNED),
        (dict(quant_scale=FAKE + 2), d.DQ_ERR_MISALIGNED),
        (dict(param_dtype=d.DQ_F32, ada_scale=FAKE + 2), d.DQ_ERR_MISALIGNED),
        (dict(weight=FAKE + 1), d.DQ_ERR_MISALIGNED),
        (dict(workspace=None), d.DQ_ERR_WORKSPACE_TOO_SMALL),
        (dict(workspace_bytes=2 * 64 * 8 - 4), d.DQ_ERR_WORKSPACE_TOO_SMALL),
        (dict(workspace=FAKE + 4), d.DQ_ERR_MISALIGNED),
    ]
    for kw, want in cases:
        assert _ada(d, **kw) == want, kw


def _ada_noalloc(d, **kw):
    args = dict(x=FAKE, x_dtype=d.DQ_BF16, batch=2, seq=8, hidden=64, ada_scale=FAKE, ada_shift=FAKE, weight=None,
                bias=None, smooth=None, param_dtype=d.DQ_BF16, epsilon=1e-6, out=FAKE, quant_scale=FAKE,
                stream=None)
    args.update(kw)
    return d.dq_ada_layernorm_quant_noalloc(**args)


def test_noalloc_checks_follow_the_regular_order(dq_lib):
    """The no-allocation AdaLN entry point validates in the regular entry
    point's order (shapes, epsilon, empty input, pointers), with its array's
    size limit where the regular one checks the workspace; every case here is
    rejected (or empty) on the host, before any CUDA call."""
    d = dq_lib
    too_big = dict(batch=33, seq=1, hidden=4096)  # 33 * 4096 > DQ_ADA_NOALLOC_MAX_TABLE
    cases = [
        (dict(batch=0, epsilon=float("nan")), d.DQ_ERR_BAD_ARGUMENT, d.DQ_ERR_BAD_ARGUMENT),
        (dict(seq=0, epsilon=-1.0), d.DQ_ERR_BAD_ARGUMENT, d.DQ_ERR_BAD_ARGUMENT),
        (dict(batch=0, x=None, out=None), d.DQ_OK, d.DQ_OK),
        (dict(hidden=0, epsilon=float("nan")), d.DQ_ERR_BAD_SHAPE, d.DQ_ERR_BAD_SHAPE),
        (dict(too_big, x=None), d.DQ_ERR_NULL_POINTER, d.DQ_ERR_NULL_POINTER),
        (dict(too_big, quant_scale=None), d.DQ_ERR_NULL_POINTER, d.DQ_ERR_NULL_POINTER),
        (dict(too_big, epsilon=float("inf")), d.DQ_ERR_BAD_ARGUMENT, d.DQ_ERR_BAD_ARGUMENT),
        (dict(too_big), d.DQ_ERR_UNSUPPORTED, d.DQ_ERR_WORKSPACE_TOO_SMALL),
    ]
    for kw, want_noalloc, want_regular in cases:
        assert _ada_noalloc(d, **kw) == want_noalloc, kw
        assert _ada(d, **dict(kw, workspace=None, workspace_bytes=0)) == want_regular, kw


def _deq(d, **kw):
    args = dict(y=FAKE, y_dtype=d.DQ_INT8, rows=4, cols=64, scale=FAKE, offset=None, scale_dtype=d.DQ_F32,
                out=FAKE, out_dtype=d.DQ_BF16, stream=None)
    args.update(kw)
    return d.dq_dequant_per_token(**args)


def test_dequant_per_token_validation(dq_lib):
    """Every invalid call is rejected on the host before any launch."""
    d = dq_lib
    assert _deq(d, rows=0, y=None, out=None) == d.DQ_OK
    cases = [
        (dict(y=None), d.DQ_ERR_NULL_POINTER),
        (dict(scale=None), d.DQ_ERR_NULL_POINTER),
        (dict(out=None), d.DQ_ERR_NULL_POINTER),
        (dict(rows=-1), d.DQ_ERR_BAD_SHAPE),
        (dict(cols=0), d.DQ_ERR_BAD_SHAPE),
        (dict(y_dtype=d.DQ_INT4X2, cols=63), d.DQ_ERR_BAD_SHAPE),
        (dict(y_dtype=d.DQ_INT32, cols=60), d.DQ_ERR_BAD_SHAPE),
        (dict(y_dtype=d.DQ_F16), d.DQ_ERR_BAD_DTYPE),
        (dict(scale_dtype=d.DQ_INT8), d.DQ_ERR_BAD_DTYPE),
        (dict(out_dtype=d.DQ_INT32), d.DQ_ERR_BAD_DTYPE),
        (dict(scale=FAKE + 2), d.DQ_ERR_MISALIGNED),
        (dict(offset=FAKE + 2), d.DQ_ERR_MISALIGNED),
        (dict(out=FAKE + 1), d.DQ_ERR_MISALIGNED),
        (dict(out_dtype=d.DQ_F32, out=FAKE + 2), d.DQ_ERR_MISALIGNED),
        (dict(y_dtype=d.DQ_INT32, y=FAKE + 2), d.DQ_ERR_MISALIGNED),
    ]
    for kw, want in cases:
        assert _deq(d, **kw) == want, kw


def test_dequant_per_group_validation(dq_lib):
    d = dq_lib

    def grp(**kw):
        args = dict(y=FAKE, y_dtype=d.DQ_INT8, rows=64, cols=64, scale=FAKE, offset=None, scale_dtype=d.DQ_F32,
                    group_size=32, k_dim=1, out=FAKE, out_dtype=d.DQ_BF16, stream=None)
        args.update(kw)
        return d.dq_dequant_per_group(**args)

    assert grp(rows=0, y=None, out=None) == d.DQ_OK
    for kw in (dict(group_size=0), dict(group_size=16), dict(group_size=48), dict(group_size=-32), dict(k_dim=2),
               dict(k_dim=-1)):
        assert grp(**kw) == d.DQ_ERR_BAD_ARGUMENT, kw
    assert grp(y=None) == d.DQ_ERR_NULL_POINTER
    assert grp(cols=0) == d.DQ_ERR_BAD_SHAPE
    assert grp(scale=FAKE + 2) == d.DQ_ERR_MISALIGNED


def test_binding_fails_loudly_without_library(tmp_path):
    """The product path has no fallback: without libdq.so the import raises."""
    pkg = os.path.join(ROOT, "token_dynamic_quantization_b200")
    dst = tmp_path / "token_dynamic_quantization_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    code = "import token_dynamic_quantization_b200.dq"
    res = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True)
    assert res.returncode != 0
    assert "ImportError" in res.stderr and "no CPU fallback" in res.stderr


def test_w8a8_gemm_validation(dq_lib):
    """Every invalid W8A8 call is rejected on the host before any launch."""
    d = dq_lib

    def mm(**kw):
        args = dict(a=FAKE, b=FAKE, m=256, n=256, k=256, a_scale=FAKE, b_scale=FAKE, out=FAKE,
                    out_dtype=d.DQ_BF16, accumulate=0, stream=None)
        args.update(kw)
        return d.dq_w8a8_gemm(**args)

    assert mm(m=0, a=None, out=None) == d.DQ_OK  # empty: nothing launched
    assert mm(n=0, b=None, out=None) == d.DQ_OK
    cases = [
        (dict(k=0), d.DQ_ERR_BAD_SHAPE),
        (dict(k=(1 << 17) + 16), d.DQ_ERR_BAD_SHAPE),  # int32 sums could overflow
        (dict(k=1 << 17), d.DQ_ERR_BAD_SHAPE),  # all codes -128: the sum 2^31 does not fit int32
        (dict(m=-1), d.DQ_ERR_BAD_SHAPE),
        (dict(out_dtype=d.DQ_INT8), d.DQ_ERR_BAD_DTYPE),
        (dict(accumulate=2), d.DQ_ERR_BAD_ARGUMENT),
        (dict(accumulate=1), d.DQ_ERR_BAD_ARGUMENT),  # the in-place add needs an f32 out
        (dict(a=None), d.DQ_ERR_NULL_POINTER),
        (dict(b_scale=None), d.DQ_ERR_NULL_POINTER),
        (dict(a_scale=FAKE + 2), d.DQ_ERR_MISALIGNED),
        (dict(out=FAKE + 1), d.DQ_ERR_MISALIGNED),
        (dict(out_dtype=d.DQ_F32, out=FAKE + 2), d.DQ_ERR_MISALIGNED),
    ]
    for kw, want in cases:
        assert mm(**kw) == want, kw


def test_w8a8_helper_checks_shapes_on_the_host(dq_lib):
    import torch

    a = torch.zeros(4, 32, dtype=torch.int8)
    with pytest.raises(ValueError):
        dq_lib.w8a8_gemm(a, torch.zeros(8, 16, dtype=torch.int8), torch.ones(4), torch.ones(8))
    with pytest.raises(TypeError):
        dq_lib.w8a8_gemm(a, torch.zeros(8, 32, dtype=torch.int8), torch.ones(3), torch.ones(8))
    with pytest.raises(TypeError):
        dq_lib.w8a8_gemm(a.float(), torch.zeros(8, 32, dtype=torch.int8), torch.ones(4), torch.ones(8))


C_PROGRAM = r"""
#include <stdio.h>
#include "dq.h"

int main(void) {
  size_t bytes = 123;
  /* host-only calls: argument validation and the workspace query */
  if (dq_get_workspace_size(32768, 7168, DQ_BF16, DQ_SYMMETRIC, DQ_INT8, 64, &bytes) != DQ_OK || bytes != 4) return 1;
  if (dq_get_workspace_size(4, 7, DQ_F16, DQ_SYMMETRIC, DQ_INT4X2, 0, &bytes) != DQ_ERR_BAD_SHAPE) return 2;
  if (dq_w8a8_gemm(NULL, NULL, 0, 16, 32, NULL, NULL, NULL, DQ_BF16, 0, 0) != DQ_OK) return 3;
  if (dq_w8a8_gemm(NULL, NULL, 16, 16, 32, NULL, NULL, NULL, DQ_BF16, 0, 0) != DQ_ERR_NULL_POINTER) return 4;
  printf("%s|%s\n", dq_status_string(DQ_OK), dq_status_string(DQ_ERR_MISALIGNED));
  return 0;
}
"""


def test_plain_c_program_uses_the_header_and_library(dq_lib, tmp_path):
    """include/dq.h is plain C (no C++ types in the signatures): a C program
    compiles against it with gcc, links libdq.so and runs its host-side calls
    (no device needed)."""
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no gcc")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(dq_lib.LIBRARY_PATH)
    build = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
                            str(src), "-L", lib_dir, "-l:libdq.so", "-Wl,-rpath," + lib_dir, "-o", str(exe)],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, (run.returncode, run.stderr)
    ok, mis = run.stdout.strip().split("|")
    assert ok == dq_lib.dq_status_string(dq_lib.DQ_OK)
    assert mis == dq_lib.dq_status_string(dq_lib.DQ_ERR_MISALIGNED)
