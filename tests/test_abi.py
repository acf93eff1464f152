"""The C-ABI library loads without a GPU, exports every symbol include/muon.h
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from newton_schulz_12_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon.h")


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(muon_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return _lib.lib()


def test_header_lists_the_boundary():
    names = declared_functions()
    for required in ("muon_ns_orthogonalize", "muon_step", "muon_get_status", "muon_last_error"):
        assert required in names
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_kernel_kinds_match_the_header():
    """The binding's names for muon_profile_end's slots follow the header's enum."""
    with open(HEADER) as f:
        text = f.read()
    kinds = dict((name, int(v)) for name, v in re.findall(r"MUON_KERNEL_([A-Z_]+)\s*=\s*(\d+)", text))
    count = kinds.pop("KINDS")
    assert count == len(_lib.KERNEL_KINDS)
    assert sorted(kinds.values()) == list(range(count))
    for name, v in kinds.items():
        assert _lib.KERNEL_KINDS[v] == name.lower(), name


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_build_targets_sm100a_only():
    from newton_schulz_12_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert os.path.exists(_lib.LIB_PATH)


def test_version(lib):
    assert lib.muon_version() == 100


def _err(lib):
    return lib.muon_last_error().decode()


def test_argument_errors_need_no_device(lib):
    null = ctypes.c_void_p(0)
    # negative batch, too many steps, unknown dtype, bad shape, null array
    assert lib.muon_ns_orthogonalize(-1, 4, 4, None, 1.0, 0.0, 0.0, 5, 0, null) == -1
    assert "batch" in _err(lib)
    assert lib.muon_ns_orthogonalize(1, 4, 4, None, 1.0, 0.0, 0.0, 101, 0, null) == -1
    assert lib.muon_ns_orthogonalize(1, 4, 4, None, 1.0, 0.0, 0.0, 5, 7, null) == -1
    assert lib.muon_ns_orthogonalize(1, 0, 4, None, 1.0, 0.0, 0.0, 5, 0, null) == -2
    assert lib.muon_ns_orthogonalize(1, 4, 40000, None, 1.0, 0.0, 0.0, 5, 0, null) == -2
    assert lib.muon_ns_orthogonalize(1, 4, 4, None, 1.0, 0.0, 0.0, 5, 0, null) == -1
    assert lib.muon_ns_orthogonalize(1, 4, 4, None, float("nan"), 0.0, 0.0, 5, 0, null) == -1
    # misaligned / null device pointers are caught on the host
    arr = _lib.ptr_array([0x1001])
    assert lib.muon_ns_orthogonalize(1, 4, 4, arr, 1.0, 0.0, 0.0, 5, 0, null) == -1
    assert "aligned" in _err(lib)
    arr = _lib.ptr_array([0])
    assert lib.muon_ns_orthogonalize(1, 4, 4, arr, 1.0, 0.0, 0.0, 5, 0, null) == -1
    assert "NULL" in _err(lib)
    # batch 0 is a no-op that succeeds without a device
    assert lib.muon_ns_orthogonalize(0, 4, 4, None, 1.0, 0.0, 0.0, 5, 0, null) == 0


def test_schedule_argument_errors(lib):
    null = ctypes.c_void_p(0)
    table = (ctypes.c_float * 6)(3.4445, -4.775, 2.0315, 1.5, -0.5, 0.0)
    bad = (ctypes.c_float * 6)(3.4445, -4.775, 2.0315, 1.5, float("inf"), 0.0)
    arr = _lib.ptr_array([0x1000])
    assert lib.muon_ns_orthogonalize_schedule(1, 4, 4, arr, None, 2, 0, null) == -1
    assert "table" in _err(lib)
    assert lib.muon_ns_orthogonalize_schedule(1, 4, 4, arr, bad, 2, 0, null) == -1
    assert "step 1" in _err(lib)
    assert lib.muon_ns_orthogonalize_schedule(1, 4, 4, arr, table, 101, 0, null) == -1
    assert lib.muon_ns_orthogonalize_schedule(1, 4, 4, arr, table, 2, 9, null) == -1
    # no steps: the table may be NULL; batch 0 is a no-op without a device
    assert lib.muon_ns_orthogonalize_schedule(0, 4, 4, None, None, 0, 0, null) == 0
    assert lib.muon_ns_orthogonalize_schedule(0, 4, 4, None, table, 2, 0, null) == 0


def test_step_argument_errors(lib):
    null = ctypes.c_void_p(0)
    p = _lib.ptr_array([0x1000])
    shapes = _lib.shape_array([(4, 4)])
    assert lib.muon_step(-1, p, p, p, shapes, 0.9, 1, 0.1, 0.0, 5, null) == -1
    assert lib.muon_step(0, None, None, None, None, 0.9, 1, 0.1, 0.0, 5, null) == 0
    assert lib.muon_step(1, None, p, p, shapes, 0.9, 1, 0.1, 0.0, 5, null) == -1
    assert lib.muon_step(1, p, p, p, shapes, 1.5, 1, 0.1, 0.0, 5, null) == -1
    assert "beta" in _err(lib)
    assert lib.muon_step(1, p, p, p, shapes, 0.9, 1, float("inf"), 0.0, 5, null) == -1
    bad = _lib.shape_array([(4, -3)])
    assert lib.muon_step(1, p, p, p, bad, 0.9, 1, 0.1, 0.0, 5, null) == -2
    assert "shape" in _err(lib)
    mis = _lib.ptr_array([0x1008])
    assert lib.muon_step(1, p, mis, p, shapes, 0.9, 1, 0.1, 0.0, 5, null) == -1
    assert "grads[0]" in _err(lib)
    assert lib.muon_momentum(1, p, p, shapes, -0.1, 1, None, null) == -1
    assert lib.muon_apply(1, p, None, shapes, 0.1, 0.0, null) == -1
    # the extended step and apply: unknown option bits, beta2, state pointers
    assert lib.muon_step_ex(1, p, p, p, shapes, 0.9, 1, 0.1, 0.0, 5, None, 2, None, 0.95, null) == -1
    assert "flags" in _err(lib)
    assert lib.muon_step_ex(1, p, p, p, shapes, 0.9, 1, 0.1, 0.0, 5, None, 1, p, 1.5, null) == -1
    assert "beta2" in _err(lib)
    assert lib.muon_step_ex(1, p, p, p, shapes, 0.9, 1, 0.1, 0.0, 5, None, 0, _lib.ptr_array([0]), 0.95, null) == -1
    assert "neuron_state[0]" in _err(lib)
    assert lib.muon_step_ex(0, None, None, None, None, 0.9, 1, 0.1, 0.0, 5, None, 1, None, 0.95, null) == 0
    sched = (ctypes.c_float * 15)(*([1.5, -0.5, 0.0] * 4 + [1.5, float("nan"), 0.0]))
    assert lib.muon_step_ex(1, p, p, p, shapes, 0.9, 1, 0.1, 0.0, 5, sched, 0, None, 0.95, null) == -1
    assert "coefficient 1 of step 4" in _err(lib)
    assert lib.muon_apply_ex(1, p, p, shapes, 0.1, 0.0, 8, None, null) == -1
    assert lib.muon_apply_ex(1, p, p, shapes, 0.1, 0.0, 1, _lib.ptr_array([0x1002]), null) == -1
    assert "row_scale[0]" in _err(lib)


def test_stage_argument_errors(lib):
    null = ctypes.c_void_p(0)
    assert lib.muon_gram_bf16(1, 8, 8, None, None, null) == -1
    assert lib.muon_poly_bf16(1, 8, 0x1000, 0x1000, 1.0, 1.0, null) == -1  # aliasing
    assert lib.muon_bx_bf16(1, 8, 8, 0x1000, 0x2000, 0x3000, 0x2000, 1.0, null) == -1
    # the int8 low part needs 16-byte rows: n a multiple of 16
    assert lib.muon_bx_bf16(1, 8, 24, 0x1000, 0x2000, 0x3000, 0x4000, 1.0, null) == -2
    assert "multiple of 16" in _err(lib)
    assert lib.muon_gram_bf16(0, 8, 8, None, None, null) == 0
    # fused last product + apply: strides, shape order and pointers are checked on the host
    w = _lib.ptr_array([0x1000])
    assert lib.muon_bx_apply_bf16(1, 8, 24, 24, 0x1000, 8, 0x2000, 0x3000, w, 0, 1.0, 0.1, 0.0, 0, null) == -2
    assert "ldx" in _err(lib)
    assert lib.muon_bx_apply_bf16(1, 8, 24, 32, 0x1000, 4, 0x2000, 0x3000, w, 0, 1.0, 0.1, 0.0, 0, null) == -2
    assert lib.muon_bx_apply_bf16(1, 32, 16, 16, 0x1000, 32, 0x2000, 0x3000, w, 0, 1.0, 0.1, 0.0, 0, null) == -2
    assert lib.muon_bx_apply_bf16(1, 8, 24, 32, 0x1000, 8, 0x2000, 0x3008, w, 0, 1.0, 0.1, 0.0, 0, null) == -1
    assert lib.muon_bx_apply_bf16(1, 8, 24, 32, 0x1000, 8, 0x2000, 0x3000, None, 0, 1.0, 0.1, 0.0, 0, null) == -1
    assert lib.muon_bx_apply_bf16(1, 8, 24, 32, 0x1000, 8, 0x2000, 0x3000, w, 0, 1.0, float("nan"), 0.0,
                                  0, null) == -1
    assert lib.muon_bx_apply_bf16(1, 8, 32, 32, 0x1000, 8, 0x2000, 0x3000, w, 0, 1.0, 0.1, 0.0, 4, null) == -1
    assert "flags" in _err(lib)
    assert lib.muon_bx_apply_bf16(0, 8, 24, 32, None, 8, None, None, None, 0, 1.0, 0.1, 0.0, 0, null) == 0


def test_setters(lib):
    assert lib.muon_set_wait_timeout_ms(0) == -1
    assert lib.muon_set_wait_timeout_ms(2000) == 0
    assert lib.muon_set_fault_injection(5) == -1
    assert lib.muon_set_fault_injection(0) == 0


def test_python_binding_rejects_cpu_tensors():
    import torch
    import newton_schulz_12_b200 as nsb
    with pytest.raises(ValueError):
        nsb.muon_ns_orthogonalize([torch.zeros(4, 4)])
    with pytest.raises(ValueError):
        nsb.muon_step([torch.zeros(4, 4)], [torch.zeros(4, 4, dtype=torch.bfloat16)],
                      [torch.zeros(4, 4)])


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "muon.h"
int main(void) {
  if (muon_version() != 100) return 1;
  /* argument errors come back synchronously, before any device work */
  if (muon_ns_orthogonalize(-1, 8, 8, NULL, 3.4445f, -4.775f, 2.0315f, 5, MUON_BF16, NULL) != MUON_ERR_ARG)
    return 2;
  if (strlen(muon_last_error()) == 0) return 3;
  if (muon_step(-1, NULL, NULL, NULL, NULL, 0.95f, 1, 0.05f, 0.0f, 5, NULL) != MUON_ERR_ARG) return 4;
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c11"), ("g++", "-std=c++17")])
def test_plain_c_client_builds_and_runs(tmp_path, compiler, std):
    """The header compiles on its own as C11 and C++17 (no CUDA headers) and a
    program linked against the library gets its version and its synchronous
    argument errors without a GPU."""
    import shutil
    import subprocess
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not available")
    src = tmp_path / ("client.c" if compiler == "gcc" else "client.cpp")
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(_lib.LIB_PATH)
    libname = os.path.basename(_lib.LIB_PATH)
    subprocess.run([compiler, std, "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(exe), os.path.join(libdir, libname), f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)
