"""The C ABI library on the host: it loads without a GPU, exports every entry
point the header declares, its struct layouts match the Python mirror, and
host-side validation rejects bad arguments before touching CUDA."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from block_sparse_linear_mean_b200 import sla, synth
from block_sparse_linear_mean_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sla.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return sla.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SLA_API\s+[\w\s\*]+?\b(sla_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(sla.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", sla._LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (sla_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_library_has_no_libcuda_dependency(lib):
    # the runtime is linked statically and the driver is never linked, so the
    # library loads on a host without a GPU driver
    out = subprocess.run(["ldd", sla._LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_struct_layout_matches_c_compiler(lib, tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(f'''#include <stdio.h>
#include <stddef.h>
#include "{HEADER}"
int main(void) {{
  printf("%zu %zu %zu %zu %zu %zu %zu\\n", sizeof(sla_params),
         offsetof(sla_params, frac_crit), offsetof(sla_params, thr),
         offsetof(sla_params, scale), offsetof(sla_params, flags),
         sizeof(sla_block_lists), offsetof(sla_block_lists, marg_idx));
  return 0;
}}
''')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", str(src), "-o", str(exe)], check=True)
    got = list(map(int, subprocess.run([str(exe)], capture_output=True, text=True,
                                       check=True).stdout.split()))
    P, L = sla.sla_params, sla.sla_block_lists
    assert got == [ctypes.sizeof(P), P.frac_crit.offset, P.thr.offset, P.scale.offset,
                   P.flags.offset, ctypes.sizeof(L), L.marg_idx.offset]


def test_abi_version_and_status_strings(lib):
    assert sla.sla_abi_version() == 1
    for st in range(6):
        assert sla.status_string(st)
    assert sla.status_string(99) == "unknown status"


def good_params(**kw):
    p = sla.params_for(synth.WORKLOADS["sla_1p3b"])
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("field,value,expect", [
    ("N", 0, sla.SLA_ERR_INVALID_ARG),
    ("H", -1, sla.SLA_ERR_INVALID_ARG),
    ("d", 96, sla.SLA_ERR_UNSUPPORTED),
    ("block_q", 32, sla.SLA_ERR_UNSUPPORTED),
    ("dtype", 7, sla.SLA_ERR_INVALID_ARG),
    ("mask_mode", 3, sla.SLA_ERR_INVALID_ARG),
    ("frac_crit", 1.5, sla.SLA_ERR_INVALID_ARG),
    ("frac_marg", -0.1, sla.SLA_ERR_INVALID_ARG),
    ("frac_marg", 0.96, sla.SLA_ERR_INVALID_ARG),   # 0.05 + 0.96 > 1
    ("scale", float("nan"), sla.SLA_ERR_INVALID_ARG),
    ("flags", 8, sla.SLA_ERR_INVALID_ARG),
    # a withheld-load selector without the debug flag, or past the last kernel
    ("flags", sla.SLA_DEBUG_WITHHOLD(sla.SLA_WITHHOLD_GATHER), sla.SLA_ERR_INVALID_ARG),
    ("flags", sla.SLA_FLAG_DEBUG_TIMEOUT | sla.SLA_DEBUG_WITHHOLD(6), sla.SLA_ERR_INVALID_ARG),
    ("flags", 1 << 12, sla.SLA_ERR_INVALID_ARG),
])
def test_validation_rejects(lib, field, value, expect):
    assert sla.sla_validate(good_params(**{field: value})) == expect


def test_validation_accepts_every_withheld_load_selector(lib):
    for kernel in range(sla.SLA_WITHHOLD_BWD_DKDV + 1):
        flags = sla.SLA_FLAG_DEBUG_TIMEOUT | sla.SLA_DEBUG_WITHHOLD(kernel)
        assert sla.sla_validate(good_params(flags=flags)) == sla.SLA_OK


def test_validation_cdf_threshold_range(lib):
    p = sla.params_for(synth.WORKLOADS["nabla_14b"])
    assert sla.sla_validate(p) == sla.SLA_OK
    p.thr = 1.0
    assert sla.sla_validate(p) == sla.SLA_ERR_INVALID_ARG
    p.thr = 0.0
    assert sla.sla_validate(p) == sla.SLA_OK


def test_all_workloads_validate_and_size(lib):
    for name, wl in synth.WORKLOADS.items():
        p = sla.params_for(wl)
        assert sla.sla_validate(p) == sla.SLA_OK, name
        for op in (sla.SLA_OP_MASK, sla.SLA_OP_FORWARD, sla.SLA_OP_BACKWARD):
            n = sla.sla_workspace_size(p, op)
            assert n >= 256 and n % 256 == 0


def test_workspace_size_bad_op(lib):
    with pytest.raises(sla.SlaError):
        sla.sla_workspace_size(good_params(), 9)


def test_null_pointers_rejected_before_any_cuda_call(lib):
    p = good_params()
    lists = sla.sla_block_lists(0, 0, 0, 0)
    assert sla.sla_build_mask(p, None, None, None, lists, None, None, None, None, 0,
                              None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_forward(p, None, None, None, None, lists, None, None, None, None,
                           None, 0, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_backward(p, None, None, None, None, None, lists, lists, None, None,
                            None, None, None, None, None, None, 0,
                            None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_mask_lists(p, None, None, None, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_block_importance(p, None, None, None, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_mask_recall(p, None, None, None, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_check_device_status(None, None) == sla.SLA_ERR_INVALID_ARG


def test_misaligned_pointer_rejected(lib):
    # 16-byte alignment is checked on the host; a misaligned (never
    # dereferenced) address is refused before anything is enqueued
    p = good_params()
    lists = sla.sla_block_lists(16, 16, 16, 16)
    st = sla.sla_build_mask(p, 16, 24, 16, lists, None, None, None, 16, 1 << 40, None)
    assert st == sla.SLA_ERR_INVALID_ARG


def test_mask_quality_entry_points_validate_on_the_host(lib):
    p = good_params()
    # misaligned (never dereferenced) addresses
    assert sla.sla_block_importance(p, 16, 24, 16, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_mask_recall(p, 16, 16, 20, None) == sla.SLA_ERR_INVALID_ARG
    # an invalid parameter block is refused before the pointers are looked at
    bad = good_params()
    bad.d = 96
    assert sla.sla_block_importance(bad, 16, 16, 16, None) == sla.SLA_ERR_UNSUPPORTED
    assert sla.sla_mask_recall(bad, 16, 16, 16, None) == sla.SLA_ERR_UNSUPPORTED


def test_tile_order_entry_points_validate_on_the_host(lib):
    # sizes and pointers are checked before anything is enqueued (the
    # addresses below are never dereferenced)
    assert sla.sla_tile_order(0, 4, 4, 1, 1, 1, 16, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_tile_order(2, 4, 4, 1, 0, 1, 16, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_tile_order(2, 4, 4, 1, 1, 1, None, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_tile_order(2, 4, 4, 1, 1, 1, 18, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_tile_order(1 << 11, 1 << 10, 1 << 10, 1, 1, 1, 16,
                              None) == sla.SLA_ERR_UNSUPPORTED
    p = good_params()
    big = 1 << 40
    assert sla.sla_permute_tokens(p, 16, big, 16, 3, 0, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_permute_tokens(p, 16, big, 16, 2, 2, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_permute_tokens(p, 24, big, 16, 2, 0, None) == sla.SLA_ERR_INVALID_ARG
    assert sla.sla_permute_tokens(p, 16, big, 18, 2, 0, None) == sla.SLA_ERR_INVALID_ARG
    # overlapping source and destination
    assert sla.sla_permute_tokens(p, 1 << 20, (1 << 20) + 4096, 16, 2, 0,
                                  None) == sla.SLA_ERR_INVALID_ARG


def test_workspace_too_small_rejected(lib):
    p = good_params()
    lists = sla.sla_block_lists(16, 16, 16, 16)
    st = sla.sla_build_mask(p, 16, 16, 16, lists, None, None, None, 16, 255, None)
    assert st == sla.SLA_ERR_WORKSPACE
