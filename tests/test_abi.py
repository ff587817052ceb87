"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and rejects bad arguments on the host before touching CUDA."""

import ctypes
import os
import re
import subprocess

import pytest

from mla_decode_attention_13_b200 import binding
from mla_decode_attention_13_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla_b200.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(mla_[a-z0-9_]+)\s*\(", text, re.M)))


def test_header_declares_the_expected_calls():
    assert declared_functions() == sorted(binding.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    nm = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s+(mla_\w+)", nm))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_library_has_no_driver_link_dependency(lib):
    # The CUDA driver is resolved at run time; the library must load on a
    # machine without a GPU driver (it only links the static runtime).
    ldd = subprocess.run(["ldd", binding.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in ldd


def test_error_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, 7):
        assert isinstance(binding.mla_error_string(code), str) and binding.mla_error_string(code)


def test_metadata_bytes(lib):
    assert binding.mla_metadata_bytes(0, 16, 1) == 0
    assert binding.mla_metadata_bytes(1, 0, 1) == 0
    assert binding.mla_metadata_bytes(1, 129, 1) == 0
    assert binding.mla_metadata_bytes(1, 16, 17) == 0
    a = binding.mla_metadata_bytes(16, 128, 1)
    b = binding.mla_metadata_bytes(64, 128, 1)
    c = binding.mla_metadata_bytes(64, 128, 2)  # two m-tiles per batch row
    assert 0 < a < b < c and a % 16 == 0


def test_workspace_bytes_bound_without_device(lib):
    # Without a device the bound for the largest part (160 pairs) is returned:
    # 2 * (160 - 1) slots of min(R, 128) rows x (512 + 1) fp32.
    n = binding.mla_workspace_bytes(16, 128, 1)
    assert n >= 2 * 159 * 128 * 513 * 4 or n == 2 * 73 * 128 * 513 * 4
    assert binding.mla_workspace_bytes(4, 16, 1) < n
    assert binding.mla_workspace_bytes(0, 16, 1) == 0


def _decode_args(**over):
    a = dict(q=16, kv=16, num_pages=4, table=16, max_pages=4, seqlens=16, batch=1, s_q=1, h_q=16, scale=0.07,
             causal=0, out=16, lse=16, meta=16, ws=16, ws_bytes=1 << 30, stream=None)
    a.update(over)
    return [a["q"], a["kv"], a["num_pages"], a["table"], a["max_pages"], a["seqlens"], a["batch"], a["s_q"],
            a["h_q"], a["scale"], a["causal"], a["out"], a["lse"], a["meta"], a["ws"], a["ws_bytes"], a["stream"]]


@pytest.mark.parametrize("over,status", [
    (dict(q=None), binding.MLA_ERR_ARG),
    (dict(kv=None), binding.MLA_ERR_ARG),
    (dict(table=None), binding.MLA_ERR_ARG),
    (dict(seqlens=None), binding.MLA_ERR_ARG),
    (dict(out=None), binding.MLA_ERR_ARG),
    (dict(lse=None), binding.MLA_ERR_ARG),
    (dict(meta=None), binding.MLA_ERR_ARG),
    (dict(q=24), binding.MLA_ERR_ARG),            # misaligned for TMA
    (dict(kv=8), binding.MLA_ERR_ARG),
    (dict(out=2), binding.MLA_ERR_ARG),
    (dict(batch=0), binding.MLA_ERR_ARG),
    (dict(h_q=0), binding.MLA_ERR_ARG),
    (dict(s_q=0), binding.MLA_ERR_ARG),
    (dict(max_pages=0), binding.MLA_ERR_ARG),
    (dict(num_pages=0), binding.MLA_ERR_ARG),
    (dict(causal=2), binding.MLA_ERR_ARG),
    (dict(scale=float("nan")), binding.MLA_ERR_ARG),
    (dict(scale=float("inf")), binding.MLA_ERR_ARG),
    (dict(scale=-0.1), binding.MLA_ERR_ARG),
    (dict(h_q=129), binding.MLA_ERR_UNSUPPORTED),
    (dict(s_q=17), binding.MLA_ERR_UNSUPPORTED),
    (dict(num_pages=(1 << 25) + 1), binding.MLA_ERR_UNSUPPORTED),
])
def test_decode_rejects_bad_arguments_on_host(lib, over, status):
    assert lib.mla_decode(*_decode_args(**over)) == status
    assert lib.mla_decode_timed(*_decode_args(**over), None, None) == status


def test_get_metadata_rejects_bad_arguments_on_host(lib):
    assert lib.mla_get_metadata(None, 1, 16, 1, 16, None) == binding.MLA_ERR_ARG
    assert lib.mla_get_metadata(16, 1, 16, 1, None, None) == binding.MLA_ERR_ARG
    assert lib.mla_get_metadata(16, 0, 16, 1, 16, None) == binding.MLA_ERR_ARG
    assert lib.mla_get_metadata(16, 1, 16, 1, 8, None) == binding.MLA_ERR_ARG
    assert lib.mla_get_metadata(16, 1, 200, 1, 16, None) == binding.MLA_ERR_UNSUPPORTED


def test_check_device_error_rejects_null(lib):
    w = ctypes.c_uint32(0)
    assert lib.mla_check_device_error(None, None, ctypes.byref(w)) == binding.MLA_ERR_ARG


@pytest.mark.parametrize("args,status", [
    ((None, 16, 16, 4, 16, 16), binding.MLA_ERR_ARG),   # q_nope
    ((16, None, 16, 4, 16, 16), binding.MLA_ERR_ARG),   # q_rope
    ((16, 16, None, 4, 16, 16), binding.MLA_ERR_ARG),   # w_uk
    ((16, 16, 16, 4, 16, None), binding.MLA_ERR_ARG),   # q_out
    ((24, 16, 16, 4, 16, 16), binding.MLA_ERR_ARG),     # misaligned for TMA
    ((16, 8, 16, 4, 16, 16), binding.MLA_ERR_ARG),
    ((16, 16, 16, 4, 16, 40), binding.MLA_ERR_ARG),
    ((16, 16, 16, 0, 16, 16), binding.MLA_ERR_ARG),     # tokens
    ((16, 16, 16, 4, 0, 16), binding.MLA_ERR_ARG),      # h_q
    ((16, 16, 16, 4, 129, 16), binding.MLA_ERR_UNSUPPORTED),
    ((16, 16, 16, 65535 * 128 + 1, 16, 16), binding.MLA_ERR_UNSUPPORTED),
])
def test_absorb_q_rejects_bad_arguments_on_host(lib, args, status):
    assert lib.mla_absorb_q(*args, None) == status


@pytest.mark.parametrize("args,status", [
    ((None, 16, 4, 16, 16), binding.MLA_ERR_ARG),
    ((16, None, 4, 16, 16), binding.MLA_ERR_ARG),
    ((16, 16, 4, 16, None), binding.MLA_ERR_ARG),
    ((16, 32 + 8, 4, 16, 16), binding.MLA_ERR_ARG),
    ((16, 16, -1, 16, 16), binding.MLA_ERR_ARG),
    ((16, 16, 4, 0, 16), binding.MLA_ERR_ARG),
    ((16, 16, 4, 200, 16), binding.MLA_ERR_UNSUPPORTED),
    ((16, 16, 65535 * 64 + 1, 16, 16), binding.MLA_ERR_UNSUPPORTED),  # token tiles past the grid's limit
])
def test_up_project_rejects_bad_arguments_on_host(lib, args, status):
    assert lib.mla_up_project(*args, None) == status


@pytest.mark.parametrize("args,status", [
    ((None, 16, 2, 1, 1, 16, 16, 16), binding.MLA_ERR_ARG),
    ((16, None, 2, 1, 1, 16, 16, 16), binding.MLA_ERR_ARG),
    ((16, 16, 2, 1, 1, 16, None, 16), binding.MLA_ERR_ARG),
    ((16, 16, 2, 1, 1, 16, 16, None), binding.MLA_ERR_ARG),
    ((8, 16, 2, 1, 1, 16, 16, 16), binding.MLA_ERR_ARG),   # misaligned
    ((16, 16, 2, 1, 1, 16, 24, 16), binding.MLA_ERR_ARG),
    ((16, 16, 0, 1, 1, 16, 16, 16), binding.MLA_ERR_ARG),  # splits
    ((16, 16, 2, 0, 1, 16, 16, 16), binding.MLA_ERR_ARG),
    ((16, 16, 2, 1, 0, 16, 16, 16), binding.MLA_ERR_ARG),
    ((16, 16, 2, 1, 1, 0, 16, 16), binding.MLA_ERR_ARG),
    ((16, 16, 2, 1, 1, 129, 16, 16), binding.MLA_ERR_UNSUPPORTED),
    ((16, 16, 2, 1, 17, 16, 16, 16), binding.MLA_ERR_UNSUPPORTED),
])
def test_merge_splits_rejects_bad_arguments_on_host(lib, args, status):
    assert lib.mla_merge_splits(*args, None) == status


def test_binding_checks_projection_and_merge_shapes_before_the_library(lib):
    # Shape and dtype errors are raised by the binding itself (MLA_ERR_ARG),
    # before any pointer reaches the library; CPU tensors suffice.
    import torch

    bf = torch.bfloat16
    w = torch.zeros(4, 512, 128, dtype=bf)
    cases = [
        lambda: binding.mla_absorb_q(torch.zeros(2, 4, 127, dtype=bf), torch.zeros(2, 4, 64, dtype=bf), w),
        lambda: binding.mla_absorb_q(torch.zeros(2, 4, 128, dtype=bf), torch.zeros(2, 4, 32, dtype=bf), w),
        lambda: binding.mla_absorb_q(torch.zeros(2, 4, 128), torch.zeros(2, 4, 64, dtype=bf), w),
        lambda: binding.mla_absorb_q(torch.zeros(2, 3, 128, dtype=bf), torch.zeros(2, 3, 64, dtype=bf), w),
        lambda: binding.mla_up_project(torch.zeros(2, 4, 511, dtype=bf), w),
        lambda: binding.mla_up_project(torch.zeros(2, 4, 512, dtype=bf), w.transpose(1, 2)),
        lambda: binding.mla_up_project(torch.zeros(2, 4, 512, dtype=bf), w, out=torch.zeros(2, 4, 64, dtype=bf)),
        lambda: binding.mla_merge_splits(torch.zeros(2, 1, 1, 4, 512, dtype=bf), torch.zeros(2, 1, 1, 4)),
        lambda: binding.mla_merge_splits(torch.zeros(2, 1, 1, 4, 512), torch.zeros(2, 1, 4, 1)),
        lambda: binding.mla_merge_splits(torch.zeros(1, 4, 512, dtype=bf), torch.zeros(1, 4)),
    ]
    for k, call in enumerate(cases):
        with pytest.raises(binding.MLAError) as e:
            call()
        assert e.value.status == binding.MLA_ERR_ARG, k
