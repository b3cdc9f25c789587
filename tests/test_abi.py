"""The C-ABI library loads on a machine without a GPU and exports every symbol
include/pa.h declares; the Python binding declares exactly those signatures.
No device entry point is called here."""
import os
import re
import subprocess

import pytest

from paged_kv_cache_356_b200 import _lib, binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "pa.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("pa_reshape_and_cache", "pa_decode", "pa_decode_workspace_size", "pa_copy_blocks",
                     "pa_block_alloc_create", "pa_block_alloc_allocate_sequence", "pa_block_alloc_append_token",
                     "pa_block_alloc_fork", "pa_block_alloc_free_sequence", "pa_block_alloc_destroy"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert set(_declared()) <= exported
    # no C entry point beyond the header
    assert {s for s in exported if s.startswith("pa_")} == set(_declared())


def test_binding_signatures_cover_the_header():
    assert set(_lib.SIGNATURES) == set(_declared())


def test_library_needs_no_cuda_runtime_shared_object():
    out = subprocess.run(["ldd", _lib.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out


def test_version_and_error_strings():
    assert "sm_100a" in binding.pa_version()
    with pytest.raises(binding.PagedAttentionError):
        binding.pa_block_alloc_create(-1, 16)
    assert "num_blocks" in _lib.last_error()


def test_workspace_size_matches_documented_layout():
    # one partition needs no workspace; P partitions need three 256-byte aligned arrays
    assert binding.pa_decode_workspace_size(4, 8, 128, 512) == 0
    p = 16
    rows = 256 * 64 * p
    align = lambda x: (x + 255) // 256 * 256  # noqa: E731
    expect = align(rows * 128 * 4) + 2 * align(rows * 4)
    assert binding.pa_decode_workspace_size(256, 64, 128, 8192) == expect
    assert binding.pa_decode_workspace_size(3, 5, 64, 1025) == align(3 * 5 * 3 * 64 * 4) + 2 * align(3 * 5 * 3 * 4)


def test_device_calls_reject_cpu_tensors():
    import torch
    kc = torch.zeros(2, 1, 16, 64)
    with pytest.raises(TypeError):
        binding.pa_reshape_and_cache(torch.zeros(1, 1, 64), torch.zeros(1, 1, 64), torch.zeros(1, dtype=torch.int64),
                                     kc, kc.clone())
    with pytest.raises(TypeError):
        binding.pa_copy_blocks(kc, kc.clone(), torch.zeros(1, 2, dtype=torch.int64))


def test_verify_workspace_size_matches_documented_layout():
    """The pa_decode partials with T * H_q heads per sequence, then the joint kernel's plan arrays and
    the merge's item list (a count, then one int32 per query row)."""
    align = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert binding.pa_decode_verify_workspace_size(4, 3, 8, 128, 512) == 0          # one partition
    assert binding.pa_decode_verify_workspace_size(4, 0, 8, 128, 4096) == 0         # no query token
    b, t, hq, d, ctx = 256, 4, 64, 128, 8192
    parts = binding.pa_decode_workspace_size(b, t * hq, d, ctx)
    assert binding.pa_decode_verify_workspace_size(b, t, hq, d, ctx) == (
        parts + align(16 * b * t) + align(4 * b * t) + align(4 * (1 + b * t * hq)))
    assert binding.pa_decode_verify_workspace_size(3, 7, 5, 64, 1025) == (
        binding.pa_decode_workspace_size(3, 35, 64, 1025) + align(16 * 21) + align(4 * 21) + align(4 * (1 + 21 * 5)))


def test_verify_and_pool_setters_validate_on_the_host():
    with pytest.raises(binding.PagedAttentionError):
        binding.pa_set_verify_path(7)
    with pytest.raises(binding.PagedAttentionError):
        binding.pa_set_verify_tiling(12)
    binding.pa_set_verify_path(binding.PA_VERIFY_AUTO)
    binding.pa_set_verify_tiling(0)


def test_verify_rejects_cpu_tensors_and_bad_shapes():
    import torch
    kc = torch.zeros(2, 1, 16, 64, dtype=torch.bfloat16)
    tables = torch.zeros(1, 2, dtype=torch.int32)
    ctx = torch.ones(1, dtype=torch.int32)
    with pytest.raises(ValueError):   # 3-D q
        binding.pa_decode_verify(torch.zeros(1, 4, 64, dtype=torch.bfloat16), kc, kc.clone(), tables, ctx, 0.1)
    with pytest.raises(TypeError):    # host tensors
        binding.pa_decode_verify(torch.zeros(1, 2, 4, 64, dtype=torch.bfloat16), kc, kc.clone(), tables, ctx, 0.1)
