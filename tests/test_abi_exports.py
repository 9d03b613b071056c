"""The C-ABI library loads on a machine without a GPU and exports what include/kvp.h declares."""

import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvp.h")


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^KVP_API [\w\s\*]+?\b(\w+)\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_319_b200 import _lib

    return _lib.lib()


def test_header_declares_the_boundary():
    names = declared()
    for n in ("kv_pool_create", "kv_seq_append", "kv_seq_fork", "kv_seq_release",
              "kv_pool_take_copies", "kv_build_batch", "reshape_and_cache", "copy_blocks",
              "paged_attention_decode", "kvp_decode_workspace_bytes", "kvp_check_device_error"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared():
        assert hasattr(lib, n), n


def test_exports_are_exactly_the_declared_ones():
    from paged_kv_cache_319_b200 import _lib

    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines() if " T " in ln})
    assert exported == declared()


def test_binding_signatures_cover_the_header():
    from paged_kv_cache_319_b200 import _lib

    assert sorted(_lib.SIGNATURES) == declared()


def test_version_and_capacity_model(lib):
    import paged_kv_cache_319_b200 as kvp

    assert "sm_100a" in kvp.version()
    # 2 x 5120 x 40 x 2 bytes: the OPT-13B worked example
    assert kvp.kv_bytes_per_token(5120, 40, 2) == 819200


def test_workspace_size_formula(lib):
    import paged_kv_cache_319_b200 as kvp

    assert kvp.decode_workspace_bytes(64, 40, 128, 2048, 0) == 0
    assert kvp.decode_workspace_bytes(64, 40, 128, 512, 512) == 0      # one partition
    n = kvp.decode_workspace_bytes(32, 32, 128, 32768, 512)
    assert n >= 32 * 32 * 64 * (128 + 2) * 4 and n % 256 == 0


def test_device_calls_reject_bad_arguments_without_a_gpu(lib):
    import ctypes as C

    from paged_kv_cache_319_b200._lib import KVP_ERR_INVALID

    # invalid geometry is caught on the host before anything touches a device
    rc = lib.paged_attention_decode(None, None, None, None, None, 1, 4, 4, 96, 16, 8, 1, 16,
                                    C.c_float(1.0), 0, None, 0, None, 0, None)
    assert rc == KVP_ERR_INVALID
    assert b"head_dim" in lib.kvp_last_error_message()
    rc = lib.reshape_and_cache(None, None, None, None, None, 1, 4, 100, 16, 8, 0, None)
    assert rc == KVP_ERR_INVALID
    rc = lib.copy_blocks(None, None, None, 1, 8, 100, 0, None)   # 200 bytes: not 16-aligned
    assert rc == KVP_ERR_INVALID
