"""The host half of the library (block pool, prefix cache, grouping planner) built
with AddressSanitizer and UndefinedBehaviorSanitizer and driven through its C API
on random streams checked against the oracle (tests/host_sanitizer_driver.py): no
memory error, no undefined behaviour, no leak from the library, same results.
Skipped where g++ or the sanitizer runtimes are missing."""

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _runtime(name):
    p = subprocess.run(["g++", f"-print-file-name={name}"], capture_output=True, text=True)
    path = p.stdout.strip()
    return path if os.path.isabs(path) and os.path.exists(path) else None


@pytest.mark.skipif(shutil.which("g++") is None, reason="no g++")
def test_host_library_under_sanitizers(tmp_path):
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("sanitizer runtimes not installed")
    lib = tmp_path / "libkvp_host_asan.so"
    csrc = os.path.join(ROOT, "paged_kv_cache_319_b200", "csrc")
    build = subprocess.run(
        ["g++", "-std=c++17", "-O1", "-g", "-fno-omit-frame-pointer",
         "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined", "-fPIC", "-shared",
         "-I", os.path.join(ROOT, "include"), "-I", csrc, "-o", str(lib),
         os.path.join(csrc, "host", "block_pool.cpp"), os.path.join(csrc, "host", "group_plan.cpp")],
        capture_output=True, text=True)
    assert build.returncode == 0, build.stderr[-3000:]
    env = dict(os.environ, LD_PRELOAD=f"{asan}:{ubsan}",
               ASAN_OPTIONS="detect_leaks=1:halt_on_error=1",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "host_sanitizer_driver.py"),
                        str(lib)], env=env, capture_output=True, text=True, timeout=600)
    out = r.stdout + r.stderr
    assert "sanitized host streams ok" in out, out[-4000:]
    for marker in ("ERROR: AddressSanitizer", "runtime error:"):
        assert marker not in out, out[-4000:]
    # the interpreter itself leaks at exit; none of the leaks may come from the library
    assert "block_pool.cpp" not in out and "group_plan.cpp" not in out, out[-4000:]
