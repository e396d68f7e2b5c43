"""The C ABI from plain C: include/deltakv.h compiles as strict C99
(gcc -std=c99 -pedantic, no warnings) and a C program linked against
libdeltakv.so plans a layer on a host without a GPU."""
import os
import shutil
import subprocess

import pytest

from decode_attention_strided_b200 import build as dkv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_c99_and_the_library_plans_from_c(tmp_path):
    dkv_build.build()
    libdir = os.path.join(ROOT, "decode_attention_strided_b200", "_lib")
    exe = str(tmp_path / "c_abi_check")
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
                         "-L", libdir, "-ldeltakv", f"-Wl,-rpath,{libdir}", "-o", exe],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    first, second = run.stdout.strip().splitlines()
    status, cache_bytes, ws_bytes, n_ref_cap, n_code_cap = (int(x) for x in first.split())
    assert status == 0 and n_ref_cap == 8192 and n_code_cap == 131072 - 8192
    # four planes of 8 x 8 (sequence, kv-head) pairs: K and V references,
    # bf16 codes and int32 slots
    assert cache_bytes >= 64 * (8192 * 128 * 2 * 2 + (131072 - 8192) * (32 * 2 + 4 * 4))
    assert ws_bytes > 0
    assert second == "1 null"  # DELTAKV_ERR_INVALID_ARG, no plan returned
