"""The C ABI from a plain C99 caller: include/kd.h compiles as strict C, and a
program linked against libkd.so gets the documented statuses from host-side
validation (no kernel is launched, so no GPU is needed)."""

import os
import shutil
import subprocess

import pytest

from chunked_kl_loss_chunk_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_caller(tmp_path):
    lib = build.build()
    src = os.path.join(ROOT, "tests", "c", "abi_host_check.c")
    exe = str(tmp_path / "abi_host_check")
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I" + os.path.join(ROOT, "include"), src, "-o", exe,
                    "-L" + libdir, "-l:libkd.so", "-Wl,-rpath," + libdir],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"


def test_header_compiles_as_cxx(tmp_path):
    """The same header from C++ (extern "C" linkage, no C-only constructs)."""
    if shutil.which("g++") is None:
        pytest.skip("needs g++")
    src = tmp_path / "inc.cc"
    src.write_text('#include "kd.h"\nint main() { return kd_status_string(KD_OK) ? 0 : 1; }\n')
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Werror", "-I" + os.path.join(ROOT, "include"),
                    "-c", str(src), "-o", str(tmp_path / "inc.o")], check=True,
                   capture_output=True, text=True)


def test_gemm_unit_walk_matches_direct_coordinates(tmp_path):
    """The persistent GEMM's clusters walk their work units without division
    (kd_unitwalk.h); on the host, the walk must give every cluster the same
    units, tile coordinates and K ranges as the direct computation, for the
    launch shapes of the bench workloads and for every small shape."""
    if shutil.which("g++") is None:
        pytest.skip("needs g++")
    src = os.path.join(ROOT, "tests", "c", "unitwalk_check.cc")
    exe = str(tmp_path / "unitwalk_check")
    subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Werror",
                    "-I" + os.path.join(ROOT, "chunked_kl_loss_chunk_b200", "csrc"), src, "-o", exe],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
