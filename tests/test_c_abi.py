"""The C ABI from C itself: a C99 program that includes include/vdn.h and
links libvdn.so compiles without warnings and its host-only checks pass."""
import os
import shutil
import subprocess

import pytest

import softmax_attention_video_chunk_b200 as vdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def libdir():
    from softmax_attention_video_chunk_b200 import _build
    if _build.needs_build():
        _build.build()
    vdn.lib()
    return os.path.dirname(vdn.LIB_PATH)


def test_c_program_against_the_header(libdir):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(libdir, "_build")  # the package's (untracked) build directory
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "abi_host_check")
    src = os.path.join(ROOT, "tests", "c", "abi_host_check.c")
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic-errors",
                    "-Wno-gnu-zero-variadic-macro-arguments", "-I", os.path.join(ROOT, "include"),
                    src, "-o", exe, "-L", libdir, "-lvdn", "-Wl,-rpath," + libdir],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAIL" not in r.stdout
