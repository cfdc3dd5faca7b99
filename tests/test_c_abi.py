"""The C ABI from plain C99: compile tests/c/abi_check.c against the public
header with gcc (-std=c99 -pedantic -Werror), link the built library and run
its host-only checks (sizes, argument validation, status strings; no kernel
is launched)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "rna_structure_models_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_header_and_library_from_plain_c(tmp_path):
    lib = os.path.join(LIBDIR, "libflashipa_b200.so")
    if not os.path.exists(lib):
        pytest.fail("library not built (python -m rna_structure_models_b200.build)")
    exe = str(tmp_path / "abi_check")
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", exe, "-L", LIBDIR, "-lflashipa_b200",
           "-Wl,-rpath," + LIBDIR]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi ok" in r.stdout


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_end_to_end_host_buffers_from_plain_c(tmp_path):
    # tests/c/e2e_host.c: page-locked host inputs through ipa_attn_fwd_host on
    # two streams; its host result must equal ipa_attn_fwd's bit for bit
    lib = os.path.join(LIBDIR, "libflashipa_b200.so")
    cuda = "/usr/local/cuda"
    exe = str(tmp_path / "e2e_host")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "e2e_host.c"), "-o", exe,
           "-L", LIBDIR, "-lflashipa_b200", "-L", os.path.join(cuda, "lib64"), "-lcudart", "-lm",
           "-Wl,-rpath," + LIBDIR, "-Wl,-rpath," + os.path.join(cuda, "lib64")]
    assert os.path.exists(lib)
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe, "1000", "10"], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "e2e ok" in r.stdout
