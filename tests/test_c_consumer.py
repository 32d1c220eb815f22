"""The C ABI from plain C: a C99 program built against include/h3b.h alone, with
-Wall -Wextra -pedantic -Werror, links to the library and checks its host-side
contract (no GPU needed). Shows the header is a C header, not a C++ one, and that
nothing beyond it is needed to call the library."""
import os
import shutil
import subprocess

import pytest

from video_diffusion_transformer_adaln_b200 import build, h3b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_consumer", "abi_host_checks.c")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_c99_program_uses_the_abi(tmp_path):
    build.build()
    lib_dir = os.path.dirname(h3b.LIB_PATH)
    exe = str(tmp_path / "abi_host_checks")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), SRC, "-o", exe,
                    "-L", lib_dir, "-l:libh3b.so", "-Wl,-rpath," + lib_dir], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "OK"
