"""The C ABI from plain C: a C99 program built against include/h3b.h alone, with
-Wall -Wextra -pedantic -Werror, links to the library and checks its host-side
contract (no GPU needed). Shows the header is a C header, not a C++ one, and that
nothing beyond it is needed to call the library. The program also prints the
offset and size of every field of the header's structs, which must equal the
binding's ctypes mirrors of them."""
import ctypes
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
    lines = r.stdout.strip().splitlines()
    assert lines[-1] == "OK"
    # the binding's ctypes mirrors of the header's structs have the C layout
    mirrors = {"h3b_dims": h3b.Dims, "h3b_block_weights": h3b.BlockWeights, "h3b_kernel_time": h3b.KernelTime}
    seen = set()
    for line in lines[:-1]:
        parts = line.split()
        if parts[0] == "sizeof":
            assert ctypes.sizeof(mirrors[parts[1]]) == int(parts[2]), line
            continue
        struct, field, off, size = parts[0], parts[1], int(parts[2]), int(parts[3])
        desc = getattr(mirrors[struct], field)
        assert (desc.offset, desc.size) == (off, size), line
        seen.add((struct, field))
    for name, cls in mirrors.items():
        assert {(name, f[0]) for f in cls._fields_} == {s for s in seen if s[0] == name}
