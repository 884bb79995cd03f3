"""liblq from plain C: tests/c_abi_check.c includes only include/lq.h and the C
standard headers, is compiled as strict C99 with warnings as errors, links the
in-tree liblq.so and runs its host-only checks (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from recurrent_state_quantization_lq_b200 import lq

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_c_caller_compiles_links_and_passes(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler on this machine")
    libdir = os.path.dirname(lq.LIB_PATH)
    assert os.path.exists(lq.LIB_PATH), "liblq.so is built in-tree by the package build"
    exe = str(tmp_path / "c_abi_check")
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(HERE, "c_abi_check.c"),
                    "-L", libdir, "-llq", f"-Wl,-rpath,{libdir}", "-o", exe],
                   check=True, capture_output=True, text=True, timeout=120)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "c abi ok" in r.stdout
