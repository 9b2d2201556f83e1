"""The headers are plain C: a C11 program includes include/*.h, links
libditattn.so and checks argument rejection (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from diffusion_transformer_attention_attn_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_program_builds_and_runs(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    lib = build_lib.build()
    exe = tmp_path / "abi_check"
    subprocess.check_call([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), lib, "-o", str(exe),
                           f"-Wl,-rpath,{os.path.dirname(lib)}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "abi check ok" in out.stdout
