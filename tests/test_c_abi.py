"""The C ABI used from plain C: tests/c_abi_check.c is compiled with gcc as C11
against include/kda.h, linked against libkda.so and run (host-side paths only,
no GPU needed)."""
import os
import subprocess

from linear_attention_recurrence_06_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_program_links_and_validates(tmp_path):
    kbuild.build()
    lib_dir = os.path.join(ROOT, "linear_attention_recurrence_06_b200")
    exe = tmp_path / "c_abi_check"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", lib_dir, "-lkda",
                    "-Wl,-rpath," + lib_dir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert "c_abi_check ok" in out.stdout
