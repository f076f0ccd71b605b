"""The boundary from C: compile a C99 program against include/rma.h with gcc, link it to
librma.so and run its host-only checks (no GPU is touched)."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_header_compiles_as_c99_and_host_calls_answer(tmp_path):
    from bounded_memory_attention_b200 import build
    so = build.build()
    exe = tmp_path / "c_abi_host_calls"
    src = os.path.join(ROOT, "tests", "c_abi_host_calls.c")
    libdir = os.path.dirname(so)
    libname = os.path.basename(so)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                        src, "-o", str(exe), os.path.join(libdir, libname), f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.strip().endswith("ok")
