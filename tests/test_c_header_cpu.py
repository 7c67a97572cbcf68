"""include/moe.h is a C header: a C99 program (tests/c/abi_host_check.c) compiles
against it with warnings as errors, links libmoe_b200.so and calls its host-side entry
points.  CPU only (nothing touches device memory)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_c99_client_compiles_links_and_runs(tmp_path):
    from routing_dispatch_expert_moe_b200 import build
    lib = build.build()
    exe = tmp_path / "abi_host_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host_check.c"), "-L", os.path.dirname(lib), "-lmoe_b200", "-lm",
           "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    env = dict(os.environ, LD_LIBRARY_PATH=os.path.dirname(lib))
    r = subprocess.run([str(exe)], capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
