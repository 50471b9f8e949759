"""The C ABI from plain C: tests/c_abi_host.c includes include/mlra.h as C (no CUDA headers),
links libmlra.so and checks the host-side entry points.  Needs gcc, no GPU."""
import pathlib
import shutil
import subprocess

import pytest

ROOT = pathlib.Path(__file__).resolve().parents[1]
LIB_DIR = ROOT / "latent_kv_cache_mlra_b200"


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_header_compiles_as_c_and_host_calls_answer(tmp_path):
    if not (LIB_DIR / "libmlra.so").exists():
        pytest.skip("libmlra.so not built")
    exe = tmp_path / "c_abi_host"
    build = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", str(ROOT / "include"),
                            str(ROOT / "tests" / "c_abi_host.c"), "-L", str(LIB_DIR), "-lmlra",
                            f"-Wl,-rpath,{LIB_DIR}", "-o", str(exe)],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.startswith("ok")
