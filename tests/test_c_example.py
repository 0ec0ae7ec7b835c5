"""The C interface used from plain C: the example program under the package's
examples/ builds against include/dsa.h and the library with gcc alone, and (on
a B200) the fused decode step equals the three staged calls."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_long_context_indexer_b200")
SRC = os.path.join(PKG, "examples", "decode_c_api.c")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    lib = os.path.join(PKG, "libdsa_b200.so")
    if not os.path.exists(lib):
        from sparse_long_context_indexer_b200 import build
        build.build()
    exe = str(tmp_path / "decode_c_api")
    cmd = [gcc, "-O2", "-Wall", "-Wextra", "-Werror", f"-I{os.path.join(ROOT, 'include')}",
           f"-I{os.path.join(CUDA, 'include')}", SRC, f"-L{PKG}", "-ldsa_b200", f"-L{os.path.join(CUDA, 'lib64')}",
           "-lcudart", "-lm", f"-Wl,-rpath,{PKG}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    return exe


def test_c_example_builds_with_gcc(tmp_path):
    exe = _build(tmp_path)
    assert os.access(exe, os.X_OK)


@pytest.mark.gpu
def test_c_example_fused_step_equals_staged_calls(tmp_path):
    exe = _build(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok:") and "selections identical" in r.stdout
