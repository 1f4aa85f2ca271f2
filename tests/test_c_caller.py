"""libcalibatt from a plain C program: the header compiles as C, the library
links without torch, and the host entry points behave (no GPU work)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_program_calls_the_host_entry_points(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    from calibrated_block_sparse_b200 import build
    lib = build.build()
    exe = tmp_path / "abi_host_check"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host_check.c"), lib, "-lm", "-o", str(exe),
                    f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


@pytest.mark.gpu
def test_c_program_runs_attention_on_the_gpu(tmp_path):
    """A C program owns the device buffers (cudaMalloc), calls
    calibatt_sparse_attn_fwd and checks every row against dense softmax
    attention it computes itself in double precision."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    from calibrated_block_sparse_b200 import build
    lib = build.build()
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = tmp_path / "attn_c_check"
    subprocess.run([cc, "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "attn_c_check.c"), lib,
                    "-L", os.path.join(cuda, "lib64"), "-lcudart", "-lm", "-o", str(exe),
                    f"-Wl,-rpath,{os.path.dirname(lib)}", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
