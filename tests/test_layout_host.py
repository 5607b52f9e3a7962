"""Host logic of the CUDA library on the CPU: the shard-layout position helpers that the
attention kernels use for causal scheduling and masking (contiguous and zigzag layouts) and
the query-tile ranges of the backward's key-tile kernel (zigzag and packed samples),
compiled from the library's own header and checked against brute force."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_shard_layout_helpers(tmp_path):
    exe = tmp_path / "layout_check"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", os.path.join(ROOT, "sequence_parallelism_attn_b200", "csrc"),
                    "-I", cuda_inc, "-o", str(exe), os.path.join(ROOT, "tests", "layout_check.cpp")],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "mismatches: 0" in r.stdout


def test_permute_index_arithmetic(tmp_path):
    """The vector Ulysses kernels' index helpers (invariant-integer division, source vector
    of every output vector, G head groups and the GQA copy) against brute force."""
    exe = tmp_path / "permute_index_check"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", os.path.join(ROOT, "sequence_parallelism_attn_b200", "csrc"),
                    "-I", cuda_inc, "-o", str(exe), os.path.join(ROOT, "tests", "permute_index_check.cpp")],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "mismatches: 0" in r.stdout
