"""The token split's key merge (select_merge in
query_aware_kv_ts_b200/csrc/split.cu) on the CPU: the kernel's own source,
with its constants, compiled for the host by tests/select_merge_emu.cpp (one
CTA of 1024 std::threads, barriers for __syncthreads and the warp
intrinsics) and run on key sets with ties at the threshold, padded ranks,
votes of +0, k of 0 and 1, and no more real keys than k; every rank row must
be the one a sort of all the keys gives.  A guard on the merge's logic that
needs no GPU (the GPU tests run the same kernel on the device)."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SPLIT_CU = os.path.join(ROOT, "query_aware_kv_ts_b200", "csrc", "split.cu")
HARNESS = os.path.join(ROOT, "tests", "select_merge_emu.cpp")


def kernel_sources(src: str):
    """The merge's constants and its source (the block scan it calls, then
    the kernel up to its closing brace) from split.cu's text."""
    constants = "\n".join(re.findall(r"^constexpr int kSelMerge\w+ = [^;]+;", src, re.M))
    start = src.index("__device__ __forceinline__ uint32_t block_exclusive_scan")
    sig = src.index("select_merge(const unsigned long long *keys")
    end = src.index("\n}\n", sig) + 3
    return constants + "\n", src[start:end]


def test_kernel_sources_are_found():
    with open(SPLIT_CU) as f:
        constants, kernel = kernel_sources(f.read())
    assert "kSelMergeThreads" in constants and "kSelMergeBins" in constants
    assert kernel.rstrip().endswith("}") and "select_merge(" in kernel


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_key_merge_matches_a_sort(tmp_path):
    with open(SPLIT_CU) as f:
        constants, kernel = kernel_sources(f.read())
    (tmp_path / "constants.inc").write_text(constants)
    (tmp_path / "kernel.inc").write_text(kernel)
    exe = str(tmp_path / "select_merge_emu")
    subprocess.run(["g++", "-std=c++20", "-O1", "-pthread", "-I", str(tmp_path), HARNESS, "-o", exe], check=True,
                   capture_output=True, timeout=300)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0 and run.stdout.strip().endswith("12 cases, 0 failures"), run.stdout
