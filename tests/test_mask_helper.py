"""The kernels' mask helper (visible_keys, a host/device function of
fa_internal.h) against enumeration of the mask's definition, on the CPU: a
host-only build of tests/mask_helper_check.cu prints the helper's first and
last visible key for a grid of cases."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _visible(i, j, s_q, n, causal, left, right):
    a = i + n - s_q                      # the query's bottom-right aligned key
    if causal and j > a:
        return False
    if right >= 0 and j > a + right:
        return False
    if left >= 0 and j < a - left:
        return False
    return True


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not available")
def test_visible_keys_matches_enumeration(tmp_path):
    exe = tmp_path / "mask_helper_check"
    subprocess.run([NVCC if os.path.exists(NVCC) else "nvcc", "-std=c++17", "-gencode",
                    "arch=compute_100a,code=sm_100a", "-I", os.path.join(ROOT, "include"), "-I",
                    os.path.join(ROOT, "rotary_embedding_b200", "csrc"), os.path.join(HERE, "mask_helper_check.cu"),
                    "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    lines = [ln for ln in out if ln]
    assert len(lines) > 1000
    for ln in lines:
        i, n, s_q, causal, left, right, first, last = map(int, ln.split())
        keys = [j for j in range(n) if _visible(i, j, s_q, n, causal, left, right)]
        if keys:
            # the visible keys form one interval, reported exactly
            assert keys == list(range(first, last + 1)), ln
        else:
            assert first > last, ln
