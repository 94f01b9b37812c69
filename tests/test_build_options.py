"""The attention kernel's compile-time options still build for sm_100a (no GPU needed).

The default build is covered by every other test; these are the alternatives kept in the
source (two softmax warps per row, P in four or one parts, polynomial exp2 for part of
the scores, direct epilogue stores, no split items, the first prologue layout, a 64-thread
prologue block). Each is compiled to an object file with nvcc, in parallel.
"""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "unified_text_pixel_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

OPTIONS = {
    "two_warps_per_row": ["-DHGX_SOFTMAX_SPLIT=2"],
    "p_in_four_parts": ["-DHGX_P_PARTS=4"],
    "p_in_one_part": ["-DHGX_P_PARTS=1"],
    "polynomial_exp2": ["-DHGX_EXP_POLY_MASK=0x0101"],
    "no_split_items": ["-DHGX_SPLIT_KV=0"],
    "direct_epilogue_stores": ["-DHGX_EPI_TMA=0"],
    "first_prologue_layout": ["-DHGX_PRO_V2=0"],
    "prologue_64_threads": ["-DHGX_PRO_V2_THREADS=64"],
}


@pytest.mark.skipif(not os.path.exists(NVCC) and shutil.which("nvcc") is None, reason="nvcc not found")
def test_attention_options_compile():
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    src = os.path.join(CSRC, "attention.cu")
    with tempfile.TemporaryDirectory() as tmp:
        procs = {}
        for name, flags in OPTIONS.items():
            target = (os.path.join(CSRC, "api.cu") if "SPLIT_KV" in flags[0] else
                      os.path.join(CSRC, "prologue.cu") if "PRO_" in flags[0] else src)
            cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                   "-I", CSRC, *flags, "-c", target, "-o", os.path.join(tmp, name + ".o")]
            procs[name] = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
        failed = {}
        for name, proc in procs.items():
            out, _ = proc.communicate(timeout=600)
            if proc.returncode != 0:
                failed[name] = out.decode(errors="replace")[-2000:]
        assert not failed, failed
