"""Resource report of the CUDA build (`nvcc -Xptxas -v`, no GPU needed): no kernel
spills registers to local memory beyond the recorded ceilings, so a change that
adds spills is caught before it reaches a GPU.  The report is read only for its
register, stack and spill counts."""
import os
import re
import shutil
import subprocess
import tempfile

import pytest

from sparse_attention_long_phi_b200 import build as nbuild

# current ceilings (bytes of spill stores, spill loads); every other kernel: none
CEILINGS = {"bwd_query_mma": (36, 84), "phi_fixup_kernel": (4, 4)}


@pytest.fixture(scope="module")
def report():
    nvcc = os.environ.get("NVCC", "nvcc")
    if shutil.which(nvcc) is None:
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as d:
        cmd = [nvcc, *nbuild.NVCC_FLAGS, "-Xptxas", "-v", "-o", os.path.join(d, "x.so"),
               os.path.join(nbuild.CSRC, "nsa_capi.cu")]
        r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    rows, cur = [], None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and cur:
            rows.append((cur, int(m.group(1)), int(m.group(2)), int(m.group(3))))
        m = re.search(r"Used (\d+) registers", line)
        if m and rows and rows[-1][0] == cur:
            rows[-1] = rows[-1] + (int(m.group(1)),)
    return rows


def test_every_kernel_is_reported(report):
    names = " ".join(r[0] for r in report)
    for k in ("attn_packed_kernel", "attn_sel_kernel", "topn_kernel", "phi_linear_kernel", "dec_cmp_stream",
              "dec_slcwin_stream", "bwd_query_mma", "bwd_kv_mma", "decode_append_kernel", "phi_dw_kernel"):
        assert k in names, k


def test_no_register_spills_beyond_the_ceilings(report):
    for name, stack, st, ld, *regs in report:
        ceil = next((v for k, v in CEILINGS.items() if k in name), (0, 0))
        assert st <= ceil[0] and ld <= ceil[1], (name, st, ld)
        if "attn_" in name or "dec_" in name or "topn" in name:
            assert st == 0 and ld == 0 and stack <= 8, (name, stack)
        if regs:
            assert regs[0] <= 255, name
