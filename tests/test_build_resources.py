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
CEILINGS = {"phi_fixup_kernel": (4, 4)}


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
    # ptxas prints, per entry function: "Compiling entry function 'X'", then
    # "Function properties for X" with its stack/spill line, then "Used N registers".
    # Non-inlined device functions get a "Function properties for Y" block of their
    # own: their spill line belongs to Y, not to the entry function before it.
    entries, rows, props = set(), {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            entries.add(m.group(1))
            continue
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            props = m.group(1)
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and props:
            rows.setdefault(props, {}).update(stack=int(m.group(1)), st=int(m.group(2)), ld=int(m.group(3)))
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and props:
            rows.setdefault(props, {})["regs"] = int(m.group(1))
    return [(name, v.get("stack", 0), v.get("st", 0), v.get("ld", 0), v.get("regs"))
            for name, v in rows.items() if name in entries]


def test_every_kernel_is_reported(report):
    names = " ".join(r[0] for r in report)
    for k in ("attn_packed_kernel", "attn_sel_kernel", "topn_kernel", "phi_linear_kernel", "dec_cmp_stream",
              "dec_slcwin_stream", "dec_win_stream", "dec_final", "bwd_q_sel", "bwd_kv_tc", "bwd_q_dense",
              "decode_append_kernel",
              "phi_dw_kernel"):
        assert k in names, k


def test_no_register_spills_beyond_the_ceilings(report):
    for name, stack, st, ld, regs in report:
        ceil = next((v for k, v in CEILINGS.items() if k in name), (0, 0))
        assert st <= ceil[0] and ld <= ceil[1], (name, st, ld)
        if "attn_" in name or "dec_" in name or "topn" in name or "bwd_" in name:
            assert st == 0 and ld == 0 and stack <= 8, (name, stack)


# registers per thread that a kernel's launch shape relies on for its residency:
# top-n over rows of at most 1024 blocks runs 3 CTAs of 256 threads per SM; the
# decode window stream (128 threads) shares each SM with a combine CTA (256
# threads): 128 x 168 + 256 x 168 registers fill the register file
REG_CEILINGS = {"topn_kernelILi32E": 80, "dec_win_stream": 168, "dec_cmp_combine": 168}


def test_register_ceilings_of_occupancy_sensitive_kernels(report):
    seen = set()
    for name, stack, st, ld, regs in report:
        for k, lim in REG_CEILINGS.items():
            if k in name:
                seen.add(k)
                assert regs is not None and regs <= lim, (name, regs, lim)
    assert seen == set(REG_CEILINGS)
