"""The C-ABI library builds, exports every entry point include/nsa.h declares,
and validates its arguments on the host (no GPU needed: every case below is
rejected before any CUDA call)."""
import ctypes
import os
import re

import pytest

from sparse_attention_long_phi_b200 import build as nbuild
from sparse_attention_long_phi_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    nbuild.build()
    from sparse_attention_long_phi_b200 import nsa
    return nsa


@pytest.fixture
def host_only():
    """The validation cases pass made-up device addresses that the host checks reject
    before any CUDA call; they run only where no GPU is visible, so that a regressed
    check can never hand such an address to a device."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("made-up device addresses are passed only where no GPU is visible")


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "nsa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(nsa_[a-z_]+)\s*\(", txt)))


def test_library_exports_every_declared_entry_point(L):
    names = declared_functions()
    assert {"nsa_forward", "nsa_decode", "nsa_backward", "nsa_workspace_size",
            "nsa_status_string", "nsa_compress", "nsa_sync_status", "nsa_num_cmp_blocks"} <= set(names)
    lib = ctypes.CDLL(L.library_path())
    for n in names:
        assert hasattr(lib, n), n


def declared_arity():
    """Parameter count of every function include/nsa.h declares."""
    txt = open(os.path.join(ROOT, "include", "nsa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(nsa_[a-z_]+)\s*\(([^()]*)\)\s*;", txt):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header(L):
    lib = L.lib()
    arity = declared_arity()
    assert len(arity) >= 14
    for name, n in arity.items():
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None, f"{name}: no argtypes in the binding"
        assert len(argtypes) == n, f"{name}: binding has {len(argtypes)} arguments, header {n}"


def test_status_strings_and_shape_helpers(L):
    lib = L.lib()
    for code in range(6):
        assert lib.nsa_status_string(code)
    c = I.WORKLOADS["prefill_fwd_T65536"]
    assert L.num_cmp_blocks(c, 65536) == 4095
    assert L.num_cmp_blocks(c, 31) == 0 and L.num_cmp_blocks(c, 32) == 1
    for mode in (0, 1, 2):
        assert L.workspace_size(c, mode) > 0


def _fwd(L, c, ptrs=True, ws_bytes=1 << 30):
    lib = L.lib()
    cfg = L.make_config(c)
    fake = ctypes.c_void_p(1 << 20) if ptrs else None     # never dereferenced: rejected first
    return lib.nsa_forward(ctypes.byref(cfg), fake, fake, fake, fake, None, fake, fake, None, None,
                           None, ctypes.c_void_p(1 << 20), ws_bytes, None)


def test_forward_argument_validation_on_host(L, host_only):
    base = dict(I.WORKLOADS["prefill_fwd_T8192"], phi="mean")
    assert _fwd(L, dict(base, d=12)) == 1                   # d does not divide l
    assert _fwd(L, dict(base, l=128)) == 1                  # l > l'
    assert _fwd(L, dict(base, n=2)) == 1                    # n < forced blocks
    assert _fwd(L, dict(base, H=63)) == 1                   # heads not a multiple of groups
    assert _fwd(L, dict(base, T=0)) == 1
    assert _fwd(L, base, ptrs=False) == 1                   # null tensors
    assert _fwd(L, dict(base, dk=128)) == 2                 # no kernel for d_k = 128
    assert _fwd(L, dict(base, lp=32, l=16)) == 2            # selection block != 64
    assert _fwd(L, dict(base, n=17)) == 2
    assert _fwd(L, dict(base, T=131073)) == 2                # beyond the largest supported context
    assert _fwd(L, base, ws_bytes=1024) == 3                # workspace too small


def test_select_blocks_validation_on_host(L, host_only):
    lib = L.lib()
    fake = ctypes.c_void_p(1 << 20)
    base = dict(I.WORKLOADS["prefill_fwd_T8192"])
    cfg = L.make_config(base)
    assert lib.nsa_select_blocks(ctypes.byref(cfg), None, fake, None) == 1       # null scores
    assert lib.nsa_select_blocks(ctypes.byref(cfg), fake, None, None) == 1       # null output
    assert lib.nsa_select_blocks(ctypes.byref(L.make_config(dict(base, n=2))), fake, fake, None) == 1
    assert lib.nsa_select_blocks(ctypes.byref(L.make_config(dict(base, n=33))), fake, fake, None) == 2
    assert lib.nsa_select_blocks(ctypes.byref(L.make_config(dict(base, T=131073))), fake, fake, None) == 2


def test_decode_append_and_rows_validation_on_host(L, host_only):
    lib = L.lib()
    c = dict(I.WORKLOADS["decode_S32_L8k_64k"])
    cfg = L.make_config(c, batch=32, seqlen=65536)
    fake = ctypes.c_void_p(1 << 20)
    nine = [fake] * 9
    assert lib.nsa_decode_append(ctypes.byref(cfg), 4, None, *nine[1:], None, None) == 1     # null k_new
    assert lib.nsa_decode_append(ctypes.byref(cfg), 4, *nine, None, None) == 1               # linear phi, no params
    assert lib.nsa_decode_append(ctypes.byref(cfg), 0, *([None] * 9), None, None) == 0      # nothing to do
    assert lib.nsa_decode_append(ctypes.byref(cfg), -1, *nine, None, None) == 1
    assert lib.nsa_decode_rows(ctypes.byref(cfg), 33, *([fake] * 13), 1 << 30, None) == 1   # more seqs than sized
    assert lib.nsa_decode_rows(ctypes.byref(cfg), 8, *([fake] * 13), 16, None) == 3         # workspace too small
    args = [fake] * 13
    args[4] = None                                                                           # no lengths
    assert lib.nsa_decode_rows(ctypes.byref(cfg), 8, *args, 1 << 30, None) == 1
    assert len(L.lib().nsa_decode_rows.argtypes) == 17 and len(L.lib().nsa_decode.argtypes) == 16


@pytest.mark.parametrize("l,d", [(32, 16), (32, 32), (16, 16), (64, 16)])
def test_append_completion_rule_matches_block_count(L, l, d):
    # nsa_decode_append compresses block (L - l)/d exactly when the new length L
    # adds one to nsa_num_cmp_blocks (page 2, 令牌压缩: block i = tokens [i*d, i*d + l))
    import oracle
    c = dict(I.WORKLOADS["prefill_fwd_T8192"], l=l, d=d)
    for n in range(1, 600):
        grows = L.num_cmp_blocks(c, n) - L.num_cmp_blocks(c, n - 1)
        assert grows == int(n >= l and (n - l) % d == 0), n
        assert L.num_cmp_blocks(c, n) == oracle.num_cmp_blocks(c, n)


def test_phi_parameter_gradient_validation_on_host(L, host_only):
    lib = L.lib()
    fake = ctypes.c_void_p(1 << 20)
    phi = ctypes.byref(L.CPhi(fake, fake, fake, fake))
    lin = L.make_config(I.WORKLOADS["train_fwd_bwd_B2_T16384"])
    mean = L.make_config(dict(I.WORKLOADS["train_fwd_bwd_B2_T16384"], phi="mean"))
    out = [fake] * 4
    assert lib.nsa_backward_phi_params(ctypes.byref(mean), fake, fake, phi, *out, fake, 1 << 40, None) == 1
    assert lib.nsa_backward_phi_params(ctypes.byref(lin), fake, fake, None, *out, fake, 1 << 40, None) == 1
    assert lib.nsa_backward_phi_params(ctypes.byref(lin), fake, fake, phi, *out, fake, 64, None) == 3


def test_decode_and_backward_validation_on_host(L, host_only):
    lib = L.lib()
    c = dict(I.WORKLOADS["decode_S32_L8k_64k"], B=32, T=65536)
    cfg = L.make_config(c, batch=32, seqlen=65536)
    fake = ctypes.c_void_p(1 << 20)
    args = [fake] * 12
    assert lib.nsa_decode(ctypes.byref(cfg), 33, *args, 1 << 30, None) == 1   # more seqs than sized
    assert lib.nsa_decode(ctypes.byref(cfg), 8, *args, 16, None) == 3         # workspace too small
    assert lib.nsa_decode(ctypes.byref(cfg), 0, *args, 16, None) == 0         # nothing to do
    big = L.make_config(dict(c, B=4096), batch=4096, seqlen=8192)
    assert lib.nsa_decode(ctypes.byref(big), 3000, *args, 1 << 40, None) == 2  # > 2048 sequences per call
    cb = L.make_config(I.WORKLOADS["train_fwd_bwd_B2_T16384"])
    assert lib.nsa_backward(ctypes.byref(cb), fake, fake, fake, fake, None, fake, fake, fake, fake,
                            fake, fake, fake, 64, None) == 3
    assert lib.nsa_backward(ctypes.byref(cb), None, fake, fake, fake, None, fake, fake, fake, fake,
                            fake, fake, fake, 1 << 40, None) == 1


def test_forward_branches_validation_and_score_table_on_host(L, host_only):
    lib = L.lib()
    base = dict(I.WORKLOADS["prefill_fwd_T8192"], phi="mean")
    cfg = L.make_config(base)
    fake = ctypes.c_void_p(1 << 20)
    ws = 1 << 34
    seven = [fake] * 7                     # q, k_cmp, v_cmp, k_slc, v_slc, k_win, v_win
    missing = list(seven)
    missing[5] = None                      # no window keys
    assert lib.nsa_forward_branches(ctypes.byref(cfg), *missing, fake, None, fake, fake, None, None, None,
                                    fake, ws, None) == 1
    small = L.workspace_size(base, L.NSA_MODE_FORWARD)
    assert lib.nsa_forward_branches(ctypes.byref(cfg), *seven, fake, None, fake, fake, None, None, None,
                                    fake, small, None) == 3          # needs the larger workspace
    assert L.workspace_size(base, L.NSA_MODE_FORWARD_BRANCHES) > small
    stride = ctypes.c_int64(0)
    off = lib.nsa_forward_score_table(ctypes.byref(cfg), ctypes.byref(stride))
    assert 0 < off < small and off % 256 == 0 and stride.value == 128
    assert off + 4 * 8192 * 4 * 128 <= small
    assert lib.nsa_forward_score_table(ctypes.byref(L.make_config(dict(base, d=12))), None) == -1
    assert lib.nsa_check_timeout_path(0, None) == 1                  # limit outside 1 .. 2e9 ns


def test_training_forward_and_saved_backward_validation_on_host(L, host_only):
    lib = L.lib()
    cb = L.make_config(dict(I.WORKLOADS["train_fwd_bwd_B2_T16384"]))
    fake = ctypes.c_void_p(1 << 20)
    big = 1 << 40
    # nsa_forward_train(cfg, q, k, v, gates, phi, out, sel_idx, lse, o_branch, ws, bytes, stream)
    assert lib.nsa_forward_train(ctypes.byref(cb), fake, fake, fake, fake, None, fake, fake, None, fake,
                                 fake, big, None) == 1                  # lse is required
    assert lib.nsa_forward_train(ctypes.byref(cb), fake, fake, fake, fake, None, fake, fake, fake, None,
                                 fake, big, None) == 1                  # o_branch is required
    assert lib.nsa_forward_train(ctypes.byref(cb), fake, fake, fake, fake, None, fake, fake, fake,
                                 ctypes.c_void_p((1 << 20) + 4), fake, big, None) == 1   # misaligned
    assert lib.nsa_forward_train(ctypes.byref(cb), fake, fake, fake, fake, None, fake, fake, fake, fake,
                                 fake, 64, None) == 3                   # workspace too small
    # nsa_backward_saved(cfg, q, k, v, gates, phi, dout, sel_idx, lse, o_branch, dq, dk, dv, dgates,
    #                    ws, bytes, stream)
    args = [fake] * 4
    assert lib.nsa_backward_saved(ctypes.byref(cb), *args, None, fake, fake, None, fake, *args, fake, big,
                                  None) == 1                            # no saved LSE
    assert lib.nsa_backward_saved(ctypes.byref(cb), *args, None, fake, fake, fake, None, *args, fake, big,
                                  None) == 1                            # no saved branch outputs
    assert lib.nsa_backward_saved(ctypes.byref(cb), *args, None, fake, fake, fake, fake, *args, fake, 64,
                                  None) == 3
