"""GPU parity of nsa_forward against the fp64 oracle (same seeded inputs).

Sizes: the tiny configuration in full; ragged and edge shapes in full; the
T=8192 and T=65536 prefill configurations on sampled rows (first/last 64
tokens plus random rows), in the launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

from helpers import check_forward, sample_rows
from sparse_attention_long_phi_b200 import inputs as I

pytestmark = pytest.mark.gpu


def wl(name, **kw):
    c = dict(I.WORKLOADS[name])
    c.update(kw)
    return c


def test_tiny_forward_all_rows():
    rep = {}
    check_forward(wl("tiny_fwd_T1024"), report=rep)


@pytest.mark.parametrize("T", [1000, 333, 64, 31, 20])
def test_ragged_and_short_sequences_small_heads(T):
    # T not a multiple of 8/64; T < l (no compressed block); T < n*l' (all blocks)
    check_forward(wl("tiny_fwd_T1024", T=T, seed=2000 + T))


def test_batch_of_two_and_linear_phi_small_heads():
    check_forward(wl("tiny_fwd_T1024", B=2, T=700, phi="linear", seed=2100))


@pytest.mark.parametrize("l,d", [(64, 64), (16, 16), (64, 32)])
def test_other_compression_blockings(l, d):
    check_forward(wl("tiny_fwd_T1024", T=1500, l=l, d=d, w=100, seed=2200 + l + d))


def test_large_heads_ragged_T():
    c = wl("prefill_fwd_T8192", T=2000, seed=2300)
    check_forward(c)


def test_large_heads_batch2_window_and_n():
    c = wl("prefill_fwd_T8192", B=2, T=1400, w=200, n=8, seed=2400)
    check_forward(c)


def test_prefill_T8192_sampled_rows():
    c = wl("prefill_fwd_T8192")
    rows = sample_rows(1, c["T"], 256, seed=1)
    check_forward(c, rows=rows)


def test_forward_is_deterministic():
    from sparse_attention_long_phi_b200 import nsa
    from helpers import phi_params
    c = wl("prefill_fwd_T8192", T=3000, seed=2500)
    x = I.make_forward_inputs(c, "cuda")
    a = nsa.forward(c, x["q"], x["k"], x["v"], x["gates"], phi_params(x))
    b = nsa.forward(c, x["q"], x["k"], x["v"], x["gates"], phi_params(x))
    torch.cuda.synchronize()
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["idx"], b["idx"])


def test_prefill_T65536_sampled_rows():
    # 4096 query positions: every t < 1024 (the rows where all blocks are
    # candidates and the first compressed blocks appear), the last 64, and
    # seeded uniform draws over the rest
    c = wl("prefill_fwd_T65536")
    T = c["T"]
    rng = np.random.default_rng(2)
    fixed = set(range(1024)) | set(range(T - 64, T))
    rest = rng.choice(np.arange(1024, T - 64), 4096 - len(fixed), replace=False)
    rows = np.array(sorted(fixed | set(int(r) for r in rest)), np.int64)
    assert rows.size == 4096
    rep = {}
    check_forward(c, rows=rows, report=rep)
    print("T=65536 sample:", rep)


def test_prefill_largest_supported_context_sampled_rows():
    # T = 131072, the largest context the library accepts (2048 selection blocks,
    # 64 candidates per top-n lane); first/last tokens and random rows
    c = wl("prefill_fwd_T65536", T=131072, seed=2131)
    rows = sample_rows(1, c["T"], 16, seed=3, edge=8)
    check_forward(c, rows=rows)
