"""Independent keys and values per branch (page 2, 滑动窗口): nsa_forward_branches
against the oracle given the three branches' own keys/values, and equal to
nsa_forward bit for bit when one k/v is passed to every branch."""
import pytest
import torch

from helpers import check_forward, phi_params
from sparse_attention_long_phi_b200 import inputs as I

pytestmark = pytest.mark.gpu


def test_branches_tiny_configuration_all_rows():
    check_forward(dict(I.WORKLOADS["tiny_fwd_T1024"], seed=8000), branches=True)


def test_branches_ragged_linear_phi_batch2():
    check_forward(dict(I.WORKLOADS["tiny_fwd_T1024"], B=2, T=777, phi="linear", seed=8100), branches=True)


def test_branches_prefill_T8192_sampled_rows():
    from helpers import sample_rows
    c = dict(I.WORKLOADS["prefill_fwd_T8192"], seed=8200)
    check_forward(c, rows=sample_rows(1, c["T"], 256, seed=5), branches=True)


def test_branches_with_shared_keys_equal_the_shared_forward():
    from sparse_attention_long_phi_b200 import nsa
    c = dict(I.WORKLOADS["prefill_fwd_T8192"], T=3000, seed=8300)
    x = I.make_forward_inputs(c, "cuda")
    kv = {n: x[n[0]] for n in ("k_cmp", "v_cmp", "k_slc", "v_slc", "k_win", "v_win")}
    a = nsa.forward(c, x["q"], x["k"], x["v"], x["gates"], phi_params(x))
    b = nsa.forward_branches(c, x["q"], kv, x["gates"], phi_params(x))
    torch.cuda.synchronize()
    nsa.sync_status()
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["idx"], b["idx"])
    assert torch.equal(a["lse"], b["lse"])
