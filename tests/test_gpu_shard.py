"""Group sharding of one sequence through libnsa on the GPU: the operator run on
each rank's contiguous range of GQA groups (here one after another on one GPU)
gives, concatenated along the heads, exactly the single-run result -- outputs,
selections and softmax statistics bit for bit -- because the selection and all
three branches are per group (page 2, 重要性分数计算: scores summed over a
group's heads; every head of the group attends the same blocks)."""
import pytest
import torch

from helpers import phi_params
from sparse_attention_long_phi_b200 import inputs as I
from sparse_attention_long_phi_b200 import shard

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4])
def test_group_slices_concatenate_to_the_full_run(world):
    from sparse_attention_long_phi_b200 import nsa
    c = dict(I.WORKLOADS["prefill_fwd_T8192"], T=4100, seed=7100)
    x = I.make_forward_inputs(c, "cuda")
    full = nsa.forward(c, x["q"], x["k"], x["v"], x["gates"], phi_params(x))
    outs, idxs, lses = [], [], []
    for rank in range(world):
        g0, g1 = shard.group_range(c["G"], rank, world)
        cs, xs = shard.slice_groups(c, x, g0, g1)
        r = nsa.forward(cs, xs["q"], xs["k"], xs["v"], xs["gates"], phi_params(xs))
        outs.append(r["out"])
        idxs.append(r["idx"])
        lses.append(r["lse"])
    torch.cuda.synchronize()
    nsa.sync_status()
    assert torch.equal(torch.cat(idxs, dim=2), full["idx"])
    assert torch.equal(torch.cat(outs, dim=2), full["out"])
    assert torch.equal(torch.cat(lses, dim=2), full["lse"])
