"""nsa_compress_static: token compression for callers that cannot allocate
device memory (graph-captured loops, plugins whose host framework owns all
device memory).  It must produce exactly what nsa_compress produces, call
after call, while sharing one fixed device scratch array."""
import pytest
import torch

from sparse_attention_long_phi_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _call_static(nsa, c, x):
    phi = {n: x[n] for n in ("wk", "ek", "wv", "ev")} if "wk" in x else None
    return nsa.compress_static(c, x["k"], x["v"], phi)


@pytest.mark.parametrize("name,T,seed", [("prefill_fwd_T8192", 8192, 5000), ("tiny_fwd_T1024", 1024, 5001)])
def test_static_compress_matches_workspace_compress_twice(name, T, seed):
    from sparse_attention_long_phi_b200 import nsa
    for call in range(2):   # two calls in a row: the shared scratch must not leak state
        c = dict(I.WORKLOADS[name], T=T, seed=seed + call)
        x = I.make_forward_inputs(c, "cuda")
        phi = {n: x[n] for n in ("wk", "ek", "wv", "ev")} if "wk" in x else None
        rc, kc, vc = _call_static(nsa, c, x)
        assert rc == 0, rc
        kref, vref = nsa.compress(c, x["k"], x["v"], phi)
        torch.cuda.synchronize()
        nsa.sync_status()
        assert torch.equal(kc.view(torch.int16), kref.contiguous().view(torch.int16))
        assert torch.equal(vc.view(torch.int16), vref.contiguous().view(torch.int16))


def test_static_compress_rejects_sizes_beyond_its_scratch():
    from sparse_attention_long_phi_b200 import nsa
    c = dict(I.WORKLOADS["prefill_fwd_T65536"])     # 5.2M compressed elements > 16 MiB of scratch
    x = I.make_forward_inputs(c, "cuda")            # real tensors of the right sizes
    phi = {n: x[n] for n in ("wk", "ek", "wv", "ev")}
    rc, kc, vc = nsa.compress_static(c, x["k"], x["v"], phi)
    torch.cuda.synchronize()
    assert rc == 3                                   # NSA_ERR_WORKSPACE, nothing launched
    assert torch.isnan(kc.float()).all() and torch.isnan(vc.float()).all()
