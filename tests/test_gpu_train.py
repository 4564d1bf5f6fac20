"""GPU checks of the training pair nsa_forward_train / nsa_backward_saved.

The training forward must return nsa_forward's results bit for bit plus each
branch's own output o_c (before its gate), which is compared with the oracle's
per-branch outputs under the GPU's selection.  The saved-statistics backward
must give the oracle's gradients (relative L2 <= 1e-2) and agree with
nsa_backward, which recomputes the same statistics with the same kernels, up to
the order of its floating-point additions."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close_out, host, phi_params, rel_l2, sample_rows
from sparse_attention_long_phi_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _train_pair(c, check_rows=None):
    from sparse_attention_long_phi_b200 import nsa
    B, T, H, G = c["B"], c["T"], c["H"], c["G"]
    x = I.make_forward_inputs(c, "cuda", with_dout=True)
    ph = phi_params(x)
    ref = nsa.forward(c, x["q"], x["k"], x["v"], x["gates"], ph, want_lse=True)
    tr = nsa.forward_train(c, x["q"], x["k"], x["v"], x["gates"], ph)
    torch.cuda.synchronize()
    nsa.sync_status()
    # same kernels, same arithmetic: bit-identical results
    assert torch.equal(tr["out"], ref["out"])
    assert torch.equal(tr["idx"], ref["idx"])
    assert torch.equal(tr["lse"], ref["lse"])
    # the gated sum of the saved branch outputs is the output
    gates = x["gates"].float()
    recon = sum(gates[..., br:br + 1] * tr["o_branch"][br] for br in range(3))
    assert rel_l2(recon.cpu().numpy(), tr["out"].cpu().numpy()) <= 1e-6
    # each branch's own output against the oracle's, under the GPU's selection
    hx = host(x)
    kc_o, vc_o = oracle.phi(c, hx["k"], hx["v"], hx.get("wk"), hx.get("ek"), hx.get("wv"), hx.get("ev"))
    rows = np.arange(B * T) if check_rows is None else np.asarray(check_rows, np.int64)
    got_idx = tr["idx"].reshape(B * T, G, c["n"]).cpu().numpy()[rows]
    want = oracle.forward_rows(c, hx["q"], hx["k"], hx["v"], hx["gates"], kc_o, vc_o, rows,
                               idx_in=got_idx, want=("out", "obr"))
    obr = tr["o_branch"].reshape(3, B * T, H, c["dv"]).cpu().numpy()[:, rows]
    for br, name in enumerate(("o_cmp", "o_slc", "o_win")):
        assert np.isfinite(obr[br]).all(), name
        assert_close_out(obr[br], want["obr"][:, :, br], name)
    return x, tr


@pytest.mark.parametrize("c", [
    dict(I.WORKLOADS["tiny_fwd_T1024"], T=600, seed=5000),
    dict(I.WORKLOADS["tiny_fwd_T1024"], B=2, T=333, phi="linear", seed=5100),
    dict(I.WORKLOADS["train_fwd_bwd_B2_T16384"], B=1, T=1200, seed=5200),
], ids=["tiny_mean", "tiny_linear_B2", "large_heads_T1200"])
def test_training_pair_against_oracle(c):
    from sparse_attention_long_phi_b200 import nsa
    x, tr = _train_pair(c)
    ph = phi_params(x)
    r = nsa.backward_saved(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], tr["idx"], tr["lse"],
                           tr["o_branch"], ph)
    rr = nsa.backward(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], tr["idx"], ph)
    torch.cuda.synchronize()
    nsa.sync_status()
    hx = host(x)
    want = oracle.backward_tail(c, hx["q"], hx["k"], hx["v"], hx["gates"], hx["dout"],
                                tr["idx"].cpu().numpy(), hx.get("wk"), hx.get("ek"), hx.get("wv"),
                                hx.get("ev"))
    for key in ("dq", "dk", "dv", "dgates"):
        got = r[key].cpu().numpy()
        assert np.isfinite(got).all(), key
        err = rel_l2(got, want[key])
        assert err <= 1e-2, f"{key}: rel L2 {err:.3e} against the oracle"
        same = rel_l2(got, rr[key].cpu().numpy())
        # summation order only; dk/dv through bf16-rounded dK~ (see the full-size test)
        assert same <= (1e-3 if key in ("dk", "dv") else 1e-5), f"{key}: rel L2 {same:.3e} against nsa_backward"
    # d(gate_c) = <dO, o_c> is one dot product of saved values: equal to the recompute's
    assert torch.equal(r["dgates"], rr["dgates"])


def test_training_pair_B2_T16384_full_size():
    """The benchmark's training workload: forward_train's branch outputs on sampled rows
    against the oracle, and the saved-statistics backward against nsa_backward."""
    from sparse_attention_long_phi_b200 import nsa
    c = dict(I.WORKLOADS["train_fwd_bwd_B2_T16384"])
    rows = sample_rows(c["B"], c["T"], 96, seed=11, edge=16)
    x, tr = _train_pair(c, check_rows=rows)
    ph = phi_params(x)
    r = nsa.backward_saved(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], tr["idx"], tr["lse"],
                           tr["o_branch"], ph)
    rr = nsa.backward(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], tr["idx"], ph)
    torch.cuda.synchronize()
    nsa.sync_status()
    # Both runs add the same terms in different orders (atomic accumulation).  dk and dv
    # also take the linear phi's transposed products, whose operand dK~/dV~ is rounded
    # to bf16 after such an fp32 sum: an element near a rounding midpoint can land one
    # bf16 ulp (2^-8 relative) apart in the two runs, hence their looser bound.
    bounds = {"dq": 1e-5, "dk": 1e-3, "dv": 1e-3}
    for key, bound in bounds.items():
        a, b = r[key], rr[key]
        assert torch.isfinite(a).all(), key
        err = float((a - b).norm() / b.norm())
        assert err <= bound, f"{key}: rel L2 {err:.3e} against nsa_backward"
    assert torch.equal(r["dgates"], rr["dgates"])
