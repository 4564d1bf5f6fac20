"""GPU parity of nsa_backward (and, for the linear phi, nsa_backward_phi_params)
against the fp64 oracle, with the same (valid, seeded) block selection on both
sides.  Gradients: relative L2 <= 1e-2."""
import numpy as np
import pytest
import torch

import oracle
from helpers import host, phi_params, rel_l2
from sparse_attention_long_phi_b200 import inputs as I

pytestmark = pytest.mark.gpu


def run_backward(c, t_lo=0):
    from sparse_attention_long_phi_b200 import nsa
    x = I.make_forward_inputs(c, "cuda", with_dout=True)
    idx = I.random_selection(c, "cuda")
    # the linear phi's parameter gradients need the complete dK~/dV~ (every row): t_lo = 0
    phi_grads = c.get("phi") == "linear" and t_lo == 0
    r = nsa.backward(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], idx, phi_params(x),
                     want_phi_grads=phi_grads)
    torch.cuda.synchronize()
    nsa.sync_status()
    hx = host(x)
    want = oracle.backward_tail(c, hx["q"], hx["k"], hx["v"], hx["gates"], hx["dout"],
                                idx.cpu().numpy(), hx.get("wk"), hx.get("ek"), hx.get("wv"),
                                hx.get("ev"), t_lo=t_lo, want_cmp=phi_grads)
    if phi_grads:
        want.update(oracle.phi_param_grads(c, hx["k"], hx["v"], hx["wk"], hx["ek"], hx["wv"], hx["ev"],
                                           want["dkc"], want["dvc"]))
        for key in ("dwk", "dwv", "dev"):
            got = r[key].cpu().numpy()
            assert np.isfinite(got).all(), key
            err = rel_l2(got, want[key])
            assert err <= 1e-2, f"{key}: rel L2 {err:.3e}"
        # E_K adds one vector, w_k vec(E_K), to every compressed key: the softmax does not
        # see it, so dE_K is zero (each row's dS sums to zero).  The GPU's products take
        # dS rounded to bf16, which leaves a residual of order 2^-9 of the terms
        dek = r["dek"].cpu().numpy()
        assert np.isfinite(dek).all()
        assert np.abs(dek).max() <= 2e-3 * np.abs(want["dwk"]).max()
    for key in ("dq", "dk", "dv", "dgates"):
        got = r[key].cpu().numpy()[:, t_lo:]
        exp = want[key][:, t_lo:]
        assert np.isfinite(got).all(), key
        err = rel_l2(got, exp)
        assert err <= 1e-2, f"{key}: rel L2 {err:.3e}"


def test_backward_small_heads_mean_phi():
    run_backward(dict(I.WORKLOADS["tiny_fwd_T1024"], T=600, seed=4000))


def test_backward_small_heads_linear_phi_batch2():
    run_backward(dict(I.WORKLOADS["tiny_fwd_T1024"], B=2, T=333, phi="linear", seed=4100))


def test_backward_large_heads():
    run_backward(dict(I.WORKLOADS["train_fwd_bwd_B2_T16384"], B=1, T=1200, seed=4200))


def test_backward_B2_T16384_tail():
    # exact for rows and keys at or after t_lo (every gradient of a key comes from later rows)
    run_backward(dict(I.WORKLOADS["train_fwd_bwd_B2_T16384"]), t_lo=16384 - 160)


def test_backward_B2_T16384_full_size_on_sampled_rows():
    """The full B=2, T=16384 backward, in the launch configuration the benchmark
    times, with the upstream gradient kept on a seeded sample of query rows and
    zero elsewhere: the result is then the gradient of the sampled rows alone,
    which the oracle computes row by row.  Every key those rows read is checked
    at full size -- block 0 (selected by every row), the selected blocks, the
    windows and, through phi transposed, the compressed blocks at any position."""
    from sparse_attention_long_phi_b200 import nsa
    c = dict(I.WORKLOADS["train_fwd_bwd_B2_T16384"])
    B, T = c["B"], c["T"]
    x = I.make_forward_inputs(c, "cuda", with_dout=True)
    idx = I.random_selection(c, "cuda")
    rng = np.random.default_rng(7)
    ts = sorted(set([0, 1, 31, 63, 64, 511, 512, 1023, 4095, 8191, T - 1]) |
                set(int(t) for t in rng.integers(0, T, 37)))
    rows = np.array([b * T + t for b in range(B) for t in ts], np.int64)
    keep = torch.zeros(B * T, dtype=torch.bool, device="cuda")
    keep[torch.from_numpy(rows).cuda()] = True
    x["dout"] = (x["dout"].reshape(B * T, -1) * keep[:, None]).reshape(x["dout"].shape).contiguous()
    r = nsa.backward(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], idx, phi_params(x))
    torch.cuda.synchronize()
    nsa.sync_status()
    hx = host(x)
    want = oracle.backward_rows(c, hx["q"], hx["k"], hx["v"], hx["gates"], hx["dout"], idx.cpu().numpy(),
                                rows, hx["wk"], hx["ek"], hx["wv"], hx["ev"])
    on = keep.cpu().numpy()
    for key in ("dq", "dgates"):
        got = r[key].cpu().numpy().reshape(B * T, -1)
        exp = want[key].reshape(B * T, -1)
        assert np.isfinite(got).all(), key
        assert not got[~on].any(), f"{key}: nonzero outside the sampled rows"
        err = rel_l2(got[on], exp[on])
        assert err <= 1e-2, f"{key}: rel L2 {err:.3e}"
    for key in ("dk", "dv"):
        got = r[key].cpu().numpy()
        exp = want[key]
        assert np.isfinite(got).all(), key
        err = rel_l2(got, exp)
        assert err <= 1e-2, f"{key}: rel L2 {err:.3e}"
        for b in range(B):                                 # block 0, read by every row
            e0 = rel_l2(got[b, :64], exp[b, :64])
            assert e0 <= 1e-2, f"{key} block 0 of sequence {b}: rel L2 {e0:.3e}"
        far = np.ones(T, bool)                              # keys outside every sampled window:
        for t in ts:                                        # selected blocks and phi^T only
            far[max(0, t - c["w"] + 1):t + 1] = False
        ef = rel_l2(got[:, far], exp[:, far])
        assert ef <= 1e-2, f"{key} outside the windows: rel L2 {ef:.3e}"
