"""The seeded input generator shared by the tests, the bench and the oracle
(sparse_attention_long_phi_b200/inputs.py): reproducible, slice-consistent,
with the stated distributions, and producing valid structured inputs (block
selections, decode offsets).  CPU only."""
import math

import numpy as np
import torch

import oracle
from sparse_attention_long_phi_b200 import inputs as I


def test_generator_is_reproducible_and_slice_consistent():
    a = I.normal64(7, 3, 5000)
    b = I.normal64(7, 3, 5000)
    assert torch.equal(a, b)
    # element k does not depend on where the draw starts
    assert torch.equal(I.normal64(7, 3, 1000, start=2000), a[2000:3000])
    assert torch.equal(I.uniform64(7, 3, 100, start=50), I.uniform64(7, 3, 150)[50:])
    # streams and seeds are independent draws
    assert not torch.equal(I.normal64(7, 4, 5000), a)
    assert not torch.equal(I.normal64(8, 3, 5000), a)


def test_distributions():
    z = I.normal64(11, 1, 400_000).numpy()
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    assert abs((np.abs(z) < 1).mean() - 0.6827) < 0.005           # one-sigma mass
    u = I.uniform64(11, 2, 400_000).numpy()
    assert u.min() >= 0.0 and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 0.005 and abs(u.var() - 1 / 12) < 0.002
    # bf16 tensors are the round-to-nearest-even cast of the fp32 values
    x = I.normal_bf16(11, 1, (1000,), std=0.5)
    ref = (I.normal64(11, 1, 1000) * 0.5).to(torch.float32).to(torch.bfloat16)
    assert torch.equal(x.view(torch.int16), ref.view(torch.int16))


def test_phi_parameters_have_the_stated_scales():
    c = dict(I.WORKLOADS["prefill_fwd_T8192"])
    p = I.make_phi_params(c)
    l, dk, dv = c["l"], c["dk"], c["dv"]
    assert p["wk"].shape == (dk, l * dk) and p["ek"].shape == (l, dk)
    assert p["wv"].shape == (dv, l * dv) and p["ev"].shape == (l, dv)
    assert abs(p["wk"].float().std().item() * math.sqrt(l * dk) - 1.0) < 0.02
    assert abs(p["wv"].float().std().item() * math.sqrt(l * dv) - 1.0) < 0.02
    assert abs(p["ek"].float().std().item() - 1.0) < 0.1


def test_random_selection_is_valid():
    c = dict(I.WORKLOADS["tiny_fwd_T1024"], B=2, T=700, G=2, n=5, seed=9)
    sel = I.random_selection(c).numpy()
    B, T, G, n, lp, fi, fl = c["B"], c["T"], c["G"], c["n"], c["lp"], c["fi"], c["fl"]
    assert sel.shape == (B, T, G, n)
    for b in range(B):
        for t in range(T):
            bt = t // lp
            for g in range(G):
                row = sel[b, t, g]
                got = row[row >= 0]
                assert np.all(row[len(got):] == -1)                  # -1 padding at the end
                assert np.all(np.diff(got) > 0)                      # ascending, distinct
                assert len(got) == min(n, bt + 1)
                assert got.min() >= 0 and got.max() <= bt            # causal candidates
                forced = set(range(fi)) | set(range(max(0, bt - fl + 1), bt + 1))
                assert forced & set(range(bt + 1)) <= set(got.tolist())


def test_decode_inputs_offsets_match_the_lengths():
    c = dict(I.WORKLOADS["decode_S32_L8k_64k"], S=5)
    L = I.decode_lengths(c)
    assert L.min() >= c["Lmin"] and L.max() <= c["Lmax"]
    x = I.make_decode_inputs(c, lambda n: oracle.num_cmp_blocks(c, n), "cpu", lengths=[1, 31, 32, 100, 4000])
    assert np.array_equal(np.diff(x["kv_off"]), [1, 31, 32, 100, 4000])
    assert np.array_equal(np.diff(x["cmp_off"]), [oracle.num_cmp_blocks(c, n) for n in (1, 31, 32, 100, 4000)])
    assert x["k_cache"].shape == (int(x["kv_off"][-1]), c["G"], c["dk"])
    assert x["kc_cache"].shape == (int(x["cmp_off"][-1]), c["G"], c["dk"])
    g = x["gates"]
    assert g.shape == (5, c["H"], 3) and float(g.min()) > 0 and float(g.max()) < 1
