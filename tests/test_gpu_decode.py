"""GPU parity of nsa_decode against the fp64 oracle.  The compressed cache
is an input of the decode step; it is drawn from the seeded generator with the
distribution of a linear phi output, so both sides read identical caches and
the selection must match exactly except at near-ties."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close_out, host, near_tie_bound, selection_ok, selections_valid
from sparse_attention_long_phi_b200 import inputs as I

pytestmark = pytest.mark.gpu


def run_decode(c, lengths=None):
    from sparse_attention_long_phi_b200 import nsa
    cmp_len = lambda L: oracle.num_cmp_blocks(c, L)
    x = I.make_decode_inputs(c, cmp_len, "cuda", lengths=lengths)
    Lmax = int(x["lengths"].max())
    kv_off = torch.from_numpy(x["kv_off"]).cuda()
    cmp_off = torch.from_numpy(x["cmp_off"]).cuda()
    r = nsa.decode(c, x["q"], x["k_cache"], x["v_cache"], kv_off, x["kc_cache"], x["vc_cache"],
                   cmp_off, x["gates"], max_len=Lmax)
    torch.cuda.synchronize()
    nsa.sync_status()
    hx = host({k: v for k, v in x.items() if isinstance(v, torch.Tensor)})
    want = oracle.decode(c, hx["q"], hx["k_cache"], hx["v_cache"], x["kv_off"], hx["kc_cache"],
                         hx["vc_cache"], x["cmp_off"], hx["gates"], want_pgrp=True)
    got_idx = r["idx"].cpu().numpy()
    S, G = got_idx.shape[:2]
    ts = np.asarray(x["lengths"], np.int64) - 1          # each sequence's query position
    selections_valid(c, ts, got_idx)
    fixed = []
    for s in range(S):
        for g in range(G):
            if not np.array_equal(got_idx[s, g], want["idx"][s, g]):
                assert selection_ok(c, ts[s], want["pgrp"][s, g], got_idx[s, g], want["idx"][s, g], 0.0), \
                    (s, g, got_idx[s, g], want["idx"][s, g])
                fixed.append(s)
    print(f"decode near-tie selections accepted: {len(fixed)} of {S * G}")
    assert len(fixed) <= near_tie_bound(S * G)
    if fixed:
        # recompute those sequences under the GPU's (valid) selection
        for s in sorted(set(fixed)):
            L = int(x["lengths"][s])
            cs = dict(c, B=1, T=L)
            k0, k1 = x["kv_off"][s], x["kv_off"][s + 1]
            c0, c1 = x["cmp_off"][s], x["cmp_off"][s + 1]
            qq = np.zeros((1, L, c["H"], c["dk"]), np.uint16)
            qq[0, L - 1] = hx["q"][s]
            gg = np.zeros((1, L, c["H"], 3), np.float32)
            gg[0, L - 1] = hx["gates"][s]
            rr = oracle.forward_rows(cs, qq, hx["k_cache"][k0:k1][None], hx["v_cache"][k0:k1][None],
                                     gg, hx["kc_cache"][c0:c1][None], hx["vc_cache"][c0:c1][None],
                                     [L - 1], idx_in=got_idx[s][None])
            want["out"][s] = rr["out"][0]
            want["lse"][s] = rr["lse"][0]
    out = r["out"].cpu().numpy()
    assert np.isfinite(out).all()
    assert_close_out(out, want["out"])
    lse = r["lse"].cpu().numpy()
    fin = np.isfinite(want["lse"])
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.abs(lse[fin] - want["lse"][fin]).max() <= 2e-3
    return r


def test_decode_small_heads_short_contexts():
    c = dict(I.WORKLOADS["tiny_fwd_T1024"], kind="decode", S=5, seed=3000)
    run_decode(c, lengths=[1, 20, 33, 700, 2500])


def test_decode_large_heads_mixed_lengths():
    c = dict(I.WORKLOADS["decode_S32_L8k_64k"], S=6, seed=3100)
    run_decode(c, lengths=[31, 64, 1025, 1100, 5000, 9000])


def test_decode_S32_full_configuration():
    run_decode(dict(I.WORKLOADS["decode_S32_L8k_64k"]))
