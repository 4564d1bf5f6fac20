"""Pins of the fp64 oracle to facts other than itself (CPU only).

Each test ties one oracle step to something the pages or the mathematics fix:
library routines (torch's bf16 cast, scaled_dot_product_attention), closed
forms, brute force on tiny inputs, invariants of the definitions, numbers the
pages print (tests/golden/page_numbers.json), and finite differences for the
backward.  A plausible mistake in any step (a dropped term, a wrong sign,
index or tap, a transposed operand) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_phi_b200 import inputs as I

HERE = os.path.dirname(os.path.abspath(__file__))


def small_cfg(**kw):
    c = dict(B=1, T=160, H=4, G=2, dk=16, dv=8, l=8, d=4, lp=16, n=4, fi=1, fl=2, w=24,
             phi="mean", seed=7)
    c.update(kw)
    return c


def make(c, with_dout=False):
    x = I.make_forward_inputs(c, "cpu", with_dout=with_dout)
    out = {k: (I.bits(v) if v.dtype == torch.bfloat16 else v.numpy()) for k, v in x.items()}
    return out


def run_rows(c, x, rows=None, want=("out", "idx", "lse", "obr", "pgrp", "pcmp"), idx_in=None,
             exact=False):
    if rows is None:
        rows = np.arange(c["B"] * c["T"])
    ph = oracle.phi(c, x["k"], x["v"], x.get("wk"), x.get("ek"), x.get("wv"), x.get("ev"),
                    exact=exact)
    kc, vc = (ph[2], ph[3]) if exact else (ph[0], ph[1])
    return oracle.forward_rows(c, x["q"], x["k"], x["v"], x["gates"], kc, vc, rows,
                               idx_in=idx_in, want=want)


def f64(bits):
    return oracle.bf16_to_f64(bits)


def full_causal(q, k, v, scale):
    """library reference: torch SDPA, causal, fp64, GQA by repeating k/v"""
    B, T, H, dk = q.shape
    G = k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(H // G, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(H // G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


# ---------------------------------------------------------------- bf16 cast

def test_bf16_rounding_matches_torch_and_is_single_step():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(4000).astype(np.float32),
                        (rng.standard_normal(2000) * 1e-30).astype(np.float32),
                        np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, 2.0 ** -130])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_round(float(v)) for v in x], np.uint16)
    np.testing.assert_array_equal(got, ref)
    # a value just above a bf16 midpoint rounds up; rounding through fp32 first
    # would land on the midpoint and tie to even (down)
    assert oracle.bf16_round(1 + 2 ** -8 + 2 ** -40) == 0x3F81
    for b in (0x3F80, 0xC2F7, 0x0001, 0x7F7F):
        assert oracle.bf16_round(oracle.bf16_value(b)) == b


# --------------------------------------------------------------------- phi

def test_phi_mean_of_a_ramp_is_its_midpoint():
    c = small_cfg(T=128, G=1, dk=8, dv=8, l=32, d=16, lp=64)
    t = np.arange(128, dtype=np.float32) / 16.0          # exact in bf16
    kf = np.broadcast_to(t[None, :, None, None], (1, 128, 1, 8)).astype(np.float32)
    kb = torch.from_numpy(np.ascontiguousarray(kf)).to(torch.bfloat16)
    kbits = I.bits(kb)
    kc, vc = oracle.phi(c, kbits, kbits)
    C = oracle.num_cmp_blocks(c, 128)
    assert C == (128 - 32) // 16 + 1
    for i in range(C):
        mid = (i * 16 + (32 - 1) / 2) / 16.0              # mean of t/16 over the block
        assert f64(kc[0, i, 0]).tolist() == [mid] * 8


def test_linear_phi_reduces_to_mean_and_selects_positions():
    c = small_cfg(phi="linear", T=96, l=8, d=4, dk=16, dv=8)
    x = make(c)
    l, dk, dv = c["l"], c["dk"], c["dv"]
    # W = (1/l)[I ... I], E = 0 equals mean-pool
    wk = np.tile(np.eye(dk, dtype=np.float32) / l, (1, l))
    wv = np.tile(np.eye(dv, dtype=np.float32) / l, (1, l))
    tb = lambda a: I.bits(torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16))
    zk, zv = np.zeros((l, dk), np.uint16), np.zeros((l, dv), np.uint16)
    kc_lin, vc_lin = oracle.phi(c, x["k"], x["v"], tb(wk), zk, tb(wv), zv)
    kc_mean, vc_mean = oracle.phi(dict(c, phi="mean"), x["k"], x["v"])
    np.testing.assert_array_equal(kc_lin, kc_mean)
    np.testing.assert_array_equal(vc_lin, vc_mean)
    # W selecting position j of the block (position-major flattening), E added
    j = 3
    sel_k = np.zeros((dk, l * dk), np.float32)
    sel_k[:, j * dk:(j + 1) * dk] = np.eye(dk)
    sel_v = np.zeros((dv, l * dv), np.float32)
    sel_v[:, j * dv:(j + 1) * dv] = np.eye(dv)
    kc_sel, _ = oracle.phi(c, x["k"], x["v"], tb(sel_k), x["ek"], tb(sel_v), x["ev"])
    C = oracle.num_cmp_blocks(c, c["T"])
    for i in range(C):
        want = f64(x["k"][0, i * c["d"] + j]) + f64(x["ek"][j])[None, :]
        want_bits = np.array([[oracle.bf16_round(w) for w in row] for row in want], np.uint16)
        np.testing.assert_array_equal(kc_sel[0, i], want_bits)


# ------------------------------------------------------ compressed attention

def test_compressed_branch_is_full_attention_when_l_d_1_and_phi_identity():
    c = small_cfg(phi="linear", l=1, d=1, lp=1, n=200, T=64, dk=16, dv=8, H=4, G=2)
    x = make(c)
    # identity phi: W = I (dk x dk since l = 1), E = 0
    x["wk"] = I.bits(torch.eye(16).to(torch.bfloat16))
    x["wv"] = I.bits(torch.eye(8).to(torch.bfloat16))
    x["ek"] = np.zeros((1, 16), np.uint16)
    x["ev"] = np.zeros((1, 8), np.uint16)
    r = run_rows(c, x)
    ref = full_causal(f64(x["q"]), f64(x["k"]), f64(x["v"]), 1 / math.sqrt(16))
    np.testing.assert_allclose(r["obr"][:, :, 0, :], ref.reshape(-1, 4, 8), rtol=0, atol=1e-12)
    # LSE of the compressed branch = logsumexp of the scaled causal logits
    qd, kd = f64(x["q"])[0], f64(x["k"])[0]
    t, h = 37, 3
    s = (kd[: t + 1, h // 2] @ qd[t, h]) / 4.0
    assert abs(r["lse"][t, h, 0] - (s.max() + np.log(np.exp(s - s.max()).sum()))) < 1e-12


def test_compressed_probabilities_rows_sum_to_one():
    c = small_cfg()
    x = make(c)
    r = run_rows(c, x)
    C = oracle.num_cmp_blocks(c, c["T"])
    for t in range(c["T"]):
        nv = oracle.ncmp_visible(c, t)
        s = r["pcmp"][t].sum(-1)
        if nv == 0:
            assert np.all(r["pcmp"][t] == 0) and np.all(r["obr"][t, :, 0] == 0)
            assert np.all(np.isneginf(r["lse"][t, :, 0]))
        else:
            np.testing.assert_allclose(s, 1.0, atol=1e-12)
            assert np.all(r["pcmp"][t, :, nv:C] == 0)
            # visibility: block i complete, i*d + l - 1 <= t
            assert (nv - 1) * c["d"] + c["l"] - 1 <= t < nv * c["d"] + c["l"] - 1


# ----------------------------------------------------------- score mapping

def test_score_map_identity_when_blockings_equal_and_group_sum():
    c = small_cfg(l=8, d=8, lp=8, n=40)
    x = make(c)
    r = run_rows(c, x)
    Hg = c["H"] // c["G"]
    C = oracle.num_cmp_blocks(c, c["T"])
    for g in range(c["G"]):
        want = r["pcmp"][:, g * Hg:(g + 1) * Hg, :C].sum(1)
        np.testing.assert_allclose(r["pgrp"][:, g, :C], want, atol=1e-13)
    # one head per group: the group score is the head's own mapped score
    c1 = small_cfg(l=8, d=8, lp=8, n=40, H=2, G=2)
    r1 = run_rows(c1, make(c1))
    np.testing.assert_allclose(r1["pgrp"][:, :, :C], r1["pcmp"][:, :, :C], atol=1e-13)


@pytest.mark.parametrize("l,d,lp", [(32, 16, 64), (16, 8, 64), (8, 8, 32), (16, 16, 16)])
def test_score_map_taps_follow_block_geometry(l, d, lp):
    """Make one compressed block dominate (q . K~_i large) so p_cmp is one-hot;
    the group score then equals Hg * (number of stride-d segments of block i
    that fall inside selection block j), computed here from interval overlap."""
    T = 8 * lp
    c = small_cfg(T=T, l=l, d=d, lp=lp, H=2, G=1, dk=16, dv=8, n=T // lp + 1, phi="linear")
    x = make(c)
    dk, dv = 16, 8
    sel_k = np.zeros((dk, l * dk), np.float32)
    sel_k[:, :dk] = np.eye(dk)                              # K~[i] = k[i*d] + E[0]
    x["wk"] = I.bits(torch.from_numpy(sel_k).to(torch.bfloat16))
    x["ek"] = np.zeros((l, dk), np.uint16)
    x["wv"] = I.bits(torch.zeros(dv, l * dv).to(torch.bfloat16))
    k = np.zeros((1, T, 1, dk), np.float32)
    q = np.zeros((1, T, 2, dk), np.float32)
    q[..., 0] = 4.0
    C = oracle.num_cmp_blocks(c, T)
    for i_star in [1, 2, 3, 4, 5, C - 2]:
        k[:] = 0
        k[0, i_star * d, 0, 0] = 30.0                       # logit 4*30/4 = 30
        x["k"] = I.bits(torch.from_numpy(k).to(torch.bfloat16))
        x["q"] = I.bits(torch.from_numpy(q).to(torch.bfloat16))
        t = T - 1
        r = run_rows(c, x, rows=[t])
        for j in range(T // lp):
            lo, hi = max(i_star * d, j * lp), min(i_star * d + l, (j + 1) * lp)
            want = 2 * max(0, hi - lo) / d
            assert abs(r["pgrp"][0, 0, j] - want) < 1e-9, (i_star, j, r["pgrp"][0, 0, j], want)


def test_score_map_row_sums_equal_segments_per_block():
    c = small_cfg()
    r = run_rows(c, make(c))
    Hg = c["H"] // c["G"]
    for t in range(c["T"]):
        if oracle.ncmp_visible(c, t) > 0:
            np.testing.assert_allclose(r["pgrp"][t].sum(-1), Hg * c["l"] / c["d"], rtol=1e-12)


# -------------------------------------------------------------------- top-n

def _brute(c, t, score):
    bt = t // c["lp"]
    cand = list(range(bt + 1))
    if len(cand) <= c["n"]:
        return cand
    forced = set(range(c["fi"])) | set(range(bt - c["fl"] + 1, bt + 1))
    rest = [j for j in cand if j not in forced]
    best = max(itertools.combinations(rest, c["n"] - len(forced)),
               key=lambda s: sum(score[j] for j in s))
    return sorted(forced | set(best))


def test_topn_matches_brute_force_and_structure():
    c = small_cfg(T=200, lp=16, n=6, G=1)
    rng = np.random.default_rng(3)
    rows = np.arange(200)
    NS = oracle.num_sel_blocks(c, 200)
    score = rng.random((200, 1, NS))
    idx = oracle.topn(c, rows, score)
    for t in rows:
        got = [j for j in idx[t, 0] if j >= 0]
        assert got == _brute(c, t, score[t, 0]), t
        bt = t // 16
        assert len(got) == min(c["n"], bt + 1)
        assert got == sorted(got) and 0 in got and bt in got
        assert list(idx[t, 0, len(got):]) == [-1] * (c["n"] - len(got))
    # ties go to the lower block index
    flat = oracle.topn(c, [199], np.ones((1, 1, NS)))
    assert list(flat[0, 0]) == [0, 1, 2, 3, 11, 12]


# ------------------------------------------------ selected / window branches

def test_selected_and_window_equal_full_attention_when_they_cover_everything():
    c = small_cfg(T=96, lp=16, n=6, w=96)                  # n*l' >= T, w >= T
    x = make(c)
    r = run_rows(c, x)
    ref = full_causal(f64(x["q"]), f64(x["k"]), f64(x["v"]), 1 / 4.0).reshape(-1, 4, 8)
    np.testing.assert_allclose(r["obr"][:, :, 1], ref, atol=1e-12)
    np.testing.assert_allclose(r["obr"][:, :, 2], ref, atol=1e-12)
    np.testing.assert_allclose(r["lse"][:, :, 1], r["lse"][:, :, 2], atol=1e-12)


def test_window_is_the_last_w_tokens():
    c = small_cfg(T=64, w=5)
    x = make(c)
    r = run_rows(c, x, rows=[40])
    qd, kd, vd = f64(x["q"])[0, 40], f64(x["k"])[0], f64(x["v"])[0]
    for h in range(4):
        s = kd[36:41, h // 2] @ qd[h] / 4.0
        p = np.exp(s - s.max())
        p /= p.sum()
        np.testing.assert_allclose(r["obr"][0, h, 2], p @ vd[36:41, h // 2], atol=1e-12)


def test_constant_values_give_the_constant_times_gate_sum():
    c = small_cfg(phi="mean")
    x = make(c)
    vconst = np.float32(np.linspace(-1, 1, 8))
    x["v"] = I.bits(torch.from_numpy(np.broadcast_to(vconst, (1, 160, 2, 8)).copy())
                    .to(torch.bfloat16))
    r = run_rows(c, x)
    vb = f64(x["v"][0, 0, 0])
    g = x["gates"].reshape(-1, 4, 3).astype(np.float64)
    for t in range(160):
        gs = g[t].sum(-1) if oracle.ncmp_visible(c, t) > 0 else g[t, :, 1] + g[t, :, 2]
        np.testing.assert_allclose(r["out"][t], gs[:, None] * vb[None, :], atol=1e-12)


def test_one_hot_gates_isolate_branches():
    c = small_cfg()
    x = make(c)
    base = run_rows(c, x)
    for br in range(3):
        g = np.zeros_like(x["gates"])
        g[..., br] = 1.0
        r = run_rows(c, dict(x, gates=g))
        np.testing.assert_allclose(r["out"], base["obr"][:, :, br], atol=0)


# ------------------------------------------------------ pages' token counts

def test_independent_window_keys_and_values():
    # page 2, sliding-window paragraph: the window branch may keep its own keys/values
    c = small_cfg(T=96, lp=16, n=6, w=96)                  # w >= T: the window sees every u <= t
    x = make(c)
    kw = I.bits(I.normal_bf16(99, 1, (1, 96, 2, 16)))
    vw = I.bits(I.normal_bf16(99, 2, (1, 96, 2, 8)))
    kc, vc = oracle.phi(c, x["k"], x["v"])
    rows = np.arange(96)
    want = ("out", "idx", "lse", "obr", "pgrp")
    same = oracle.forward_rows(c, x["q"], x["k"], x["v"], x["gates"], kc, vc, rows, want=want,
                               k_win=x["k"], v_win=x["v"])
    base = oracle.forward_rows(c, x["q"], x["k"], x["v"], x["gates"], kc, vc, rows, want=want)
    for key in want:                                       # passing the shared k/v changes nothing
        np.testing.assert_array_equal(same[key], base[key])
    sep = oracle.forward_rows(c, x["q"], x["k"], x["v"], x["gates"], kc, vc, rows, want=want,
                              k_win=kw, v_win=vw)
    # the window branch is full causal attention over its own keys/values (library)
    ref = full_causal(f64(x["q"]), f64(kw), f64(vw), 1 / 4.0).reshape(-1, 4, 8)
    np.testing.assert_allclose(sep["obr"][:, :, 2], ref, atol=1e-12)
    # the compressed and selected branches, the scores and the selection do not see them
    np.testing.assert_array_equal(sep["obr"][:, :, :2], base["obr"][:, :, :2])
    np.testing.assert_array_equal(sep["idx"], base["idx"])
    np.testing.assert_array_equal(sep["pgrp"], base["pgrp"])
    np.testing.assert_array_equal(sep["lse"][:, :, :2], base["lse"][:, :, :2])
    assert not np.allclose(sep["obr"][:, :, 2], base["obr"][:, :, 2])


def test_token_counts_reproduce_the_pages_numbers():
    gold = json.load(open(os.path.join(HERE, "golden", "page_numbers.json")))
    hp = {k: gold["hyperparameters"][k] for k in ("l", "d", "lp", "n", "fi", "fl", "w")}
    c = dict(hp, B=1, T=65536, H=64, G=4, dk=192, dv=128)
    n64 = sum(oracle.key_counts(c, 65535))
    # the page's count uses 65536/16 compressed tokens; the exact count at the
    # last query is floor((65536-32)/16)+1 = 4095
    assert abs(n64 - gold["tokens_per_query_64k"]["value"]) <= 1
    assert round(65536 / n64, 1) == gold["decode_speedup_64k"]["value"]
    assert round(1 - n64 / 65536, 3) == gold["sparsity_64k"]["value"]
    c32 = dict(c, T=32768)
    g32 = gold["avg_tokens_per_query_32k"]
    counts = np.array([oracle.key_counts(c32, t) for t in range(0, 32768, 7)])
    dec = g32["decomposition"]
    # the page's 2560 = average compressed count + n*l' + w
    assert abs(counts[:, 0].mean() - dec["avg_compressed"]) / dec["avg_compressed"] < 0.01
    assert counts[:, 1].max() == dec["selected_max"] == c["n"] * c["lp"]
    assert counts[:, 2].max() == dec["window_max"] == c["w"]
    assert sum(dec.values()) == g32["value"]
    tot = counts.sum(1).mean()
    assert abs(tot - g32["value"]) / g32["value"] < g32["rel_tol"]


# ---------------------------------------------------------------- decode

def test_decode_equals_forward_at_the_last_position():
    c = small_cfg(phi="mean", T=0)
    lens = [50, 97, 160]
    xs = [make(dict(c, T=L, seed=20 + i)) for i, L in enumerate(lens)]
    kcs = [oracle.phi(dict(c, T=L), x["k"], x["v"]) for L, x in zip(lens, xs)]
    q = np.concatenate([x["q"][0, -1:] for x in xs])
    g = np.concatenate([x["gates"][0, -1:] for x in xs])
    kv_off = np.concatenate([[0], np.cumsum(lens)])
    cmp_off = np.concatenate([[0], np.cumsum([k[0].shape[1] for k in kcs])])
    cat = lambda key: np.concatenate([x[key][0] for x in xs])
    d = oracle.decode(c, q, cat("k"), cat("v"), kv_off, np.concatenate([k[0][0] for k in kcs]),
                      np.concatenate([k[1][0] for k in kcs]), cmp_off, g)
    for s, L in enumerate(lens):
        cs = dict(c, T=L)
        r = oracle.forward_rows(cs, xs[s]["q"], xs[s]["k"], xs[s]["v"], xs[s]["gates"], kcs[s][0],
                                kcs[s][1], [L - 1])
        np.testing.assert_array_equal(d["out"][s], r["out"][0])
        np.testing.assert_array_equal(d["idx"][s], r["idx"][0])
    with pytest.raises(ValueError):
        oracle.decode(c, q, cat("k"), cat("v"), kv_off, np.concatenate([k[0][0] for k in kcs]),
                      np.concatenate([k[1][0] for k in kcs]), cmp_off + np.array([0, 1, 1, 1]), g)


# --------------------------------------------------------------- backward

def _loss(c, x, idx, exact=True):
    """sum(dO * out) with the selection held fixed, from the oracle forward"""
    r = run_rows(dict(c, cmp_exact=1), x, want=("out",), idx_in=idx.reshape(-1, c["G"], c["n"]),
                 exact=exact)
    dO = f64(x["dout"]).reshape(r["out"].shape)
    return float((dO * r["out"]).sum())


@pytest.mark.parametrize("phi", ["mean", "linear"])
def test_backward_matches_central_differences(phi):
    c = small_cfg(T=56, H=2, G=1, dk=8, dv=8, l=8, d=4, lp=8, n=3, w=9, phi=phi)
    x = make(c, with_dout=True)
    idx = oracle.forward_rows(c, x["q"], x["k"], x["v"], x["gates"],
                              *oracle.phi(c, x["k"], x["v"], x.get("wk"), x.get("ek"), x.get("wv"),
                                          x.get("ev")), np.arange(56))["idx"].reshape(1, 56, 1, 3)
    rng = np.random.default_rng(11)
    eps = 2.0 ** -10
    checks = ([("q", (0, t, h, ch)) for t, h, ch in zip(rng.integers(0, 56, 6), rng.integers(0, 2, 6),
                                                        rng.integers(0, 8, 6))] +
              [("k", (0, t, 0, ch)) for t, ch in zip(rng.integers(0, 56, 8), rng.integers(0, 8, 8))] +
              [("v", (0, t, 0, ch)) for t, ch in zip(rng.integers(0, 56, 8), rng.integers(0, 8, 8))])
    for name, pos in checks:
        xz = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in x.items()}
        xz[name][pos] = 0                                   # expand around 0 so +-eps is exact
        g = oracle.backward_tail(dict(c, cmp_exact=1), xz["q"], xz["k"], xz["v"], xz["gates"],
                                 xz["dout"], idx, xz.get("wk"), xz.get("ek"), xz.get("wv"),
                                 xz.get("ev"))
        vals = []
        for sgn in (1, -1):
            xp = dict(xz)
            xp[name] = xz[name].copy()
            xp[name][pos] = oracle.bf16_round(sgn * eps)
            vals.append(_loss(c, xp, idx))
        fd = (vals[0] - vals[1]) / (2 * eps)
        an = g["d" + name][pos]
        assert abs(fd - an) <= 1e-6 + 1e-5 * abs(an), (name, pos, fd, an)
    # d(gates) = <dO, o_c> and equals the derivative in the gate
    g = oracle.backward_tail(dict(c, cmp_exact=1), x["q"], x["k"], x["v"], x["gates"], x["dout"],
                             idx, x.get("wk"), x.get("ek"), x.get("wv"), x.get("ev"))
    r = run_rows(dict(c, cmp_exact=1), x, want=("out", "obr"), idx_in=idx.reshape(-1, 1, 3),
                 exact=True)
    dO = f64(x["dout"]).reshape(56, 2, 8)
    np.testing.assert_allclose(g["dgates"].reshape(56, 2, 3),
                               np.einsum("thc,thbc->thb", dO, r["obr"]), atol=1e-12)


def test_phi_parameter_gradients_match_central_differences():
    # token compression: K~[i] = W vec(k_blk + E); dW and dE from the backward's dK~, dV~
    c = small_cfg(T=56, H=2, G=1, dk=8, dv=8, l=8, d=4, lp=8, n=3, w=9, phi="linear")
    x = make(c, with_dout=True)
    idx = oracle.forward_rows(c, x["q"], x["k"], x["v"], x["gates"],
                              *oracle.phi(c, x["k"], x["v"], x["wk"], x["ek"], x["wv"], x["ev"]),
                              np.arange(56))["idx"].reshape(1, 56, 1, 3)
    rng = np.random.default_rng(12)
    eps = 2.0 ** -10
    checks = ([("wk", (o, e)) for o, e in zip(rng.integers(0, 8, 5), rng.integers(0, 64, 5))] +
              [("ek", (j, ch)) for j, ch in zip(rng.integers(0, 8, 5), rng.integers(0, 8, 5))] +
              [("wv", (o, e)) for o, e in zip(rng.integers(0, 8, 5), rng.integers(0, 64, 5))] +
              [("ev", (j, ch)) for j, ch in zip(rng.integers(0, 8, 5), rng.integers(0, 8, 5))])
    for name, pos in checks:
        xz = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in x.items()}
        xz[name][pos] = 0                                   # expand around 0 so +-eps is exact
        g = oracle.backward_tail(dict(c, cmp_exact=1), xz["q"], xz["k"], xz["v"], xz["gates"], xz["dout"],
                                 idx, xz["wk"], xz["ek"], xz["wv"], xz["ev"], want_cmp=True)
        pg = oracle.phi_param_grads(c, xz["k"], xz["v"], xz["wk"], xz["ek"], xz["wv"], xz["ev"],
                                    g["dkc"], g["dvc"])
        vals = []
        for sgn in (1, -1):
            xp = dict(xz)
            xp[name] = xz[name].copy()
            xp[name][pos] = oracle.bf16_round(sgn * eps)
            vals.append(_loss(c, xp, idx))
        fd = (vals[0] - vals[1]) / (2 * eps)
        an = pg["d" + name][pos]
        assert abs(fd - an) <= 1e-6 + 1e-5 * abs(an), (name, pos, fd, an)
    # closed form: E_K shifts every compressed key by the same vector w_k vec(E_K), which
    # the softmax does not see, so dE_K = 0 (each row's dS sums to zero); E_V shifts every
    # output by w_v vec(E_V) weighted by the gate, so dE_V does not vanish
    assert np.abs(pg["dwk"]).max() > 0
    assert np.abs(pg["dek"]).max() <= 1e-12 * np.abs(pg["dwk"]).max()
    assert np.abs(pg["dev"]).max() > 1e-6


def test_backward_tail_is_exact_above_the_cut():
    c = small_cfg(T=80, H=2, G=1, dk=8, dv=8, l=8, d=4, lp=8, n=3, w=9, phi="linear")
    x = make(c, with_dout=True)
    idx = I.random_selection(dict(c, seed=3)).numpy()
    full = oracle.backward_tail(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], idx, x["wk"],
                                x["ek"], x["wv"], x["ev"])
    tail = oracle.backward_tail(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], idx, x["wk"],
                                x["ek"], x["wv"], x["ev"], t_lo=50)
    for key in ("dq", "dk", "dv", "dgates"):
        np.testing.assert_array_equal(full[key][:, 50:], tail[key][:, 50:])


@pytest.mark.parametrize("l,d,lp", [(32, 16, 64), (16, 8, 64), (8, 8, 32)])
def test_unweighted_score_map_counts_each_overlapping_block_once(l, d, lp):
    """score_map = 1, the unweighted reading of the blockings-differ paragraph:
    with p_cmp one-hot at block i*, selection block j scores Hg for every j that
    block i* overlaps (interval overlap > 0) and 0 elsewhere."""
    T = 8 * lp
    c = small_cfg(T=T, l=l, d=d, lp=lp, H=2, G=1, dk=16, dv=8, n=T // lp + 1, phi="linear",
                  score_map=1)
    x = make(c)
    dk, dv = 16, 8
    sel_k = np.zeros((dk, l * dk), np.float32)
    sel_k[:, :dk] = np.eye(dk)
    x["wk"] = I.bits(torch.from_numpy(sel_k).to(torch.bfloat16))
    x["ek"] = np.zeros((l, dk), np.uint16)
    x["wv"] = I.bits(torch.zeros(dv, l * dv).to(torch.bfloat16))
    k = np.zeros((1, T, 1, dk), np.float32)
    q = np.zeros((1, T, 2, dk), np.float32)
    q[..., 0] = 4.0
    C = oracle.num_cmp_blocks(c, T)
    for i_star in [1, 3, 4, C - 2]:
        k[:] = 0
        k[0, i_star * d, 0, 0] = 30.0
        x["k"] = I.bits(torch.from_numpy(k).to(torch.bfloat16))
        x["q"] = I.bits(torch.from_numpy(q).to(torch.bfloat16))
        r = run_rows(c, x, rows=[T - 1])
        for j in range(T // lp):
            lo, hi = max(i_star * d, j * lp), min(i_star * d + l, (j + 1) * lp)
            want = 2.0 if hi > lo else 0.0
            assert abs(r["pgrp"][0, 0, j] - want) < 1e-9, (i_star, j, r["pgrp"][0, 0, j], want)


def test_backward_rows_is_the_backward_of_the_listed_rows_only():
    """Restricting the backward to a row set R is the backward with dout zeroed
    outside R (the loss sum_t <dout_t, out_t> is linear in dout): checked against
    the full backward of such a dout, and the full list equals the full backward."""
    c = small_cfg(T=96, H=4, G=2, dk=8, dv=8, l=8, d=4, lp=8, n=4, w=11, phi="linear", B=2)
    x = make(c, with_dout=True)
    idx = I.random_selection(dict(c, seed=5)).numpy()
    B, T = c["B"], c["T"]
    rows = np.array([0, 7, 31, 50, 95, T + 3, T + 64, 2 * T - 1])
    dz = np.zeros_like(x["dout"]).reshape(B * T, -1)
    dz[rows] = x["dout"].reshape(B * T, -1)[rows]
    dz = dz.reshape(x["dout"].shape)
    args = (x["wk"], x["ek"], x["wv"], x["ev"])
    full = oracle.backward_tail(c, x["q"], x["k"], x["v"], x["gates"], dz, idx, *args, want_cmp=True)
    part = oracle.backward_rows(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], idx, rows, *args,
                                want_cmp=True)
    for key in ("dq", "dk", "dv", "dkc", "dvc"):
        np.testing.assert_allclose(part[key], full[key], rtol=1e-12, atol=1e-14, err_msg=key)
    on = np.zeros(B * T, bool)
    on[rows] = True
    ref = oracle.backward_tail(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], idx, *args)
    dg = part["dgates"].reshape(B * T, -1)
    np.testing.assert_array_equal(dg[on], ref["dgates"].reshape(B * T, -1)[on])
    assert not dg[~on].any()
    every = oracle.backward_rows(c, x["q"], x["k"], x["v"], x["gates"], x["dout"], idx, np.arange(B * T), *args)
    for key in ("dq", "dk", "dv", "dgates"):
        np.testing.assert_array_equal(every[key], ref[key])
