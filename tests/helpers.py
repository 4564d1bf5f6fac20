"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare.

Tolerances (from the operator's contract): bf16-in / fp32-accumulate outputs
max abs error <= 2e-2 and relative L2 error <= 5e-3; gradients relative L2
<= 1e-2; selected block indices bit-exact except at near-ties.

Near-ties.  The selection is decided on fp32 scores by the kernel and on fp64
scores by the oracle.  Where the two index sets differ, the GPU's set is
accepted when it is also optimal, up to a relative slack, under the oracle's
own scores: every block only the GPU chose scores at least
(1 - eps) x every block only the oracle chose.  eps = 1e-5 plus the largest
effect the compressed keys can have on the scores: the kernel's K~ may differ
from the oracle's by 1 bf16 ulp (fp32 vs fp64 accumulation before rounding),
which moves a logit by at most delta = scale * |q . dK~| and a ratio of two
scores by at most exp(4 delta).  delta is measured per row from the actual
K~ differences, so it is 0 wherever the keys agree.  Rows whose GPU set is
accepted are then compared under the GPU's set (the oracle recomputes them
with it); rows that fail fail the test.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from sparse_attention_long_phi_b200 import inputs as I


def f64(bits):
    return oracle.bf16_to_f64(bits)


def bf16_ulp_diff(a_bits, b_bits):
    """|a - b| in bf16 ulps (same-sign values; sign changes count as large)."""
    a = a_bits.astype(np.int32)
    b = b_bits.astype(np.int32)
    sa, sb = a >> 15, b >> 15
    ma, mb = a & 0x7FFF, b & 0x7FFF
    oa = np.where(sa == 1, -ma, ma)
    ob = np.where(sb == 1, -mb, mb)
    return np.abs(oa - ob)


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_close_out(got, want, what="out", max_abs=2e-2, rl2=5e-3):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want).max() if got.size else 0.0
    r = rel_l2(got, want)
    assert err <= max_abs and r <= rl2, f"{what}: max abs {err:.3e}, rel L2 {r:.3e}"


def host(x: dict) -> dict:
    return {k: (I.bits(v) if v.dtype == torch.bfloat16 else v.detach().cpu().numpy())
            for k, v in x.items()}


def phi_params(x):
    return {k: x[k] for k in ("wk", "ek", "wv", "ev")} if "wk" in x else None


def selection_ok(c, q_row, pg, got, want, delta):
    """GPU index row `got` vs oracle `want` for one (row, group); pg = oracle scores."""
    A = set(int(j) for j in got if j >= 0) - set(int(j) for j in want if j >= 0)
    B = set(int(j) for j in want if j >= 0) - set(int(j) for j in got if j >= 0)
    if not A and not B:
        return True
    if len(A) != len(B):
        return False
    eps = 1e-5 + (math.exp(4 * delta) - 1)
    return min(pg[j] for j in A) >= max(pg[j] for j in B) * (1 - eps)


def check_forward(c: dict, rows=None, device="cuda", x=None, report=None):
    """Run nsa_forward on the workload, compare with the oracle on `rows`."""
    from sparse_attention_long_phi_b200 import nsa
    B, T, H, G, n = c["B"], c["T"], c["H"], c["G"], c["n"]
    if x is None:
        x = I.make_forward_inputs(c, device)
    r = nsa.forward(c, x["q"], x["k"], x["v"], x["gates"], phi_params(x), want_lse=True, want_kc=True)
    torch.cuda.synchronize()
    nsa.sync_status()
    hx = host(x)
    C = oracle.num_cmp_blocks(c, T)
    kc_o, vc_o = oracle.phi(c, hx["k"], hx["v"], hx.get("wk"), hx.get("ek"), hx.get("wv"), hx.get("ev"))
    dK = np.zeros(kc_o.shape)
    if C > 0:
        kc_g = I.bits(r["kc"][:, :C].contiguous())
        vc_g = I.bits(r["vc"][:, :C].contiguous())
        uk, uv = bf16_ulp_diff(kc_g, kc_o), bf16_ulp_diff(vc_g, vc_o)
        assert uk.max() <= 1 and uv.max() <= 1, f"phi: {uk.max()} / {uv.max()} ulp"
        assert (uk > 0).mean() < 1e-2 and (uv > 0).mean() < 1e-2
        if c.get("phi", "mean") == "mean":
            assert uk.max() == 0 and uv.max() == 0, "mean phi must be correctly rounded"
        dK = f64(kc_g) - f64(kc_o)
    if rows is None:
        rows = np.arange(B * T)
    rows = np.asarray(rows, np.int64)
    want = oracle.forward_rows(c, hx["q"], hx["k"], hx["v"], hx["gates"], kc_o, vc_o, rows,
                               want=("out", "idx", "lse", "pgrp"))
    got_idx = r["idx"].reshape(B * T, G, n).cpu().numpy()[rows]
    Hg = H // G
    scale = c.get("scale", 0) or 1 / math.sqrt(c["dk"])
    qd = None
    bad, fixed = [], []
    for a in range(rows.size):
        for g in range(G):
            if np.array_equal(got_idx[a, g], want["idx"][a, g]):
                continue
            b, t = divmod(int(rows[a]), T)
            nv = oracle.ncmp_visible(c, t)
            delta = 0.0
            if nv > 0 and np.any(dK[b, :nv, g]):
                if qd is None:
                    qd = {}
                qr = f64(hx["q"][b, t, g * Hg:(g + 1) * Hg])
                delta = scale * float(np.abs(qr @ dK[b, :nv, g].T).max())
            if selection_ok(c, None, want["pgrp"][a, g], got_idx[a, g], want["idx"][a, g], delta):
                fixed.append(a)
            else:
                bad.append((int(rows[a]), g, got_idx[a, g].tolist(), want["idx"][a, g].tolist()))
    assert not bad, f"{len(bad)} selection mismatches beyond near-ties, e.g. {bad[:3]}"
    if fixed:
        fixed = np.unique(fixed)
        redo = oracle.forward_rows(c, hx["q"], hx["k"], hx["v"], hx["gates"], kc_o, vc_o,
                                   rows[fixed], idx_in=got_idx[fixed], want=("out", "idx", "lse"))
        want["out"][fixed] = redo["out"]
        want["lse"][fixed] = redo["lse"]
    out_g = r["out"].reshape(B * T, H, c["dv"]).cpu().numpy()[rows]
    assert np.isfinite(out_g).all()
    assert_close_out(out_g, want["out"])
    lse_g = r["lse"].reshape(B * T, H, 3).cpu().numpy()[rows]
    fin = np.isfinite(want["lse"])
    assert np.array_equal(np.isfinite(lse_g), fin), "lse: -inf pattern differs"
    assert np.abs(lse_g[fin] - want["lse"][fin]).max() <= 2e-3, "lse"
    if report is not None:
        report.update(near_ties=len(fixed), rows=int(rows.size))
    return r, x


def sample_rows(B, T, k, seed=0, edge=64):
    """first/last `edge` tokens of every batch plus k random rows"""
    rng = np.random.default_rng(seed)
    s = set()
    for b in range(B):
        s.update(b * T + t for t in range(min(edge, T)))
        s.update(b * T + t for t in range(max(0, T - edge), T))
    s.update(int(v) for v in rng.integers(0, B * T, k))
    return np.array(sorted(s), np.int64)
