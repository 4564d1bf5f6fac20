"""Top-n block selection on its own (nsa_select_blocks) against the oracle's
top-n, bit-exact, on crafted score tables: random scores, heavy ties, rows of
zeros, a heavy-tailed mix, and scores concentrated in one candidate lane (so
that both the threshold-and-sort path and the round-by-round path of the
kernel are taken).  The oracle decides on the same values (fp32 scores widened
to fp64), so every selection must match exactly.

Reference: page 2 (硬件对齐+原生训练！DeepSeek NSA打造高效稀疏Attention),
Top-n 块选择 and its hyperparameter paragraph (1 initial + 2 local blocks
always selected)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_phi_b200 import inputs as I

pytestmark = pytest.mark.gpu

BASE = I.WORKLOADS["prefill_fwd_T8192"]


def _nsa():
    from sparse_attention_long_phi_b200 import nsa
    return nsa


def _scores(kind, rng, shape):
    B, T, G, NS = shape
    if kind == "uniform":
        s = rng.random(shape)
    elif kind == "ties":
        s = rng.integers(0, 4, shape).astype(np.float64)
    elif kind == "sparse":
        s = np.zeros(shape)
        s.reshape(-1)[rng.integers(0, s.size, s.size // 50)] = 1.0
    elif kind == "zeros":
        s = np.zeros(shape)
    elif kind == "heavy":
        s = np.exp(rng.normal(0.0, 3.0, shape))
    elif kind == "one_lane":
        s = rng.random(shape)
        s[..., 4::32] += 2.0           # every 32nd block after the initial one: one lane wins all
    elif kind == "tiny":
        s = rng.integers(0, 8, shape) * 1e-42   # fp32 subnormals
    else:
        raise ValueError(kind)
    return s.astype(np.float32)


def _check(c, kind, seed, nrows=None):
    nsa = _nsa()
    B, T, G = c["B"], c["T"], c["G"]
    NS = -(-T // c["lp"])
    rng = np.random.default_rng(seed)
    s = _scores(kind, rng, (B, T, G, NS))
    got = nsa.select_blocks(c, torch.from_numpy(s).cuda()).cpu().numpy().reshape(B * T, G, c["n"])
    torch.cuda.synchronize()
    nsa.sync_status()
    rows = np.arange(B * T) if nrows is None else np.sort(rng.choice(B * T, nrows, replace=False))
    want = oracle.topn(c, rows, s.reshape(B * T, G, NS)[rows].astype(np.float64))
    bad = np.nonzero(np.any(got[rows] != want, axis=(1, 2)))[0]
    assert bad.size == 0, (kind, rows[bad[:3]], got[rows[bad[:3]]], want[bad[:3]])


@pytest.mark.parametrize("kind", ["uniform", "ties", "sparse", "zeros", "heavy", "one_lane", "tiny"])
def test_select_blocks_matches_oracle(kind):
    _check(dict(BASE, B=2, T=4096 + 37, G=4), kind, seed=11)


@pytest.mark.parametrize("n,fi,fl", [(16, 1, 2), (8, 0, 0), (3, 1, 2), (32, 2, 3)])
def test_select_blocks_counts_and_forced_blocks(n, fi, fl):
    _check(dict(BASE, B=1, T=8192, G=2, n=n, fi=fi, fl=fl), "uniform", seed=n)
    _check(dict(BASE, B=1, T=8192, G=2, n=n, fi=fi, fl=fl), "ties", seed=n + 1)


@pytest.mark.parametrize("kind", ["uniform", "ties", "one_lane", "zeros", "sparse", "tiny", "heavy"])
def test_select_blocks_rows_beyond_1024_blocks(kind):
    # up to 1563 candidate blocks per row: one CTA per row, the selection routine the
    # decode step also uses (ties at the threshold, all-equal rows, subnormals)
    _check(dict(BASE, B=1, T=100000, G=1), kind, seed=5, nrows=1500)


def _select_valid_only(c, t, row):
    """The selection rule the library states for scores outside the pages' domain:
    negative and NaN scores are never selected (fewer picks, -1 padded); -0 is 0."""
    n, lp, fi, fl = c["n"], c["lp"], c["fi"], c["fl"]
    bt = t // lp
    if bt + 1 <= n:
        got = list(range(bt + 1))
    else:
        cand = [j for j in range(fi, bt - fl + 1) if row[j] >= 0]          # False for NaN
        best = sorted(cand, key=lambda j: (-float(row[j]), j))[: n - fi - fl]
        got = sorted(set(range(fi)) | set(range(bt - fl + 1, bt + 1)) | set(best))
    return got + [-1] * (n - len(got))


def test_select_blocks_long_rows_skip_negative_and_nan_scores():
    # the CTA selection on rows of up to 1563 blocks with negative and NaN scores mixed
    # in, and rows where fewer valid scores than slots remain
    nsa = _nsa()
    c = dict(BASE, B=1, T=100000, G=1)
    NS = -(-100000 // c["lp"])
    rng = np.random.default_rng(9)
    s = rng.random((1, 100000, 1, NS)).astype(np.float32)
    s[..., 1::3] = -1.0
    s[..., 2::7] = np.nan
    s[0, 99000:, 0, 8:] = -0.5                  # these rows: only blocks 0..7 (and the forced) remain
    s[0, 99500:, 0, 3] = -0.0                   # negative zero counts as a zero score
    got = nsa.select_blocks(c, torch.from_numpy(s).cuda()).cpu().numpy()[0, :, 0]
    torch.cuda.synchronize()
    nsa.sync_status()
    rows = np.concatenate([np.sort(rng.choice(np.arange(64000, 99000), 300, replace=False)),
                           np.arange(99000, 99010), np.arange(99500, 99510), np.arange(99990, 100000)])
    for t in rows:
        assert got[t].tolist() == _select_valid_only(c, int(t), s[0, t, 0]), t
