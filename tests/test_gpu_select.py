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


@pytest.mark.parametrize("kind", ["uniform", "ties", "one_lane"])
def test_select_blocks_rows_beyond_1024_blocks(kind):
    # 1563 candidate blocks per row at the end: the 64-slot-per-lane kernel
    _check(dict(BASE, B=1, T=100000, G=1), kind, seed=5, nrows=1500)


def test_select_blocks_full_context_row_lengths():
    # every row length of a T=65536 sequence (1..1024 blocks), sampled rows
    _check(dict(BASE, B=1, T=65536, G=4), "heavy", seed=7, nrows=3000)


def test_select_blocks_never_takes_negative_or_nan_scores():
    nsa = _nsa()
    c = dict(BASE, B=1, T=4096, G=1)
    NS = 64
    rng = np.random.default_rng(3)
    s = rng.random((1, 4096, 1, NS)).astype(np.float32)
    s[..., 5:] = -1.0                      # only blocks 0..4 carry a score
    s[..., 2] = np.nan
    got = nsa.select_blocks(c, torch.from_numpy(s).cuda()).cpu().numpy()[0, :, 0]
    torch.cuda.synchronize()
    for t in (1024, 2047, 4095):
        bt = t // 64
        row = got[t]
        picked = set(row[row >= 0].tolist())
        forced = {0, bt - 1, bt}
        assert forced <= picked
        assert picked - forced <= {1, 3, 4}, row       # never 2 (NaN) nor a negative score
        assert (row >= 0).sum() == len(forced | ({1, 3, 4} - forced))
