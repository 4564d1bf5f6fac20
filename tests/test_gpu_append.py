"""Decode-step cache maintenance (nsa_decode_append) and decode over caches with
spare capacity (nsa_decode_rows).

Reference: page 2 (硬件对齐+原生训练！DeepSeek NSA打造高效稀疏Attention), 令牌压缩
(block i covers tokens [i*d, i*d + l)) and 效率分析 解码速度 (the decode step reads
the compressed cache).  The appended compressed block must be the oracle's phi
of the block, the raw row must be the new token, nothing else may change, and a
decode over the capacity layout must equal the decode over a packed copy of the
same rows bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_ulp_diff
from sparse_attention_long_phi_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _nsa():
    from sparse_attention_long_phi_b200 import nsa
    return nsa


def _phi_params(c, seed):
    if c.get("phi", "mean") != "linear":
        return None
    return I.make_phi_params(dict(c, seed=seed), "cuda")


def _capacity_caches(c, L_before, seed, spare=3):
    """Packed caches drawn for the lengths after the append, laid out again with
    `spare` free rows after every sequence (raw and compressed)."""
    cmp_len = lambda n: oracle.num_cmp_blocks(c, n)
    L_after = np.asarray(L_before, np.int64) + 1
    x = I.make_decode_inputs(dict(c, seed=seed), cmp_len, "cuda", lengths=L_after)
    S = len(L_after)
    cap = L_after + spare
    ccap = np.array([cmp_len(int(n)) for n in L_after]) + spare
    kv_start = np.concatenate([[0], np.cumsum(cap)[:-1]]).astype(np.int64)
    cmp_start = np.concatenate([[0], np.cumsum(ccap)[:-1]]).astype(np.int64)
    G, dk, dv = c["G"], c["dk"], c["dv"]
    sentinel = 0x1234
    def fill(rows, width):
        return torch.full((rows, G, width), sentinel, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    kc_ = fill(int(cap.sum()), dk); vc_ = fill(int(cap.sum()), dv)
    kcc = fill(int(ccap.sum()), dk); vcc = fill(int(ccap.sum()), dv)
    k_new = torch.empty(S, G, dk, dtype=torch.bfloat16, device="cuda")
    v_new = torch.empty(S, G, dv, dtype=torch.bfloat16, device="cuda")
    for s in range(S):
        a, b = int(x["kv_off"][s]), int(x["kv_off"][s + 1])
        n = b - a
        kc_[kv_start[s]:kv_start[s] + n - 1] = x["k_cache"][a:b - 1]
        vc_[kv_start[s]:kv_start[s] + n - 1] = x["v_cache"][a:b - 1]
        k_new[s] = x["k_cache"][b - 1]
        v_new[s] = x["v_cache"][b - 1]
        ca, cb = int(x["cmp_off"][s]), int(x["cmp_off"][s + 1])
        kcc[cmp_start[s]:cmp_start[s] + (cb - ca)] = x["kc_cache"][ca:cb]
        vcc[cmp_start[s]:cmp_start[s] + (cb - ca)] = x["vc_cache"][ca:cb]
    return x, dict(k_cache=kc_, v_cache=vc_, kc_cache=kcc, vc_cache=vcc, k_new=k_new, v_new=v_new,
                   kv_start=torch.from_numpy(kv_start).cuda(), cmp_start=torch.from_numpy(cmp_start).cuda(),
                   kv_len=torch.as_tensor(np.asarray(L_before, np.int64)).cuda())


def _check_append(c, L_before, seed):
    nsa = _nsa()
    x, cc = _capacity_caches(c, L_before, seed)
    phi = _phi_params(c, seed)
    before = {k: cc[k].clone() for k in ("k_cache", "v_cache", "kc_cache", "vc_cache")}
    nsa.decode_append(c, cc["k_new"], cc["v_new"], cc["k_cache"], cc["v_cache"], cc["kv_start"], cc["kv_len"],
                      cc["kc_cache"], cc["vc_cache"], cc["cmp_start"], phi)
    torch.cuda.synchronize()
    nsa.sync_status()
    l, d = c["l"], c["d"]
    kv_start = cc["kv_start"].cpu().numpy()
    cmp_start = cc["cmp_start"].cpu().numpy()
    expect = {k: v.clone() for k, v in before.items()}
    hphi = {k: I.bits(v) for k, v in phi.items()} if phi else {}
    completed = 0
    for s, L in enumerate(L_before):
        expect["k_cache"][kv_start[s] + L] = cc["k_new"][s]
        expect["v_cache"][kv_start[s] + L] = cc["v_new"][s]
        L1 = L + 1
        if L1 >= l and (L1 - l) % d == 0:
            i = (L1 - l) // d
            rows = slice(kv_start[s] + L1 - l, kv_start[s] + L1)
            kb = expect["k_cache"][rows][None]         # [1, l, G, dk], the new token included
            vb = expect["v_cache"][rows][None]
            kc_o, vc_o = oracle.phi(dict(c, B=1, T=l), I.bits(kb), I.bits(vb),
                                    hphi.get("wk"), hphi.get("ek"), hphi.get("wv"), hphi.get("ev"))
            got_k = I.bits(cc["kc_cache"][cmp_start[s] + i])
            got_v = I.bits(cc["vc_cache"][cmp_start[s] + i])
            uk, uv = bf16_ulp_diff(got_k, kc_o[0, 0]), bf16_ulp_diff(got_v, vc_o[0, 0])
            if c.get("phi", "mean") == "mean":
                assert uk.max() == 0 and uv.max() == 0, (s, L)
            else:
                assert uk.max() <= 1 and uv.max() <= 1, (s, L)
                assert (uk > 0).mean() <= 0.01 and (uv > 0).mean() <= 0.01
            expect["kc_cache"][cmp_start[s] + i] = cc["kc_cache"][cmp_start[s] + i]
            expect["vc_cache"][cmp_start[s] + i] = cc["vc_cache"][cmp_start[s] + i]
            completed += 1
    for k in expect:
        assert np.array_equal(I.bits(expect[k]), I.bits(cc[k])), k
    return x, cc, completed


def _lengths(c, S, rng):
    l, d = c["l"], c["d"]
    # about half complete a block: L + 1 = l + m*d; the rest fall between
    out = []
    for s in range(S):
        if s % 2 == 0:
            out.append(l - 1 + d * int(rng.integers(0, 600)))
        else:           # L mod d != d - 1: the new token completes no block
            out.append(d * int(rng.integers(0, 600)) + int(rng.integers(0, d - 1)))
    out[0] = 0           # first token of a sequence: no block
    out[1 % S] = l - 1   # completes block 0
    return out


def test_append_mean_phi_small_heads():
    c = dict(I.WORKLOADS["tiny_fwd_T1024"], kind="decode", S=9, phi="mean")
    rng = np.random.default_rng(1)
    _, _, n = _check_append(c, _lengths(c, 9, rng), seed=4100)
    assert n >= 3


def test_append_linear_phi_large_heads():
    c = dict(I.WORKLOADS["decode_S32_L8k_64k"], S=12, phi="linear")
    rng = np.random.default_rng(2)
    _, _, n = _check_append(c, _lengths(c, 12, rng), seed=4200)
    assert n >= 5


def test_decode_rows_equals_packed_decode_after_append():
    nsa = _nsa()
    c = dict(I.WORKLOADS["decode_S32_L8k_64k"], S=6, phi="linear")
    rng = np.random.default_rng(3)
    L_before = _lengths(c, 6, rng)
    x, cc, _ = _check_append(c, L_before, seed=4300)
    L_after = np.asarray(L_before, np.int64) + 1
    kv_start = cc["kv_start"].cpu().numpy()
    cmp_start = cc["cmp_start"].cpu().numpy()
    # packed copy of exactly the rows the capacity layout holds
    ks, vs, kcs, vcs = [], [], [], []
    for s, L in enumerate(L_after):
        C = oracle.num_cmp_blocks(c, int(L))
        ks.append(cc["k_cache"][kv_start[s]:kv_start[s] + L]); vs.append(cc["v_cache"][kv_start[s]:kv_start[s] + L])
        kcs.append(cc["kc_cache"][cmp_start[s]:cmp_start[s] + C]); vcs.append(cc["vc_cache"][cmp_start[s]:cmp_start[s] + C])
    kv_off = torch.from_numpy(np.concatenate([[0], np.cumsum(L_after)]).astype(np.int64)).cuda()
    Cs = [oracle.num_cmp_blocks(c, int(L)) for L in L_after]
    cmp_off = torch.from_numpy(np.concatenate([[0], np.cumsum(Cs)]).astype(np.int64)).cuda()
    Lmax = int(L_after.max())
    packed = nsa.decode(c, x["q"], torch.cat(ks), torch.cat(vs), kv_off, torch.cat(kcs), torch.cat(vcs),
                        cmp_off, x["gates"], max_len=Lmax)
    rows = nsa.decode_rows(c, x["q"], cc["k_cache"], cc["v_cache"], cc["kv_start"],
                           torch.from_numpy(L_after).cuda(), cc["kc_cache"], cc["vc_cache"], cc["cmp_start"],
                           x["gates"], max_len=Lmax)
    torch.cuda.synchronize()
    nsa.sync_status()
    for k in ("out", "idx", "lse"):
        assert torch.equal(packed[k], rows[k]), k
