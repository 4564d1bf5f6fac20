"""Seeded synthetic inputs for the NSA operator (tests, smoke check and bench).

This module holds no arithmetic of the method: it draws i.i.d. random tensors
of the workloads' shapes and value distributions, and nothing else.  It is
shared by the CUDA path's callers and by the oracle's callers so that both see
the same bits.

Generator: a counter-based stream.  Element ``i`` of stream ``s`` under seed
``seed`` is built from two splitmix64 hashes of (key(seed, s), 2i) and
(key(seed, s), 2i+1) -> two 53-bit uniforms -> Box-Muller in fp64 -> fp32.
bf16 tensors are the fp32 values rounded to nearest-even (torch's cast).
The same integer arithmetic runs on the CPU and on the GPU, so any slice can
be regenerated on either device (``start`` offset) without drawing the rest.

Workloads (the five configurations the operator is measured on; names say what
they are, sizes in the dicts):
  tiny_fwd_T1024        B1 T1024 H4 G1 d64/64, l32 d16 l'64 n4 w128, mean phi
  prefill_fwd_T8192     B1 T8192 H64 G4 d192/128, l32 d16 l'64 n16 w512, linear phi
  prefill_fwd_T65536    as above, T65536
  decode_S32_L8k_64k    32 sequences, L ~ U[8192, 65536], one query each, linear phi cache
  train_fwd_bwd_B2_T16384  B2 T16384, the T8192 architecture, upstream gradient dO
"""
from __future__ import annotations

import math

import numpy as np
import torch

_M64 = (1 << 64) - 1


def _s64(x: int) -> int:
    x &= _M64
    return x - (1 << 64) if x >= (1 << 63) else x


_C_GOLD = _s64(0x9E3779B97F4A7C15)
_C_MIX1 = _s64(0xBF58476D1CE4E5B9)
_C_MIX2 = _s64(0x94D049BB133111EB)


def _py_mix(z: int) -> int:
    z = (z + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = z + _C_GOLD
    z = (z ^ _srl(z, 30)) * _C_MIX1
    z = (z ^ _srl(z, 27)) * _C_MIX2
    return z ^ _srl(z, 31)


# stream ids, in the generation order q, k, v, gates, W_K, E_K, W_V, E_V, dO,
# lengths (+ the decode caches and the random selection used by backward tests)
STREAMS = {"q": 1, "k": 2, "v": 3, "gates": 4, "wk": 5, "ek": 6, "wv": 7, "ev": 8, "dout": 9,
           "lengths": 10, "kc_cache": 11, "vc_cache": 12, "sel": 13}

_CHUNK = 1 << 25


def _key(seed: int, stream: int) -> int:
    return _s64(_py_mix(_py_mix(seed & _M64) ^ (stream * 0x632BE59BD9B4E019 & _M64)))


def uniform64(seed: int, stream: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    """n uniforms in [0, 1) as fp64 (53-bit), elements start .. start+n-1."""
    key = _key(seed, stream)
    out = torch.empty(n, dtype=torch.float64, device=device)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        i = torch.arange(start + c0, start + c1, dtype=torch.int64, device=device)
        out[c0:c1] = _srl(_mix(i + key), 11).to(torch.float64) * (2.0 ** -53)
    return out


def normal64(seed: int, stream: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    """n standard normals (fp64), elements start .. start+n-1."""
    key = _key(seed, stream)
    out = torch.empty(n, dtype=torch.float64, device=device)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        i = torch.arange(start + c0, start + c1, dtype=torch.int64, device=device) * 2 + key
        u1 = (_srl(_mix(i), 11).to(torch.float64) + 0.5) * (2.0 ** -53)
        u2 = _srl(_mix(i + 1), 11).to(torch.float64) * (2.0 ** -53)
        out[c0:c1] = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
    return out


def normal_bf16(seed, stream, shape, std=1.0, device="cpu") -> torch.Tensor:
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        x = normal64(seed, stream, c1 - c0, device, start=c0)
        if std != 1.0:
            x = x * std
        out[c0:c1] = x.to(torch.float32).to(torch.bfloat16)
    return out.view(*shape)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(b: np.ndarray, device="cpu") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(device)


WORKLOADS = {
    "tiny_fwd_T1024": dict(kind="forward", B=1, T=1024, H=4, G=1, dk=64, dv=64, l=32, d=16,
                           lp=64, n=4, fi=1, fl=2, w=128, phi="mean", seed=1000),
    "prefill_fwd_T8192": dict(kind="forward", B=1, T=8192, H=64, G=4, dk=192, dv=128, l=32,
                              d=16, lp=64, n=16, fi=1, fl=2, w=512, phi="linear", seed=1001),
    "prefill_fwd_T65536": dict(kind="forward", B=1, T=65536, H=64, G=4, dk=192, dv=128, l=32,
                               d=16, lp=64, n=16, fi=1, fl=2, w=512, phi="linear", seed=1002),
    "decode_S32_L8k_64k": dict(kind="decode", S=32, Lmin=8192, Lmax=65536, H=64, G=4, dk=192,
                               dv=128, l=32, d=16, lp=64, n=16, fi=1, fl=2, w=512,
                               phi="linear", seed=1003),
    "train_fwd_bwd_B2_T16384": dict(kind="backward", B=2, T=16384, H=64, G=4, dk=192, dv=128,
                                    l=32, d=16, lp=64, n=16, fi=1, fl=2, w=512, phi="linear",
                                    seed=1004),
}


def make_forward_inputs(wl: dict, device="cpu", with_dout: bool = False) -> dict:
    """q [B,T,H,dk], k [B,T,G,dk], v [B,T,G,dv] bf16 N(0,1); gates [B,T,H,3] fp32
    sigmoid(N(0,1)); for the linear phi W_K [dk, l*dk] ~ N(0, 1/(l*dk)),
    E_K [l, dk] ~ N(0,1) (and W_V, E_V likewise); dO [B,T,H,dv] bf16 N(0,1)."""
    s = wl["seed"]
    B, T, H, G, dk, dv, l = wl["B"], wl["T"], wl["H"], wl["G"], wl["dk"], wl["dv"], wl["l"]
    out = {
        "q": normal_bf16(s, STREAMS["q"], (B, T, H, dk), device=device),
        "k": normal_bf16(s, STREAMS["k"], (B, T, G, dk), device=device),
        "v": normal_bf16(s, STREAMS["v"], (B, T, G, dv), device=device),
    }
    z = normal64(s, STREAMS["gates"], B * T * H * 3, device)
    out["gates"] = torch.sigmoid(z).to(torch.float32).view(B, T, H, 3)
    if wl.get("phi", "mean") == "linear":
        out.update(make_phi_params(wl, device))
    if with_dout:
        out["dout"] = normal_bf16(s, STREAMS["dout"], (B, T, H, dv), device=device)
    return out


def make_phi_params(wl: dict, device="cpu") -> dict:
    """Linear phi parameters: W_K [dk, l*dk] ~ N(0, 1/(l*dk)), E_K [l, dk] ~ N(0,1),
    W_V [dv, l*dv] ~ N(0, 1/(l*dv)), E_V [l, dv] ~ N(0,1), bf16."""
    s, dk, dv, l = wl["seed"], wl["dk"], wl["dv"], wl["l"]
    return {"wk": normal_bf16(s, STREAMS["wk"], (dk, l * dk), std=1.0 / math.sqrt(l * dk), device=device),
            "ek": normal_bf16(s, STREAMS["ek"], (l, dk), device=device),
            "wv": normal_bf16(s, STREAMS["wv"], (dv, l * dv), std=1.0 / math.sqrt(l * dv), device=device),
            "ev": normal_bf16(s, STREAMS["ev"], (l, dv), device=device)}


def decode_lengths(wl: dict) -> np.ndarray:
    """S context lengths, integers uniform in [Lmin, Lmax] inclusive."""
    u = uniform64(wl["seed"], STREAMS["lengths"], wl["S"]).numpy()
    span = wl["Lmax"] - wl["Lmin"] + 1
    return (wl["Lmin"] + np.floor(u * span)).astype(np.int64)


def make_decode_inputs(wl: dict, cmp_len, device="cpu", lengths=None) -> dict:
    """Packed varlen caches for one decode step.

    ``cmp_len(L)`` gives the compressed-cache length for a context of L tokens
    (the caller supplies it from the operator's contract).  The compressed
    cache is drawn i.i.d. N(0, 2) in bf16: the variance of a linear phi output
    with W ~ N(0, 1/(l*d)) over inputs k + E with k, E ~ N(0,1).
    """
    s = wl["seed"]
    S, H, G, dk, dv = wl["S"], wl["H"], wl["G"], wl["dk"], wl["dv"]
    L = decode_lengths(wl) if lengths is None else np.asarray(lengths, np.int64)
    Cs = np.array([cmp_len(int(x)) for x in L], np.int64)
    kv_off = np.concatenate([[0], np.cumsum(L)]).astype(np.int64)
    cmp_off = np.concatenate([[0], np.cumsum(Cs)]).astype(np.int64)
    NL, NC = int(kv_off[-1]), int(cmp_off[-1])
    out = {
        "lengths": L, "kv_off": kv_off, "cmp_off": cmp_off,
        "q": normal_bf16(s, STREAMS["q"], (S, H, dk), device=device),
        "k_cache": normal_bf16(s, STREAMS["k"], (NL, G, dk), device=device),
        "v_cache": normal_bf16(s, STREAMS["v"], (NL, G, dv), device=device),
        "kc_cache": normal_bf16(s, STREAMS["kc_cache"], (NC, G, dk), std=math.sqrt(2.0),
                                device=device),
        "vc_cache": normal_bf16(s, STREAMS["vc_cache"], (NC, G, dv), std=math.sqrt(2.0),
                                device=device),
    }
    z = normal64(s, STREAMS["gates"], S * H * 3, device)
    out["gates"] = torch.sigmoid(z).to(torch.float32).view(S, H, 3)
    return out


def random_selection(wl: dict, device="cpu") -> torch.Tensor:
    """A random valid block selection [B,T,G,n] int32 (ascending, -1 padded):
    blocks 0..fi-1 and the fl blocks ending at floor(t/l') always, plus distinct
    uniformly drawn other candidate blocks; all candidates when there are at
    most n.  Used as the fixed selection input of backward tests."""
    B, T, G, n, lp, fi, fl = wl["B"], wl["T"], wl["G"], wl["n"], wl["lp"], wl["fi"], wl["fl"]
    NS = (T + lp - 1) // lp
    t = torch.arange(T, device=device)
    bt = (t // lp).view(1, T, 1, 1)
    j = torch.arange(NS, device=device).view(1, 1, 1, NS)
    keys = uniform64(wl["seed"], STREAMS["sel"], B * T * G * NS, device).view(B, T, G, NS)
    cand = j <= bt
    forced = (j < fi) | ((j > bt - fl) & cand)
    few = (bt + 1) <= n
    pri = torch.where(forced | (cand & few), torch.full_like(keys, 3.0),
                      torch.where(cand, keys + 1.0, torch.zeros_like(keys)))
    top = torch.topk(pri, min(n, NS), dim=-1).indices
    valid = torch.gather(pri, -1, top) > 0.5
    sel = torch.where(valid, top, torch.full_like(top, 1 << 30))
    sel = torch.sort(sel, dim=-1).values
    sel = torch.where(sel == (1 << 30), torch.full_like(sel, -1), sel)
    if sel.shape[-1] < n:
        pad = torch.full((B, T, G, n - sel.shape[-1]), -1, dtype=sel.dtype, device=device)
        sel = torch.cat([sel, pad], -1)
    return sel.to(torch.int32).contiguous()
