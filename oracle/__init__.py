"""fp64 CPU oracle of the NSA per-layer attention operator.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it; the product library never does.  It
shares no code with the CUDA path.  The arithmetic lives in ``nsa_oracle.c``
(plain C, fp64, OpenMP over independent rows); this module only builds it and
marshals numpy arrays through ctypes.

Every function follows the NSA pages (see the header of ``nsa_oracle.c`` for
the sections each step cites).  Parity pins live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nsa_oracle.c")
_SO = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile nsa_oracle.c into oracle/_build/liboracle.so (gcc, OpenMP)."""
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


class OCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("B", "T", "H", "G", "dk", "dv", "l", "d", "lp", "n", "fi", "fl", "w",
                 "phi", "score_map", "cmp_exact")] + [("scale", ctypes.c_double)]


_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        pc = ctypes.POINTER(OCfg)
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        for f in ("oracle_num_cmp_blocks", "oracle_num_sel_blocks", "oracle_ncmp_visible"):
            getattr(lib, f).restype = _I64
            getattr(lib, f).argtypes = [pc, _I64]
        lib.oracle_phi.restype = None
        lib.oracle_phi.argtypes = [pc] + [_P] * 10
        lib.oracle_topn.restype = None
        lib.oracle_topn.argtypes = [pc, _I64, _P, _P, _P]
        lib.oracle_forward_rows.restype = None
        lib.oracle_forward_rows.argtypes = [pc, _P, _P, _P, _P, _P, _P, _I64, _P, _P, _P, _P, _P,
                                            _P, _P, _P]
        lib.oracle_forward_rows_branches.restype = None
        lib.oracle_forward_rows_branches.argtypes = [pc] + [_P] * 8 + [_I64] + [_P] * 8
        lib.oracle_key_counts.restype = None
        lib.oracle_key_counts.argtypes = [pc, _I64, _P]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [pc, _I64] + [_P] * 12 + [_I64]
        lib.oracle_backward_tail.restype = None
        lib.oracle_backward_tail.argtypes = [pc] + [_P] * 10 + [_I64] + [_P] * 6
        lib.oracle_backward_rows.restype = None
        lib.oracle_backward_rows.argtypes = [pc] + [_P] * 10 + [_I64] + [_P] * 7
        lib.oracle_phi_param_grads.restype = None
        lib.oracle_phi_param_grads.argtypes = [pc, _I64] + [_P] * 6
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def make_cfg(c: dict) -> OCfg:
    """Build the C config from a workload dict (keys as in the input module)."""
    phi = c.get("phi", "mean")
    phi = {"mean": 0, "linear": 1}.get(phi, phi)
    return OCfg(int(c.get("B", 1)), int(c.get("T", 0)), int(c["H"]), int(c["G"]), int(c["dk"]),
                int(c["dv"]), int(c["l"]), int(c["d"]), int(c["lp"]), int(c["n"]),
                int(c.get("fi", 1)), int(c.get("fl", 2)), int(c["w"]), int(phi),
                int(c.get("score_map", 0)), int(c.get("cmp_exact", 0)), float(c.get("scale", 0.0)))


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return None if a is None else np.ascontiguousarray(a, dtype=dt)


def bf16_to_f64(bits_arr) -> np.ndarray:
    """bf16 bit patterns -> exact fp64 values."""
    b = np.ascontiguousarray(bits_arr, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _vals(a):
    """compressed keys/values as fp64: bf16 bits are widened exactly, fp64 kept"""
    if a is None:
        return None
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return bf16_to_f64(a)
    return np.ascontiguousarray(a, np.float64)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def bf16_round(x: float) -> int:
    return int(_load().oracle_double_to_bf16(float(x)))


def bf16_value(bits: int) -> float:
    return float(_load().oracle_bf16_to_double(int(bits)))


def num_cmp_blocks(c: dict, T: int) -> int:
    return int(_load().oracle_num_cmp_blocks(ctypes.byref(make_cfg(c)), int(T)))


def num_sel_blocks(c: dict, T: int) -> int:
    return int(_load().oracle_num_sel_blocks(ctypes.byref(make_cfg(c)), int(T)))


def ncmp_visible(c: dict, t: int) -> int:
    return int(_load().oracle_ncmp_visible(ctypes.byref(make_cfg(c)), int(t)))


def key_counts(c: dict, t: int):
    out = np.zeros(3, np.int64)
    _load().oracle_key_counts(ctypes.byref(make_cfg(c)), int(t), _ptr(out))
    return tuple(int(x) for x in out)


def phi(c: dict, k, v, wk=None, ek=None, wv=None, ev=None, exact: bool = False):
    """Token compression: returns (kc, vc) bf16 bits [B,C,G,*] (and fp64 exact values)."""
    cf = make_cfg(c)
    B, T, G = cf.B, cf.T, cf.G
    C = num_cmp_blocks(c, T)
    kc = np.zeros((B, C, G, cf.dk), np.uint16)
    vc = np.zeros((B, C, G, cf.dv), np.uint16)
    kx = np.zeros(kc.shape, np.float64) if exact else None
    vx = np.zeros(vc.shape, np.float64) if exact else None
    args = [_c(k, np.uint16), _c(v, np.uint16), _c(wk, np.uint16), _c(ek, np.uint16),
            _c(wv, np.uint16), _c(ev, np.uint16)]
    if cf.phi == 1:
        assert all(a is not None for a in args), "linear phi needs W_K, E_K, W_V, E_V"
    _load().oracle_phi(ctypes.byref(cf), *[_ptr(a) for a in args], _ptr(kc), _ptr(vc), _ptr(kx),
                       _ptr(vx))
    return (kc, vc, kx, vx) if exact else (kc, vc)


def forward_rows(c: dict, q, k, v, gates, kc, vc, rows, idx_in=None, want=("out", "idx", "lse"),
                 k_win=None, v_win=None):
    """Forward for the rows r = b*T + t listed in ``rows``.

    ``kc``/``vc`` are the compressed keys/values [B,C,G,*], as bf16 bits (the
    operator) or fp64 values (unrounded, for gradient checks).

    Returns a dict with any of: out [R,H,dv], idx [R,G,n], lse [R,H,3] (natural
    log, cmp/slc/win), pgrp [R,G,Nsel] (group importance scores), pcmp [R,H,C]
    (compressed probabilities), obr [R,H,3,dv] (per-branch outputs).
    ``idx_in`` ([R,G,n]) replaces the oracle's selection for these rows.
    ``k_win``/``v_win`` give the window branch its own keys/values (independent
    K/V per branch); by default it reads k/v like the selected branch.
    """
    cf = make_cfg(c)
    rows = np.ascontiguousarray(rows, np.int64).reshape(-1)
    R = rows.size
    C = num_cmp_blocks(c, cf.T)
    NS = num_sel_blocks(c, cf.T)
    res = {"out": np.zeros((R, cf.H, cf.dv)), "idx": np.zeros((R, cf.G, cf.n), np.int32)}
    if "lse" in want:
        res["lse"] = np.zeros((R, cf.H, 3))
    if "pgrp" in want:
        res["pgrp"] = np.zeros((R, cf.G, NS))
    if "pcmp" in want:
        res["pcmp"] = np.zeros((R, cf.H, max(C, 1)))
    if "obr" in want:
        res["obr"] = np.zeros((R, cf.H, 3, cf.dv))
    kb, vb = _c(k, np.uint16), _c(v, np.uint16)
    kw = kb if k_win is None else _c(k_win, np.uint16)
    vw = vb if v_win is None else _c(v_win, np.uint16)
    assert kw.shape == kb.shape and vw.shape == vb.shape
    _load().oracle_forward_rows_branches(
        ctypes.byref(cf), _ptr(_c(q, np.uint16)), _ptr(kb), _ptr(vb), _ptr(kw), _ptr(vw),
        _ptr(_c(gates, np.float32)), _ptr(_vals(kc)), _ptr(_vals(vc)), R,
        _ptr(rows), _ptr(_c(idx_in, np.int32)), _ptr(res["out"]), _ptr(res["idx"]),
        _ptr(res.get("lse")), _ptr(res.get("pgrp")), _ptr(res.get("pcmp")), _ptr(res.get("obr")))
    return res


def topn(c: dict, rows, pgrp):
    cf = make_cfg(c)
    rows = np.ascontiguousarray(rows, np.int64).reshape(-1)
    pgrp = np.ascontiguousarray(pgrp, np.float64)
    idx = np.zeros((rows.size, cf.G, cf.n), np.int32)
    _load().oracle_topn(ctypes.byref(cf), rows.size, _ptr(rows), _ptr(pgrp), _ptr(idx))
    return idx


def decode(c: dict, q, k_cache, v_cache, kv_off, kc_cache, vc_cache, cmp_off, gates,
           want_pgrp: bool = False):
    """Decode step: one query per sequence at t = L-1.  Returns dict(out, idx, lse[, pgrp])."""
    cf = make_cfg(c)
    kv_off = np.ascontiguousarray(kv_off, np.int64)
    cmp_off = np.ascontiguousarray(cmp_off, np.int64)
    S = kv_off.size - 1
    lens = np.diff(kv_off)
    ns_stride = int(max(1, max(num_sel_blocks(c, int(L)) for L in lens))) if S else 1
    out = np.zeros((S, cf.H, cf.dv))
    idx = np.zeros((S, cf.G, cf.n), np.int32)
    lse = np.zeros((S, cf.H, 3))
    pg = np.zeros((S, cf.G, ns_stride)) if want_pgrp else None
    rc = _load().oracle_decode(
        ctypes.byref(cf), S, _ptr(_c(q, np.uint16)), _ptr(_c(k_cache, np.uint16)),
        _ptr(_c(v_cache, np.uint16)), _ptr(kv_off), _ptr(_c(kc_cache, np.uint16)),
        _ptr(_c(vc_cache, np.uint16)), _ptr(cmp_off), _ptr(_c(gates, np.float32)), _ptr(out),
        _ptr(idx), _ptr(lse), _ptr(pg), ns_stride)
    if rc != 0:
        raise ValueError("oracle_decode: a compressed-cache length does not equal N_cmp(L-1)")
    res = {"out": out, "idx": idx, "lse": lse}
    if want_pgrp:
        res["pgrp"] = pg
    return res


def backward_tail(c: dict, q, k, v, gates, dout, idx, wk=None, ek=None, wv=None, ev=None,
                  t_lo: int = 0, want_cmp: bool = False):
    """Backward with the selection ``idx`` [B,T,G,n] held fixed.

    dk/dv are exact for tokens u >= t_lo, dq/dgates for rows t >= t_lo.
    Returns dict(dq [B,T,H,dk], dk [B,T,G,dk], dv [B,T,G,dv], dgates [B,T,H,3]), and with
    want_cmp the compressed-key gradients dkc [B,C,G,dk], dvc [B,C,G,dv] (exact with t_lo = 0).
    """
    cf = make_cfg(c)
    B, T, H, G = cf.B, cf.T, cf.H, cf.G
    C = num_cmp_blocks(c, T)
    dq = np.zeros((B, T, H, cf.dk))
    dk = np.zeros((B, T, G, cf.dk))
    dv = np.zeros((B, T, G, cf.dv))
    dg = np.zeros((B, T, H, 3))
    dkc = np.zeros((B, C, G, cf.dk)) if want_cmp else None
    dvc = np.zeros((B, C, G, cf.dv)) if want_cmp else None
    _load().oracle_backward_tail(
        ctypes.byref(cf), _ptr(_c(q, np.uint16)), _ptr(_c(k, np.uint16)), _ptr(_c(v, np.uint16)),
        _ptr(_c(gates, np.float32)), _ptr(_c(wk, np.uint16)), _ptr(_c(ek, np.uint16)),
        _ptr(_c(wv, np.uint16)), _ptr(_c(ev, np.uint16)), _ptr(_c(dout, np.uint16)),
        _ptr(_c(idx, np.int32)), int(t_lo), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dkc), _ptr(dvc))
    out = {"dq": dq, "dk": dk, "dv": dv, "dgates": dg}
    if want_cmp:
        out.update(dkc=dkc, dvc=dvc)
    return out


def backward_rows(c: dict, q, k, v, gates, dout, idx, rows, wk=None, ek=None, wv=None, ev=None,
                  want_cmp: bool = False):
    """Backward restricted to the query rows r = b*T + t in ``rows``: the gradient of the
    sum over those rows of <dout, out> (rows outside contribute nothing, as if their dout
    were zero).  Same outputs as backward_tail; dq/dgates are zero outside the listed rows,
    dk/dv/dkc/dvc hold the listed rows' contributions at every key position."""
    cf = make_cfg(c)
    B, T, H, G = cf.B, cf.T, cf.H, cf.G
    C = num_cmp_blocks(c, T)
    rows = np.ascontiguousarray(rows, np.int64).reshape(-1)
    dq = np.zeros((B, T, H, cf.dk))
    dk = np.zeros((B, T, G, cf.dk))
    dv = np.zeros((B, T, G, cf.dv))
    dg = np.zeros((B, T, H, 3))
    dkc = np.zeros((B, C, G, cf.dk)) if want_cmp else None
    dvc = np.zeros((B, C, G, cf.dv)) if want_cmp else None
    _load().oracle_backward_rows(
        ctypes.byref(cf), _ptr(_c(q, np.uint16)), _ptr(_c(k, np.uint16)), _ptr(_c(v, np.uint16)),
        _ptr(_c(gates, np.float32)), _ptr(_c(wk, np.uint16)), _ptr(_c(ek, np.uint16)),
        _ptr(_c(wv, np.uint16)), _ptr(_c(ev, np.uint16)), _ptr(_c(dout, np.uint16)),
        _ptr(_c(idx, np.int32)), int(rows.size), _ptr(rows), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
        _ptr(dkc), _ptr(dvc))
    out = {"dq": dq, "dk": dk, "dv": dv, "dgates": dg}
    if want_cmp:
        out.update(dkc=dkc, dvc=dvc)
    return out


def phi_param_grads(c: dict, k, v, wk, ek, wv, ev, dkc, dvc):
    """Gradients of the linear phi's W_K, E_K, W_V, E_V from dK~ = dkc, dV~ = dvc
    (token compression: K~[i] = W vec(k_blk + E)).  fp64 dict(dwk, dek, dwv, dev)."""
    cf = make_cfg(c)
    lib = _load()
    out = {}
    for name, x, W, E, dY, D in (("k", k, wk, ek, dkc, cf.dk), ("v", v, wv, ev, dvc, cf.dv)):
        dW = np.zeros((D, cf.l * D))
        dE = np.zeros((cf.l, D))
        lib.oracle_phi_param_grads(ctypes.byref(cf), int(D), _ptr(_c(x, np.uint16)), _ptr(_c(W, np.uint16)),
                                   _ptr(_c(E, np.uint16)), _ptr(np.ascontiguousarray(dY, np.float64)),
                                   _ptr(dW), _ptr(dE))
        out["dw" + name], out["de" + name] = dW, dE
    return out
