"""Python binding of libnsa (include/nsa.h): argument marshalling only.

Every step of the operator runs in the library's CUDA kernels; this module
allocates outputs and the workspace with torch (device memory, streams) and
passes raw pointers through ctypes.  There is no fallback: if libnsa.so is
missing or a call fails, it raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libnsa.so")

NSA_MODE_FORWARD, NSA_MODE_DECODE, NSA_MODE_BACKWARD, NSA_MODE_FORWARD_BRANCHES = 0, 1, 2, 3
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "workspace",
          4: "CUDA error", 5: "device timeout"}


class NsaError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn}: {STATUS.get(code, code)} ({code})")
        self.code = code


class CConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("batch", "seqlen", "num_q_heads", "num_kv_groups", "d_k", "d_v", "cmp_block",
                 "cmp_stride", "sel_block", "sel_count", "forced_initial", "forced_local", "window",
                 "phi", "score_map")] + [("scale", ctypes.c_float)]


class CPhi(ctypes.Structure):
    _fields_ = [("w_k", ctypes.c_void_p), ("e_k", ctypes.c_void_p), ("w_v", ctypes.c_void_p),
                ("e_v", ctypes.c_void_p)]


_lib = None
_P = ctypes.c_void_p


def library_path() -> str:
    return _SO


def lib():
    """Load libnsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_SO):
            raise ImportError(f"libnsa.so not found at {_SO}: build it with "
                              "`python -m sparse_attention_long_phi_b200.build`")
        L = ctypes.CDLL(_SO)
        pc = ctypes.POINTER(CConfig)
        pp = ctypes.POINTER(CPhi)
        L.nsa_workspace_size.restype = ctypes.c_size_t
        L.nsa_workspace_size.argtypes = [pc, ctypes.c_int32]
        L.nsa_num_cmp_blocks.restype = ctypes.c_int64
        L.nsa_num_cmp_blocks.argtypes = [pc, ctypes.c_int64]
        L.nsa_forward_score_table.restype = ctypes.c_int64
        L.nsa_forward_score_table.argtypes = [pc, ctypes.POINTER(ctypes.c_int64)]
        L.nsa_compress.restype = ctypes.c_int
        L.nsa_compress.argtypes = [pc, _P, _P, pp, _P, _P, _P, ctypes.c_size_t, _P]
        L.nsa_compress_static.restype = ctypes.c_int
        L.nsa_compress_static.argtypes = [pc, _P, _P, pp, _P, _P, _P]
        L.nsa_forward.restype = ctypes.c_int
        L.nsa_forward.argtypes = [pc, _P, _P, _P, _P, pp, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.nsa_forward_train.restype = ctypes.c_int
        L.nsa_forward_train.argtypes = [pc, _P, _P, _P, _P, pp, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.nsa_backward_saved.restype = ctypes.c_int
        L.nsa_backward_saved.argtypes = [pc, _P, _P, _P, _P, pp, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                         ctypes.c_size_t, _P]
        L.nsa_forward_branches.restype = ctypes.c_int
        L.nsa_forward_branches.argtypes = [pc] + [_P] * 8 + [pp] + [_P] * 6 + [ctypes.c_size_t, _P]
        L.nsa_decode_rows.restype = ctypes.c_int
        L.nsa_decode_rows.argtypes = [pc, ctypes.c_int32] + [_P] * 13 + [ctypes.c_size_t, _P]
        L.nsa_decode_append.restype = ctypes.c_int
        L.nsa_decode_append.argtypes = [pc, ctypes.c_int32] + [_P] * 9 + [pp, _P]
        L.nsa_select_blocks.restype = ctypes.c_int
        L.nsa_select_blocks.argtypes = [pc, _P, _P, _P]
        L.nsa_decode.restype = ctypes.c_int
        L.nsa_decode.argtypes = [pc, ctypes.c_int32] + [_P] * 12 + [ctypes.c_size_t, _P]
        L.nsa_backward.restype = ctypes.c_int
        L.nsa_backward.argtypes = [pc, _P, _P, _P, _P, pp, _P, _P, _P, _P, _P, _P, _P,
                                   ctypes.c_size_t, _P]
        L.nsa_backward_phi_params.restype = ctypes.c_int
        L.nsa_backward_phi_params.argtypes = [pc, _P, _P, pp, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
        L.nsa_check_timeout_path.restype = ctypes.c_int
        L.nsa_check_timeout_path.argtypes = [ctypes.c_uint64, _P]
        L.nsa_sync_status.restype = ctypes.c_int
        L.nsa_sync_status.argtypes = [_P]
        L.nsa_profile_enable.restype = ctypes.c_int
        L.nsa_profile_enable.argtypes = [ctypes.c_int32]
        L.nsa_profile_read.restype = ctypes.c_int32
        L.nsa_profile_read.argtypes = [ctypes.c_int32, ctypes.c_char_p, _P, _P]
        L.nsa_status_string.restype = ctypes.c_char_p
        L.nsa_status_string.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def make_config(c: dict, batch=None, seqlen=None) -> CConfig:
    """nsa_config_t from a workload dict (keys B, T, H, G, dk, dv, l, d, lp, n, fi, fl, w, phi)."""
    phi = c.get("phi", "mean")
    phi = {"mean": 0, "linear": 1}.get(phi, phi)
    return CConfig(int(batch if batch is not None else c.get("B", 1)),
                   int(seqlen if seqlen is not None else c.get("T", 0)), int(c["H"]), int(c["G"]),
                   int(c["dk"]), int(c["dv"]), int(c["l"]), int(c["d"]), int(c["lp"]), int(c["n"]),
                   int(c.get("fi", 1)), int(c.get("fl", 2)), int(c["w"]), int(phi),
                   int(c.get("score_map", 0)), float(c.get("scale", 0.0)))


def _p(t):
    if t is None:
        return None
    assert t.is_contiguous(), "libnsa tensors must be contiguous"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, code):
    if code != 0:
        raise NsaError(fn, code)


def _phi(phi):
    if phi is None:
        return None
    return ctypes.byref(CPhi(*(ctypes.c_void_p(phi[k].data_ptr()) for k in ("wk", "ek", "wv", "ev"))))


def workspace_size(c: dict, mode: int, batch=None, seqlen=None) -> int:
    return int(lib().nsa_workspace_size(ctypes.byref(make_config(c, batch, seqlen)), mode))


def num_cmp_blocks(c: dict, length: int) -> int:
    return int(lib().nsa_num_cmp_blocks(ctypes.byref(make_config(c)), int(length)))


def alloc_workspace(c: dict, mode: int, device, batch=None, seqlen=None) -> torch.Tensor:
    n = workspace_size(c, mode, batch, seqlen)
    if n == 0:
        raise NsaError("nsa_workspace_size", 1)
    return torch.empty(n, dtype=torch.uint8, device=device)


@dataclass
class ForwardBuffers:
    out: torch.Tensor
    idx: torch.Tensor
    lse: torch.Tensor | None
    kc: torch.Tensor | None
    vc: torch.Tensor | None
    ws: torch.Tensor


def forward_buffers(c: dict, device, want_lse=True, want_kc=False) -> ForwardBuffers:
    B, T, H, G, dk, dv = c["B"], c["T"], c["H"], c["G"], c["dk"], c["dv"]
    C = num_cmp_blocks(c, T)
    f32 = dict(dtype=torch.float32, device=device)
    return ForwardBuffers(
        out=torch.empty(B, T, H, dv, **f32),
        idx=torch.empty(B, T, G, c["n"], dtype=torch.int32, device=device),
        lse=torch.empty(B, T, H, 3, **f32) if want_lse else None,
        kc=torch.empty(B, max(C, 1), G, dk, dtype=torch.bfloat16, device=device) if want_kc else None,
        vc=torch.empty(B, max(C, 1), G, dv, dtype=torch.bfloat16, device=device) if want_kc else None,
        ws=alloc_workspace(c, NSA_MODE_FORWARD, device))


def forward_into(c: dict, q, k, v, gates, phi, buf: ForwardBuffers, stream=None):
    """nsa_forward into preallocated buffers (asynchronous on the stream)."""
    cfg = make_config(c)
    _check("nsa_forward", lib().nsa_forward(
        ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(gates), _phi(phi), _p(buf.out), _p(buf.idx),
        _p(buf.lse), _p(buf.kc), _p(buf.vc), _p(buf.ws), buf.ws.numel(), _stream(stream)))


def score_table(c: dict, ws: torch.Tensor) -> torch.Tensor:
    """View of the group importance-score table [B,T,G,NSp] fp32 that nsa_forward leaves in
    its workspace `ws` (valid for blocks j <= t // l' of rows t >= l - 1)."""
    stride = ctypes.c_int64(0)
    off = int(lib().nsa_forward_score_table(ctypes.byref(make_config(c)), ctypes.byref(stride)))
    if off < 0:
        raise NsaError("nsa_forward_score_table", 1)
    B, T, G = c["B"], c["T"], c["G"]
    n = B * T * G * stride.value
    return ws[off:off + 4 * n].view(torch.float32).view(B, T, G, stride.value)


def forward(c: dict, q, k, v, gates, phi=None, want_lse=True, want_kc=False, stream=None,
            want_scores=False) -> dict:
    """Prefill forward.  q [B,T,H,dk], k [B,T,G,dk], v [B,T,G,dv] bf16; gates [B,T,H,3] fp32;
    phi = dict(wk, ek, wv, ev) for the linear map.  Returns out, idx, lse, kc, vc (and with
    want_scores the importance-score table left in the workspace)."""
    buf = forward_buffers(c, q.device, want_lse, want_kc)
    forward_into(c, q, k, v, gates, phi, buf, stream)
    res = {"out": buf.out, "idx": buf.idx, "lse": buf.lse, "kc": buf.kc, "vc": buf.vc}
    if want_scores:
        res["scores"] = score_table(c, buf.ws)
    return res


def forward_train(c: dict, q, k, v, gates, phi=None, stream=None, ws=None, res=None) -> dict:
    """Training forward: forward()'s out, idx, lse plus o_branch [3,B,T,H,dv] fp32, each
    branch's own output before its gate (compressed, selected, window), for backward_saved.
    `res` (a previous result) is written in place instead of allocating new tensors."""
    B, T, H, G, dv = c["B"], c["T"], c["H"], c["G"], c["dv"]
    f32 = dict(dtype=torch.float32, device=q.device)
    if res is None:
        res = {"out": torch.empty(B, T, H, dv, **f32),
               "idx": torch.empty(B, T, G, c["n"], dtype=torch.int32, device=q.device),
               "lse": torch.empty(B, T, H, 3, **f32), "o_branch": torch.empty(3, B, T, H, dv, **f32)}
    if ws is None:
        ws = alloc_workspace(c, NSA_MODE_FORWARD, q.device)
    _check("nsa_forward_train", lib().nsa_forward_train(
        ctypes.byref(make_config(c)), _p(q), _p(k), _p(v), _p(gates), _phi(phi), _p(res["out"]),
        _p(res["idx"]), _p(res["lse"]), _p(res["o_branch"]), _p(ws), ws.numel(), _stream(stream)))
    return res


def backward_saved(c: dict, q, k, v, gates, dout, idx, lse, o_branch, phi=None, stream=None,
                   ws=None, want_phi_grads=False, res=None) -> dict:
    """backward() from the statistics forward_train saved (lse, o_branch) for the same inputs
    and selection idx: dq, dk, dv, dgates (fp32), and the phi parameter gradients as backward().
    `res` (a previous result) is written in place instead of allocating new tensors."""
    B, T, H, G, dk, dv = c["B"], c["T"], c["H"], c["G"], c["dk"], c["dv"]
    f32 = dict(dtype=torch.float32, device=q.device)
    if res is None:
        res = {"dq": torch.empty(B, T, H, dk, **f32), "dk": torch.empty(B, T, G, dk, **f32),
               "dv": torch.empty(B, T, G, dv, **f32), "dgates": torch.empty(B, T, H, 3, **f32)}
    if ws is None:
        ws = alloc_workspace(c, NSA_MODE_BACKWARD, q.device)
    cfg = make_config(c)
    _check("nsa_backward_saved", lib().nsa_backward_saved(
        ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(gates), _phi(phi), _p(dout), _p(idx),
        _p(lse), _p(o_branch), _p(res["dq"]), _p(res["dk"]), _p(res["dv"]), _p(res["dgates"]), _p(ws),
        ws.numel(), _stream(stream)))
    if want_phi_grads:
        _phi_grads(c, cfg, k, v, phi, ws, stream, res)
    return res


def _phi_grads(c, cfg, k, v, phi, ws, stream, res):
    """nsa_backward_phi_params after a backward that left dK~/dV~ in ws (into res's
    dwk/dek/dwv/dev when it has them)."""
    dk, dv, l = c["dk"], c["dv"], c["l"]
    f32 = dict(dtype=torch.float32, device=k.device)
    if "dwk" not in res:
        res.update(dwk=torch.empty(dk, l * dk, **f32), dek=torch.empty(l, dk, **f32),
                   dwv=torch.empty(dv, l * dv, **f32), dev=torch.empty(l, dv, **f32))
    _check("nsa_backward_phi_params", lib().nsa_backward_phi_params(
        ctypes.byref(cfg), _p(k), _p(v), _phi(phi), _p(res["dwk"]), _p(res["dek"]), _p(res["dwv"]),
        _p(res["dev"]), _p(ws), ws.numel(), _stream(stream)))


def forward_branches(c: dict, q, kv: dict, gates, phi=None, want_lse=True, want_kc=False,
                     stream=None, want_scores=False) -> dict:
    """Prefill forward with independent keys/values per branch: kv = dict(k_cmp, v_cmp,
    k_slc, v_slc, k_win, v_win), each shaped like k / v.  Returns as forward()."""
    B, T, H, G, dk, dv = c["B"], c["T"], c["H"], c["G"], c["dk"], c["dv"]
    C = num_cmp_blocks(c, T)
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = torch.empty(B, T, H, dv, **f32)
    idx = torch.empty(B, T, G, c["n"], dtype=torch.int32, device=dev)
    lse = torch.empty(B, T, H, 3, **f32) if want_lse else None
    kc = torch.empty(B, max(C, 1), G, dk, dtype=torch.bfloat16, device=dev) if want_kc else None
    vc = torch.empty(B, max(C, 1), G, dv, dtype=torch.bfloat16, device=dev) if want_kc else None
    ws = alloc_workspace(c, NSA_MODE_FORWARD_BRANCHES, dev)
    _check("nsa_forward_branches", lib().nsa_forward_branches(
        ctypes.byref(make_config(c)), _p(q), _p(kv["k_cmp"]), _p(kv["v_cmp"]), _p(kv["k_slc"]),
        _p(kv["v_slc"]), _p(kv["k_win"]), _p(kv["v_win"]), _p(gates), _phi(phi), _p(out), _p(idx), _p(lse),
        _p(kc), _p(vc), _p(ws), ws.numel(), _stream(stream)))
    res = {"out": out, "idx": idx, "lse": lse, "kc": kc, "vc": vc}
    if want_scores:
        res["scores"] = score_table(c, ws)
    return res


def compress(c: dict, k, v, phi=None, stream=None):
    B, T, G = c["B"], c["T"], c["G"]
    C = num_cmp_blocks(c, T)
    kc = torch.empty(B, max(C, 1), G, c["dk"], dtype=torch.bfloat16, device=k.device)
    vc = torch.empty(B, max(C, 1), G, c["dv"], dtype=torch.bfloat16, device=k.device)
    ws = alloc_workspace(c, NSA_MODE_FORWARD, k.device)
    _check("nsa_compress", lib().nsa_compress(ctypes.byref(make_config(c)), _p(k), _p(v), _phi(phi),
                                              _p(kc), _p(vc), _p(ws), ws.numel(), _stream(stream)))
    return kc[:, :C], vc[:, :C]


def select_blocks(c: dict, scores, stream=None) -> torch.Tensor:
    """Top-n block selection alone.  scores [B,T,G,NS] fp32 (NS = ceil(T / l')) ->
    sel_idx [B,T,G,n] int32, ascending, -1 padded."""
    B, T, G = c["B"], c["T"], c["G"]
    assert scores.dtype == torch.float32 and scores.is_cuda
    assert tuple(scores.shape) == (B, T, G, -(-T // c["lp"])), "scores must be [B,T,G,ceil(T/l')]"
    idx = torch.empty(B, T, G, c["n"], dtype=torch.int32, device=scores.device)
    _check("nsa_select_blocks", lib().nsa_select_blocks(ctypes.byref(make_config(c)), _p(scores), _p(idx),
                                                        _stream(stream)))
    return idx


def compress_static(c: dict, k, v, phi=None, stream=None) -> tuple:
    """Token compression with the library's fixed device scratch (no workspace).
    Returns (status, kc, vc); status NSA_ERR_WORKSPACE (3) when the sizes exceed it."""
    B, T, G = c["B"], c["T"], c["G"]
    C = num_cmp_blocks(c, T)
    kc = torch.full((B, max(C, 1), G, c["dk"]), float("nan"), dtype=torch.bfloat16, device=k.device)
    vc = torch.full((B, max(C, 1), G, c["dv"]), float("nan"), dtype=torch.bfloat16, device=k.device)
    rc = lib().nsa_compress_static(ctypes.byref(make_config(c)), _p(k), _p(v), _phi(phi), _p(kc), _p(vc),
                                   _stream(stream))
    return rc, kc[:, :C], vc[:, :C]


@dataclass
class DecodeBuffers:
    out: torch.Tensor
    idx: torch.Tensor
    lse: torch.Tensor | None
    ws: torch.Tensor


def decode_buffers(c: dict, num_seqs: int, max_len: int, device, want_lse=True) -> DecodeBuffers:
    f32 = dict(dtype=torch.float32, device=device)
    return DecodeBuffers(
        out=torch.empty(num_seqs, c["H"], c["dv"], **f32),
        idx=torch.empty(num_seqs, c["G"], c["n"], dtype=torch.int32, device=device),
        lse=torch.empty(num_seqs, c["H"], 3, **f32) if want_lse else None,
        ws=alloc_workspace(c, NSA_MODE_DECODE, device, batch=num_seqs, seqlen=max_len))


def decode_into(c: dict, max_len: int, q, k_cache, v_cache, kv_off, kc_cache, vc_cache, cmp_off,
                gates, buf: DecodeBuffers, stream=None):
    S = q.shape[0]
    cfg = make_config(c, batch=S, seqlen=max_len)
    _check("nsa_decode", lib().nsa_decode(
        ctypes.byref(cfg), S, _p(q), _p(k_cache), _p(v_cache), _p(kv_off), _p(kc_cache),
        _p(vc_cache), _p(cmp_off), _p(gates), _p(buf.out), _p(buf.idx), _p(buf.lse), _p(buf.ws),
        buf.ws.numel(), _stream(stream)))


def decode(c: dict, q, k_cache, v_cache, kv_off, kc_cache, vc_cache, cmp_off, gates, max_len: int,
           want_lse=True, stream=None) -> dict:
    """One decode step: q [S,H,dk]; packed caches with int64 device offsets [S+1]."""
    buf = decode_buffers(c, q.shape[0], max_len, q.device, want_lse)
    decode_into(c, max_len, q, k_cache, v_cache, kv_off, kc_cache, vc_cache, cmp_off, gates, buf,
                stream)
    return {"out": buf.out, "idx": buf.idx, "lse": buf.lse}


def decode_rows(c: dict, q, k_cache, v_cache, kv_start, kv_len, kc_cache, vc_cache, cmp_start, gates,
                max_len: int, want_lse=True, stream=None) -> dict:
    """One decode step over caches with spare capacity: sequence s holds kv_len[s] tokens
    from row kv_start[s] and its compressed blocks from row cmp_start[s] (int64 device [S])."""
    S = q.shape[0]
    buf = decode_buffers(c, S, max_len, q.device, want_lse)
    cfg = make_config(c, batch=S, seqlen=max_len)
    _check("nsa_decode_rows", lib().nsa_decode_rows(
        ctypes.byref(cfg), S, _p(q), _p(k_cache), _p(v_cache), _p(kv_start), _p(kv_len), _p(kc_cache),
        _p(vc_cache), _p(cmp_start), _p(gates), _p(buf.out), _p(buf.idx), _p(buf.lse), _p(buf.ws),
        buf.ws.numel(), _stream(stream)))
    return {"out": buf.out, "idx": buf.idx, "lse": buf.lse}


def decode_append(c: dict, k_new, v_new, k_cache, v_cache, kv_start, kv_len, kc_cache, vc_cache, cmp_start,
                  phi=None, stream=None):
    """Append token kv_len[s] of each sequence (k_new [S,G,dk], v_new [S,G,dv]) to the raw caches and
    write phi of the compressed block it completes, if any.  kv_len is not advanced here."""
    S = k_new.shape[0]
    cfg = make_config(c, batch=S, seqlen=c.get("T", 1))   # the context length plays no part here
    _check("nsa_decode_append", lib().nsa_decode_append(
        ctypes.byref(cfg), S, _p(k_new), _p(v_new), _p(k_cache), _p(v_cache), _p(kv_start), _p(kv_len),
        _p(kc_cache), _p(vc_cache), _p(cmp_start), _phi(phi), _stream(stream)))


def backward(c: dict, q, k, v, gates, dout, idx, phi=None, stream=None, want_phi_grads=False,
             ws=None) -> dict:
    """Gradients with the selection idx [B,T,G,n] held fixed: dq, dk, dv, dgates (fp32); with
    want_phi_grads (linear phi) also dwk [dk, l*dk], dek [l, dk], dwv [dv, l*dv], dev [l, dv]."""
    B, T, H, G, dk, dv = c["B"], c["T"], c["H"], c["G"], c["dk"], c["dv"]
    f32 = dict(dtype=torch.float32, device=q.device)
    res = {"dq": torch.empty(B, T, H, dk, **f32), "dk": torch.empty(B, T, G, dk, **f32),
           "dv": torch.empty(B, T, G, dv, **f32), "dgates": torch.empty(B, T, H, 3, **f32)}
    if ws is None:
        ws = alloc_workspace(c, NSA_MODE_BACKWARD, q.device)
    cfg = make_config(c)
    _check("nsa_backward", lib().nsa_backward(
        ctypes.byref(cfg), _p(q), _p(k), _p(v), _p(gates), _phi(phi), _p(dout), _p(idx),
        _p(res["dq"]), _p(res["dk"]), _p(res["dv"]), _p(res["dgates"]), _p(ws), ws.numel(),
        _stream(stream)))
    if want_phi_grads:
        _phi_grads(c, cfg, k, v, phi, ws, stream, res)
    return res


def check_timeout_path(limit_ns: int = 1_000_000, stream=None):
    """Launch the failure-detection self-test: a bounded wait that nothing satisfies
    expires after limit_ns; the next sync_status() raises NsaError (device timeout)."""
    _check("nsa_check_timeout_path", lib().nsa_check_timeout_path(int(limit_ns), _stream(stream)))


def sync_status(stream=None):
    """Synchronise and raise if a kernel's bounded wait expired since the last check."""
    _check("nsa_sync_status", lib().nsa_sync_status(_stream(stream)))


def profile_enable(on: bool = True):
    """Bracket every kernel launch of the entry points with CUDA events."""
    lib().nsa_profile_enable(1 if on else 0)


def profile_read(max_kernels: int = 64) -> dict:
    """{kernel name: (launches, total device ms)} since the previous read."""
    names = ctypes.create_string_buffer(48 * max_kernels)
    launches = (ctypes.c_int32 * max_kernels)()
    ms = (ctypes.c_float * max_kernels)()
    n = lib().nsa_profile_read(max_kernels, names, ctypes.cast(launches, _P), ctypes.cast(ms, _P))
    if n < 0:
        raise NsaError("nsa_profile_read", 4)
    out = {}
    for k in range(n):
        name = names.raw[48 * k:48 * (k + 1)].split(b"\0", 1)[0].decode()
        out[name] = (int(launches[k]), float(ms[k]))
    return out
