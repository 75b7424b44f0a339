"""ctypes binding of the C oracle (``nsa_oracle.c``), built with gcc + OpenMP.

Test infrastructure only: see the package docstring.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nsa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libnsa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/_build/libnsa_oracle.so."""
    os.makedirs(_BUILD, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Params(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("l", ctypes.c_int), ("d", ctypes.c_int), ("lsel", ctypes.c_int),
                ("n", ctypes.c_int), ("w", ctypes.c_int), ("scale", ctypes.c_double)]


class _DsaParams(ctypes.Structure):
    _fields_ = [("Hi", ctypes.c_int), ("Di", ctypes.c_int), ("top_k", ctypes.c_int)]


@dataclasses.dataclass(frozen=True)
class OracleParams:
    head_dim: int
    num_q_heads: int
    num_kv_heads: int
    cmp_block: int
    cmp_stride: int
    sel_block: int
    top_n: int
    window: int
    scale: float = 0.0

    @classmethod
    def of(cls, cfg) -> "OracleParams":
        return cls(cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads, cfg.cmp_block,
                   cfg.cmp_stride, cfg.sel_block, cfg.top_n, cfg.window)

    def c(self) -> _Params:
        s = self.scale if self.scale > 0 else 1.0 / math.sqrt(self.head_dim)
        return _Params(self.head_dim, self.num_q_heads, self.num_kv_heads, self.cmp_block,
                       self.cmp_stride, self.sel_block, self.top_n, self.window, s)


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.POINTER(_Params)
            vp = ctypes.c_void_p
            lib.oracle_compress.argtypes = [P, ctypes.c_int, vp, vp, vp, vp]
            lib.oracle_compress.restype = None
            lib.oracle_nsa_rows.argtypes = [P, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp,
                                            ctypes.c_int, vp, vp, vp, vp, vp, vp, ctypes.c_int,
                                            vp, vp]
            lib.oracle_nsa_rows.restype = ctypes.c_int
            lib.oracle_nsa_query.argtypes = [P, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp,
                                             vp, vp, vp, vp, ctypes.c_int, vp, vp]
            lib.oracle_nsa_query.restype = ctypes.c_int
            lib.oracle_select_f32.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, vp,
                                              ctypes.c_int, vp, vp]
            lib.oracle_select_f32.restype = None
            lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
            lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
            lib.oracle_num_cmp_blocks.argtypes = [P, ctypes.c_int]
            lib.oracle_num_cmp_blocks.restype = ctypes.c_int
            lib.oracle_block_means.argtypes = [P, ctypes.c_int, vp, vp, vp]
            lib.oracle_block_means.restype = None
            lib.oracle_block_select_rows.argtypes = [P, ctypes.c_int, vp, vp, vp, vp, vp,
                                                     ctypes.c_int, vp, vp, ctypes.c_int, vp, vp]
            lib.oracle_block_select_rows.restype = ctypes.c_int
            lib.oracle_block_select_query.argtypes = [P, ctypes.c_int, vp, vp, vp, vp, vp, vp,
                                                      ctypes.c_int, vp, vp]
            lib.oracle_block_select_query.restype = ctypes.c_int
            lib.oracle_dsa_rows.argtypes = [P, ctypes.POINTER(_DsaParams), ctypes.c_int, vp, vp, vp,
                                            vp, vp, vp, vp, ctypes.c_int, vp, vp, vp, vp]
            lib.oracle_dsa_rows.restype = ctypes.c_int
            lib.oracle_backward.argtypes = [P, ctypes.c_int] + [vp] * 11 + [ctypes.c_int] + [vp] * 8
            lib.oracle_backward.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_cmp_blocks(p: OracleParams, T: int) -> int:
    return int(_load().oracle_num_cmp_blocks(ctypes.byref(p.c()), int(T)))


def bf16_round_f64(x: float) -> int:
    """fp64 -> bf16 bits, one rounding to nearest even."""
    return int(_load().oracle_f64_to_bf16(float(x)))


def compress(p: OracleParams, x_bits: np.ndarray, w: np.ndarray):
    """Step 1 for one sequence: x [T,Hkv,D] bf16 bits, w [Hkv,D,l*D] fp32.
    Returns (fp64 [C,Hkv,D], bf16 bits [C,Hkv,D])."""
    x = _c(x_bits, np.uint16)
    w = _c(w, np.float32)
    T = x.shape[0]
    C = num_cmp_blocks(p, T)
    f = np.zeros((C, p.num_kv_heads, p.head_dim), dtype=np.float64)
    b = np.zeros((C, p.num_kv_heads, p.head_dim), dtype=np.uint16)
    if C:
        _load().oracle_compress(ctypes.byref(p.c()), T, _ptr(x), _ptr(w), _ptr(f), _ptr(b))
    return f, b


def nsa_rows(p: OracleParams, q, k, v, kc, vc, gates, rows, cmax: int | None = None) -> dict:
    """Steps 2-7 for the query rows `rows` of one sequence.

    q [T,Hq,D], k/v [T,Hkv,D], kc/vc [C,Hkv,D] (bf16 bits), gates [T,Hq,3].
    Returns fp64 o_cmp/o_slc/o_win/out [R,Hq,D], lse [R,Hq], scores
    [R,Hkv,cmax], sel [R,Hkv,n] (int32) and gap [R,Hkv]."""
    q, k, v = _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    kc, vc = _c(kc, np.uint16), _c(vc, np.uint16)
    gates = _c(gates, np.float32)
    rows = _c(rows, np.int32)
    T = q.shape[0]
    R, Hq, Hkv, D, n = len(rows), p.num_q_heads, p.num_kv_heads, p.head_dim, p.top_n
    if cmax is None:
        cmax = max(1, T // p.cmp_block)
    res = {name: np.zeros((R, Hq, D)) for name in ("o_cmp", "o_slc", "o_win", "out")}
    res["lse"] = np.zeros((R, Hq))
    res["scores"] = np.zeros((R, Hkv, cmax))
    res["sel"] = np.zeros((R, Hkv, n), dtype=np.int32)
    res["gap"] = np.zeros((R, Hkv))
    rc = _load().oracle_nsa_rows(ctypes.byref(p.c()), T, _ptr(q), _ptr(k), _ptr(v), _ptr(kc),
                                 _ptr(vc), _ptr(gates), _ptr(rows), R, _ptr(res["o_cmp"]),
                                 _ptr(res["o_slc"]), _ptr(res["o_win"]), _ptr(res["out"]),
                                 _ptr(res["lse"]), _ptr(res["scores"]), cmax, _ptr(res["sel"]),
                                 _ptr(res["gap"]))
    if rc != 0:
        raise ValueError("oracle rejected the geometry or a row index")
    return res


def nsa_query(p: OracleParams, t: int, q_row, k, v, kc, vc, gates_row, cmax: int) -> dict:
    """Steps 2-7 for a single query at position t (decode): q_row [Hq,D],
    k/v [>=t+1,Hkv,D], kc/vc [>=C,Hkv,D], gates_row [Hq,3]."""
    q_row, k, v = _c(q_row, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    kc, vc, gates_row = _c(kc, np.uint16), _c(vc, np.uint16), _c(gates_row, np.float32)
    Hq, Hkv, D, n = p.num_q_heads, p.num_kv_heads, p.head_dim, p.top_n
    res = {name: np.zeros((Hq, D)) for name in ("o_cmp", "o_slc", "o_win", "out")}
    res["lse"] = np.zeros(Hq)
    res["scores"] = np.zeros((Hkv, cmax))
    res["sel"] = np.zeros((Hkv, n), dtype=np.int32)
    res["gap"] = np.zeros(Hkv)
    rc = _load().oracle_nsa_query(ctypes.byref(p.c()), int(t), _ptr(q_row), _ptr(k), _ptr(v),
                                  _ptr(kc), _ptr(vc), _ptr(gates_row), _ptr(res["o_cmp"]),
                                  _ptr(res["o_slc"]), _ptr(res["o_win"]), _ptr(res["out"]),
                                  _ptr(res["lse"]), _ptr(res["scores"]), cmax,
                                  _ptr(res["sel"]), _ptr(res["gap"]))
    if rc != 0:
        raise ValueError("oracle rejected the geometry")
    return res


def select_f32(scores: np.ndarray, ncand: np.ndarray, cmp_n: np.ndarray, n: int):
    """Step 4 alone on fp32 score rows [R, cstride]: returns (sel [R,n], gap [R])."""
    s = _c(scores, np.float32)
    R, cs = s.shape
    sel = np.zeros((R, n), dtype=np.int32)
    gap = np.zeros(R)
    _load().oracle_select_f32(_ptr(s), R, cs, _ptr(_c(ncand, np.int32)), _ptr(_c(cmp_n, np.int32)),
                              n, _ptr(sel), _ptr(gap))
    return sel, gap


def prefill_reference(p: OracleParams, inputs: dict, rows_per_seq=None, kc_override=None,
                      vc_override=None) -> list[dict]:
    """Oracle over a packed prefill batch from ``workloads.prefill_inputs``.

    rows_per_seq: per sequence, the local rows to evaluate (default: all).
    kc_override / vc_override: packed [C_total,Hkv,D] bf16 compressed KV to
    use in steps 2-7 instead of the oracle's own step 1 (stage-wise checks).
    Returns one dict per sequence (with "kc"/"vc" fp64 + bf16 of step 1)."""
    cu = inputs["cu_seqlens"]
    out = []
    coff = 0
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        T = e - s
        C = num_cmp_blocks(p, T)
        kc64, kc16 = compress(p, inputs["k"][s:e], inputs["w_k"])
        vc64, vc16 = compress(p, inputs["v"][s:e], inputs["w_v"])
        kc_use = kc16 if kc_override is None else kc_override[coff:coff + C]
        vc_use = vc16 if vc_override is None else vc_override[coff:coff + C]
        coff += C
        rows = np.arange(T) if rows_per_seq is None else np.asarray(rows_per_seq[b])
        r = nsa_rows(p, inputs["q"][s:e], inputs["k"][s:e], inputs["v"][s:e],
                     kc_use if C else np.zeros((1, p.num_kv_heads, p.head_dim), np.uint16),
                     vc_use if C else np.zeros((1, p.num_kv_heads, p.head_dim), np.uint16),
                     inputs["gates"][s:e], rows)
        r.update(rows=rows, kc64=kc64, kc16=kc16, vc64=vc64, vc16=vc16)
        out.append(r)
    return out


def decode_reference(p: OracleParams, inputs: dict, b: int, kc=None, vc=None) -> dict:
    """Oracle for decode sequence b of ``workloads.decode_inputs``: the query is
    the token at t = len-1; the compressed cache is used as given, except the
    block completed by the new token (len % l == 0), which step 1 computes."""
    L = int(inputs["seqlens"][b])
    t = L - 1
    k, v = inputs["k"][b], inputs["v"][b]
    kc = np.array(inputs["kc"][b] if kc is None else kc, copy=True)
    vc = np.array(inputs["vc"][b] if vc is None else vc, copy=True)
    C = num_cmp_blocks(p, L)
    # the newest token completes compressed block C - 1 when its last token
    # (C - 1) * d + l - 1 is the newest one
    if C > 0 and (C - 1) * p.cmp_stride + p.cmp_block == L:
        blk = C - 1
        s = blk * p.cmp_stride
        _, kb = compress(p, k[s:s + p.cmp_block], inputs["w_k"])
        _, vb = compress(p, v[s:s + p.cmp_block], inputs["w_v"])
        kc[blk], vc[blk] = kb[0], vb[0]
    r = nsa_query(p, t, inputs["q"][b], k, v, kc, vc, inputs["gates"][b], cmax=kc.shape[0])
    r.update(kc_used=kc, vc_used=vc, t=t)
    return r


# ---------------------------------------------------------------- select-only block attention
def block_means(p: OracleParams, x_bits: np.ndarray):
    """Mean keys of the complete l'-token blocks of one sequence: x [T,Hkv,D]
    bf16 bits.  Returns (fp64 [T//l',Hkv,D], bf16 bits [T//l',Hkv,D])."""
    x = _c(x_bits, np.uint16)
    nb = x.shape[0] // p.sel_block
    f = np.zeros((nb, p.num_kv_heads, p.head_dim), dtype=np.float64)
    b = np.zeros((nb, p.num_kv_heads, p.head_dim), dtype=np.uint16)
    if nb:
        _load().oracle_block_means(ctypes.byref(p.c()), x.shape[0], _ptr(x), _ptr(f), _ptr(b))
    return f, b


def block_select_rows(p: OracleParams, q, k, v, kbar, rows, cmax: int | None = None) -> dict:
    """Select-only block attention for the query rows `rows` of one sequence.

    q [T,Hq,D], k/v [T,Hkv,D], kbar [>=1,Hkv,D] (bf16 bits).  Returns fp64 out
    [R,Hq,D], scores [R,Hkv,cmax] (routing scores of the complete blocks
    before each row's block), sel [R,Hkv,n] (int32) and gap [R,Hkv]."""
    q, k, v, kbar = _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16), _c(kbar, np.uint16)
    rows = _c(rows, np.int32)
    T = q.shape[0]
    R, Hq, Hkv, D, n = len(rows), p.num_q_heads, p.num_kv_heads, p.head_dim, p.top_n
    if cmax is None:
        cmax = max(1, T // p.sel_block)
    res = {"out": np.zeros((R, Hq, D)), "scores": np.zeros((R, Hkv, cmax)),
           "sel": np.zeros((R, Hkv, n), dtype=np.int32), "gap": np.zeros((R, Hkv))}
    rc = _load().oracle_block_select_rows(ctypes.byref(p.c()), T, _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(kbar), _ptr(rows), R, _ptr(res["out"]),
                                          _ptr(res["scores"]), cmax, _ptr(res["sel"]),
                                          _ptr(res["gap"]))
    if rc != 0:
        raise ValueError("oracle rejected the geometry or a row index")
    return res


def block_select_reference(p: OracleParams, inputs: dict, rows_per_seq=None,
                           kbar_override=None) -> list[dict]:
    """Select-only block attention over a packed batch from
    ``workloads.prefill_inputs`` (q, k, v, cu_seqlens are used).
    kbar_override: packed [sum T_b // l', Hkv, D] bf16 mean keys to route with
    instead of the oracle's own (stage-wise checks)."""
    cu = inputs["cu_seqlens"]
    out = []
    boff = 0
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        T = e - s
        nb = T // p.sel_block
        kb64, kb16 = block_means(p, inputs["k"][s:e])
        use = kb16 if kbar_override is None else kbar_override[boff:boff + nb]
        boff += nb
        rows = np.arange(T) if rows_per_seq is None else np.asarray(rows_per_seq[b])
        r = block_select_rows(p, inputs["q"][s:e], inputs["k"][s:e], inputs["v"][s:e],
                              use if nb else np.zeros((1, p.num_kv_heads, p.head_dim), np.uint16),
                              rows)
        r.update(rows=rows, kbar64=kb64, kbar16=kb16)
        out.append(r)
    return out


def block_select_query(p: OracleParams, t: int, q_row, k, v, kbar, cmax: int) -> dict:
    """Select-only block attention for a single query at position t (decode):
    q_row [Hq,D], k/v [>=t+1,Hkv,D], kbar [>=max(1, t // l'),Hkv,D]."""
    q_row, k, v, kbar = _c(q_row, np.uint16), _c(k, np.uint16), _c(v, np.uint16), _c(kbar, np.uint16)
    Hq, Hkv, D, n = p.num_q_heads, p.num_kv_heads, p.head_dim, p.top_n
    res = {"out": np.zeros((Hq, D)), "scores": np.zeros((Hkv, cmax)),
           "sel": np.zeros((Hkv, n), dtype=np.int32), "gap": np.zeros(Hkv)}
    rc = _load().oracle_block_select_query(ctypes.byref(p.c()), int(t), _ptr(q_row), _ptr(k),
                                           _ptr(v), _ptr(kbar), _ptr(res["out"]),
                                           _ptr(res["scores"]), cmax, _ptr(res["sel"]),
                                           _ptr(res["gap"]))
    if rc != 0:
        raise ValueError("oracle rejected the geometry")
    return res


def block_select_decode_reference(p: OracleParams, q_row, k_seq, v_seq, kmean, L: int) -> dict:
    """Select-only decode of the newest token (t = L - 1) of one sequence:
    k_seq/v_seq [>=L,Hkv,D] the caches, kmean [>=1,Hkv,D] the routing keys of
    the complete blocks before the newest token.  The routing key of the block
    the newest token completes (L % l' == 0) is computed here ("written")."""
    ls = p.sel_block
    t = L - 1
    written = None
    if L % ls == 0:
        _, written = block_means(p, k_seq[L - ls:L])
        written = written[0]
    kb = kmean if kmean.shape[0] else np.zeros((1, p.num_kv_heads, p.head_dim), np.uint16)
    r = block_select_query(p, t, q_row, k_seq, v_seq, kb, cmax=max(1, kb.shape[0]))
    r.update(t=t, written=written)
    return r


# ---------------------------------------------------------------- token-level selection (DSA style)
def dsa_rows(p: OracleParams, top_k: int, q, k, v, qi, w, ki, rows, with_index: bool = False) -> dict:
    """Token-level top-k attention for the query rows `rows` of one sequence:
    q [T,Hq,D], k/v [T,Hkv,D], qi [T,Hi,Di], ki [T,Di] (bf16 bits), w [T,Hi]
    fp32.  Returns fp64 out [R,Hq,D], sel [R,top_k] (int32), gap [R] and,
    with_index, the index scores [R,T] (entries > t are 0)."""
    q, k, v = _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    qi, ki, w = _c(qi, np.uint16), _c(ki, np.uint16), _c(w, np.float32)
    rows = _c(rows, np.int32)
    T, Hi, Di = qi.shape
    R, Hq, D = len(rows), p.num_q_heads, p.head_dim
    x = _DsaParams(Hi, Di, int(top_k))
    res = {"out": np.zeros((R, Hq, D)), "sel": np.zeros((R, top_k), dtype=np.int32),
           "gap": np.zeros(R)}
    idx = np.zeros((R, T)) if with_index else None
    rc = _load().oracle_dsa_rows(ctypes.byref(p.c()), ctypes.byref(x), T, _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(qi), _ptr(w), _ptr(ki), _ptr(rows), R, _ptr(res["out"]),
                                 _ptr(idx) if with_index else None, _ptr(res["sel"]),
                                 _ptr(res["gap"]))
    if rc != 0:
        raise ValueError("oracle rejected the geometry or a row index")
    if with_index:
        res["index"] = idx
    return res


def backward_c(p: OracleParams, q, k, v, gates, w_k, w_v, sel, dout, kc=None, vc=None,
               rows=None) -> dict:
    """The backward of ``oracle.backward.backward`` (same arguments and
    results: fp64 inputs, the selection held fixed) in C with OpenMP over
    query rows, for sizes where the numpy loops are slow."""
    D, Hq, Hkv = p.head_dim, p.num_q_heads, p.num_kv_heads
    q, k, v = _c(q, np.float64), _c(k, np.float64), _c(v, np.float64)
    gates, dout = _c(gates, np.float64), _c(dout, np.float64)
    w_k, w_v = _c(w_k, np.float64), _c(w_v, np.float64)
    sel = _c(sel, np.int32)
    T = q.shape[0]
    C = num_cmp_blocks(p, T)
    kc = None if kc is None else _c(kc, np.float64)
    vc = None if vc is None else _c(vc, np.float64)
    rr = None if rows is None else _c(rows, np.int32)
    res = {"dq": np.zeros((T, Hq, D)), "dk": np.zeros((T, Hkv, D)), "dv": np.zeros((T, Hkv, D)),
           "dgates": np.zeros((T, Hq, 3)), "dw_k": np.zeros(w_k.shape), "dw_v": np.zeros(w_v.shape),
           "dkc": np.zeros((C, Hkv, D)), "dvc": np.zeros((C, Hkv, D))}
    none = ctypes.c_void_p(None)
    rc = _load().oracle_backward(
        ctypes.byref(p.c()), T, _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(w_k), _ptr(w_v),
        _ptr(sel), _ptr(dout), none if kc is None else _ptr(kc), none if vc is None else _ptr(vc),
        none if rr is None else _ptr(rr), 0 if rr is None else len(rr),
        *[_ptr(res[name]) for name in ("dq", "dk", "dv", "dgates", "dw_k", "dw_v", "dkc", "dvc")])
    if rc != 0:
        raise ValueError("oracle rejected the geometry")
    return res
