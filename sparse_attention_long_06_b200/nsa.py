"""ctypes binding of libnsa_b200.so (declared in include/nsa.h).

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels of the library.  torch supplies device memory and streams.  There is
no fallback: if the library is missing or a call fails, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libnsa_b200.so")

NSA_OK = 0
NSA_ERR_INVALID_ARG = 1
NSA_ERR_UNSUPPORTED = 2
NSA_ERR_MISALIGNED = 3
NSA_ERR_WORKSPACE = 4
NSA_ERR_CUDA = 5
NSA_ERR_DEVICE_TIMEOUT = 6
NSA_ERR_DEVICE_BAD_INPUT = 7
OUT_BF16, OUT_F32 = 0, 1
MODE_PREFILL, MODE_DECODE, MODE_BLOCK_SELECT, MODE_BLOCK_SELECT_DECODE = 0, 1, 2, 3
WS_STATUS, WS_O_CMP, WS_LSE, WS_SCORES, WS_SEL, WS_WIN, WS_SEL_SCORES = 0, 1, 2, 3, 4, 5, 6

EXPORTED = ["nsa_plan_create", "nsa_plan_destroy", "nsa_workspace_size", "nsa_workspace_region",
            "nsa_cmp_rows", "nsa_prefill", "nsa_decode", "nsa_read_device_status",
            "nsa_selftest_timeout", "nsa_strerror", "nsa_last_launch_count",
            "nsa_profile_enable", "nsa_profile_stage_ms", "nsa_prefill_noalloc",
            "nsa_plan", "nsa_noalloc_read_device_status", "nsa_block_select_prefill",
            "nsa_block_rows", "nsa_block_select_decode", "nsa_token_select_prefill",
            "nsa_token_select_workspace_size"]


class NsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {strerror(code)} ({code})")
        self.code = code


class Params(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int), ("num_q_heads", ctypes.c_int),
                ("num_kv_heads", ctypes.c_int), ("cmp_block", ctypes.c_int),
                ("cmp_stride", ctypes.c_int), ("sel_block", ctypes.c_int),
                ("top_n", ctypes.c_int), ("window", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("max_batch", ctypes.c_int),
                ("max_seqlen", ctypes.c_int), ("max_total_tokens", ctypes.c_int),
                ("out_dtype", ctypes.c_int)]


_lib = None
_lock = threading.Lock()


def lib():
    """Load the library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m sparse_attention_long_06_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            L.nsa_plan_create.argtypes = [ctypes.POINTER(Params), ctypes.POINTER(vp)]
            L.nsa_plan_create.restype = i
            L.nsa_plan.argtypes = [ctypes.POINTER(Params), ctypes.POINTER(vp)]
            L.nsa_plan.restype = i
            L.nsa_plan_destroy.argtypes = [vp]
            L.nsa_plan_destroy.restype = None
            L.nsa_workspace_size.argtypes = [vp, i]
            L.nsa_workspace_size.restype = sz
            L.nsa_workspace_region.argtypes = [vp, i, i, ctypes.POINTER(sz), ctypes.POINTER(sz)]
            L.nsa_workspace_region.restype = i
            L.nsa_cmp_rows.argtypes = [vp, i]
            L.nsa_cmp_rows.restype = i
            L.nsa_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, vp, vp, sz, vp]
            L.nsa_prefill.restype = i
            L.nsa_prefill_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, vp, vp]
            L.nsa_prefill_noalloc.restype = i
            L.nsa_block_select_prefill.argtypes = [vp, vp, vp, vp, vp, i, i, vp, vp, vp, vp, sz, vp]
            L.nsa_block_select_prefill.restype = i
            L.nsa_block_select_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, sz, vp]
            L.nsa_block_select_decode.restype = i
            L.nsa_token_select_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, vp, i, i,
                                                    vp, vp, vp, sz, vp]
            L.nsa_token_select_prefill.restype = i
            L.nsa_token_select_workspace_size.argtypes = [vp, i]
            L.nsa_token_select_workspace_size.restype = sz
            L.nsa_block_rows.argtypes = [vp, i]
            L.nsa_block_rows.restype = i
            L.nsa_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, vp, vp, vp, vp, vp, vp, sz, vp]
            L.nsa_decode.restype = i
            L.nsa_read_device_status.argtypes = [vp, vp]
            L.nsa_read_device_status.restype = i
            L.nsa_noalloc_read_device_status.argtypes = [vp]
            L.nsa_noalloc_read_device_status.restype = i
            L.nsa_selftest_timeout.argtypes = [vp, sz, ctypes.c_longlong, vp]
            L.nsa_selftest_timeout.restype = i
            L.nsa_strerror.argtypes = [i]
            L.nsa_strerror.restype = ctypes.c_char_p
            L.nsa_last_launch_count.argtypes = []
            L.nsa_last_launch_count.restype = i
            L.nsa_profile_enable.argtypes = [i]
            L.nsa_profile_enable.restype = i
            L.nsa_profile_stage_ms.argtypes = [ctypes.POINTER(ctypes.c_float), i]
            L.nsa_profile_stage_ms.restype = i
            _lib = L
    return _lib


def strerror(code: int) -> str:
    try:
        return lib().nsa_strerror(int(code)).decode()
    except Exception:  # pragma: no cover - library missing
        return "library unavailable"


def _check(code: int, what: str):
    if code != NSA_OK:
        raise NsaError(code, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Plan:
    """An nsa_plan_t with the NSA geometry and the per-call upper bounds."""

    def __init__(self, head_dim, num_q_heads, num_kv_heads, cmp_block, cmp_stride, sel_block,
                 top_n, window, max_batch, max_seqlen, max_total_tokens=0, out_dtype=OUT_BF16,
                 softmax_scale=0.0):
        self.params = Params(head_dim, num_q_heads, num_kv_heads, cmp_block, cmp_stride,
                             sel_block, top_n, window, float(softmax_scale), max_batch,
                             max_seqlen, max_total_tokens, out_dtype)
        h = ctypes.c_void_p()
        _check(lib().nsa_plan(ctypes.byref(self.params), ctypes.byref(h)), "nsa_plan")
        self.handle = h

    @classmethod
    def for_config(cls, cfg, max_batch, max_seqlen, max_total_tokens=0, out_dtype=OUT_BF16):
        return cls(cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads, cfg.cmp_block,
                   cfg.cmp_stride, cfg.sel_block, cfg.top_n, cfg.window, max_batch, max_seqlen,
                   max_total_tokens, out_dtype)

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            try:
                lib().nsa_plan_destroy(self.handle)
            except (TypeError, AttributeError):  # interpreter shutdown: module state is gone
                pass
            self.handle = None

    __del__ = close

    def workspace_size(self, mode=MODE_PREFILL) -> int:
        return int(lib().nsa_workspace_size(self.handle, mode))

    def workspace_region(self, region, mode=MODE_PREFILL):
        off, nb = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().nsa_workspace_region(self.handle, mode, region, ctypes.byref(off),
                                          ctypes.byref(nb)), "nsa_workspace_region")
        return off.value, nb.value

    def cmp_rows(self, total_tokens: int) -> int:
        return int(lib().nsa_cmp_rows(self.handle, total_tokens))

    def alloc_workspace(self, mode=MODE_PREFILL, device="cuda"):
        import torch
        return torch.empty(max(self.workspace_size(mode), 256), dtype=torch.uint8, device=device)

    def prefill(self, q, k, v, gates, w_k, w_v, cu_seqlens, out, k_cmp, v_cmp, workspace,
                sel_idx=None, stream=None):
        """Packed causal prefill; all tensors are CUDA tensors (bf16 stored as
        torch.bfloat16 or int16/uint16).  Launches asynchronously."""
        batch = cu_seqlens.numel() - 1
        total = q.shape[0]
        rc = lib().nsa_prefill(self.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(w_k),
                               _ptr(w_v), _ptr(cu_seqlens), batch, total, _ptr(out), _ptr(k_cmp),
                               _ptr(v_cmp), _ptr(sel_idx), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
        _check(rc, "nsa_prefill")

    def prefill_noalloc(self, q, k, v, gates, w_k, w_v, cu_seqlens, out, k_cmp, v_cmp,
                        sel_idx=None, stream=None):
        """nsa_prefill on the library's static device workspace (no caller
        workspace; for plans whose workspace fits in 32 MiB)."""
        batch = cu_seqlens.numel() - 1
        total = q.shape[0]
        rc = lib().nsa_prefill_noalloc(self.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(gates),
                                       _ptr(w_k), _ptr(w_v), _ptr(cu_seqlens), batch, total,
                                       _ptr(out), _ptr(k_cmp), _ptr(v_cmp), _ptr(sel_idx),
                                       _stream(stream))
        _check(rc, "nsa_prefill_noalloc")

    def block_rows(self, total_tokens: int) -> int:
        return int(lib().nsa_block_rows(self.handle, total_tokens))

    def block_select_prefill(self, q, k, v, cu_seqlens, out, k_mean, workspace, sel_idx=None,
                             stream=None):
        """Select-only block attention over a packed batch (the own block plus
        the n - 1 best-routed earlier blocks of l' tokens); workspace of
        workspace_size(MODE_BLOCK_SELECT) bytes."""
        batch = cu_seqlens.numel() - 1
        total = q.shape[0]
        rc = lib().nsa_block_select_prefill(self.handle, _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(cu_seqlens), batch, total, _ptr(out),
                                            _ptr(k_mean), _ptr(sel_idx), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(),
                                            _stream(stream))
        _check(rc, "nsa_block_select_prefill")

    def token_select_workspace_size(self, top_k: int) -> int:
        return int(lib().nsa_token_select_workspace_size(self.handle, int(top_k)))

    def token_select_prefill(self, q, k, v, q_index, w_index, k_index, top_k, cu_seqlens, out,
                             workspace, sel_idx=None, stream=None):
        """Token-level top-k attention over a packed batch: an indexer
        (q_index [T, Hi, Di], w_index [T, Hi], k_index [T, Di]) picks each
        query's top_k earlier tokens, every query head attends to them."""
        batch = cu_seqlens.numel() - 1
        total = q.shape[0]
        rc = lib().nsa_token_select_prefill(self.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(q_index),
                                            _ptr(w_index), _ptr(k_index), q_index.shape[1],
                                            q_index.shape[2], int(top_k), _ptr(cu_seqlens),
                                            batch, total, _ptr(out), _ptr(sel_idx),
                                            _ptr(workspace),
                                            workspace.numel() * workspace.element_size(),
                                            _stream(stream))
        _check(rc, "nsa_token_select_prefill")

    def block_select_decode(self, q, k_cache, v_cache, k_mean_cache, seqlens, out, workspace,
                            sel_idx=None, stream=None):
        """One select-only decode step (caches include the newest token);
        workspace of workspace_size(MODE_BLOCK_SELECT_DECODE) bytes."""
        batch = q.shape[0]
        cap = k_cache.shape[1]
        rc = lib().nsa_block_select_decode(self.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                           _ptr(k_mean_cache), _ptr(seqlens), batch, cap,
                                           _ptr(out), _ptr(sel_idx), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream))
        _check(rc, "nsa_block_select_decode")

    def decode(self, q, k_cache, v_cache, k_cmp_cache, v_cmp_cache, seqlens, gates, w_k, w_v,
               out, workspace, sel_idx=None, stream=None):
        """One decode step for a batch (caches include the newest token)."""
        batch = q.shape[0]
        cap = k_cache.shape[1]
        rc = lib().nsa_decode(self.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache),
                              _ptr(k_cmp_cache), _ptr(v_cmp_cache), _ptr(seqlens), batch, cap,
                              _ptr(gates), _ptr(w_k), _ptr(w_v), _ptr(out), _ptr(sel_idx),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(stream))
        _check(rc, "nsa_decode")


def read_device_status(workspace, stream=None) -> int:
    return int(lib().nsa_read_device_status(_ptr(workspace), _stream(stream)))


def noalloc_read_device_status(stream=None) -> int:
    """Status word of the last nsa_prefill_noalloc call on the current device
    (synchronises the stream, then clears the word)."""
    return int(lib().nsa_noalloc_read_device_status(_stream(stream)))


def selftest_timeout(workspace, cycles: int, stream=None):
    _check(lib().nsa_selftest_timeout(_ptr(workspace), workspace.numel(), int(cycles),
                                      _stream(stream)), "nsa_selftest_timeout")


def last_launch_count() -> int:
    return int(lib().nsa_last_launch_count())


def profile_enable(on: bool = True):
    lib().nsa_profile_enable(1 if on else 0)


def profile_stage_ms(max_stages: int = 16) -> list[float]:
    """Per-launch milliseconds of the last profiled call (synchronises)."""
    buf = (ctypes.c_float * max_stages)()
    n = lib().nsa_profile_stage_ms(buf, max_stages)
    if n < 0:
        raise NsaError(NSA_ERR_CUDA, "nsa_profile_stage_ms")
    return [float(buf[i]) for i in range(min(n, max_stages))]
