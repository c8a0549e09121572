"""Thin Python binding of libssa (the C ABI in include/ssa.h).

Two layers, both argument marshalling only:

* ``ssa_*`` functions with the C names and signatures; pointers and the
  stream are plain integers.
* ``select_blocks``, ``attn_fwd_dual``, ``align_loss``, ``attn_bwd``,
  ``attn_fwd_sparse``, ``diagnostics`` and ``DecodeCache`` (a key/value cache
  with its pooled keys, for ``ssa_decode_pool`` / ``ssa_decode_step``): take
  torch CUDA tensors, allocate the outputs and the workspace with torch, pass
  raw device pointers and torch's current stream to the C entry point and
  raise ``SsaError`` on a non-zero status.

Every compute step runs in the library's CUDA kernels.  There is no fallback:
importing this module without a built ``libssa.so`` raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from ctypes import POINTER, c_float, c_int, c_size_t, c_uint, c_void_p

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssa.so")

SSA_OK, SSA_ERR_INVALID_ARG, SSA_ERR_UNSUPPORTED = 0, -1, -2
SSA_ERR_WORKSPACE, SSA_ERR_CUDA, SSA_ERR_TIMEOUT = -3, -4, -5
SSA_F32, SSA_BF16 = 0, 1
SSA_FLAG_FORCE_SINK, SSA_FLAG_FORCE_SIMT = 1, 2
SSA_WS_SELECT, SSA_WS_FWD, SSA_WS_LOSS, SSA_WS_BWD, SSA_WS_FWD_SPARSE, SSA_WS_DECODE = range(6)

# every symbol include/ssa.h declares
EXPORTS = (
    "ssa_workspace_size", "ssa_select_blocks", "ssa_select_blocks_noalloc",
    "ssa_attn_fwd_dual", "ssa_attn_fwd_sparse", "ssa_attn_diagnostics", "ssa_attn_fwd_dual_diag",
    "ssa_decode_pool",
    "ssa_decode_step", "ssa_align_loss",
    "ssa_attn_bwd", "ssa_device_status", "ssa_status_string", "ssa_last_error",
    "ssa_kernel_path", "ssa_bwd_heads_per_group", "ssa_selftest_math", "ssa_selftest_wait_timeout",
    "ssa_debug_set_wait_limit_ns", "ssa_debug_set_ds_budget_bytes", "ssa_debug_set_kernel_events",
    "ssa_version",
)


class SsaError(RuntimeError):
    def __init__(self, where: str, status: int, detail: str):
        super().__init__(f"{where}: {status_string(status)} ({status}): {detail}")
        self.status = status


class ssa_params_t(ctypes.Structure):
    _fields_ = [("B", c_int), ("H", c_int), ("T", c_int), ("D", c_int), ("block", c_int),
                ("topk", c_int), ("dtype", c_int), ("sm_scale", c_float), ("flags", c_uint)]

    def __repr__(self):
        return ("ssa_params_t(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_)
                + ")")


_P = POINTER(ssa_params_t)
_SIGNATURES = {
    "ssa_workspace_size": (c_size_t, [_P, c_int]),
    "ssa_select_blocks": (c_int, [_P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_size_t, c_void_p]),
    "ssa_select_blocks_noalloc": (c_int, [_P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                          c_void_p]),
    "ssa_attn_fwd_dual": (c_int, [_P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_size_t, c_void_p]),
    "ssa_attn_fwd_sparse": (c_int, [_P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "ssa_attn_diagnostics": (c_int, [_P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p]),
    "ssa_attn_fwd_dual_diag": (c_int, [_P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                       c_void_p]),
    "ssa_decode_pool": (c_int, [_P, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "ssa_decode_step": (c_int, [_P, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "ssa_align_loss": (c_int, [_P, c_void_p, c_float, c_float, c_void_p, c_void_p, c_size_t,
                               c_void_p]),
    "ssa_attn_bwd": (c_int, [_P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_float, c_float, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_size_t, c_void_p]),
    "ssa_device_status": (c_int, [c_void_p]),
    "ssa_status_string": (ctypes.c_char_p, [c_int]),
    "ssa_last_error": (ctypes.c_char_p, []),
    "ssa_kernel_path": (c_int, [_P]),
    "ssa_bwd_heads_per_group": (c_int, [_P]),
    "ssa_selftest_math": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "ssa_version": (c_int, []),
    "ssa_debug_set_wait_limit_ns": (None, [ctypes.c_ulonglong]),
    "ssa_debug_set_ds_budget_bytes": (None, [ctypes.c_ulonglong]),
    "ssa_debug_set_kernel_events": (c_int, [c_void_p, c_int]),
    "ssa_selftest_wait_timeout": (c_int, [ctypes.c_ulonglong, c_void_p, c_void_p]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m block_sparse_full_b200.build` (no fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


# ------------------------------------------------------------ C-named entry points

def ssa_workspace_size(params, which):
    return _lib.ssa_workspace_size(ctypes.byref(params), which)


def ssa_select_blocks(params, q, k, idx, cnt, mask, ws, ws_bytes, stream):
    return _lib.ssa_select_blocks(ctypes.byref(params), q, k, idx, cnt, mask, ws, ws_bytes,
                                  stream)


def ssa_select_blocks_noalloc(params, q, k, idx, cnt, mask, stream):
    """Selection with the library's built-in scratch (no workspace argument)."""
    return _lib.ssa_select_blocks_noalloc(ctypes.byref(params), q, k, idx, cnt, mask, stream)


def ssa_attn_fwd_dual(params, q, k, v, idx, cnt, mask, h_full, h_sparse, delta, lse_full,
                      lse_sparse, sqdiff_rows, ws, ws_bytes, stream):
    return _lib.ssa_attn_fwd_dual(ctypes.byref(params), q, k, v, idx, cnt, mask, h_full,
                                  h_sparse, delta, lse_full, lse_sparse, sqdiff_rows, ws,
                                  ws_bytes, stream)


def ssa_attn_fwd_sparse(params, q, k, v, idx, cnt, mask, h_sparse, lse_sparse, ws, ws_bytes,
                        stream):
    return _lib.ssa_attn_fwd_sparse(ctypes.byref(params), q, k, v, idx, cnt, mask, h_sparse,
                                    lse_sparse, ws, ws_bytes, stream)


def ssa_attn_diagnostics(params, q, k, lse_full, delta, sink_rows, head_stats, stream):
    return _lib.ssa_attn_diagnostics(ctypes.byref(params), q, k, lse_full, delta, sink_rows,
                                     head_stats, stream)


def ssa_attn_fwd_dual_diag(params, q, k, v, idx, cnt, mask, h_full, h_sparse, delta, lse_full,
                           lse_sparse, sqdiff_rows, sink_rows, head_stats, ws, ws_bytes, stream):
    return _lib.ssa_attn_fwd_dual_diag(ctypes.byref(params), q, k, v, idx, cnt, mask, h_full,
                                       h_sparse, delta, lse_full, lse_sparse, sqdiff_rows,
                                       sink_rows, head_stats, ws, ws_bytes, stream)


def ssa_decode_pool(params, j0, j1, k_cache, kbar, stream):
    return _lib.ssa_decode_pool(ctypes.byref(params), j0, j1, k_cache, kbar, stream)


def ssa_decode_step(params, t, q, k_cache, v_cache, kbar, h, lse, idx, ws, ws_bytes, stream):
    return _lib.ssa_decode_step(ctypes.byref(params), t, q, k_cache, v_cache, kbar, h, lse, idx, ws,
                                ws_bytes, stream)


def ssa_align_loss(params, sqdiff_rows, w_sparsity, w_commit, loss_out, ws, ws_bytes, stream):
    return _lib.ssa_align_loss(ctypes.byref(params), sqdiff_rows, w_sparsity, w_commit,
                               loss_out, ws, ws_bytes, stream)


def ssa_attn_bwd(params, q, k, v, idx, cnt, mask, h_full, h_sparse, lse_full, lse_sparse,
                 dh_full, dh_sparse, w_sparsity, w_commit, dq, dk, dv, ws, ws_bytes, stream):
    return _lib.ssa_attn_bwd(ctypes.byref(params), q, k, v, idx, cnt, mask, h_full, h_sparse,
                             lse_full, lse_sparse, dh_full, dh_sparse, w_sparsity, w_commit,
                             dq, dk, dv, ws, ws_bytes, stream)


def ssa_device_status(stream):
    return _lib.ssa_device_status(stream)


def ssa_status_string(status):
    return _lib.ssa_status_string(status).decode()


def ssa_last_error():
    return _lib.ssa_last_error().decode()


def ssa_kernel_path(params):
    return _lib.ssa_kernel_path(ctypes.byref(params))


def ssa_selftest_math(x, n, exp2_poly, exp2_mufu, bf16_alu, stream):
    return _lib.ssa_selftest_math(x, n, exp2_poly, exp2_mufu, bf16_alu, stream)


def ssa_selftest_wait_timeout(limit_ns, gave_up, stream):
    return _lib.ssa_selftest_wait_timeout(limit_ns, gave_up, stream)


def ssa_debug_set_wait_limit_ns(ns):
    _lib.ssa_debug_set_wait_limit_ns(ns)


def ssa_debug_set_ds_budget_bytes(nbytes):
    _lib.ssa_debug_set_ds_budget_bytes(nbytes)


def ssa_bwd_heads_per_group(params):
    return _lib.ssa_bwd_heads_per_group(ctypes.byref(params))


def ssa_debug_set_kernel_events(events, n):
    return _lib.ssa_debug_set_kernel_events(events, n)


def ssa_version():
    return _lib.ssa_version()


status_string = ssa_status_string


def check(status: int, where: str):
    if status != SSA_OK:
        raise SsaError(where, status, ssa_last_error())


# ------------------------------------------------------------ tensor-level helpers

_DT = {torch.float32: SSA_F32, torch.bfloat16: SSA_BF16}


def make_params(B, H, T, D, block, topk, dtype, sm_scale=None, flags=0) -> ssa_params_t:
    if isinstance(dtype, torch.dtype):
        dtype = _DT[dtype]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    return ssa_params_t(B, H, T, D, block, topk, dtype, sm_scale, flags)


def params_for(q: torch.Tensor, block: int, topk: int, sm_scale=None, flags=0) -> ssa_params_t:
    B, H, T, D = q.shape
    return make_params(B, H, T, D, block, topk, q.dtype, sm_scale, flags)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def workspace(params, which, device) -> torch.Tensor:
    n = ssa_workspace_size(params, which)
    if n == ctypes.c_size_t(-1).value:
        raise SsaError("ssa_workspace_size", SSA_ERR_INVALID_ARG, ssa_last_error())
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device)


def select_blocks(params, q, k, ws=None):
    """Selection sets of the sparse stream -> (idx, cnt, mask) int32/int32/int32-bits."""
    _need(q, "q"), _need(k, "k")
    B, H, n = params.B, params.H, params.T // params.block
    words = (n + 31) // 32
    dev = q.device
    idx = torch.empty((B, H, n, params.topk), dtype=torch.int32, device=dev)
    cnt = torch.empty((B, H, n), dtype=torch.int32, device=dev)
    mask = torch.empty((B, H, n, words), dtype=torch.int32, device=dev)  # uint32 bits
    ws = workspace(params, SSA_WS_SELECT, dev) if ws is None else ws
    check(ssa_select_blocks(params, _ptr(q), _ptr(k), _ptr(idx), _ptr(cnt), _ptr(mask),
                            _ptr(ws), ws.numel(), _stream(dev)), "ssa_select_blocks")
    return idx, cnt, mask


def attn_fwd_dual(params, q, k, v, mask, idx=None, cnt=None, ws=None, out=None):
    """Both streams -> dict(h_full, h_sparse, delta, lse_full, lse_sparse, sqdiff)."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (mask, "mask")):
        _need(t, nm)
    dev = q.device
    rows = (params.B, params.H, params.T)
    if out is None:
        out = {
            "h_full": torch.empty_like(q), "h_sparse": torch.empty_like(q),
            **{nm: torch.empty(rows, dtype=torch.float32, device=dev)
               for nm in ("delta", "lse_full", "lse_sparse", "sqdiff")},
        }
    ws = workspace(params, SSA_WS_FWD, dev) if ws is None else ws
    check(ssa_attn_fwd_dual(params, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                            _ptr(mask), _ptr(out["h_full"]), _ptr(out["h_sparse"]),
                            _ptr(out["delta"]), _ptr(out["lse_full"]),
                            _ptr(out["lse_sparse"]), _ptr(out["sqdiff"]), _ptr(ws),
                            ws.numel(), _stream(dev)), "ssa_attn_fwd_dual")
    return out


def attn_fwd_sparse(params, q, k, v, mask, idx=None, cnt=None, ws=None, out=None):
    """The sparse stream alone (inference) -> dict(h_sparse, lse_sparse)."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (mask, "mask")):
        _need(t, nm)
    dev = q.device
    if out is None:
        out = {"h_sparse": torch.empty_like(q),
               "lse_sparse": torch.empty((params.B, params.H, params.T), dtype=torch.float32,
                                         device=dev)}
    ws = workspace(params, SSA_WS_FWD_SPARSE, dev) if ws is None else ws
    check(ssa_attn_fwd_sparse(params, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                              _ptr(mask), _ptr(out["h_sparse"]), _ptr(out["lse_sparse"]),
                              _ptr(ws), ws.numel(), _stream(dev)), "ssa_attn_fwd_sparse")
    return out


def diagnostics(params, q, k, fwd):
    """Sink mass per row and per-head means of delta and sink -> dict(sink, head_stats)."""
    _need(q, "q"), _need(k, "k")
    dev = q.device
    sink = torch.empty((params.B, params.H, params.T), dtype=torch.float32, device=dev)
    stats = torch.empty((params.B, params.H, 2), dtype=torch.float32, device=dev)
    check(ssa_attn_diagnostics(params, _ptr(q), _ptr(k), _ptr(fwd["lse_full"]), _ptr(fwd["delta"]),
                               _ptr(sink), _ptr(stats), _stream(dev)), "ssa_attn_diagnostics")
    return {"sink": sink, "head_stats": stats}


def attn_fwd_dual_diag(params, q, k, v, mask, idx=None, cnt=None, ws=None, out=None):
    """Both streams plus the diagnostics in one call -> the dict of
    ``attn_fwd_dual`` with ``sink`` [B,H,T] and ``head_stats`` [B,H,2] added."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (mask, "mask")):
        _need(t, nm)
    dev = q.device
    rows = (params.B, params.H, params.T)
    if out is None:
        out = {
            "h_full": torch.empty_like(q), "h_sparse": torch.empty_like(q),
            **{nm: torch.empty(rows, dtype=torch.float32, device=dev)
               for nm in ("delta", "lse_full", "lse_sparse", "sqdiff", "sink")},
            "head_stats": torch.empty((params.B, params.H, 2), dtype=torch.float32, device=dev),
        }
    ws = workspace(params, SSA_WS_FWD, dev) if ws is None else ws
    check(ssa_attn_fwd_dual_diag(params, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                                 _ptr(mask), _ptr(out["h_full"]), _ptr(out["h_sparse"]),
                                 _ptr(out["delta"]), _ptr(out["lse_full"]),
                                 _ptr(out["lse_sparse"]), _ptr(out["sqdiff"]), _ptr(out["sink"]),
                                 _ptr(out["head_stats"]), _ptr(ws), ws.numel(), _stream(dev)),
          "ssa_attn_fwd_dual_diag")
    return out


class DecodeCache:
    """Key/value cache of capacity params.T and the pooled keys of its completed
    blocks, for ssa_decode_step.  Tensors are allocated on ``device``."""

    def __init__(self, params, device, dtype):
        B, H, T, D = params.B, params.H, params.T, params.D
        self.params = params
        self.k = torch.zeros((B, H, T, D), dtype=dtype, device=device)
        self.v = torch.zeros_like(self.k)
        self.kbar = torch.zeros((B, H, T // params.block, D), dtype=torch.float64, device=device)
        self.pooled = 0  # completed blocks whose pooled keys are in kbar
        self.ws = workspace(params, SSA_WS_DECODE, device)

    def pool_upto(self, n_blocks):
        if n_blocks > self.pooled:
            check(ssa_decode_pool(self.params, self.pooled, n_blocks, _ptr(self.k), _ptr(self.kbar),
                                  _stream(self.k.device)), "ssa_decode_pool")
            self.pooled = n_blocks

    def step(self, t, q_t, idx=True):
        """Attend q_t [B,H,D] at position t (keys/values 0..t already written)."""
        p = self.params
        self.pool_upto(t // p.block)
        h = torch.empty((p.B, p.H, p.D), dtype=self.k.dtype, device=self.k.device)
        lse = torch.empty((p.B, p.H), dtype=torch.float32, device=self.k.device)
        ix = torch.empty((p.B, p.H, p.topk), dtype=torch.int32, device=self.k.device) if idx else None
        check(ssa_decode_step(p, t, _ptr(q_t), _ptr(self.k), _ptr(self.v), _ptr(self.kbar), _ptr(h),
                              _ptr(lse), _ptr(ix), _ptr(self.ws), self.ws.numel(),
                              _stream(self.k.device)), "ssa_decode_step")
        return {"h": h, "lse": lse, "idx": ix}


def align_loss(params, sqdiff, w_sparsity=1.0, w_commit=1.0, ws=None, out=None):
    """(w_s * L_sparsity, w_c * L_commit) as a float32 CUDA tensor of 2."""
    _need(sqdiff, "sqdiff")
    dev = sqdiff.device
    out = torch.empty(2, dtype=torch.float32, device=dev) if out is None else out
    ws = workspace(params, SSA_WS_LOSS, dev) if ws is None else ws
    check(ssa_align_loss(params, _ptr(sqdiff), w_sparsity, w_commit, _ptr(out), _ptr(ws),
                         ws.numel(), _stream(dev)), "ssa_align_loss")
    return out


def attn_bwd(params, q, k, v, mask, fwd, dh_full=None, dh_sparse=None, w_sparsity=0.0,
             w_commit=0.0, ws=None, out=None):
    """Gradients (dq, dk, dv) of both streams plus the alignment terms."""
    dev = q.device
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dv = out
    ws = workspace(params, SSA_WS_BWD, dev) if ws is None else ws
    check(ssa_attn_bwd(params, _ptr(q), _ptr(k), _ptr(v), None, None, _ptr(mask),
                       _ptr(fwd["h_full"]), _ptr(fwd["h_sparse"]), _ptr(fwd["lse_full"]),
                       _ptr(fwd["lse_sparse"]), _ptr(dh_full), _ptr(dh_sparse), w_sparsity,
                       w_commit, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                       _stream(dev)), "ssa_attn_bwd")
    return dq, dk, dv


def device_status(device=None):
    check(ssa_device_status(_stream(device)), "ssa_device_status")
