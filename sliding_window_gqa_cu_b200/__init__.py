"""B200 (sm_100a) packed-THD sliding-window GQA attention forward.

Python binding over the C ABI in ``include/thd_attn.h`` (``libthdattn.so``,
built in-tree by :mod:`sliding_window_gqa_cu_b200.build`).  This module only
marshals arguments: every step of the computation runs in the CUDA library.
PyTorch supplies device memory and the current stream.

The operation is the local THD attention of ``MuseMagiPlan.attention`` /
``FlintMagiPlan.attention`` (NeMo AutoModel "muse_spark.magi_cp" and
"flint.magi" pages): q ``[T, Hq, D]``, k/v ``[T, Hkv, D]`` packed by
``cu_seqlens``, causal or sliding-window (the window counts the current
token), GQA by ``repeat_kv`` head mapping, optional per-head sink logits,
bf16 output ``[T, Hq, D]`` and fp32 log-sum-exp ``[T, Hq]``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

__all__ = ["thd_attn_fwd", "thd_attn_fwd_noalloc", "thd_attn_fwd_range", "thd_attn_merge",
           "thd_attn_fwd_host",
           "thd_attn_bwd", "thd_attn_bwd_workspace_bytes", "thd_qk_norm_rope",
           "thd_sparse_mla_fwd", "thd_sparse_mla_workspace_bytes", "thd_sparse_mla_get_error",
           "thd_attn_get_error", "thd_attn_noalloc_get_error", "thd_attn_selftest_stall", "thd_attn_plan", "thd_attn_plan_range",
           "thd_attn_plan_range_keys", "ThdAttnError", "library_path", "load_library", "STATUS"]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libthdattn.so"
_lib = None

STATUS = {0: "THD_OK", -1: "THD_ERR_INVALID_ARG", -2: "THD_ERR_UNSUPPORTED", -3: "THD_ERR_CUDA",
          -4: "THD_ERR_TIMEOUT", -5: "THD_ERR_NO_MEMORY", -6: "THD_ERR_TOO_LARGE",
          -7: "THD_ERR_STALE_SCRATCH", -8: "THD_ERR_BAD_ITEM"}

WORK_ITEM_FIELDS = ("q0", "q1", "doc_start", "head0", "kv_start", "n_kv", "n_heads", "block_n")


class ThdAttnError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        msg = f"{STATUS.get(code, code)}: {_status_string(code)}"
        super().__init__(f"{what}: {msg}" if what else msg)


class _WorkItem(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in WORK_ITEM_FIELDS]


def library_path() -> str:
    return os.path.join(_PKG, _LIB_NAME)


def load_library():
    """Load ``libthdattn.so``; raises if it has not been built (no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m sliding_window_gqa_cu_b200.build` "
            "(there is no CPU fallback)")
    _lib = bind(ctypes.CDLL(path))
    return _lib


def bind(lib):
    """Declare the argument and result types of every entry point on a loaded
    copy of the library (``load_library`` does this for the in-tree build)."""
    vp, i32p, c_int = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_int
    lib.thd_attn_fwd.argtypes = [vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int,
                                 ctypes.c_float, vp, vp, vp, vp]
    lib.thd_attn_fwd.restype = c_int
    lib.thd_attn_get_error.argtypes = [vp]
    lib.thd_attn_get_error.restype = c_int
    lib.thd_attn_status_string.argtypes = [c_int]
    lib.thd_attn_status_string.restype = ctypes.c_char_p
    lib.thd_attn_plan.argtypes = [i32p, c_int, c_int, c_int, c_int, c_int,
                                  ctypes.POINTER(_WorkItem), ctypes.c_int64,
                                  ctypes.POINTER(ctypes.c_int64)]
    lib.thd_attn_plan.restype = c_int
    lib.thd_attn_fwd_noalloc.argtypes = [vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int,
                                         ctypes.c_float, vp, vp, vp, vp, vp]
    lib.thd_attn_fwd_noalloc.restype = c_int
    lib.thd_attn_noalloc_get_error.argtypes = [vp]
    lib.thd_attn_noalloc_get_error.restype = c_int
    lib.thd_attn_bwd_workspace_bytes.argtypes = [ctypes.c_int64, c_int]
    lib.thd_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.thd_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int,
                                 ctypes.c_float, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.thd_attn_bwd.restype = c_int
    lib.thd_attn_fwd_range.argtypes = [vp, vp, vp, i32p, c_int, ctypes.c_int64, ctypes.c_int64,
                                       c_int, c_int, c_int, c_int, ctypes.c_float, vp, vp, vp, vp]
    lib.thd_attn_fwd_range.restype = c_int
    lib.thd_attn_fwd_range_keys.argtypes = [vp, vp, vp, i32p, c_int, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_int64, c_int, c_int, c_int, c_int, ctypes.c_float,
                                            vp, vp, vp, vp]
    lib.thd_attn_fwd_range_keys.restype = c_int
    lib.thd_attn_merge.argtypes = [vp, vp, vp, vp, ctypes.c_int64, c_int, c_int, vp, vp, vp]
    lib.thd_attn_merge.restype = c_int
    lib.thd_attn_fwd_host.argtypes = [vp, vp, vp, i32p, c_int, c_int, c_int, c_int, c_int,
                                      ctypes.c_float, vp, vp, vp, vp, vp, vp, vp, vp, vp, c_int, vp]
    lib.thd_attn_fwd_host.restype = c_int
    lib.thd_attn_selftest_stall.argtypes = [ctypes.POINTER(ctypes.c_int64)]
    lib.thd_attn_selftest_stall.restype = c_int
    lib.thd_attn_plan_range.argtypes = [i32p, c_int, ctypes.c_int64, ctypes.c_int64, c_int, c_int,
                                        c_int, c_int, vp, ctypes.c_int64,
                                        ctypes.POINTER(ctypes.c_int64)]
    lib.thd_attn_plan_range.restype = c_int
    lib.thd_attn_plan_range_keys.argtypes = [i32p, c_int, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_int64, c_int, c_int, c_int, c_int, vp,
                                             ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]
    lib.thd_attn_plan_range_keys.restype = c_int
    lib.thd_sparse_mla_workspace_bytes.argtypes = [ctypes.c_int64, c_int, c_int]
    lib.thd_sparse_mla_workspace_bytes.restype = ctypes.c_size_t
    lib.thd_sparse_mla_fwd.argtypes = [vp, vp, vp, vp, ctypes.c_int64, ctypes.c_int64, c_int, c_int,
                                       c_int, ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
    lib.thd_sparse_mla_fwd.restype = c_int
    lib.thd_sparse_mla_get_error.argtypes = [vp]
    lib.thd_sparse_mla_get_error.restype = c_int
    lib.thd_qk_norm_rope.argtypes = [vp, vp, i32p, c_int, vp, c_int, c_int, c_int, ctypes.c_float,
                                     ctypes.c_float, c_int, vp]
    lib.thd_qk_norm_rope.restype = c_int
    lib.thd_attn_abi_version.argtypes = []
    lib.thd_attn_abi_version.restype = c_int
    return lib


def _status_string(code: int) -> str:
    try:
        return load_library().thd_attn_status_string(int(code)).decode()
    except Exception:  # library missing while formatting an error
        return "?"


def _cu_array(cu_seqlens) -> np.ndarray:
    try:
        import torch
        if isinstance(cu_seqlens, torch.Tensor):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    if cu.ndim != 1 or cu.size < 1:
        raise ValueError("cu_seqlens must be a 1-D array of documents + 1 boundaries")
    return cu


def thd_attn_plan(cu_seqlens, Hq: int, Hkv: int, D: int, window: int) -> np.ndarray:
    """The tile schedule (structured numpy array, one record per work item)."""
    lib = load_library()
    cu = _cu_array(cu_seqlens)
    n = ctypes.c_int64(0)
    cup = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    rc = lib.thd_attn_plan(cup, cu.size - 1, Hq, Hkv, D, window, None, 0, ctypes.byref(n))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_plan")
    buf = (_WorkItem * max(1, n.value))()
    rc = lib.thd_attn_plan(cup, cu.size - 1, Hq, Hkv, D, window, buf, n.value, ctypes.byref(n))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_plan")
    dt = np.dtype([(f, np.int32) for f in WORK_ITEM_FIELDS])
    return np.frombuffer(bytes(buf), dtype=dt, count=n.value).copy()


def thd_attn_fwd(q, k, v, cu_seqlens, window: int = 0, scale: Optional[float] = None,
                 sinks=None, out=None, lse=None, return_lse: bool = True, stream=None):
    """Packed-THD attention forward on the current CUDA device.

    q: bf16 CUDA tensor [T, Hq, D]; k, v: bf16 CUDA [T, Hkv, D] (contiguous);
    cu_seqlens: host int32 boundaries [documents + 1] (numpy, list or CPU tensor);
    window: 0 = full causal, W > 0 = W keys including the query's own token;
    scale: score scale (default D ** -0.5); sinks: fp32 CUDA [Hq] or None.
    Returns ``(out, lse)`` (``lse`` is None when ``return_lse`` is False).
    """
    import torch

    lib = load_library()
    if q.dim() != 3 or k.dim() != 3 or v.dim() != 3:
        raise ValueError("q, k, v must be [tokens, heads, head_dim]")
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if k.shape != (T, Hkv, D) or v.shape != (T, Hkv, D):
        raise ValueError("k and v must be [tokens, kv_heads, head_dim] like q")
    cu = _cu_array(cu_seqlens)
    if int(cu[-1]) != T:
        raise ValueError(f"cu_seqlens[-1]={int(cu[-1])} does not match {T} tokens")
    if scale is None:
        scale = D ** -0.5
    if sinks is not None:
        if sinks.dtype != torch.float32 or not sinks.is_cuda or sinks.numel() != Hq:
            raise ValueError("sinks must be an fp32 CUDA tensor of Hq values")
        sinks = sinks.contiguous()
    if out is None:
        out = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        rc = lib.thd_attn_fwd(
            q.data_ptr(), k.data_ptr(), v.data_ptr(),
            cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1,
            Hq, Hkv, D, int(window), float(scale),
            sinks.data_ptr() if sinks is not None else None,
            out.data_ptr(), lse.data_ptr() if lse is not None else None,
            ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_fwd")
    return out, lse


def thd_attn_bwd(q, k, v, out, lse, dout, cu_seqlens, window: int = 0,
                 scale: Optional[float] = None, sinks=None, dq=None, dk=None, dv=None,
                 workspace=None, stream=None):
    """Backward of :func:`thd_attn_fwd` (head dim 64, 128 or 256).

    q, k, v, cu_seqlens, window, scale, sinks: as passed to the forward;
    out, lse: the forward's results; dout: bf16 CUDA [T, Hq, D] gradient of the
    loss w.r.t. out.  Returns ``(dq, dk, dv, dsinks)`` (``dsinks`` is None
    without sinks).  ``workspace`` (optional) is a CUDA byte tensor of at least
    ``thd_attn_bwd_workspace_bytes(T, Hq)`` bytes.
    """
    import torch

    lib = load_library()
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if out.shape != q.shape or dout.shape != q.shape:
        raise ValueError("out and dout must be [tokens, heads, head_dim] like q")
    if k.shape != (T, Hkv, D) or v.shape != (T, Hkv, D):
        raise ValueError("k and v must be [tokens, kv_heads, head_dim] like q")
    if lse is None or lse.dtype != torch.float32 or not lse.is_contiguous() or lse.shape != (T, Hq):
        raise ValueError("lse must be the forward's contiguous fp32 [tokens, heads] log-sum-exp")
    cu = _cu_array(cu_seqlens)
    if int(cu[-1]) != T:
        raise ValueError(f"cu_seqlens[-1]={int(cu[-1])} does not match {T} tokens")
    if scale is None:
        scale = D ** -0.5
    dsinks = None
    if sinks is not None:
        if sinks.dtype != torch.float32 or not sinks.is_cuda or sinks.numel() != Hq:
            raise ValueError("sinks must be an fp32 CUDA tensor of Hq values")
        sinks = sinks.contiguous()
        dsinks = torch.empty((Hq,), dtype=torch.float32, device=q.device)
    dq = dq if dq is not None else torch.empty_like(q)
    dk = dk if dk is not None else torch.empty_like(k)
    dv = dv if dv is not None else torch.empty_like(v)
    need = int(lib.thd_attn_bwd_workspace_bytes(T, Hq))
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        rc = lib.thd_attn_bwd(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
            dout.data_ptr(), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1,
            Hq, Hkv, D, int(window), float(scale),
            sinks.data_ptr() if sinks is not None else None,
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
            dsinks.data_ptr() if dsinks is not None else None,
            workspace.data_ptr(), workspace.numel(), ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_bwd")
    return dq, dk, dv, dsinks


def thd_attn_bwd_workspace_bytes(T: int, Hq: int) -> int:
    """Workspace bytes :func:`thd_attn_bwd` needs for T tokens and Hq query heads."""
    return int(load_library().thd_attn_bwd_workspace_bytes(int(T), int(Hq)))


def thd_qk_norm_rope(q, k, cu_seqlens, eps: float = 1e-5, theta: float = 500000.0,
                     apply_rope: bool = True, positions=None, stream=None):
    """In-place Q/K prologue: scaleless RMSNorm of every head vector, then
    split-half RoPE at per-document positions (or ``positions``, an int32 CUDA
    tensor [T]).  q: bf16 CUDA [T, Hq, D]; k: bf16 CUDA [T, Hkv, D] or None.
    Returns (q, k)."""
    import torch

    lib = load_library()
    T, Hq, D = q.shape
    for name, t in (("q", q), ("k", k)):
        if t is None:
            continue
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [tokens, heads, head_dim]")
        if t.shape[0] != T or t.shape[2] != D:
            raise ValueError("q and k must share tokens and head_dim")
    Hkv = k.shape[1] if k is not None else 0
    cu = _cu_array(cu_seqlens)
    if int(cu[-1]) != T:
        raise ValueError(f"cu_seqlens[-1]={int(cu[-1])} does not match {T} tokens")
    if positions is not None:
        if positions.dtype != torch.int32 or not positions.is_cuda or positions.numel() != T:
            raise ValueError("positions must be an int32 CUDA tensor [tokens]")
        positions = positions.contiguous()
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        rc = lib.thd_qk_norm_rope(
            q.data_ptr(), k.data_ptr() if k is not None else None,
            cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1,
            positions.data_ptr() if positions is not None else None,
            Hq, Hkv, D, float(eps), float(theta), int(bool(apply_rope)),
            ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise ThdAttnError(rc, "thd_qk_norm_rope")
    return q, k


def thd_attn_fwd_range(q, k, v, cu_seqlens, q_begin: int, q_end: int, window: int = 0,
                       scale: Optional[float] = None, sinks=None, out=None, lse=None,
                       return_lse: bool = True, stream=None, k_end: Optional[int] = None):
    """Forward of the query rows [q_begin, q_end) of the pack against K/V of
    the whole pack (the local step of a context-parallel forward).

    q: bf16 CUDA [q_end - q_begin, Hq, D]; k, v: bf16 CUDA [T, Hkv, D];
    cu_seqlens: host boundaries of the whole pack.  ``k_end`` (default T)
    restricts the keys to j < k_end (``thd_attn_fwd_range_keys``; only those
    rows of k and v are read).  Returns ``(out, lse)`` for those rows.
    """
    import torch

    lib = load_library()
    Tq, Hq, D = q.shape
    T, Hkv = k.shape[0], k.shape[1]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if v.shape != k.shape or k.shape[2] != D:
        raise ValueError("k and v must be [tokens, kv_heads, head_dim] with q's head_dim")
    cu = _cu_array(cu_seqlens)
    if int(cu[-1]) != T:
        raise ValueError(f"cu_seqlens[-1]={int(cu[-1])} does not match {T} key tokens")
    if not (0 <= q_begin <= q_end <= T) or q_end - q_begin != Tq:
        raise ValueError("q must hold exactly the rows [q_begin, q_end) of the pack")
    if k_end is None:
        k_end = T
    if not (0 <= k_end <= T):
        raise ValueError(f"k_end={k_end} outside [0, {T}]")
    if scale is None:
        scale = D ** -0.5
    if sinks is not None:
        if sinks.dtype != torch.float32 or not sinks.is_cuda or sinks.numel() != Hq:
            raise ValueError("sinks must be an fp32 CUDA tensor of Hq values")
        sinks = sinks.contiguous()
    if out is None:
        out = torch.empty((Tq, Hq, D), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((Tq, Hq), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        rc = lib.thd_attn_fwd_range_keys(
            q.data_ptr(), k.data_ptr(), v.data_ptr(),
            cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1,
            int(q_begin), int(q_end), int(k_end), Hq, Hkv, D, int(window), float(scale),
            sinks.data_ptr() if sinks is not None else None,
            out.data_ptr(), lse.data_ptr() if lse is not None else None,
            ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_fwd_range")
    return out, lse


def thd_attn_merge(out_a, lse_a, out_b, lse_b, out=None, lse=None, stream=None):
    """Merge two partial results of the same rows over disjoint key sets
    (log-sum-exp combination, ``thd_attn_merge``).  out_*: bf16 CUDA
    [rows, Hq, D]; lse_*: fp32 CUDA [rows, Hq].  ``out`` / ``lse`` default to
    new tensors and may be ``out_a`` / ``lse_a``.  Returns ``(out, lse)``."""
    import torch

    lib = load_library()
    rows, Hq, D = out_a.shape
    for name, t, dt, shape in (("out_a", out_a, torch.bfloat16, (rows, Hq, D)),
                               ("out_b", out_b, torch.bfloat16, (rows, Hq, D)),
                               ("lse_a", lse_a, torch.float32, (rows, Hq)),
                               ("lse_b", lse_b, torch.float32, (rows, Hq))):
        if t.dtype != dt or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape:
            raise ValueError(f"{name} must be a contiguous {dt} CUDA tensor of shape {shape}")
    if out is None:
        out = torch.empty_like(out_a)
    if lse is None:
        lse = torch.empty_like(lse_a)
    if stream is None:
        stream = torch.cuda.current_stream(out_a.device)
    with torch.cuda.device(out_a.device):
        rc = lib.thd_attn_merge(out_a.data_ptr(), lse_a.data_ptr(), out_b.data_ptr(), lse_b.data_ptr(),
                                rows, Hq, D, out.data_ptr(), lse.data_ptr(),
                                ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_merge")
    return out, lse


def thd_attn_fwd_host(q_host, k_host, v_host, cu_seqlens, window: int = 0,
                      scale: Optional[float] = None, sinks_host=None, out_host=None,
                      lse_host=None, device_buffers=None, n_chunks: int = 8, stream=None):
    """The forward from host tensors with the copies overlapped with the
    attention (token ranges pipelined over two copy streams and ``stream``).

    q_host, k_host, v_host: bf16 CPU tensors [T, Hq, D] / [T, Hkv, D]
    (page-locked for the copies to overlap); sinks_host: fp32 CPU [Hq] or
    None.  ``device_buffers`` is an optional dict of CUDA staging tensors
    ``q, k, v, out, lse`` (and ``sinks``) of the same shapes, reused across
    calls; missing ones are allocated on the current device.  Returns
    ``(out_host, lse_host)``; they are valid once ``stream`` (default: the
    current stream) has been synchronised.
    """
    import torch

    lib = load_library()
    T, Hq, D = q_host.shape
    Hkv = k_host.shape[1]
    for name, t in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host)):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor")
    if v_host.shape != k_host.shape or k_host.shape[0] != T or k_host.shape[2] != D:
        raise ValueError("k and v must be [tokens, kv_heads, head_dim] with q's tokens and head_dim")
    cu = _cu_array(cu_seqlens)
    if int(cu[-1]) != T:
        raise ValueError(f"cu_seqlens[-1]={int(cu[-1])} does not match {T} tokens")
    if scale is None:
        scale = D ** -0.5
    dev = torch.device("cuda", torch.cuda.current_device())
    bufs = dict(device_buffers or {})
    shapes = {"q": ((T, Hq, D), torch.bfloat16), "k": ((T, Hkv, D), torch.bfloat16),
              "v": ((T, Hkv, D), torch.bfloat16), "out": ((T, Hq, D), torch.bfloat16),
              "lse": ((T, Hq), torch.float32)}
    if sinks_host is not None:
        if sinks_host.dtype != torch.float32 or sinks_host.is_cuda or sinks_host.numel() != Hq:
            raise ValueError("sinks_host must be an fp32 CPU tensor of Hq values")
        sinks_host = sinks_host.contiguous()
        shapes["sinks"] = ((Hq,), torch.float32)
    for name, (shape, dtype) in shapes.items():
        if name not in bufs:
            bufs[name] = torch.empty(shape, dtype=dtype, device=dev)
        t = bufs[name]
        if tuple(t.shape) != shape or t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"device buffer {name} must be a contiguous CUDA {dtype} tensor {shape}")
    if out_host is None:
        out_host = torch.empty((T, Hq, D), dtype=torch.bfloat16, pin_memory=True)
    if lse_host is None:
        lse_host = torch.empty((T, Hq), dtype=torch.float32, pin_memory=True)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    rc = lib.thd_attn_fwd_host(
        q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1, Hq, Hkv, D, int(window),
        float(scale), sinks_host.data_ptr() if sinks_host is not None else None,
        out_host.data_ptr(), lse_host.data_ptr(), bufs["q"].data_ptr(), bufs["k"].data_ptr(),
        bufs["v"].data_ptr(), bufs["sinks"].data_ptr() if sinks_host is not None else None,
        bufs["out"].data_ptr(), bufs["lse"].data_ptr(), int(n_chunks),
        ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_fwd_host")
    return out_host, lse_host


def thd_attn_plan_range_keys(cu_seqlens, q_begin: int, q_end: int, k_end: int, Hq: int, Hkv: int,
                             D: int, window: int) -> np.ndarray:
    """Host-only: the work list of :func:`thd_attn_fwd_range` with keys below
    ``k_end`` only (structured array)."""
    lib = load_library()
    cu = _cu_array(cu_seqlens)
    n = ctypes.c_int64(0)
    args = (cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1, int(q_begin), int(q_end),
            int(k_end), Hq, Hkv, D, int(window))
    rc = lib.thd_attn_plan_range_keys(*args, None, 0, ctypes.byref(n))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_plan_range_keys")
    dt = np.dtype([(f, np.int32) for f in WORK_ITEM_FIELDS])
    items = np.zeros(max(1, n.value), dtype=dt)
    rc = lib.thd_attn_plan_range_keys(*args, items.ctypes.data, n.value, ctypes.byref(n))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_plan_range_keys")
    return items[:n.value].copy()


def thd_attn_plan_range(cu_seqlens, q_begin: int, q_end: int, Hq: int, Hkv: int, D: int,
                        window: int) -> np.ndarray:
    """Host-only: the work list of :func:`thd_attn_fwd_range` (structured array)."""
    lib = load_library()
    cu = _cu_array(cu_seqlens)
    n = ctypes.c_int64(0)
    rc = lib.thd_attn_plan_range(cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1,
                                 int(q_begin), int(q_end), Hq, Hkv, D, int(window), None, 0,
                                 ctypes.byref(n))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_plan_range")
    dt = np.dtype([(f, np.int32) for f in WORK_ITEM_FIELDS])
    items = np.zeros(max(1, n.value), dtype=dt)
    rc = lib.thd_attn_plan_range(cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1,
                                 int(q_begin), int(q_end), Hq, Hkv, D, int(window),
                                 items.ctypes.data, n.value, ctypes.byref(n))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_plan_range")
    return items[:n.value].copy()


def thd_sparse_mla_fwd(q, kv, indices, value_weight, scale: float, out=None, workspace=None,
                       stream=None):
    """Sparse MLA forward.  q: bf16 CUDA [T, H, 576]; kv: bf16 CUDA [Tg, 576];
    indices: int32 CUDA [T, K] (-1 = invalid slot); value_weight: bf16 CUDA
    [H, value_dim, 512].  Returns out: bf16 [T, H, value_dim]."""
    import torch

    lib = load_library()
    T, H, dq = q.shape
    Tg = kv.shape[0]
    K = indices.shape[1] if indices.dim() == 2 else 0
    vd = value_weight.shape[1]
    for name, t, dt in (("q", q, torch.bfloat16), ("kv", kv, torch.bfloat16),
                        ("indices", indices, torch.int32), ("value_weight", value_weight, torch.bfloat16)):
        if t.dtype != dt or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {dt} CUDA tensor")
    if dq != 576 or kv.shape[1] != 576 or indices.shape[0] != T or value_weight.shape != (H, vd, 512):
        raise ValueError("shapes: q [T, H, 576], kv [Tg, 576], indices [T, K], value_weight [H, vd, 512]")
    if out is None:
        out = torch.empty((T, H, vd), dtype=torch.bfloat16, device=q.device)
    need = int(lib.thd_sparse_mla_workspace_bytes(T, H, K))
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        rc = lib.thd_sparse_mla_fwd(q.data_ptr(), kv.data_ptr(), indices.data_ptr(),
                                    value_weight.data_ptr(), T, Tg, H, K, vd, float(scale),
                                    out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                    ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise ThdAttnError(rc, "thd_sparse_mla_fwd")
    return out


def thd_sparse_mla_workspace_bytes(T: int, H: int, K: int) -> int:
    """Workspace bytes :func:`thd_sparse_mla_fwd` needs (the bf16 latent
    [T, H, 512], compacted indices [T, K], counts [T])."""
    return int(load_library().thd_sparse_mla_workspace_bytes(int(T), int(H), int(K)))


def thd_sparse_mla_get_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the sparse-MLA status word."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(load_library().thd_sparse_mla_get_error(ctypes.c_void_p(stream.cuda_stream)))


def thd_attn_selftest_stall() -> tuple:
    """Runs the stall-detector self-test (about 2.5 s; see thd_attn.h) and
    returns how long its two blocks waited, in ns.  Afterwards
    :func:`thd_attn_get_error` returns the timeout status once."""
    lib = load_library()
    w = (ctypes.c_int64 * 2)()
    rc = lib.thd_attn_selftest_stall(w)
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_selftest_stall")
    return int(w[0]), int(w[1])


def thd_attn_get_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(load_library().thd_attn_get_error(ctypes.c_void_p(stream.cuda_stream)))


def thd_attn_fwd_noalloc(q, k, v, cu_seqlens, out, lse=None, window: int = 0,
                         scale: Optional[float] = None, sinks=None, device_status=None,
                         stream=None):
    """Allocation-free forward for callers that may not allocate device memory.

    Same computation as :func:`thd_attn_fwd`, but the caller supplies every
    buffer (``out`` and, if wanted, ``lse``; optionally a device int32
    ``device_status`` word) and the library uses only a fixed scratch array
    compiled into its device image.  This wrapper allocates nothing either.
    The first call on a device does a one-time synchronous set-up; calls that
    overlap on the GPU share the scratch and must be serialised.  Without
    ``device_status``, errors are read with :func:`thd_attn_noalloc_get_error`.
    """
    import torch

    lib = load_library()
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    cu = _cu_array(cu_seqlens)
    if scale is None:
        scale = D ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        rc = lib.thd_attn_fwd_noalloc(
            q.data_ptr(), k.data_ptr(), v.data_ptr(),
            cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1,
            Hq, Hkv, D, int(window), float(scale),
            sinks.data_ptr() if sinks is not None else None,
            out.data_ptr(), lse.data_ptr() if lse is not None else None,
            device_status.data_ptr() if device_status is not None else None,
            ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise ThdAttnError(rc, "thd_attn_fwd_noalloc")
    return out, lse


def thd_attn_noalloc_get_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the status word of the
    allocation-free entry point's scratch."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(load_library().thd_attn_noalloc_get_error(ctypes.c_void_p(stream.cuda_stream)))
