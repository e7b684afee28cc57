"""CPU oracle for the packed-THD sliding-window GQA attention forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm may import this package.  It shares no
code with the CUDA path and the CUDA path never imports it.

Two independent formulations live here:

* :func:`attention` / :func:`attention_rows` -- the plain fp64 loop over
  documents, heads and queries in ``thd_attn_oracle.c`` (see that file's
  header for the definition and the page passages it restates);
* :func:`attention_bwd` / :func:`attention_bwd_q_rows` /
  :func:`attention_bwd_kv_rows` -- the fp64 gradient of that forward (dq, dk,
  dv, dsink), the plain derivative written out in the same C file, for the
  whole pack or for selected query rows (dq) or key rows (dk, dv);
  :func:`attention_dsink` -- the sink gradient alone from the forward's
  output and log-sum-exp;
* :mod:`oracle.prologue` -- the Q/K prologue (scaleless RMSNorm, then
  split-half RoPE at per-document positions) in plain fp64 numpy;
* :mod:`oracle.sparse_mla` -- sparse MLA over gathered latent KV with the
  absorbed value projection, fp64 numpy;
* :func:`dense_attention` -- a dense brute force for tiny packs: it builds the
  boolean ``[query_tokens, key_tokens]`` causal document mask the way
  ``SequenceLayout.allowed`` is described ("mistral_large4.attention" page),
  expands K/V to the query-head count like ``repeat_kv`` ("muse_glimmer.model"
  page), appends the sink as an extra logit column with a zero value row
  ("flint.magi" page, ``sink`` parameter) and runs one dense softmax.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "thd_attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

F64, BF16 = 0, 1


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the C oracle (gcc -O2 -fopenmp, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", src, "-o", out, "-lm"]
        subprocess.run(cmd, check=True)
    return out


def load(path: Optional[str] = None):
    """Load (building first if needed) the oracle library; returns the ctypes handle."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _bind(lib):
    vp, i32p, i64p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)
    dp, fp = ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_float)
    c_int, c_double = ctypes.c_int, ctypes.c_double
    lib.oracle_thd_attn.argtypes = [vp, vp, vp, c_int, i32p, c_int, c_int, c_int, c_int,
                                    c_int, c_double, fp, dp, dp]
    lib.oracle_thd_attn.restype = c_int
    lib.oracle_thd_attn_rows.argtypes = [vp, vp, vp, c_int, i32p, c_int, c_int, c_int, c_int,
                                         c_int, c_double, fp, i64p, ctypes.c_int64, dp, dp]
    lib.oracle_thd_attn_rows.restype = c_int
    lib.oracle_thd_attn_bwd.argtypes = [vp, vp, vp, vp, c_int, i32p, c_int, c_int, c_int, c_int,
                                        c_int, c_double, fp, dp, dp, dp, dp]
    lib.oracle_thd_attn_bwd.restype = c_int
    lib.oracle_thd_attn_bwd_q_rows.argtypes = [vp, vp, vp, vp, c_int, i32p, c_int, c_int, c_int,
                                               c_int, c_int, c_double, fp, i64p, ctypes.c_int64, dp]
    lib.oracle_thd_attn_bwd_q_rows.restype = c_int
    lib.oracle_thd_attn_bwd_kv_rows.argtypes = [vp, vp, vp, vp, c_int, i32p, c_int, c_int, c_int,
                                                c_int, c_int, c_double, fp, i64p, ctypes.c_int64,
                                                dp, dp]
    lib.oracle_thd_attn_bwd_kv_rows.restype = c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = c_int
    return lib


def _as_input(x) -> tuple[np.ndarray, int]:
    """numpy float64 -> (F64), or bf16 given as a torch tensor / uint16 bits -> (BF16)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            if x.dtype == torch.bfloat16:
                bits = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
                return np.ascontiguousarray(bits), BF16
            return np.ascontiguousarray(x.detach().cpu().double().numpy()), F64
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), BF16
    return np.ascontiguousarray(x, dtype=np.float64), F64


def _sinks(sinks) -> Optional[np.ndarray]:
    if sinks is None:
        return None
    try:
        import torch
        if isinstance(sinks, torch.Tensor):
            sinks = sinks.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(sinks, dtype=np.float32))


def _common(q, k, v, cu_seqlens):
    qa, qt = _as_input(q)
    ka, kt = _as_input(k)
    va, vt = _as_input(v)
    if not (qt == kt == vt):
        raise ValueError("q, k, v must share one dtype")
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    T, Hq, D = qa.shape
    Hkv = ka.shape[1]
    if ka.shape != (T, Hkv, D) or va.shape != (T, Hkv, D):
        raise ValueError("k/v shape mismatch")
    if int(cu[-1]) != T:
        raise ValueError("cu_seqlens[-1] must equal the token count")
    return qa, ka, va, qt, cu, T, Hq, Hkv, D


def attention(q, k, v, cu_seqlens, window: int, scale: float, sinks=None, lib=None):
    """Full fp64 forward.  Returns (out [T, Hq, D] float64, lse [T, Hq] float64)."""
    lib = lib or load()
    qa, ka, va, dt, cu, T, Hq, Hkv, D = _common(q, k, v, cu_seqlens)
    s = _sinks(sinks)
    out = np.zeros((T, Hq, D), dtype=np.float64)
    lse = np.zeros((T, Hq), dtype=np.float64)
    rc = lib.oracle_thd_attn(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, dt,
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(cu) - 1, Hq, Hkv, D,
        int(window), float(scale),
        s.ctypes.data_as(ctypes.POINTER(ctypes.c_float)) if s is not None else None,
        out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
        lse.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out, lse


def attention_rows(q, k, v, cu_seqlens, window: int, scale: float, rows, sinks=None, lib=None):
    """fp64 forward for selected (token, query_head) rows.

    ``rows`` is an int array [n, 2].  Returns (out [n, D], lse [n]).
    """
    lib = lib or load()
    qa, ka, va, dt, cu, T, Hq, Hkv, D = _common(q, k, v, cu_seqlens)
    s = _sinks(sinks)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    n = r.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = lib.oracle_thd_attn_rows(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, dt,
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(cu) - 1, Hq, Hkv, D,
        int(window), float(scale),
        s.ctypes.data_as(ctypes.POINTER(ctypes.c_float)) if s is not None else None,
        r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n,
        out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
        lse.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out, lse


def _dout(dout, dt):
    da, ddt = _as_input(dout)
    if ddt != dt:
        raise ValueError("dout must share the dtype of q, k, v")
    return da


def attention_bwd(q, k, v, dout, cu_seqlens, window: int, scale: float, sinks=None, lib=None):
    """Full fp64 backward (the derivative of :func:`attention`, see the C
    source).  Returns (dq [T, Hq, D], dk [T, Hkv, D], dv [T, Hkv, D],
    dsink [Hq] or None), all float64."""
    lib = lib or load()
    qa, ka, va, dt, cu, T, Hq, Hkv, D = _common(q, k, v, cu_seqlens)
    da = _dout(dout, dt)
    if da.shape != (T, Hq, D):
        raise ValueError("dout shape mismatch")
    s = _sinks(sinks)
    dq = np.zeros((T, Hq, D))
    dk = np.zeros((T, Hkv, D))
    dv = np.zeros((T, Hkv, D))
    dsink = np.zeros((Hq,)) if s is not None else None
    dptr = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if a is not None else None
    rc = lib.oracle_thd_attn_bwd(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data, dt,
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(cu) - 1, Hq, Hkv, D,
        int(window), float(scale),
        s.ctypes.data_as(ctypes.POINTER(ctypes.c_float)) if s is not None else None,
        dptr(dq), dptr(dk), dptr(dv), dptr(dsink))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return dq, dk, dv, dsink


def attention_bwd_q_rows(q, k, v, dout, cu_seqlens, window: int, scale: float, rows, sinks=None,
                         lib=None):
    """fp64 dq for selected (token, query_head) rows ``rows`` [n, 2]; returns [n, D]."""
    lib = lib or load()
    qa, ka, va, dt, cu, T, Hq, Hkv, D = _common(q, k, v, cu_seqlens)
    da = _dout(dout, dt)
    s = _sinks(sinks)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    out = np.zeros((r.shape[0], D))
    rc = lib.oracle_thd_attn_bwd_q_rows(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data, dt,
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(cu) - 1, Hq, Hkv, D,
        int(window), float(scale),
        s.ctypes.data_as(ctypes.POINTER(ctypes.c_float)) if s is not None else None,
        r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), r.shape[0],
        out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def attention_bwd_kv_rows(q, k, v, dout, cu_seqlens, window: int, scale: float, rows, sinks=None,
                          lib=None):
    """fp64 dk and dv for selected (key token, kv_head) rows ``rows`` [n, 2];
    returns (dk [n, D], dv [n, D])."""
    lib = lib or load()
    qa, ka, va, dt, cu, T, Hq, Hkv, D = _common(q, k, v, cu_seqlens)
    da = _dout(dout, dt)
    s = _sinks(sinks)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    dk = np.zeros((r.shape[0], D))
    dv = np.zeros((r.shape[0], D))
    rc = lib.oracle_thd_attn_bwd_kv_rows(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data, dt,
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(cu) - 1, Hq, Hkv, D,
        int(window), float(scale),
        s.ctypes.data_as(ctypes.POINTER(ctypes.c_float)) if s is not None else None,
        r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), r.shape[0],
        dk.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
        dv.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return dk, dv


def attention_dsink(q, k, v, dout, cu_seqlens, window: int, scale: float, sinks, lib=None):
    """fp64 sink gradient alone: dsink[h] = -sum_i exp(sink_h - lse[i,h]) *
    D[i,h] with D[i,h] = sum_c dO[i,h,c] out[i,h,c], where out and lse are the
    forward oracle's (:func:`attention`).  Returns [Hq]."""
    out, lse = attention(q, k, v, cu_seqlens, window, scale, sinks, lib=lib)
    da = _dout(dout, _as_input(q)[1])
    if da.dtype == np.uint16:
        da = _bits_to_f64(da)
    Di = np.einsum("ihc,ihc->ih", da, out)
    s = _sinks(sinks).astype(np.float64)
    return -(np.exp(s[None, :] - lse) * Di).sum(0)


def num_threads(lib=None) -> int:
    return int((lib or load()).oracle_num_threads())


# --------------------------------------------------------------------------
# Dense brute force (tiny packs only): a second, independent formulation.
# --------------------------------------------------------------------------

def dense_mask(cu_seqlens, window: int) -> np.ndarray:
    """bool [T, T]: key j visible to query i -- same document, j <= i, and
    (window == 0 or i - j < window).  Built from per-token document ids and
    positions, as the ``SequenceLayout.allowed`` causal document mask is."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = int(cu[-1])
    lengths = np.diff(cu)
    doc_id = np.repeat(np.arange(len(lengths)), lengths)
    pos = np.arange(T)
    same = doc_id[:, None] == doc_id[None, :]
    causal = pos[None, :] <= pos[:, None]
    mask = same & causal
    if window > 0:
        mask &= (pos[:, None] - pos[None, :]) < window
    return mask


def repeat_kv(x: np.ndarray, n_rep: int) -> np.ndarray:
    """[T, Hkv, D] -> [T, Hkv * n_rep, D], each kv head repeated n_rep times in place."""
    return np.repeat(x, n_rep, axis=1)


def dense_attention(q, k, v, cu_seqlens, window: int, scale: float, sinks=None):
    """Dense softmax over the masked score matrix.  Returns (out, lse) in fp64."""
    qa, ka, va, _, cu, T, Hq, Hkv, D = _common(q, k, v, cu_seqlens)
    if qa.dtype == np.uint16:
        qa, ka, va = (_bits_to_f64(a) for a in (qa, ka, va))
    kx = repeat_kv(ka, Hq // Hkv)
    vx = repeat_kv(va, Hq // Hkv)
    mask = dense_mask(cu, window)                          # [T, T]
    scores = scale * np.einsum("ihc,jhc->hij", qa, kx)     # [Hq, T, T]
    scores = np.where(mask[None], scores, -np.inf)
    s = _sinks(sinks)
    sink_col = (np.full((Hq, T, 1), -np.inf) if s is None
                else np.broadcast_to(s.astype(np.float64)[:, None, None], (Hq, T, 1)))
    logits = np.concatenate([scores, sink_col], axis=2)    # [Hq, T, T + 1]
    m = logits.max(axis=2, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(logits - m_safe)
    Z = w.sum(axis=2, keepdims=True)
    vals = np.concatenate([vx.transpose(1, 0, 2), np.zeros((Hq, 1, D))], axis=1)  # [Hq, T+1, D]
    with np.errstate(invalid="ignore", divide="ignore"):
        p = np.where(Z > 0, w / np.where(Z > 0, Z, 1.0), 0.0)
        out = np.einsum("hij,hjc->ihc", p, vals)
        lse = np.where(Z[..., 0] > 0, np.log(np.where(Z[..., 0] > 0, Z[..., 0], 1.0)) + m_safe[..., 0], -np.inf)
    return out, lse.T.copy()


def _bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def valid_pairs(cu_seqlens, window: int) -> int:
    """Number of (query, key) pairs with key visible to query, summed over documents."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    total = 0
    for L in np.diff(cu):
        L = int(L)
        if window <= 0 or window >= L:
            total += L * (L + 1) // 2
        else:
            total += window * (window + 1) // 2 + (L - window) * window
    return total
