"""CPU oracle for the Q/K prologue: parameter-free RMSNorm, then split-half RoPE.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Plain fp64 numpy.

What it computes (restated from the "muse_glimmer.model" page):

* ``MuseGlimmerScalelessRMSNorm`` -- "parameter-free RMSNorm used for
  embedding and Q/K normalization", ``eps`` default 1e-5; applied to each
  query / key head vector of ``D`` elements (the attention's Q/K RMSNorm):
  ``y = x / sqrt(mean(x ** 2) + eps)``.
* ``MuseGlimmerRotaryEmbedding`` -- "split-half rotary embedding matching the
  canonical HF implementation", ``theta`` default 500000, and
  ``apply_rotary_emb`` ("apply split-half RoPE to native BSHD or THD
  tensors").  Frequencies ``f_k = theta ** (-2k / D)`` for ``k < D/2``, angle
  ``a_k = position * f_k``; element ``k`` pairs with element ``k + D/2``:
  ``out_k = y_k cos a_k - y_{k+D/2} sin a_k`` and
  ``out_{k+D/2} = y_{k+D/2} cos a_k + y_k sin a_k``.
* Order: the normalisation comes first, then the rotation (MuseGlimmerAttention
  is "GQA with Q/K RMSNorm, optional RoPE").
* Positions in a THD pack: the position of token ``i`` of the document
  ``[s, e)`` is ``i - s`` (the pages leave the reset unstated; a packed
  document is its own sequence, as the per-token "local positions / document
  IDs" of the ``SequenceLayout`` describe).
"""
from __future__ import annotations

import numpy as np


def doc_positions(cu_seqlens) -> np.ndarray:
    """int64 [T]: position of every token inside its own document."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = int(cu[-1])
    pos = np.empty(T, dtype=np.int64)
    for d in range(len(cu) - 1):
        s, e = int(cu[d]), int(cu[d + 1])
        pos[s:e] = np.arange(e - s)
    return pos


def rms_norm(x: np.ndarray, eps: float) -> np.ndarray:
    """Scaleless RMSNorm over the last axis, fp64."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope_angles(positions: np.ndarray, D: int, theta: float) -> np.ndarray:
    """fp64 angles [T, D/2]: position * theta ** (-2k / D)."""
    k = np.arange(D // 2, dtype=np.float64)
    freq = np.power(float(theta), -2.0 * k / D)
    return np.asarray(positions, dtype=np.float64)[:, None] * freq[None, :]


def rope(y: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Split-half rotation of y [T, H, D] at the given positions, fp64."""
    T, H, D = y.shape
    a = rope_angles(positions, D, theta)[:, None, :]   # [T, 1, D/2]
    c, s = np.cos(a), np.sin(a)
    y1, y2 = y[..., : D // 2], y[..., D // 2:]
    return np.concatenate([y1 * c - y2 * s, y2 * c + y1 * s], axis=-1)


def qk_norm_rope(x, cu_seqlens, eps: float = 1e-5, theta: float = 500000.0, apply_rope: bool = True,
                 positions=None) -> np.ndarray:
    """The prologue for one of q [T, Hq, D] or k [T, Hkv, D] (bf16 bits as a
    torch tensor, or float): fp64 result [T, H, D].  ``positions`` (int [T])
    defaults to the per-document positions of ``cu_seqlens``."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().double().numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x, dtype=np.float64)
    y = rms_norm(x, eps)
    if not apply_rope:
        return y
    pos = doc_positions(cu_seqlens) if positions is None else np.asarray(positions, dtype=np.int64)
    return rope(y, pos, theta)
