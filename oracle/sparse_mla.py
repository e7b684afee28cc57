"""CPU oracle for sparse MLA ("mistral_large4.attention" page, ``sparse_mla``).

TEST INFRASTRUCTURE ONLY (see the package docstring).  fp64 numpy; the
matrix products are numpy library calls.

What it computes, restated from the ``sparse_mla`` entry:

* ``q`` [local_tokens, heads, 576]: absorbed queries, the last 64
  coordinates rotary (zeros in NoPE layers);
* ``kv`` [global_tokens, 576]: one latent (512) + rotary (64) row per key,
  shared by all heads;
* ``indices`` [local_tokens, selected]: global kv rows each query attends
  to; -1 marks an invalid slot (the caller has already applied document and
  causal boundaries);
* ``value_weight`` [heads, value_dim, 512]: the KV-B value weight absorbed
  after the attention;
* ``scale``: the attention scale.

Reading (the page gives signatures, not the body): for token t and head h,
``s_j = scale * <q[t, h, :], kv[indices[t, j], :]>`` over the valid slots j
(each slot counts once, as given); ``p = softmax(s)``; the latent result
``l = sum_j p_j kv[indices[t, j], :512]`` (the latent part is the value);
``out[t, h, :] = value_weight[h] @ l``.  A row whose slots are all invalid
is zero ("empty query rows are zero").
"""
from __future__ import annotations

import numpy as np

LATENT = 512


def _f64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def sparse_mla(q, kv, indices, value_weight, scale: float, return_latent: bool = False):
    """fp64 out [T, H, value_dim] (and the normalised latent [T, H, 512] if
    ``return_latent``)."""
    q, kv, w = _f64(q), _f64(kv), _f64(value_weight)
    idx = np.asarray(indices.cpu() if hasattr(indices, "cpu") else indices, dtype=np.int64)
    T, H, _ = q.shape
    out = np.zeros((T, H, w.shape[1]))
    lat = np.zeros((T, H, LATENT))
    for t in range(T):
        sel = idx[t][idx[t] >= 0]
        if sel.size == 0:
            continue
        rows = kv[sel]                                  # [n, 576]
        s = scale * (q[t] @ rows.T)                     # [H, n]
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        lat[t] = p @ rows[:, :LATENT]                   # [H, 512]
        out[t] = np.einsum("hvc,hc->hv", w, lat[t])
    return (out, lat) if return_latent else out
