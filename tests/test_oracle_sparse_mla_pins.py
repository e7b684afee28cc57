"""Pins for the sparse-MLA oracle ("mistral_large4.attention" page,
sparse_mla): equality with PyTorch's fp64 scaled_dot_product_attention over
the whole kv with a mask built from the indices, closed forms (scale 0 is
the mean of the selected latent rows, one valid slot returns its projected
latent row, no valid slot returns zero), invariance to the slot order and,
in NoPE layers (zero rotary query), to the rotary part of kv; planted
mistakes in a copy of the oracle must each be caught."""
import importlib.util

import numpy as np
import pytest
import torch

from oracle import sparse_mla as SM

SRC = SM.__file__


def case(seed=0, T=6, Tg=9, H=3, K=5, vd=7):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, 576))
    kv = rng.standard_normal((Tg, 576))
    w = rng.standard_normal((H, vd, 512)) * 0.05
    idx = np.full((T, K), -1, dtype=np.int64)
    for t in range(T):
        n = int(rng.integers(1, K + 1))
        idx[t, :n] = rng.choice(Tg, size=n, replace=False)
        rng.shuffle(idx[t])
    return q, kv, idx, w


def _pins_fail(mod) -> list[str]:
    fails = []
    q, kv, idx, w = case()
    scale = 576 ** -0.5
    try:
        out, lat = mod.sparse_mla(q, kv, idx, w, scale, return_latent=True)
    except Exception:
        return ["raised"]
    # dense SDPA over all kv rows with the index mask
    for t in range(q.shape[0]):
        mask = np.zeros((1, kv.shape[0]), dtype=bool)
        mask[0, idx[t][idx[t] >= 0]] = True
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q[t])[:, None, :], torch.tensor(kv)[None].expand(q.shape[1], -1, -1),
            torch.tensor(kv[:, :512])[None].expand(q.shape[1], -1, -1),
            attn_mask=torch.tensor(mask)[None].expand(q.shape[1], -1, -1), scale=scale)[:, 0, :]
        if not np.allclose(lat[t], ref.numpy(), atol=1e-12):
            fails.append("sdpa")
            break
        if not np.allclose(out[t], np.einsum("hvc,hc->hv", w, ref.numpy()), atol=1e-12):
            fails.append("projection")
            break
    # scale 0: the mean of the selected latent rows
    o0, l0 = mod.sparse_mla(q, kv, idx, w, 0.0, return_latent=True)
    if not np.allclose(l0[0], kv[idx[0][idx[0] >= 0], :512].mean(0)[None], atol=1e-12):
        fails.append("scale0")
    # one valid slot returns the projected latent row; none returns zero
    idx1 = np.full_like(idx, -1)
    idx1[0, 2] = 4
    o1 = mod.sparse_mla(q, kv, idx1, w, scale)
    if not (np.allclose(o1[0], np.einsum("hvc,c->hv", w, kv[4, :512]), atol=1e-12)
            and np.abs(o1[1:]).max() == 0):
        fails.append("single")
    return fails


def test_oracle_passes_its_pins():
    assert _pins_fail(SM) == []


def test_slot_order_does_not_matter():
    q, kv, idx, w = case(1)
    perm = np.random.default_rng(2).permutation(idx.shape[1])
    assert np.allclose(SM.sparse_mla(q, kv, idx, w, 0.1), SM.sparse_mla(q, kv, idx[:, perm], w, 0.1),
                       atol=1e-13)


def test_nope_queries_ignore_the_rotary_keys():
    q, kv, idx, w = case(3)
    q[..., 512:] = 0.0
    kv2 = kv.copy()
    kv2[:, 512:] = np.random.default_rng(4).standard_normal((kv.shape[0], 64))
    assert np.allclose(SM.sparse_mla(q, kv, idx, w, 0.1), SM.sparse_mla(q, kv2, idx, w, 0.1), atol=1e-13)


MUTANTS = {
    "value_from_wrong_columns": ("lat[t] = p @ rows[:, :LATENT]", "lat[t] = p @ rows[:, 64:]"),
    "invalid_slots_kept": ("sel = idx[t][idx[t] >= 0]", "sel = idx[t]"),
    "scale_dropped": ("s = scale * (q[t] @ rows.T)", "s = (q[t] @ rows.T)"),
    "latent_not_normalised": ("p /= p.sum(axis=1, keepdims=True)", "p /= 1.0"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1
    path = tmp_path / f"sparse_mla_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"sparse_mla_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    assert _pins_fail(mod), f"mutant {name} survived every pin"
