"""Pins for the Q/K prologue oracle (scaleless RMSNorm, then split-half RoPE,
"muse_glimmer.model" page: MuseGlimmerScalelessRMSNorm,
MuseGlimmerRotaryEmbedding, apply_rotary_emb), checked against closed forms,
the textbook complex-number form of the rotation and its defining property
(scores depend only on the position difference); planted mistakes in a copy
of the oracle must each be caught."""
import importlib.util
import math
import os

import numpy as np
import pytest

from oracle import prologue as P

SRC = P.__file__


def _rand(seed, shape):
    return np.random.default_rng(seed).standard_normal(shape)


def _pins_fail(mod) -> list[str]:
    fails = []
    rng = np.random.default_rng(0)
    D, eps, theta = 16, 1e-5, 500000.0
    x = rng.standard_normal((7, 3, D)) * 3.0
    cu = [0, 3, 7]
    # RMS closed form: mean(y^2) = ms / (ms + eps)
    y = mod.rms_norm(x, eps)
    ms = np.mean(x * x, axis=-1)
    if not np.allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-13):
        fails.append("rms")
    # per-document positions
    if not np.array_equal(mod.doc_positions(cu), [0, 1, 2, 0, 1, 2, 3]):
        fails.append("positions")
    out = mod.qk_norm_rope(x, cu, eps, theta)
    # position 0 (each document's first token) is the identity rotation
    if not (np.allclose(out[0], y[0], atol=1e-14) and np.allclose(out[3], y[3], atol=1e-14)):
        fails.append("pos0")
    # textbook complex form: (y_k + i y_{k+D/2}) * exp(i * pos * theta^(-2k/D))
    pos = np.array([0, 1, 2, 0, 1, 2, 3], dtype=np.float64)
    k = np.arange(D // 2)
    ang = pos[:, None, None] * theta ** (-2.0 * k / D)[None, None, :]
    z = (y[..., : D // 2] + 1j * y[..., D // 2:]) * np.exp(1j * ang)
    if not np.allclose(out, np.concatenate([z.real, z.imag], -1), atol=1e-12):
        fails.append("complex")
    # scores depend only on the position difference
    q, kk = rng.standard_normal((1, 1, D)), rng.standard_normal((1, 1, D))
    for m, n, d in ((5, 2, 7), (100, 100, 1000), (0, 9, 40)):
        a = (mod.rope(q, np.array([m]), theta) * mod.rope(kk, np.array([n]), theta)).sum()
        b = (mod.rope(q, np.array([m + d]), theta) * mod.rope(kk, np.array([n + d]), theta)).sum()
        if abs(a - b) > 1e-9:
            fails.append("relative")
            break
    # the angles of frequency 0 are the positions; the middle frequency is theta^(-1/2)
    a = mod.rope_angles(np.array([1]), D, theta)
    if not (a[0, 0] == 1.0 and math.isclose(a[0, D // 4], theta ** -0.5, rel_tol=1e-14)):
        fails.append("freq")
    return fails


def test_oracle_passes_its_pins():
    assert _pins_fail(P) == []


def test_a_document_alone_equals_the_document_in_the_pack():
    x = _rand(1, (30, 2, 32))
    cu = [0, 11, 30]
    full = P.qk_norm_rope(x, cu)
    alone = P.qk_norm_rope(x[11:], [0, 19])
    assert np.allclose(full[11:], alone, atol=1e-14)


def test_without_rope_it_is_the_norm_only():
    x = _rand(2, (9, 4, 64))
    assert np.allclose(P.qk_norm_rope(x, [0, 9], apply_rope=False), P.rms_norm(x, 1e-5))


def test_rotation_preserves_the_split_half_pair_norms():
    x = _rand(3, (12, 2, 64))
    y = P.rms_norm(x, 1e-5)
    out = P.qk_norm_rope(x, [0, 12])
    pair = lambda a: a[..., :32] ** 2 + a[..., 32:] ** 2
    assert np.allclose(pair(out), pair(y), atol=1e-13)


MUTANTS = {
    "second_half_sign": ("y2 * c + y1 * s", "y2 * c - y1 * s"),
    "interleaved_pairs": ("y1, y2 = y[..., : D // 2], y[..., D // 2:]", "y1, y2 = y[..., 0::2], y[..., 1::2]"),
    "global_positions": ("pos[s:e] = np.arange(e - s)", "pos[s:e] = np.arange(s, e)"),
    "eps_outside_sqrt": ("np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)",
                         "(np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps)"),
    "frequency_exponent": ("np.power(float(theta), -2.0 * k / D)", "np.power(float(theta), -1.0 * k / D)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    path = tmp_path / f"prologue_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"prologue_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    assert _pins_fail(mod), f"mutant {name} survived every pin"
