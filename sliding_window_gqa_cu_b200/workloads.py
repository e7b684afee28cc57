"""Seeded synthetic workloads for the packed-THD attention forward.

This module only draws numbers: document lengths and the bf16 query/key/value
tensors (plus fp32 sink logits) of the five pack shapes the benchmark and the
parity tests use.  It holds none of the attention arithmetic, so both the CUDA
path and the CPU oracle can be fed from it without sharing any computation.

Shapes follow the packed THD convention of the Muse/Flint Magi plans
(``MuseMagiPlan.attention`` / ``FlintMagiPlan.attention`` parameter docs):
query ``[tokens, query_heads, head_dim]``, key/value ``[tokens, kv_heads,
head_dim]``, documents delimited by an int32 ``cu_seqlens`` of
``documents + 1`` boundaries (``_build_magi_plan``, ``cu_seqlens`` parameter),
and per-query-head fp32 sink logits (``FlintMagiPlan.attention``, ``sink``).

Recipe (stated once, used everywhere):

* document lengths: ``rng = numpy.random.default_rng(seed)``; repeat
  ``L = round(exp(rng.uniform(ln lo, ln hi)))``, ``L = min(L, T - used)``
  until the pack holds ``T`` tokens (the last document is truncated);
* tensors: ``rng2 = numpy.random.default_rng([seed, index])`` draws q, then k,
  then v as float32 ``standard_normal * std`` and rounds them to bf16
  (round-to-nearest-even, via ``torch.Tensor.to(torch.bfloat16)``); sink
  logits are float32 N(0, 1) ``[Hq]`` drawn after v.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class PackConfig:
    """One synthetic pack shape."""

    name: str
    index: int
    T: int
    Hq: int
    Hkv: int
    D: int
    window: int
    scale: float
    sinks: bool
    std: float = 1.0
    doc_len_range: Optional[tuple[int, int]] = None  # log-uniform [lo, hi]
    fixed_cu_seqlens: Optional[tuple[int, ...]] = None
    description: str = ""


CONFIGS: dict[str, PackConfig] = {
    c.name: c
    for c in [
        PackConfig(
            name="tiny_2doc_gqa2_d64", index=0, T=128, Hq=4, Hkv=2, D=64,
            window=0, scale=1.0 / 8.0, sinks=False,
            fixed_cu_seqlens=(0, 37, 128),
            description="2 documents of 37 and 91 tokens, Hq=4 Hkv=2 D=64, full causal, scale 1/8",
        ),
        PackConfig(
            name="pack8k_gqa4_d128_causal", index=1, T=8192, Hq=32, Hkv=8, D=128,
            window=0, scale=128 ** -0.5, sinks=False, doc_len_range=(64, 4096),
            description="8,192-token pack, log-uniform doc lengths in [64, 4096], Hq=32 Hkv=8 D=128, full causal",
        ),
        PackConfig(
            name="pack32k_gqa4_d128_w4096", index=2, T=32768, Hq=32, Hkv=8, D=128,
            window=4096, scale=128 ** -0.5, sinks=False, doc_len_range=(256, 16384),
            description="32,768-token pack, log-uniform doc lengths in [256, 16384], Hq=32 Hkv=8 D=128, window 4096",
        ),
        PackConfig(
            name="pack64k_gqa8_d128_causal_sink", index=3, T=65536, Hq=64, Hkv=8, D=128,
            window=0, scale=128 ** -0.5, sinks=True, doc_len_range=(1024, 32768),
            description="65,536-token pack, log-uniform doc lengths in [1024, 32768], Hq=64 Hkv=8 D=128, full causal, learned sinks",
        ),
        PackConfig(
            name="doc128k_mqa_d256_w8192_sink", index=4, T=131072, Hq=16, Hkv=1, D=256,
            window=8192, scale=256 ** -0.5, sinks=True, std=0.5,
            fixed_cu_seqlens=(0, 131072),
            description="single 131,072-token document, Hq=16 Hkv=1 (MQA) D=256, window 8192, learned sinks, q/k/v N(0, 0.5^2)",
        ),
    ]
}

CONFIG_ORDER: list[str] = [n for n, _ in sorted(CONFIGS.items(), key=lambda kv: kv[1].index)]


def doc_lengths(T: int, lo: int, hi: int, seed: int) -> list[int]:
    """Log-uniform document lengths in [lo, hi] filling exactly T tokens."""
    rng = np.random.default_rng(seed)
    lens: list[int] = []
    used = 0
    while used < T:
        L = int(round(math.exp(rng.uniform(math.log(lo), math.log(hi)))))
        L = max(1, min(L, T - used))
        lens.append(L)
        used += L
    return lens


def cu_seqlens_from_lengths(lengths: Sequence[int]) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def pack_cu_seqlens(cfg: PackConfig, seed: int = 0) -> np.ndarray:
    if cfg.fixed_cu_seqlens is not None:
        return np.asarray(cfg.fixed_cu_seqlens, dtype=np.int32)
    lo, hi = cfg.doc_len_range
    return cu_seqlens_from_lengths(doc_lengths(cfg.T, lo, hi, seed))


def random_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> torch.Tensor:
    """float32 N(0, std^2) rounded to bf16 (round-to-nearest-even) on the CPU."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return torch.from_numpy(x).to(torch.bfloat16)


def make_pack(cfg: PackConfig, seed: int = 0, tensor_seed: Optional[int] = None,
              T_override: Optional[int] = None) -> dict:
    """Build one pack on the CPU.

    ``tensor_seed`` (default ``seed``) seeds the tensor values separately from
    the document lengths, so that ranks of a multi-GPU run can hold packs of
    the same shape with different values.  ``T_override`` truncates the pack
    to its first ``T_override`` tokens (cut at the document containing that
    token) for reduced-size parity runs.
    """
    cu = pack_cu_seqlens(cfg, seed)
    if T_override is not None and T_override < int(cu[-1]):
        keep = [0]
        for b in cu[1:]:
            if b >= T_override:
                keep.append(T_override)
                break
            keep.append(int(b))
        cu = np.asarray(keep, dtype=np.int32)
    T = int(cu[-1])
    ts = seed if tensor_seed is None else tensor_seed
    rng2 = np.random.default_rng([ts, cfg.index])
    q = random_bf16(rng2, (T, cfg.Hq, cfg.D), cfg.std)
    k = random_bf16(rng2, (T, cfg.Hkv, cfg.D), cfg.std)
    v = random_bf16(rng2, (T, cfg.Hkv, cfg.D), cfg.std)
    sinks = None
    if cfg.sinks:
        sinks = torch.from_numpy(rng2.standard_normal(size=(cfg.Hq,), dtype=np.float32))
    return dict(q=q, k=k, v=v, cu_seqlens=cu, sinks=sinks, window=cfg.window,
                scale=cfg.scale, Hq=cfg.Hq, Hkv=cfg.Hkv, D=cfg.D, T=T, config=cfg)


def random_pack(seed: int, doc_lengths_: Sequence[int], Hq: int, Hkv: int, D: int,
                window: int, scale: float, sinks: bool, std: float = 1.0) -> dict:
    """A pack with explicitly given document lengths (zero-length allowed)."""
    cu = cu_seqlens_from_lengths(doc_lengths_)
    T = int(cu[-1])
    rng = np.random.default_rng([seed, 1000 + len(doc_lengths_)])
    q = random_bf16(rng, (T, Hq, D), std)
    k = random_bf16(rng, (T, Hkv, D), std)
    v = random_bf16(rng, (T, Hkv, D), std)
    s = torch.from_numpy(rng.standard_normal(size=(Hq,), dtype=np.float32)) if sinks else None
    return dict(q=q, k=k, v=v, cu_seqlens=cu, sinks=s, window=window, scale=scale,
                Hq=Hq, Hkv=Hkv, D=D, T=T, config=None)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a CPU bf16 tensor as a uint16 numpy array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ sparse MLA

def sparse_mla_case(seed: int, doc_lengths_: Sequence[int], H: int, K: int, value_dim: int,
                    device=None) -> dict:
    """Synthetic sparse-MLA inputs (shapes of "mistral_large4.attention"'s
    sparse_mla): q [T, H, 576] and kv [T, 576] ~ N(0, 1) in bf16 (the last 64
    query columns rotary), value_weight [H, value_dim, 512] ~ N(0, 1/512), and
    for every token a random subset of up to K of the keys it may see (same
    document, not after it; the caller's document / causal boundaries), in
    random order, padded with -1; scale (128 + 64) ** -0.5 (a 192-wide MLA
    query head: 128 latent-absorbed + 64 rotary)."""
    rng = np.random.default_rng(seed)
    cu = cu_seqlens_from_lengths(doc_lengths_)
    T = int(cu[-1])
    q = random_bf16(rng, (T, H, 576))
    kv = random_bf16(rng, (T, 576))
    w = random_bf16(rng, (H, value_dim, 512), std=512 ** -0.5)
    idx = np.full((T, K), -1, dtype=np.int32)
    for d in range(len(cu) - 1):
        s, e = int(cu[d]), int(cu[d + 1])
        for t in range(s, e):
            n = min(K, t - s + 1)
            sel = rng.choice(np.arange(s, t + 1), size=n, replace=False)
            slots = rng.permutation(K)[:n]
            idx[t, slots] = sel
    return {"q": q, "kv": kv, "value_weight": w, "indices": torch.from_numpy(idx), "T": T,
            "cu_seqlens": cu, "scale": (128 + 64) ** -0.5}
