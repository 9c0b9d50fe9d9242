"""Seeded synthetic inputs for the attention hot path.

This module only draws numbers: shapes, seeds, value distributions and length
mixes of the five workloads below.  It holds none of the attention arithmetic
(no RoPE, no softmax), so both the CUDA path and the fp64 oracle can take their
inputs from it without sharing any of the method.

All tensors are drawn on the CPU with ``torch.Generator().manual_seed(seed)``
as float32 N(0, 1) and then cast to the workload dtype, so the same bytes can
be handed to the GPU and to the oracle.

Workloads (shapes as the pages' LLaMA configurations use them):

* ``tiny_fp32``   causal GQA prefill, fp32, b1 S64 H4 Hkv2 D64, RoPE theta 1e4
* ``mha_bf16``    non-causal MHA without RoPE, bf16, b4 S128 H32 Hkv32 D128
                  (hidden 4096; the tensor-parallel demo shape [4, 128, 4096])
* ``llama7b``     causal MHA prefill, bf16, b2 S4096 H32 Hkv32 D128, RoPE 1e4
* ``llama70b``    causal GQA prefill, bf16, b1 S8192 H64 Hkv8 D128, RoPE 1e4
                  with linear position scaling factor 2.0
* ``decode70b``   GQA single-token decode, bf16, b32 H64 Hkv8 D128, cache
                  lengths uniform in [512, 4096], max cache length 4096, query
                  position = cache length, cache rows past the length poisoned
                  with NaN
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    bsz: int
    seq: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: torch.dtype
    causal: bool
    rope: bool
    theta: float = 10000.0
    factor: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return self.head_dim ** -0.5

    def unmasked_pairs(self) -> int:
        """Number of (query row, key) pairs that take part, summed over b and heads."""
        per = self.seq * (self.seq + 1) // 2 if self.causal else self.seq * self.seq
        return per * self.bsz * self.n_heads

    def flops(self) -> int:
        """Algorithmic FLOPs: 2*D for QK^T plus 2*D for PV per unmasked pair."""
        return 4 * self.head_dim * self.unmasked_pairs()


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    bsz: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    max_cache_len: int
    min_len: int
    max_len: int
    dtype: torch.dtype
    theta: float = 10000.0
    factor: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return self.head_dim ** -0.5


TINY_FP32 = PrefillConfig("tiny_fp32", 1, 64, 4, 2, 64, torch.float32, True, True, seed=1000)
MHA_BF16 = PrefillConfig("mha_bf16", 4, 128, 32, 32, 128, torch.bfloat16, False, False, seed=1001)
LLAMA7B = PrefillConfig("llama7b", 2, 4096, 32, 32, 128, torch.bfloat16, True, True, seed=1002)
LLAMA70B = PrefillConfig("llama70b", 1, 8192, 64, 8, 128, torch.bfloat16, True, True,
                         factor=2.0, seed=1003)
DECODE70B = DecodeConfig("decode70b", 32, 64, 8, 128, 4096, 512, 4096, torch.bfloat16, seed=1004)

PREFILL_CONFIGS = {c.name: c for c in (TINY_FP32, MHA_BF16, LLAMA7B, LLAMA70B)}
DECODE_CONFIGS = {DECODE70B.name: DECODE70B}


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(int(seed))


def normal(shape, dtype, gen: torch.Generator) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(dtype)


def prefill_inputs(cfg: PrefillConfig, seed: Optional[int] = None, with_mask: bool = False):
    """q [b,S,H,D], k/v [b,S,Hkv,D], pos [b,S] int64 (None when the workload has no RoPE)."""
    g = _gen(cfg.seed if seed is None else seed)
    b, S, H, Hkv, D = cfg.bsz, cfg.seq, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    q = normal((b, S, H, D), cfg.dtype, g)
    k = normal((b, S, Hkv, D), cfg.dtype, g)
    v = normal((b, S, Hkv, D), cfg.dtype, g)
    pos = torch.arange(S, dtype=torch.int64).repeat(b, 1) if cfg.rope else None
    mask = additive_mask(b, S, g) if with_mask else None
    return {"q": q, "k": k, "v": v, "pos": pos, "mask": mask}


def additive_mask(bsz: int, seq: int, gen: torch.Generator, blocked_frac: float = 0.2):
    """[b,1,S,S] float32: N(0,1) biases with a random fraction of entries set to -1e9.

    The diagonal is never blocked, so every row keeps at least one key.
    """
    m = torch.randn(bsz, 1, seq, seq, generator=gen, dtype=torch.float32)
    blocked = torch.rand(bsz, 1, seq, seq, generator=gen) < blocked_frac
    eye = torch.eye(seq, dtype=torch.bool).view(1, 1, seq, seq)
    blocked &= ~eye
    m[blocked] = -1e9
    return m


def decode_inputs(cfg: DecodeConfig, seed: Optional[int] = None, poison: bool = True,
                  lens: Optional[torch.Tensor] = None):
    """q [b,H,D] un-rotated, caches [b,Hkv,L,D], lens [b] int32, qpos [b] int64 (= lens).

    Cache rows at or past lens[b] are filled with NaN when ``poison`` is set.
    """
    g = _gen(cfg.seed if seed is None else seed)
    b, H, Hkv, D, L = cfg.bsz, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.max_cache_len
    if lens is None:
        lens = torch.randint(cfg.min_len, cfg.max_len + 1, (b,), generator=g, dtype=torch.int64)
    lens = lens.to(torch.int32)
    q = normal((b, H, D), cfg.dtype, g)
    k_cache = normal((b, Hkv, L, D), cfg.dtype, g)
    v_cache = normal((b, Hkv, L, D), cfg.dtype, g)
    if poison:
        idx = torch.arange(L).view(1, 1, L, 1)
        tail = idx >= lens.view(b, 1, 1, 1).to(torch.int64)
        k_cache = k_cache.masked_fill(tail, float("nan"))
        v_cache = v_cache.masked_fill(tail, float("nan"))
    qpos = lens.to(torch.int64).clone()
    return {"q": q, "k_cache": k_cache, "v_cache": v_cache, "lens": lens, "qpos": qpos}


def small_prefill(bsz, seq, n_heads, n_kv_heads, head_dim, dtype, causal=True, rope=True,
                  theta=10000.0, factor=1.0, seed=0, with_mask=False):
    """A random small prefill problem (same generator recipe as the named workloads)."""
    cfg = PrefillConfig("small", bsz, seq, n_heads, n_kv_heads, head_dim, dtype, causal, rope,
                        theta=theta, factor=factor, seed=seed)
    return cfg, prefill_inputs(cfg, with_mask=with_mask)


def small_decode(bsz, n_heads, n_kv_heads, head_dim, max_cache_len, dtype, min_len=1,
                 max_len=None, seed=0, poison=True, lens=None):
    cfg = DecodeConfig("small", bsz, n_heads, n_kv_heads, head_dim, max_cache_len, min_len,
                       max_cache_len if max_len is None else max_len, dtype, seed=seed)
    return cfg, decode_inputs(cfg, poison=poison, lens=lens)
