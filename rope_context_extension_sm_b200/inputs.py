"""Seeded synthetic workloads (shared by the tests, the benchmark and smoke).

This module only draws random numbers and lays them out; it holds none of the
attention method's arithmetic (no rotation, no position map, no softmax).

Recipe (every workload):
  * Q, K, V are i.i.d. N(0, 1) drawn with ``numpy.random.Generator(PCG64(seed))``
    as float32, then rounded to bf16 (round to nearest even).
  * Seeds: 0 for Q, 1 for K, 2 for V, 3 for the per-channel key scales,
    4 for the varlen lengths, 5 for the decode-walk queries.
  * "Outlier channels": K[..., c] is multiplied by u_c ~ U[0.5, 2] (one factor
    per head-dim channel, shared by every head and token) before rounding.
  * Varlen lengths: L_s = floor(exp(U(ln 4096, ln 131072))).
Tensors are token-major, packed: [T][H][d].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

SEED_Q, SEED_K, SEED_V, SEED_SCALE, SEED_LENS, SEED_DECODE = 0, 1, 2, 3, 4, 5


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    seqlens: tuple
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    w0: int
    w_pretrained: int
    rope_base: float
    outlier_k: bool

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def max_seqlen(self) -> int:
        return int(max(self.seqlens)) if self.seqlens else 0

    def useful_flops(self) -> float:
        """4*d flops per causal (q, k) pair per query head; each pair counted once."""
        return float(sum(4.0 * self.head_dim * self.n_q_heads * L * (L + 1) / 2 for L in self.seqlens))


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    cache_lens: tuple
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    w0: int
    w_pretrained: int
    rope_base: float
    walk_first_pos: int = 98176
    walk_steps: int = 256


def varlen_lengths(n: int = 8, lo: int = 4096, hi: int = 131072, seed: int = SEED_LENS) -> tuple:
    g = np.random.Generator(np.random.PCG64(seed))
    u = g.uniform(math.log(lo), math.log(hi), size=n)
    return tuple(int(math.floor(math.exp(x))) for x in u)


TINY = PrefillConfig("tiny_L256_d64_G4", (256,), 1, 1, 64, 32, 64, 1e4, False)
QWEN3_1P7B = PrefillConfig("qwen3_1p7b_L65536_G2", (65536,), 16, 8, 128, 4096, 32768, 1e6, True)
QWEN3_8B_128K = PrefillConfig("qwen3_8b_L131072_G4", (131072,), 32, 8, 128, 4096, 32768, 1e6, True)
VARLEN = PrefillConfig("varlen_8seq_4k_128k", varlen_lengths(), 16, 8, 128, 4096, 32768, 1e6, False)
DECODE_QWEN3_4B = DecodeConfig("decode_qwen3_4b", (8192, 32768, 65536, 131072), 32, 8, 128, 4096, 32768, 1e6)
W0_SWEEP = (1024, 2048, 4096, 8192)


def with_(cfg: PrefillConfig, **kw) -> PrefillConfig:
    d = dict(cfg.__dict__)
    d.update(kw)
    return PrefillConfig(**d)


def _normal_bf16(seed: int, shape, scale: np.ndarray | None = None, chunk_rows: int = 8192) -> torch.Tensor:
    """N(0,1) float32 draws in row-major order, optionally scaled per last-dim channel, rounded to bf16."""
    g = np.random.Generator(np.random.PCG64(seed))
    out = torch.empty(shape, dtype=torch.bfloat16)
    rows = shape[0]
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = g.standard_normal((r1 - r0,) + tuple(shape[1:]), dtype=np.float32)
        if scale is not None:
            x *= scale.astype(np.float32)
        out[r0:r1] = torch.from_numpy(x).to(torch.bfloat16)
    return out


def channel_scales(d: int, seed: int = SEED_SCALE) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(seed))
    return g.uniform(0.5, 2.0, size=d)


def prefill_inputs(cfg: PrefillConfig):
    """(q, k, v, cu_seqlens) as CPU tensors: bf16 [T][H][d] and int32 [B+1]."""
    T, d = cfg.total_tokens, cfg.head_dim
    sc = channel_scales(d) if cfg.outlier_k else None
    q = _normal_bf16(SEED_Q, (T, cfg.n_q_heads, d))
    k = _normal_bf16(SEED_K, (T, cfg.n_kv_heads, d), sc)
    v = _normal_bf16(SEED_V, (T, cfg.n_kv_heads, d))
    cu = torch.zeros(len(cfg.seqlens) + 1, dtype=torch.int32)
    if cfg.seqlens:
        cu[1:] = torch.cumsum(torch.tensor(cfg.seqlens, dtype=torch.int64), 0).to(torch.int32)
    return q, k, v, cu


def decode_raw_inputs(cfg: DecodeConfig, max_len: int, batch: int = 1):
    """Raw (un-rotated) keys/values for a cache of max_len positions, and values.

    Returns k_raw, v as bf16 [batch][max_len][Hkv][d].  The base-RoPE cache a
    caller stores is R(j) k_raw[j]; producing it is the caller's job.
    """
    d = cfg.head_dim
    sc = channel_scales(d)
    k = _normal_bf16(SEED_K, (batch * max_len, cfg.n_kv_heads, d), sc).view(batch, max_len, cfg.n_kv_heads, d)
    v = _normal_bf16(SEED_V, (batch * max_len, cfg.n_kv_heads, d)).view(batch, max_len, cfg.n_kv_heads, d)
    return k, v


def decode_queries(cfg: DecodeConfig, n: int, batch: int = 1, seed: int = SEED_DECODE):
    """n raw decode queries per batch entry: bf16 [n][batch][Hq][d]."""
    return _normal_bf16(seed, (n * batch, cfg.n_q_heads, cfg.head_dim)).view(n, batch, cfg.n_q_heads, cfg.head_dim)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a CPU bf16 tensor (for the oracle's bf16 views)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
