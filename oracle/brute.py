"""NumPy fp64 brute-force twin of the C oracle, for tiny inputs.

TEST INFRASTRUCTURE ONLY.  It is written independently of ``jl_oracle.c``:
rotations use complex arithmetic (pair (c, c + d/2) as x_c + i x_{c+d/2}
multiplied by e^{i p theta_c}), and the whole L x L routed score matrix is
materialised with its explicit mask (Methodology section 1, "Dynamic Bifocal
RoPE": local window of w0 with classical RoPE, remote map f(x) = floor(x/G),
G = max(1, ceil(L / w_pretrained))).
"""
from __future__ import annotations

import numpy as np


def group_size(L: int, w_pretrained: int) -> int:
    # ceil without floating point: -(-L // w)
    return max(1, -(-L // w_pretrained))


def rotate_complex(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """R(pos) x for x [n][d] and integer positions pos [n], via complex multiplication."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    h = d // 2
    theta = base ** (-np.arange(0, d, 2, dtype=np.float64) / d)  # base^(-2c/d)
    z = x[..., :h] + 1j * x[..., h:]
    z = z * np.exp(1j * np.asarray(pos, np.float64)[:, None] * theta[None, :])
    return np.concatenate([z.real, z.imag], axis=-1)


def routed_masks(L: int, w0: int):
    """(local, remote) boolean [L][L] masks over (i, j): local 0 <= i-j < w0, remote i-j >= w0."""
    dist = np.subtract.outer(np.arange(L), np.arange(L))  # i - j
    causal = np.tri(L, L, 0, dtype=bool)  # j <= i
    local = causal & ~np.tri(L, L, -w0, dtype=bool)  # exclude i - j >= w0
    remote = causal & ~local
    assert np.all(local == ((dist >= 0) & (dist < w0)))
    return local, remote


def bifocal_single_head(q, k, v, *, w0, w_pretrained, rope_base, scale=None, plain=False):
    """Full routed attention for one head and one sequence. q, k, v: [L][d] raw.

    Returns (out [L][d], lse [L], S [L][L] with -inf where masked).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    L, d = q.shape
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    G = 1 if plain else group_size(L, w_pretrained)
    pos = np.arange(L)
    fpos = pos // G
    sb = sc * rotate_complex(q, pos, rope_base) @ rotate_complex(k, pos, rope_base).T
    sr = sc * rotate_complex(q, fpos, rope_base) @ rotate_complex(k, fpos, rope_base).T
    local, remote = routed_masks(L, L if plain else w0)
    S = np.full((L, L), -np.inf)
    S[local] = sb[local]
    S[remote] = sr[remote]
    m = S.max(axis=1, keepdims=True)
    P = np.exp(S - m)
    z = P.sum(axis=1, keepdims=True)
    out = (P / z) @ v
    lse = (m + np.log(z))[:, 0]
    return out, lse, S
