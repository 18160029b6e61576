"""Pins for the CPU oracle: it is checked against things other than itself.

Each test names the fact it checks and where that fact comes from:
  * the group-size / remote-map equations (golden tables evaluated by hand),
  * the on-grid statement for remote angles,
  * exact recovery of plain RoPE attention at short inputs,
  * additive composition of RoPE rotations,
  * inclusion-exclusion giving the exact distance-routed output,
  * library special cases (torch scaled_dot_product_attention in fp64),
  * an independent numpy brute force with an explicit L x L mask.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import brute
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(tuple(int(x) for x in line.split()))
    return rows


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- G and f ----

def test_group_size_golden():
    """G = max(1, ceil(L / w_pretrained)) (Methodology section 1, equation for G)."""
    for L, w, G in _golden("group_size.txt"):
        assert O.group_size(L, w) == G, (L, w)
        assert brute.group_size(L, w) == G, (L, w)


def test_remote_pos_golden():
    """f(x) = floor(x / G) (Methodology section 1, integer division)."""
    for x, G, f in _golden("remote_pos.txt"):
        assert O.remote_pos(x, G) == f


@pytest.mark.parametrize("w_pre", [1, 2, 3, 5, 8, 16, 17])
def test_remote_angles_on_grid_exhaustive(w_pre):
    """Every remote relative position f(i) - f(j), j <= i < L, lies in [0, w_pre - 1]
    ("each remote rotation angle stays on the pretraining grid", Methodology section 1)."""
    for L in range(1, 6 * w_pre + 3):
        G = O.group_size(L, w_pre)
        f = np.array([O.remote_pos(x, G) for x in range(L)])
        assert f[-1] <= w_pre - 1
        rel = np.subtract.outer(f, f)[np.tril_indices(L)]
        assert rel.min() >= 0 and rel.max() <= w_pre - 1
        # minimal compression: with G - 1 the last position would fall off the grid
        if G > 1:
            assert (L - 1) // (G - 1) > w_pre - 1


def test_remote_angles_on_grid_large():
    w_pre = 32768
    for L in [32768, 32769, 65536, 98304, 98305, 131072]:
        G = O.group_size(L, w_pre)
        assert O.remote_pos(L - 1, G) <= w_pre - 1
        assert O.remote_pos(0, G) == 0


# ------------------------------------------------------------- rotations ----

def test_inv_freq_closed_form():
    """theta_c = base^(-2c/d): theta_0 = 1, theta for d = 4, base = 100 is (1, 1/10)."""
    np.testing.assert_allclose(O.inv_freq(4, 100.0), [1.0, 0.1], rtol=1e-15)
    t = O.inv_freq(128, 1e6)
    assert t[0] == 1.0
    np.testing.assert_allclose(t[1:] / t[:-1], 1e6 ** (-2.0 / 128), rtol=1e-13)


def test_cos_sin_table_closed_form():
    c, s = O.rope_cos_sin(1000, 8, 1e4)
    np.testing.assert_array_equal(c[0], 1.0)
    np.testing.assert_array_equal(s[0], 0.0)
    p = np.arange(1000)
    np.testing.assert_allclose(c[:, 0], np.cos(p), atol=1e-15)  # theta_0 = 1
    np.testing.assert_allclose(s[:, 0], np.sin(p), atol=1e-15)
    np.testing.assert_allclose(c ** 2 + s ** 2, 1.0, atol=1e-15)


@pytest.mark.parametrize("d,base", [(8, 1e4), (64, 1e4), (128, 1e6)])
def test_rotation_composes_additively(d, base):
    """R(a) R(b) = R(a + b) (RoPE rotations compose additively, Methodology section 2)."""
    x = _rand(d, 1)
    for a, b in [(0, 0), (3, 5), (-7, 7), (1000, -250), (98304, -73728), (131071, -98303)]:
        lhs = O.rotate(O.rotate(x, b, base), a, base)
        rhs = O.rotate(x, a + b, base)
        np.testing.assert_allclose(lhs, rhs, atol=1e-9 * np.abs(x).max())
    np.testing.assert_array_equal(O.rotate(x, 0, base), x)  # R(0) = I
    y = O.rotate(x, 12345, base)
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12 * np.linalg.norm(x)


@pytest.mark.parametrize("d,base", [(8, 1e4), (128, 1e6)])
def test_rotation_matches_complex_multiplication(d, base):
    """Rotate-half pairing (c, c + d/2): R(p) x equals (x_c + i x_{c+d/2}) e^{i p theta_c}."""
    x = _rand((5, d), 2)
    pos = np.array([0, 1, 17, 4096, 131071])
    ref = brute.rotate_complex(x, pos, base)
    got = np.stack([O.rotate(x[r], int(pos[r]), base) for r in range(5)])
    np.testing.assert_allclose(got, ref, atol=1e-10)


def test_rotate_rows_matches_single_rotations():
    x = _rand((6, 16), 3)
    pos = np.array([0, 5, -5, 77, 131071, -98303])
    y = O.rotate_rows(x, pos, 1e6)
    for r in range(6):
        np.testing.assert_array_equal(y[r], O.rotate(x[r], int(pos[r]), 1e6))


# ---------------------------------------------------- attention helpers ----

def _seq(L, hq, hkv, d, seed):
    q = _rand((L, hq, d), seed)
    k = _rand((L, hkv, d), seed + 1)
    v = _rand((L, hkv, d), seed + 2)
    return q, k, v


def _all_rows(L, hq):
    pos = np.repeat(np.arange(L), hq)
    head = np.tile(np.arange(hq), L)
    return pos, head


def _rows(q, k, v, L, w0, w_pre, base, **kw):
    pos, head = _all_rows(L, q.shape[1])
    out, lse = O.bifocal_rows(q, k, v, L, pos, head, w0=w0, w_pretrained=w_pre, rope_base=base, **kw)
    return out.reshape(L, q.shape[1], -1), lse.reshape(L, q.shape[1])


def _sdpa(qr, kr, v, mask):
    """torch fp64 scaled_dot_product_attention with a boolean keep-mask; qr, kr, v: [L][d]."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(t(qr), t(kr), t(v), attn_mask=t(mask))
    s = (t(qr) @ t(kr).transpose(-1, -2)) / math.sqrt(qr.shape[-1])
    lse = torch.logsumexp(s.masked_fill(~t(mask), -math.inf), dim=-1)
    return out[0, 0].numpy(), lse[0, 0].numpy()


# ----------------------------------------------- exact recovery (G = 1) ----

@pytest.mark.parametrize("w0", [0, 1, 5, 16, 40])
def test_short_input_equals_plain_rope_bit_for_bit(w0):
    """L <= w_pretrained => G = 1 => the bifocal output IS plain causal RoPE attention,
    bit for bit in the oracle's own arithmetic ("recovers the base model exactly at short
    inputs", abstract)."""
    L, w_pre, base = 37, 40, 1e4
    q, k, v = _seq(L, 4, 2, 16, 10)
    ob, lb = _rows(q, k, v, L, w0, w_pre, base)
    op, lp = _rows(q, k, v, L, w0, w_pre, base, plain=True)
    np.testing.assert_array_equal(ob, op)
    np.testing.assert_array_equal(lb, lp)


def test_plain_rope_matches_library_sdpa():
    """Plain causal RoPE attention equals torch SDPA (fp64, causal) on complex-rotated q, k."""
    L, d, base = 45, 32, 1e4
    q, k, v = _seq(L, 2, 1, d, 20)
    op, lp = _rows(q, k, v, L, 0, 64, base, plain=True)
    pos = np.arange(L)
    causal = np.tri(L, L, 0, dtype=bool)
    for h in range(2):
        ref, rl = _sdpa(brute.rotate_complex(q[:, h], pos, base), brute.rotate_complex(k[:, 0], pos, base),
                        v[:, 0], causal)
        np.testing.assert_allclose(op[:, h], ref, atol=1e-12)
        np.testing.assert_allclose(lp[:, h], rl, atol=1e-12)


@pytest.mark.parametrize("w_pre", [4, 7, 16])
def test_window_covering_input_equals_plain_bit_for_bit(w_pre):
    """w0 >= L: every causal pair is local, so the output is plain RoPE for any G."""
    L = 50
    q, k, v = _seq(L, 2, 2, 8, 30)
    for w0 in [L, L + 1, 10 * L]:
        ob, lb = _rows(q, k, v, L, w0, w_pre, 1e4)
        op, lp = _rows(q, k, v, L, w0, w_pre, 1e4, plain=True)
        np.testing.assert_array_equal(ob, op)
        np.testing.assert_array_equal(lb, lp)


@pytest.mark.parametrize("w0", [1, 6, 19])
def test_rows_inside_window_equal_plain_rope(w0):
    """Rows i < w0 see only local keys, so they equal plain RoPE rows for any G."""
    L, w_pre = 64, 8  # G = 8
    q, k, v = _seq(L, 2, 1, 8, 40)
    ob, lb = _rows(q, k, v, L, w0, w_pre, 1e4)
    op, lp = _rows(q, k, v, L, w0, w_pre, 1e4, plain=True)
    np.testing.assert_array_equal(ob[:w0], op[:w0])
    np.testing.assert_array_equal(lb[:w0], lp[:w0])
    assert np.abs(ob[w0:] - op[w0:]).max() > 1e-6  # and the routing does act beyond the window


# ------------------------------------------- library pins for G > 1 ----

@pytest.mark.parametrize("L,w_pre", [(40, 10), (64, 16), (33, 8)])
def test_no_window_equals_attention_at_remote_positions(L, w_pre):
    """w0 = 0: every pair is remote, so the output is causal attention with positions f(.),
    computed here by torch SDPA on q, k rotated at f(i), f(j)."""
    d, base = 16, 1e4
    q, k, v = _seq(L, 1, 1, d, 50)
    ob, lb = _rows(q, k, v, L, 0, w_pre, base)
    G = brute.group_size(L, w_pre)
    f = np.arange(L) // G
    ref, rl = _sdpa(brute.rotate_complex(q[:, 0], f, base), brute.rotate_complex(k[:, 0], f, base), v[:, 0],
                    np.tri(L, L, 0, dtype=bool))
    np.testing.assert_allclose(ob[:, 0], ref, atol=1e-12)
    np.testing.assert_allclose(lb[:, 0], rl, atol=1e-12)


@pytest.mark.parametrize("L,w_pre,w0", [(48, 12, 5), (64, 16, 9), (70, 20, 1), (57, 10, 30)])
def test_routed_equals_lse_merge_of_two_library_softmaxes(L, w_pre, w0):
    """The distance-routed output equals the log-sum-exp merge of two library softmaxes:
    local keys (0 <= i-j < w0) with base-rotated q, k and remote keys (i-j >= w0) with
    q, k rotated at f(i), f(j) (Methodology section 2, "exact distance-based routing")."""
    d, base = 16, 1e4
    q, k, v = _seq(L, 1, 1, d, 60)
    ob, lb = _rows(q, k, v, L, w0, w_pre, base)
    G = brute.group_size(L, w_pre)
    pos = np.arange(L)
    dist = np.subtract.outer(pos, pos)
    local = (dist >= 0) & (dist < w0)
    remote = dist >= w0
    o1, l1 = _sdpa(brute.rotate_complex(q[:, 0], pos, base), brute.rotate_complex(k[:, 0], pos, base), v[:, 0],
                   local)
    o2, l2 = _sdpa(brute.rotate_complex(q[:, 0], pos // G, base), brute.rotate_complex(k[:, 0], pos // G, base),
                   v[:, 0], remote)
    has2 = remote.any(axis=1)
    lse = np.where(has2, np.logaddexp(l1, np.where(has2, l2, -np.inf)), l1)
    w1 = np.exp(l1 - lse)[:, None]
    w2 = np.where(has2, np.exp(np.where(has2, l2, 0) - lse), 0)[:, None]
    ref = w1 * o1 + w2 * np.where(has2[:, None], o2, 0)
    np.testing.assert_allclose(ob[:, 0], ref, atol=1e-12)
    np.testing.assert_allclose(lb[:, 0], lse, atol=1e-12)


# ----------------------------------------- brute-force twin (explicit mask) ----

@pytest.mark.parametrize("L,w_pre,w0,hq,hkv", [(1, 4, 2, 1, 1), (17, 4, 3, 2, 1), (64, 16, 8, 4, 2),
                                               (100, 30, 0, 2, 2), (100, 30, 100, 1, 1), (96, 25, 7, 3, 1)])
def test_c_oracle_matches_numpy_brute_force(L, w_pre, w0, hq, hkv):
    d, base = 16, 1e4
    q, k, v = _seq(L, hq, hkv, d, 70)
    ob, lb = _rows(q, k, v, L, w0, w_pre, base)
    grp = hq // hkv
    for h in range(hq):
        ref, rl, _ = brute.bifocal_single_head(q[:, h], k[:, h // grp], v[:, h // grp], w0=w0,
                                                w_pretrained=w_pre, rope_base=base)
        np.testing.assert_allclose(ob[:, h], ref, atol=1e-12)
        np.testing.assert_allclose(lb[:, h], rl, atol=1e-12)


def test_c_oracle_reads_bf16_and_fp32_views_exactly():
    L, d = 40, 16
    q, k, v = _seq(L, 2, 1, d, 80)
    qb = torch.from_numpy(q).to(torch.bfloat16)
    kb = torch.from_numpy(k).to(torch.bfloat16)
    vb = torch.from_numpy(v).to(torch.bfloat16)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    o16, l16 = _rows(bits(qb), bits(kb), bits(vb), L, 5, 8, 1e4)
    o64, l64 = _rows(qb.double().numpy(), kb.double().numpy(), vb.double().numpy(), L, 5, 8, 1e4)
    o32, l32 = _rows(qb.float().numpy(), kb.float().numpy(), vb.float().numpy(), L, 5, 8, 1e4)
    np.testing.assert_array_equal(o16, o64)
    np.testing.assert_array_equal(l16, l64)
    np.testing.assert_array_equal(o32, o64)


# ------------------------------------------------ inclusion-exclusion ----

@pytest.mark.parametrize("L", [1, 2, 7, 33, 64])
@pytest.mark.parametrize("G_target", [1, 2, 3, 4])
def test_three_pass_merge_equals_masked_definition(L, G_target):
    """Inclusion-exclusion of the three passes (local/base + causal/remote - local/remote),
    merged on their LogSumExp statistics, gives the exact distance-routed output
    (Methodology section 2); brute force over every w0 in [0, L + 1]."""
    d, base = 8, 1e4
    w_pre = max(1, -(-L // G_target))  # a w_pretrained that yields G = G_target (or less for tiny L)
    q, k, v = _seq(L, 1, 1, d, 90 + L)
    pos, head = _all_rows(L, 1)
    for w0 in range(0, L + 2):
        od, ld = O.bifocal_rows(q, k, v, L, pos, head, w0=w0, w_pretrained=w_pre, rope_base=base)
        o3, l3, pl = O.bifocal_rows(q, k, v, L, pos, head, w0=w0, w_pretrained=w_pre, rope_base=base,
                                    three_pass=True)
        np.testing.assert_allclose(o3, od, atol=1e-12, rtol=0)
        np.testing.assert_allclose(l3, ld, atol=1e-12, rtol=0)
        # pass statistics: pass 1 empty iff w0 = 0; passes 2 and 3 coincide for rows i < w0
        assert np.all(np.isneginf(pl[:, 0]) == (w0 == 0))
        inside = pos < w0
        np.testing.assert_array_equal(pl[inside, 1], pl[inside, 2])


# --------------------------------------------------------------- decode ----

@pytest.mark.parametrize("w0", [0, 3, 8, 1000])
def test_decode_on_cache_equals_last_prefill_row(w0):
    """The correction rotation on a base-RoPE cache reproduces the routed score exactly:
    R(f(i)-i) R(i) q . R(f(j)-j) R(j) k = R(f(i)) q . R(f(j)) k (additive composition,
    Methodology section 2).  Decode at length L equals the last prefill row at L, for L
    on both sides of G boundaries."""
    d, base, w_pre, hq, hkv = 16, 1e4, 12, 4, 2
    Lmax = 40
    q, k, v = _seq(Lmax, hq, hkv, d, 100)
    # base-RoPE cache in fp64 (not rounded): k_tilde_j = R(j) k_j
    kc = np.stack([np.stack([O.rotate(k[j, h], j, base) for h in range(hkv)]) for j in range(Lmax)])
    for L in [1, 11, 12, 13, 24, 25, 36, 37, 40]:
        qt = np.stack([O.rotate(q[L - 1, h], L - 1, base) for h in range(hq)])
        od, ld = O.decode_step(qt, kc, v, L, w0=w0, w_pretrained=w_pre, rope_base=base)
        pos = np.full(hq, L - 1)
        op, lp = O.bifocal_rows(q[:L], k[:L], v[:L], L, pos, np.arange(hq), w0=w0, w_pretrained=w_pre,
                                rope_base=base)
        np.testing.assert_allclose(od, op, atol=1e-12)
        np.testing.assert_allclose(ld, lp, atol=1e-12)
        # plain decode equals plain prefill's last row
        od, ld = O.decode_step(qt, kc, v, L, w0=w0, w_pretrained=w_pre, rope_base=base, plain=True)
        op, lp = O.bifocal_rows(q[:L], k[:L], v[:L], L, pos, np.arange(hq), w0=w0, w_pretrained=w_pre,
                                rope_base=base, plain=True)
        np.testing.assert_allclose(od, op, atol=1e-12)


def test_decode_does_not_modify_inputs():
    d, hq, hkv, L = 8, 2, 1, 30
    q = _rand((hq, d), 1)
    kc = _rand((L, hkv, d), 2)
    v = _rand((L, hkv, d), 3)
    before = (q.copy(), kc.copy(), v.copy())
    O.decode_step(q, kc, v, L, w0=4, w_pretrained=8, rope_base=1e4)
    for a, b in zip(before, (q, kc, v)):
        np.testing.assert_array_equal(a, b)


# ------------------------------------------ planted mistakes are caught ----

def _mutant(kind, q, k, v, L, w0, w_pre, base):
    """A brute-force variant with one plausible mistake planted (CPU only)."""
    d = q.shape[-1]
    h = d // 2
    G = brute.group_size(L, w_pre)
    if kind == "floor_G":
        G = max(1, L // w_pre)
    pos = np.arange(L)

    def rot(x, p):
        if kind == "conjugate":
            return brute.rotate_complex(x, -p, base)
        if kind == "interleaved":
            y = x.copy()
            th = base ** (-np.arange(0, d, 2) / d)
            z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * p[:, None] * th[None])
            y[:, 0::2], y[:, 1::2] = z.real, z.imag
            return y
        return brute.rotate_complex(x, p, base)

    sc = 1 / math.sqrt(d)
    sb = sc * rot(q, pos) @ rot(k, pos).T
    sr = sc * rot(q, pos // G) @ rot(k, pos // G).T
    dist = np.subtract.outer(pos, pos)
    local = (dist >= 0) & ((dist <= w0) if kind == "window_le" else (dist < w0))
    remote = (dist >= 0) & ~local
    S = np.where(local, sb, np.where(remote, sr, -np.inf))
    m = S.max(1, keepdims=True)
    P = np.exp(S - m)
    del h
    return (P / P.sum(1, keepdims=True)) @ v


@pytest.mark.parametrize("kind", ["conjugate", "interleaved", "window_le", "floor_G"])
def test_planted_mistakes_fail_the_pins(kind):
    L, w_pre, w0, d, base = 50, 16, 6, 16, 1e4
    q, k, v = _seq(L, 1, 1, d, 110)
    good = _mutant("none", q[:, 0], k[:, 0], v[:, 0], L, w0, w_pre, base)
    ob, _ = _rows(q, k, v, L, w0, w_pre, base)
    np.testing.assert_allclose(ob[:, 0], good, atol=1e-12)
    bad = _mutant(kind, q[:, 0], k[:, 0], v[:, 0], L, w0, w_pre, base)
    assert np.abs(bad - ob[:, 0]).max() > 1e-3, kind


# ------------------------------------------- frequency-interpolation variant ----

def test_interp_with_unit_factors_is_plain_rope_bit_for_bit():
    """lambda_c = 1: the remote rotation is the base rotation, so the variant is plain RoPE."""
    L, d = 60, 16
    q, k, v = _seq(L, 2, 1, d, 120)
    pos, head = _all_rows(L, 2)
    oi, li = O.interp_rows(q, k, v, L, pos, head, w0=7, rope_base=1e4, freq_scale=np.ones(d // 2))
    op, lp = O.bifocal_rows(q, k, v, L, pos, head, w0=7, w_pretrained=10 ** 6, rope_base=1e4, plain=True)
    np.testing.assert_array_equal(oi, op)
    np.testing.assert_array_equal(li, lp)


def test_interp_equals_lse_merge_of_library_softmaxes():
    """Local keys with base RoPE, remote keys with R'(p) (angle p theta_c lambda_c) via complex
    multiplication; merged on log-sum-exp, by torch SDPA with boolean masks."""
    L, d, base, w0 = 57, 16, 1e4, 9
    lam = np.linspace(0.25, 1.0, d // 2)  # a YaRN-like ramp
    q, k, v = _seq(L, 1, 1, d, 130)
    pos, head = _all_rows(L, 1)
    oi, li = O.interp_rows(q, k, v, L, pos, head, w0=w0, rope_base=base, freq_scale=lam)
    th = base ** (-np.arange(0, d, 2) / d)

    def rot(x, p, scale):
        z = (x[:, :d // 2] + 1j * x[:, d // 2:]) * np.exp(1j * p[:, None] * (th * scale)[None])
        return np.concatenate([z.real, z.imag], -1)

    p = np.arange(L).astype(np.float64)
    dist = np.subtract.outer(np.arange(L), np.arange(L))
    local, remote = (dist >= 0) & (dist < w0), dist >= w0
    o1, l1 = _sdpa(rot(q[:, 0], p, 1.0), rot(k[:, 0], p, 1.0), v[:, 0], local)
    o2, l2 = _sdpa(rot(q[:, 0], p, lam), rot(k[:, 0], p, lam), v[:, 0], remote)
    has2 = remote.any(1)
    lse = np.where(has2, np.logaddexp(l1, np.where(has2, l2, -np.inf)), l1)
    ref = np.exp(l1 - lse)[:, None] * o1 + np.where(has2, np.exp(np.where(has2, l2, 0) - lse), 0)[:, None] * \
        np.where(has2[:, None], o2, 0)
    np.testing.assert_allclose(oi, ref, atol=1e-12)
    np.testing.assert_allclose(li, lse, atol=1e-12)
