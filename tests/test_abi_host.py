"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/jetlong.h declares, and rejects bad arguments before
launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jetlong.h")


@pytest.fixture(scope="module")
def jlmod():
    from rope_context_extension_sm_b200 import build
    build.build()
    from rope_context_extension_sm_b200 import jetlong
    return jetlong


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(jl_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ["jl_rope_tables", "jl_bifocal_prefill", "jl_bifocal_decode", "jl_plain_prefill", "jl_plain_decode",
              "jl_last_error", "jl_group_size", "jl_sync_status", "jl_bifocal_decode_workspace_size"]:
        assert s in syms


def test_library_exports_every_declared_symbol(jlmod):
    lib = ctypes.CDLL(jlmod.LIB_PATH)
    for s in declared_symbols():
        assert hasattr(lib, s), s
    assert set(declared_symbols()) == set(jlmod.SIGNATURES), "binding and header disagree"


def test_group_size_matches_golden(jlmod):
    gold = os.path.join(ROOT, "tests", "golden", "group_size.txt")
    for line in open(gold):
        line = line.split("#")[0].strip()
        if line:
            L, w, G = (int(x) for x in line.split())
            assert jlmod.jl_group_size(L, w) == G
    assert jlmod.jl_group_size(10, 0) == -1


def _call_prefill(jlmod, **over):
    a = dict(q=16, k=16, v=16, cu=16, batch=1, T=256, max_seqlen=256, Hq=1, Hkv=1, d=64, w0=32, w_pre=64,
             cos=16, sin=16, n_tab=256, scale=0.0, out=16, lse=16, ws=None, ws_bytes=0, stream=None)
    a.update(over)
    return jlmod._lib.jl_bifocal_prefill(a["q"], a["k"], a["v"], a["cu"], a["batch"], a["T"], a["max_seqlen"],
                                         a["Hq"], a["Hkv"], a["d"], a["w0"], a["w_pre"], a["cos"], a["sin"],
                                         a["n_tab"], a["scale"], a["out"], a["lse"], a["ws"], a["ws_bytes"],
                                         a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(d=96), 2), (dict(Hq=3, Hkv=2), 1), (dict(w0=-1), 1), (dict(w_pre=0), 1), (dict(n_tab=100), 1),
    (dict(q=None), 1), (dict(q=24), 1), (dict(batch=-1), 1), (dict(T=-5), 1), (dict(T=1 << 31), 1),
    (dict(ws=16, ws_bytes=1000), 1), (dict(ws=24, ws_bytes=1 << 20), 1),
])
def test_prefill_rejects_bad_arguments_without_launching(jlmod, over, status):
    # the pointers are fake host addresses: a launch would fail, validation must stop first
    assert _call_prefill(jlmod, **over) == status
    assert jlmod.jl_last_error() != ""


def test_prefill_empty_batch_is_a_no_op(jlmod):
    assert _call_prefill(jlmod, batch=0) == 0
    assert _call_prefill(jlmod, T=0) == 0


def _call_decode(jlmod, **over):
    a = dict(q=16, k=16, v=16, sl=16, B=1, stride=1024, max_seqlen=1024, Hq=32, Hkv=8, d=128, w0=64, w_pre=256,
             cos=16, sin=16, n_tab=1024, scale=0.0, out=16, lse=16, ws=16, ws_bytes=1 << 30, stream=None)
    a.update(over)
    return jlmod._lib.jl_bifocal_decode(a["q"], a["k"], a["v"], a["sl"], a["B"], a["stride"], a["max_seqlen"],
                                        a["Hq"], a["Hkv"], a["d"], a["w0"], a["w_pre"], a["cos"], a["sin"],
                                        a["n_tab"], a["scale"], a["out"], a["lse"], a["ws"], a["ws_bytes"],
                                        a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(d=80), 2), (dict(Hq=34, Hkv=2), 2), (dict(Hq=30), 1), (dict(stride=512), 1), (dict(n_tab=10), 1),
    (dict(ws_bytes=10), 1), (dict(ws=None), 1), (dict(k=8), 1), (dict(max_seqlen=0), 1), (dict(w0=-3), 1),
])
def test_decode_rejects_bad_arguments_without_launching(jlmod, over, status):
    assert _call_decode(jlmod, **over) == status


def test_decode_workspace_size(jlmod):
    n = jlmod.jl_bifocal_decode_workspace_size(1, 32, 128, 131072)
    assert n > 0 and n % 16 == 0
    assert jlmod.jl_bifocal_decode_workspace_size(0, 32, 128, 131072) == 0


@pytest.mark.parametrize("B,Hq,L", [(1, 32, 131072), (2, 32, 65536), (1, 16, 8192), (4, 64, 4096), (1, 8, 300)])
def test_decode_workspace_covers_a_one_wave_split_for_every_kv_head_count(jlmod, B, Hq, L):
    # The tensor-core decode runs at most one wave of 148 CTAs (B x Hkv x splits), each
    # split a whole number of 128-key tiles; the size query does not know Hkv, so it has
    # to cover the largest split any Hkv allowed by Hq can produce, plus two 8-byte merge
    # counter words per (entry, KV head) after the partials.
    n = jlmod.jl_bifocal_decode_workspace_size(B, Hq, 128, L)
    tiles = -(-L // 128)
    for hkv in [h for h in range(1, Hq + 1) if Hq % h == 0 and Hq // h <= 16]:
        worst_split = min(tiles, max(1, 148 // (hkv * B)))
        assert n >= B * worst_split * Hq * (128 + 2) * 4 + B * hkv * 16, hkv


def test_prefill_and_cache_rejects_a_short_cache_without_launching(jlmod):
    lib = jlmod._lib
    # cache_stride below max_seqlen is refused before any pointer is touched or kernel launched
    st = lib.jl_bifocal_prefill_and_cache(None, None, None, None, 1, 100, 100, 4, 2, 128, 16, 64, None, None, 128,
                                          0.0, None, None, None, None, 99, None, 0, None)
    assert st == 1 and "cache_stride" in jlmod.jl_last_error()
    # an empty batch is a no-op, whatever the pointers
    assert lib.jl_bifocal_prefill_and_cache(None, None, None, None, 0, 0, 0, 4, 2, 128, 16, 64, None, None, 1,
                                            0.0, None, None, None, None, 1, None, 0, None) == 0
    assert lib.jl_bifocal_prefill_and_cache(None, None, None, None, 0, 0, 0, 4, 2, 128, 16, 64, None, None, 1,
                                            0.0, None, None, None, None, 1, 16, 1 << 20, None) == 0


def test_rope_tables_rejects_bad_arguments(jlmod):
    assert jlmod._lib.jl_rope_tables(16, 16, 0, 128, 1e4, None) == 1
    assert jlmod._lib.jl_rope_tables(16, 16, 10, 100, 1e4, None) == 2
    assert jlmod._lib.jl_rope_tables(None, 16, 10, 128, 1e4, None) == 1
    assert jlmod._lib.jl_rope_tables(16, 16, 10, 128, 0.5, None) == 1


def test_selftest_rejects_bad_limits(jlmod):
    assert jlmod._lib.jl_selftest_wait_timeout(10, None) == 1
    assert jlmod._lib.jl_selftest_wait_timeout(3_000_000_000, None) == 1


def test_prefill_workspace_size(jlmod):
    # two rotated key rows (base and remote) per token and KV head
    assert jlmod.jl_bifocal_prefill_workspace_size(131072, 8, 128) == 2 * 131072 * 8 * 128 * 2
    assert jlmod.jl_bifocal_prefill_workspace_size(0, 8, 128) == 0


def test_key_workspace_is_checked_before_any_launch(jlmod):
    """A key workspace too small or not 16-byte aligned is refused by every prefill entry
    point that takes one, before anything is launched (the pointers are fake host addresses)."""
    lib = jlmod._lib
    T, hkv, d = 256, 1, 64
    need = jlmod.jl_bifocal_prefill_workspace_size(T, hkv, d)
    for ws, nbytes in ((16, need - 16), (24, need)):
        st = lib.jl_bifocal_prefill_and_cache(16, 16, 16, 16, 1, T, T, 1, hkv, d, 32, 64, 16, 16, 256, 0.0, 16, 16,
                                              16, 16, 256, ws, nbytes, None)
        assert st == jlmod.JL_ERR_INVALID and "workspace" in jlmod.jl_last_error()
        st = lib.jl_interp_prefill(16, 16, 16, 16, 1, T, T, 1, hkv, d, 32, 16, 16, 256, 16, 16, 256, 0.0, 16, 16,
                                   ws, nbytes, None)
        assert st == jlmod.JL_ERR_INVALID and "workspace" in jlmod.jl_last_error()
        st = lib.jl_plain_prefill(16, 16, 16, 16, 1, T, T, 1, hkv, d, 16, 16, 256, 0.0, 16, 16, ws, nbytes, None)
        assert st == jlmod.JL_ERR_INVALID and "workspace" in jlmod.jl_last_error()
