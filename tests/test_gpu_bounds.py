"""The debug-bounds build on the GPU: the same library compiled with
-DJL_DEBUG_BOUNDS (libjetlong_bounds.so) checks, on the device, every index its
kernels derive there (RoPE table rows, TMA tile coordinates, cache and page
positions, workspace slots) and records a failed check in the status word
instead of trapping.  The prefill runs both ways: keys rotated once into a
workspace (the default), and rotated by the prefill kernel itself.  Every product kernel runs here on small parity cases; each
must pass its oracle comparison with no check failing.  A paged decode given a
page index outside its pool (which the normal build reads as zeros) must be
reported.  This is the stand-in for a memory checker on this machine.
"""
import ctypes

import numpy as np
import pytest
import torch

import test_gpu_parity as P
from rope_context_extension_sm_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def jlb():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from rope_context_extension_sm_b200 import build
    build.build()
    path = build.build_bounds()
    from rope_context_extension_sm_b200 import jetlong
    lib = ctypes.CDLL(path)
    for name, (res, args) in jetlong.SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    assert lib.jl_debug_bounds_enabled() == 1
    saved = jetlong._lib
    jetlong._lib = lib
    try:
        yield jetlong
    finally:
        jetlong._lib = saved


@pytest.mark.parametrize("name", ["gqa4_G4_w0_100", "gqa4_G4_w0_0", "w0_covers_all", "G1_short", "varlen_ragged",
                                  "group3_d64", "d64_gqa2", "group3_d128_G4", "group3_d128_varlen",
                                  "group1_d128_w0_0"])
def test_bounds_build_prefill(jlb, name):
    case = next(c for c in P.SMALL if c[0] == name)
    _, seqlens, hq, hkv, d, w0, w_pre = case
    P._compare_all_rows(jlb, I.PrefillConfig(name, seqlens, hq, hkv, d, w0, w_pre, 1e4, True))


@pytest.mark.parametrize("name", ["gqa4_G4_w0_100", "varlen_ragged", "group3_d64", "group3_d128_G4"])
def test_bounds_build_prefill_in_kernel_key_rotation(jlb, name):
    """The path without a key workspace: the prefill kernel's rotation warps rotate the keys."""
    case = next(c for c in P.SMALL if c[0] == name)
    _, seqlens, hq, hkv, d, w0, w_pre = case
    P._compare_all_rows(jlb, I.PrefillConfig(name, seqlens, hq, hkv, d, w0, w_pre, 1e4, True), in_kernel=True)


def test_bounds_build_tiny_and_empty_sequences(jlb):
    P._compare_all_rows(jlb, I.TINY)
    P._compare_all_rows(jlb, I.PrefillConfig("with_empty", (0, 200, 0, 5), 2, 1, 128, 16, 64, 1e4, False))


@pytest.mark.parametrize("in_kernel", [False, True], ids=["key_workspace", "in_kernel_rotation"])
@pytest.mark.parametrize("case", P.PREFILL_AND_CACHE, ids=[c[0] for c in P.PREFILL_AND_CACHE])
def test_bounds_build_prefill_and_cache(jlb, case, in_kernel):
    P.test_prefill_and_cache_writes_the_base_rope_cache(jlb, case, in_kernel)


def test_bounds_build_chunked_three_pass_interp(jlb):
    P.test_chunked_prefill_single_sequence_across_G(jlb)
    P.test_chunked_prefill_d64_group3(jlb)
    P.test_chunked_prefill_d128_group3(jlb)
    P.test_three_pass_merge_on_gpu(jlb, P.THREE_PASS[0])
    P.test_interp_prefill_matches_oracle(jlb, P.INTERP[1], False)
    P.test_interp_prefill_matches_oracle(jlb, P.INTERP[1], True)


@pytest.mark.parametrize("case", [c for c in P.DECODE_GROUPS if c[0] in ("d64_g3", "d64_g16", "d128_g3")],
                         ids=lambda c: c[0])
@pytest.mark.parametrize("L", [1, 101, 257])
def test_bounds_build_decode(jlb, case, L):
    P.test_decode_head_dims_and_groups(jlb, case, L)


def test_bounds_build_batched_and_paged_decode(jlb):
    P.test_batched_decode_each_sequence_its_own_G(jlb)
    P.test_decode_d64_batched_and_long(jlb, 6, 2)
    P.test_paged_decode_equals_contiguous_and_oracle(jlb)
    P.test_streaming_decode_from_raw_tokens_across_G_boundary(jlb)


def test_bounds_build_reports_a_page_outside_the_pool(jlb):
    """A block table that points past the page pool: the normal build reads that page as zeros
    (the TMA load is bounded by the pool), the bounds build also reports it."""
    cfg = P.SMALL_DECODE
    lens, page, max_len = [1000], 256, 1024
    k_cache, v = P._decode_setup(cfg, max_len)
    q_t = P._query_tilde(cfg, I.decode_queries(cfg, 1)[0, 0], lens[0])[None]
    cos, sin = P._tables(jlb, max_len, 128, cfg.rope_base)
    kp, table = P._paginate(k_cache, lens, page)
    vp, _ = P._paginate(v, lens, page)
    bad = table.clone()
    bad[0, 1] = kp.shape[0] + 5
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    jlb.jl_bifocal_decode_paged(q_t.cuda(), kp.cuda(), vp.cuda(), bad.cuda(), sl, max_len, cfg.w0, cfg.w_pretrained,
                                cos, sin)
    with pytest.raises(jlb.JetLongError) as err:
        jlb.jl_sync_status()
    assert err.value.status == jlb.JL_ERR_INVALID
    assert "debug-bounds" in jlb.jl_last_error()
    jlb.jl_sync_status()  # cleared
