"""The single-launch decode build on the GPU: libjetlong_lastcta.so, compiled with
-DJL_DECODE_LAST_CTA_MERGE=1, merges the split partials of each (entry, KV head) in
the last of its split CTAs, found through atomic tickets on counter words in the
workspace, instead of in a second kernel.  The decode cases of the parity suite run
on it: the oracle comparisons, a workspace of random bytes (counter words with
arbitrary contents), more CTAs than one wave, entries with one active split, and a
CUDA graph replayed across G changes (the counters must be clear after every call).
"""
import ctypes

import pytest
import torch

import test_gpu_parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def jll():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from rope_context_extension_sm_b200 import build
    build.build()
    path = build.build_last_cta()
    from rope_context_extension_sm_b200 import jetlong
    lib = ctypes.CDLL(path)
    for name, (res, args) in jetlong.SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    assert lib.jl_decode_single_launch_enabled() == 1
    saved = jetlong._lib
    jetlong._lib = lib
    try:
        yield jetlong
    finally:
        jetlong._lib = saved


@pytest.mark.parametrize("L", [1, 2, 100, 257, 700, 1024])
def test_last_cta_small_decode_steps(jll, L):
    P.test_small_decode_steps(jll, L)


@pytest.mark.parametrize("case", [c for c in P.DECODE_GROUPS if c[3] == 128], ids=lambda c: c[0])
@pytest.mark.parametrize("L", [1, 101, 257])
def test_last_cta_decode_groups(jll, case, L):
    P.test_decode_head_dims_and_groups(jll, case, L)


def test_last_cta_workspace_of_random_bytes(jll):
    P.test_decode_workspace_of_random_bytes(jll)


def test_last_cta_more_ctas_than_one_wave(jll):
    P.test_batched_decode_more_ctas_than_one_wave(jll)


def test_last_cta_batched_each_sequence_its_own_G(jll):
    P.test_batched_decode_each_sequence_its_own_G(jll)


def test_last_cta_graph_replay_across_G(jll):
    P.test_decode_replayed_from_a_cuda_graph_follows_the_device_lengths(jll)


@pytest.mark.parametrize("L", [8192, 131072])
def test_last_cta_qwen3_4b(jll, L):
    P.test_decode_qwen3_4b_cache_lengths(jll, L)
