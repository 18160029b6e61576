"""jl_bifocal_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (an engine plugin handed only its input and output
buffers, a serving loop that forbids cudaMalloc once running).  It uses the
library's static per-device scratch instead of a caller workspace; its output
must match jl_bifocal_decode's, call after call, even though the scratch keeps
the previous call's contents.

This file is collected last on purpose: a run that stops at the first failure
has already run every other test by the time it gets here.
"""
import numpy as np
import pytest
import torch

OUT_MAX, LSE_MAX = 2e-2, 1e-2


def _lib():
    from rope_context_extension_sm_b200 import build
    build.build()
    from rope_context_extension_sm_b200 import jetlong
    return jetlong


def test_noalloc_rejects_sizes_beyond_its_static_scratch():
    jl = _lib()
    cap = jl.jl_bifocal_decode_noalloc_scratch_bytes()
    assert cap > 0
    # B = 8 at 131072 needs ~8x the B = 1 scratch; validation stops before any CUDA call
    assert jl.jl_bifocal_decode_workspace_size(8, 32, 128, 131072) > cap
    st = jl._lib.jl_bifocal_decode_noalloc(16, 16, 16, 16, 8, 131072, 131072, 32, 8, 128, 4096, 32768, 16, 16,
                                           131072, 0.0, 16, 16, None)
    assert st == jl.JL_ERR_INVALID
    assert "static scratch" in jl.jl_last_error()
    assert jl.jl_bifocal_decode_workspace_size(1, 32, 128, 131072) <= cap


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    jl = _lib()
    from rope_context_extension_sm_b200 import inputs as I
    assert torch.cuda.is_available()
    dev = torch.device("cuda", 0)
    cfg = I.DECODE_QWEN3_4B
    max_len = 65536
    k_cache, v = I.decode_raw_inputs(cfg, max_len)  # random rows stand for base-rotated keys
    kd, vd = k_cache.to(dev), v.to(dev)
    qs = I.decode_queries(cfg, 2).to(dev)
    cos, sin = jl.jl_rope_tables(max_len, cfg.head_dim, cfg.rope_base, device=dev)
    # two calls in a row with different lengths (G = 2, then G = 1) and different queries
    for call, L in enumerate([65536, 9000]):
        sl = torch.tensor([L], dtype=torch.int32, device=dev)
        q = qs[call].contiguous()
        ref, ref_lse = jl.jl_bifocal_decode(q, kd, vd, sl, max_len, cfg.w0, cfg.w_pretrained, cos, sin)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((1, cfg.n_q_heads), float("nan"), dtype=torch.float32, device=dev)
        jl.jl_bifocal_decode_noalloc(q, kd, vd, sl, max_len, cfg.w0, cfg.w_pretrained, cos, sin, out=out, lse=lse)
        jl.jl_sync_status()
        got, want = out.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.isfinite(got).all(), f"call {call}"
        assert np.abs(got - want).max() <= OUT_MAX, f"call {call}: out differs"
        assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= LSE_MAX, f"call {call}: lse differs"


@pytest.mark.gpu
def test_noalloc_decode_head_dim_64_matches_workspace_decode():
    """head_dim 64 runs the CUDA-core split kernel: two calls in a row (G = 3, then G = 1)."""
    jl = _lib()
    from rope_context_extension_sm_b200 import inputs as I
    dev = torch.device("cuda", 0)
    cfg = I.DecodeConfig("noalloc_d64", (), 8, 2, 64, 100, 1024, 1e4)
    max_len = 3000
    k_cache, v = I.decode_raw_inputs(cfg, max_len)
    kd, vd = k_cache.to(dev), v.to(dev)
    qs = I.decode_queries(cfg, 2).to(dev)
    cos, sin = jl.jl_rope_tables(max_len, cfg.head_dim, cfg.rope_base, device=dev)
    for call, L in enumerate([3000, 700]):
        sl = torch.tensor([L], dtype=torch.int32, device=dev)
        q = qs[call].contiguous()
        ref, ref_lse = jl.jl_bifocal_decode(q, kd, vd, sl, max_len, cfg.w0, cfg.w_pretrained, cos, sin)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((1, cfg.n_q_heads), float("nan"), dtype=torch.float32, device=dev)
        jl.jl_bifocal_decode_noalloc(q, kd, vd, sl, max_len, cfg.w0, cfg.w_pretrained, cos, sin, out=out, lse=lse)
        jl.jl_sync_status()
        got, want = out.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.isfinite(got).all(), f"call {call}"
        assert np.abs(got - want).max() <= OUT_MAX, f"call {call}: out differs"
        assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= LSE_MAX, f"call {call}: lse differs"


@pytest.mark.gpu
def test_noalloc_rejects_a_query_outside_device_memory():
    """The static scratch is only valid on its own device, so the call checks that q is device
    memory of the current device (and that the stream is that device's) before launching."""
    jl = _lib()
    assert torch.cuda.is_available()
    torch.cuda.init()
    host_q = np.zeros((1, 32, 128), dtype=np.uint16)  # pageable host memory
    st = jl._lib.jl_bifocal_decode_noalloc(host_q.ctypes.data, 16, 16, 16, 1, 4096, 4096, 32, 8, 128, 64, 1024, 16,
                                           16, 4096, 0.0, 16, 16, None)
    assert st == jl.JL_ERR_INVALID
    assert "not device memory" in jl.jl_last_error()
