"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on the
same seeded bf16 inputs.

Acceptance (bf16 inputs, fp32 accumulation): output max-abs <= 2e-2, output
mean-abs <= 2e-3, LSE max-abs <= 1e-2.  Small cases compare every row; the
model-sized cases compare sampled rows plus the critical rows (window edge,
pretraining-window edge, tile edges, last rows).
"""
import numpy as np
import pytest
import torch

import _headroom
from oracle import oracle as O
from rope_context_extension_sm_b200 import inputs as I

pytestmark = pytest.mark.gpu

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-2


@pytest.fixture(scope="module")
def jl():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    from rope_context_extension_sm_b200 import build
    build.build()
    from rope_context_extension_sm_b200 import jetlong
    return jetlong


def _tables(jl, n, d, base):
    return jl.jl_rope_tables(n, d, base)


def _check(got_out, got_lse, ref_out, ref_lse, what):
    err = np.abs(got_out.astype(np.float64) - ref_out)
    lerr = np.abs(got_lse.astype(np.float64) - ref_lse)
    assert np.isfinite(got_out).all() and np.isfinite(got_lse).all(), what
    assert err.max() <= OUT_MAX, f"{what}: out max-abs {err.max():.3e}"
    assert err.mean() <= OUT_MEAN, f"{what}: out mean-abs {err.mean():.3e}"
    assert lerr.max() <= LSE_MAX, f"{what}: lse max-abs {lerr.max():.3e}"
    _headroom.record(what, err.max(), err.mean(), lerr.max())
    return err.max(), err.mean(), lerr.max()


def _prefill_gpu(jl, q, k, v, cu, cfg, plain=False, in_kernel=False):
    """in_kernel: the prefill kernel rotates the keys itself (no key workspace); otherwise
    the keys are rotated once into a workspace before it (the default path)."""
    dev = "cuda"
    qd, kd, vd, cud = q.to(dev), k.to(dev), v.to(dev), cu.to(dev)
    cos, sin = _tables(jl, max(cfg.max_seqlen, 1), cfg.head_dim, cfg.rope_base)
    if plain:
        out, lse = jl.jl_plain_prefill(qd, kd, vd, cud, cfg.max_seqlen, cos, sin, rotate_keys_in_kernel=in_kernel)
    else:
        out, lse = jl.jl_bifocal_prefill(qd, kd, vd, cud, cfg.max_seqlen, cfg.w0, cfg.w_pretrained, cos, sin,
                                         rotate_keys_in_kernel=in_kernel)
    jl.jl_sync_status()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _oracle_rows(q, k, v, cu, cfg, seq, rows, heads, plain=False):
    s0, s1 = int(cu[seq]), int(cu[seq + 1])
    qb, kb, vb = I.bf16_bits(q[s0:s1]), I.bf16_bits(k[s0:s1]), I.bf16_bits(v[s0:s1])
    return O.bifocal_rows(qb, kb, vb, s1 - s0, rows, heads, w0=cfg.w0, w_pretrained=cfg.w_pretrained,
                          rope_base=cfg.rope_base, plain=plain)


def _compare_all_rows(jl, cfg, plain=False, in_kernel=False):
    q, k, v, cu = I.prefill_inputs(cfg)
    out, lse = _prefill_gpu(jl, q, k, v, cu, cfg, plain, in_kernel)
    for s in range(len(cfg.seqlens)):
        L = cfg.seqlens[s]
        if L == 0:
            continue
        pos = np.repeat(np.arange(L), cfg.n_q_heads)
        head = np.tile(np.arange(cfg.n_q_heads), L)
        ro, rl = _oracle_rows(q, k, v, cu, cfg, s, pos, head, plain)
        s0 = int(cu[s])
        _check(out[s0 + pos, head], lse[head, s0 + pos], ro, rl,
               f"{cfg.name} seq {s}" + (" (in-kernel key rotation)" if in_kernel else ""))
    return out, lse


# ------------------------------------------------------------------ tables ----

@pytest.mark.parametrize("n,d,base", [(256, 64, 1e4), (131072, 128, 1e6)])
def test_rope_tables_match_fp64_rounded_once(jl, n, d, base):
    """fp32 tables = fp64 cos/sin rounded once.  The device's fp64 pow/sincos and the
    host's agree to ~1e-11 rad at p ~ 1.3e5, so compare absolutely: within half an fp32
    ulp at magnitude 1 (2^-25) plus that slack, and bit-equal for almost every entry."""
    cos, sin = _tables(jl, n, d, base)
    jl.jl_sync_status()
    rc, rs = O.rope_cos_sin(n, d, base)
    for got, ref in ((cos, rc), (sin, rs)):
        g = got.cpu().numpy().astype(np.float64)
        assert np.abs(g - ref).max() <= 2.0 ** -25 + 1e-9
        assert (g != ref.astype(np.float32)).mean() < 1e-3


# --------------------------------------------------------- failure detection ----

def test_bounded_wait_reports_timeout_and_context_stays_usable(jl):
    """A wait that nothing completes ends after its limit with JL_ERR_TIMEOUT (no trap,
    no hang); jl_sync_status reports and clears it; the context keeps working."""
    jl.jl_selftest_wait_timeout(2_000_000)
    with pytest.raises(jl.JetLongError) as err:
        jl.jl_sync_status()
    assert err.value.status == jl.JL_ERR_TIMEOUT
    jl.jl_sync_status()  # cleared
    _compare_all_rows(jl, I.TINY)


# ----------------------------------------------------------------- prefill ----

def test_tiny_prefill_all_rows(jl):
    """L = 256, d = 64, G = 4, w0 = 32: every row against the oracle."""
    _compare_all_rows(jl, I.TINY)


def test_tiny_plain_prefill_all_rows(jl):
    _compare_all_rows(jl, I.TINY, plain=True)


def test_tiny_prefill_in_kernel_key_rotation(jl):
    """The path without a key workspace: the prefill kernel rotates every key tile itself."""
    _compare_all_rows(jl, I.TINY, in_kernel=True)
    _compare_all_rows(jl, I.TINY, plain=True, in_kernel=True)


SMALL = [
    # name, seqlens, Hq, Hkv, d, w0, w_pre
    ("gqa4_G4_w0_100", (1000,), 8, 2, 128, 100, 256),
    ("gqa4_G4_w0_0", (1000,), 8, 2, 128, 0, 256),
    ("gqa4_G4_w0_1", (1000,), 8, 2, 128, 1, 256),
    ("gqa4_G4_w0_127", (777,), 4, 1, 128, 127, 200),
    ("gqa4_G4_w0_128", (777,), 4, 1, 128, 128, 200),
    ("gqa4_G4_w0_129", (777,), 4, 1, 128, 129, 200),
    ("gqa2_G3_w0_300", (700,), 4, 2, 128, 300, 256),
    ("w0_covers_all", (600,), 4, 2, 128, 5000, 100),
    ("G1_short", (300,), 4, 2, 128, 64, 512),
    ("varlen_ragged", (1, 130, 257, 700, 64, 129), 4, 2, 128, 50, 128),
    ("group3_d64", (500,), 3, 1, 64, 40, 100),
    ("group1_d128", (384,), 2, 2, 128, 64, 100),
    # odd groups at head_dim 128 run the one-head double-buffered kernel
    ("group3_d128_G4", (1000,), 6, 2, 128, 100, 256),
    ("group1_d128_G5_w0_129", (600,), 3, 3, 128, 129, 128),
    ("group3_d128_varlen", (1, 130, 257, 700, 0, 64), 3, 1, 128, 50, 128),
    ("group1_d128_w0_0", (500,), 2, 2, 128, 0, 128),
    ("group3_d128_w0_covers", (300,), 3, 1, 128, 5000, 100),
    ("d64_gqa2", (450,), 4, 2, 64, 33, 64),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_prefill_all_rows(jl, case):
    name, seqlens, hq, hkv, d, w0, w_pre = case
    cfg = I.PrefillConfig(name, seqlens, hq, hkv, d, w0, w_pre, 1e4, True)
    _compare_all_rows(jl, cfg)


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_prefill_in_kernel_key_rotation(jl, case):
    name, seqlens, hq, hkv, d, w0, w_pre = case
    cfg = I.PrefillConfig(name, seqlens, hq, hkv, d, w0, w_pre, 1e4, True)
    _compare_all_rows(jl, cfg, in_kernel=True)


def test_prefill_key_workspace_contents_do_not_matter(jl):
    """A key workspace full of random bytes and one of zeros give the same result, bit for
    bit: every row the kernel reads is written by the key rotation first (the remote rows
    of a G = 1 sequence are neither written nor read)."""
    cfg = I.PrefillConfig("ws_garbage", (700, 64, 300), 8, 2, 128, 100, 256, 1e4, True)
    q, k, v, cu = I.prefill_inputs(cfg)
    dev = "cuda"
    qd, kd, vd, cud = q.to(dev), k.to(dev), v.to(dev), cu.to(dev)
    cos, sin = _tables(jl, cfg.max_seqlen, cfg.head_dim, cfg.rope_base)
    n = jl.jl_bifocal_prefill_workspace_size(qd.shape[0], cfg.n_kv_heads, cfg.head_dim)
    gen = torch.Generator(device="cpu").manual_seed(3)
    results = []
    for ws in (torch.randint(0, 256, (n,), dtype=torch.uint8, generator=gen).to(dev),
               torch.zeros(n, dtype=torch.uint8, device=dev)):
        out, lse = jl.jl_bifocal_prefill(qd, kd, vd, cud, cfg.max_seqlen, cfg.w0, cfg.w_pretrained, cos, sin,
                                         workspace=ws)
        jl.jl_sync_status()
        results.append((out.clone(), lse.clone()))
    assert torch.equal(results[0][0], results[1][0]) and torch.equal(results[0][1], results[1][1])


def test_short_input_gpu_bifocal_equals_plain_bitwise(jl):
    """L <= w_pretrained (G = 1): the kernel takes the plain path, so the outputs are identical."""
    cfg = I.PrefillConfig("G1", (900,), 8, 2, 128, 100, 1024, 1e6, True)
    q, k, v, cu = I.prefill_inputs(cfg)
    ob, lb = _prefill_gpu(jl, q, k, v, cu, cfg)
    op, lp = _prefill_gpu(jl, q, k, v, cu, cfg, plain=True)
    np.testing.assert_array_equal(ob, op)
    np.testing.assert_array_equal(lb, lp)


def test_empty_and_zero_length_sequences(jl):
    cfg = I.PrefillConfig("with_empty", (0, 200, 0, 5), 2, 1, 128, 16, 64, 1e4, False)
    _compare_all_rows(jl, cfg)


def _critical_rows(L, w0, w_pre, extra_seed, n_random):
    rows = {0, 1, 2, 126, 127, 128, 129, w0 - 2, w0 - 1, w0, w0 + 1, w0 + 127, w0 + 128, w_pre - 1, w_pre,
            w_pre + 1, L - 129, L - 128, L - 2, L - 1}
    rng = np.random.default_rng(extra_seed)
    rows |= set(rng.integers(0, L, n_random).tolist())
    return sorted(r for r in rows if 0 <= r < L)


def _compare_sampled(jl, cfg, n_random=24, heads_per_row=4, seed=11, in_kernel=False):
    q, k, v, cu = I.prefill_inputs(cfg)
    out, lse = _prefill_gpu(jl, q, k, v, cu, cfg, in_kernel=in_kernel)
    rng = np.random.default_rng(seed)
    worst = (0.0, 0.0, 0.0)
    for s in range(len(cfg.seqlens)):
        L = cfg.seqlens[s]
        rows = _critical_rows(L, cfg.w0, cfg.w_pretrained, seed + s, n_random)
        pos, head = [], []
        for r in rows:
            hs = rng.choice(cfg.n_q_heads, size=min(heads_per_row, cfg.n_q_heads), replace=False)
            pos += [r] * len(hs)
            head += hs.tolist()
        pos, head = np.array(pos), np.array(head)
        ro, rl = _oracle_rows(q, k, v, cu, cfg, s, pos, head)
        s0 = int(cu[s])
        e = _check(out[s0 + pos, head], lse[head, s0 + pos], ro, rl, f"{cfg.name} seq {s}")
        worst = tuple(max(a, b) for a, b in zip(worst, e))
    assert np.isfinite(out).all()
    return worst


@pytest.mark.parametrize("w0", I.W0_SWEEP)
def test_qwen3_1p7b_64k_sampled_rows(jl, w0):
    _compare_sampled(jl, I.with_(I.QWEN3_1P7B, w0=w0), n_random=12 if w0 != 4096 else 24)


def test_qwen3_8b_128k_sampled_rows(jl):
    _compare_sampled(jl, I.QWEN3_8B_128K, n_random=24)


def test_qwen3_8b_128k_sampled_rows_in_kernel_key_rotation(jl):
    _compare_sampled(jl, I.QWEN3_8B_128K, n_random=12, in_kernel=True)


@pytest.mark.parametrize("L", [32768, 32769])
def test_group_boundary_32768(jl, L):
    """G jumps from 1 to 2 between L = 32768 and L = 32769."""
    _compare_sampled(jl, I.with_(I.QWEN3_8B_128K, seqlens=(L,)), n_random=8)


def test_varlen_sampled_rows(jl):
    _compare_sampled(jl, I.VARLEN, n_random=6, heads_per_row=2)


# ------------------------------------------------------------------ decode ----

def _decode_setup(cfg, max_len, batch=1):
    """Raw keys -> base-RoPE cache k~_j = bf16(R(j) k_j) (rotated by the oracle in fp64)."""
    k_raw, v = I.decode_raw_inputs(cfg, max_len, batch)
    d = cfg.head_dim
    kr = k_raw.float().numpy().reshape(batch, max_len, cfg.n_kv_heads, d)
    pos = np.broadcast_to(np.arange(max_len)[None, :, None], (batch, max_len, cfg.n_kv_heads)).reshape(-1)
    kc = O.rotate_rows(kr.reshape(-1, d), pos, cfg.rope_base).reshape(batch, max_len, cfg.n_kv_heads, d)
    k_cache = torch.from_numpy(kc).to(torch.bfloat16)
    return k_cache, v


def _query_tilde(cfg, q_raw, L):
    """bf16(R(L-1) q) for q_raw [Hq][d] bf16."""
    qt = O.rotate_rows(q_raw.float().numpy(), np.full(q_raw.shape[0], L - 1), cfg.rope_base)
    return torch.from_numpy(qt).to(torch.bfloat16)


def _decode_oracle(cfg, q_t, k_cache_b, v_b, L, plain=False):
    return O.decode_step(I.bf16_bits(q_t), I.bf16_bits(k_cache_b[:L]), I.bf16_bits(v_b[:L]), L, w0=cfg.w0,
                         w_pretrained=cfg.w_pretrained, rope_base=cfg.rope_base, plain=plain)


def _run_decode(jl, cfg, q_t, k_cache_d, v_d, seqlens, max_len, cos, sin, plain=False):
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    if plain:
        out, lse = jl.jl_plain_decode(q_t.cuda(), k_cache_d, v_d, sl, max_len, cos, sin)
    else:
        out, lse = jl.jl_bifocal_decode(q_t.cuda(), k_cache_d, v_d, sl, max_len, cfg.w0, cfg.w_pretrained, cos,
                                        sin)
    jl.jl_sync_status()
    return out.float().cpu().numpy(), lse.cpu().numpy()


SMALL_DECODE = I.DecodeConfig("small_decode", (), 8, 2, 128, 100, 256, 1e4)


@pytest.mark.parametrize("L", [1, 2, 100, 101, 255, 256, 257, 700, 1000, 1024])
def test_small_decode_steps(jl, L):
    cfg = SMALL_DECODE
    max_len = 1024
    k_cache, v = _decode_setup(cfg, max_len)
    q_raw = I.decode_queries(cfg, 1)[0, 0]
    q_t = _query_tilde(cfg, q_raw, L)
    cos, sin = _tables(jl, max_len, cfg.head_dim, cfg.rope_base)
    out, lse = _run_decode(jl, cfg, q_t[None], k_cache.cuda(), v.cuda(), [L], max_len, cos, sin)
    ro, rl = _decode_oracle(cfg, q_t, k_cache[0], v[0], L)
    _check(out[0], lse[0], ro, rl, f"decode L={L}")
    out, lse = _run_decode(jl, cfg, q_t[None], k_cache.cuda(), v.cuda(), [L], max_len, cos, sin, plain=True)
    ro, rl = _decode_oracle(cfg, q_t, k_cache[0], v[0], L, plain=True)
    _check(out[0], lse[0], ro, rl, f"plain decode L={L}")


DECODE_GROUPS = [
    # name, Hq, Hkv, head_dim: head_dim 64 runs the CUDA-core split kernel, 128 the tensor-core one;
    # groups between the built capacities (1, 2, 4, 8, 16) run in the next capacity up
    ("d64_g1", 2, 2, 64),
    ("d64_g2", 4, 2, 64),
    ("d64_g3", 6, 2, 64),
    ("d64_g4", 8, 2, 64),
    ("d64_g8", 8, 1, 64),
    ("d64_g16", 16, 1, 64),
    ("d128_g3", 6, 2, 128),
    ("d128_g12", 12, 1, 128),
]


@pytest.mark.parametrize("case", DECODE_GROUPS, ids=[c[0] for c in DECODE_GROUPS])
@pytest.mark.parametrize("L", [1, 100, 101, 255, 256, 257])
def test_decode_head_dims_and_groups(jl, case, L):
    """Bifocal and plain decode against the oracle for every decode kernel and GQA shape:
    w0 = 40, w_pretrained = 64, so these lengths give G = 1, 2, 2, 4, 4, 5."""
    name, hq, hkv, d = case
    cfg = I.DecodeConfig(name, (), hq, hkv, d, 40, 64, 1e4)
    max_len = 300
    k_cache, v = _decode_setup(cfg, max_len)
    q_t = _query_tilde(cfg, I.decode_queries(cfg, 1)[0, 0], L)
    cos, sin = _tables(jl, max_len, d, cfg.rope_base)
    for plain in (False, True):
        out, lse = _run_decode(jl, cfg, q_t[None], k_cache.cuda(), v.cuda(), [L], max_len, cos, sin, plain=plain)
        ro, rl = _decode_oracle(cfg, q_t, k_cache[0], v[0], L, plain=plain)
        _check(out[0], lse[0], ro, rl, f"{name} {'plain' if plain else 'bifocal'} decode L={L}")


@pytest.mark.parametrize("hq,hkv", [(8, 2), (6, 2)])
def test_decode_d64_batched_and_long(jl, hq, hkv):
    """head_dim 64 (CUDA-core kernel): a batch whose entries each have their own G, with a cache
    long enough that the split size grows past its minimum (20000 keys: 128-key chunks)."""
    cfg = I.DecodeConfig("d64_batch", (), hq, hkv, 64, 100, 1024, 1e4)
    max_len, lens = 20000, [20000, 1024, 1025, 7, 5000]
    k_cache, v = _decode_setup(cfg, max_len, batch=len(lens))
    qs = I.decode_queries(cfg, 1, batch=len(lens))[0]
    q_t = torch.stack([_query_tilde(cfg, qs[b], lens[b]) for b in range(len(lens))])
    cos, sin = _tables(jl, max_len, 64, cfg.rope_base)
    out, lse = _run_decode(jl, cfg, q_t, k_cache.cuda(), v.cuda(), lens, max_len, cos, sin)
    for b, L in enumerate(lens):
        ro, rl = _decode_oracle(cfg, q_t[b], k_cache[b], v[b], L)
        _check(out[b], lse[b], ro, rl, f"d64 batched decode b={b} L={L} G={O.group_size(L, 1024)}")


def test_decode_refuses_more_than_16_heads_per_kv_head(jl):
    cfg = I.DecodeConfig("g32", (), 32, 1, 128, 40, 64, 1e4)
    k_cache, v = _decode_setup(cfg, 64)
    cos, sin = _tables(jl, 64, 128, cfg.rope_base)
    q = torch.zeros((1, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(jl.JetLongError) as err:
        _run_decode(jl, cfg, q, k_cache.cuda(), v.cuda(), [64], 64, cos, sin)
    assert err.value.status == jl.JL_ERR_UNSUPPORTED


def test_decode_replayed_from_a_cuda_graph_follows_the_device_lengths(jl):
    # The decode entry point reads the lengths (and so G) only on the device, so one captured
    # call serves every step: replaying it after the lengths change must give the eager result
    # for the new lengths, bit for bit, crossing G = 4 -> 5 at L = 1024 -> 1025.
    cfg = SMALL_DECODE
    max_len = 1100
    k_cache, v = _decode_setup(cfg, max_len)
    kd, vd = k_cache.cuda(), v.cuda()
    cos, sin = _tables(jl, max_len, cfg.head_dim, cfg.rope_base)
    q_raw = I.decode_queries(cfg, 1)[0, 0]
    sl = torch.tensor([1024], dtype=torch.int32, device="cuda")
    qd = _query_tilde(cfg, q_raw, 1024)[None].cuda().contiguous()
    out = torch.empty_like(qd)
    lse = torch.empty((1, cfg.n_q_heads), dtype=torch.float32, device="cuda")
    ws = torch.empty(jl.jl_bifocal_decode_workspace_size(1, cfg.n_q_heads, cfg.head_dim, max_len),
                     dtype=torch.uint8, device="cuda")

    def step():
        jl.jl_bifocal_decode(qd, kd, vd, sl, max_len, cfg.w0, cfg.w_pretrained, cos, sin, out=out, lse=lse,
                             workspace=ws)

    step()  # one-time setup outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for L in (1024, 1025, 700):
        sl.fill_(L)
        qd.copy_(_query_tilde(cfg, q_raw, L)[None].cuda())
        g.replay()
        torch.cuda.synchronize()
        got_out, got_lse = out.clone(), lse.clone()
        step()
        jl.jl_sync_status()
        assert torch.equal(got_out, out) and torch.equal(got_lse, lse), f"graph replay differs at L={L}"
        ro, rl = _decode_oracle(cfg, _query_tilde(cfg, q_raw, L), k_cache[0], v[0], L)
        _check(got_out.float().cpu().numpy()[0], got_lse.cpu().numpy()[0], ro, rl, f"graph decode L={L}")
    del g


def test_decode_workspace_of_random_bytes(jl):
    """The last CTA of each (entry, KV head) merges the split partials; it is found through
    counter words in the workspace that carry a per-call tag.  A workspace full of random
    bytes (counter words with arbitrary tags and counts) must give the oracle's result, and
    so must a second call on the same workspace and a call after the words were zeroed."""
    cfg = SMALL_DECODE
    max_len, L = 1024, 1000  # 8 splits of one 128-key tile per KV head
    k_cache, v = _decode_setup(cfg, max_len)
    kd, vd = k_cache.cuda(), v.cuda()
    cos, sin = _tables(jl, max_len, cfg.head_dim, cfg.rope_base)
    q_t = _query_tilde(cfg, I.decode_queries(cfg, 1)[0, 0], L)
    qd = q_t[None].cuda().contiguous()
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    n = jl.jl_bifocal_decode_workspace_size(1, cfg.n_q_heads, cfg.head_dim, max_len)
    gen = torch.Generator(device="cpu").manual_seed(7)
    ws = torch.randint(0, 256, (n,), dtype=torch.uint8, generator=gen).cuda()
    ro, rl = _decode_oracle(cfg, q_t, k_cache[0], v[0], L)
    first = None
    for call in ("random", "again", "zeroed"):
        if call == "zeroed":
            ws.zero_()
        out, lse = jl.jl_bifocal_decode(qd, kd, vd, sl, max_len, cfg.w0, cfg.w_pretrained, cos, sin, workspace=ws)
        jl.jl_sync_status()
        got = (out.float().cpu().numpy()[0], lse.cpu().numpy()[0])
        _check(got[0], got[1], ro, rl, f"decode, workspace {call}")
        if first is None:
            first = got
        else:
            assert np.array_equal(first[0], got[0]) and np.array_equal(first[1], got[1]), call


def test_batched_decode_more_ctas_than_one_wave(jl):
    """10 entries x 8 KV heads x 2 splits = 160 CTAs on 148 SMs: the split CTAs of one (entry,
    KV head) can run in different waves, and entries no longer than the split size (16384
    keys) have one active split, which is then its own last CTA.  Random rows stand for the
    base-rotated keys (the decode only reads the cache)."""
    cfg = I.DecodeConfig("wave", (), 32, 8, 128, 1024, 4096, 1e6)
    lens = [20000, 19000, 300, 16385, 129, 20000, 8000, 16384, 1, 12345]
    max_len = 20000
    k_cache, v = I.decode_raw_inputs(cfg, max_len, len(lens))
    qs = I.decode_queries(cfg, 1, batch=len(lens))[0]
    q_t = torch.stack([_query_tilde(cfg, qs[b], lens[b]) for b in range(len(lens))])
    cos, sin = _tables(jl, max_len, cfg.head_dim, cfg.rope_base)
    out, lse = _run_decode(jl, cfg, q_t, k_cache.cuda(), v.cuda(), lens, max_len, cos, sin)
    for b, L in enumerate(lens):
        ro, rl = _decode_oracle(cfg, q_t[b], k_cache[b], v[b], L)
        _check(out[b], lse[b], ro, rl, f"multi-wave decode b={b} L={L} G={O.group_size(L, 4096)}")


def test_batched_decode_each_sequence_its_own_G(jl):
    cfg = SMALL_DECODE
    max_len, lens = 1024, [1024, 250, 513, 7]
    k_cache, v = _decode_setup(cfg, max_len, batch=len(lens))
    qs = I.decode_queries(cfg, 1, batch=len(lens))[0]
    q_t = torch.stack([_query_tilde(cfg, qs[b], lens[b]) for b in range(len(lens))])
    cos, sin = _tables(jl, max_len, cfg.head_dim, cfg.rope_base)
    out, lse = _run_decode(jl, cfg, q_t, k_cache.cuda(), v.cuda(), lens, max_len, cos, sin)
    for b, L in enumerate(lens):
        ro, rl = _decode_oracle(cfg, q_t[b], k_cache[b], v[b], L)
        _check(out[b], lse[b], ro, rl, f"batched decode b={b} L={L}")


@pytest.mark.parametrize("L", I.DECODE_QWEN3_4B.cache_lens)
def test_decode_qwen3_4b_cache_lengths(jl, L):
    cfg = I.DECODE_QWEN3_4B
    k_cache, v = _decode_setup(cfg, L)
    q_raw = I.decode_queries(cfg, 1)[0, 0]
    q_t = _query_tilde(cfg, q_raw, L)
    cos, sin = _tables(jl, L, cfg.head_dim, cfg.rope_base)
    kd, vd = k_cache.cuda(), v.cuda()
    before = (kd.view(torch.int16).sum(dtype=torch.int64).item(), vd.view(torch.int16).sum(dtype=torch.int64).item())
    out, lse = _run_decode(jl, cfg, q_t[None], kd, vd, [L], L, cos, sin)
    after = (kd.view(torch.int16).sum(dtype=torch.int64).item(), vd.view(torch.int16).sum(dtype=torch.int64).item())
    assert before == after, "the cache must not be written"
    ro, rl = _decode_oracle(cfg, q_t, k_cache[0], v[0], L)
    _check(out[0], lse[0], ro, rl, f"decode Qwen3-4B L={L}")


def test_decode_walk_across_G_boundary(jl):
    """Generation across L = 98304 -> 98305 (G 3 -> 4) with no cache rewrite: every one of the
    256 steps of the walk (query positions 98176 .. 98431) against the oracle.  The cache is
    rotated once; each step reads its prefix.  The GPU steps run first (each output kept), then
    the oracle checks them one by one."""
    cfg = I.DECODE_QWEN3_4B
    first, steps = cfg.walk_first_pos, cfg.walk_steps
    max_len = first + steps
    k_cache, v = _decode_setup(cfg, max_len)
    qs = I.decode_queries(cfg, steps)
    cos, sin = _tables(jl, max_len, cfg.head_dim, cfg.rope_base)
    kd, vd = k_cache.cuda(), v.cuda()
    kbits, vbits = I.bf16_bits(k_cache[0]), I.bf16_bits(v[0])
    results = []
    for t in range(steps):
        L = first + t + 1
        q_t = _query_tilde(cfg, qs[t, 0], L)
        out, lse = _run_decode(jl, cfg, q_t[None], kd, vd, [L], max_len, cos, sin)
        results.append((L, q_t, out[0], lse[0]))
    groups = set()
    for t, (L, q_t, out, lse) in enumerate(results):
        ro, rl = O.decode_step(I.bf16_bits(q_t), kbits[:L], vbits[:L], L, w0=cfg.w0,
                               w_pretrained=cfg.w_pretrained, rope_base=cfg.rope_base)
        G = O.group_size(L, cfg.w_pretrained)
        groups.add(G)
        _check(out, lse, ro, rl, f"walk step {t} (L={L}, G={G})")
    assert groups == {3, 4}


# ------------------------------------------------- KV cache writers (append) ----

def test_kv_cache_fill_writes_base_rope_keys(jl):
    """cache[b][p] = R(p) k (fp32 math, one bf16 rounding) and v copied, for packed varlen prompts."""
    cfg = I.PrefillConfig("fill", (300, 1, 129, 0, 64), 4, 2, 128, 32, 64, 1e4, True)
    q, k, v, cu = I.prefill_inputs(cfg)
    stride = 320
    kc = torch.zeros((len(cfg.seqlens), stride, 2, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    cos, sin = _tables(jl, stride, 128, cfg.rope_base)
    jl.jl_kv_cache_fill(k.cuda(), v.cuda(), cu.cuda(), cos, sin, kc, vc)
    jl.jl_sync_status()
    kc, vc = kc.cpu(), vc.cpu()
    for b, L in enumerate(cfg.seqlens):
        s0 = int(cu[b])
        if L == 0:
            continue
        pos = np.repeat(np.arange(L), 2)
        ref = O.rotate_rows(k[s0:s0 + L].float().numpy().reshape(-1, 128), pos, cfg.rope_base).reshape(L, 2, 128)
        got = kc[b, :L].float().numpy()
        np.testing.assert_allclose(got, ref, rtol=2.0 ** -7, atol=1e-6)
        assert torch.equal(vc[b, :L], v[s0:s0 + L])
        assert torch.count_nonzero(kc[b, L:]) == 0  # nothing written past the sequence


PREFILL_AND_CACHE = [
    ("varlen_G_to_10", (300, 1, 129, 0, 640), 4, 2, 128, 32, 64),
    ("G1_plain", (200,), 4, 2, 128, 32, 256),
    ("w0_0_writer_fallback", (300,), 4, 2, 128, 0, 64),
    ("d64_group3", (257, 70), 3, 1, 64, 16, 64),
    ("d128_group3", (257, 700), 3, 1, 128, 16, 64),
    ("d128_group1_w0_0", (300,), 2, 2, 128, 0, 64),
]


@pytest.mark.parametrize("in_kernel", [False, True], ids=["key_workspace", "in_kernel_rotation"])
@pytest.mark.parametrize("case", PREFILL_AND_CACHE, ids=[c[0] for c in PREFILL_AND_CACHE])
def test_prefill_and_cache_writes_the_base_rope_cache(jl, case, in_kernel):
    """Same attention as jl_bifocal_prefill on the same key path, bit for bit; the cache
    holds R(p) k (one bf16 rounding of fp32 math) and v for every position of every
    sequence, nothing beyond."""
    name, seqlens, hq, hkv, d, w0, w_pre = case
    cfg = I.PrefillConfig(name, seqlens, hq, hkv, d, w0, w_pre, 1e4, True)
    q, k, v, cu = I.prefill_inputs(cfg)
    stride = cfg.max_seqlen + 5
    kc = torch.zeros((len(seqlens), stride, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    cos, sin = _tables(jl, stride, d, cfg.rope_base)
    qd, kd, vd, cud = q.cuda(), k.cuda(), v.cuda(), cu.cuda()
    out, lse = jl.jl_bifocal_prefill_and_cache(qd, kd, vd, cud, cfg.max_seqlen, w0, w_pre, cos, sin, kc, vc,
                                               rotate_keys_in_kernel=in_kernel)
    ref_out, ref_lse = jl.jl_bifocal_prefill(qd, kd, vd, cud, cfg.max_seqlen, w0, w_pre, cos, sin,
                                             rotate_keys_in_kernel=in_kernel)
    jl.jl_sync_status()
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    kc, vc = kc.cpu(), vc.cpu()
    for b, L in enumerate(seqlens):
        s0 = int(cu[b])
        assert torch.count_nonzero(kc[b, L:]) == 0 and torch.count_nonzero(vc[b, L:]) == 0
        if L == 0:
            continue
        pos = np.repeat(np.arange(L), hkv)
        ref = O.rotate_rows(k[s0:s0 + L].float().numpy().reshape(-1, d), pos, cfg.rope_base).reshape(L, hkv, d)
        np.testing.assert_allclose(kc[b, :L].float().numpy(), ref, rtol=2.0 ** -7, atol=1e-6)
        assert torch.equal(vc[b, :L], v[s0:s0 + L])


def test_cache_writer_reports_positions_outside_the_cache(jl):
    cos, sin = _tables(jl, 64, 128, 1e4)
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 16, 2, 128), dtype=torch.bfloat16, device="cuda")
    jl.jl_decode_append(q, kv, kv, torch.tensor([40], dtype=torch.int32, device="cuda"), cos, sin, kc, kc.clone())
    with pytest.raises(jl.JetLongError) as err:
        jl.jl_sync_status()
    assert err.value.status == jl.JL_ERR_INVALID
    jl.jl_sync_status()
    assert torch.count_nonzero(kc) == 0


def test_streaming_decode_from_raw_tokens_across_G_boundary(jl):
    """Prompt -> jl_kv_cache_fill; then per step jl_decode_append (raw token) + jl_bifocal_decode.
    Each step must equal the routed attention of the raw sequence's last row (direct definition),
    across L = 768 -> 769 where G steps from 3 to 4, with no cache rewrite."""
    L0, steps, w_pre, w0 = 765, 6, 256, 100
    cfg = I.PrefillConfig("stream", (L0 + steps,), 8, 2, 128, w0, w_pre, 1e4, True)
    q, k, v, _ = I.prefill_inputs(cfg)
    stride = L0 + steps
    cos, sin = _tables(jl, stride, 128, cfg.rope_base)
    kc = torch.zeros((1, stride, 2, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    cu0 = torch.tensor([0, L0], dtype=torch.int32, device="cuda")
    jl.jl_kv_cache_fill(k[:L0].cuda(), v[:L0].cuda(), cu0, cos, sin, kc, vc)
    qb, kb, vb = I.bf16_bits(q), I.bf16_bits(k), I.bf16_bits(v)
    for t in range(steps):
        L = L0 + t + 1
        sl = torch.tensor([L], dtype=torch.int32, device="cuda")
        qt = jl.jl_decode_append(q[L - 1:L].cuda(), k[L - 1:L].cuda(), v[L - 1:L].cuda(), sl, cos, sin, kc, vc)
        out, lse = jl.jl_bifocal_decode(qt, kc, vc, sl, stride, w0, w_pre, cos, sin)
        jl.jl_sync_status()
        ro, rl = O.bifocal_rows(qb[:L], kb[:L], vb[:L], L, np.full(8, L - 1), np.arange(8), w0=w0,
                                w_pretrained=w_pre, rope_base=cfg.rope_base)
        _check(out.float().cpu().numpy()[0], lse.cpu().numpy()[0], ro, rl,
               f"stream step L={L} G={O.group_size(L, w_pre)}")


# ----------------------------------- literal three-pass inclusion-exclusion ----

THREE_PASS = [
    ("tp_G4_w0_100", (1000,), 8, 2, 128, 100, 256),
    ("tp_G4_w0_0", (600,), 4, 2, 128, 0, 160),
    ("tp_G3_w0_128", (700,), 4, 1, 128, 128, 256),
    ("tp_G1", (300,), 4, 2, 128, 64, 512),
    ("tp_varlen", (1, 130, 257, 700, 0, 64), 4, 2, 128, 50, 128),
    ("tp_w0_covers", (400,), 2, 2, 128, 5000, 100),
    ("tp_d64_group3", (500,), 3, 1, 64, 40, 100),
    ("tp_d128_group3", (700,), 3, 1, 128, 100, 256),
]


@pytest.mark.parametrize("case", THREE_PASS, ids=[c[0] for c in THREE_PASS])
def test_three_pass_merge_on_gpu(jl, case):
    """The pages' own realisation (pass 1 + pass 2 - pass 3 merged on their LSEs) on the GPU:
    the merged rows and each pass's LSE match the oracle's direct definition and its
    three-pass statistics."""
    name, seqlens, hq, hkv, d, w0, w_pre = case
    cfg = I.PrefillConfig(name, seqlens, hq, hkv, d, w0, w_pre, 1e4, True)
    q, k, v, cu = I.prefill_inputs(cfg)
    cos, sin = _tables(jl, max(cfg.max_seqlen, 1), d, cfg.rope_base)
    out, lse, ws = jl.jl_bifocal_prefill_three_pass(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), cfg.max_seqlen, w0,
                                                    w_pre, cos, sin)
    jl.jl_sync_status()
    T = cfg.total_tokens
    out, lse = out.float().cpu().numpy(), lse.cpu().numpy()
    plane = T * hq * d
    lse_p = ws[3 * plane * 4:].view(torch.float32)[:3 * hq * T].cpu().numpy().reshape(3, hq, T)
    for s in range(len(seqlens)):
        L = seqlens[s]
        if L == 0:
            continue
        pos = np.repeat(np.arange(L), hq)
        head = np.tile(np.arange(hq), L)
        s0 = int(cu[s])
        qb, kb, vb = I.bf16_bits(q[s0:s0 + L]), I.bf16_bits(k[s0:s0 + L]), I.bf16_bits(v[s0:s0 + L])
        ro, rl, rp = O.bifocal_rows(qb, kb, vb, L, pos, head, w0=w0, w_pretrained=w_pre, rope_base=cfg.rope_base,
                                    three_pass=True)
        _check(out[s0 + pos, head], lse[head, s0 + pos], ro, rl, f"{name} seq {s} merged")
        for pss in range(3):
            got = lse_p[pss][head, s0 + pos]
            ref = rp[:, pss]
            assert np.array_equal(np.isneginf(got), np.isneginf(ref)), f"{name} pass {pss + 1} emptiness"
            fin = np.isfinite(ref)
            assert np.abs(got[fin] - ref[fin]).max(initial=0.0) <= LSE_MAX, f"{name} pass {pss + 1} lse"


# ---------------------------------------------- chunked prefill over a cache ----

def _chunked_run(jl, name, lens_total, chunk_plan, hq, hkv, d, w0, w_pre):
    """Prefill each sequence in chunks: append the chunk's keys after the cached ones, then
    attend the chunk's queries over the cache; every chunk row must equal the direct
    definition over the raw prefix of length L = past + chunk."""
    B = len(lens_total)
    cfg = I.PrefillConfig(name, tuple(lens_total), hq, hkv, d, w0, w_pre, 1e4, True)
    q, k, v, cu = I.prefill_inputs(cfg)
    stride = max(lens_total)
    cos, sin = _tables(jl, stride, d, cfg.rope_base)
    kc = torch.zeros((B, stride, hkv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    past = [0] * B
    for step in chunk_plan:  # step: chunk length per sequence
        rows_q, rows_k, rows_v, cu_c = [], [], [], [0]
        for b in range(B):
            s0 = int(cu[b]) + past[b]
            rows_q.append(q[s0:s0 + step[b]])
            rows_k.append(k[s0:s0 + step[b]])
            rows_v.append(v[s0:s0 + step[b]])
            cu_c.append(cu_c[-1] + step[b])
        qc, kk, vv = torch.cat(rows_q), torch.cat(rows_k), torch.cat(rows_v)
        cu_t = torch.tensor(cu_c, dtype=torch.int32, device="cuda")
        past_t = torch.tensor(past, dtype=torch.int32, device="cuda")
        jl.jl_kv_cache_fill(kk.cuda(), vv.cuda(), cu_t, cos, sin, kc, vc, past_lens=past_t)
        out, lse = jl.jl_bifocal_prefill_chunk(qc.cuda(), cu_t, past_t, max(max(step), 1),
                                               max(p + s for p, s in zip(past, step)), kc, vc, w0, w_pre, cos, sin)
        jl.jl_sync_status()
        out, lse = out.float().cpu().numpy(), lse.cpu().numpy()
        for b in range(B):
            n = step[b]
            if n == 0:
                continue
            L = past[b] + n
            s0 = int(cu[b])
            pos = np.repeat(np.arange(past[b], L), hq)
            head = np.tile(np.arange(hq), n)
            ro, rl = O.bifocal_rows(I.bf16_bits(q[s0:s0 + L]), I.bf16_bits(k[s0:s0 + L]), I.bf16_bits(v[s0:s0 + L]),
                                    L, pos, head, w0=w0, w_pretrained=w_pre, rope_base=cfg.rope_base)
            r0 = cu_c[b] + (pos - past[b])
            _check(out[r0, head], lse[head, r0], ro, rl, f"{name} seq {b} chunk past={past[b]} L={L}")
        past = [p + s for p, s in zip(past, step)]


def test_chunked_prefill_single_sequence_across_G(jl):
    # L after each chunk: 300 (G 2), 777 (G 4), 1100 (G 5); chunk starts not multiples of 128
    _chunked_run(jl, "chunk1", [1100], [[300], [477], [323]], 8, 2, 128, 100, 256)


def test_chunked_prefill_batched_mixed_pasts(jl):
    _chunked_run(jl, "chunk_b", [700, 260, 513], [[128, 0, 100], [200, 260, 1], [372, 0, 412]], 4, 2, 128, 64, 128)


def test_chunked_prefill_d64_group3(jl):
    _chunked_run(jl, "chunk_d64", [500], [[129], [371]], 3, 1, 64, 40, 100)


def test_chunked_prefill_d128_group3(jl):
    # odd group at head_dim 128: the one-head double-buffered kernel with cached keys
    _chunked_run(jl, "chunk_d128_g3", [900, 300], [[130, 0], [400, 300], [370, 0]], 3, 1, 128, 64, 200)


# --------------------------------------------------------------- paged caches ----

def _paginate(cache, lens, page_size, seed=3):
    """Scatter contiguous caches [B][stride][Hkv][d] into a shuffled page pool + block table."""
    B = cache.shape[0]
    max_pages = max(-(-L // page_size) for L in lens)
    n_pages = sum(-(-L // page_size) for L in lens) + 3
    order = np.random.default_rng(seed).permutation(n_pages)
    pool = torch.zeros((n_pages, page_size) + tuple(cache.shape[2:]), dtype=cache.dtype)
    table = torch.zeros((B, max_pages), dtype=torch.int32)
    nxt = 0
    for b, L in enumerate(lens):
        for pg in range(-(-L // page_size)):
            page = int(order[nxt])
            nxt += 1
            table[b, pg] = page
            rows = cache[b, pg * page_size:min(L, (pg + 1) * page_size)]
            pool[page, :rows.shape[0]] = rows
    return pool, table


def test_paged_decode_equals_contiguous_and_oracle(jl):
    cfg = SMALL_DECODE
    lens, page = [1000, 300], 256
    max_len = 1024
    k_cache, v = _decode_setup(cfg, max_len, batch=2)
    qs = I.decode_queries(cfg, 1, batch=2)[0]
    q_t = torch.stack([_query_tilde(cfg, qs[b], lens[b]) for b in range(2)])
    cos, sin = _tables(jl, max_len, 128, cfg.rope_base)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ref, ref_lse = jl.jl_bifocal_decode(q_t.cuda(), k_cache.cuda(), v.cuda(), sl, max_len, cfg.w0, cfg.w_pretrained,
                                        cos, sin)
    kp, table = _paginate(k_cache, lens, page)
    vp, _ = _paginate(v, lens, page)
    out, lse = jl.jl_bifocal_decode_paged(q_t.cuda(), kp.cuda(), vp.cuda(), table.cuda(), sl, max_len, cfg.w0,
                                          cfg.w_pretrained, cos, sin)
    jl.jl_sync_status()
    assert torch.equal(out, ref) and torch.equal(lse, ref_lse)
    for b, L in enumerate(lens):
        ro, rl = _decode_oracle(cfg, q_t[b], k_cache[b], v[b], L)
        _check(out[b].float().cpu().numpy(), lse[b].cpu().numpy(), ro, rl, f"paged b={b}")


def test_paged_cache_writers_match_contiguous(jl):
    cfg = I.PrefillConfig("pfill", (500, 130), 4, 2, 128, 32, 64, 1e4, True)
    q, k, v, cu = I.prefill_inputs(cfg)
    cos, sin = _tables(jl, 1024, 128, cfg.rope_base)
    kc = torch.zeros((2, 512, 2, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    jl.jl_kv_cache_fill(k.cuda(), v.cuda(), cu.cuda(), cos, sin, kc, vc)
    _, table = _paginate(kc.cpu(), [512, 512], 128)
    n_pages = int(table.max()) + 1
    kp = torch.zeros((n_pages, 128, 2, 128), dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    tb = table.cuda()
    jl.jl_kv_cache_fill_paged(k.cuda(), v.cuda(), cu.cuda(), cos, sin, kp, vp, tb)
    # one decode-step append at position 500 of entry 0 and 130 of entry 1
    q1 = torch.randn((2, 4, 128)).to(torch.bfloat16).cuda()
    k1 = torch.randn((2, 2, 128)).to(torch.bfloat16).cuda()
    sl = torch.tensor([501, 131], dtype=torch.int32, device="cuda")
    qa = jl.jl_decode_append(q1, k1, k1, sl, cos, sin, kc, vc)
    qb = jl.jl_decode_append_paged(q1, k1, k1, sl, cos, sin, kp, vp, tb)
    jl.jl_sync_status()
    assert torch.equal(qa, qb)
    for b, L in enumerate([501, 131]):
        for pos in range(L):
            page, off = int(table[b, pos // 128]), pos % 128
            assert torch.equal(kp[page, off], kc[b, pos]) and torch.equal(vp[page, off], vc[b, pos])
    bad = tb.clone()
    bad[0, 0] = n_pages + 7
    jl.jl_kv_cache_fill_paged(k.cuda(), v.cuda(), cu.cuda(), cos, sin, kp, vp, bad)
    with pytest.raises(jl.JetLongError) as err:
        jl.jl_sync_status()
    assert err.value.status == jl.JL_ERR_INVALID
    jl.jl_sync_status()


# ------------------------------------------- frequency-interpolation variant ----

def _yarn_ramp(d, s, base, w_pre, alpha=1.0, beta=32.0):
    """A YaRN-style by-parts factor per frequency: 1/s for long wavelengths, 1 for short."""
    th = base ** (-np.arange(0, d, 2) / d)
    r = w_pre * th / (2 * np.pi)  # rotations within the pretraining window
    gamma = np.clip((r - alpha) / (beta - alpha), 0.0, 1.0)
    return (1 - gamma) / s + gamma


INTERP = [
    ("pi_G4", (1000,), 8, 2, 128, 100, "pi", 4.0),
    ("yarn_s4", (1000,), 8, 2, 128, 100, "yarn", 4.0),
    ("yarn_varlen", (300, 129, 700), 4, 2, 128, 64, "yarn", 3.0),
    ("pi_d64_w0_0", (400,), 3, 1, 64, 0, "pi", 2.0),
    ("yarn_d128_group3", (600, 129), 3, 1, 128, 64, "yarn", 4.0),
]


@pytest.mark.parametrize("in_kernel", [False, True], ids=["key_workspace", "in_kernel_rotation"])
@pytest.mark.parametrize("case", INTERP, ids=[c[0] for c in INTERP])
def test_interp_prefill_matches_oracle(jl, case, in_kernel):
    """Keys rotated once into a workspace (remote rows: the interpolated rotation at the raw
    position), or rotated by the prefill kernel itself."""
    name, seqlens, hq, hkv, d, w0, kind, s = case
    cfg = I.PrefillConfig(name, seqlens, hq, hkv, d, w0, 256, 1e4, True)
    lam = np.full(d // 2, 1.0 / s) if kind == "pi" else _yarn_ramp(d, s, cfg.rope_base, 256)
    q, k, v, cu = I.prefill_inputs(cfg)
    n = max(cfg.max_seqlen, 1)
    cos, sin = _tables(jl, n, d, cfg.rope_base)
    cr, sr = jl.jl_rope_tables_scaled(n, d, cfg.rope_base, lam)
    out, lse = jl.jl_interp_prefill(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), cfg.max_seqlen, w0, cos, sin, cr, sr,
                                    rotate_keys_in_kernel=in_kernel)
    jl.jl_sync_status()
    out, lse = out.float().cpu().numpy(), lse.cpu().numpy()
    for b, L in enumerate(seqlens):
        s0 = int(cu[b])
        pos = np.repeat(np.arange(L), hq)
        head = np.tile(np.arange(hq), L)
        ro, rl = O.interp_rows(I.bf16_bits(q[s0:s0 + L]), I.bf16_bits(k[s0:s0 + L]), I.bf16_bits(v[s0:s0 + L]), L,
                               pos, head, w0=w0, rope_base=cfg.rope_base, freq_scale=lam)
        _check(out[s0 + pos, head], lse[head, s0 + pos], ro, rl,
               f"{name} seq {b}" + (" (in-kernel key rotation)" if in_kernel else ""))
