"""The bench's reference arm runs on the host cores alone: its JSON line must carry the
keys the line contract names, and ranks other than 0 must print nothing."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def oracle_built():
    sys.path.insert(0, ROOT)
    from oracle import build
    build.build()


def _run(extra_env, *args, timeout=300):
    env = dict(os.environ)
    env.update(extra_env)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line(oracle_built):
    r = _run({}, "--impl", "reference", "--steps", "1", "--warmup", "0")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 0
    assert d["value"] > 0 and d["config"]["workload"] == bench.WORKLOAD and d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing(oracle_built):
    r = _run({"RANK": "1", "WORLD_SIZE": "2"}, "--impl", "reference", "--steps", "1", "--warmup", "0", timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_cpu_baseline_covers_prefill_decode_and_tiny(oracle_built):
    """The bench's cpu_baseline object: the prefill row sample (the metric's unit), one oracle decode
    step at every cache length plus the walk steps around the G = 3 -> 4 boundary, the tiny layer
    in full, and the host's core count (affinity-aware) beside the oracle's thread count."""
    sys.path.insert(0, ROOT)
    import bench
    cb = bench.cpu_baseline(seconds=0.3)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["unit"] == bench.UNIT
    assert cb["cores"] == len(os.sched_getaffinity(0)) and cb["omp_threads"] >= 1
    dec = cb["decode"]
    assert set(dec["us_per_token_at_cache_len"]) == {str(L) for L in bench.DECODE.cache_lens}
    assert all(v > 0 for v in dec["us_per_token_at_cache_len"].values())
    assert dec["walk_sample"]["G"] == [3, 3, 4, 4] and dec["walk_256_tokens_estimate_s"] > 0
    assert cb["tiny"]["ms_per_layer"] > 0 and cb["tiny"]["useful_tflops"] > 0
