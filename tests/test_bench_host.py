"""Host logic of bench.py on CPU: the cross-rank reduction with two gloo
ranks (max of device times, sum of bytes), the expected-bytes formula, the
store-dtype override, the sysfs cpu-list parser, the lookup of a profiled
traffic ratio, the reference arm's line and the prefill attention's tile
count."""
import json
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms, nb = bench.reduce_over_ranks(1.5 + rank, 100.0 * (rank + 1))
    out[rank] = (ms, nb)
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = 29500 + os.getpid() % 2000
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (2.5, 300.0)


def test_reduce_without_process_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(3.0, 7.0) == (3.0, 7.0)


def test_expected_bytes_of_the_default_workload():
    sys.path.insert(0, ROOT)
    import bench
    from synth import configs
    wl = configs.QWEN8B_CTX8K
    b = bench.expected_bytes_per_step(wl)
    # 288 heads, about 512 + 0.16 * 7680 kept tokens each, 512 bytes per token
    assert 200e6 < b < 300e6


def test_kv_dtype_override_renames_and_resizes():
    sys.path.insert(0, ROOT)
    import bench
    from synth import configs
    wl = bench.with_kv_dtype(configs.QWEN8B_CTX8K, "int4")
    assert wl.name == "qwen3-8b_l36_b1_ctx8192_s128_w512_int4g32" and wl.kv_dtype == "int4"
    assert wl.kv_row_bytes() == 72 and configs.QWEN8B_CTX8K.kv_row_bytes() == 256
    b8 = bench.with_kv_dtype(configs.QWEN8B_FP8_B8_CTX32K, "int4")
    assert b8.name == "qwen3-8b_l36_b8_ctx32768_s256_w512_int4g32"
    assert bench.with_kv_dtype(configs.QWEN8B_CTX8K, None) is configs.QWEN8B_CTX8K
    assert bench.with_kv_dtype(configs.QWEN8B_CTX8K, "bf16") is configs.QWEN8B_CTX8K
    # retained bytes scale with the row size: 2 x 72 instead of 2 x 256 bytes a token
    r = bench.expected_bytes_per_step(wl) / bench.expected_bytes_per_step(configs.QWEN8B_CTX8K)
    assert abs(r - 72 / 256) < 1e-12


def test_parse_cpulist():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.parse_cpulist("0-3,8,10-11\n") == {0, 1, 2, 3, 8, 10, 11}
    assert bench.parse_cpulist("5") == {5}


def test_profiled_traffic_ratio_matches_workload_and_source(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    h = bench.attn_source_hash()
    (tmp_path / "decode_attn_a.md").write_text(
        f"workload: wl_a\nkernel source hash: {h}\n| dram bytes per algorithmic byte: 1.0200 | x |\n")
    (tmp_path / "decode_attn_b.md").write_text(
        "workload: wl_b\nkernel source hash: 0000000000000000\n| dram bytes per algorithmic byte: 1.5 |\n")
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    assert bench.profiled_traffic_ratio("wl_a") == (1.02, h)
    assert bench.profiled_traffic_ratio("wl_b") == (None, None)   # taken on other sources
    assert bench.profiled_traffic_ratio("wl_c") == (None, None)   # no summary


@pytest.mark.slow
def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "3", "--cpu-heads", "8", "--cpu-steps", "3",
                        "--workload", "llama3.2-1b_l16_b1_ctx8192_s128_w512_bf16"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["compaction"]["ms_per_layer"] > 0


def test_prefill_tile_counts_reduce_to_closed_forms():
    """bench.prefill_tiles (the FLOP count of the prefill attention line):
    the dense count is the number of causal tiles n (n + 1) / 2; with no
    evict flag every old key sits in the store, so the far tiles are the old
    tiles themselves and the sparse count equals the dense one; with every
    key flagged only the band is read (for w = 128: the diagonal tile and
    the one before it); any flags give a count between the two."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    P, w = 1000, 128
    n = (P + 127) // 128
    none = np.zeros((2, P, 3), np.uint8)
    dense, sparse = bench.prefill_tiles(none, P, w)
    assert dense == n * (n + 1) // 2
    assert (sparse == dense).all()
    allf = np.ones((1, P, 2), np.uint8)
    _, sp = bench.prefill_tiles(allf, P, w)
    assert (sp == 1 + 2 * (n - 1)).all()
    rng = np.random.default_rng(3)
    f = (rng.random((1, P, 4)) < 0.8).astype(np.uint8)
    _, sp = bench.prefill_tiles(f, P, w)
    assert (sp >= 1 + 2 * (n - 1)).all() and (sp <= dense).all()
    # a window shorter than a tile with few kept keys: far tiles whose slots
    # would run past the head's kept rows fall back to the causal tiles
    f = (rng.random((1, P, 1)) < 0.97).astype(np.uint8)
    _, sp = bench.prefill_tiles(f, P, 16)
    assert sp[0, 0] <= dense
