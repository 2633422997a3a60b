"""Host logic of bench.py on CPU: the cross-rank reduction with two gloo
ranks (max of device times, sum of bytes), the expected-bytes formula and the
reference arm's line."""
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


@pytest.mark.slow
def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "3", "--cpu-heads", "8", "--cpu-steps", "3",
                        "--workload", "llama3.2-1b_l16_b1_ctx8192_s128_w512_bf16"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
