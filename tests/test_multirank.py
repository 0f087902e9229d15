"""Multi-rank host logic of bench.py on CPU with world_size = 2 (gloo).

Token rows are independent, so N GPUs run N independent shards; the only
collectives are the timing barrier and the max-over-ranks of the elapsed time.
These tests run that logic on two gloo ranks (no GPU needed)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from w3a3_quantization_online_b200 import inputs
        elapsed = [10.0, 12.5][rank]
        dist.barrier()
        worst = bench.max_over_ranks(elapsed)
        rate = bench.whole_job_rate(16384, world, 100, worst)
        a = inputs.align_case(8, 256, 8, bench.shard_seed(rank), dtype="bf16", n_outliers=2,
                              outlier_scale=10.0, qm_seed=1)
        q.put((rank, worst, rate, a.x.copy(), a.Q.copy(), a.M.copy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_max_elapsed_and_shard_their_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, worst, rate, x, Q, M = q.get(timeout=120)
        res[r] = (worst, rate, x, Q, M)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][0] == res[1][0] == 12.5                     # max over ranks
    assert res[0][1] == pytest.approx(16384 * 2 * 100 / 12.5e-3)
    assert not np.array_equal(res[0][2], res[1][2])           # different token shards
    np.testing.assert_array_equal(res[0][3], res[1][3])       # Q replicated
    np.testing.assert_array_equal(res[0][4], res[1][4])       # M replicated


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_rate(100, 1, 10, 1000.0) == pytest.approx(1000.0)
    assert bench.shard_seed(0) != bench.shard_seed(1)


def test_traffic_record_follows_code_not_comments(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "k.cu"
    src.write_text("// a kernel\n__global__ void k(int *p) { p[0] = 1; }  /* store */\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha(["k.cu"])
    src.write_text("// the same kernel, reworded comment\n__global__ void k(int *p) {\n    p[0] = 1;\n}\n")
    assert bench.kernel_source_sha(["k.cu"]) == h0
    src.write_text("__global__ void k(int *p) { p[0] = 2; }\n")
    assert bench.kernel_source_sha(["k.cu"]) != h0
