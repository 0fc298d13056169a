"""The bench's N > 1 path (independent replicas, one per rank) on CPU with gloo.

Each rank times its own replica; the job time is the max over ranks and the
whole-job rate is world * steps / max. The reference arm prints on rank 0 only.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = [0.5, 0.8][rank]
        got = bench.max_over_ranks(torch, dist, mine, "cpu")
        out[rank] = (got, bench.job_rate(world, 10, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_max_over_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert out[0] == out[1] == (0.8, 2 * 10 / 0.8)


def test_reference_arm_other_ranks_exit_quietly(capsys):
    import bench

    class A:
        steps, warmup, gpus = 1, 1, 2
    assert bench.run_reference(A, rank=1) == 0
    assert capsys.readouterr().out == ""


def test_job_rate_single():
    import bench
    assert bench.job_rate(1, 20, 0.5) == pytest.approx(40.0)


def test_attention_work_units_and_traffic_key(tmp_path, monkeypatch):
    # the units the roofline figures are built from, and the key that voids a
    # stored DRAM-traffic figure once any attention source changes
    import shutil

    import bench
    assert bench.attn_flops_layer(4096, 320) == 4.0 * 16 * 8 * 4096 * (5 * 4096) * 40
    assert abs(bench.attn_flops_layer(4096, 320) / 1e12 - 1.718) < 1e-3
    assert bench.exp2_level64() == 16 * 8 * 4096 * 5 * 4096
    src = os.path.join(bench.ROOT, "denoise_step_b200", "csrc")
    dst = tmp_path / "denoise_step_b200" / "csrc"
    dst.mkdir(parents=True)
    names = ("attn.cu", "attn.cuh", "ptx.cuh", "fastmath.cuh")
    for f in names:
        shutil.copy(os.path.join(src, f), dst / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_hash()
    for f in names:
        keep = (dst / f).read_bytes()
        (dst / f).write_bytes(keep + b"\n")
        assert bench.kernel_hash() != base, f
        (dst / f).write_bytes(keep)
    assert bench.kernel_hash() == base
