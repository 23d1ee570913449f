"""The multi-GPU host logic of bench.py on CPU ranks (gloo, world size 2): each
rank encodes its own clips with the same weights, the step time is the slowest
rank's, and the reported value is the whole job's. No GPU: the ranks only run
the host-side helpers bench.py uses between its CUDA launches."""
import datetime
import os
import socket

import pytest

import bench
import synthetic as S

CFG = S.EncoderConfig(name="ranks", n_mels=8, d_model=128, n_layers=1, n_heads=2, ffn_dim=256, frames=40, batch=2,
                      dtype="fp32", seed=3)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        rc = bench.rank_config(CFG, rank)
        mel = S.make_mel(rc)
        w = S.make_weights(CFG.replace(seed=bench.rank_weight_seed(CFG)))
        mine = torch.tensor([float(mel.astype("float64").sum()), float(sum(v.astype("float64").sum()
                                                                              for v in w.values()))],
                            dtype=torch.float64)
        every = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(every, mine)
        slowest = bench.max_over_ranks(10.0 + rank, world, torch.device("cpu"))
        dist.barrier()
        queue.put((rank, [e.tolist() for e in every], slowest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(queue.get(timeout=180) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [r for r, _, _ in results] == [0, 1]
    for _, every, slowest in results:
        assert slowest == 11.0                           # the slower rank's time
        (mel0, w0), (mel1, w1) = every
        assert mel0 != mel1                              # each rank its own clips
        assert w0 == w1                                  # the same weights everywhere
    assert all(p.exitcode == 0 for p in procs)


def test_job_throughput_counts_every_rank():
    # 16 clips of 30 s per rank in a 40 ms step
    assert bench.job_throughput(1, 480.0, 40.0) == pytest.approx(12000.0)
    assert bench.job_throughput(8, 480.0, 40.0) == pytest.approx(96000.0)
    assert bench.rank_config(CFG, 0) is CFG
    assert bench.rank_config(CFG, 3).seed == CFG.seed + 3000
