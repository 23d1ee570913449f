"""The multi-GPU host logic of bench.py on CPU ranks (gloo, world size 2): the
global batch is split by the library's cost-balanced shard plan (every rank
computes the same plan, each gets its own clips, the weights are the same
everywhere), the step time is the slowest rank's, and the reported value is
the whole job's audio over that time. No GPU: the ranks only run the host-side
helpers bench.py uses between its CUDA launches (the plan is a host-only call
of the C ABI)."""
import datetime
import os
import socket

import pytest

import bench
import synthetic as S

CFG = S.EncoderConfig(name="ranks", n_mels=8, d_model=128, n_layers=1, n_heads=2, ffn_dim=256, frames=40, batch=4,
                      dtype="fp32", seed=3, ragged=(5, 40))


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
        g, clips, lengths = bench.rank_clips(CFG, rank, world)
        mel = bench.rank_mel(g, clips)
        w = S.make_weights(CFG.replace(seed=bench.rank_weight_seed(CFG)))
        wsum = float(sum(v.astype("float64").sum() for v in w.values()))
        flops = bench.workload_flops(CFG, lengths)
        mine = torch.tensor([wsum, flops] + [float(c) for c in clips], dtype=torch.float64)
        every = [torch.zeros_like(mine) for _ in range(world)]
        dist.all_gather(every, mine)
        cpu = torch.device("cpu")
        slowest = bench.max_over_ranks(10.0 + rank, world, cpu)
        audio = bench.sum_over_ranks(float(lengths.sum()) / bench.FRAMES_PER_SECOND, world, cpu)
        dist.barrier()
        queue.put((rank, [e.tolist() for e in every], slowest, audio, mel.shape, lengths.tolist(),
                   [S.mel_clip(g, int(c)).tolist() == m.tolist() for c, m in zip(clips, mel)]))
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
    assert [r[0] for r in results] == [0, 1]
    g = CFG.replace(batch=2 * CFG.batch)
    all_lengths = S.make_lengths(g)
    for rank, every, slowest, audio, shape, lengths, same_mel in results:
        assert slowest == 11.0                           # the slower rank's time
        assert audio == float(all_lengths.sum()) / bench.FRAMES_PER_SECOND   # every rank's audio
        assert every[0][0] == every[1][0]                # the same weights everywhere
        clips0, clips1 = [set(int(c) for c in e[2:]) for e in every]
        assert len(clips0) == len(clips1) == CFG.batch   # cfg.batch clips per rank
        assert clips0 | clips1 == set(range(g.batch)) and not clips0 & clips1
        mine = sorted(clips0 if rank == 0 else clips1)
        assert lengths == all_lengths[mine].tolist()     # clips in global order with their lengths
        assert shape == (CFG.batch, CFG.n_mels, CFG.frames) and all(same_mel)
        # the plan's loads are balanced: the two ranks' FLOPs within the largest clip's
        assert abs(every[0][1] - every[1][1]) <= bench.workload_flops(CFG, [int(all_lengths.max())])
    assert results[0][1] == results[1][1]                # both ranks saw the same plan
    assert all(p.exitcode == 0 for p in procs)


def test_job_throughput_counts_every_rank():
    # 16 clips of 30 s per rank in a 40 ms step
    assert bench.job_throughput(480.0, 40.0) == pytest.approx(12000.0)
    assert bench.job_throughput(8 * 480.0, 40.0) == pytest.approx(96000.0)
    # one rank: the one-GPU batch itself
    g, clips, lengths = bench.rank_clips(CFG, 0, 1)
    assert g.batch == CFG.batch and clips.tolist() == list(range(CFG.batch))
    assert lengths.tolist() == S.make_lengths(CFG).tolist()
    assert (bench.rank_mel(g, clips) == S.make_mel(CFG)).all()
    # more ranks: the global batch starts with the one-GPU batch
    g4, _, _ = bench.rank_clips(CFG, 2, 4)
    assert S.make_lengths(g4)[:CFG.batch].tolist() == S.make_lengths(CFG).tolist()
