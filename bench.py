#!/usr/bin/env python
"""Throughput of the Whisper-style audio encoder tower forward pass on B200.

Default workload: the Whisper-large encoder (32 layers, d_model 1280, 20 heads
x 64, FFN 5120, 128 mel bins x 3000 frames = 30 s per clip -> 1500 positions),
batch 16 per GPU, bf16 operands with fp32 accumulation, synthetic seeded inputs
and random weights of that architecture.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
    python bench.py --kernel qkv|out|fc1|fc2|attention|frontend|cache [--steps K] [--warmup W]   (one step alone)
    python bench.py --kernel sidestream [--steps K]   (encoder on a side stream beside a decoder stand-in)
    python bench.py --kernel block [--steps K]        (the workload's geometry with one encoder block)

One step = one enc_forward over a batch of 16 clips. Multi-GPU (torchrun, one
process per GPU) runs independent replicas, each with its own batch of 16
(weak scaling, no collective on the data path); the time is the max over ranks.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synthetic as S  # noqa: E402

METRIC = "audio-sec/s and TFLOP/s (% of BF16 peak), Whisper-large encoder, B=16, bf16, 1 B200"
UNIT = "audio-s/s"
FRAMES_PER_SECOND = 100.0          # 16 kHz audio, hop 160
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's published dense BF16 tensor rate of one B200 (its 4.5 PFLOP/s figure
# assumes 2:4 sparsity); reported beside the measured peaks
PUBLISHED_DENSE_BF16_TFLOPS = 2250.0
GEMM_CLASSES = ("conv1", "conv2", "qkv", "out", "fc1", "fc2", "proj1", "proj2")


# ----------------------------------------------------------------- workload
def workload_flops(cfg, lengths, layers=None) -> float:
    """Algorithmic FLOPs (multiply-add = 2) over the valid positions of each clip."""
    d, m, f = cfg.d_model, cfg.n_mels, cfg.ffn_dim
    L = cfg.n_layers if layers is None else layers
    total = 0.0
    for ln in lengths:
        n = (int(ln) + 1) // 2
        total += 2.0 * (2 * n) * d * 3 * m + 2.0 * n * d * 3 * d
        c = cfg.attn_chunk if cfg.attn_chunk else n      # block-local attention: per chunk
        attn = sum(min(c, n - c0) ** 2 for c0 in range(0, n, c))
        total += L * (6.0 * n * d * d + 4.0 * attn * d + 2.0 * n * d * d + 4.0 * n * d * f)
        if cfg.proj_hidden:
            no = n // cfg.pool_step if cfg.pool_step > 1 else n
            total += 2.0 * no * (d * cfg.proj_hidden + cfg.proj_hidden * cfg.proj_out)
    return total


def workload_desc(cfg, n_gpus):
    return {
        "workload": (f"{cfg.name}: Whisper-style encoder {cfg.n_layers}L d{cfg.d_model} {cfg.n_heads}x64 heads "
                     f"FFN{cfg.ffn_dim}, {cfg.n_mels} mel x {cfg.frames} frames, B={cfg.batch} per GPU"
                     + (f", pool {cfg.pool_step}" if cfg.pool_step > 1 else "")
                     + (f", projector {cfg.d_model}->{cfg.proj_hidden}->{cfg.proj_out}" if cfg.proj_hidden else "")
                     + (f", lengths U[{cfg.ragged[0]},{cfg.ragged[1]}] frames" if cfg.ragged else "")
                     + (f", block-local attention over {cfg.attn_chunk}-position chunks" if cfg.attn_chunk else "")),
        "global_batch": cfg.batch * n_gpus,
        "frames": cfg.frames,
        "positions": cfg.positions,
        "parallelism": (f"replicas x{n_gpus} (global batch of {cfg.batch * n_gpus} clips split by the cost-balanced "
                        f"shard plan, {cfg.batch} per GPU; no collective)" if n_gpus > 1 else "replicas x1"),
        "l2": "per-step working set >> 126 MB L2 (weights 1.27 GB bf16 + activations), no explicit flush",
    }


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ------------------------------------------------------------- oracle legs
def oracle_sample(cfg, w, mel_clip, length, layers):
    """Time the oracle on one clip: conv stem + `layers` blocks + final LN."""
    import oracle as O
    t0 = time.perf_counter()
    O.encode_clip(cfg, w, mel_clip, int(length), layers=layers)
    return time.perf_counter() - t0


# Both CPU legs (cpu_baseline and --impl reference) time the same sample: one
# clip of the workload through the conv stem, ORACLE_SAMPLE_BLOCKS of its
# blocks and the final LayerNorm, converted to audio-s/s at the full workload's
# FLOPs per audio second.
ORACLE_SAMPLE_BLOCKS = 4


def oracle_sample_setup(cfg):
    lengths = S.make_lengths(cfg)
    w = S.make_weights(cfg, layers=list(range(ORACLE_SAMPLE_BLOCKS)))
    mel = S.mel_clip(cfg, 0)
    sample_flops = workload_flops(cfg, lengths[:1], ORACLE_SAMPLE_BLOCKS)
    flops_per_audio_s = workload_flops(cfg, lengths) / (float(np.sum(lengths)) / FRAMES_PER_SECOND)
    desc = (f"1 clip ({lengths[0]} frames), conv stem + {ORACLE_SAMPLE_BLOCKS} of {cfg.n_layers} blocks + final "
            f"LN, float64 numpy/BLAS; audio-s/s at the full workload's FLOPs per audio second")
    return lengths, w, mel, sample_flops, flops_per_audio_s, desc


def cpu_baseline(cfg, repeats=5):
    """The oracle on the host cores, on a bounded sample of the same workload
    (the median of `repeats` runs of the common sample, about 10 s in all)."""
    lengths, w, mel, sample_flops, flops_per_audio_s, desc = oracle_sample_setup(cfg)
    times = [oracle_sample(cfg, w, mel, lengths[0], ORACLE_SAMPLE_BLOCKS) for _ in range(repeats)]
    secs = statistics.median(times)
    return {"value": sample_flops / secs / flops_per_audio_s, "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle", "sample": f"median of {repeats} runs of: {desc}; {secs:.2f} s per run",
            "seconds": secs}


def run_reference(args, cfg):
    """--impl reference: the oracle (float64, host cores) timed on this workload,
    one run of the common sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    lengths, w, mel, sample_flops, flops_per_audio_s, desc = oracle_sample_setup(cfg)
    for _ in range(args.warmup):
        oracle_sample(cfg, w, mel, lengths[0], ORACLE_SAMPLE_BLOCKS)
    times = [oracle_sample(cfg, w, mel, lengths[0], ORACLE_SAMPLE_BLOCKS) for _ in range(args.steps)]
    tot = sum(times)
    value = sample_flops * args.steps / tot / flops_per_audio_s
    sample = f"each step: {desc}"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_desc(cfg, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = "clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown," \
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown," \
             "clocks_event_reasons.sw_power_cap"

    def __init__(self, device_index: int):
        self.proc = None
        self.rows = []
        ident = str(device_index)
        try:
            import torch
            u = getattr(torch.cuda.get_device_properties(device_index), "uuid", None)
            if u is not None:
                ident = "GPU-" + str(u)
        except Exception:
            pass
        self.ident = ident

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.ident, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 8:
                self.rows.append(parts)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[4 + i].lower() == "active"})
        pw = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows), "power_w_max": max(pw) if pw else None}


def gemm_traffic_record():
    """DRAM traffic of the GEMM kernel from a committed ncu summary, if it matches the current source."""
    p = os.path.join(ROOT, "profiles", "gemm_tc_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for fn in ("gemm_tc.cu", "common.cuh"):
        with open(os.path.join(ROOT, "audio_encoder_tower_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return rec if rec.get("source_sha256") == h.hexdigest() else None


# ------------------------------------------------------------ multi-rank
def tower_config(cfg, max_batch=None):
    """The library's enc_config for a workload (max_batch = clips per rank)."""
    from audio_encoder_tower_b200 import encoder_config
    return encoder_config(n_mels=cfg.n_mels, d_model=cfg.d_model, n_layers=cfg.n_layers, n_heads=cfg.n_heads,
                          ffn_dim=cfg.ffn_dim, max_frames=cfg.frames,
                          max_batch=cfg.batch if max_batch is None else max_batch, dtype=cfg.dtype,
                          pool_step=cfg.pool_step, proj_hidden=cfg.proj_hidden, proj_out=cfg.proj_out,
                          attn_chunk=cfg.attn_chunk)


def rank_clips(cfg, rank: int, world: int):
    """The clips of one rank: one seeded global batch of world x cfg.batch clips
    (its first cfg.batch clips are the one-GPU batch) split over the ranks by the
    library's cost-balanced plan (enc_shard_plan: largest clip first onto the
    least loaded rank, cfg.batch clips per rank). Every rank computes the same
    plan from the same lengths, so no rank sends it to another.
    Returns (global-batch config, clip indices of this rank, their lengths)."""
    g = cfg.replace(batch=cfg.batch * world)
    lengths = S.make_lengths(g)
    if world == 1:
        return g, np.arange(cfg.batch), lengths
    from audio_encoder_tower_b200 import shard_plan
    rank_of, _, _, _ = shard_plan(tower_config(cfg), lengths, world)
    mine = np.flatnonzero(rank_of == rank)     # clip order, as the plan's index_of
    return g, mine, lengths[mine]


def rank_mel(g, clips):
    """The mel of the given clips of global-batch config g, [len(clips), n_mels, T]."""
    if len(clips) == g.batch:
        return S.make_mel(g)
    return np.stack([S.mel_clip(g, int(b)) for b in clips])


def rank_weight_seed(cfg) -> int:
    """Every rank draws the weights from the unshifted seed."""
    return cfg.seed


def max_over_ranks(v: float, world: int, device) -> float:
    """The slowest rank's time: all-reduce MAX over the process group (any backend)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v: float, world: int, device) -> float:
    """A per-rank amount summed over the process group (any backend)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_throughput(audio_s_all_ranks: float, ms_per_step: float) -> float:
    """Whole-job audio-seconds per second: the audio of every rank's batch in the slowest rank's step time."""
    return audio_s_all_ranks / (ms_per_step / 1e3)


# ------------------------------------------------------- one kernel alone
def run_kernel(args, cfg):
    """Time one step of the workload alone through the C ABI (for profiling): a
    layer GEMM shape (qkv, out, fc1, fc2) at M = batch x positions, the
    attention, the log-mel front end over the batch's 30 s clips, or the
    encoder behind its embeddings cache with half of every step's clips seen
    in the step before."""
    import torch
    from audio_encoder_tower_b200.binding import attention_bf16, linear_bf16
    torch.cuda.set_device(0)
    n = cfg.frames // 2
    M, d, f, H = cfg.batch * n, cfg.d_model, cfg.ffn_dim, cfg.n_heads
    g = torch.Generator(device="cuda").manual_seed(cfg.seed)
    if args.kernel == "block":
        # every kernel of a forward once (stem, one block with its fused LayerNorms, final LN)
        from audio_encoder_tower_b200 import Encoder
        one = cfg.replace(n_layers=1)
        w_dev = {k: torch.from_numpy(v).to(device="cuda", dtype=torch.bfloat16)
                 for k, v in S.make_weights(one).items()}
        enc = Encoder(n_mels=one.n_mels, d_model=one.d_model, n_layers=1, n_heads=one.n_heads,
                      ffn_dim=one.ffn_dim, max_frames=one.frames, max_batch=one.batch, dtype=one.dtype,
                      pool_step=one.pool_step, proj_hidden=one.proj_hidden, proj_out=one.proj_out,
                      attn_chunk=one.attn_chunk, weights=w_dev)
        del w_dev
        mel = torch.from_numpy(S.make_mel(one)).to(device="cuda", dtype=torch.bfloat16)
        lengths = S.make_lengths(one)
        launch = lambda: enc.forward(mel, lengths)   # noqa: E731
        flops = workload_flops(one, lengths)
        shape = {"clips": one.batch, "layers": 1, "audio_s": float(np.sum(lengths)) / FRAMES_PER_SECOND}
    elif args.kernel == "cache":
        from audio_encoder_tower_b200 import Cache, Encoder
        w_np = S.make_weights(cfg)
        w_dev = {k: torch.from_numpy(v).to(device="cuda", dtype=torch.bfloat16) for k, v in w_np.items()}
        del w_np
        enc = Encoder(n_mels=cfg.n_mels, d_model=cfg.d_model, n_layers=cfg.n_layers, n_heads=cfg.n_heads,
                      ffn_dim=cfg.ffn_dim, max_frames=cfg.frames, max_batch=cfg.batch, dtype=cfg.dtype,
                      pool_step=cfg.pool_step, proj_hidden=cfg.proj_hidden, proj_out=cfg.proj_out,
                      attn_chunk=cfg.attn_chunk, weights=w_dev)
        del w_dev
        mel = torch.from_numpy(S.make_mel(cfg)).to(device="cuda", dtype=torch.bfloat16)
        cache = Cache(enc, 4 * cfg.batch)
        half, step_no = cfg.batch // 2, [0]

        def launch():   # keys of step i: half * i .. half * i + B - 1 (the first half seen in step i - 1)
            i = step_no[0]
            step_no[0] += 1
            cache.forward(mel, list(range(half * i, half * i + cfg.batch)))

        flops = workload_flops(cfg, S.make_lengths(cfg)[:half])   # the clips computed per step
        shape = {"clips": cfg.batch, "hits_per_step": half, "capacity": 4 * cfg.batch,
                 "audio_s": cfg.batch * cfg.frames / FRAMES_PER_SECOND}
    elif args.kernel == "frontend":
        from audio_encoder_tower_b200 import Frontend
        fe = Frontend(n_mels=cfg.n_mels, max_batch=cfg.batch)
        audio = torch.from_numpy(S.make_audio(cfg.batch)).cuda()
        mel_out = torch.empty((cfg.batch, cfg.n_mels, 3000), dtype=torch.bfloat16, device="cuda")
        launch = lambda: fe.log_mel(audio, out=mel_out)   # noqa: E731
        rows = cfg.batch * 3003   # frame rows as computed (3000 kept per clip)
        flops = 2.0 * rows * 404 * 400 + 2.0 * rows * cfg.n_mels * 204   # the two fp32 GEMMs as executed
        shape = {"clips": cfg.batch, "samples": 480000, "n_mels": cfg.n_mels, "frames": 3000,
                 "audio_s": 30.0 * cfg.batch}
    elif args.kernel == "attention":
        qkv = torch.randn(M, 3 * d, device="cuda", generator=g).to(torch.bfloat16)
        out = torch.empty(M, d, device="cuda", dtype=torch.bfloat16)
        cu = torch.arange(0, (cfg.batch + 1) * n, n, device="cuda", dtype=torch.int32)
        launch = lambda: attention_bf16(qkv, cu, n, H, out=out)   # noqa: E731
        flops = 4.0 * cfg.batch * n * n * d
        shape = {"clips": cfg.batch, "positions": n, "heads": H, "head_dim": 64}
    else:
        N, K, gelu, resid = {"qkv": (3 * d, d, False, False), "out": (d, d, False, True),
                             "fc1": (f, d, True, False), "fc2": (d, f, False, True)}[args.kernel]
        A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
        W = (torch.randn(N, K, device="cuda", generator=g) * 0.03).to(torch.bfloat16)
        b = torch.randn(N, device="cuda", generator=g) * 0.1
        x = torch.zeros(M, N, device="cuda", dtype=torch.float32) if resid else None
        launch = lambda: linear_bf16(A, W, b, gelu=gelu, resid=x)   # noqa: E731
        flops = 2.0 * M * N * K
        shape = {"M": M, "N": N, "K": K, "gelu": gelu, "residual": resid}
    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        launch()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    line = {"kernel": args.kernel, "workload": cfg.name, "shape": shape, "launches": args.steps,
            "ms_per_launch": ms, "tflops": flops / ms / 1e9}
    if args.kernel in ("frontend", "cache", "block"):
        line["audio_s_per_s"] = shape["audio_s"] / (ms / 1e3)
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ encoder side stream
# A decoder-like stand-in for the side-stream measurement: per layer the four
# projections of a 3072-wide transformer LLM (the width the Voxtral projector
# maps into): fused q/k/v 3072 -> 6144, attention output 4096 -> 3072, gate and
# up 3072 -> 2 x 8192, down 8192 -> 3072, at M = 64 tokens (one decode step of
# 64 sequences), each a tcgen05 GEMM of this library (enc_linear_bf16).
DECODER_WIDTH, DECODER_LAYERS, DECODER_TOKENS = 3072, 30, 64
DECODER_SHAPES = [(6144, 3072), (3072, 4096), (16384, 3072), (3072, 8192)]   # (N, K) per layer


def run_sidestream(args, cfg):
    """The encoder on a low-priority side stream while the decoder stand-in runs
    decode steps on a high-priority stream ("Multimodal Encoder Side Stream"):
    each workload alone, then both at once, timed with CUDA events on their own
    streams. Reports per-forward and per-decode-step times alone and overlapped,
    and the overlap gain = (sum of the times alone) / (time of both at once)."""
    import torch
    from audio_encoder_tower_b200 import Encoder
    from audio_encoder_tower_b200.binding import linear_bf16
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w_np = S.make_weights(cfg)
    w_dev = {k: torch.from_numpy(v).to(device=dev, dtype=torch.bfloat16) for k, v in w_np.items()}
    del w_np
    enc = Encoder(n_mels=cfg.n_mels, d_model=cfg.d_model, n_layers=cfg.n_layers, n_heads=cfg.n_heads,
                  ffn_dim=cfg.ffn_dim, max_frames=cfg.frames, max_batch=cfg.batch, dtype=cfg.dtype,
                  pool_step=cfg.pool_step, proj_hidden=cfg.proj_hidden, proj_out=cfg.proj_out,
                  attn_chunk=cfg.attn_chunk, weights=w_dev)
    del w_dev
    lengths = S.make_lengths(cfg)
    mel = torch.from_numpy(S.make_mel(cfg)).to(device=dev, dtype=torch.bfloat16)
    _, p_out, d_out = enc.output_positions(cfg.batch, lengths)
    out = torch.empty((cfg.batch, p_out, d_out), dtype=torch.bfloat16, device=dev)
    g = torch.Generator(device=dev).manual_seed(cfg.seed)
    dec_w = [[(torch.randn(n, k, device=dev, generator=g) * 0.02).to(torch.bfloat16) for n, k in DECODER_SHAPES]
             for _ in range(DECODER_LAYERS)]
    dec_x = {k: torch.randn(DECODER_TOKENS, k, device=dev, generator=g).to(torch.bfloat16)
             for k in {k for _, k in DECODER_SHAPES}}
    dec_y = {n: torch.empty(DECODER_TOKENS, n, device=dev, dtype=torch.bfloat16) for n, _ in DECODER_SHAPES}
    s_enc = torch.cuda.Stream(dev, priority=0)     # background: the encoder
    s_dec = torch.cuda.Stream(dev, priority=-1)    # latency-bound: the decoder

    def decode_step():
        for layer in dec_w:
            for (n, k), wt in zip(DECODER_SHAPES, layer):
                linear_bf16(dec_x[k], wt, out=dec_y[n], stream=s_dec)

    def timed(n_enc, n_dec):
        """n_enc forwards on s_enc and n_dec decode steps on s_dec, started together.
        Returns (ms of the encoder span, per-step decode ms list, ms of the whole)."""
        torch.cuda.synchronize(dev)
        start = torch.cuda.Event(enable_timing=True)
        start.record(torch.cuda.current_stream(dev))
        s_enc.wait_event(start)
        s_dec.wait_event(start)
        e_end = torch.cuda.Event(enable_timing=True)
        d_ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_dec + 1)]
        d_ev[0].record(s_dec)
        i_enc = i_dec = 0
        while i_enc < n_enc or i_dec < n_dec:   # interleave the host's enqueueing of the two streams
            if i_enc < n_enc:
                enc.forward(mel, lengths, out, s_enc)
                i_enc += 1
            for _ in range(2):
                if i_dec < n_dec:
                    decode_step()
                    i_dec += 1
                    d_ev[i_dec].record(s_dec)
        e_end.record(s_enc)
        torch.cuda.synchronize(dev)
        enc_ms = start.elapsed_time(e_end) if n_enc else 0.0
        dec = [d_ev[i].elapsed_time(d_ev[i + 1]) for i in range(n_dec)]
        whole = max(enc_ms, start.elapsed_time(d_ev[n_dec]) if n_dec else 0.0)
        return enc_ms, dec, whole

    for _ in range(max(args.warmup, 3)):
        enc.forward(mel, lengths, out, s_enc)
        decode_step()
    torch.cuda.synchronize(dev)
    n_enc = max(args.steps, 3)
    enc_alone, _, _ = timed(n_enc, 0)
    t_enc = enc_alone / n_enc
    _, dec_alone, _ = timed(0, 20)
    t_dec = statistics.median(dec_alone)
    n_dec = max(1, int(round(enc_alone / t_dec)))   # decode steps spanning the encoder's run
    enc_both, dec_both, whole = timed(n_enc, n_dec)
    enc.status(s_enc)
    enc.close()
    q = lambda v, f: sorted(v)[min(len(v) - 1, int(f * len(v)))]   # noqa: E731
    line = {"kernel": "sidestream", "workload": cfg.name,
            "decoder_stand_in": {"width": DECODER_WIDTH, "layers": DECODER_LAYERS, "tokens": DECODER_TOKENS,
                                 "gemms_per_layer": [f"{k}->{n}" for n, k in DECODER_SHAPES],
                                 "kernel": "enc_linear_bf16 (tcgen05 GEMM)", "stream_priority": "high"},
            "encoder": {"stream_priority": "low", "forwards": n_enc, "ms_alone": t_enc,
                        "ms_overlapped": enc_both / n_enc, "slowdown": (enc_both / n_enc) / t_enc,
                        "audio_s_per_s_alone": cfg.batch * cfg.frames / FRAMES_PER_SECOND / (t_enc / 1e3),
                        "audio_s_per_s_overlapped": cfg.batch * cfg.frames / FRAMES_PER_SECOND /
                        (enc_both / n_enc / 1e3)},
            "decoder": {"steps": n_dec, "ms_alone_median": t_dec, "ms_alone_p90": q(dec_alone, 0.9),
                        "ms_overlapped_median": statistics.median(dec_both), "ms_overlapped_p90": q(dec_both, 0.9),
                        "slowdown": statistics.median(dec_both) / t_dec},
            "ms_both_at_once": whole, "ms_sum_alone": n_enc * t_enc + n_dec * t_dec,
            "overlap_gain": (n_enc * t_enc + n_dec * t_dec) / whole}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="large_b16", choices=S.CONFIG_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=["qkv", "out", "fc1", "fc2", "attention", "frontend", "cache", "sidestream",
                                        "block"],
                    help="time one layer kernel of the workload alone (profiling aid)")
    args = ap.parse_args()
    cfg = S.CONFIGS[args.config]
    if args.kernel == "sidestream":
        return run_sidestream(args, cfg)
    if args.kernel:
        return run_kernel(args, cfg)
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch
    import torch.distributed as dist
    from audio_encoder_tower_b200 import Encoder

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- synthetic inputs and weights (per rank: own clips, same weights)
    w_np = S.make_weights(cfg.replace(seed=rank_weight_seed(cfg)))
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    w_dev = {k: torch.from_numpy(v).to(device=dev, dtype=dt) for k, v in w_np.items()}
    del w_np
    gcfg, clips, lengths = rank_clips(cfg, rank, world)
    mel_np = rank_mel(gcfg, clips)
    enc = Encoder(n_mels=cfg.n_mels, d_model=cfg.d_model, n_layers=cfg.n_layers, n_heads=cfg.n_heads,
                  ffn_dim=cfg.ffn_dim, max_frames=cfg.frames, max_batch=cfg.batch, dtype=cfg.dtype,
                  pool_step=cfg.pool_step, proj_hidden=cfg.proj_hidden, proj_out=cfg.proj_out,
                  attn_chunk=cfg.attn_chunk, weights=w_dev)
    del w_dev
    torch.cuda.empty_cache()
    mel = torch.from_numpy(mel_np).to(device=dev, dtype=dt)
    _, p_out, d_out = enc.output_positions(cfg.batch, lengths)
    out = torch.empty((cfg.batch, p_out, d_out), dtype=dt, device=dev)
    stream = torch.cuda.current_stream(dev)
    audio_s = float(np.sum(lengths)) / FRAMES_PER_SECOND
    flops = workload_flops(cfg, lengths)
    audio_s_job = sum_over_ranks(audio_s, world, dev)     # ragged clips: ranks differ in audio, not in cost
    flops_job = sum_over_ranks(flops, world, dev)

    # ---- device-resident timing (inputs in HBM when the region starts)
    for _ in range(args.warmup):
        enc.forward(mel, lengths, out, stream)
    enc.status(stream)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    n0 = enc.launch_count()
    e0.record(stream)
    for _ in range(args.steps):
        enc.forward(mel, lengths, out, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    launches = enc.launch_count() - n0
    clocks.stop()
    enc.status(stream)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)

    # ---- per-kernel-class breakdown: the same steps again with the library's
    # CUDA-event profiler on (kept out of the headline timing above)
    enc.profile(True)
    for _ in range(args.steps):
        enc.forward(mel, lengths, out, stream)
    torch.cuda.synchronize(dev)
    enc.profile(False)
    prof = enc.collect_profile()
    enc.status(stream)

    # ---- end to end through the public call with host buffers. Every step
    # copies its mel in from pinned host memory and its output back to pinned
    # host memory. Inputs and outputs are double-buffered and the copies run on
    # their own streams (one per direction), so a step's copies overlap the
    # neighbouring steps' forward passes, as a serving loop would run them.
    mel_host = torch.from_numpy(mel_np).to(dtype=dt).pin_memory()
    out_host = [torch.empty(out.shape, dtype=dt).pin_memory() for _ in range(2)]
    mel_in = [torch.empty_like(mel) for _ in range(2)]
    outs = [out, torch.empty_like(out)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # slot's mel landed on the device
    ev_fwd = [torch.cuda.Event() for _ in range(2)]   # slot's forward done: mel_in free, output ready
    ev_out = [torch.cuda.Event() for _ in range(2)]   # slot's output copied to the host: output free
    for k in range(2):
        ev_fwd[k].record(stream)
        ev_out[k].record(stream)
    step_no = [0]

    def e2e_step():
        k = step_no[0] % 2
        step_no[0] += 1
        s_in.wait_event(ev_fwd[k])
        with torch.cuda.stream(s_in):
            mel_in[k].copy_(mel_host, non_blocking=True)
        ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        stream.wait_event(ev_out[k])
        enc.forward(mel_in[k], lengths, outs[k], stream)
        ev_fwd[k].record(stream)
        s_out.wait_event(ev_fwd[k])
        with torch.cuda.stream(s_out):
            out_host[k].copy_(outs[k], non_blocking=True)
        ev_out[k].record(s_out)
        return k

    for _ in range(args.warmup):
        e2e_step()
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    last = 0
    for _ in range(args.steps):
        last = e2e_step()
    stream.wait_event(ev_out[last])   # the last output is on the host
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    enc.status(stream)
    if not np.all(np.isfinite(out_host[last][0, :10].float().numpy())):
        raise RuntimeError("non-finite encoder output")

    # ---- roofline of the dominant kernel (the tcgen05 GEMM, every GEMM launch of the region)
    peaks, peak_src = load_peaks()
    g_ms = sum(prof[k][0] for k in GEMM_CLASSES if k in prof)
    g_fl = sum(prof[k][1] for k in GEMM_CLASSES if k in prof)
    g_n = sum(prof[k][2] for k in GEMM_CLASSES if k in prof)
    step_ms_prof = sum(v[0] for v in prof.values())
    peak_tf = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    ach = (g_fl / g_n) / (g_ms / g_n) / 1e9 if g_n else 0.0
    traffic = gemm_traffic_record()
    roofline = {"kernel": ("tcgen05 GEMM: gemm_tc2_kernel on SM pairs where N % 256 == 0 (every GEMM of the "
                           "Whisper workloads), else gemm_tc_kernel; all GEMM launches of the timed region"),
                "bound": "tensor", "achieved": ach, "peak": peak_tf, "unit": "TFLOP/s", "frac": ach / peak_tf,
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)",
                "frac_of_burst_peak": ach / float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])),
                "traffic": (traffic["bytes_per_launch"] if traffic else None),
                "share_of_step": g_ms / step_ms_prof if step_ms_prof else None,
                "launches": g_n, "flops_per_launch": g_fl / g_n if g_n else None}
    kernels = {k: {"ms_per_step": v[0] / args.steps, "tflops": (v[1] / v[0] / 1e9 if v[0] and v[1] else None),
                   "share": v[0] / step_ms_prof} for k, v in prof.items()}

    tflops = flops_job / world / ms / 1e9     # per GPU
    line = {"metric": METRIC, "value": job_throughput(audio_s_job, ms), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded; random weights)",
            "config": workload_desc(cfg, world),
            "tflops": world * tflops,
            "frac_bf16_peak": tflops / float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])),
            "frac_bf16_peak_sustained": tflops / peak_tf,
            "frac_bf16_published_dense_peak": tflops / PUBLISHED_DENSE_BF16_TFLOPS,
            "peaks": f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback",
            "roofline": roofline,
            "kernels": kernels,
            "e2e": {"value": job_throughput(audio_s_job, ms_e2e), "unit": UNIT,
                    "h2d_bytes_per_step": int(mel_host.numel() * mel_host.element_size()),
                    "d2h_bytes_per_step": int(out_host[0].numel() * out_host[0].element_size()),
                    "ms_per_step": ms_e2e,
                    "api": "enc_forward (C ABI); pinned host copies in and out every step on two copy streams, double-buffered"},
            "gpu_launches": int(launches),
            "clocks": clocks.summary()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    enc.close()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
