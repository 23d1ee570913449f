"""The shard planner of the C ABI (include/enc_shard.h): host-only calls, run
here without a GPU. The cost of a clip is pinned to a hand-computed FLOP count
and to bench.py's own formula; the plan is checked for what every plan must
satisfy (each clip once, capacity, order within a rank, loads that add up) and
against the optimum found by brute force on tiny batches."""
import ctypes
import itertools

import numpy as np
import pytest

import bench
import synthetic as S
from audio_encoder_tower_b200 import EncError, binding, build, clip_flops, encoder_config, shard_plan
from audio_encoder_tower_b200.binding import ENC_ERR_INVALID_ARG, ENC_ERR_UNSUPPORTED


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    return binding.load_library()


def cfg_of(c, max_batch=None):
    return bench.tower_config(c, max_batch)


TINY = S.EncoderConfig(name="shard", n_mels=8, d_model=128, n_layers=1, n_heads=2, ffn_dim=128, frames=40,
                       batch=4, dtype="bf16", seed=11)


def test_clip_flops_closed_form():
    # len 3 -> n 2 positions; d 128, 8 mel, F 128, one layer, no chunks, no projector
    #   conv1 2*4*128*3*8 = 24,576        conv2 2*2*128*384 = 196,608
    #   QKV 6*2*128^2 = 196,608   attention 4*2^2*128 = 2,048
    #   out 2*2*128^2 = 65,536    FFN 4*2*128*128 = 131,072
    assert clip_flops(cfg_of(TINY), 3) == 24576 + 196608 + 196608 + 2048 + 65536 + 131072
    # odd and even lengths share a position count
    assert clip_flops(cfg_of(TINY), 4) == clip_flops(cfg_of(TINY), 3)


@pytest.mark.parametrize("name", S.CONFIG_ORDER)
def test_clip_flops_matches_the_workload_formula(name):
    c = S.CONFIGS[name]
    for ln in (1, 2, 99, 100, 101, c.frames - 1, c.frames):
        assert clip_flops(cfg_of(c), ln) == pytest.approx(bench.workload_flops(c, [ln]), rel=1e-12)


def test_chunked_attention_cost_is_per_chunk():
    c = TINY.replace(attn_chunk=3)
    full, chunked = clip_flops(cfg_of(TINY), 40), clip_flops(cfg_of(c), 40)
    # 20 positions: one 20^2 segment against six chunks of 3 and one of 2
    assert full - chunked == 4 * 128 * (20 ** 2 - (6 * 9 + 4))


def _check_plan(lengths, world, cap, rank_of, index_of, count, flops, cfg):
    B = len(lengths)
    assert rank_of.min() >= 0 and rank_of.max() < world
    assert count.tolist() == np.bincount(rank_of, minlength=world).tolist()
    assert count.max() <= cap
    for r in range(world):
        mine = np.flatnonzero(rank_of == r)
        assert index_of[mine].tolist() == list(range(len(mine)))   # a rank keeps the input order
        assert flops[r] == pytest.approx(sum(clip_flops(cfg, int(lengths[b])) for b in mine), rel=1e-12)
    assert flops.sum() == pytest.approx(sum(clip_flops(cfg, int(x)) for x in lengths), rel=1e-12)
    assert B == count.sum()


def test_full_length_clips_go_round_robin():
    cfg = cfg_of(TINY)
    rank_of, index_of, count, flops = shard_plan(cfg, 10, 3)
    assert rank_of.tolist() == [b % 3 for b in range(10)]
    assert count.tolist() == [4, 3, 3]
    _check_plan(np.full(10, 40), 3, 4, rank_of, index_of, count, flops, cfg)


def test_plan_is_deterministic_and_valid_on_ragged_batches():
    rng = np.random.default_rng(0)
    for world, cap, B in [(2, 8, 16), (3, 5, 13), (8, 16, 128), (4, 64, 100), (1, 7, 7)]:
        cfg = cfg_of(TINY, cap)
        lengths = rng.integers(1, 41, size=B).astype(np.int32)
        a = shard_plan(cfg, lengths, world)
        b = shard_plan(cfg, lengths, world)
        for x, y in zip(a, b):
            assert (x == y).all()
        _check_plan(lengths, world, cap, *a, cfg)


def _optimum(costs, world, cap):
    best = float("inf")
    for assign in itertools.product(range(world), repeat=len(costs)):
        if max(np.bincount(assign, minlength=world)) > cap:
            continue
        load = [0.0] * world
        for c, r in zip(costs, assign):
            load[r] += c
        best = min(best, max(load))
    return best


def test_makespan_against_brute_force():
    # Without a binding capacity the longest-first rule is within 4/3 - 1/(3m) of the
    # optimum (Graham's bound for longest-processing-time scheduling); here it is
    # checked against the optimum itself, found by brute force. With a binding
    # capacity (ceil(B / m) clips per rank) the plan must stay feasible; on these
    # fixed seeded batches it also stays within the same factor of that optimum.
    rng = np.random.default_rng(1)
    cfg_free = cfg_of(TINY.replace(frames=3000), 64)
    for trial in range(12):
        world = 2 + trial % 2
        B = 5 + trial % 4
        lengths = rng.integers(1, 3001, size=B).astype(np.int32)
        costs = [clip_flops(cfg_free, int(x)) for x in lengths]
        _, _, _, flops = shard_plan(cfg_free, lengths, world)
        assert flops.max() <= (4 / 3 - 1 / (3 * world)) * _optimum(costs, world, B) * (1 + 1e-12)
        cap = -(-B // world)
        cfg_cap = cfg_of(TINY.replace(frames=3000), cap)
        rank_of, index_of, count, flops = shard_plan(cfg_cap, lengths, world)
        _check_plan(lengths, world, cap, rank_of, index_of, count, flops, cfg_cap)
        assert flops.max() <= (4 / 3 - 1 / (3 * world)) * _optimum(costs, world, cap) * (1 + 1e-12)


def test_ragged_whisper_large_batch_balances():
    # 8 ranks x 64 clips of U[500, 3000] frames (the ragged Whisper-large workload)
    c = S.CONFIGS["large_ragged_b64"]
    g = c.replace(batch=8 * c.batch)
    lengths = S.make_lengths(g)
    _, _, count, flops = shard_plan(cfg_of(c), lengths, 8)
    assert count.tolist() == [c.batch] * 8
    assert flops.max() / flops.min() < 1.001
    # an index split (clips 64r .. 64r+63) is visibly worse on the same lengths
    naive = [bench.workload_flops(c, lengths[r * c.batch:(r + 1) * c.batch]) for r in range(8)]
    assert max(naive) / flops.max() > 1.04


def test_argument_errors():
    cfg = cfg_of(TINY)
    with pytest.raises(EncError) as e:
        shard_plan(cfg, 9, 2)                   # 9 clips > 2 ranks x 4
    assert e.value.code == ENC_ERR_INVALID_ARG
    for world in (0, -1):
        with pytest.raises(EncError) as e:
            shard_plan(cfg, 2, world)
        assert e.value.code == ENC_ERR_INVALID_ARG
    for bad in ([0, 5], [5, 41], [-3, 5]):
        with pytest.raises(EncError) as e:
            shard_plan(cfg, bad, 2)
        assert e.value.code == ENC_ERR_INVALID_ARG
    with pytest.raises(EncError) as e:
        clip_flops(cfg, 41)
    assert e.value.code == ENC_ERR_INVALID_ARG
    bad_cfg = encoder_config(n_mels=8, d_model=128, n_layers=1, n_heads=4, head_dim=32, ffn_dim=128,
                             max_frames=40, max_batch=4)
    with pytest.raises(EncError) as e:
        clip_flops(bad_cfg, 10)
    assert e.value.code == ENC_ERR_UNSUPPORTED
    lib = binding.load_library()
    i32 = np.zeros(4, np.int32)
    i32p = ctypes.POINTER(ctypes.c_int32)
    # a NULL rank_of, a NULL config, a NULL flops pointer
    assert lib.enc_shard_plan(ctypes.byref(cfg), None, 2, 2, None, None, None, None) == ENC_ERR_INVALID_ARG
    assert lib.enc_shard_plan(None, None, 2, 2, i32.ctypes.data_as(i32p), None, None, None) == ENC_ERR_INVALID_ARG
    assert lib.enc_clip_flops(ctypes.byref(cfg), 10, None) == ENC_ERR_INVALID_ARG
    # nothing written on an error
    out = np.full(4, -7, np.int32)
    assert lib.enc_shard_plan(ctypes.byref(cfg), None, 9, 2, out.ctypes.data_as(i32p), None, None,
                              None) == ENC_ERR_INVALID_ARG
    assert (out == -7).all()


def test_plan_properties_on_random_batches():
    hyp = pytest.importorskip("hypothesis")
    st = pytest.importorskip("hypothesis.strategies")

    @hyp.settings(max_examples=150, deadline=None, derandomize=True)
    @hyp.given(world=st.integers(1, 9), cap=st.integers(1, 12), data=st.data())
    def check(world, cap, data):
        B = data.draw(st.integers(1, world * cap))
        lengths = np.array(data.draw(st.lists(st.integers(1, 40), min_size=B, max_size=B)), np.int32)
        cfg = cfg_of(TINY, cap)
        rank_of, index_of, count, flops = shard_plan(cfg, lengths, world)
        _check_plan(lengths, world, cap, rank_of, index_of, count, flops, cfg)
        # without a binding capacity (max_batch >= B) every clip goes onto the rank that
        # is least loaded at that moment, so the most loaded rank ends at most the cost
        # of its last clip above the final minimum
        free = cfg_of(TINY, B)
        _, _, _, f_free = shard_plan(free, lengths, world)
        costs = np.array([clip_flops(free, int(x)) for x in lengths])
        assert f_free.max() - f_free.min() <= costs.max() * (1 + 1e-12)

    check()
