"""Device-side failure detection without a fault: a bounded wait inside a
kernel runs out (a phase that nothing completes), the kernel records
ENC_ERR_TIMEOUT in the handle's status word and returns, the host reads it,
and the context stays usable: the next forward is bit-identical to one before."""
import numpy as np
import pytest

import synthetic as S
from audio_encoder_tower_b200 import EncError
from audio_encoder_tower_b200.binding import ENC_ERR_INVALID_ARG, ENC_ERR_TIMEOUT
from tests.encoder_cases import make_encoder, run_gpu, to_device

pytestmark = pytest.mark.gpu


def test_timeout_is_reported_and_the_context_survives():
    import torch
    cfg = S.EncoderConfig(name="fail", n_mels=80, d_model=256, n_layers=1, n_heads=4, ffn_dim=512, frames=200,
                          batch=2, dtype="bf16", seed=13)
    lengths = np.array([200, 77], np.int32)
    enc = make_encoder(cfg, to_device(cfg, S.make_weights(cfg)))
    mel = S.make_mel(cfg)
    before = run_gpu(enc, cfg, mel, lengths)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    enc.selftest_timeout(2_000_000)            # 2 ms
    e1.record(stream)
    with pytest.raises(EncError) as ei:
        enc.status()
    assert ei.value.code == ENC_ERR_TIMEOUT
    ms = e0.elapsed_time(e1)
    # it waited out its limit, and the second warp left on the abort flag, not on its own 2 s limit
    assert 1.8 <= ms < 500.0, ms
    enc.status()                               # reading the word cleared it
    np.testing.assert_array_equal(run_gpu(enc, cfg, mel, lengths), before)
    for bad in (0, 999, 100_000_001):
        with pytest.raises(EncError) as ei:
            enc.selftest_timeout(bad)
        assert ei.value.code == ENC_ERR_INVALID_ARG
    enc.status()
    enc.close()


def test_allocation_failure_at_every_point_frees_everything(monkeypatch):
    """ENC_FAIL_ALLOC=N makes the N-th device allocation of one enc_create report
    failure: a host-side failure, no device fault. For every N up to the number of
    allocations a handle makes, enc_create returns ENC_ERR_OOM and leaves nothing
    allocated (the device's free memory is the same after the whole sweep); the
    counter restarts with every enc_create, and without the hook creation works."""
    import torch
    from audio_encoder_tower_b200.binding import ENC_ERR_OOM
    # a 30 s workspace, so that a leaked buffer would show in the free memory
    cfg = S.EncoderConfig(name="oom", n_mels=128, d_model=256, n_layers=2, n_heads=4, ffn_dim=1024, frames=3000,
                          batch=2, dtype="bf16", seed=14)
    w = to_device(cfg, S.make_weights(cfg))
    monkeypatch.delenv("ENC_FAIL_ALLOC", raising=False)
    make_encoder(cfg, w).close()               # modules loaded, runtime pools warm
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    failed = 0
    for n in range(1, 500):
        monkeypatch.setenv("ENC_FAIL_ALLOC", str(n))
        try:
            enc = make_encoder(cfg, w)
        except EncError as e:
            assert e.code == ENC_ERR_OOM, (n, e.code)
            failed += 1
            continue
        enc.close()                            # n is past the last allocation
        break
    else:
        pytest.fail("enc_create never got past the hook")
    monkeypatch.delenv("ENC_FAIL_ALLOC")
    assert failed >= 30                        # weights, biases, workspace: every one was a failure point
    torch.cuda.synchronize()
    assert abs(torch.cuda.mem_get_info()[0] - free0) < (8 << 20)
    enc = make_encoder(cfg, w)
    enc.close()


def test_guard_regions_report_a_changed_byte():
    """ENC_FLAG_GUARD: a forward leaves every guard region intact, and a guard
    byte changed from the host (no kernel, no fault) on either side of a buffer
    is reported with the buffer's name, then the restored guard passes again."""
    cfg = S.EncoderConfig(name="guard", n_mels=80, d_model=256, n_layers=1, n_heads=4, ffn_dim=512, frames=200,
                          batch=2, dtype="bf16", seed=15)
    enc = make_encoder(cfg, to_device(cfg, S.make_weights(cfg)), guard=True)
    run_gpu(enc, cfg, S.make_mel(cfg), np.array([200, 77], np.int32))    # checks the guards
    for buffer, offset in [(0, -1), (0, 1), (2, -262144), (2, 262144), (4, 17), (4, -4096)]:
        enc.guard_selftest(buffer, offset)
    enc.check_guards()
    with pytest.raises(EncError):
        enc.guard_selftest(0, 0)                # offset 0 is inside the buffer
    enc.close()
    plain = make_encoder(cfg, to_device(cfg, S.make_weights(cfg)), guard=False)
    with pytest.raises(EncError):
        plain.check_guards()                    # no guards on this handle
    plain.close()
