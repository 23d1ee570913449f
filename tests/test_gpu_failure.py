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
