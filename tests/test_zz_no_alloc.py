"""enc_forward_static_scratch: the forward pass for callers that cannot
allocate device memory while they run, such as a serving process whose device
memory is handed out up front by its own pool allocator (a cudaMalloc there
would fail, or break the pool's accounting). Its workspace lives in the
library's fixed 64 MiB static device array, reserved when enc_create resolves
the array's address. Checked here through the C ABI:

* its output equals enc_forward's bit for bit on the same handle and inputs,
  on two calls in a row (the array keeps the previous call's contents, so the
  second call shows that nothing stale leaks through), and matches the CPU
  oracle within the workload tolerance;
* the calls leave the device's free memory unchanged, the first call on a
  fresh handle included;
* a batch whose workspace exceeds 64 MiB is rejected before anything runs.

Kept in a file of its own, collected last, so that a run stopping at the first
failure has already run every other test."""
import numpy as np
import pytest

import synthetic as S
from tests.encoder_cases import assert_parity, compare, make_encoder, oracle_clip, to_device

pytestmark = pytest.mark.gpu


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)


CASES = [
    (S.EncoderConfig("na_bf16", n_mels=80, d_model=256, n_layers=2, n_heads=4, ffn_dim=512, frames=333, batch=3,
                     dtype="bf16", seed=21), [333, 200, 1]),
    (S.EncoderConfig("na_bf16_pool_proj", n_mels=128, d_model=256, n_layers=1, n_heads=4, ffn_dim=512, frames=301,
                     batch=2, dtype="bf16", seed=22, pool_step=2, proj_hidden=384, proj_out=256), [301, 77]),
    (S.CONFIGS["tiny_fp32"], [200]),
]


@pytest.mark.parametrize("cfg,lengths", CASES, ids=[c.name for c, _ in CASES])
def test_static_scratch_matches_enc_forward(cfg, lengths):
    import torch
    lengths = np.array(lengths, np.int32)
    w = S.make_weights(cfg)
    enc = make_encoder(cfg, to_device(cfg, w))
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    mel_np = S.make_mel(cfg)
    mel = torch.from_numpy(mel_np).to("cuda", dt)
    ref = _host(enc.forward(mel, lengths))
    enc.status()
    n_out, p_out, d_out = enc.output_positions(cfg.batch, lengths)
    outs = [torch.full((cfg.batch, p_out, d_out), float("nan"), dtype=dt, device="cuda") for _ in range(2)]
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for call in range(2):
        enc.forward_static_scratch(mel, lengths, outs[call])
        enc.status()
        np.testing.assert_array_equal(_host(outs[call]), ref)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "enc_forward_static_scratch changed the device's free memory"
    enc.close()
    # and against the CPU oracle
    got = _host(outs[1])
    for b, ln in enumerate(lengths):
        assert_parity(cfg, compare(cfg, got[b], oracle_clip(cfg, w, mel_np[b], ln), int(n_out[b])))


def test_static_scratch_rejects_batches_beyond_capacity():
    import torch
    from audio_encoder_tower_b200 import EncError
    # Whisper-large geometry, one block: one 30 s clip fits the 64 MiB array, two do not
    cfg = S.CONFIGS["large_b16"].replace(n_layers=1, batch=2)
    enc = make_encoder(cfg, to_device(cfg, S.make_weights(cfg)))
    mel = torch.from_numpy(S.make_mel(cfg)).to("cuda", torch.bfloat16)
    _, p_out, d_out = enc.output_positions(2)
    out = torch.empty((2, p_out, d_out), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(EncError) as ei:
        enc.forward_static_scratch(mel, None, out)
    assert ei.value.code == 1
    one = enc.forward_static_scratch(mel[:1], None, out[:1])
    ref = enc.forward(mel[:1])
    enc.status()
    np.testing.assert_array_equal(_host(one), _host(ref))
    enc.close()
