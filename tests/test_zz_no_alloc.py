"""enc_forward_static_scratch: the forward pass for callers that cannot
allocate device memory while they run (their device memory is handed out up
front by their own pool allocator). Its workspace lives in the library's fixed
64 MiB static device array; its output must match enc_forward's on the same
handle and inputs, on two calls in a row (the array keeps the previous call's
contents, so the second call checks that nothing stale leaks through).

Kept in a file of its own, collected last, so that a run stopping at the first
failure has already run every other test."""
import numpy as np
import pytest

import synthetic as S
from tests.encoder_cases import assert_parity, compare, make_encoder, to_device

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
    enc = make_encoder(cfg, to_device(cfg, S.make_weights(cfg)))
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    mel = torch.from_numpy(S.make_mel(cfg)).to("cuda", dt)
    ref = _host(enc.forward(mel, lengths))
    enc.status()
    n_out, p_out, d_out = enc.output_positions(cfg.batch, lengths)
    for call in range(2):
        out = torch.full((cfg.batch, p_out, d_out), float("nan"), dtype=dt, device="cuda")
        enc.forward_static_scratch(mel, lengths, out)
        enc.status()
        got = _host(out)
        for b in range(cfg.batch):
            assert_parity(cfg, compare(cfg, got[b], ref[b], int(n_out[b])))
    enc.close()


def test_static_scratch_rejects_batches_beyond_capacity():
    import torch
    from audio_encoder_tower_b200 import EncError
    # Whisper-large geometry, one block: one 30 s clip fits the 64 MiB array, two do not
    cfg = S.CONFIGS["large_b16"].replace(n_layers=1, batch=2)
    enc = make_encoder(cfg, to_device(cfg, S.make_weights(cfg)))
    mel = torch.from_numpy(S.make_mel(cfg)).to("cuda", torch.bfloat16)
    with pytest.raises(EncError) as ei:
        enc.forward_static_scratch(mel)
    assert ei.value.code == 1
    one = enc.forward_static_scratch(mel[:1])
    ref = enc.forward(mel[:1])
    enc.status()
    n_out, _, _ = enc.output_positions(1)
    assert_parity(cfg, compare(cfg, _host(one)[0], _host(ref)[0], int(n_out[0])))
    enc.close()
