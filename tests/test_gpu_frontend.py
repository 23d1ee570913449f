"""Log-mel front end on the GPU (include/enc_frontend.h) against the float64
oracle (oracle/frontend.py) on the same seeded audio.

Tolerance (fp32 output): the DFT runs in fp32 over 400 products per bin, so a
mel value carries a relative error of about 1e-6 and its log10 a few 1e-7;
values pushed below the 8-decade clamp agree exactly once clamped. 2e-4
absolute on the normalised features leaves a wide margin; bf16 output adds its
own rounding (one bf16 step is 2^-7 for values of magnitude 1 to 2)."""
import numpy as np
import pytest

import synthetic as S
from oracle import frontend as F

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def audio():
    return S.make_audio(3)


@pytest.mark.parametrize("n_mels,dtype", [(128, "fp32"), (80, "fp32"), (128, "bf16")])
def test_log_mel_parity(audio, n_mels, dtype):
    import torch
    from audio_encoder_tower_b200 import Frontend
    fe = Frontend(n_mels=n_mels, max_batch=4)
    got = fe.log_mel(torch.from_numpy(audio).cuda(), dtype=dtype)
    torch.cuda.synchronize()
    got = got.float().cpu().numpy().astype(np.float64)
    fe.close()
    assert got.shape == (3, n_mels, 3000)
    tol_abs, tol_rel = (2e-4, 1e-5) if dtype == "fp32" else (2.0 ** -7, 4e-3)
    for b in range(3):
        ref = F.log_mel(audio[b].astype(np.float64), n_mels)
        err = np.abs(got[b] - ref)
        assert err.max() <= tol_abs, (b, float(err.max()))
        assert np.linalg.norm(got[b] - ref) / np.linalg.norm(ref) <= tol_rel, b
    # the silent last two seconds of clip 1 sit exactly at the clamp (the clip's minimum)
    assert np.all(got[1][:, -150:] == got[1].min())


def test_silence_and_argument_errors():
    import torch
    from audio_encoder_tower_b200 import EncError, Frontend
    fe = Frontend(n_mels=80, max_batch=2)
    z = torch.zeros((2, 480000), dtype=torch.float32, device="cuda")
    out = fe.log_mel(z, dtype="fp32")
    torch.cuda.synchronize()
    assert torch.all(out == -1.5)                       # log10(1e-10) = -10 -> (-10 + 4) / 4
    with pytest.raises(EncError):
        fe.log_mel(torch.zeros((3, 480000), dtype=torch.float32, device="cuda"))   # B > max_batch
    out = torch.full((1, 80, 3000), 3.0, dtype=torch.bfloat16, device="cuda")   # B = 0, valid pointers
    assert fe.lib.enc_frontend_log_mel(fe.h, z.data_ptr(), 0, out.data_ptr(), 0,
                                       torch.cuda.current_stream().cuda_stream) == 1
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)
    fe.close()
    with pytest.raises(EncError):
        Frontend(n_mels=64)


def test_front_end_feeds_the_encoder(audio):
    """The front end's bf16 output is the encoder's input layout: a small encoder
    runs on it and matches the oracle tower run on the oracle's own features
    (oracle.frontend.log_mel rounded to bf16), within the workloads' bf16
    tolerance (relative Frobenius <= 1e-2, max-abs <= 5e-2). The two feature sets
    differ by at most one bf16 step, so this also bounds how such differences
    propagate through the tower."""
    import torch
    import oracle as O
    from audio_encoder_tower_b200 import Frontend
    from tests.encoder_cases import assert_parity, compare, make_encoder, run_gpu, to_device
    cfg = S.EncoderConfig(name="fe", n_mels=128, d_model=256, n_layers=2, n_heads=4, ffn_dim=512, frames=3000,
                          batch=1, dtype="bf16", seed=12)
    w = S.make_weights(cfg)
    fe = Frontend(n_mels=cfg.n_mels, max_batch=1)
    mel = fe.log_mel(torch.from_numpy(audio[:1]).cuda(), dtype="bf16")
    torch.cuda.synchronize()
    mel_np = mel.float().cpu().numpy()
    fe.close()
    enc = make_encoder(cfg, to_device(cfg, w))
    got = run_gpu(enc, cfg, mel_np, np.array([3000], np.int32))
    enc.close()
    feats = S.round_bf16(F.log_mel(audio[0].astype(np.float64), cfg.n_mels).astype(np.float32))
    ref = O.encode_clip(cfg, w, feats.astype(np.float64), 3000)
    assert_parity(cfg, compare(cfg, got[0], ref, 1500))
