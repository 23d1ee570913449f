"""Embeddings cache (include/enc_cache.h) on the GPU: hits return exactly what
enc_forward computes for the clip (bit for bit: the encoder's result for a clip
does not depend on its batch), repeated keys are computed once, the least
recently used entry is replaced when the cache is full."""
import numpy as np
import pytest

import synthetic as S
from tests.encoder_cases import make_encoder, to_device

pytestmark = pytest.mark.gpu


def _setup(capacity):
    import torch
    from audio_encoder_tower_b200 import Cache
    cfg = S.EncoderConfig(name="cache", n_mels=80, d_model=256, n_layers=2, n_heads=4, ffn_dim=512, frames=300,
                          batch=4, dtype="bf16", seed=21)
    enc = make_encoder(cfg, to_device(cfg, S.make_weights(cfg)))
    mel = torch.from_numpy(S.make_mel(cfg.replace(batch=6))).to(device="cuda", dtype=torch.bfloat16)
    return cfg, enc, mel, Cache(enc, capacity)


def test_hits_equal_fresh_forward_bit_for_bit():
    import torch
    cfg, enc, mel, cache = _setup(8)
    lengths = np.array([300, 201, 77, 300, 150, 9], np.int32)
    sel = [0, 1, 2]
    out, hits = cache.forward(mel[sel].contiguous(), keys=[10, 11, 12], lengths=lengths[sel])
    ref = enc.forward(mel[sel].contiguous(), lengths[sel])
    torch.cuda.synchronize()
    assert list(hits) == [0, 0, 0] and cache.size() == 3
    assert torch.equal(out, ref)
    sel = [1, 3, 0, 3]                                   # keys 11 and 10 hit; key 13 twice, computed once
    out, hits = cache.forward(mel[sel].contiguous(), keys=[11, 13, 10, 13], lengths=lengths[sel])
    ref = enc.forward(mel[sel].contiguous(), lengths[sel])
    torch.cuda.synchronize()
    assert list(hits) == [1, 0, 1, 0] and cache.size() == 4
    assert torch.equal(out, ref)
    enc.status()
    cache.close()
    enc.close()


def test_least_recently_used_is_replaced():
    import torch
    cfg, enc, mel, cache = _setup(2)
    one = lambda i, key: cache.forward(mel[i:i + 1].contiguous(), keys=[key])[1][0]   # noqa: E731
    assert one(0, 1) == 0 and one(1, 2) == 0 and cache.size() == 2
    assert one(0, 1) == 1                                # key 1 used last: key 2 is now the oldest
    assert one(2, 3) == 0 and cache.size() == 2          # replaces key 2
    assert one(0, 1) == 1 and one(1, 2) == 0             # key 2 was dropped, key 1 kept
    out, _ = cache.forward(mel[2:3].contiguous(), keys=[3])   # key 3 was replaced by key 2 just now
    ref = enc.forward(mel[2:3].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    enc.status()
    cache.close()
    enc.close()


def test_argument_errors():
    from audio_encoder_tower_b200 import Cache, EncError
    cfg, enc, mel, cache = _setup(2)
    with pytest.raises(EncError):
        cache.forward(mel[:5].contiguous(), keys=[1, 2, 3, 4, 5])          # B > max_batch
    with pytest.raises(EncError):
        cache.forward(mel[:1].contiguous(), keys=[1], lengths=[301])       # length > T
    with pytest.raises(EncError):
        Cache(enc, 0)
    # B = 0 with valid pointers
    import ctypes
    import torch
    _, p_out, d_out = enc.output_positions(1)
    out = mel.new_zeros((1, p_out, d_out))
    keys = np.zeros(1, np.uint64)
    kp = keys.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64))
    stream = torch.cuda.current_stream().cuda_stream
    assert cache.lib.enc_forward_cached(cache.h, mel.data_ptr(), None, kp, 0, out.data_ptr(), None, stream) == 1
    assert cache.lib.enc_cache_content_keys(cache.h, mel.data_ptr(), None, 0, kp, stream) == 1
    assert cache.size() == 0
    cache.close()
    enc.close()


def test_content_keys():
    """enc_cache_content_keys: equal clips (same length, same valid frames) get
    equal keys and hit; one changed valid frame changes the key (a miss); frames
    past the length change neither the key nor the output; a cached output matches
    the CPU oracle within the bf16 tolerance."""
    import torch
    from tests.encoder_cases import assert_parity, compare, oracle_clip
    cfg, enc, mel, cache = _setup(8)
    w = S.make_weights(cfg)
    mel_np = S.make_mel(cfg.replace(batch=6))
    lengths = np.array([300, 201, 77, 201], np.int32)
    sel = mel[[0, 1, 2, 1]].contiguous()
    keys = cache.content_keys(sel, lengths)
    assert keys[1] == keys[3] and len(set(keys[:3].tolist())) == 3
    past = sel.clone()
    past[1, :, 201:] = 5.0                          # frames past clip 1's length
    assert np.array_equal(cache.content_keys(past, lengths), keys)
    assert cache.content_keys(sel, [300, 200, 77, 201])[1] != keys[1]      # the length enters the key
    one = sel.clone()
    one[2, 40, 13] = one[2, 40, 13] + 0.5           # one valid frame of clip 2
    k2 = cache.content_keys(one, lengths)
    assert k2[2] != keys[2] and np.array_equal(k2[[0, 1, 3]], keys[[0, 1, 3]])
    out, hits = cache.forward(sel, None, lengths)   # keys from content: clip 3 repeats clip 1
    assert list(hits) == [0, 0, 0, 0] and cache.size() == 3
    out2, hits2 = cache.forward(past, None, lengths)
    assert list(hits2) == [1, 1, 1, 1]
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
    _, hits3 = cache.forward(one, None, lengths)
    assert list(hits3) == [1, 1, 0, 1]
    got = out2.float().cpu().numpy().astype(np.float64)
    for b, src in ((1, 1), (2, 2)):
        n = (int(lengths[b]) + 1) // 2
        assert_parity(cfg, compare(cfg, got[b], oracle_clip(cfg, w, mel_np[src], lengths[b]), n))
    enc.status()
    cache.close()
    enc.close()


def _content_key(mel_clip_bits: np.ndarray, length: int, frames: int) -> int:
    """The documented content key, restated on the host: the sum modulo 2^64 of
    the SplitMix64 mix of ((c * T + t) << 32 | value bits) + golden over the
    valid frames t < length, mixed with the mix of length * golden."""
    mask = (1 << 64) - 1
    g = 0x9E3779B97F4A7C15

    def mix(z):
        z &= mask
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & mask
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & mask
        return z ^ (z >> 31)

    n_mels = mel_clip_bits.shape[0]
    idx = (np.arange(n_mels, dtype=np.uint64)[:, None] * np.uint64(frames)
           + np.arange(length, dtype=np.uint64)[None, :])
    words = (idx << np.uint64(32)) | mel_clip_bits[:, :length].astype(np.uint64)
    z = (words + np.uint64(g))                        # wraps modulo 2^64
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    z = z ^ (z >> np.uint64(31))
    total = int(np.sum(z, dtype=np.uint64))           # modulo 2^64
    return mix(total ^ mix(length * g))


def test_content_keys_match_their_definition():
    """The device's content keys equal the documented hash computed on the host,
    bit for bit, for full and ragged clips."""
    import torch
    cfg, enc, mel, cache = _setup(8)
    lengths = np.array([300, 1, 177, 64], np.int32)
    sel = mel[:4].contiguous()
    keys = cache.content_keys(sel, lengths)
    bits = sel.view(torch.int16).cpu().numpy().view(np.uint16)
    for b in range(4):
        assert int(keys[b]) == _content_key(bits[b], int(lengths[b]), cfg.frames), b
    cache.close()
    enc.close()
