"""Single-kernel parity on the GPU: the tcgen05 linear layer and the flash
attention kernel against the oracle's float64 steps (same bf16 inputs)."""
import numpy as np
import pytest

import oracle as O
import synthetic as S

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(7)


def _bf16(a):
    return S.round_bf16(np.asarray(a, np.float32))


def _dev(a, dtype=None):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype or torch.bfloat16)


# N % 256 == 0 runs 256 x 256 tiles on pairs of SMs: M = 129 leaves the second
# CTA of the pair one valid row, M = 257 starts a second tile row
@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (127, 256, 128), (128, 384, 64), (129, 256, 64), (257, 512, 64),
                                   (300, 1280, 1280), (1000, 512, 320), (4000, 3840, 1280)])
@pytest.mark.parametrize("gelu", [False, True])
def test_linear_bf16(M, N, K, gelu):
    import torch
    from audio_encoder_tower_b200.binding import linear_bf16
    A = _bf16(RNG.standard_normal((M, K)))
    W = _bf16(RNG.standard_normal((N, K)) * 0.05)
    b = RNG.standard_normal(N).astype(np.float32) * 0.1
    out = linear_bf16(_dev(A), _dev(W), _dev(b, torch.float32), gelu=gelu)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    ref = O.linear(A, W, b)
    if gelu:
        ref = O.gelu(ref)
    err = np.abs(got - ref)
    assert np.all(err <= 8e-3 * np.maximum(1.0, np.abs(ref))), float(err.max())


# reduce-add epilogue on pairs of SMs: a ragged second tile row (129) and a long K (5120)
@pytest.mark.parametrize("M,N,K", [(77, 256, 64), (129, 512, 512), (513, 1280, 5120)])
def test_linear_residual(M, N, K):
    import torch
    from audio_encoder_tower_b200.binding import linear_bf16
    A = _bf16(RNG.standard_normal((M, K)))
    W = _bf16(RNG.standard_normal((N, K)) * 0.02)
    b = RNG.standard_normal(N).astype(np.float32)
    x0 = RNG.standard_normal((M, N)).astype(np.float32)
    x = _dev(x0, torch.float32)
    linear_bf16(_dev(A), _dev(W), _dev(b, torch.float32), resid=x)
    torch.cuda.synchronize()
    got = x.cpu().numpy().astype(np.float64)
    ref = x0 + O.linear(A, W, b)
    assert np.abs(got - ref).max() < 1e-4 * max(1.0, np.abs(ref).max())


@pytest.mark.parametrize("lengths,heads,qscale", [([1, 77, 300], 2, 1.0), ([64, 128, 129], 1, 1.0),
                                                  ([1500], 3, 1.0), ([200, 513], 2, 6.0)])
def test_attention_bf16(lengths, heads, qscale):
    import torch
    from audio_encoder_tower_b200.binding import attention_bf16
    d = 64 * heads
    R = sum(lengths)
    q = _bf16(RNG.standard_normal((R, d)) * qscale)
    k = _bf16(RNG.standard_normal((R, d)))
    v = _bf16(RNG.standard_normal((R, d)))
    qkv = np.concatenate([q, k, v], axis=1)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    out = attention_bf16(_dev(qkv), _dev(cu, torch.int32), max(lengths), heads)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    for b, n in enumerate(lengths):
        s = slice(cu[b], cu[b + 1])
        ref = O.attention(q[s], k[s], v[s], heads, n)
        err = np.abs(got[s] - ref)
        # bf16 probabilities and bf16 output: a few 2^-8 of the value range
        assert err.max() < 3e-2, (b, float(err.max()))
        assert np.linalg.norm(got[s] - ref) / np.linalg.norm(ref) < 1e-2


def test_attention_bf16_late_large_scores():
    """Scores far above the row maximum taken over a segment's first key tile:
    every query shares a component u, and keys 250, 1100 and 1400 are 4u, 8u and
    30u, so their exponentials exceed that maximum's by factors of about 2^41,
    2^92 and 2^346. Each makes the row's sum for its key tile overflow the bound, so
    the row moves to a higher maximum and rescales what it has accumulated, the
    last time by more than 2^126 (the old values drop to zero). Compared with the
    oracle's softmax, which subtracts the exact maximum."""
    import torch
    from audio_encoder_tower_b200.binding import attention_bf16
    rng = np.random.default_rng(78)
    heads, lengths = 2, [300, 1500]
    d = 64 * heads
    R = sum(lengths)
    q = rng.standard_normal((R, d)) + 1.0
    k = rng.standard_normal((R, d))
    for pos, c in ((250, 4.0), (1100, 8.0), (1400, 30.0)):
        k[lengths[0] + pos] = c                     # c * u, u = all ones in every head
    q, k = _bf16(q), _bf16(k)
    v = _bf16(rng.standard_normal((R, d)))
    qkv = np.concatenate([q, k, v], axis=1)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    out = attention_bf16(_dev(qkv), _dev(cu, torch.int32), max(lengths), heads)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    for b, n in enumerate(lengths):
        s = slice(cu[b], cu[b + 1])
        ref = O.attention(q[s], k[s], v[s], heads, n)
        assert np.abs(got[s] - ref).max() < 3e-2, b
        assert np.linalg.norm(got[s] - ref) / np.linalg.norm(ref) < 1e-2, b


def test_attention_bf16_many_short_segments():
    """Segments of at most 192 positions (block-local attention) run as runs of
    work items per CTA (two CTAs per SM, each looping over its items): 700
    segments of 1 .. 190 positions x 2 heads is far more items than resident CTAs,
    so every CTA crosses item boundaries with odd and even tile counts, skipped
    query tiles and both score buffers. Every segment is compared with the oracle."""
    import torch
    from audio_encoder_tower_b200.binding import attention_bf16
    rng = np.random.default_rng(77)
    heads = 2
    d = 64 * heads
    lengths = rng.integers(1, 191, size=700).tolist()
    R = sum(lengths)
    q = _bf16(rng.standard_normal((R, d)))
    k = _bf16(rng.standard_normal((R, d)))
    v = _bf16(rng.standard_normal((R, d)))
    qkv = np.concatenate([q, k, v], axis=1)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    out = attention_bf16(_dev(qkv), _dev(cu, torch.int32), max(lengths), heads)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    worst = 0.0
    for b, n in enumerate(lengths):
        s = slice(cu[b], cu[b + 1])
        ref = O.attention(q[s], k[s], v[s], heads, n)
        worst = max(worst, float(np.abs(got[s] - ref).max()))
        assert np.linalg.norm(got[s] - ref) / np.linalg.norm(ref) < 1e-2, b
    assert worst < 3e-2, worst
