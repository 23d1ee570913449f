"""Pins of the bf16 rounding-point model (oracle/bf16_model.py), CPU only.

The model is the oracle's computation with bf16 rounding at the points where a
tensor-core implementation stores 16-bit values. Its error against the exact
oracle is the band that bounds the GPU's error on the stress case (weights ten
times the workloads' scale), where bf16 rounding alone exceeds the workloads'
1e-2 relative tolerance."""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from oracle.bf16_model import encode_clip_bf16, round_bf16


def _small(name, **kw):
    base = dict(name=name, n_mels=80, d_model=256, n_layers=2, n_heads=4, ffn_dim=512, frames=333, batch=3,
                dtype="bf16", seed=11)
    base.update(kw)
    return S.EncoderConfig(**base)


PEAKY = (_small("peaky", weight_std=0.2, frames=260), [260, 131, 65])
STANDARD = (_small("small_ragged"), [333, 200, 1])


def _errors(cfg, lengths, rounding=True):
    w = S.make_weights(cfg)
    mel = S.make_mel(cfg)
    out = []
    for b, ln in enumerate(lengths):
        n = O.valid_output_rows(cfg, ln)
        ref = O.encode_clip(cfg, w, mel[b], ln)[:n]
        got = encode_clip_bf16(cfg, w, mel[b], ln, rounding)[:n]
        out.append((float(np.linalg.norm(got - ref) / np.linalg.norm(ref)), float(np.abs(got - ref).max())))
    return out


def test_rounding_is_torch_bfloat16():
    """round_bf16 equals PyTorch's float32 -> bfloat16 conversion (nearest, ties to even)."""
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 1.0 + 2 ** -9, 1.0 + 3 * 2 ** -9, 65504.0]])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(round_bf16(x), ref)
    # ties go to the even neighbour: 1 + 2^-8 (halfway) -> 1, 1 + 3*2^-8 -> 1 + 2^-6
    assert round_bf16(np.array([1.0 + 2 ** -8]))[0] == 1.0
    assert round_bf16(np.array([1.0 + 3 * 2 ** -8]))[0] == 1.0 + 2 ** -6


@pytest.mark.parametrize("case", [PEAKY, STANDARD], ids=["peaky", "standard"])
def test_without_rounding_the_model_is_the_oracle(case):
    cfg, lengths = case
    for rel, mx in _errors(cfg, lengths, rounding=False):
        assert rel < 1e-12 and mx < 1e-11


def test_model_variants_reduce_to_the_oracle():
    """Pool, projector and block-local attention follow the oracle too."""
    for cfg, lengths in [(_small("pp", pool_step=2, proj_hidden=256, proj_out=128, frames=120), [120, 51, 4]),
                         (_small("ck", attn_chunk=7, frames=90), [90, 33, 2])]:
        for rel, mx in _errors(cfg, lengths, rounding=False):
            assert rel < 1e-12 and mx < 1e-11


def test_band_at_the_workloads_scale_is_inside_the_tolerance():
    """At N(0, 0.02) weights bf16 rounding alone costs about 0.2%: the workloads'
    1e-2 / 5e-2 tolerance leaves a five-fold margin for accumulation order and
    the approximate exponentials."""
    for rel, mx in _errors(*STANDARD):
        assert 5e-4 < rel < 2e-3 and mx < 1e-2


def test_band_of_the_stress_case():
    """At N(0, 0.2) weights bf16 rounding alone costs 1.5-1.9%: above the
    workloads' 1e-2, which is why the stress case has its own bound, computed from
    this model in the GPU test."""
    errs = _errors(*PEAKY)
    for rel, mx in errs:
        assert 1.2e-2 < rel < 2.2e-2 and 0.08 < mx < 0.25
    # rounding the probabilities contributes: without it the band shrinks
    import oracle.bf16_model as M
    keep = M._attention
    try:
        M._attention = lambda q, k, v, h, hd, rb: keep(q, k, v, h, hd, lambda x: np.asarray(x, np.float64))
        no_p = _errors(*PEAKY)
    finally:
        M._attention = keep
    assert all(a[0] != b[0] for a, b in zip(errs, no_p))
