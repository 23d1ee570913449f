"""Planted mistakes in the oracle (on the CPU) must be caught by the pins.

Each case swaps one oracle step for a plausible wrong variant and checks that
the independent torch.nn composition used in test_oracle_pins disagrees.
"""
import math

import numpy as np
import pytest

import oracle.encoder as E
from tests.test_oracle_pins import Geo, _rand_weights, _torch_tower

RNG = np.random.default_rng(99)


def _tanh_gelu(x):
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))


def _cos_first(p, c, max_timescale=10000.0):
    half = c // 2
    inv = np.exp(-math.log(max_timescale) / (half - 1) * np.arange(half))
    ang = np.arange(p)[:, None] * inv[None]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1)


def _interleaved(p, c, max_timescale=10000.0):
    half = c // 2
    inv = np.exp(-math.log(max_timescale) / (half - 1) * np.arange(half))
    ang = np.arange(p)[:, None] * inv[None]
    out = np.empty((p, c)); out[:, 0::2] = np.sin(ang); out[:, 1::2] = np.cos(ang)
    return out


def _ln_unbiased(x, g, b, eps=1e-5):
    x = np.asarray(x, np.float64)
    mu = x.mean(-1, keepdims=True)
    var = ((x - mu) ** 2).sum(-1, keepdims=True) / (x.shape[-1] - 1)
    return (x - mu) / np.sqrt(var + eps) * g + b


def _ln_eps_outside(x, g, b, eps=1e-5):
    x = np.asarray(x, np.float64)
    mu = x.mean(-1, keepdims=True)
    return (x - mu) / (np.sqrt(((x - mu) ** 2).mean(-1, keepdims=True)) + eps) * g + b


def _attn_scale_hd(q, k, v, n_heads, n_valid=None, head_dim=64):
    return _ORIG_ATTN(q * (1.0 / math.sqrt(head_dim)), k, v, n_heads, n_valid, head_dim)


def _stem_no_frame_mask(mel, length, w):                            # frames past the clip kept
    return _ORIG_STEM(mel, mel.shape[1], w)


def _stem_trailing_rows(mel, length, w):                           # clip run alone, not zero padded
    y = _ORIG_STEM(mel[:, :length], length, w)
    full = _ORIG_STEM(mel, length, w)
    full[: y.shape[0]] = y
    return full


def _conv_shifted(x, w, b, stride):
    y = _ORIG_CONV(x, w, b, stride)
    return np.roll(y, 1, axis=1)


def _post_ln_layer(x, lw, n_heads, eps, head_dim=64, attn_chunk=0):
    q = E.linear(x, lw["q_w"], lw["q_b"]); k = E.linear(x, lw["k_w"], None); v = E.linear(x, lw["v_w"], lw["v_b"])
    x = E.layer_norm(x + E.linear(E.attention(q, k, v, n_heads, None, head_dim), lw["o_w"], lw["o_b"]),
                     lw["ln1_g"], lw["ln1_b"], eps)
    return E.layer_norm(x + E.linear(E.gelu(E.linear(x, lw["fc1_w"], lw["fc1_b"])), lw["fc2_w"], lw["fc2_b"]),
                        lw["ln2_g"], lw["ln2_b"], eps)


def _k_biased_layer(x, lw, n_heads, eps, head_dim=64, attn_chunk=0):
    lw = dict(lw); lw["k_b"] = lw["q_b"]
    a = E.layer_norm(x, lw["ln1_g"], lw["ln1_b"], eps)
    q = E.linear(a, lw["q_w"], lw["q_b"]); k = E.linear(a, lw["k_w"], lw["k_b"]); v = E.linear(a, lw["v_w"], lw["v_b"])
    x = x + E.linear(E.attention(q, k, v, n_heads, None, head_dim), lw["o_w"], lw["o_b"])
    a = E.layer_norm(x, lw["ln2_g"], lw["ln2_b"], eps)
    return x + E.linear(E.gelu(E.linear(a, lw["fc1_w"], lw["fc1_b"])), lw["fc2_w"], lw["fc2_b"])


def _pool_max(x, step):
    n = x.shape[0] // step
    return x[: n * step].reshape(n, step, x.shape[1]).max(axis=1)


_ORIG_ATTN = E.attention
_ORIG_CONV = E.conv1d
_ORIG_STEM = E.conv_stem

MUTANTS = [("gelu", _tanh_gelu), ("sinusoids", _cos_first), ("sinusoids", _interleaved),
           ("layer_norm", _ln_unbiased), ("layer_norm", _ln_eps_outside), ("attention", _attn_scale_hd),
           ("conv_stem", _stem_no_frame_mask), ("conv_stem", _stem_trailing_rows), ("conv1d", _conv_shifted),
           ("encoder_layer", _post_ln_layer), ("avg_pool", _pool_max)]


@pytest.mark.parametrize("name,bad", MUTANTS, ids=[f"{n}:{b.__name__}" for n, b in MUTANTS])
def test_planted_mistake_is_caught(monkeypatch, name, bad):
    d, m, f, heads, layers, t = 128, 8, 256, 2, 2, 41
    length, pool = (29, 2)   # odd length: the last valid conv2 window reaches frame `length`
    w = _rand_weights(d, m, f, layers, None, std=0.2)
    mel = RNG.uniform(-1.5, 1.5, (m, t))
    geo = Geo(layers, heads, pool)
    ref = _torch_tower(w, mel, length, d, heads, layers, pool, None)
    nv = ref.shape[0]
    np.testing.assert_allclose(E.encode_clip(geo, w, mel, length)[:nv], ref, atol=1e-10)
    monkeypatch.setattr(E, name, bad)
    if name == "layer_norm":   # small eps effects need small-variance rows to show
        w = {k: (v * 1e-3 if k.startswith("conv") else v) for k, v in w.items()}
        ref = _torch_tower(w, mel, length, d, heads, layers, pool, None)
    got = E.encode_clip(geo, w, mel, length)[:nv]
    assert not np.allclose(got, ref, atol=1e-6), f"planted mistake in {name} not detected"


def test_key_bias_is_softmax_invariant(monkeypatch):
    """A bias on k adds q.b_k to every score of a row, which softmax removes:
    the unbiased k of the tower is therefore not a detectable choice."""
    d, m, f, heads, layers, t = 128, 8, 256, 2, 1, 20
    w = _rand_weights(d, m, f, layers, None, std=0.2)
    mel = RNG.uniform(-1.5, 1.5, (m, t))
    geo = Geo(layers, heads)
    base = E.encode_clip(geo, w, mel, t)
    monkeypatch.setattr(E, "encoder_layer", _k_biased_layer)
    np.testing.assert_allclose(E.encode_clip(geo, w, mel, t), base, atol=1e-12)
