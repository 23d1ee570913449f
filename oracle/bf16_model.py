"""Rounding-point model of the bf16 tensor-core encoder (TEST INFRASTRUCTURE).

This module is test infrastructure, like the rest of ``oracle/``: only the
tests, the smoke check and the benchmark's CPU legs may import it, and the
product never calls it.

It answers one question: how far from the exact (float64) encoder output can a
correct bf16 implementation land?  It recomputes the oracle's steps
(``oracle.encoder``) in float64, but rounds to bfloat16 (round to nearest,
ties to even) at the points where a bf16 tensor-core implementation stores a
value in 16 bits:

* the conv1 output (after its GELU), which conv2 reads back;
* every GEMM operand: the LayerNorm outputs, q / k / v, the attention
  output, the FFN hidden activation, the projector input and hidden layer;
* the softmax probabilities that multiply V (the row sums stay unrounded);
* the final output.

The residual stream, every accumulation and every LayerNorm statistic stay in
float64 here; in the library they are fp32, whose rounding (2^-24) is far
below bf16's (2^-9) and is left out of the model.

With ``rounding=False`` every rounding point is the identity and the model is
the oracle's computation (to float64 rounding order): that is how its
arithmetic is pinned to the oracle, and its rounding function is pinned to
PyTorch's own float32 -> bfloat16 conversion.  Sources of the steps are the
same as the oracle's: Qwen2-Audio-7B-Instruct, "(1) AUDIO ENCODER";
Voxtral-Mini-3B-2507, "(1) AUDIO ENCODER", "Preprocessor", "PROJECTOR";
MiniCPM-o-2.6, "(2) AUDIO".
"""
from __future__ import annotations

import math

import numpy as np

from .encoder import (avg_pool, conv1d, encoder_positions, gelu, layer_norm, layer_weights, linear,
                      pooled_positions, sinusoids, valid_positions)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 (nearest) -> bfloat16 (nearest, ties to even), returned as float64."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def _identity(x):
    return np.asarray(x, np.float64)


def _attention(q, k, v, n_heads, head_dim, rb):
    """Per-head softmax(q k^T / sqrt(hd)) v with the probabilities rounded before
    they multiply V and the row sums taken over the unrounded probabilities."""
    s = q.shape[0]
    out = np.zeros((s, n_heads * head_dim), np.float64)
    scale = 1.0 / math.sqrt(head_dim)
    for h in range(n_heads):
        c = slice(h * head_dim, (h + 1) * head_dim)
        sc = (q[:, c] @ k[:, c].T) * scale
        p = np.exp(sc - sc.max(axis=1, keepdims=True))
        out[:, c] = (rb(p) @ v[:, c]) / p.sum(axis=1, keepdims=True)
    return out


def _chunked(q, k, v, n_heads, head_dim, chunk, rb):
    out = np.zeros((q.shape[0], n_heads * head_dim), np.float64)
    for c0 in range(0, q.shape[0], chunk):
        c1 = min(q.shape[0], c0 + chunk)
        out[c0:c1] = _attention(q[c0:c1], k[c0:c1], v[c0:c1], n_heads, head_dim, rb)
    return out


def encode_clip_bf16(cfg, w: dict, mel: np.ndarray, length: int, rounding: bool = True) -> np.ndarray:
    """oracle.encode_clip with bf16 rounding at the storage points listed above.

    ``w`` and ``mel`` hold the bf16-representable values the GPU receives.
    Returns [P_out, d_out]; rows past the valid count are 0."""
    rb = round_bf16 if rounding else _identity
    chunk = getattr(cfg, "attn_chunk", 0)
    n = valid_positions(length)
    x = np.array(mel, dtype=np.float64)
    x[:, length:] = 0.0
    y1 = rb(gelu(conv1d(x, w["conv1_w"], w["conv1_b"], 1)))          # stored bf16
    h = gelu(conv1d(y1, w["conv2_w"], w["conv2_b"], 2)).T             # residual stream: not rounded
    x = (h + sinusoids(h.shape[0], h.shape[1]))[:n]
    for l in range(cfg.n_layers):
        lw = layer_weights(w, l)
        a = rb(layer_norm(x, lw["ln1_g"], lw["ln1_b"], cfg.ln_eps))
        q = rb(linear(a, lw["q_w"], lw["q_b"]))
        k = rb(linear(a, lw["k_w"], None))
        v = rb(linear(a, lw["v_w"], lw["v_b"]))
        att = (_chunked(q, k, v, cfg.n_heads, cfg.head_dim, chunk, rb) if chunk > 0
               else _attention(q, k, v, cfg.n_heads, cfg.head_dim, rb))
        x = x + linear(rb(att), lw["o_w"], lw["o_b"])
        a = rb(layer_norm(x, lw["ln2_g"], lw["ln2_b"], cfg.ln_eps))
        f = rb(gelu(linear(a, lw["fc1_w"], lw["fc1_b"])))
        x = x + linear(f, lw["fc2_w"], lw["fc2_b"])
    y = layer_norm(x, w["lnpost_g"], w["lnpost_b"], cfg.ln_eps)
    if cfg.pool_step > 1:
        y = avg_pool(y, cfg.pool_step)
    if cfg.proj_hidden:
        e = rb(y)
        p1 = rb(gelu(linear(e, w["proj1_w"], w["proj1_b"])))
        y = linear(p1, w["proj2_w"], w["proj2_b"])
    p_out = pooled_positions(encoder_positions(mel.shape[1]), cfg.pool_step)
    out = np.zeros((p_out, y.shape[1]), np.float64)
    out[: y.shape[0]] = rb(y)
    return out
