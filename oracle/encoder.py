"""CPU oracle for the Whisper-style audio encoder tower (TEST INFRASTRUCTURE).

This module is test infrastructure.  Only the tests, the smoke check and the
CPU-baseline leg of the benchmark may import it.  The product (the CUDA
library and its Python binding) never calls it and shares no code with it.

It is a plain, slow, float64 restatement of what the encoder computes, written
clip by clip so that a reader can check each step against the model pages:

* Qwen2-Audio-7B-Instruct page, "(1) AUDIO ENCODER": the tower is the
  Whisper-large encoder (d_model 1280, 32 layers, 20 heads, FFN 5120, gelu,
  128 mel bins, 1500 source positions), one bidirectional pass, no KV cache.
* Voxtral-Mini-3B-2507 page, "(1) AUDIO ENCODER" and "Preprocessor": head_dim
  64, MHA (as many KV heads as heads); 30 s at 16 kHz with hop 160 gives 3000
  mel frames and 1500 encoder positions; "PROJECTOR": a 2-layer gelu MLP from
  the 1280-wide encoder into the 3072-wide LLM.
* MiniCPM-o-2.6 page, "(2) AUDIO": a medium-sized Whisper encoder (d_model
  1024, 24 layers, 16 heads, FFN 4096) whose audio_pool_step 2 halves the
  token rate (about 750 tokens per 30 s).

Steps the pages leave open follow the plainest reading of "the Whisper-large
encoder verbatim":

* conv stem: conv1 (n_mels -> d, kernel 3, padding 1) + GELU, conv2 (d -> d,
  kernel 3, stride 2, padding 1) + GELU; frames at or beyond a clip's length
  are zero before conv1, and the convolutions run over all T frames.
* position table: sin of the first d/2 channels then cos of the last d/2, with
  inverse timescales exp(-i ln(10000) / (d/2 - 1)).
* pre-LN blocks: x += out_proj(attn(LN1(x))); x += fc2(GELU(fc1(LN2(x)))).
  q, v, out, fc1, fc2 carry biases, k does not.
* attention: softmax(q k^T / sqrt(64)) v per head over the clip's valid keys
  (a key-padding mask; padded query rows are not part of the result).
* LayerNorm: biased variance, eps 1e-5 inside the square root.
* GELU: the exact form 0.5 x (1 + erf(x / sqrt 2)).
* final LayerNorm, then (optionally) average-pool kernel 2 stride 2 (floor),
  then (optionally) the projector fc1 -> GELU -> fc2 on every position.

Every function works in float64; library primitives used as single steps are
numpy's matmul/exp and scipy's erf.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

SQRT1_2 = 1.0 / math.sqrt(2.0)


# ----------------------------------------------------------------- counts
def frames_for_seconds(seconds: float, sampling_rate: int = 16000, hop: int = 160) -> int:
    """Mel frames for an audio span (Voxtral page, "Preprocessor": hop 160 at 16 kHz)."""
    return int(round(seconds * sampling_rate)) // hop


def conv_output_length(t: int, kernel: int = 3, stride: int = 1, pad: int = 1) -> int:
    """Length of a 1-D convolution output (standard zero-padded convolution)."""
    return (t + 2 * pad - kernel) // stride + 1


def encoder_positions(frames: int) -> int:
    """Positions after the stem: conv1 keeps the length, conv2 halves it."""
    return conv_output_length(conv_output_length(frames, 3, 1, 1), 3, 2, 1)


def valid_positions(length: int) -> int:
    """Positions whose conv2 window starts inside the clip: ceil(length / 2)."""
    return encoder_positions(length)


def pooled_positions(positions: int, pool_step: int) -> int:
    """Average pool with kernel = stride = pool_step, floor mode (MiniCPM-o page)."""
    return positions // pool_step if pool_step > 1 else positions


# ------------------------------------------------------------- elementwise
def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU: x * Phi(x) = 0.5 x (1 + erf(x / sqrt(2)))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + erf(x * SQRT1_2))


def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float = 1e-5) -> np.ndarray:
    """Row LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * gamma + beta."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def linear(x: np.ndarray, w: np.ndarray, b: np.ndarray | None) -> np.ndarray:
    """y = x W^T + b with W in PyTorch layout [out, in]."""
    y = np.asarray(x, np.float64) @ np.asarray(w, np.float64).T
    if b is not None:
        y = y + np.asarray(b, np.float64)
    return y


# -------------------------------------------------------------- conv stem
def conv1d(x: np.ndarray, w: np.ndarray, b: np.ndarray | None, stride: int) -> np.ndarray:
    """Cross-correlation, kernel 3, zero padding 1.

    x: [C_in, T]; w: [C_out, C_in, 3]; returns [C_out, T_out] with
    y[o, j] = b[o] + sum_{c,k} w[o, c, k] * x[c, stride*j + k - 1].
    """
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    c_in, t = x.shape
    t_out = conv_output_length(t, 3, stride, 1)
    xp = np.zeros((c_in, t + 2), np.float64)
    xp[:, 1:t + 1] = x
    y = np.zeros((w.shape[0], t_out), np.float64)
    for k in range(3):
        cols = xp[:, k: k + stride * (t_out - 1) + 1: stride]   # x[c, stride*j + k - 1]
        y += w[:, :, k] @ cols
    if b is not None:
        y += np.asarray(b, np.float64)[:, None]
    return y


def sinusoids(positions: int, channels: int, max_timescale: float = 10000.0) -> np.ndarray:
    """[positions, channels] table: sin in the first half, cos in the second."""
    assert channels % 2 == 0
    half = channels // 2
    log_inc = math.log(max_timescale) / (half - 1)
    inv = np.exp(-log_inc * np.arange(half, dtype=np.float64))
    ang = np.arange(positions, dtype=np.float64)[:, None] * inv[None, :]
    return np.concatenate([np.sin(ang), np.cos(ang)], axis=1)


def conv_stem(mel: np.ndarray, length: int, w: dict) -> np.ndarray:
    """mel [n_mels, T] of one clip -> [P, d] (GELU(conv2(GELU(conv1))) + PE)."""
    x = np.array(mel, dtype=np.float64)
    x[:, length:] = 0.0                                   # frames past the clip are silence
    h = gelu(conv1d(x, w["conv1_w"], w["conv1_b"], 1))
    h = gelu(conv1d(h, w["conv2_w"], w["conv2_b"], 2))    # [d, P]
    h = h.T
    return h + sinusoids(h.shape[0], h.shape[1])


# --------------------------------------------------------------- attention
def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, n_heads: int, n_valid: int | None = None,
              head_dim: int = 64) -> np.ndarray:
    """Bidirectional multi-head attention of one clip.

    q, k, v: [S, H*hd]; keys j >= n_valid are masked out (probability 0).
    Returns [S, H*hd] = concat_h softmax(q_h k_h^T / sqrt(hd)) v_h.
    """
    s = q.shape[0]
    n_valid = s if n_valid is None else n_valid
    out = np.zeros((s, n_heads * head_dim), np.float64)
    scale = 1.0 / math.sqrt(head_dim)
    for h in range(n_heads):
        c = slice(h * head_dim, (h + 1) * head_dim)
        sc = (np.asarray(q[:, c], np.float64) @ np.asarray(k[:n_valid, c], np.float64).T) * scale
        sc = sc - sc.max(axis=1, keepdims=True)
        p = np.exp(sc)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, c] = p @ np.asarray(v[:n_valid, c], np.float64)
    return out


def chunked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, n_heads: int, chunk: int,
                      head_dim: int = 64) -> np.ndarray:
    """Block-local attention of one clip (MiniCPM-o-2.6, "(2) AUDIO": audio_chunk_length
    1.0 s): position i attends only to the positions of its own chunk
    [chunk * floor(i / chunk), chunk * floor(i / chunk) + chunk), a block-diagonal mask."""
    s = q.shape[0]
    out = np.zeros((s, n_heads * head_dim), np.float64)
    for c0 in range(0, s, chunk):
        c1 = min(s, c0 + chunk)
        out[c0:c1] = attention(q[c0:c1], k[c0:c1], v[c0:c1], n_heads, None, head_dim)
    return out


# ------------------------------------------------------------------ blocks
def encoder_layer(x: np.ndarray, lw: dict, n_heads: int, eps: float, head_dim: int = 64,
                  attn_chunk: int = 0) -> np.ndarray:
    """One pre-LN block on the valid rows x [n, d] of a clip (attn_chunk > 0: block-local attention)."""
    a = layer_norm(x, lw["ln1_g"], lw["ln1_b"], eps)
    q = linear(a, lw["q_w"], lw["q_b"])
    k = linear(a, lw["k_w"], None)
    v = linear(a, lw["v_w"], lw["v_b"])
    att = (chunked_attention(q, k, v, n_heads, attn_chunk, head_dim) if attn_chunk > 0
           else attention(q, k, v, n_heads, None, head_dim))
    x = x + linear(att, lw["o_w"], lw["o_b"])
    a = layer_norm(x, lw["ln2_g"], lw["ln2_b"], eps)
    return x + linear(gelu(linear(a, lw["fc1_w"], lw["fc1_b"])), lw["fc2_w"], lw["fc2_b"])


def layer_weights(w: dict, l: int) -> dict:
    p = f"layers.{l}."
    return {k[len(p):]: v for k, v in w.items() if k.startswith(p)}


def avg_pool(x: np.ndarray, step: int) -> np.ndarray:
    """Average of consecutive groups of `step` rows; a trailing partial group is dropped."""
    n = x.shape[0] // step
    return x[: n * step].reshape(n, step, x.shape[1]).mean(axis=1)


def encode_clip(cfg, w: dict, mel: np.ndarray, length: int, layers: int | None = None) -> np.ndarray:
    """Encoder output of one clip, [P_out, d_out]; rows past the valid count are 0.

    cfg carries the geometry (n_heads, n_layers, frames, pool_step, proj_*, ln_eps,
    and attn_chunk: 0 for full attention, else the block-local chunk in positions).
    `layers` (default all) limits the number of blocks, for timing samples.
    """
    p = encoder_positions(mel.shape[1])
    n = valid_positions(length)
    chunk = getattr(cfg, "attn_chunk", 0)
    x = conv_stem(mel, length, w)[:n]                     # key-padding mask: keep valid rows
    for l in range(cfg.n_layers if layers is None else layers):
        x = encoder_layer(x, layer_weights(w, l), cfg.n_heads, cfg.ln_eps, cfg.head_dim, chunk)
    y = layer_norm(x, w["lnpost_g"], w["lnpost_b"], cfg.ln_eps)
    p_out = pooled_positions(p, cfg.pool_step)
    if cfg.pool_step > 1:
        y = avg_pool(y, cfg.pool_step)
    if cfg.proj_hidden:
        y = linear(gelu(linear(y, w["proj1_w"], w["proj1_b"])), w["proj2_w"], w["proj2_b"])
    out = np.zeros((p_out, y.shape[1]), np.float64)
    out[: y.shape[0]] = y
    return out


def valid_output_rows(cfg, length: int) -> int:
    """Rows of encode_clip's output that carry data (the rest are zero)."""
    n = valid_positions(length)
    return n // cfg.pool_step if cfg.pool_step > 1 else n
