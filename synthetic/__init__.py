"""Seeded synthetic inputs for the Whisper-style audio encoder tower.

This module is shared by the CPU oracle tests, the GPU parity tests and the
benchmark.  It holds no arithmetic of the encoder itself: it only draws random
numbers, shapes them into tensors and rounds them to the storage precision the
GPU receives.  Both sides of every parity check are fed the *same* arrays.

Generator (counter based, so any tensor can be drawn on its own):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): state advances by the golden-ratio increment
  0x9E3779B97F4A7C15 and each output is the published 64-bit finaliser of the
  state.  Element ``i`` of a stream with key ``k`` is ``mix(k + (i+1)*G)``.
* The key of tensor number ``t`` under seed ``s`` is
  ``mix(((s + 1) * G) xor ((t + 1) * 0xD1B54A32D192ED03))``.
* Uniform in [0, 1): the top 53 bits times 2**-53.
* Normal: Box-Muller on consecutive uniform pairs (u1, u2):
  ``r = sqrt(-2 ln(1 - u1))``; element 2p gets ``r cos(2 pi u2)`` and element
  2p+1 gets ``r sin(2 pi u2)``.

Distributions (the workloads of the encoder configurations):

* mel ~ U(-1.5, 1.5)
* every weight matrix ~ N(0, 0.02); biases and LayerNorm beta ~ N(0, 0.02);
  LayerNorm gamma = 1 + N(0, 0.02)
* per-clip lengths for the ragged sweep: uniform integer in [500, 3000] frames

Values are drawn in float64, cast to float32, and for bf16 workloads rounded
to bfloat16 (round to nearest, ties to even) and widened back to float32, so
the float32 arrays hold exactly the values the GPU stores.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess

import numpy as np

_MASK = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
_KEYMUL = 0xD1B54A32D192ED03
_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "_gen.c")
_SO = os.path.join(_HERE, "_gen.so")
_LIB = None


def _mix(z: int) -> int:
    """SplitMix64 output finaliser on a Python int (64-bit wrapping)."""
    z &= _MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_index: int) -> int:
    return _mix((((seed + 1) * GOLDEN) & _MASK) ^ (((tensor_index + 1) * _KEYMUL) & _MASK))


def build_generator(force: bool = False) -> str:
    """Compile the C drawing routines next to this file (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _lib():
    global _LIB
    if _LIB is None:
        lib = ctypes.CDLL(build_generator())
        f32p = ctypes.POINTER(ctypes.c_float)
        lib.synth_uniform.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_double, ctypes.c_double, f32p]
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_double,
                                     ctypes.c_double, f32p]
        lib.synth_round_bf16.argtypes = [f32p, ctypes.c_int64]
        for f in (lib.synth_uniform, lib.synth_normal, lib.synth_round_bf16):
            f.restype = None
        _LIB = lib
    return _LIB


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def uniform_f32(seed: int, tensor_index: int, n: int, scale: float = 1.0, shift: float = 0.0,
                start: int = 0) -> np.ndarray:
    """float32(u * scale + shift) for uniforms u of stream (seed, tensor_index), elements start.."""
    out = np.empty(n, np.float32)
    _lib().synth_uniform(stream_key(seed, tensor_index), start, n, scale, shift, _ptr(out))
    return out


def normal_f32(seed: int, tensor_index: int, n: int, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    """float32(z * std + mean) for standard normals z of stream (seed, tensor_index)."""
    out = np.empty(n, np.float32)
    _lib().synth_normal(stream_key(seed, tensor_index), n, std, mean, _ptr(out))
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return float32."""
    out = np.array(x, dtype=np.float32, copy=True, order="C")
    _lib().synth_round_bf16(_ptr(out), out.size)
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of bf16-representable float32 values (the bf16 encoding)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# --------------------------------------------------------------------------
# Encoder configurations (geometry and workload of each case)
# --------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class EncoderConfig:
    name: str
    n_mels: int
    d_model: int
    n_layers: int
    n_heads: int
    ffn_dim: int
    frames: int          # T, mel frames per clip (zero padded)
    batch: int
    dtype: str           # "bf16" or "fp32"
    seed: int
    pool_step: int = 1
    proj_hidden: int = 0
    proj_out: int = 0
    ragged: tuple | None = None   # (min_frames, max_frames) for uniform lengths
    head_dim: int = 64
    ln_eps: float = 1e-5
    weight_std: float = 0.02
    attn_chunk: int = 0           # 0: full attention; else block-local chunks of this many positions

    @property
    def positions(self) -> int:       # conv2 (k3, s2, p1) output length
        return (self.frames + 2 - 3) // 2 + 1

    def replace(self, **kw) -> "EncoderConfig":
        return dataclasses.replace(self, **kw)


# Workloads: tiny fp32 check case, MiniCPM-o medium tower with pool, Whisper-large
# tower, Whisper-large + Voxtral projector, ragged sweep, Whisper-large at 12.5 Hz,
# MiniCPM-o medium tower with 1 s block-local attention.
CONFIGS = {
    "tiny_fp32": EncoderConfig("tiny_fp32", 128, 1280, 2, 20, 5120, 200, 1, "fp32", 0),
    "medium_pool": EncoderConfig("medium_pool", 80, 1024, 24, 16, 4096, 3000, 8, "bf16", 1,
                                 pool_step=2),
    "large_b16": EncoderConfig("large_b16", 128, 1280, 32, 20, 5120, 3000, 16, "bf16", 2),
    "large_proj_b32": EncoderConfig("large_proj_b32", 128, 1280, 32, 20, 5120, 3000, 32, "bf16", 3,
                                    proj_hidden=3072, proj_out=3072),
    "large_ragged_b64": EncoderConfig("large_ragged_b64", 128, 1280, 32, 20, 5120, 3000, 64, "bf16", 4,
                                      ragged=(500, 3000)),
    # rate reduction to 12.5 Hz (Kimi-Audio-7B-Instruct: "Whisper encoder (downsampled to 12.5Hz)")
    "large_pool4_b16": EncoderConfig("large_pool4_b16", 128, 1280, 32, 20, 5120, 3000, 16, "bf16", 6,
                                     pool_step=4),
    # MiniCPM-o tower with block-local attention over 1 s chunks (50 positions):
    # MiniCPM-o-2.6, "(2) AUDIO", audio_chunk_length 1.0
    "medium_chunk50": EncoderConfig("medium_chunk50", 80, 1024, 24, 16, 4096, 3000, 8, "bf16", 7,
                                    pool_step=2, attn_chunk=50),
}
CONFIG_ORDER = ["tiny_fp32", "medium_pool", "large_b16", "large_proj_b32", "large_ragged_b64", "large_pool4_b16",
                "medium_chunk50"]

LAYER_TENSORS = ["ln1_g", "ln1_b", "q_w", "q_b", "k_w", "v_w", "v_b", "o_w", "o_b",
                 "ln2_g", "ln2_b", "fc1_w", "fc1_b", "fc2_w", "fc2_b"]


def weight_shapes(cfg: EncoderConfig) -> list[tuple[str, tuple]]:
    """(name, shape) of every parameter, in drawing order (PyTorch layouts)."""
    d, m, f = cfg.d_model, cfg.n_mels, cfg.ffn_dim
    out = [("conv1_w", (d, m, 3)), ("conv1_b", (d,)), ("conv2_w", (d, d, 3)), ("conv2_b", (d,))]
    per = {"ln1_g": (d,), "ln1_b": (d,), "q_w": (d, d), "q_b": (d,), "k_w": (d, d),
           "v_w": (d, d), "v_b": (d,), "o_w": (d, d), "o_b": (d,), "ln2_g": (d,), "ln2_b": (d,),
           "fc1_w": (f, d), "fc1_b": (f,), "fc2_w": (d, f), "fc2_b": (d,)}
    for l in range(cfg.n_layers):
        for nm in LAYER_TENSORS:
            out.append((f"layers.{l}.{nm}", per[nm]))
    out += [("lnpost_g", (d,)), ("lnpost_b", (d,))]
    if cfg.proj_hidden:
        out += [("proj1_w", (cfg.proj_hidden, d)), ("proj1_b", (cfg.proj_hidden,)),
                ("proj2_w", (cfg.proj_out, cfg.proj_hidden)), ("proj2_b", (cfg.proj_out,))]
    return out


def _store(cfg: EncoderConfig, x: np.ndarray) -> np.ndarray:
    if cfg.dtype == "bf16":
        _lib().synth_round_bf16(_ptr(x), x.size)
    return x


def draw_tensor(cfg: EncoderConfig, index: int, name: str, shape: tuple,
                std: float | None = None) -> np.ndarray:
    n = int(np.prod(shape))
    std = cfg.weight_std if std is None else std
    z = normal_f32(cfg.seed, index, n, std, 1.0 if name.endswith("_g") else 0.0)
    return _store(cfg, z).reshape(shape)


def make_weights(cfg: EncoderConfig, layers: list[int] | None = None,
                 std: float | None = None) -> dict[str, np.ndarray]:
    """All parameters (or the stem/post ones plus the chosen layers)."""
    w = {}
    for idx, (name, shape) in enumerate(weight_shapes(cfg)):
        if layers is not None and name.startswith("layers."):
            if int(name.split(".")[1]) not in layers:
                continue
        w[name] = draw_tensor(cfg, idx, name, shape, std)
    return w


def input_index(cfg: EncoderConfig) -> int:
    return len(weight_shapes(cfg))


def make_lengths(cfg: EncoderConfig) -> np.ndarray:
    """Per-clip valid frame counts (int32); full length unless ragged."""
    if cfg.ragged is None:
        return np.full(cfg.batch, cfg.frames, dtype=np.int32)
    lo, hi = cfg.ragged
    key = stream_key(cfg.seed, input_index(cfg) + 1)
    u = np.array([_mix(key + (i + 1) * GOLDEN) >> 11 for i in range(cfg.batch)], dtype=np.float64)
    u *= 2.0 ** -53
    return (np.floor(u * (hi - lo + 1)).astype(np.int64) + lo).astype(np.int32)


def make_mel(cfg: EncoderConfig, batch: int | None = None) -> np.ndarray:
    """Log-mel input [B, n_mels, T] ~ U(-1.5, 1.5) in the storage precision."""
    b = cfg.batch if batch is None else batch
    n = b * cfg.n_mels * cfg.frames
    u = uniform_f32(cfg.seed, input_index(cfg), n, 3.0, -1.5)
    return _store(cfg, u).reshape(b, cfg.n_mels, cfg.frames)


def mel_clip(cfg: EncoderConfig, b: int) -> np.ndarray:
    """Clip b of make_mel(cfg) without drawing the whole batch."""
    n = cfg.n_mels * cfg.frames
    u = uniform_f32(cfg.seed, input_index(cfg), n, 3.0, -1.5, start=b * n)
    return _store(cfg, u).reshape(cfg.n_mels, cfg.frames)


def make_audio(batch: int, seed: int = 5) -> np.ndarray:
    """[batch, 480000] float32 test audio (30 s at 16 kHz) for the log-mel front
    end: white noise (std 0.05) under a piecewise-constant envelope of 0.5 s
    segments, one sine tone per clip (100 Hz .. 7.1 kHz, amplitude 0.05 .. 0.35),
    and the last two seconds of every odd clip silent."""
    n = 480000
    t = np.arange(n, dtype=np.float64) / 16000.0
    out = np.empty((batch, n), np.float32)
    for b in range(batch):
        noise = normal_f32(seed, 3 * b, n, std=0.05).astype(np.float64)
        env = np.repeat(uniform_f32(seed, 3 * b + 1, 60).astype(np.float64), n // 60)
        u = uniform_f32(seed, 3 * b + 2, 2).astype(np.float64)
        tone = (0.05 + 0.3 * u[1]) * np.sin(2.0 * np.pi * (100.0 + 7000.0 * u[0]) * t)
        x = (noise * env + tone).astype(np.float32)
        if b % 2:
            x[-32000:] = 0.0
        out[b] = x
    return out
