"""Helpers shared by the GPU parity tests: upload synthetic weights, run the
library through its C ABI, and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np

import oracle as O
import synthetic as S

# bf16 tensor-core mode and fp32 check mode tolerances on the final output
BF16_REL_FRO = 1e-2
BF16_MAX_ABS = 5e-2
FP32_MAX_ABS = 1e-4


def torch_dtype(cfg):
    import torch
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def to_device(cfg, arrays: dict) -> dict:
    """float32 numpy arrays (already in the storage precision) -> device tensors."""
    import torch
    dt = torch_dtype(cfg)
    return {k: torch.from_numpy(np.ascontiguousarray(v)).to(device="cuda", dtype=dt) for k, v in arrays.items()}


def make_encoder(cfg, dev_w, max_batch=None, guard=True):
    """An encoder handle for a test; by default with guard regions around every
    workspace buffer (ENC_FLAG_GUARD), which run_gpu checks after each forward."""
    from audio_encoder_tower_b200 import Encoder
    return Encoder(n_mels=cfg.n_mels, d_model=cfg.d_model, n_layers=cfg.n_layers, n_heads=cfg.n_heads,
                   ffn_dim=cfg.ffn_dim, max_frames=cfg.frames, max_batch=max_batch or cfg.batch, dtype=cfg.dtype,
                   pool_step=cfg.pool_step, proj_hidden=cfg.proj_hidden, proj_out=cfg.proj_out,
                   ln_eps=cfg.ln_eps, attn_chunk=cfg.attn_chunk, guard=guard, weights=dev_w)


def run_gpu(enc, cfg, mel_np, lengths):
    import torch
    mel = torch.from_numpy(np.ascontiguousarray(mel_np)).to(device="cuda", dtype=torch_dtype(cfg))
    out = enc.forward(mel, lengths)
    enc.status()
    if enc.cfg.flags:
        enc.check_guards()          # no kernel wrote outside its workspace buffer
    return out.float().cpu().numpy().astype(np.float64)


def compare(cfg, got: np.ndarray, ref: np.ndarray, n_valid: int) -> dict:
    """Parity metrics over one clip's valid rows; rows past n_valid must be exact zeros."""
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(got[n_valid:] == 0.0), "rows past the valid count are not exact zeros"
    g, r = got[:n_valid], ref[:n_valid]
    assert np.all(np.isfinite(g))
    diff = g - r
    return {"rel_fro": float(np.linalg.norm(diff) / max(np.linalg.norm(r), 1e-30)),
            "max_abs": float(np.abs(diff).max()) if diff.size else 0.0}


def assert_parity(cfg, m: dict):
    if cfg.dtype == "fp32":
        assert m["max_abs"] <= FP32_MAX_ABS, m
    else:
        assert m["rel_fro"] <= BF16_REL_FRO and m["max_abs"] <= BF16_MAX_ABS, m


def oracle_clip(cfg, w, mel_clip, length):
    return O.encode_clip(cfg, w, mel_clip, int(length))
