"""Log-mel front end of the audio encoder, in float64 (TEST INFRASTRUCTURE ONLY).

The pages give the front end's geometry and nothing else: a
WhisperFeatureExtractor with 30 s chunks, 480,000 samples at 16 kHz, hop 160,
3000 frames and 128 features (Voxtral-Mini-3B-2507, "Preprocessor"; 80 for the
MiniCPM-o-2.6 tower, "(2) AUDIO"). Everything else is a reading of "the
Whisper feature extractor", each listed in the design notes:

- F1 window: periodic Hann of length n_fft = 400 (25 ms at 16 kHz)
- F2 framing: frames centred on samples 0, 160, 320, ... with the signal
  reflected at both ends (200 samples each side, edge sample not repeated);
  3001 frames for 480,000 samples, the last one dropped -> 3000
- F3 spectrum: power |X_k|^2 of the 201 one-sided DFT bins
- F4 mel filterbank: the Slaney mel scale (linear 0..1 kHz at 200/3 Hz per mel,
  logarithmic above with 27 mels per factor 6.4), n_mels + 2 equally spaced
  mel points from 0 Hz to 8 kHz, triangular filters on the bin frequencies
  k * 40 Hz, each scaled by 2 / (upper edge - lower edge) (unit area)
- F5 compression: log10(max(mel, 1e-10)); values below (clip maximum - 8) are
  raised to it; then (x + 4) / 4

Nothing here is shared with the CUDA path; `tests/` and `bench.py`'s CPU legs
are the only callers.
"""
from __future__ import annotations

import numpy as np

SAMPLE_RATE = 16000
N_FFT = 400
HOP = 160
N_SAMPLES = 480000          # 30 s at 16 kHz
N_FRAMES = N_SAMPLES // HOP  # 3000
N_BINS = N_FFT // 2 + 1      # 201


def hann_periodic(n: int = N_FFT) -> np.ndarray:
    """F1: w[k] = 1/2 - 1/2 cos(2 pi k / n), k = 0 .. n-1 (periodic form)."""
    k = np.arange(n, dtype=np.float64)
    return 0.5 - 0.5 * np.cos(2.0 * np.pi * k / n)


def frames(audio: np.ndarray, n_fft: int = N_FFT, hop: int = HOP) -> np.ndarray:
    """F2: [n_frames, n_fft] windows of the reflect-padded signal, frame f centred
    on sample f * hop; all 1 + len // hop frames (the caller drops the last)."""
    x = np.asarray(audio, dtype=np.float64)
    half = n_fft // 2
    padded = np.pad(x, (half, half), mode="reflect")
    n = 1 + len(x) // hop
    idx = np.arange(n)[:, None] * hop + np.arange(n_fft)[None, :]
    return padded[idx]


def power_spectrum(audio: np.ndarray) -> np.ndarray:
    """F2 + F3: [N_FRAMES, N_BINS] power of the windowed frames, last frame dropped."""
    fr = frames(audio) * hann_periodic()[None, :]
    spec = np.fft.rfft(fr, axis=-1)
    return (spec.real ** 2 + spec.imag ** 2)[:-1]


def hz_to_mel(f):
    """F4: Slaney mel scale. Linear below 1 kHz (3 mels per 200 Hz), then
    logarithmic: 15 mels at 1 kHz plus 27 mels per factor 6.4 in frequency."""
    f = np.asarray(f, dtype=np.float64)
    lin = f * 3.0 / 200.0
    log = 15.0 + np.log(np.maximum(f, 1e-300) / 1000.0) * (27.0 / np.log(6.4))
    return np.where(f >= 1000.0, log, lin)


def mel_to_hz(m):
    """Inverse of hz_to_mel."""
    m = np.asarray(m, dtype=np.float64)
    lin = m * 200.0 / 3.0
    log = 1000.0 * np.exp((m - 15.0) * (np.log(6.4) / 27.0))
    return np.where(m >= 15.0, log, lin)


def mel_filterbank(n_mels: int, sr: int = SAMPLE_RATE, n_fft: int = N_FFT) -> np.ndarray:
    """F4: [n_mels, N_BINS] triangular filters with unit-area (Slaney) scaling."""
    edges = mel_to_hz(np.linspace(hz_to_mel(0.0), hz_to_mel(sr / 2.0), n_mels + 2))
    freqs = np.arange(n_fft // 2 + 1, dtype=np.float64) * sr / n_fft
    fb = np.zeros((n_mels, len(freqs)))
    for m in range(n_mels):
        lo, mid, hi = edges[m], edges[m + 1], edges[m + 2]
        rise = (freqs - lo) / (mid - lo)
        fall = (hi - freqs) / (hi - mid)
        fb[m] = np.maximum(0.0, np.minimum(rise, fall)) * (2.0 / (hi - lo))
    return fb


def log_mel(audio: np.ndarray, n_mels: int) -> np.ndarray:
    """F1-F5 for one clip of N_SAMPLES samples: [n_mels, N_FRAMES] float64."""
    assert len(audio) == N_SAMPLES
    mel = power_spectrum(audio) @ mel_filterbank(n_mels).T          # [N_FRAMES, n_mels]
    lg = np.log10(np.maximum(mel, 1e-10)).T
    lg = np.maximum(lg, lg.max() - 8.0)
    return (lg + 4.0) / 4.0
