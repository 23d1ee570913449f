"""Planted mistakes in the front-end oracle (on the CPU) must be caught by the
pins of tests/test_oracle_frontend.py.

Each case swaps one step of oracle/frontend.py for a plausible wrong variant
and runs every pin; at least one must fail."""
import numpy as np
import pytest

from oracle import frontend as F
import tests.test_oracle_frontend as pins


def _run_all_pins() -> int:
    failures = 0
    cases = [
        (pins.test_geometry_matches_the_pages, ()),
        (pins.test_hann_window_closed_forms, ()),
        (pins.test_reflect_framing, ()),
        (pins.test_power_spectrum_against_brute_force_dft, ()),
        (pins.test_parseval_per_frame, ()),
        (pins.test_slaney_mel_scale_anchor_points, ()),
        (pins.test_log_mel_compression_closed_forms, ()),
        (pins.test_log_mel_of_a_tone_peaks_in_its_channel, ()),
    ]
    cases += [(pins.test_cosine_at_a_bin_closed_form, a) for a in ((25, 0.3), (100, 1.7), (3, 0.05))]
    cases += [(pins.test_filterbank_triangles_partition_unity, (m,)) for m in (80, 128)]
    for fn, args in cases:
        try:
            fn(*args)
        except (AssertionError, ValueError, IndexError):
            failures += 1
    return failures


def _symmetric_hann(n=F.N_FFT):
    k = np.arange(n, dtype=np.float64)
    return 0.5 - 0.5 * np.cos(2.0 * np.pi * k / (n - 1))


def _zero_padded_frames(audio, n_fft=F.N_FFT, hop=F.HOP):
    x = np.pad(np.asarray(audio, np.float64), (n_fft // 2, n_fft // 2))
    n = 1 + len(audio) // hop
    return x[np.arange(n)[:, None] * hop + np.arange(n_fft)[None, :]]


def _hop_161_frames(audio, n_fft=F.N_FFT, hop=F.HOP):
    x = np.pad(np.asarray(audio, np.float64), (n_fft // 2, n_fft // 2), mode="reflect")
    n = 1 + len(audio) // hop
    idx = np.minimum(np.arange(n)[:, None] * 161 + np.arange(n_fft)[None, :], len(x) - 1)
    return x[idx]


def _magnitude_not_power(audio):
    spec = np.fft.rfft(F.frames(audio) * F.hann_periodic()[None, :], axis=-1)
    return np.abs(spec)[:-1]


def _htk_mel(f):
    return 2595.0 * np.log10(1.0 + np.asarray(f, np.float64) / 700.0)


def _unnormalised_filterbank(n_mels, sr=F.SAMPLE_RATE, n_fft=F.N_FFT):
    fb = ORIGINAL["mel_filterbank"](n_mels, sr, n_fft)
    edges = F.mel_to_hz(np.linspace(0.0, F.hz_to_mel(sr / 2.0), n_mels + 2))
    return fb * ((edges[2:] - edges[:-2]) / 2.0)[:, None]


def _clamp_10(audio, n_mels):
    mel = F.power_spectrum(audio) @ F.mel_filterbank(n_mels).T
    lg = np.log10(np.maximum(mel, 1e-10)).T
    return (np.maximum(lg, lg.max() - 10.0) + 4.0) / 4.0


def _natural_log(audio, n_mels):
    mel = F.power_spectrum(audio) @ F.mel_filterbank(n_mels).T
    lg = np.log(np.maximum(mel, 1e-10)).T
    return (np.maximum(lg, lg.max() - 8.0) + 4.0) / 4.0


ORIGINAL = {"mel_filterbank": F.mel_filterbank}

MUTANTS = {
    "symmetric Hann window": ("hann_periodic", _symmetric_hann),
    "zero padding instead of reflection": ("frames", _zero_padded_frames),
    "hop 161": ("frames", _hop_161_frames),
    "magnitude instead of power": ("power_spectrum", _magnitude_not_power),
    "HTK mel scale": ("hz_to_mel", _htk_mel),
    "filters without unit-area scaling": ("mel_filterbank", _unnormalised_filterbank),
    "10-decade clamp": ("log_mel", _clamp_10),
    "natural log": ("log_mel", _natural_log),
}


def test_pins_pass_on_the_oracle():
    assert _run_all_pins() == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(monkeypatch, name):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(F, attr, fn)
    assert _run_all_pins() > 0, name
