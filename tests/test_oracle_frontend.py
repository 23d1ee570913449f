"""Pins of the log-mel front-end oracle (oracle/frontend.py) against closed
forms, brute force and textbook identities; no GPU.

The front end follows the reading of the Whisper feature extractor stated in
the oracle's header (the pages give only 16 kHz, 480,000 samples, hop 160,
3000 frames and 128 / 80 features: Voxtral-Mini-3B-2507, "Preprocessor";
MiniCPM-o-2.6, "(2) AUDIO")."""
import numpy as np
import pytest

from oracle import frontend as F

RNG = np.random.default_rng(11)


def test_geometry_matches_the_pages():
    # 30 s at 16 kHz is 480,000 samples; hop 160 gives 3000 frames (Voxtral "Preprocessor")
    assert F.N_SAMPLES == 30 * 16000
    assert F.N_SAMPLES // F.HOP == 3000 == F.N_FRAMES
    assert F.frames(np.zeros(F.N_SAMPLES)).shape == (3001, 400)
    assert F.power_spectrum(np.zeros(F.N_SAMPLES)).shape == (3000, 201)


def test_hann_window_closed_forms():
    w = F.hann_periodic(400)
    assert w[0] == 0.0 and abs(w[200] - 1.0) < 1e-15
    assert abs(w.sum() - 200.0) < 1e-9                 # periodic Hann of even length N sums to N/2
    assert np.allclose(w[1:], w[1:][::-1])              # w[k] = w[N-k]


def test_reflect_framing():
    x = RNG.standard_normal(1600)
    fr = F.frames(x)
    assert fr.shape == (1 + 1600 // 160, 400)
    j = np.arange(1, 200)
    assert np.array_equal(fr[0, 200 + j], x[j])        # frame 0 is centred on sample 0 ...
    assert np.array_equal(fr[0, 200 - j], x[j])        # ... with the signal reflected (no repeat)
    assert fr[0, 200] == x[0]
    assert np.array_equal(fr[3, :], x[3 * 160 - 200:3 * 160 + 200])   # interior frames are plain slices
    last = fr[-1]                                       # centred on sample 1600: reflected tail
    assert np.array_equal(last[200 - j], x[1600 - j])
    assert np.array_equal(last[200:], x[::-1][1:201])


@pytest.mark.parametrize("k0,amp", [(25, 0.3), (100, 1.7), (3, 0.05)])
def test_cosine_at_a_bin_closed_form(k0, amp):
    """A cosine at bin k0 through a periodic Hann window of length N: |X[k0]| = A N / 4,
    |X[k0 +- 1]| = A N / 8, every other bin 0 (the window's DFT has three nonzero terms)."""
    n = np.arange(F.N_SAMPLES)
    x = amp * np.cos(2 * np.pi * k0 * n / F.N_FFT)     # k0 * 40 Hz
    P = F.power_spectrum(x)[100:2900]                  # interior frames (no reflection)
    N = F.N_FFT
    assert np.allclose(P[:, k0], (amp * N / 4) ** 2, rtol=1e-9)
    assert np.allclose(P[:, k0 - 1], (amp * N / 8) ** 2, rtol=1e-9)
    assert np.allclose(P[:, k0 + 1], (amp * N / 8) ** 2, rtol=1e-9)
    others = np.delete(P, [k0 - 1, k0, k0 + 1], axis=1)
    assert others.max() < 1e-12 * (amp * N) ** 2


def test_power_spectrum_against_brute_force_dft():
    x = RNG.standard_normal(F.N_SAMPLES) * 0.2
    P = F.power_spectrum(x)
    w = F.hann_periodic()
    n = np.arange(400)
    for f in (0, 1, 1234, 2999):
        seg = F.frames(x)[f] * w
        for k in (0, 1, 57, 200):
            X = np.sum(seg * np.exp(-2j * np.pi * k * n / 400))
            assert abs(P[f, k] - abs(X) ** 2) <= 1e-9 * max(1.0, abs(X) ** 2)


def test_parseval_per_frame():
    x = RNG.standard_normal(F.N_SAMPLES)
    P = F.power_spectrum(x)
    seg = F.frames(x)[:-1] * F.hann_periodic()[None, :]
    c = np.full(201, 2.0)
    c[0] = c[200] = 1.0                                 # one-sided sum: DC and Nyquist once
    assert np.allclose(P @ c, 400.0 * np.sum(seg ** 2, axis=1), rtol=1e-10)


def test_slaney_mel_scale_anchor_points():
    assert F.hz_to_mel(0.0) == 0.0
    assert abs(F.hz_to_mel(200.0) - 3.0) < 1e-12        # linear: 3 mels per 200 Hz
    assert abs(F.hz_to_mel(1000.0) - 15.0) < 1e-12
    assert abs(F.hz_to_mel(6400.0) - 42.0) < 1e-12      # 27 mels per factor 6.4 above 1 kHz
    f = np.array([0.0, 30.0, 999.0, 1000.0, 1001.0, 4321.0, 8000.0])
    assert np.allclose(F.mel_to_hz(F.hz_to_mel(f)), f, rtol=1e-12, atol=1e-9)


@pytest.mark.parametrize("n_mels", [80, 128])
def test_filterbank_triangles_partition_unity(n_mels):
    fb = F.mel_filterbank(n_mels)
    assert fb.shape == (n_mels, 201) and fb.min() >= 0.0
    edges = F.mel_to_hz(np.linspace(0.0, F.hz_to_mel(8000.0), n_mels + 2))
    width = (edges[2:] - edges[:-2]) / 2.0              # undo the unit-area scaling
    tri = fb * width[:, None]
    assert tri.max() <= 1.0 + 1e-12
    freqs = np.arange(201) * 40.0
    inside = (freqs >= edges[1]) & (freqs <= edges[n_mels])
    # neighbouring triangles share edges, so the unscaled filters sum to 1 between
    # the first and last centre
    assert np.allclose(tri[:, inside].sum(axis=0), 1.0, atol=1e-12)
    # each filter is zero outside its own two neighbours' centres
    for m in (0, n_mels // 2, n_mels - 1):
        outside = (freqs <= edges[m]) | (freqs >= edges[m + 2])
        assert np.all(fb[m, outside] == 0.0)


def test_log_mel_compression_closed_forms():
    silence = F.log_mel(np.zeros(F.N_SAMPLES), 128)
    assert silence.shape == (128, 3000)
    assert np.all(silence == (-10.0 + 4.0) / 4.0)       # floor 1e-10 -> log10 = -10 -> -1.5
    x = RNG.standard_normal(F.N_SAMPLES) * 0.1
    x[:16000] *= 1e-6                                   # a near-silent first second
    y = F.log_mel(x, 80)
    assert abs(y.max() - y.min() - 2.0) < 1e-12          # the 8-decade clamp becomes a range of 2
    assert np.all(y[:, :90] == y.min())                 # the quiet frames sit at the clamp


def test_log_mel_of_a_tone_peaks_in_its_channel():
    n = np.arange(F.N_SAMPLES)
    x = 0.5 * np.cos(2 * np.pi * 1000.0 * n / F.SAMPLE_RATE)
    y = F.log_mel(x, 128)
    fb = F.mel_filterbank(128)
    assert int(np.argmax(y[:, 1500])) == int(np.argmax(fb[:, 25]))   # 1000 Hz is bin 25
