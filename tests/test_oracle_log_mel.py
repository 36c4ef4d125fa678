"""Pins of the oracle's streaming log-mel frontend (16 kHz, n_fft 400, hop
160, periodic Hann, slaney filterbank 128 x 0-8000 Hz, fixed global max 1.5)."""
import math

import numpy as np
import pytest
import torch
import torchaudio.functional as TAF

import oracle


def test_slaney_scale_closed_forms():
    np.testing.assert_allclose(oracle._hz_to_mel([0.0, 500.0, 1000.0]), [0.0, 7.5, 15.0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle._hz_to_mel(6400.0), 15.0 + 27.0, rtol=1e-12)   # one factor 6.4 above 1 kHz
    f = np.array([10.0, 999.0, 1000.0, 1234.5, 7999.0])
    np.testing.assert_allclose(oracle._mel_to_hz(oracle._hz_to_mel(f)), f, rtol=1e-12)


def test_filterbank_matches_torchaudio_slaney():
    # torchaudio builds its filterbank in float32: agreement to fp32 rounding
    want = TAF.melscale_fbanks(201, 0.0, 8000.0, 128, 16000, norm="slaney", mel_scale="slaney").double().numpy().T
    got = oracle.slaney_mel_filterbank()
    assert np.max(np.abs(got - want)) <= 1e-5 * np.max(np.abs(want))
    assert np.array_equal(got > 0, want > 0) or np.max(np.abs(got[(got > 0) != (want > 0)])) < 1e-6


def test_silence_is_the_floor_everywhere():
    out = oracle.log_mel(np.zeros((1, 1600)))
    assert out.shape == (1, 128, 10)
    np.testing.assert_array_equal(out, np.full_like(out, (1.5 - 8.0 + 4.0) / 4.0))


def test_bin_centred_tone_power_and_band():
    # 1000 Hz = bin 25 of a 400-point DFT at 16 kHz: |X[25]| = A * sum(w) / 2 = 100 A
    # for a periodic Hann window (sum 200); the band with the largest output
    # is the one whose triangle is highest at 1000 Hz.
    A = 0.3
    n = np.arange(400)
    frame = A * np.cos(2 * math.pi * 1000.0 * n / 16000.0)
    spec = np.abs(np.fft.rfft(frame * oracle._hann_periodic())) ** 2
    assert abs(spec[25] - (100.0 * A) ** 2) < 1e-9
    fb = oracle.slaney_mel_filterbank()
    out = oracle.log_mel_frames(frame[None, :])[0]
    assert int(np.argmax(out)) == int(np.argmax(fb[:, 25]))


def test_parseval_per_frame():
    rng = np.random.default_rng(0)
    frame = rng.standard_normal(400)
    wx = frame * oracle._hann_periodic()
    X = np.fft.rfft(wx)
    p = np.abs(X) ** 2
    assert abs((p[0] + p[200] + 2 * p[1:200].sum()) - 400 * np.sum(wx * wx)) < 1e-8 * 400 * np.sum(wx * wx)


def test_centred_frame_sits_on_its_sample():
    # An impulse at sample 160 t is at the centre of centred frame t, where the
    # window is 1: the frame's power spectrum is flat (1 at every bin).
    x = np.zeros((1, 3200))
    x[0, 160 * 5] = 1.0
    pad = np.pad(x, ((0, 0), (200, 200)), mode="reflect")
    spec = np.abs(np.fft.rfft(pad[0, 160 * 5:160 * 5 + 400] * oracle._hann_periodic())) ** 2
    np.testing.assert_allclose(spec, np.ones(201), atol=1e-12)
    flat = oracle.log_mel_frames(pad[0, 160 * 5:160 * 5 + 400][None, :])[0]
    np.testing.assert_allclose(oracle.log_mel(x)[0, :, 5], flat, rtol=0, atol=1e-12)


@pytest.mark.parametrize("N,center,F", [(16000, True, 100), (16000, False, 98), (399, False, 0), (400, False, 1),
                                        (960000, True, 6000)])
def test_frame_counts(N, center, F):
    if N > 20000:
        assert N // 160 == F   # the 60 s clip of the encoder workload: 6000 mel frames
        return
    assert oracle.log_mel(np.zeros((1, N)), center=center).shape == (1, 128, F)


def test_streaming_continuation_equals_whole_clip_interior():
    # The fixed global maximum makes every frame independent: interior centred
    # frames t equal uncentred frames over the samples [160 t0 - 200, ...).
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 8000)) * 0.1
    whole = oracle.log_mel(x, center=True)
    t0 = 7
    cont = oracle.log_mel(x[:, 160 * t0 - 200:], center=False)
    n = cont.shape[2]
    np.testing.assert_allclose(cont[:, :, :min(n, whole.shape[2] - t0 - 2)],
                               whole[:, :, t0:t0 + min(n, whole.shape[2] - t0 - 2)], rtol=0, atol=1e-12)


def _torchaudio_fb():
    """The slaney filterbank as torchaudio builds it (float32), [128, 201] float64."""
    return TAF.melscale_fbanks(201, 0.0, 8000.0, 128, 16000, norm="slaney", mel_scale="slaney").double().numpy().T


@pytest.mark.parametrize("A", [1.0, 0.03, 1e-3])
def test_impulse_at_frame_centre_band_values_closed_form(A):
    # An impulse of amplitude A at sample 160 t sits at the centre of centred
    # frame t, where the periodic Hann window is exactly 1, so that frame's
    # power spectrum is A^2 at every bin and band m holds A^2 * sum_k fb[m, k].
    # The normalisation then fixes every value: log10, the fixed floor
    # 1.5 - 8 = -6.5, and (x + 4) / 4.  A = 1e-3 puts every band below the
    # floor, A = 0.03 and 1.0 none (a natural log or a missing clamp fails).
    x = np.zeros((1, 3200))
    x[0, 160 * 5] = A
    got = oracle.log_mel(x)[0, :, 5]
    mel = A * A * _torchaudio_fb().sum(axis=1)
    want = (np.maximum(np.log10(mel), -6.5) + 4.0) / 4.0
    np.testing.assert_allclose(got, want, rtol=0, atol=2e-6)


def test_bin_centred_tone_band_values_closed_form():
    # A 1000 Hz cosine of amplitude A is 25 whole periods of a 400-sample
    # frame.  With the periodic Hann window its DFT has |X[25]| = 100 A and
    # |X[24]| = |X[26]| = 50 A and nothing else, whatever the phase; so band m
    # of every interior frame is A^2 (2500 fb[m,24] + 1e4 fb[m,25] + 2500
    # fb[m,26]), and bands without those bins sit at the -6.5 floor.
    A = 0.25
    n = np.arange(16000)
    x = (A * np.cos(2 * math.pi * 1000.0 * n / 16000.0 + 0.7))[None, :]
    out = oracle.log_mel(x)[0]
    fb = _torchaudio_fb()
    mel = A * A * (2500.0 * fb[:, 24] + 1e4 * fb[:, 25] + 2500.0 * fb[:, 26])
    want = (np.maximum(np.log10(np.maximum(mel, 1e-30)), -6.5) + 4.0) / 4.0
    assert np.sum(want > -0.625) >= 2 and np.sum(want == -0.625) >= 100
    for t in (3, 50, 97):
        np.testing.assert_allclose(out[:, t], want, rtol=0, atol=2e-6)
