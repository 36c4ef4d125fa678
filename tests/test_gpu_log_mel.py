"""GPU parity of the streaming log-mel frontend against the float64 oracle
(fp32 path: max-abs 1e-4)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import compare_f32, dev, host

pytestmark = pytest.mark.gpu


def _vx():
    import sliding_window_attention_tcgen05_b200 as vx
    return vx


def _audio(B, N, seed, scale=0.1):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, N)) * scale).astype(np.float32)


@pytest.mark.parametrize("N", [16000, 16123, 201])
def test_log_mel_centred(N):
    x = _audio(2, N, seed=N)
    got = host(_vx().log_mel_fwd(dev(x), center=True))
    compare_f32(got, oracle.log_mel(x, center=True), f"log-mel centred N={N}")


@pytest.mark.parametrize("N", [400, 8000, 8123])
def test_log_mel_uncentred(N):
    x = _audio(3, N, seed=N + 1)
    got = host(_vx().log_mel_fwd(dev(x), center=False))
    compare_f32(got, oracle.log_mel(x, center=False), f"log-mel uncentred N={N}")


def test_log_mel_silence_is_the_floor():
    got = host(_vx().log_mel_fwd(dev(np.zeros((1, 3200), np.float32))))
    np.testing.assert_array_equal(got, np.full((1, 128, 20), -0.625, np.float32))


def test_log_mel_tone_peaks_in_the_oracles_band():
    n = np.arange(16000)
    x = (0.3 * np.cos(2 * np.pi * 1000.0 * n / 16000.0)).astype(np.float32)[None, :]
    got = host(_vx().log_mel_fwd(dev(x)))
    want = oracle.log_mel(x)
    assert np.array_equal(np.argmax(got[0, :, 10:-10], axis=0), np.argmax(want[0, :, 10:-10], axis=0))
    compare_f32(got, want, "log-mel tone")


def test_log_mel_chunked_stream_equals_whole_clip_interior():
    vx = _vx()
    x = _audio(2, 12000, seed=5)
    whole = host(vx.log_mel_fwd(dev(x), center=True))
    t0 = 9
    cont = host(vx.log_mel_fwd(dev(np.ascontiguousarray(x[:, 160 * t0 - 200:])), center=False))
    n = min(cont.shape[2], whole.shape[2] - t0 - 2)
    np.testing.assert_array_equal(cont[:, :, :n], whole[:, :, t0:t0 + n])   # same samples, same arithmetic


def test_log_mel_short_inputs():
    vx = _vx()
    with pytest.raises(vx.VxError, match="UNSUPPORTED"):
        vx.log_mel_fwd(dev(np.zeros((1, 200), np.float32)), center=True)
    assert tuple(vx.log_mel_fwd(dev(np.zeros((1, 399), np.float32)), center=False).shape) == (1, 128, 0)


def test_log_mel_full_size_sampled_frames():
    # 4 clips x 60 s at 16 kHz -> [4, 128, 6000], the encoder workload's input.
    x = _audio(4, 960000, seed=7)
    got = host(_vx().log_mel_fwd(dev(x)))
    assert got.shape == (4, 128, 6000)
    pad = np.pad(x.astype(np.float64), ((0, 0), (200, 200)), mode="reflect")
    for t in (0, 1, 2999, 5998, 5999):
        want = oracle.log_mel_frames(pad[:, 160 * t:160 * t + 400])
        compare_f32(got[:, :, t], want, f"log-mel frame {t}")
