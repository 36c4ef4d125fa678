"""Float64 CPU oracle for the Voxtral Realtime causal sliding-window encoder.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the CUDA library and its Python binding) never
imports, links or runs it, and this package shares no code with it.

Every function is a plain, slow statement of what the encoder computes,
written from the transcribe.cpp porting notes "Voxtral", section
"Architecture -> Voxtral Realtime 2602 (voxtral_realtime)": a causal conv stem
(left-pad-only CausalConv1d, conv2 stride 2), then 32 causal sliding-window
(750) transformer layers with RoPE (theta 1e6, head_dim 64), RMSNorm pre-norm,
a SwiGLU/silu MLP, 32-head MHA, no bias on k_proj and FFN bias only on the down
projection; plus the streaming schedule of the same section (4 encoder frames
per step).  Numpy matmuls serve as library steps; nothing is blocked, fused or
reordered beyond the definitions below.

Readings where the page is silent (each pinned by a test in tests/):
  * window: query i sees keys j with i - W < j <= i (exactly W keys incl. itself);
  * RoPE: split-halves pairing (x_m, x_{m+D/2}), inv_freq_m = theta^(-2m/D),
    angle = position * inv_freq_m, applied to q and k after the bias add;
    positions are absolute 0-based frame indices (pos0 + t);
  * softmax scale 1/sqrt(head_dim); RMSNorm x / sqrt(mean(x^2) + eps) * g;
  * SwiGLU: silu(x W_g^T [+ b_g]) * (x W_u^T [+ b_u]) with silu(z) = z * sigmoid(z);
  * conv stem: left zero padding of k - 1 = 2 frames before each conv, exact
    (erf) GELU, output length floor((Tm - 1) / 2) + 1;
  * streaming: the ring holds frame f in slot f mod W; a step reads every old
    in-window slot before any new frame is written;
  * streaming conv stem (the "conv padding cache" of the Frontend section):
    a chunk of an even number of mel frames continues the left context of
    the previous chunk: the last 2 mel frames (conv1 taps) and the last 2
    conv1 outputs (conv2 taps) are carried; the first chunk starts from zeros;
  * projector: frames 4j .. 4j+3 are concatenated in time order into token j
    (frame-major reshape of [B, T, d] to [B, T/4, 4d]), exact (erf) GELU;
  * log-mel frontend (section "Frontend"): power spectrum |STFT|^2 of
    400-sample frames (periodic Hann, hop 160, n_fft 400) at 16 kHz, a slaney
    filterbank of 128 bands over 0-8000 Hz (slaney mel scale, area
    normalisation), log10 of max(mel, 1e-10), the fixed global maximum of the
    Realtime model: max(log, 1.5 - 8), then (x + 4) / 4; with centring
    (the first chunk / a whole clip) the signal is reflect-padded by 200
    samples on both sides and the last STFT frame is dropped; without it the
    frames are those lying wholly inside the given samples.

Parity against the real checkpoint is unpinned: the pages print no
activations and no trained weights are available.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "rms_norm", "rope_inv_freq", "rope", "swa_attention", "swa_attention_rows",
    "silu", "gelu", "encoder_layer", "ring_from_sequence", "stream_step_layer",
    "stream_step", "conv_stem", "conv_out_len", "encoder", "as64", "conv_stem_step",
    "projector", "slaney_mel_filterbank", "log_mel", "log_mel_frames",
]


def as64(a):
    """Upcast (bf16-exact float32 or float32) inputs to float64, exactly."""
    return None if a is None else np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------- elementwise

def rms_norm(x, g, eps=1e-5):
    """RMSNorm (the pre-norm of each 2602 encoder sub-block):
    y = x / sqrt(mean(x^2 over the model dimension) + eps) * g."""
    x = as64(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * as64(g)


def silu(z):
    """silu(z) = z * sigmoid(z) (the MLP activation of the 2602 encoder)."""
    return z / (1.0 + np.exp(-z))


def gelu(z):
    """Exact GELU, 0.5 z (1 + erf(z / sqrt(2))) (the conv-stem activation)."""
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


# ----------------------------------------------------------------------- RoPE

def rope_inv_freq(head_dim, theta):
    """inv_freq_m = theta^(-2m / head_dim), m = 0 .. head_dim/2 - 1."""
    m = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * m / head_dim)


def rope(x, pos, theta):
    """Rotary position embedding (theta 1e6, head_dim 64 for the encoder).

    x: [..., T, H, D]; pos: [T] absolute frame positions.  Each pair
    (x_m, x_{m+D/2}) is rotated by the angle pos * inv_freq_m.
    """
    x = as64(x)
    D = x.shape[-1]
    half = D // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * rope_inv_freq(D, theta)[None, :]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


# ------------------------------------------------------------------ attention

def swa_attention_rows(q, k, v, window, rows, scale=None):
    """Causal sliding-window attention for selected query rows.

    o_i = sum_{j : i - W < j <= i} softmax_j(<q_i, k_j> * scale) v_j, per head
    (the 2602 encoder's causal attention restricted to a window of W frames).
    q, k, v: [B, T, H, D] (RoPE already applied).  Returns [B, len(rows), H, D].
    """
    q, k, v = as64(q), as64(k), as64(v)
    B, T, H, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = np.empty((B, len(rows), H, D))
    for n, i in enumerate(rows):
        lo = max(0, i - window + 1)
        s = np.einsum("bhd,bjhd->bhj", q[:, i], k[:, lo:i + 1]) * scale
        s = s - np.max(s, axis=-1, keepdims=True)
        p = np.exp(s)
        p /= np.sum(p, axis=-1, keepdims=True)
        out[:, n] = np.einsum("bhj,bjhd->bhd", p, v[:, lo:i + 1])
    return out


def swa_attention(q, k, v, window, scale=None):
    """swa_attention_rows over every query row: [B, T, H, D] -> [B, T, H, D]."""
    T = np.shape(q)[1]
    return swa_attention_rows(q, k, v, window, range(T), scale)


# ------------------------------------------------------------- encoder layer

def _qkv(y, p, dims, pos):
    """Projections q = y Wq^T + bq, k = y Wk^T (no bias), v = y Wv^T + bv,
    split into heads, RoPE on q and k at `pos` (per row of the T axis)."""
    H, D = dims.n_heads, dims.head_dim
    lead = y.shape[:-1]
    q = y @ as64(p["wq"]).T + as64(p["bq"])
    k = y @ as64(p["wk"]).T
    v = y @ as64(p["wv"]).T + as64(p["bv"])
    q = q.reshape(*lead, H, D)
    k = k.reshape(*lead, H, D)
    v = v.reshape(*lead, H, D)
    return rope(q, pos, dims.rope_theta), rope(k, pos, dims.rope_theta), v


def _mlp(h, p, dims):
    """SwiGLU MLP branch: (silu(y Wg^T [+bg]) * (y Wu^T [+bu])) Wd^T + bd, y = RMSNorm(h)."""
    y1 = rms_norm(h, p["ffn_norm_g"], dims.eps)
    g = y1 @ as64(p["wg"]).T
    u = y1 @ as64(p["wu"]).T
    if p.get("bg") is not None:
        g = g + as64(p["bg"])
    if p.get("bu") is not None:
        u = u + as64(p["bu"])
    return (silu(g) * u) @ as64(p["wd"]).T + as64(p["bd"])


def encoder_layer(x, p, dims, pos0=0, return_kv=False):
    """One pre-norm encoder layer over whole clips.

    x: [B, T, d] -> [B, T, d]:
      h   = x + SWA(RoPE(q), RoPE(k), v) Wo^T + bo
      out = h + MLP(RMSNorm(h))
    with y0 = RMSNorm(x) feeding the q/k/v projections, positions pos0 + t.
    """
    x = as64(x)
    B, T, d = x.shape
    pos = pos0 + np.arange(T)
    y0 = rms_norm(x, p["attn_norm_g"], dims.eps)
    q, k, v = _qkv(y0, p, dims, pos)
    a = swa_attention(q, k, v, dims.window).reshape(B, T, dims.hd)
    h = x + a @ as64(p["wo"]).T + as64(p["bo"])
    out = h + _mlp(h, p, dims)
    return (out, k, v) if return_kv else out


# ------------------------------------------------------------------ streaming

def ring_from_sequence(k, v, window):
    """Ring cache after appending a whole sequence: frame f sits in slot f mod W.

    k, v: [S, T, H, D] -> ring_k, ring_v: [S, H, W, D] (slots never written are 0).
    """
    k, v = as64(k), as64(v)
    S, T, H, D = k.shape
    rk = np.zeros((S, H, window, D))
    rv = np.zeros((S, H, window, D))
    for f in range(max(0, T - window), T):
        rk[:, :, f % window] = k[:, f]
        rv[:, :, f % window] = v[:, f]
    return rk, rv


def stream_step_layer(x_new, p, dims, ring_k, ring_v, pos):
    """One layer of an incremental streaming step over a W-slot ring cache.

    x_new: [S, n, d] (frames pos[s] .. pos[s]+n-1 of each stream);
    ring_k/ring_v: [S, H, W, D] holding frames max(0, pos-W) .. pos-1 at slot f mod W.
    Query frame f_q attends frames f with f_q - W < f <= f_q; frames before pos[s]
    come from the ring, the others from this step.  All ring reads happen before
    the n new frames are written to slots (pos[s] + t) mod W.
    Returns (out [S, n, d], new ring_k, new ring_v).
    """
    x_new = as64(x_new)
    S, n, d = x_new.shape
    H, D, W = dims.n_heads, dims.head_dim, dims.window
    scale = 1.0 / math.sqrt(D)
    ring_k, ring_v = as64(ring_k), as64(ring_v)
    y0 = rms_norm(x_new, p["attn_norm_g"], dims.eps)
    a = np.empty((S, n, H, D))
    knew_all, vnew_all = [], []
    for s in range(S):
        ps = int(pos[s])
        q, knew, vnew = _qkv(y0[s], p, dims, ps + np.arange(n))     # [n, H, D]
        knew_all.append(knew)
        vnew_all.append(vnew)
        for i in range(n):
            fq = ps + i
            keys, vals = [], []
            for f in range(max(0, fq - W + 1), fq + 1):
                if f < ps:
                    keys.append(ring_k[s, :, f % W])
                    vals.append(ring_v[s, :, f % W])
                else:
                    keys.append(knew[f - ps])
                    vals.append(vnew[f - ps])
            K = np.stack(keys, axis=1)                  # [H, J, D]
            V = np.stack(vals, axis=1)
            sc = np.einsum("hd,hjd->hj", q[i], K) * scale
            sc = sc - np.max(sc, axis=-1, keepdims=True)
            pr = np.exp(sc)
            pr /= np.sum(pr, axis=-1, keepdims=True)
            a[s, i] = np.einsum("hj,hjd->hd", pr, V)
    new_k, new_v = ring_k.copy(), ring_v.copy()
    for s in range(S):
        ps = int(pos[s])
        for t in range(n):
            new_k[s, :, (ps + t) % W] = knew_all[s][t]
            new_v[s, :, (ps + t) % W] = vnew_all[s][t]
    h = x_new + a.reshape(S, n, dims.hd) @ as64(p["wo"]).T + as64(p["bo"])
    out = h + _mlp(h, p, dims)
    return out, new_k, new_v


def stream_step(x_new, layers, dims, rings, pos, final_g=None):
    """A streaming step through a stack of layers: each layer's output feeds the
    next; rings is a list of (ring_k, ring_v) per layer.  Returns
    (out, new_rings, pos + n); a final RMSNorm is applied when final_g is given."""
    x = as64(x_new)
    new_rings = []
    for p, (rk, rv) in zip(layers, rings):
        x, nk, nv = stream_step_layer(x, p, dims, rk, rv, pos)
        new_rings.append((nk, nv))
    if final_g is not None:
        x = rms_norm(x, final_g, dims.eps)
    return x, new_rings, np.asarray(pos) + x.shape[1]


# ------------------------------------------------------------------ conv stem

def conv_out_len(Tm):
    """Frames out of the stride-2 causal conv with left padding 2 and kernel 3."""
    return (Tm - 1) // 2 + 1


def conv_stem(mel, w1, b1, w2, b2):
    """Causal conv stem (left-pad-only CausalConv1d, conv2 stride 2):
      h1[t] = GELU(b1 + sum_{k,c} w1[:, c, k] x[c, t + k - 2]),      t < Tm
      h2[t] = GELU(b2 + sum_{k,c} w2[:, c, k] h1[c, 2t + k - 2]),    t < floor((Tm-1)/2)+1
    with x[., t<0] = h1[., t<0] = 0.  mel: [B, C, Tm] -> [B, T_out, d] (frame-major)."""
    x = as64(mel)
    w1, b1, w2, b2 = as64(w1), as64(b1), as64(w2), as64(b2)
    B, C, Tm = x.shape
    xp = np.concatenate([np.zeros((B, C, 2)), x], axis=2)            # [B, C, Tm+2]
    h1 = np.zeros((B, w1.shape[0], Tm)) + b1[None, :, None]
    for k in range(3):
        h1 += np.einsum("oc,bct->bot", w1[:, :, k], xp[:, :, k:k + Tm], optimize=True)
    h1 = gelu(h1)
    To = conv_out_len(Tm)
    hp = np.concatenate([np.zeros((B, h1.shape[1], 2)), h1], axis=2)  # [B, d, Tm+2]
    h2 = np.zeros((B, w2.shape[0], To)) + b2[None, :, None]
    for k in range(3):
        h2 += np.einsum("oc,bct->bot", w2[:, :, k], hp[:, :, k:k + 2 * To - 1:2], optimize=True)
    return np.transpose(gelu(h2), (0, 2, 1))


def encoder(mel, conv, layers, final_g, dims):
    """Whole-clip encoder: conv stem -> layers (positions from 0) -> final RMSNorm."""
    x = conv_stem(mel, conv["w1"], conv["b1"], conv["w2"], conv["b2"])
    for p in layers:
        x = encoder_layer(x, p, dims, pos0=0)
    return rms_norm(x, final_g, dims.eps)


def conv_stem_step(mel_new, w1, b1, w2, b2, cache_x, cache_h1):
    """One streaming chunk of the causal conv stem with a conv padding cache.

    mel_new: [B, C, n] (n even) new mel frames; cache_x: [B, C, 2] the last two
    mel frames of the previous chunk; cache_h1: [B, d, 2] its last two conv1
    outputs (GELU applied); zeros before the first chunk (the left padding).
    Returns (out [B, n/2, d], new cache_x, new cache_h1), where out continues
    conv_stem of the concatenated stream: conv1 reads mel t-2 .. t, conv2
    output u reads conv1 outputs 2u-2 .. 2u."""
    x = as64(mel_new)
    w1, b1, w2, b2 = as64(w1), as64(b1), as64(w2), as64(b2)
    B, C, n = x.shape
    assert n % 2 == 0, "chunks must keep the stride-2 phase"
    xp = np.concatenate([as64(cache_x), x], axis=2)                      # [B, C, n+2]
    h1 = np.zeros((B, w1.shape[0], n)) + b1[None, :, None]
    for k in range(3):
        h1 += np.einsum("oc,bct->bot", w1[:, :, k], xp[:, :, k:k + n], optimize=True)
    h1 = gelu(h1)
    hp = np.concatenate([as64(cache_h1), h1], axis=2)                    # [B, d, n+2]
    To = n // 2
    h2 = np.zeros((B, w2.shape[0], To)) + b2[None, :, None]
    for k in range(3):
        h2 += np.einsum("oc,bct->bot", w2[:, :, k], hp[:, :, k:k + 2 * To - 1:2], optimize=True)
    return np.transpose(gelu(h2), (0, 2, 1)), xp[:, :, -2:], hp[:, :, -2:]


def projector(x, w1, w2, factor=4):
    """Audio projector of the 2602 model (transcribe.cpp notes "Voxtral",
    section "Architecture -> Voxtral Realtime 2602"): reshape [B, T, d] to
    [B, T // factor, factor * d] (the last T % factor frames dropped, frames
    4j .. 4j+3 concatenated in time order), then Linear(4d -> H) without bias,
    GELU, Linear(H -> H) without bias.  w1: [H, 4d], w2: [H, H]."""
    x = as64(x)
    B, T, d = x.shape
    T4 = T // factor
    tok = x[:, :T4 * factor, :].reshape(B, T4, factor * d)
    return gelu(tok @ as64(w1).T) @ as64(w2).T


# ------------------------------------------------------------------ frontend

SAMPLE_RATE, N_FFT, HOP, N_MELS, F_MAX, LOG_MEL_MAX = 16000, 400, 160, 128, 8000.0, 1.5


def _hz_to_mel(f):
    """Slaney mel scale: linear (3 f / 200) below 1000 Hz, logarithmic above
    (27 mels per factor 6.4 in frequency), 15 mels at 1000 Hz."""
    f = np.asarray(f, dtype=np.float64)
    lin = f / (200.0 / 3.0)
    log = 15.0 + np.log(np.maximum(f, 1e-300) / 1000.0) / (math.log(6.4) / 27.0)
    return np.where(f >= 1000.0, log, lin)


def _mel_to_hz(m):
    m = np.asarray(m, dtype=np.float64)
    lin = m * (200.0 / 3.0)
    log = 1000.0 * np.exp((m - 15.0) * (math.log(6.4) / 27.0))
    return np.where(m >= 15.0, log, lin)


def slaney_mel_filterbank(n_mels=N_MELS, n_fft=N_FFT, sr=SAMPLE_RATE, f_min=0.0, f_max=F_MAX):
    """[n_mels, n_fft // 2 + 1] triangles between n_mels + 2 points evenly spaced
    on the slaney mel scale from f_min to f_max, each scaled by 2 / (its width
    in Hz) (area normalisation)."""
    hz = _mel_to_hz(np.linspace(_hz_to_mel(f_min), _hz_to_mel(f_max), n_mels + 2))
    freqs = np.arange(n_fft // 2 + 1) * (sr / n_fft)
    fb = np.zeros((n_mels, freqs.size))
    for m in range(n_mels):
        lo, mid, hi = hz[m], hz[m + 1], hz[m + 2]
        up = (freqs - lo) / (mid - lo)
        down = (hi - freqs) / (hi - mid)
        fb[m] = np.maximum(0.0, np.minimum(up, down)) * (2.0 / (hi - lo))
    return fb


def _hann_periodic(n=N_FFT):
    return 0.5 - 0.5 * np.cos(2.0 * math.pi * np.arange(n) / n)


def log_mel_frames(frames):
    """Normalised log-mel of already cut frames [..., 400] (float64)."""
    spec = np.abs(np.fft.rfft(as64(frames) * _hann_periodic(), n=N_FFT, axis=-1)) ** 2    # [..., 201]
    mel = spec @ slaney_mel_filterbank().T                                               # [..., 128]
    log = np.log10(np.maximum(mel, 1e-10))
    log = np.maximum(log, LOG_MEL_MAX - 8.0)
    return (log + 4.0) / 4.0


def log_mel(audio, center=True):
    """Streaming log-mel frontend of the Realtime model: audio [B, N] at 16 kHz
    -> [B, 128, F].  center: reflect-pad 200 samples on both sides, frames at
    hop 160, last frame dropped (F = N // 160); else frames wholly inside the
    samples (F = 1 + (N - 400) // 160 for N >= 400)."""
    x = as64(audio)
    if center:
        x = np.pad(x, ((0, 0), (N_FFT // 2, N_FFT // 2)), mode="reflect")
    n_frames = 1 + (x.shape[1] - N_FFT) // HOP if x.shape[1] >= N_FFT else 0
    if center:
        n_frames -= 1
    idx = np.arange(n_frames)[:, None] * HOP + np.arange(N_FFT)[None, :]
    return np.transpose(log_mel_frames(x[:, idx]), (0, 2, 1))

