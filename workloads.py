"""Seeded synthetic PCM workloads for the batched log-mel spectrogram.

This module only *makes input audio*.  It holds none of the log-mel
arithmetic (no framing, window, transform, filterbank or log): both the
float64 oracle and the CUDA path are fed from here, and neither shares
anything else.

Signals follow the shapes the pages describe (16 kHz mono fp32 PCM in
[-1, 1]; "从零理解 ASR ... Qwen3-ASR", section 2.1) and the five workloads of
the benchmark table:

  1. single 1 s three-tone clip                   -> 98 frames
  2. dense batch 64 x 30 s speech-like clips       -> 64 x 2998 frames
  3. ragged batch of 256 clips, lengths U[1, 30] s -> packed, int64 offsets
  4. long-form 87 min recording, 174 x 30 s chunks, 20 % silent segments
  5. streaming: 1024 streams x 600 pushes of 80 ms (1280 samples)

The speech-like generator is our own recipe (the pages name no dataset):
harmonic series on f0 ~ U(80, 300) Hz with 1/k amplitudes below 8 kHz and
uniform random phases, a 4 Hz syllabic envelope 0.5 (1 + sin), pink noise
(white Gaussian shaped by 1/sqrt(f) in the frequency domain) at -30 dB
relative to the modulated harmonics, and a peak normalisation to 0.9.
The harmonic series is evaluated from a one-period wavetable of 16384
points with linear interpolation, which keeps 786 M samples affordable.
"""
from __future__ import annotations

import numpy as np

SR = 16000
CLIP_30S = 480000

__all__ = [
    "SR", "CLIP_30S", "three_tone", "speech_like", "dense_batch", "ragged_batch",
    "long_form", "stream_signals", "page1_test_tones", "offsets_from_lengths",
]

_TABLE_LEN = 16384


def three_tone(n_samples: int = 16000, seed: int = 0) -> np.ndarray:
    """0.3 sin 440 Hz + 0.2 sin 1200 Hz + 0.1 sin 3500 Hz + U(-0.01, 0.01), clipped."""
    rng = np.random.default_rng(seed)
    t = np.arange(n_samples, dtype=np.float64) / SR
    x = (0.3 * np.sin(2 * np.pi * 440.0 * t)
         + 0.2 * np.sin(2 * np.pi * 1200.0 * t)
         + 0.1 * np.sin(2 * np.pi * 3500.0 * t)
         + rng.uniform(-0.01, 0.01, n_samples))
    return np.clip(x, -1.0, 1.0).astype(np.float32)


def page1_test_tones(duration_s: float = 3.0, noise: bool = False, seed: int = 0) -> np.ndarray:
    """The page-1 demo tones (0.4 sin 200 Hz + 0.3 sin 400 Hz [+ 0.02 randn]).

    The page spaces time with ``linspace``; we use t = n / sr so the tones sit
    exactly on the 40 Hz bin grid (200 Hz = bin 5, 400 Hz = bin 10).
    """
    n = int(round(duration_s * SR))
    t = np.arange(n, dtype=np.float64) / SR
    x = 0.4 * np.sin(2 * np.pi * 200.0 * t) + 0.3 * np.sin(2 * np.pi * 400.0 * t)
    if noise:
        x = x + 0.02 * np.random.default_rng(seed).standard_normal(n)
    return x.astype(np.float32)


def _pink(n: int, rng: np.random.Generator) -> np.ndarray:
    white = rng.standard_normal(n)
    spec = np.fft.rfft(white)
    f = np.arange(spec.shape[0], dtype=np.float64)
    spec[0] = 0.0
    spec[1:] /= np.sqrt(f[1:])
    return np.fft.irfft(spec, n)


def speech_like(n_samples: int, seed: int) -> np.ndarray:
    """One seeded speech-like clip, float32, peak 0.9 (0 samples -> empty)."""
    if n_samples <= 0:
        return np.zeros(0, np.float32)
    rng = np.random.default_rng(seed)
    f0 = rng.uniform(80.0, 300.0)
    n_harm = int(np.ceil(8000.0 / f0)) - 1          # k * f0 < 8 kHz
    phases = rng.uniform(0.0, 2 * np.pi, n_harm)
    env_phase = rng.uniform(0.0, 2 * np.pi)

    theta = np.arange(_TABLE_LEN, dtype=np.float64) / _TABLE_LEN
    k = np.arange(1, n_harm + 1, dtype=np.float64)
    table = (np.sin(2 * np.pi * k[:, None] * theta[None, :] + phases[:, None]) / k[:, None]).sum(0)
    table = np.append(table, table[0])

    n = np.arange(n_samples, dtype=np.float64)
    pos = np.mod(n * (f0 / SR), 1.0) * _TABLE_LEN
    i0 = pos.astype(np.int64)
    frac = pos - i0
    harm = table[i0] * (1.0 - frac) + table[i0 + 1] * frac

    period = SR // 4                                   # the 4 Hz envelope repeats every 4000 samples
    env_one = 0.5 * (1.0 + np.sin(2 * np.pi * 4.0 * np.arange(period) / SR + env_phase))
    env = np.resize(env_one, n_samples)
    voiced = harm * env

    pink = _pink(n_samples, rng)
    rms_v = np.sqrt(np.mean(voiced ** 2))
    rms_p = np.sqrt(np.mean(pink ** 2))
    if rms_p > 0:
        pink *= rms_v * 10.0 ** (-30.0 / 20.0) / rms_p
    x = voiced + pink
    peak = np.max(np.abs(x))
    if peak > 0:
        x *= 0.9 / peak
    return x.astype(np.float32)


def offsets_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    off = np.zeros(lengths.shape[0] + 1, np.int64)
    np.cumsum(lengths, out=off[1:])
    return off


def dense_batch(n_clips: int = 64, clip_len: int = CLIP_30S, seed0: int = 1000):
    """Config 2: n_clips speech-like clips of clip_len samples, packed; CSR offsets."""
    pcm = np.empty(n_clips * clip_len, np.float32)
    for i in range(n_clips):
        pcm[i * clip_len:(i + 1) * clip_len] = speech_like(clip_len, seed0 + i)
    return pcm, offsets_from_lengths([clip_len] * n_clips)


def ragged_batch(n_utt: int = 256, min_len: int = SR, max_len: int = CLIP_30S,
                 seed: int = 3, seed0: int = 1000, lengths=None):
    """Config 3: lengths ~ integer U[min_len, max_len] (seeded), packed contiguously."""
    if lengths is None:
        lengths = np.random.default_rng(seed).integers(min_len, max_len + 1, n_utt)
    lengths = np.asarray(lengths, np.int64)
    off = offsets_from_lengths(lengths)
    pcm = np.empty(int(off[-1]), np.float32)
    for i, L in enumerate(lengths):
        pcm[off[i]:off[i + 1]] = speech_like(int(L), seed0 + i)
    return pcm, off


def long_form(total: int = 83_520_000, seed: int = 4, silence_p: float = 0.2, seed0: int = 4000):
    """Config 4: one recording cut into U(1, 5) s segments; each segment is exact
    zeros with probability ``silence_p`` (Bernoulli per segment), else speech-like.
    Returns (pcm, offsets of 30 s chunks) with the chunking as a ragged batch."""
    rng = np.random.default_rng(seed)
    pcm = np.zeros(total, np.float32)
    pos, i = 0, 0
    while pos < total:
        seg = int(round(rng.uniform(1.0, 5.0) * SR))
        seg = min(seg, total - pos)
        silent = rng.random() < silence_p
        if not silent:
            pcm[pos:pos + seg] = speech_like(seg, seed0 + i)
        pos += seg
        i += 1
    n_chunks = total // CLIP_30S
    lengths = [CLIP_30S] * n_chunks
    if total - n_chunks * CLIP_30S:
        lengths.append(total - n_chunks * CLIP_30S)
    return pcm, offsets_from_lengths(lengths)


def _speech_rows(args):
    n_samples, seeds = args
    return np.stack([speech_like(n_samples, s) for s in seeds])


def stream_signals(n_streams: int = 1024, n_samples: int = 768_000, seed0: int = 5000,
                   first: int = 0, workers: int = 0) -> np.ndarray:
    """Config 5: [n_streams, n_samples] float32, stream s seeded with seed0 + first + s.
    ``workers`` > 1 generates in a spawn-started process pool (same values)."""
    out = np.empty((n_streams, n_samples), np.float32)
    seeds = [seed0 + first + s for s in range(n_streams)]
    if workers and workers > 1 and n_streams > 1:
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        step = max(1, n_streams // (4 * workers))
        jobs = [(n_samples, seeds[i:i + step]) for i in range(0, n_streams, step)]
        with ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as ex:
            for i, rows in zip(range(0, n_streams, step), ex.map(_speech_rows, jobs)):
                out[i:i + rows.shape[0]] = rows
        return out
    for s in range(n_streams):
        out[s] = speech_like(n_samples, seeds[s])
    return out
