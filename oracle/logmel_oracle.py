"""Float64 CPU oracle for the batched log-mel spectrogram (test infrastructure).

THIS IS TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it.  The CUDA library shares
no code, table or constant generator with it.

It is the plain definition of the pipeline that "从零理解 ASR：音频基础、
Qwen3-ASR 架构，以及离线 vs 流式推理原理" lays out in section 2.3
("Log-Mel Spectrogram 提取流水线"), steps 1-5, written in float64:

  step 1  framing: frames of n_fft = 400 samples every hop = 160 samples,
          no padding; frame count floor((N - 400) / 160) + 1 (0 if N < 400)
  step 2  Hamming window (the page multiplies by ``np.hamming(400)``, i.e.
          the symmetric form 0.54 - 0.46 cos(2 pi n / (N - 1)))
  step 3  real DFT to n_fft / 2 + 1 = 201 bins, power |X|^2
  step 4  128 triangular filters spaced uniformly on mel = 2595 log10(1 + f / 700)
  step 5  ln(max(mel_energy, 1e-10))

The DFT is written out as a direct O(n^2) sum (a cos / sin matrix product,
with the index product k*n reduced mod n_fft before scaling to an angle);
the filterbank is built explicitly as a dense [n_mels, n_fft/2+1] matrix.
Frames are processed in batches of independent frames purely to bound
memory; no frame's arithmetic is split or reordered.

Readings taken where the pages are silent or disagree:
  * frame count: the exact no-padding count (2998 for 30 s), not the page's
    rounded "3000";
  * triangles are linear in Hz between mel-spaced edges (130 edges for 128
    filters over fmin..fmax), unnormalised;
  * fmin = 0 Hz, fmax = sr / 2 = 8000 Hz;
  * natural log, floor 1e-10 applied to the mel energy.

Streaming (page 1 section 6 and the 80 ms audio clock of the
"Audio8-ASR-Infinite" page) emits, after each push, every frame that the
concatenated audio so far completes; the samples not yet consumed by a
frame are carried.  ``stream_emit_counts`` states that definition.
"""
from __future__ import annotations

from dataclasses import dataclass
from functools import lru_cache

import numpy as np

__all__ = [
    "Params", "DEFAULT", "LOG_FLOOR", "ENERGY_FLOOR", "hz_to_mel", "mel_to_hz", "hamming_symmetric",
    "num_frames", "frame_offsets", "frame_signal", "dft_matrices", "power_spectrum",
    "mel_edges", "mel_filterbank", "log_mel", "log_mel_batch", "log_mel_frames",
    "stream_emit_counts",
]

ENERGY_FLOOR = 1e-10
LOG_FLOOR = float(np.log(ENERGY_FLOOR))          # -23.025850929940457


@dataclass(frozen=True)
class Params:
    """Preprocessor parameters (section 2.3: n_mels 128, n_fft 400, hop 160, 16 kHz)."""
    sr: int = 16000
    n_fft: int = 400
    hop: int = 160
    n_mels: int = 128
    fmin: float = 0.0
    fmax: float = 8000.0

    @property
    def n_bins(self) -> int:
        return self.n_fft // 2 + 1


DEFAULT = Params()


# --- step 4: mel scale ------------------------------------------------------
def hz_to_mel(f):
    """mel = 2595 * log10(1 + f / 700)  (section 2.3, step 4)."""
    return 2595.0 * np.log10(1.0 + np.asarray(f, np.float64) / 700.0)


def mel_to_hz(m):
    """Inverse of ``hz_to_mel``: f = 700 * (10^(m / 2595) - 1)."""
    return 700.0 * (10.0 ** (np.asarray(m, np.float64) / 2595.0) - 1.0)


# --- step 2: window ---------------------------------------------------------
def hamming_symmetric(n: int) -> np.ndarray:
    """w[i] = 0.54 - 0.46 cos(2 pi i / (n - 1)), i = 0..n-1 (step 2)."""
    i = np.arange(n, dtype=np.float64)
    return 0.54 - 0.46 * np.cos(2.0 * np.pi * i / (n - 1))


# --- step 1: framing --------------------------------------------------------
def num_frames(n_samples: int, n_fft: int = 400, hop: int = 160) -> int:
    """floor((N - n_fft) / hop) + 1 frames, none if N < n_fft (step 1, no padding)."""
    n_samples = int(n_samples)
    if n_samples < n_fft:
        return 0
    return (n_samples - n_fft) // hop + 1


def frame_offsets(offsets, n_fft: int = 400, hop: int = 160) -> np.ndarray:
    """CSR sample offsets [n+1] -> CSR frame offsets [n+1] (exclusive prefix sum)."""
    offsets = np.asarray(offsets, np.int64)
    counts = [num_frames(offsets[i + 1] - offsets[i], n_fft, hop) for i in range(len(offsets) - 1)]
    out = np.zeros(len(offsets), np.int64)
    out[1:] = np.cumsum(counts, dtype=np.int64)
    return out


def frame_signal(x: np.ndarray, n_fft: int = 400, hop: int = 160, first: int = 0,
                 count: int | None = None) -> np.ndarray:
    """Frames first..first+count-1 of x as a [count, n_fft] float64 array."""
    total = num_frames(len(x), n_fft, hop)
    if count is None:
        count = total - first
    idx = (first + np.arange(count))[:, None] * hop + np.arange(n_fft)[None, :]
    return np.asarray(x, np.float64)[idx]


# --- step 3: DFT and power --------------------------------------------------
@lru_cache(maxsize=8)
def dft_matrices(n_fft: int = 400):
    """cos and -sin of 2 pi ((n k) mod n_fft) / n_fft, shape [n_fft, n_fft/2+1]."""
    n = np.arange(n_fft, dtype=np.int64)[:, None]
    k = np.arange(n_fft // 2 + 1, dtype=np.int64)[None, :]
    angle = 2.0 * np.pi * ((n * k) % n_fft).astype(np.float64) / n_fft
    return np.cos(angle), -np.sin(angle)


def power_spectrum(frames_windowed: np.ndarray) -> np.ndarray:
    """|X[k]|^2 with X[k] = sum_n x[n] e^{-2 pi i k n / N}, k = 0..N/2 (step 3)."""
    n_fft = frames_windowed.shape[-1]
    c, s = dft_matrices(n_fft)
    re = frames_windowed @ c
    im = frames_windowed @ s
    return re * re + im * im


# --- step 4: filterbank -----------------------------------------------------
def mel_edges(p: Params = DEFAULT) -> np.ndarray:
    """n_mels + 2 edge frequencies (Hz), uniform on the mel scale over fmin..fmax;
    the end edges are fmin and fmax themselves (not their mel round trip)."""
    m = np.linspace(hz_to_mel(p.fmin), hz_to_mel(p.fmax), p.n_mels + 2)
    e = mel_to_hz(m)
    e[0], e[-1] = p.fmin, p.fmax
    return e


def mel_filterbank(p: Params = DEFAULT) -> np.ndarray:
    """Dense H[m, k]: triangle m rises linearly in Hz from edge m to edge m+1
    and falls to edge m+2; bin k sits at k * sr / n_fft Hz; no normalisation."""
    e = mel_edges(p)
    f = np.arange(p.n_bins, dtype=np.float64) * p.sr / p.n_fft
    H = np.zeros((p.n_mels, p.n_bins), np.float64)
    for m in range(p.n_mels):
        lo, mid, hi = e[m], e[m + 1], e[m + 2]
        rise = (f - lo) / (mid - lo)
        fall = (hi - f) / (hi - mid)
        H[m] = np.maximum(0.0, np.minimum(rise, fall))
    return H


# --- the whole pipeline -----------------------------------------------------
_BATCH = 8192


def _mel_energy_of_frames(frames: np.ndarray, p: Params) -> np.ndarray:
    w = hamming_symmetric(p.n_fft)
    H = mel_filterbank(p)
    out = np.empty((frames.shape[0], p.n_mels), np.float64)
    for b in range(0, frames.shape[0], _BATCH):
        fw = frames[b:b + _BATCH] * w[None, :]
        out[b:b + _BATCH] = power_spectrum(fw) @ H.T
    return out


def log_mel(x: np.ndarray, p: Params = DEFAULT, return_energy: bool = False):
    """[T, n_mels] log-mel of one utterance (steps 1-5); optionally also the
    pre-log mel energy M so callers can apply the tolerance bands."""
    T = num_frames(len(x), p.n_fft, p.hop)
    frames = frame_signal(x, p.n_fft, p.hop, 0, T)
    M = _mel_energy_of_frames(frames, p)
    L = np.log(np.maximum(M, ENERGY_FLOOR))
    return (L, M) if return_energy else L


def log_mel_batch(pcm: np.ndarray, offsets, p: Params = DEFAULT, return_energy: bool = False):
    """Ragged batch: utterance u is pcm[offsets[u]:offsets[u+1]]; outputs are
    concatenated frames-major, utterance u at rows frame_offsets[u]..."""
    offsets = np.asarray(offsets, np.int64)
    Ls, Ms = [], []
    for u in range(len(offsets) - 1):
        L, M = log_mel(pcm[offsets[u]:offsets[u + 1]], p, return_energy=True)
        Ls.append(L)
        Ms.append(M)
    L = np.concatenate(Ls) if Ls else np.zeros((0, p.n_mels))
    M = np.concatenate(Ms) if Ms else np.zeros((0, p.n_mels))
    return (L, M) if return_energy else L


def log_mel_frames(pcm: np.ndarray, offsets, rows, p: Params = DEFAULT):
    """Only the requested output rows of ``log_mel_batch`` (for sampled parity
    at sizes where the whole batch would take too long). Returns (L, M)."""
    offsets = np.asarray(offsets, np.int64)
    fo = frame_offsets(offsets, p.n_fft, p.hop)
    rows = np.asarray(rows, np.int64)
    u = np.searchsorted(fo, rows, side="right") - 1
    t = rows - fo[u]
    start = offsets[u] + t * p.hop
    frames = np.asarray(pcm, np.float64)[start[:, None] + np.arange(p.n_fft)[None, :]]
    M = _mel_energy_of_frames(frames, p)
    return np.log(np.maximum(M, ENERGY_FLOOR)), M


def stream_emit_counts(push_lengths, n_fft: int = 400, hop: int = 160):
    """Frames emitted by each push of a stream, and the carried sample count
    after it: after a push the stream has emitted exactly the frames that the
    audio received so far completes, num_frames(total so far)."""
    emitted, total, out, carry = 0, 0, [], []
    for n in push_lengths:
        total += int(n)
        now = num_frames(total, n_fft, hop)
        out.append(now - emitted)
        emitted = now
        carry.append(total - emitted * hop)
    return out, carry
