"""Pins for the float64 oracle (CPU only).

The oracle is tied here to things other than itself: closed forms, invariants,
library routines it reduces to, brute force on tiny inputs, and the facts the
pages print ("从零理解 ASR：音频基础、Qwen3-ASR 架构，以及离线 vs 流式推理原理",
sections 2.1 and 2.3).  ``test_planted_mistakes_are_caught`` plants plausible
mistakes in the oracle (on the CPU) and checks that some pin fails for each.
"""
import math
import os

import numpy as np
import pytest

import oracle as O
import oracle.logmel_oracle as OM
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
N = 400


def _page_facts():
    facts = {}
    with open(os.path.join(GOLDEN, "page_facts.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("="))
                facts[k] = float(v)
    return facts


# --- closed-form spectrum of a Hamming-windowed cosine ----------------------
def _geom(beta):
    """sum_{n=0}^{N-1} exp(2 pi i n beta) in closed form (Dirichlet kernel)."""
    beta = np.asarray(beta, np.float64)
    out = np.empty(beta.shape, np.complex128)
    near = np.abs(beta - np.round(beta)) < 1e-13
    b = beta[~near]
    out[~near] = np.exp(1j * np.pi * (N - 1) * b) * np.sin(np.pi * N * b) / np.sin(np.pi * b)
    out[near] = N
    return out


def _windowed_cosine_spectrum(nu, phi):
    """X[k] of w[n] cos(2 pi nu n + phi), w = 0.54 - 0.46 cos(2 pi n / (N-1)), by
    expanding both factors into exponentials and summing geometric series."""
    k = np.arange(N // 2 + 1) / N
    d = 1.0 / (N - 1)
    out = np.zeros(k.shape, np.complex128)
    for sgn in (1.0, -1.0):
        base = sgn * nu - k
        term = 0.54 * _geom(base) - 0.23 * (_geom(base + d) + _geom(base - d))
        out += 0.5 * np.exp(1j * sgn * phi) * term
    return out


# --- pins, written as functions so the planted-mistake test can rerun them --
def pin_frame_counts():
    f = _page_facts()
    assert O.num_frames(int(f["samples_30s"])) == 2998          # page's "≈3000", exact count
    assert abs(O.num_frames(int(f["samples_30s"])) - f["frames_30s_page"]) <= 2
    for n, t in [(0, 0), (399, 0), (400, 1), (401, 1), (559, 1), (560, 2), (16000, 98),
                 (480000, 2998), (83_520_000, 521_998), (768_000, 4798)]:
        assert O.num_frames(n) == t, (n, O.num_frames(n), t)
    fo = O.frame_offsets(np.arange(0, 174 * 480000 + 1, 480000))
    assert fo[-1] == 174 * 2998 == 521_652
    counts, carry = O.stream_emit_counts([1280] * 600)
    assert counts[0] == 6 and all(c == 8 for c in counts[1:]) and sum(counts) == 4798
    assert all(c == 320 for c in carry)


def pin_window():
    w = O.hamming_symmetric(N)
    assert np.allclose(w, np.hamming(N), rtol=0, atol=1e-15)           # the page's np.hamming(400)
    assert abs(w[0] - 0.08) < 1e-15 and abs(w[-1] - 0.08) < 1e-15
    assert np.allclose(w, w[::-1], atol=1e-15)
    # sum_{n=0}^{399} cos(2 pi n / 399) = 1 (a full period plus the n = 399 term)
    assert abs(w.sum() - (0.54 * N - 0.46)) < 1e-11


def pin_dft_closed_form():
    rng = np.random.default_rng(7)
    n = np.arange(N)
    for nu, phi in [(25 / N, 0.0), (0.0623, 0.4), (0.3, 0.7), (101.5 / N, -1.1), (0.0, 0.3)]:
        x = np.cos(2 * np.pi * nu * n + phi)
        P = O.power_spectrum((x * O.hamming_symmetric(N))[None, :])[0]
        X = _windowed_cosine_spectrum(nu, phi)
        ref = (X * X.conj()).real
        assert np.max(np.abs(P - ref)) <= 1e-9 * max(ref.max(), 1.0), (nu, phi)
    # Parseval on random frames: sum x^2 = (|X0|^2 + |X_{N/2}|^2 + 2 sum_{0<k<N/2} |Xk|^2) / N
    fw = rng.standard_normal((16, N))
    P = O.power_spectrum(fw)
    lhs = (fw ** 2).sum(1)
    rhs = (P[:, 0] + P[:, -1] + 2 * P[:, 1:-1].sum(1)) / N
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=0)


def pin_dft_library():
    fw = np.random.default_rng(11).standard_normal((8, N))
    P = O.power_spectrum(fw)
    ref = np.abs(np.fft.rfft(fw, n=N, axis=1)) ** 2
    assert np.max(np.abs(P - ref) / ref.max()) < 1e-12


def pin_sinusoid_peak():
    # A sin(2 pi 40k t), bin-centred at bin k: |X[k]| = A * sum(w) / 2 up to the
    # negative-frequency image (~1.5e-6 relative for k = 25)
    A, k = 0.8, 25
    x = A * np.sin(2 * np.pi * (k * 40.0) * np.arange(N) / 16000.0)
    P = O.power_spectrum((x * O.hamming_symmetric(N))[None, :])[0]
    assert int(np.argmax(P)) == k
    assert abs(P[k] / (A * 215.54 / 2) ** 2 - 1) < 1e-5


def pin_zero_and_floor():
    L, M = O.log_mel(np.zeros(16000), return_energy=True)
    assert L.shape == (98, 128) and np.all(M == 0)
    assert np.all(L == math.log(1e-10)) and O.LOG_FLOOR == math.log(1e-10)
    assert O.log_mel(np.zeros(399)).shape == (0, 128)


def pin_mel_scale():
    f = _page_facts()
    assert abs(O.hz_to_mel(1000.0) - 1000.0) < 0.05                    # HTK mel: 1000 Hz ~ 1000 mel
    assert abs(O.hz_to_mel(f["mel_b"]) - f["mel_a"] * math.log10(2.0)) < 1e-9
    fr = np.linspace(0, 8000, 101)
    assert np.allclose(O.mel_to_hz(O.hz_to_mel(fr)), fr, atol=1e-9)
    e = O.mel_edges()
    assert e.shape == (130,) and e[0] == 0.0 and e[-1] == 8000.0
    assert np.allclose(np.diff(O.hz_to_mel(e)), O.hz_to_mel(8000.0) / 129.0, atol=1e-9)


def pin_filterbank_invariants():
    H = O.mel_filterbank()
    e = O.mel_edges()
    f = np.arange(201) * 40.0
    assert H.shape == (128, 201) and H.min() >= 0 and H.max() <= 1 + 1e-12
    assert (H > 0).sum(0).max() <= 2                                   # each bin feeds <= 2 filters
    inner = (f >= e[1]) & (f <= e[128])                                # between filter 0 and 127 centres
    assert np.allclose(H[:, inner].sum(0), 1.0, atol=1e-12)            # partition of unity
    for m in range(128):
        nz = np.nonzero(H[m])[0]
        assert np.all((f[nz] > e[m]) & (f[nz] < e[m + 2]))
    # a filter is empty exactly when no 40 Hz bin lies strictly inside (e_m, e_{m+2}),
    # found here by scanning the bin grid against the edges
    empty = [m for m in range(128) if not np.any((f > e[m]) & (f < e[m + 2]))]
    assert list(np.nonzero(H.sum(1) == 0)[0]) == empty == [0, 3, 6, 13]
    # bins 0 (0 Hz = fmin) and 200 (8000 Hz = fmax) sit on the outer edges: no weight
    assert np.all(H[:, 0] == 0) and np.all(H[:, 200] == 0)
    assert int((H > 0).sum()) == 394


def pin_filterbank_library():
    from transformers.audio_utils import mel_filter_bank
    ref = mel_filter_bank(num_frequency_bins=201, num_mel_filters=128, min_frequency=0.0,
                          max_frequency=8000.0, sampling_rate=16000, norm=None, mel_scale="htk")
    assert np.allclose(O.mel_filterbank(), ref.T, rtol=0, atol=1e-12)


def pin_pipeline_library():
    from transformers.audio_utils import mel_filter_bank, spectrogram, window_function
    fb = mel_filter_bank(num_frequency_bins=201, num_mel_filters=128, min_frequency=0.0,
                         max_frequency=8000.0, sampling_rate=16000, norm=None, mel_scale="htk")
    win = window_function(400, "hamming", periodic=False)
    for x in (W.three_tone(16000).astype(np.float64),
              np.random.default_rng(5).uniform(-1, 1, 4321)):
        ref = spectrogram(x, win, frame_length=400, hop_length=160, fft_length=400, power=2.0,
                          center=False, mel_filters=fb, mel_floor=1e-10, log_mel="log",
                          dtype=np.float64).T
        L = O.log_mel(x)
        assert L.shape == ref.shape
        # the library keeps its spectrum as complex64, so agreement is ~1e-7
        assert np.max(np.abs(L - ref)) < 2e-6


def _brute_force_logmel(x):
    """Pure-Python scalar loops on a tiny input: frame, window, DFT, power,
    triangle filters, log floor."""
    sr, nfft, hop, nm = 16000, 400, 160, 128
    T = 0 if len(x) < nfft else (len(x) - nfft) // hop + 1
    m_lo, m_hi = 0.0, 2595.0 * math.log10(1.0 + 8000.0 / 700.0)
    edges = [700.0 * (10.0 ** ((m_lo + (m_hi - m_lo) * j / (nm + 1)) / 2595.0) - 1.0)
             for j in range(nm + 2)]
    out = []
    for t in range(T):
        xw = [x[t * hop + n] * (0.54 - 0.46 * math.cos(2 * math.pi * n / (nfft - 1)))
              for n in range(nfft)]
        P = []
        for k in range(nfft // 2 + 1):
            re = sum(xw[n] * math.cos(2 * math.pi * k * n / nfft) for n in range(nfft))
            im = -sum(xw[n] * math.sin(2 * math.pi * k * n / nfft) for n in range(nfft))
            P.append(re * re + im * im)
        row = []
        for m in range(nm):
            acc = 0.0
            for k in range(nfft // 2 + 1):
                fk = k * sr / nfft
                wt = max(0.0, min((fk - edges[m]) / (edges[m + 1] - edges[m]),
                                  (edges[m + 2] - fk) / (edges[m + 2] - edges[m + 1])))
                acc += wt * P[k]
            row.append(math.log(max(acc, 1e-10)))
        out.append(row)
    return np.array(out).reshape(T, nm)


def pin_brute_force_tiny():
    rng = np.random.default_rng(3)
    for n in (399, 400, 401, 559, 560):
        x = rng.uniform(-1, 1, n)
        ref = _brute_force_logmel(list(x))
        L = O.log_mel(x)
        assert L.shape == ref.shape == (O.num_frames(n), 128)
        if L.size:
            assert np.max(np.abs(L - ref)) < 1e-8, n


def pin_page1_tones():
    # 0.4 sin 200 Hz + 0.3 sin 400 Hz: tones on bins 5 and 10; the power at each
    # tone bin is (A sum(w) / 2)^2 up to leakage from the other tone
    x = W.page1_test_tones(3.0).astype(np.float64)
    fr = O.frame_signal(x, 400, 160, 0, 4) * O.hamming_symmetric(400)
    P = O.power_spectrum(fr)
    assert np.all(np.argsort(P, axis=1)[:, -2:].min(1) >= 5)
    for k, A in ((5, 0.4), (10, 0.3)):
        assert np.allclose(P[:, k] / (A * 215.54 / 2) ** 2, 1.0, rtol=2e-3)


def pin_golden_rows():
    L = O.log_mel(W.three_tone(16000, seed=0))
    with open(os.path.join(GOLDEN, "three_tone_1s_rows.txt")) as f:
        for line in f:
            if line.startswith("#"):
                continue
            vals = line.split()
            r = int(vals[0])
            ref = np.array([float(v) for v in vals[1:]])
            assert np.array_equal(L[r], ref), r


def pin_shapes():
    f = _page_facts()
    x = np.zeros(int(f["samples_30s"]))
    fr = O.frame_signal(x, int(f["frame_length"]), int(f["hop_length"]))
    assert fr.shape == (2998, 400)
    assert O.power_spectrum(fr[:3]).shape == (3, int(f["rfft_bins"]))
    assert O.log_mel(x[:16000]).shape == (98, int(f["n_mels"]))
    assert O.DEFAULT.sr == f["sample_rate"] and O.DEFAULT.n_fft == f["n_fft"]
    assert O.DEFAULT.hop == f["hop_length"] and O.DEFAULT.n_mels == f["n_mels"]
    assert O.ENERGY_FLOOR == f["energy_floor"]


PINS = [pin_frame_counts, pin_window, pin_dft_closed_form, pin_dft_library, pin_sinusoid_peak,
        pin_zero_and_floor, pin_mel_scale, pin_filterbank_invariants, pin_filterbank_library,
        pin_pipeline_library, pin_brute_force_tiny, pin_page1_tones, pin_golden_rows, pin_shapes]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def test_ragged_batch_concatenates_utterances():
    pcm, off = W.ragged_batch(lengths=[399, 16000, 400, 0, 5000])
    L, M = O.log_mel_batch(pcm, off, return_energy=True)
    fo = O.frame_offsets(off)
    assert list(fo) == [0, 0, 98, 99, 99, 128] and L.shape == (128, 128)
    for u in range(5):
        ref = O.log_mel(pcm[off[u]:off[u + 1]])
        assert np.array_equal(L[fo[u]:fo[u + 1]], ref)
    rows = np.array([0, 50, 97, 98, 99, 127])
    Ls, Ms = O.log_mel_frames(pcm, off, rows)
    assert np.allclose(Ls, L[rows], atol=1e-12)


def test_stream_counts_any_push_sizes():
    rng = np.random.default_rng(9)
    pushes = rng.integers(0, 700, 200)
    counts, carry = O.stream_emit_counts(pushes)
    assert sum(counts) == O.num_frames(int(pushes.sum()))
    tot = np.cumsum(pushes)
    for c, t in zip(carry, tot):
        assert (c == t) if t < 400 else (240 <= c < 400)


# --- planted mistakes -------------------------------------------------------
def _periodic_hamming(n):
    i = np.arange(n, dtype=np.float64)
    return 0.54 - 0.46 * np.cos(2.0 * np.pi * i / n)


def _power_dropped_imag(fw):
    c, s = O.dft_matrices(fw.shape[-1])
    re = fw @ c
    return re * re


def _mel_in_natural_log(f):
    return 2595.0 * np.log(1.0 + np.asarray(f, np.float64) / 700.0)


def _filterbank_shifted(p=O.DEFAULT):
    return np.roll(OM._orig_filterbank(p), 1, axis=1)


def _num_frames_plus_one(n, n_fft=400, hop=160):
    return 0 if n < n_fft else (n - n_fft) // hop + 2


def _filterbank_in_mel_space(p=O.DEFAULT):
    e = O.hz_to_mel(O.mel_edges(p))
    f = O.hz_to_mel(np.arange(p.n_bins) * p.sr / p.n_fft)
    H = np.zeros((p.n_mels, p.n_bins))
    for m in range(p.n_mels):
        H[m] = np.maximum(0, np.minimum((f - e[m]) / (e[m + 1] - e[m]), (e[m + 2] - f) / (e[m + 2] - e[m + 1])))
    return H


MISTAKES = {
    "periodic window": ("hamming_symmetric", _periodic_hamming),
    "dropped imaginary part": ("power_spectrum", _power_dropped_imag),
    "natural log in mel scale": ("hz_to_mel", _mel_in_natural_log),
    "filterbank shifted one bin": ("mel_filterbank", _filterbank_shifted),
    "frame count off by one": ("num_frames", _num_frames_plus_one),
    "triangles linear in mel": ("mel_filterbank", _filterbank_in_mel_space),
}


@pytest.mark.parametrize("name", list(MISTAKES))
def test_planted_mistakes_are_caught(name, monkeypatch):
    attr, bad = MISTAKES[name]
    monkeypatch.setattr(OM, "_orig_filterbank", OM.mel_filterbank, raising=False)
    monkeypatch.setattr(OM, attr, bad)
    monkeypatch.setattr(O, attr, bad)
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"no pin caught: {name}"
