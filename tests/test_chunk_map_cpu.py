"""The encoder-ready index maps of the C library (logmel_encoder_chunks,
logmel_stream_windows) against the pinned oracle, exactly, plus their
zero-copy views and error behaviour."""
import numpy as np
import pytest

from oracle import chunk_oracle as C


# ---- C functions against the oracle ------------------------------------------
@pytest.fixture(scope="module")
def lm():
    import __graft_entry__
    __graft_entry__._builder().build()
    import log_mel_spectrogram_logmel_b200 as m
    return m


@pytest.mark.parametrize("seed", range(8))
def test_encoder_chunks_match_oracle(lm, seed):
    rng = np.random.default_rng(100 + seed)
    n_utt = int(rng.integers(0, 40))
    n = rng.integers(0, 20000, n_utt)
    n[rng.random(n_utt) < 0.2] = 0
    fo = (int(rng.integers(0, 50)) + np.concatenate([[0], np.cumsum(n)])).astype(np.int64)
    for chunk, quantum in ((3000, None), (3000, 500), (2000, 128), (1, 1)):
        want = C.encoder_chunks(fo, chunk, chunk if quantum is None else quantum)
        got = lm.encoder_chunks(fo, chunk, quantum)
        assert np.array_equal(got, want)


@pytest.mark.parametrize("seed", range(8))
def test_stream_windows_match_oracle(lm, seed):
    rng = np.random.default_rng(200 + seed)
    for _ in range(25):
        n = int(rng.integers(0, 5000))
        chunk = int(rng.integers(1, 700))
        ctx = int(rng.integers(0, 120))
        for finished in (False, True):
            assert np.array_equal(lm.stream_windows(n, finished, chunk, ctx), C.stream_windows(n, finished, chunk, ctx))


def test_views_are_zero_copy(lm):
    out = np.arange(12 * 3, dtype=np.float32).reshape(12, 3)
    ch = lm.encoder_chunks([0, 5, 12], chunk_frames=4)
    views = lm.chunk_views(out, ch)
    assert [v.shape[0] for v in views] == [4, 1, 4, 3]
    assert all(np.shares_memory(v, out) for v in views)
    assert np.array_equal(np.concatenate(views), out)


def test_errors(lm):
    with pytest.raises(lm.LogMelError):
        lm.encoder_chunks([0, 5], chunk_frames=0)
    with pytest.raises(lm.LogMelError):
        lm.encoder_chunks([0, 5], quantum=0)
    with pytest.raises(lm.LogMelError):
        lm.encoder_chunks([0, 9, 5])                        # decreasing offsets
    with pytest.raises(ValueError):
        C.encoder_chunks([0, 9, 5])
    with pytest.raises(lm.LogMelError):
        lm.stream_windows(-1, True)
    with pytest.raises(lm.LogMelError):
        lm.stream_windows(10, True, context=-1)
    import ctypes
    n = ctypes.c_int64(0)
    fo = np.array([0, 9000], np.int64)
    buf = np.zeros((1, 4), np.int64)
    # capacity too small: nothing written, the needed count reported
    code = lm._lib.logmel_encoder_chunks(fo.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), 1, 3000, 3000,
                                         ctypes.c_void_p(buf.ctypes.data), 1, ctypes.byref(n))
    assert code == 1 and n.value == 3 and not buf.any()
