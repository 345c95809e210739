"""The C-ABI library loads and exports every entry point include/logmel.h
declares; argument checks that precede any CUDA call work without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "logmel.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(logmel_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def cdll():
    import __graft_entry__
    path = __graft_entry__._builder().build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("logmel_plan_create", "logmel_plan_destroy", "logmel_num_frames",
                     "logmel_frame_offsets", "logmel_compute", "logmel_stream_create",
                     "logmel_stream_push", "logmel_stream_push_batch", "logmel_stream_get_state",
                     "logmel_stream_set_state", "logmel_stream_destroy", "logmel_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(cdll):
    missing = [n for n in _declared() if not hasattr(cdll, n)]
    assert not missing, missing


def test_binding_wraps_every_declared_symbol():
    import log_mel_spectrogram_logmel_b200 as lm
    assert lm.exported_symbols() == _declared()


def test_status_strings(cdll):
    f = cdll.logmel_status_string
    f.restype = ctypes.c_char_p
    f.argtypes = [ctypes.c_int]
    assert f(0) == b"ok"
    for code in range(1, 7):
        assert f(code) and f(code) != b"unknown status"
    assert f(99) == b"unknown status"


def test_plan_argument_checks_precede_cuda(cdll):
    create = cdll.logmel_plan_create
    create.restype = ctypes.c_int
    create.argtypes = [ctypes.c_int] * 4 + [ctypes.c_float] * 2 + [ctypes.POINTER(ctypes.c_void_p)]
    h = ctypes.c_void_p()
    assert create(16000, 512, 160, 128, 0.0, 8000.0, ctypes.byref(h)) == 2      # n_fft != 400
    assert create(16000, 400, 100, 128, 0.0, 8000.0, ctypes.byref(h)) == 2      # hop != 160
    assert create(16000, 400, 160, 202, 0.0, 8000.0, ctypes.byref(h)) == 2      # n_mels > 201
    assert create(16000, 400, 160, 128, 0.0, 9000.0, ctypes.byref(h)) == 1      # fmax > sr / 2
    assert create(16000, 400, 160, 128, 500.0, 100.0, ctypes.byref(h)) == 1     # fmin >= fmax
    assert create(0, 400, 160, 128, 0.0, 8000.0, ctypes.byref(h)) == 1          # sr <= 0
    assert create(16000, 400, 160, 128, 0.0, 8000.0, None) == 1                 # null out
    assert not h.value


def test_null_handles_are_rejected(cdll):
    nf = cdll.logmel_num_frames
    nf.restype = ctypes.c_int64
    nf.argtypes = [ctypes.c_void_p, ctypes.c_int64]
    assert nf(None, 16000) == -1
    comp = cdll.logmel_compute
    comp.restype = ctypes.c_int
    comp.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] + [ctypes.c_void_p] * 2
    assert comp(None, None, None, 0, None, None) == 1
    cdll.logmel_plan_destroy.argtypes = [ctypes.c_void_p]
    cdll.logmel_plan_destroy(None)
    cdll.logmel_stream_destroy.argtypes = [ctypes.c_void_p]
    cdll.logmel_stream_destroy(None)


def test_noalloc_limits_precede_cuda(cdll):
    """The allocation-free entry point refuses batches beyond its fixed
    scratch (4096 utterances, 32768 tiles) before any CUDA call."""
    f = cdll.logmel_compute_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64] + [ctypes.c_void_p] * 3
    import numpy as np
    many = np.arange(4098, dtype=np.int64) * 400                     # 4097 utterances of one frame
    assert f(ctypes.c_void_p(16), many.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), 4097, ctypes.c_void_p(16),
             None, None) == 7
    long_one = np.array([0, 32768 * 32 * 160 + 400], dtype=np.int64)  # 32769 tiles
    assert f(ctypes.c_void_p(16), long_one.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), 1, ctypes.c_void_p(16),
             None, None) == 7
    bad = np.array([0, 10, 5], dtype=np.int64)                         # decreasing offsets
    assert f(ctypes.c_void_p(16), bad.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), 2, ctypes.c_void_p(16),
             None, None) == 1


def test_noalloc_total_frames_is_the_frame_count(cdll):
    """The plan-free row count of the allocation-free entry point equals the
    oracle's frame count (section 2.3 step 1) on ragged lengths around the
    400-sample frame and the 160-sample hop, and refuses bad offsets."""
    import numpy as np

    import oracle as O
    f = cdll.logmel_noalloc_total_frames
    f.restype = ctypes.c_int64
    f.argtypes = [ctypes.POINTER(ctypes.c_int64), ctypes.c_int64]
    lens = [0, 1, 399, 400, 401, 559, 560, 561, 16000, 480000, 83_520_000]
    off = 7 + np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    p64 = off.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
    assert f(p64, len(lens)) == O.frame_offsets(off)[-1] == sum(O.num_frames(n) for n in lens)
    assert f(p64, 0) == 0
    bad = np.array([0, 10, 5], dtype=np.int64)
    assert f(bad.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), 2) == -1
    assert f(None, 1) == -1
    assert f(p64, -1) == -1


def test_fp32_probe_library_exports_its_entry_point():
    """The FP32 FMA probe bench.py measures the FP32 roof with is built beside
    the library and exports the call its header declares."""
    import __graft_entry__
    path = __graft_entry__._builder().build_peak_probe()
    lib = ctypes.CDLL(path)
    src = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "fp32_peak.h")).read(), flags=re.S)
    names = set(re.findall(r"\b(fp32_[a-z_]+)\s*\(", src))
    assert names == {"fp32_fma_probe"}
    assert hasattr(lib, "fp32_fma_probe")
