"""Python binding of the B200 batched log-mel spectrogram C ABI (include/logmel.h).

Argument marshalling only: every step of the log-mel pipeline runs in the
CUDA library ``liblogmel_b200.so`` built in this directory.  PyTorch supplies
device memory and the current CUDA stream.  Importing fails loudly when the
library has not been built (``python log_mel_spectrogram_logmel_b200/build.py``).

    import torch, log_mel_spectrogram_logmel_b200 as lm
    plan = lm.Plan()                                  # sr 16000, n_fft 400, hop 160, 128 mels, 0-8 kHz
    out = plan.compute(pcm_cuda_f32, offsets_int64)   # [total_frames, 128] fp32 on the GPU

    st = lm.Stream(plan, n_streams=1024)
    out, n = st.push_batch(chunks_cuda_f32)           # [1024, cap, 128], frames per stream

    chunks = lm.encoder_chunks(plan.frame_offsets(offsets_int64))   # 3000-row encoder inputs
    views = lm.chunk_views(out, chunks)                # zero-copy row views
    windows = lm.stream_windows(frames_so_far, finished=False)      # 500-frame chunks, +-50 context

    lm.compute_noalloc(pcm_cuda_f32, offsets_int64, out)  # no device allocation (fixed scratch)
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = ["Plan", "Stream", "LogMelError", "compute_noalloc", "encoder_chunks", "stream_windows", "chunk_views",
           "partition_utterances", "partition_streams", "lib_path", "exported_symbols", "STATUS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblogmel_b200.so")

STATUS = {
    0: "LOGMEL_OK", 1: "LOGMEL_ERR_INVALID_ARG", 2: "LOGMEL_ERR_UNSUPPORTED", 3: "LOGMEL_ERR_CUDA",
    4: "LOGMEL_ERR_OOM", 5: "LOGMEL_ERR_INPUT_TOO_LONG", 6: "LOGMEL_ERR_DEVICE_STATUS",
    7: "LOGMEL_ERR_NOALLOC_LIMIT",
}


class LogMelError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        msg = f"{what}: {STATUS.get(code, code)} ({_lib.logmel_status_string(code).decode()})"
        if code == 3:
            msg += ": " + _lib.logmel_last_error().decode()
        super().__init__(msg)


def lib_path() -> str:
    return _LIB_PATH


if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing; build it with `python log_mel_spectrogram_logmel_b200/build.py`")
_lib = ctypes.CDLL(_LIB_PATH)

_p, _i, _i64, _f, _vp = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
_i64p = ctypes.POINTER(ctypes.c_int64)
_SIGS = {
    "logmel_status_string": (ctypes.c_char_p, [_i]),
    "logmel_last_error": (ctypes.c_char_p, []),
    "logmel_plan_create": (_i, [_i, _i, _i, _i, _f, _f, ctypes.POINTER(_p)]),
    "logmel_plan_destroy": (None, [_p]),
    "logmel_num_frames": (_i64, [_p, _i64]),
    "logmel_frame_offsets": (_i, [_p, _i64p, _i64, _i64p]),
    "logmel_total_frames": (_i64, [_p, _i64p, _i64]),
    "logmel_compute": (_i, [_p, _vp, _i64p, _i64, _vp, _vp]),
    "logmel_compute_noalloc": (_i, [_vp, _i64p, _i64, _vp, _vp, _vp]),
    "logmel_noalloc_total_frames": (_i64, [_i64p, _i64]),
    "logmel_stream_create": (_i, [_p, _i, ctypes.POINTER(_p)]),
    "logmel_stream_destroy": (None, [_p]),
    "logmel_stream_frames_for_push": (_i64, [_p, _i, _i64]),
    "logmel_stream_push": (_i, [_p, _i, _vp, _i64, _vp, _i64, _i64p, _vp]),
    "logmel_stream_push_batch": (_i, [_p, _vp, _i64, _i64, _vp, _i64, _i64p, _vp]),
    "logmel_stream_max_frames": (_i64, [_p, _i64]),
    "logmel_stream_push_batch_ragged": (_i, [_p, _vp, _i64p, _vp, _i64, _i64p, _vp]),
    "logmel_stream_max_frames_ragged": (_i64, [_p, _i64p]),
    "logmel_stream_state_bytes": (_i64, [_p]),
    "logmel_stream_get_state": (_i, [_p, _vp, _i64, _vp]),
    "logmel_stream_set_state": (_i, [_p, _vp, _i64, _vp]),
    "logmel_stream_reset": (_i, [_p, _i, _vp]),
    "logmel_plan_device_status": (_i, [_p, ctypes.POINTER(_i), _vp]),
    "logmel_plan_set_wait_test": (_i, [_p, _i, _i]),
    "logmel_encoder_chunk_count": (_i64, [_i64p, _i64, _i64]),
    "logmel_encoder_chunks": (_i, [_i64p, _i64, _i64, _i64, _vp, _i64, _i64p]),
    "logmel_stream_windows": (_i, [_i64, _i, _i64, _i64, _vp, _i64, _i64p]),
    "logmel_partition_utterances": (_i, [_i64p, _i64, _i, _i64p]),
    "logmel_partition_streams": (_i, [_i64, _i, _i64p]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def exported_symbols() -> list[str]:
    """Names of the C entry points this binding wraps (all must resolve)."""
    return sorted(_SIGS)


def _check(code: int, what: str) -> None:
    if code != 0:
        raise LogMelError(code, what)


def _offsets(offsets) -> np.ndarray:
    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
    if off.ndim != 1 or off.shape[0] < 1:
        raise ValueError("offsets must be a 1-D CSR array of n_utt + 1 int64 entries")
    return off


def _ptr64(a: np.ndarray):
    return a.ctypes.data_as(_i64p)


def _torch():
    import torch
    return torch


def _stream_handle(stream, device):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _check_cuda_f32(t, name, device):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32:
        raise TypeError(f"{name} must be a CUDA float32 tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the plan on {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def compute_noalloc(pcm, offsets, out, device_status=None, stream=None):
    """The allocation-free entry point (logmel_compute_noalloc): the default
    front-end (sr 16000, n_fft 400, hop 160, 128 mels, 0-8 kHz) of a ragged
    batch, written into the caller's ``out`` with no device or pinned
    allocation, for callers whose device memory belongs to another allocator
    or whose thread must not block in cudaMalloc / cudaFree.

    ``out`` (CUDA float32, at least total_frames x 128) and the optional
    ``device_status`` (CUDA int32, one element) are the caller's.  At most
    4096 utterances and 32768 tiles of 32 frames per call; calls that overlap
    on the GPU share one scratch array and race.  Returns ``out``."""
    torch = _torch()
    device = pcm.device if isinstance(pcm, torch.Tensor) else None
    _check_cuda_f32(pcm, "pcm", device)
    _check_cuda_f32(out, "out", device)
    off = _offsets(offsets)
    if off[-1] > pcm.numel():
        raise ValueError("offsets reach beyond pcm")
    total = int(_lib.logmel_noalloc_total_frames(_ptr64(off), off.shape[0] - 1))
    if total < 0:
        raise ValueError("offsets must be non-negative and non-decreasing")
    if out.numel() < total * 128:
        raise ValueError("out is too small")
    st = _vp(0)
    if device_status is not None:
        if (not isinstance(device_status, torch.Tensor) or device_status.dtype != torch.int32
                or device_status.device != device or device_status.numel() < 1):
            raise TypeError("device_status must be an int32 tensor on the device of pcm")
        st = _vp(device_status.data_ptr())
    with torch.cuda.device(device):
        _check(_lib.logmel_compute_noalloc(_vp(pcm.data_ptr()), _ptr64(off), off.shape[0] - 1,
                                           _vp(out.data_ptr()), st, _stream_handle(stream, device)),
               "logmel_compute_noalloc")
    return out


def encoder_chunks(frame_offsets, chunk_frames: int = 3000, quantum: int | None = None) -> np.ndarray:
    """Offline encoder chunks over the rows of a log-mel batch
    (logmel_encoder_chunks): int64 [n, 4] rows (utt, row, frames, padded).
    frame_offsets are the batch's row offsets (Plan.frame_offsets).  Each
    utterance's rows are cut into chunks of at most chunk_frames rows (3000 =
    30 s), padded to a multiple of quantum rows (default chunk_frames: pad to
    3000; smaller: length buckets).  Nothing is copied: see chunk_views."""
    fo = _offsets(frame_offsets)
    n_utt = fo.shape[0] - 1
    q = chunk_frames if quantum is None else int(quantum)
    count = int(_lib.logmel_encoder_chunk_count(_ptr64(fo), n_utt, int(chunk_frames)))
    if count < 0:
        _check(1, "logmel_encoder_chunk_count")
    out = np.zeros((count, 4), dtype=np.int64)
    n = ctypes.c_int64(0)
    _check(_lib.logmel_encoder_chunks(_ptr64(fo), n_utt, int(chunk_frames), q, _vp(out.ctypes.data), count,
                                      ctypes.byref(n)), "logmel_encoder_chunks")
    return out


def stream_windows(n_frames: int, finished: bool, chunk_frames: int = 500, context: int = 50) -> np.ndarray:
    """Streaming encoder windows (logmel_stream_windows): int64 [n, 5] rows
    (chunk, core_begin, core_end, ctx_begin, ctx_end) over a stream's frames,
    for the chunks whose right context has arrived (all chunks once the
    stream has finished)."""
    n = ctypes.c_int64(0)
    code = _lib.logmel_stream_windows(int(n_frames), int(bool(finished)), int(chunk_frames), int(context), None, 0,
                                      ctypes.byref(n))
    if code != 0 and n.value == 0:
        _check(code, "logmel_stream_windows")
    out = np.zeros((n.value, 5), dtype=np.int64)
    _check(_lib.logmel_stream_windows(int(n_frames), int(bool(finished)), int(chunk_frames), int(context),
                                      _vp(out.ctypes.data), n.value, ctypes.byref(n)), "logmel_stream_windows")
    return out


def partition_utterances(frame_offsets, n_parts: int) -> np.ndarray:
    """Data-parallel split of a batch (logmel_partition_utterances): int64
    utt_begin [n_parts + 1]; rank r takes utterances utt_begin[r] ..
    utt_begin[r + 1] - 1 and writes rows frame_offsets[utt_begin[r]] ..
    frame_offsets[utt_begin[r + 1]] of the batch, balanced by frame count."""
    fo = _offsets(frame_offsets)
    out = np.zeros(int(n_parts) + 1, dtype=np.int64)
    _check(_lib.logmel_partition_utterances(_ptr64(fo), fo.shape[0] - 1, int(n_parts), _ptr64(out)),
           "logmel_partition_utterances")
    return out


def partition_streams(n_streams: int, n_parts: int) -> np.ndarray:
    """Stream ids split over ranks (logmel_partition_streams): int64
    stream_begin [n_parts + 1]; rank r takes ids stream_begin[r] .. stream_begin[r + 1] - 1."""
    out = np.zeros(int(n_parts) + 1, dtype=np.int64)
    _check(_lib.logmel_partition_streams(int(n_streams), int(n_parts), _ptr64(out)), "logmel_partition_streams")
    return out


def chunk_views(out, chunks: np.ndarray) -> list:
    """Zero-copy views out[row:row + frames] of the chunks' rows."""
    return [out[int(r):int(r) + int(f)] for _, r, f, _ in chunks]


class Plan:
    """A log-mel plan on the current CUDA device (window, twiddles, filterbank)."""

    def __init__(self, sr: int = 16000, n_fft: int = 400, hop: int = 160, n_mels: int = 128,
                 fmin: float = 0.0, fmax: float = 8000.0, device=None):
        torch = _torch()
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.sr, self.n_fft, self.hop, self.n_mels = sr, n_fft, hop, n_mels
        self.fmin, self.fmax = fmin, fmax
        h = _p()
        with torch.cuda.device(self.device):
            _check(_lib.logmel_plan_create(sr, n_fft, hop, n_mels, fmin, fmax, ctypes.byref(h)),
                   "logmel_plan_create")
        self._h = h
        self._destroy = _lib.logmel_plan_destroy   # kept: module globals may be gone at exit

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._destroy(h)
            self._h = None

    def num_frames(self, n_samples: int) -> int:
        return int(_lib.logmel_num_frames(self._h, int(n_samples)))

    def frame_offsets(self, offsets) -> np.ndarray:
        off = _offsets(offsets)
        fo = np.zeros_like(off)
        _check(_lib.logmel_frame_offsets(self._h, _ptr64(off), off.shape[0] - 1, _ptr64(fo)),
               "logmel_frame_offsets")
        return fo

    def compute(self, pcm, offsets=None, out=None, stream=None):
        """Log-mel of a ragged batch: utterance u = pcm[offsets[u]:offsets[u+1]].
        Returns (or fills) a [total_frames, n_mels] float32 CUDA tensor."""
        torch = _torch()
        _check_cuda_f32(pcm, "pcm", self.device)
        off = _offsets([0, pcm.numel()] if offsets is None else offsets)
        if off[-1] > pcm.numel():
            raise ValueError("offsets reach beyond pcm")
        n_utt = off.shape[0] - 1
        total = int(_lib.logmel_total_frames(self._h, _ptr64(off), n_utt))
        if total < 0:
            _check(1, "logmel_total_frames")
        if out is None:
            out = torch.empty((total, self.n_mels), dtype=torch.float32, device=self.device)
        else:
            _check_cuda_f32(out, "out", self.device)
            if out.numel() < total * self.n_mels:
                raise ValueError("out is too small")
        _check(_lib.logmel_compute(self._h, _vp(pcm.data_ptr()), _ptr64(off), n_utt,
                                   _vp(out.data_ptr()), _stream_handle(stream, self.device)),
               "logmel_compute")
        return out

    def set_wait_test(self, extra_tx_bytes: int, poll_limit: int) -> None:
        """Test hook (logmel_plan_set_wait_test): make the bounded wait on
        each tile's span copies run out (extra expected bytes that never
        arrive, at most poll_limit polls); (0, 0) restores normal operation."""
        _check(_lib.logmel_plan_set_wait_test(self._h, int(extra_tx_bytes), int(poll_limit)),
               "logmel_plan_set_wait_test")

    def device_status(self, stream=None) -> int:
        code = ctypes.c_int(0)
        _check(_lib.logmel_plan_device_status(self._h, ctypes.byref(code), _stream_handle(stream, self.device)),
               "logmel_plan_device_status")
        return code.value


class Stream:
    """Carry state of n_streams independent audio streams on a plan."""

    def __init__(self, plan: Plan, n_streams: int):
        torch = _torch()
        self.plan = plan
        self.n_streams = n_streams
        h = _p()
        with torch.cuda.device(plan.device):
            _check(_lib.logmel_stream_create(plan._h, n_streams, ctypes.byref(h)), "logmel_stream_create")
        self._h = h
        self._destroy = _lib.logmel_stream_destroy   # kept: module globals may be gone at exit

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._destroy(h)
            self._h = None

    def frames_for_push(self, stream_id: int, length: int) -> int:
        """Frames the next push of `length` samples to one stream emits."""
        return int(_lib.logmel_stream_frames_for_push(self._h, stream_id, int(length)))

    def max_frames(self, length: int) -> int:
        """Largest per-stream count the NEXT push_batch of `length` samples
        emits; it grows as the carries fill (a carry holds at most n_fft - 1
        samples), so a buffer reused across pushes is sized with
        (length - 1) // hop + 1 rows, the count for a full carry."""
        return int(_lib.logmel_stream_max_frames(self._h, int(length)))

    def push(self, stream_id: int, chunk, out=None, stream=None):
        """Push a 1-D chunk to one stream; returns the [n, n_mels] frames it completes."""
        torch = _torch()
        _check_cuda_f32(chunk, "chunk", self.plan.device)
        n = self.frames_for_push(stream_id, chunk.numel())
        if n < 0:
            raise ValueError("bad stream id")
        cap = max(n, 1)
        if out is None:
            out = torch.empty((cap, self.plan.n_mels), dtype=torch.float32, device=self.plan.device)
        nf = ctypes.c_int64(0)
        _check(_lib.logmel_stream_push(self._h, stream_id, _vp(chunk.data_ptr()), chunk.numel(),
                                       _vp(out.data_ptr()), out.shape[0], ctypes.byref(nf),
                                       _stream_handle(stream, self.plan.device)), "logmel_stream_push")
        return out[:nf.value]

    def push_batch(self, chunks, out=None, stream=None):
        """Push chunks[s] ([n_streams, len]) to every stream s.  Returns
        (out [n_streams, cap, n_mels], n_frames int64 numpy [n_streams])."""
        torch = _torch()
        if not isinstance(chunks, torch.Tensor) or not chunks.is_cuda or chunks.dtype != torch.float32:
            raise TypeError("chunks must be a CUDA float32 tensor")
        if chunks.dim() != 2 or chunks.shape[0] != self.n_streams or chunks.stride(1) != 1:
            raise ValueError("chunks must be [n_streams, len] with contiguous rows")
        length = chunks.shape[1]
        need = self.max_frames(length)
        nm = self.plan.n_mels
        if out is None:
            out = torch.empty((self.n_streams, max(need, 1), nm), dtype=torch.float32,
                              device=self.plan.device)
        if (not isinstance(out, torch.Tensor) or not out.is_cuda or out.dtype != torch.float32
                or out.dim() != 3 or out.shape[0] != self.n_streams or out.shape[2] != nm
                or out.stride(2) != 1 or out.stride(1) != nm or out.stride(0) % nm):
            raise ValueError("out must be a [n_streams, frames, n_mels] float32 CUDA view with n_mels-contiguous rows")
        if out.shape[1] < need:
            raise ValueError(f"out holds {out.shape[1]} frames per stream, the push emits up to {need}")
        cap = out.stride(0) // nm
        n = np.zeros(self.n_streams, np.int64)
        _check(_lib.logmel_stream_push_batch(self._h, _vp(chunks.data_ptr()), chunks.stride(0), length,
                                             _vp(out.data_ptr()), cap, _ptr64(n),
                                             _stream_handle(stream, self.plan.device)),
               "logmel_stream_push_batch")
        return out, n

    def push_batch_ragged(self, chunks, offsets, out=None, stream=None):
        """Push chunks[offsets[s]:offsets[s + 1]] to every stream s, each its
        own length (0 leaves a stream as it is), in one launch.  chunks is a
        1-D CUDA float32 tensor, offsets host int64 [n_streams + 1].  Returns
        (out [n_streams, cap, n_mels], n_frames int64 numpy [n_streams])."""
        torch = _torch()
        _check_cuda_f32(chunks, "chunks", self.plan.device)
        off = _offsets(offsets)
        if off.shape[0] != self.n_streams + 1:
            raise ValueError("offsets must hold n_streams + 1 entries")
        if off[-1] > chunks.numel():
            raise ValueError("offsets reach beyond chunks")
        need = int(_lib.logmel_stream_max_frames_ragged(self._h, _ptr64(off)))
        if need < 0:
            raise ValueError("offsets must be non-negative and non-decreasing")
        nm = self.plan.n_mels
        if out is None:
            out = torch.empty((self.n_streams, max(need, 1), nm), dtype=torch.float32, device=self.plan.device)
        if (not isinstance(out, torch.Tensor) or not out.is_cuda or out.dtype != torch.float32
                or out.dim() != 3 or out.shape[0] != self.n_streams or out.shape[2] != nm
                or out.stride(2) != 1 or out.stride(1) != nm or out.stride(0) % nm):
            raise ValueError("out must be a [n_streams, frames, n_mels] float32 CUDA view with n_mels-contiguous rows")
        if out.shape[1] < need:
            raise ValueError(f"out holds {out.shape[1]} frames per stream, the push emits up to {need}")
        n = np.zeros(self.n_streams, np.int64)
        _check(_lib.logmel_stream_push_batch_ragged(self._h, _vp(chunks.data_ptr()), _ptr64(off),
                                                    _vp(out.data_ptr()), out.stride(0) // nm, _ptr64(n),
                                                    _stream_handle(stream, self.plan.device)),
               "logmel_stream_push_batch_ragged")
        return out, n

    def state_bytes(self) -> int:
        return int(_lib.logmel_stream_state_bytes(self._h))

    def get_state(self, stream=None) -> bytes:
        buf = ctypes.create_string_buffer(self.state_bytes())
        _check(_lib.logmel_stream_get_state(self._h, buf, len(buf), _stream_handle(stream, self.plan.device)),
               "logmel_stream_get_state")
        return buf.raw

    def set_state(self, blob: bytes, stream=None) -> None:
        buf = ctypes.create_string_buffer(bytes(blob), len(blob))
        _check(_lib.logmel_stream_set_state(self._h, buf, len(blob), _stream_handle(stream, self.plan.device)),
               "logmel_stream_set_state")

    def reset(self, stream_id: int = -1, stream=None) -> None:
        _check(_lib.logmel_stream_reset(self._h, stream_id, _stream_handle(stream, self.plan.device)),
               "logmel_stream_reset")
