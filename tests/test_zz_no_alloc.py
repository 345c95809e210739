"""The allocation-free entry point, logmel_compute_noalloc.

It exists for callers that cannot call cudaMalloc: code whose device memory
belongs to another allocator (a serving runtime or host application that
reserves the GPU's memory and hands out buffers) and real-time audio code
that must not block in cudaMalloc / cudaFree.  It keeps its tables, ragged
metadata and tile descriptors in one fixed device array shared by every
call, so these tests check that calls in a row -- the first at the array's
maximum size (4096 utterances: its index map and tile descriptors fill the
scratch), then a small ragged batch whose index map travels in the launch,
then 300 ragged utterances at unaligned offsets that go through the scratch
again with fewer tiles than the first call left there -- each match the
plan-based logmel_compute bit for bit, and that a call made after the
one-time set-up changes neither the device's free memory nor the PyTorch
allocator's counters.

This file is collected last on purpose: the first call on a device does the
entry point's one-time set-up, and the tests must pass both alone in a fresh
process and after every other test has run.
"""
import ctypes

import numpy as np
import pytest

from _tolerance import TOL

MAX_UTT, MAX_TILES = 4096, 32768


def _total_rows(lib, off):
    offs = np.ascontiguousarray(off, dtype=np.int64)
    n = lib._lib.logmel_noalloc_total_frames(offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                             offs.shape[0] - 1)
    assert n >= 0
    return int(n)


def _noalloc(lib, pcm, off, out, status):
    import torch
    offs = np.ascontiguousarray(off, dtype=np.int64)
    return lib._lib.logmel_compute_noalloc(
        ctypes.c_void_p(pcm.data_ptr()), offs.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        offs.shape[0] - 1, ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _max_size_batch(dev):
    """4096 utterances of 41200 samples (256 frames, 8 tiles each): exactly
    the scratch's 4096 utterances and 32768 tiles; offsets 16-byte aligned."""
    import torch
    g = torch.Generator(device=dev).manual_seed(11)
    n = 255 * 160 + 400
    off = np.arange(MAX_UTT + 1, dtype=np.int64) * n
    pcm = 0.3 * torch.randn(int(off[-1]), generator=g, device=dev)
    return pcm, off


def _small_ragged_batch(dev):
    """13 utterances whose lengths are not multiples of 160, some below 400
    samples (no rows) or empty, starting at sample 3, so most utterances
    start off the 16-byte grid and the 160-sample row grid."""
    import torch
    lens = np.array([16000, 399, 400, 401, 5117, 0, 47999, 160 * 33 + 400, 123457, 250, 9001, 32000, 777],
                    dtype=np.int64)
    off = 3 + np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    g = torch.Generator(device=dev).manual_seed(12)
    pcm = 0.5 * torch.randn(int(off[-1]) + 5, generator=g, device=dev)
    return pcm, off


def _ragged_beyond_inline(dev):
    """300 utterances (more than the 256 whose index map fits in the launch)
    of 401..20000 samples at odd offsets: the index map and the tile
    descriptors go through the scratch again, with far fewer tiles than the
    maximum-size call left there."""
    import torch
    lens = np.random.default_rng(13).integers(401, 20000, 300).astype(np.int64)
    off = 1 + np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    g = torch.Generator(device=dev).manual_seed(14)
    pcm = 0.4 * torch.randn(int(off[-1]) + 3, generator=g, device=dev)
    return pcm, off


@pytest.mark.gpu
def test_noalloc_matches_compute_on_calls_in_a_row():
    import torch
    import log_mel_spectrogram_logmel_b200 as lm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    plan = lm.Plan(device=dev)
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    for make in (_max_size_batch, _small_ragged_batch, _ragged_beyond_inline):
        pcm, off = make(dev)
        total = _total_rows(lm, off)
        got = torch.full((total, 128), float("nan"), device=dev)
        assert _noalloc(lm, pcm, off, got, status) == 0
        torch.cuda.synchronize()
        want = plan.compute(pcm, off)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.isfinite(got).all()
        err = (got - want).abs().max().item()
        assert err <= TOL, (make.__name__, err)
        # same kernel and tables: the two entry points agree bit for bit
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), make.__name__
        del pcm, got, want
    assert plan.device_status() == 0


@pytest.mark.gpu
def test_noalloc_call_allocates_nothing():
    """After the one-time set-up on the device, a call at the maximum size
    leaves the device's free memory (cudaMemGetInfo) and the PyTorch caching
    allocator's counters exactly as they were."""
    import torch
    import log_mel_spectrogram_logmel_b200 as lm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    pcm, off = _max_size_batch(dev)
    out = torch.empty((_total_rows(lm, off), 128), device=dev)
    assert _noalloc(lm, pcm, off, out, status) == 0            # set-up (first call on this device)
    torch.cuda.synchronize()
    keys = ("allocation.all.allocated", "segment.all.allocated", "reserved_bytes.all.current",
            "allocated_bytes.all.current")
    before_stats = {k: torch.cuda.memory_stats(dev).get(k) for k in keys}
    free_before, _ = torch.cuda.mem_get_info(dev)
    for _ in range(2):
        assert _noalloc(lm, pcm, off, out, status) == 0
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info(dev)
    after_stats = {k: torch.cuda.memory_stats(dev).get(k) for k in keys}
    assert free_after == free_before, (free_before, free_after)
    assert after_stats == before_stats
    assert int(status.item()) == 0


@pytest.mark.gpu
def test_noalloc_binding_and_limits():
    import torch
    import log_mel_spectrogram_logmel_b200 as lm

    dev = torch.device("cuda", 0)
    pcm = torch.zeros(MAX_UTT * 400 + 400, device=dev)
    out = torch.empty(1, 128, device=dev)
    too_many = np.arange(MAX_UTT + 2, dtype=np.int64) * 400         # 4097 utterances
    with pytest.raises(lm.LogMelError, match="NOALLOC_LIMIT"):
        lm.compute_noalloc(pcm, too_many, torch.empty(MAX_UTT + 1, 128, device=dev))
    long_one = np.array([0, (MAX_TILES * 32) * 160 + 400], dtype=np.int64)   # 32769 tiles
    big = torch.zeros(int(long_one[-1]), device=dev)
    with pytest.raises(lm.LogMelError, match="NOALLOC_LIMIT"):
        lm.compute_noalloc(big, long_one, torch.empty(MAX_TILES * 32 + 1, 128, device=dev))
    del big
    # through the binding, with the default status word inside the scratch
    x = torch.sin(torch.arange(16000, device=dev, dtype=torch.float32) * (2 * np.pi * 440 / 16000))
    plan = lm.Plan(device=dev)
    got = lm.compute_noalloc(x, [0, 16000], torch.empty(98, 128, device=dev))
    assert torch.equal(got, plan.compute(x, [0, 16000]))
    assert lm.compute_noalloc(x, [0, 399], out) is out               # no frames: nothing to do
