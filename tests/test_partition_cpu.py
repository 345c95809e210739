"""The data-parallel split of a batch over ranks: the oracle's definition
pinned by closed forms and invariants, the C library equal to the oracle,
and the split exercised by two gloo ranks on CPU."""
import os
import socket
import sys

import numpy as np
import pytest

from oracle import partition_oracle as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fo(frames):
    return np.concatenate([[0], np.cumsum(frames)]).astype(np.int64)


# --- pins of the oracle -----------------------------------------------------
def test_equal_utterances_split_equally():
    for n, g in ((64, 1), (64, 2), (64, 8), (12, 3), (2998, 7)):
        cuts = P.partition_utterances(_fo([2998] * n), g)
        sizes = np.diff(cuts)
        assert sizes.sum() == n
        if n % g == 0:
            assert np.all(sizes == n // g)
        assert sizes.max() - sizes.min() <= 1


def test_nearest_boundary_not_first_past_the_target():
    # frames 10, 2, 10, 6 (total 28, half 14): boundary 12 is nearer than 22
    assert P.partition_utterances([0, 10, 12, 22, 28], 2) == [0, 2, 4]
    # one utterance over three ranks: targets 1/3 and 2/3 of it
    assert P.partition_utterances([0, 100], 3) == [0, 0, 1, 1]
    # ties go to the smaller index: boundaries 10 and 11 around 10.5 (scaled 21)
    assert P.partition_utterances([0, 10, 11, 21], 2) == [0, 1, 3]
    # utterances without frames: the cut is the first index of a plateau
    assert P.partition_utterances([0, 5, 5, 5, 10], 2) == [0, 1, 4]
    # no frames at all: everything on the last rank
    assert P.partition_utterances([0, 0, 0, 0], 3) == [0, 0, 0, 3]


def test_partition_invariants_on_random_batches():
    rng = np.random.default_rng(1)
    for trial in range(200):
        n = int(rng.integers(0, 60))
        frames = rng.integers(0, 3000, n) * (rng.random(n) > 0.15)
        g = int(rng.integers(1, 9))
        fo = _fo(frames) + int(rng.integers(0, 50))
        cuts = P.partition_utterances(fo, g)
        assert cuts[0] == 0 and cuts[-1] == n and len(cuts) == g + 1
        assert all(a <= b for a, b in zip(cuts[:-1], cuts[1:]))
        loads = np.diff(fo[cuts])
        assert loads.sum() == fo[-1] - fo[0]
        longest = int(frames.max()) if n else 0
        mean = (fo[-1] - fo[0]) / g
        assert np.all(np.abs(loads - mean) <= longest + 1e-9), (frames, g, loads)


def test_stream_split():
    assert P.partition_streams(1024, 8) == [128 * r for r in range(9)]
    for s, g in ((10, 3), (1, 4), (0, 2), (1023, 8)):
        b = P.partition_streams(s, g)
        sizes = np.diff(b)
        assert b[0] == 0 and b[-1] == s and sizes.max() - sizes.min() <= 1


def test_planted_mistake_fails_a_pin():
    """Cutting at the first boundary at or past the target, instead of the
    nearest one, breaks the pinned 10 / 2 / 10 / 6 case."""
    def first_past(fo, g):
        tot = fo[-1] - fo[0]
        return [0] + [next(u for u in range(len(fo)) if g * (fo[u] - fo[0]) >= r * tot)
                      for r in range(1, g)] + [len(fo) - 1]
    assert first_past([0, 10, 12, 22, 28], 2) != [0, 2, 4]


# --- the C library equals the oracle -----------------------------------------
def test_library_partition_equals_oracle():
    import log_mel_spectrogram_logmel_b200 as lm
    rng = np.random.default_rng(2)
    for trial in range(300):
        n = int(rng.integers(0, 80))
        frames = rng.integers(0, 4000, n) * (rng.random(n) > 0.2)
        g = int(rng.integers(1, 17))
        fo = _fo(frames) + int(rng.integers(0, 7))
        assert lm.partition_utterances(fo, g).tolist() == P.partition_utterances(fo, g), (frames, g)
    for s, g in ((1024, 8), (10, 3), (0, 5), (7, 1)):
        assert lm.partition_streams(s, g).tolist() == P.partition_streams(s, g)
    with pytest.raises(lm.LogMelError):
        lm.partition_utterances([0, 10, 5], 2)
    with pytest.raises(lm.LogMelError):
        lm.partition_utterances([0, 10], 0)


# --- two ranks on CPU ----------------------------------------------------------
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import log_mel_spectrogram_logmel_b200 as lm
    import workloads as W
    from oracle import logmel_oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # the ragged batch's lengths (config 3): every rank computes the same
        # split and keeps its own part
        lengths = np.random.default_rng(3).integers(W.SR, W.CLIP_30S + 1, 256)
        off = W.offsets_from_lengths(lengths)
        fo = O.frame_offsets(off)
        begin = lm.partition_utterances(fo, world)
        mine = (int(begin[rank]), int(begin[rank + 1]))
        rows = (int(fo[mine[0]]), int(fo[mine[1]]))
        parts = [None] * world
        dist.all_gather_object(parts, (mine, rows))
        q.put((rank, parts, int(fo[-1]), int(np.diff(fo).max())))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_cover_the_batch_once_and_balanced():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, parts0, total, longest), (_, parts1, _, _) = res
    assert parts0 == parts1                                   # every rank agrees on the split
    (u0, r0), (u1, r1) = parts0
    assert u0[0] == 0 and u0[1] == u1[0] and u1[1] == 256     # every utterance exactly once
    assert r0[0] == 0 and r0[1] == r1[0] and r1[1] == total   # rows tile the batch's rows
    for a, b in (r0, r1):
        assert abs((b - a) - total / 2) <= longest            # within one utterance of the mean
