"""Pins of the encoder-ready index-map oracle (offline 30 s chunks,
streaming windows) against the pages' printed windows and parameters,
tiling invariants and a per-frame brute force; planted mistakes must fail
a pin.  Integer bookkeeping only, so every comparison is exact."""
import os

import numpy as np
import pytest

from oracle import chunk_oracle as C

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _facts():
    facts = {}
    with open(os.path.join(GOLDEN, "page_facts.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("="))
                facts[k] = float(v)
    return facts


def _page_windows():
    rows = []
    with open(os.path.join(GOLDEN, "stream_windows_page.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k1, cb, ce, xb, xe = map(int, line.split())
                rows.append((k1 - 1, cb, ce, xb, xe))       # the page counts chunks from 1
    return np.array(rows, np.int64)


# ---- oracle pins -----------------------------------------------------------
def test_page_windows_are_reproduced():
    f = _facts()
    chunk, ctx = int(f["stream_chunk_frames"]), int(f["stream_context_frames"])
    page = _page_windows()
    # once frame 1550 has arrived, the right context of the third chunk is in
    got = C.stream_windows(1550, finished=False, chunk_frames=chunk, context=ctx)
    assert np.array_equal(got, page)
    # one frame fewer and the third chunk must wait
    assert np.array_equal(C.stream_windows(1549, False, chunk, ctx), page[:2])


def test_page_chunk_length_and_padding():
    f = _facts()
    frames_per_chunk = int(f["chunk_length_s"] * f["sample_rate"] / f["hop_length"])
    assert frames_per_chunk == int(f["chunk_frames"]) == 3000
    # a 30 s utterance has 2998 frames (no padding in the front-end): one chunk, padded to 3000
    got = C.encoder_chunks([0, 2998])
    assert got.tolist() == [[0, 0, 2998, 3000]]


@pytest.mark.parametrize("seed", range(6))
def test_chunks_tile_every_utterance(seed):
    rng = np.random.default_rng(seed)
    n = rng.integers(0, 9000, 12)
    fo = np.concatenate([[0], np.cumsum(n)])
    for chunk, quantum in ((3000, 3000), (3000, 500), (1000, 128), (7, 3)):
        got = C.encoder_chunks(fo, chunk, quantum)
        for u in range(len(n)):
            mine = got[got[:, 0] == u]
            assert len(mine) == -(-int(n[u]) // chunk)
            if len(mine):
                assert mine[0, 1] == fo[u] and mine[-1, 1] + mine[-1, 2] == fo[u + 1]
                assert np.all(mine[1:, 1] == mine[:-1, 1] + mine[:-1, 2])      # contiguous, disjoint
            assert np.all(mine[:, 2] >= 1) and np.all(mine[:, 2] <= chunk)
            assert np.all(mine[:, 3] >= mine[:, 2]) and np.all(mine[:, 3] <= chunk)
            capped = mine[:, 3] == chunk
            assert np.all((mine[:, 3] % quantum == 0) | capped)
            assert np.all(mine[:, 3] - mine[:, 2] < quantum)                    # the smallest such padding


def _brute_windows(n, finished, chunk, ctx):
    """Per frame: frame f belongs to chunk f // chunk; a chunk is ready when
    frame (k + 1) chunk + ctx - 1 exists (or the stream has finished)."""
    rows = []
    for k in sorted({f // chunk for f in range(n)}):
        core = [f for f in range(n) if f // chunk == k]
        if not finished and (k + 1) * chunk + ctx > n:
            continue
        if finished:
            ctx_frames = [f for f in range(n) if k * chunk - ctx <= f < (k + 1) * chunk + ctx]
        else:
            ctx_frames = [f for f in range(max(0, k * chunk - ctx), (k + 1) * chunk + ctx)]
        core_end = core[-1] + 1 if finished else (k + 1) * chunk
        rows.append((k, core[0], core_end, ctx_frames[0], ctx_frames[-1] + 1))
    return np.array(rows, np.int64).reshape(-1, 5)


@pytest.mark.parametrize("n", [0, 1, 7, 49, 50, 51, 99, 100, 101, 149, 150, 151, 333])
@pytest.mark.parametrize("finished", [False, True])
def test_windows_match_brute_force(n, finished):
    assert np.array_equal(C.stream_windows(n, finished, 50, 10), _brute_windows(n, finished, 50, 10))


def _pins_hold(encoder_chunks, stream_windows):
    """The page pins, for any implementation of the two maps."""
    page = _page_windows()
    ok = np.array_equal(stream_windows(1550, False, 500, 50), page)
    ok &= np.array_equal(stream_windows(1549, False, 500, 50), page[:2])
    ok &= encoder_chunks([0, 2998], 3000, 3000).tolist() == [[0, 0, 2998, 3000]]
    ok &= encoder_chunks([0, 998], 3000, 500).tolist() == [[0, 0, 998, 1000]]
    ok &= encoder_chunks([0, 6998], 3000, 3000)[:, 2].tolist() == [3000, 3000, 998]
    return bool(ok)


def test_planted_mistakes_fail_a_pin():
    assert _pins_hold(C.encoder_chunks, C.stream_windows)

    def unclipped(n, finished, chunk, ctx):               # context not clipped at frame 0
        w = C.stream_windows(n, finished, chunk, ctx).copy()
        w[:, 3] = w[:, 1] - ctx
        return w

    def eager(n, finished, chunk, ctx):                   # released before the right context arrives
        return C.stream_windows(n + ctx, finished, chunk, ctx)

    def drop_tail(fo, chunk, quantum):                    # the last partial chunk dropped
        c = C.encoder_chunks(fo, chunk, quantum)
        return c[c[:, 2] == chunk]

    def no_buckets(fo, chunk, quantum):                   # quantum ignored: always padded to the chunk
        c = C.encoder_chunks(fo, chunk, quantum).copy()
        c[:, 3] = chunk
        return c

    assert not _pins_hold(C.encoder_chunks, unclipped)
    assert not _pins_hold(C.encoder_chunks, eager)
    assert not _pins_hold(drop_tail, C.stream_windows)
    assert not _pins_hold(no_buckets, C.stream_windows)


