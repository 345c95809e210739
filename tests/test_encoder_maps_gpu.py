"""The encoder-ready index maps applied to the library's real output: the
ragged batch (config 3) through logmel_compute, cut into encoder chunks
(30 s = 3000 frames, padded to 3000 or to 500-frame buckets), and a
stream's pushes cut into 500-frame windows with 50 frames of context on each
side.  The maps equal their oracle and every row a chunk or a window points
at equals the float64 oracle's log-mel row within the tolerance."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from _tolerance import check_against_oracle
from oracle import chunk_oracle as C

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def plan(lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib.Plan()


@pytest.fixture(scope="module")
def ragged(plan):
    pcm, off = W.ragged_batch()
    out = plan.compute(torch.from_numpy(pcm).cuda(), off)
    torch.cuda.synchronize()
    return pcm, off, out


@pytest.mark.parametrize("quantum", [3000, 500])
def test_offline_chunks_of_the_ragged_batch(lib, plan, ragged, quantum):
    pcm, off, out = ragged
    fo = plan.frame_offsets(off)
    chunks = lib.encoder_chunks(fo, 3000, quantum)
    assert np.array_equal(chunks, C.encoder_chunks(fo, 3000, quantum))
    views = lib.chunk_views(out, chunks)
    assert len(views) == len(chunks) and sum(v.shape[0] for v in views) == out.shape[0]
    for (u, row, frames, padded), v in zip(chunks, views):
        assert v.data_ptr() == out[row].data_ptr()            # a view of the rows, not a copy
        assert frames <= padded <= 3000 and padded % quantum == 0 or padded == 3000
        t0 = row - fo[u]                                      # the chunk's first frame in its utterance
        rows = np.arange(t0, t0 + frames)
        L, M = O.log_mel_frames(pcm[off[u]:off[u + 1]], [0, off[u + 1] - off[u]], rows)
        check_against_oracle(v.cpu().numpy(), L, M)


def test_stream_windows_of_pushed_rows(lib, plan):
    S, L, pushes = 2, 1280, 150                               # 12 s per stream at the 80 ms clock
    x = torch.from_numpy(W.stream_signals(S, L * pushes, seed0=9800)).cuda()
    st = lib.Stream(plan, S)
    rows, released = [], []
    for i in range(pushes):
        o, n = st.push_batch(x[:, i * L:(i + 1) * L])
        rows.append(o[0, :n[0]].clone())
        got = torch.cat(rows, 0)
        w = lib.stream_windows(got.shape[0], finished=False)
        assert np.array_equal(w, C.stream_windows(got.shape[0], False))
        released = w
    got = torch.cat(rows, 0)
    final = lib.stream_windows(got.shape[0], finished=True)
    assert np.array_equal(final, C.stream_windows(got.shape[0], True))
    assert len(final) >= len(released) and len(final) == -(-got.shape[0] // 500)
    xs = x[0].cpu().numpy()
    L_, M_ = O.log_mel(xs, return_energy=True)
    assert got.shape[0] == L_.shape[0]
    for k, c0, c1, b0, b1 in final:
        check_against_oracle(got[b0:b1].cpu().numpy(), L_[b0:b1], M_[b0:b1])
    # the page's first windows: [0, 500) with context [0, 550), [500, 1000) with [450, 1050)
    assert tuple(final[0]) == (0, 0, 500, 0, 550) and tuple(final[1]) == (1, 500, 1000, 450, 1050)
