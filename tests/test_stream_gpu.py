"""Streaming pushes through the C ABI: the frames emitted across pushes equal
the offline log-mel of the concatenated audio bit for bit, for the 80 ms
clock of the benchmark and for arbitrary push sizes; checkpoint / resume of
the carry state is exact."""
import os

import numpy as np
import pytest

import oracle as O
import workloads as W
from _tolerance import check_against_oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def plan(lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib.Plan()


def _offline(plan, x2d):
    S, N = x2d.shape
    out = plan.compute(x2d.reshape(-1), np.arange(S + 1, dtype=np.int64) * N)
    return out.view(S, -1, plan.n_mels)


def _bits(t):
    return t.contiguous().view(torch.int32)


def test_batch_pushes_80ms_equal_offline(plan, lib):
    S, pushes, L = 16, 60, 1280
    x = torch.from_numpy(W.stream_signals(S, pushes * L, seed0=9000)).cuda()
    st = lib.Stream(plan, S)
    outs = []
    for i in range(pushes):
        o, n = st.push_batch(x[:, i * L:(i + 1) * L])
        assert np.all(n == (6 if i == 0 else 8))
        outs.append(o[:, :n[0]].clone())
    got = torch.cat(outs, 1)
    ref = _offline(plan, x)
    assert got.shape == ref.shape == (S, O.num_frames(pushes * L), 128)
    assert torch.equal(_bits(got), _bits(ref))
    xs = x[3].cpu().numpy()
    L_, M_ = O.log_mel(xs, return_energy=True)
    check_against_oracle(got[3].cpu().numpy(), L_, M_)


@pytest.mark.parametrize("L", [1920, 2560, 160, 100, 399, 401, 5000])
def test_batch_pushes_other_clocks(plan, lib, L):
    S, total = 6, 40000
    pushes = total // L
    x = torch.from_numpy(W.stream_signals(S, pushes * L, seed0=9100)).cuda()
    st = lib.Stream(plan, S)
    outs = []
    for i in range(pushes):
        o, n = st.push_batch(x[:, i * L:(i + 1) * L])
        assert len(set(n.tolist())) == 1
        outs.append(o[:, :n[0]].clone())
    got = torch.cat(outs, 1)
    assert torch.equal(_bits(got), _bits(_offline(plan, x)))


def test_single_stream_arbitrary_pushes(plan, lib):
    rng = np.random.default_rng(21)
    sizes = [0, 1, 159, 160, 399, 400, 1, 1280, 1920, 2560, 7000, 20000, 3, 12345, 0, 6000, 40000, 161]
    total = sum(sizes)
    x = torch.from_numpy(W.speech_like(total, 9200)).cuda()
    st = lib.Stream(plan, 3)
    outs, pos = [], 0
    for L in sizes:
        n_expect = st.frames_for_push(1, L)
        o = st.push(1, x[pos:pos + L])
        assert o.shape[0] == n_expect
        outs.append(o.clone())
        pos += L
    got = torch.cat(outs, 0)
    counts, _ = O.stream_emit_counts(sizes)
    assert [t.shape[0] for t in outs] == counts
    ref = plan.compute(x, [0, total])
    assert torch.equal(_bits(got), _bits(ref))
    assert rng is not None


def test_streams_in_different_states(plan, lib):
    S, L = 8, 1280
    x = torch.from_numpy(W.stream_signals(S, 60000, seed0=9300)).cuda()
    st = lib.Stream(plan, S)
    pre = [0, 17, 160, 333, 399, 400, 1000, 5555]           # warm each stream differently
    outs = [[] for _ in range(S)]
    for s in range(S):
        outs[s].append(st.push(s, x[s, :pre[s]]).clone())
    pos = np.array(pre)
    chunk = torch.empty((S, L), device="cuda")
    for _ in range(20):
        for s in range(S):
            chunk[s] = x[s, pos[s]:pos[s] + L]
        expect = [st.frames_for_push(s, L) for s in range(S)]
        # the next push's largest count; a full carry (n_fft - 1 samples) bounds it
        assert st.max_frames(L) == max(expect) <= (L - 1) // 160 + 1
        o, n = st.push_batch(chunk)
        assert n.tolist() == expect
        for s in range(S):
            outs[s].append(o[s, :n[s]].clone())
        pos += L
    for s in range(S):
        got = torch.cat(outs[s], 0)
        ref = plan.compute(x[s, :pos[s]].contiguous(), [0, int(pos[s])])
        assert torch.equal(_bits(got), _bits(ref)), s


def test_long_pushes_use_several_tiles(plan, lib):
    S, L = 3, 30000                                           # 187 frames per stream per push
    x = torch.from_numpy(W.stream_signals(S, 4 * L, seed0=9400)).cuda()
    st = lib.Stream(plan, S)
    outs = []
    for i in range(4):
        o, n = st.push_batch(x[:, i * L:(i + 1) * L])
        outs.append(o[:, :n[0]].clone())
    got = torch.cat(outs, 1)
    assert torch.equal(_bits(got), _bits(_offline(plan, x)))


def test_checkpoint_resume(plan, lib):
    S, L, pushes, cut = 5, 1280, 30, 13
    x = torch.from_numpy(W.stream_signals(S, pushes * L + 777, seed0=9500)).cuda()
    a = lib.Stream(plan, S)
    ref = []
    for i in range(pushes):
        o, n = a.push_batch(x[:, i * L:(i + 1) * L])
        ref.append(o[:, :n[0]].clone())
        if i == cut:
            blob = a.get_state()
    b = lib.Stream(plan, S)
    b.set_state(blob)
    resumed = []
    for i in range(cut + 1, pushes):
        o, n = b.push_batch(x[:, i * L:(i + 1) * L])
        resumed.append(o[:, :n[0]].clone())
    assert torch.equal(_bits(torch.cat(resumed, 1)), _bits(torch.cat(ref[cut + 1:], 1)))
    with pytest.raises(lib.LogMelError):
        lib.Stream(plan, S + 1).set_state(blob)
    bad = bytearray(blob)
    bad[0] ^= 0xFF
    with pytest.raises(lib.LogMelError):
        b.set_state(bytes(bad))


def test_reset(plan, lib):
    x = torch.from_numpy(W.speech_like(5000, 9600)).cuda()
    st = lib.Stream(plan, 2)
    st.push(0, x[:3000])
    st.reset(0)
    assert st.frames_for_push(0, 399) == 0 and st.frames_for_push(0, 400) == 1
    got = torch.cat([st.push(0, x[:2000]), st.push(0, x[2000:])], 0)
    assert torch.equal(_bits(got), _bits(plan.compute(x, [0, 5000])))


def test_streaming_full_size_1024x600(plan, lib):
    S, pushes, L = 1024, 600, 1280
    N = pushes * L
    workers = max(1, min(16, (os.cpu_count() or 2)))
    xh = W.stream_signals(S, N, workers=workers)
    x = torch.from_numpy(xh).cuda()
    st = lib.Stream(plan, S)
    F = O.num_frames(N)
    got = torch.empty((S, F, 128), device="cuda")
    f = 0
    for i in range(pushes):
        n_expect = st.max_frames(L)
        o, n = st.push_batch(x[:, i * L:(i + 1) * L], out=got[:, f:f + n_expect])
        assert np.all(n == n_expect)
        f += int(n[0])
    assert f == F == 4798
    ref = _offline(plan, x)
    assert torch.equal(_bits(got), _bits(ref))
    # every row of 16 streams against the oracle (76,768 frames), on top of
    # the bitwise equality with offline for all 1024 streams
    rng = np.random.default_rng(5)
    picked = rng.choice(S, 16, replace=False)
    g = got[torch.from_numpy(picked).cuda()].cpu().numpy()
    for i, s in enumerate(picked):
        L_, M_ = O.log_mel(xh[s], return_energy=True)
        check_against_oracle(g[i], L_, M_)
    assert plan.device_status() == 0


def test_long_form_streamed_equals_offline_whole_recording(plan, lib):
    # the 87-minute recording pushed through one stream in pieces from one
    # sample to 3 M samples equals the offline log-mel of the whole recording
    # taken as one utterance: 521,998 frames (continuous, not cut at 30 s)
    pcm, _ = W.long_form()
    N = pcm.shape[0]
    x = torch.from_numpy(pcm).cuda()
    rng = np.random.default_rng(44)
    st = lib.Stream(plan, 1)
    outs, pos = [], 0
    while pos < N:
        L = int(rng.integers(1, 3_000_000)) if rng.random() < 0.7 else int(rng.integers(1, 2000))
        L = min(L, N - pos)
        n_expect = st.frames_for_push(0, L)
        o = st.push(0, x[pos:pos + L])
        assert o.shape[0] == n_expect
        outs.append(o)
        pos += L
    got = torch.cat(outs, 0)
    assert got.shape == (O.num_frames(N), 128) == (521_998, 128)
    ref = plan.compute(x, [0, N])
    assert torch.equal(_bits(got), _bits(ref))
    # every row against the oracle, 20,000 rows at a time
    g = got.cpu().numpy()
    for r0 in range(0, g.shape[0], 20_000):
        rows = np.arange(r0, min(g.shape[0], r0 + 20_000))
        L_, M_ = O.log_mel_frames(pcm, [0, N], rows)
        check_against_oracle(g[rows], L_, M_)
    assert plan.device_status() == 0


def test_ragged_batch_pushes_equal_offline(plan, lib):
    """One launch per call, every stream advancing by its own length (0 to
    5000 samples, mixed across streams and calls): each stream's frames equal
    the offline log-mel of its concatenated audio bit for bit, and the
    per-push counts follow the oracle's emission rule."""
    S, calls = 12, 50
    sizes = np.array([0, 1, 159, 160, 399, 1280, 1920, 2560, 5000])
    rng = np.random.default_rng(61)
    lens = rng.choice(sizes, size=(calls, S))
    lens[7] = 0                                               # a call where nothing arrives
    lens[8] = 5000                                            # a call where every stream emits > 28 frames
    total = lens.sum(0)
    x = torch.from_numpy(W.stream_signals(S, int(total.max()), seed0=9700)).cuda()
    st = lib.Stream(plan, S)
    outs = [[] for _ in range(S)]
    pos = np.zeros(S, np.int64)
    for c in range(calls):
        off = np.concatenate([[0], np.cumsum(lens[c])]).astype(np.int64)
        packed = torch.cat([x[s, pos[s]:pos[s] + lens[c, s]] for s in range(S)]).contiguous()
        if packed.numel() == 0:
            packed = torch.zeros(1, device="cuda")
        o, n = st.push_batch_ragged(packed, off)
        for s in range(S):
            outs[s].append(o[s, :n[s]].clone())
        pos += lens[c]
    for s in range(S):
        counts, carry = O.stream_emit_counts(lens[:, s].tolist())
        assert [t.shape[0] for t in outs[s]] == counts, s
        got = torch.cat(outs[s], 0)
        ref = plan.compute(x[s, :pos[s]].contiguous(), [0, int(pos[s])])
        assert torch.equal(_bits(got), _bits(ref)), s
    # the ragged form equals the uniform one when all lengths are equal
    a, b = lib.Stream(plan, S), lib.Stream(plan, S)
    L = 1280
    for i in range(6):
        chunk = x[:, i * L:(i + 1) * L].contiguous()
        oa, na = a.push_batch(chunk)
        ob, nb = b.push_batch_ragged(chunk.reshape(-1), np.arange(S + 1, dtype=np.int64) * L)
        assert np.array_equal(na, nb)
        assert torch.equal(_bits(oa[:, :na[0]]), _bits(ob[:, :nb[0]]))
    assert plan.device_status() == 0
