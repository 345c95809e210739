"""GPU parity of the offline path (logmel_compute through the C ABI) against
the float64 oracle, on the benchmark workloads and the edge cases."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from _tolerance import FLOOR32, check_against_oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def plan(lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib.Plan()


def _run(plan, pcm, off):
    x = torch.from_numpy(np.ascontiguousarray(pcm, np.float32)).cuda()
    out = plan.compute(x, off)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_three_tone_1s(plan):
    x = W.three_tone(16000, seed=0)
    g = _run(plan, x, [0, len(x)])
    L, M = O.log_mel(x, return_energy=True)
    assert g.shape == (98, 128)
    s = check_against_oracle(g, L, M)
    assert s["zero_cells"] == 98 * 4          # filters 0, 3, 6, 13 hold no bin


def test_dense_batch_small_full_compare(plan):
    pcm, off = W.dense_batch(4)
    g = _run(plan, pcm, off)
    L, M = O.log_mel_batch(pcm, off, return_energy=True)
    check_against_oracle(g, L, M)


def test_ragged_batch_small_full_compare(plan):
    pcm, off = W.ragged_batch(n_utt=24, seed=33)
    g = _run(plan, pcm, off)
    L, M = O.log_mel_batch(pcm, off, return_energy=True)
    check_against_oracle(g, L, M)


def test_batch_beyond_inline_metadata(plan):
    """More than 256 utterances: the ragged index map goes to the device by a
    copy and the tile descriptors through the kernel's scratch, instead of
    travelling in the launch parameters.  Both routes give the same bits."""
    lengths = np.random.default_rng(71).integers(200, 9000, 300)
    pcm, off = W.ragged_batch(lengths=lengths, seed0=5000)
    g = _run(plan, pcm, off)
    L, M = O.log_mel_batch(pcm, off, return_energy=True)
    check_against_oracle(g, L, M)
    # the same audio as two batches of 150 utterances (parameter route)
    h = 150
    first = _run(plan, pcm[:off[h]], off[:h + 1])
    second = _run(plan, pcm[off[h]:], off[h:] - off[h])
    both = np.concatenate([first, second])
    assert np.array_equal(both.view(np.int32), g.view(np.int32))


def check_all_rows(g, pcm, off, utts_per_chunk=16):
    """Every row of a full-size batch against the oracle, a few utterances at
    a time (the oracle's float64 energies of a whole long-form batch would
    take about 1 GB of host memory at once)."""
    fo = O.frame_offsets(off)
    assert g.shape == (fo[-1], 128)
    worst, cells = 0.0, 0
    for u0 in range(0, len(off) - 1, utts_per_chunk):
        u1 = min(len(off) - 1, u0 + utts_per_chunk)
        sub = off[u0:u1 + 1]
        L, M = O.log_mel_batch(pcm[sub[0]:sub[-1]], sub - sub[0], return_energy=True)
        st = check_against_oracle(g[fo[u0]:fo[u1]], L, M)
        worst = max(worst, st.get("max_err", 0.0))
        cells += st["cells"]
    assert cells == g.size
    return worst


def test_dense_batch_full_size(plan):
    pcm, off = W.dense_batch(64)
    g = _run(plan, pcm, off)
    assert g.shape == (64 * 2998, 128)
    check_all_rows(g, pcm, off)


def test_ragged_batch_full_size(plan):
    pcm, off = W.ragged_batch()
    g = _run(plan, pcm, off)
    assert g.shape == (O.frame_offsets(off)[-1], 128)
    check_all_rows(g, pcm, off)


def test_long_form_full_size(plan):
    pcm, off = W.long_form()
    g = _run(plan, pcm, off)
    fo = O.frame_offsets(off)
    assert g.shape == (174 * 2998, 128) == (521_652, 128)
    # the all-zero frames are many (about a fifth of the recording), and every
    # one of them must be the exact floor in every band
    nz = np.concatenate([[0], np.cumsum(pcm != 0, dtype=np.int64)])
    silent = []
    for u in range(len(off) - 1):
        t = np.arange(fo[u + 1] - fo[u])
        s0 = off[u] + 160 * t
        silent.append((nz[s0 + 400] - nz[s0]) == 0)
    silent = np.concatenate(silent)
    assert silent.sum() > 50_000
    assert np.all(g[silent] == FLOOR32)
    check_all_rows(g, pcm, off)


def test_edge_lengths_and_unaligned_offsets(plan):
    lengths = [0, 399, 400, 401, 559, 560, 160 * 31 + 400, 160 * 32 + 400, 160 * 63 + 400, 17, 16000, 3]
    rng = np.random.default_rng(8)
    pcm = rng.uniform(-1, 1, 5 + sum(lengths)).astype(np.float32)
    off = 5 + W.offsets_from_lengths(lengths)           # offsets[0] = 5: odd, unaligned starts
    g = _run(plan, pcm, off)
    L, M = O.log_mel_batch(pcm, off, return_energy=True)
    assert g.shape[0] == O.frame_offsets(off)[-1] == sum(O.num_frames(n) for n in lengths)
    check_against_oracle(g, L, M)


@pytest.mark.parametrize("base_shift", [0, 1, 2, 3])
def test_span_staging_at_every_alignment(plan, base_shift):
    """Utterances whose starts cover every residue mod 4 and several mod 160,
    in a buffer that ends at the last utterance, with the buffer itself
    starting 0..3 floats past a 16-byte boundary.  Tiles are staged by the
    row tensor copy, the shifted tensor copy, per-block bulk copies (shifted
    or not) or cp.async, depending on where they start and how close they
    end to the buffer's end; every route must give the oracle's values."""
    lengths = [16000 + 160 * 3, 4001, 16002, 8003, 12004, 160 * 50 + 1, 400, 20397, 9000 + 157, 5001, 402]
    pcm_np, off = W.ragged_batch(lengths=lengths, seed0=7100)
    starts = off[:-1] + base_shift
    assert {int(v % 4) for v in starts} == {0, 1, 2, 3}
    big = torch.zeros(len(pcm_np) + 8, dtype=torch.float32, device="cuda")
    pcm = big[base_shift:base_shift + len(pcm_np)]
    pcm.copy_(torch.from_numpy(pcm_np).cuda())
    assert pcm.is_contiguous() and (pcm.data_ptr() - big.data_ptr()) == 4 * base_shift
    g = plan.compute(pcm, off)
    torch.cuda.synchronize()
    L, M = O.log_mel_batch(pcm_np, off, return_energy=True)
    check_against_oracle(g.cpu().numpy(), L, M)
    assert plan.device_status() == 0


def test_zero_input_is_exact_floor(plan):
    g = _run(plan, np.zeros(48000, np.float32), [0, 48000])
    assert g.shape == (298, 128) and np.all(g == FLOOR32)


def test_empty_batches(plan):
    x = torch.zeros(1000, device="cuda")
    assert plan.compute(x, [0]).shape == (0, 128)
    assert plan.compute(x, [0, 100, 399, 399]).shape == (0, 128)


@pytest.mark.parametrize("n_mels,fmin,fmax", [(80, 20.0, 7600.0), (201, 0.0, 8000.0), (1, 100.0, 4000.0),
                                              (40, 0.0, 8000.0)])
def test_other_filterbanks(lib, n_mels, fmin, fmax):
    p = lib.Plan(n_mels=n_mels, fmin=fmin, fmax=fmax)
    pcm, off = W.ragged_batch(lengths=[16000, 7000, 30000], seed0=77)
    g = _run(p, pcm, off)
    L, M = O.log_mel_batch(pcm, off, O.Params(n_mels=n_mels, fmin=fmin, fmax=fmax), return_energy=True)
    check_against_oracle(g, L, M)


@pytest.mark.parametrize("sr,n_mels,fmax", [(8000, 64, 4000.0), (22050, 128, 11025.0), (24000, 80, 12000.0)])
def test_other_sample_rates(lib, sr, n_mels, fmax):
    """The plan places bin k at k * sr / 400 Hz: other rates move every
    triangle onto other bins (same 400-sample frames and 160-sample hop)."""
    p = lib.Plan(sr=sr, n_mels=n_mels, fmin=0.0, fmax=fmax)
    pcm, off = W.ragged_batch(lengths=[16000, 7001, 30000], seed0=78)
    g = _run(p, pcm, off)
    L, M = O.log_mel_batch(pcm, off, O.Params(sr=sr, n_mels=n_mels, fmin=0.0, fmax=fmax), return_energy=True)
    check_against_oracle(g, L, M)


def test_bounded_span_wait_runs_out_and_reports(lib):
    """The bounded wait on a tile's span copies: with the test hook arming
    each tile's barrier with 64 more bytes than its copies bring (every copy
    still lands), the wait gives up after 1024 polls, the plan's status word
    reads 3 (copy timeout) and the call returns; with the hook off, the same
    plan computes the batch correctly again."""
    p = lib.Plan()
    pcm, off = W.dense_batch(4)
    x = torch.from_numpy(pcm).cuda()
    p.set_wait_test(64, 1 << 10)
    p.compute(x, off)
    torch.cuda.synchronize()
    assert p.device_status() == 3
    p.set_wait_test(0, 0)
    g = _run(p, pcm, off)
    assert p.device_status() == 0
    L, M = O.log_mel_batch(pcm, off, return_energy=True)
    check_against_oracle(g, L, M)
    with pytest.raises(lib.LogMelError):
        p.set_wait_test(-16, 0)


def test_bitwise_deterministic(plan):
    pcm, off = W.ragged_batch(n_utt=8, seed=12)
    a = _run(plan, pcm, off)
    b = _run(plan, pcm, off)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_errors_are_reported(lib, plan):
    x = torch.zeros(1000, device="cuda")
    with pytest.raises(lib.LogMelError) as e:
        plan.compute(x, [0, 500, 400])
    assert e.value.code == 1
    with pytest.raises(lib.LogMelError) as e:
        lib.Plan(hop=100)
    assert e.value.code == 2
    assert plan.device_status() == 0


def test_sizes_beyond_the_kernels_index_range_are_refused(lib, plan):
    """Frame counts past int32 return LOGMEL_ERR_INPUT_TOO_LONG before any
    work is enqueued (nothing is truncated); the buffers are never touched,
    so small ones stand in for the huge input the offsets describe."""
    import ctypes
    x = torch.zeros(1024, device="cuda")
    out = torch.zeros(16, 128, device="cuda")
    for off in ([0, 160 * (2 ** 31) + 400], [0, 160 * (2 ** 30) + 400, 2 * 160 * (2 ** 30) + 800]):
        o = np.ascontiguousarray(off, np.int64)
        code = lib._lib.logmel_compute(plan._h, ctypes.c_void_p(x.data_ptr()),
                                       o.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), len(off) - 1,
                                       ctypes.c_void_p(out.data_ptr()), None)
        assert code == 5, code
    torch.cuda.synchronize()
    assert not out.any()
    assert plan.device_status() == 0


@pytest.mark.parametrize("n_parts", [2, 3, 8])
def test_partitioned_batch_equals_whole(lib, plan, n_parts):
    """The data-parallel split: each part of the ragged batch, copied into a
    buffer of its own and computed as a batch of its own (as a rank would on
    its GPU), writes exactly the whole batch's rows for its utterances."""
    pcm, off = W.ragged_batch(n_utt=40, seed=31, seed0=3100)
    whole = _run(plan, pcm, off)
    fo = O.frame_offsets(off)
    begin = lib.partition_utterances(fo, n_parts)
    pieces = []
    for r in range(n_parts):
        u0, u1 = int(begin[r]), int(begin[r + 1])
        sub = off[u0:u1 + 1]
        part = _run(plan, pcm[sub[0]:sub[-1]], sub - sub[0])
        assert part.shape[0] == fo[u1] - fo[u0]
        pieces.append(part)
    got = np.concatenate(pieces)
    assert np.array_equal(got.view(np.int32), whole.view(np.int32))
    longest = int(np.diff(fo).max())
    for r in range(n_parts):
        assert abs(int(fo[begin[r + 1]] - fo[begin[r]]) - fo[-1] / n_parts) <= longest


def test_accuracy_guard_on_pure_tones(lib, plan):
    """On-bin tones with no noise (the first page's demo signal without its
    noise term): the Hamming window's sidelobes leave most bands of every
    frame far below the frame's energy, so the float64 recomputation runs on
    every frame.  A 2 s clip is 7 tiles of 32 frames, one per tile group, so
    each group's queue of 16 deferred frames fills and its other flagged
    frames are recomputed inside their tile.  The offline result must meet
    the oracle on every row; streaming (which recomputes inside the tile,
    warps taking frames in turn) must equal it bit for bit; and the generic
    filterbank layout (recomputed inside the tile offline) must meet its
    oracle too."""
    x = W.page1_test_tones(2.0)
    g = _run(plan, x, [0, len(x)])
    L, M = O.log_mel(x, return_energy=True)
    check_against_oracle(g, L, M)
    st = lib.Stream(plan, 1)
    xs = torch.from_numpy(x).cuda()
    rows = [st.push(0, xs[i:i + 1280]).clone() for i in range(0, len(x), 1280)]
    got = torch.cat(rows, 0).cpu().numpy()
    assert got.shape == g.shape
    assert np.array_equal(got.view(np.int32), g.view(np.int32))
    p80 = lib.Plan(n_mels=80, fmin=20.0, fmax=7600.0)
    g80 = _run(p80, x, [0, len(x)])
    L80, M80 = O.log_mel(x, O.Params(n_mels=80, fmin=20.0, fmax=7600.0), return_energy=True)
    check_against_oracle(g80, L80, M80)


def test_accuracy_guard_after_the_queue_overflows(plan):
    """160 s of the same tones: 500 tiles, so some tile groups run two. A
    group's first tile overflows its queue of deferred frames; from then on
    every warp of the group recomputes its tiles' flagged frames in place."""
    x = W.page1_test_tones(160.0)
    g = _run(plan, x, [0, len(x)])
    L, M = O.log_mel(x, return_energy=True)
    assert g.shape[0] == 15998
    check_against_oracle(g, L, M)
