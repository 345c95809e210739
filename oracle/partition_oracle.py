"""Data-parallel partition of a log-mel batch over ranks: the plain definition.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline may use this module; the product path never does.

The front-end of "从零理解 ASR：音频基础、Qwen3-ASR 架构，以及离线 vs 流式推理原理"
(section 2.3) works frame by frame, every frame reading only its own 400
samples, so a batch of utterances (or a set of streams) is split over GPUs
with no exchange of data between them.  Reading taken here (the pages do not
say how to balance the split): each rank gets a contiguous run of whole
utterances, so that its output rows are one contiguous slice of the batch's
rows, and the cut before rank r is the utterance boundary whose frame prefix
sum is nearest to r / G of the batch's frames (the smaller index on a tie).
Streams are split into G contiguous runs of ids whose sizes differ by at
most one.
"""
from __future__ import annotations


def partition_utterances(frame_offsets, n_parts: int) -> list[int]:
    """utt_begin[0..n_parts]: rank r takes utterances utt_begin[r] ..
    utt_begin[r + 1] - 1.  frame_offsets is the batch's CSR frame prefix sum
    (n_utt + 1 entries); each inner cut is found by scanning every boundary."""
    fo = [int(v) for v in frame_offsets]
    if n_parts < 1 or len(fo) < 1:
        raise ValueError("need at least one part and one offset")
    if any(b < a for a, b in zip(fo[:-1], fo[1:])):
        raise ValueError("frame offsets must not decrease")
    n_utt, total = len(fo) - 1, fo[-1] - fo[0]
    cuts = [0]
    for r in range(1, n_parts):
        # distance of boundary u to the target r * total / n_parts, scaled by n_parts
        best = min(range(n_utt + 1), key=lambda u: (abs(n_parts * (fo[u] - fo[0]) - r * total), u))
        cuts.append(best)
    cuts.append(n_utt)
    return cuts


def partition_streams(n_streams: int, n_parts: int) -> list[int]:
    """stream_begin[0..n_parts]: rank r takes stream ids floor(r S / G) ..
    floor((r + 1) S / G) - 1."""
    if n_parts < 1 or n_streams < 0:
        raise ValueError("need at least one part and no negative stream count")
    return [r * n_streams // n_parts for r in range(n_parts + 1)]
