"""Encoder-ready index maps over log-mel rows: the plain definitions.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline may use this module; the product path never does.

Two maps, both pure integer bookkeeping over the rows the log-mel pipeline
writes (no data is copied; a consumer takes views of the rows):

* Offline chunks.  "从零理解 ASR：音频基础、Qwen3-ASR 架构，以及离线 vs 流式推理原理",
  section 2.3 (the preprocessor configuration): chunk_length = 30 s, i.e.
  3000 frames per encoder input.  "Qwen3-ASR详解transcribe.cpp中audio-LLM
  token注入架构原理" (section "4. Padding 浪费"): the audio encoder pads every
  input to 3000 frames, and bucketing by length reduces the padded work.
  Reading: each utterance's rows are cut into consecutive chunks of at most
  `chunk_frames` rows; a chunk is padded up to the next multiple of
  `quantum` rows, capped at `chunk_frames` (quantum = chunk_frames pads
  every chunk to 3000, the page's behaviour; a smaller quantum gives length
  buckets).  Utterances with no rows give no chunks.

* Streaming windows.  First page, section 5.2 ("流式模式的滑动窗口机制"):
  chunk k covers frames [500 k, 500 (k + 1)) and is processed with
  n_window = 50 frames of context on each side, clipped at the stream's
  start (chunk 1: [0, 500) with context [0, 550); chunk 2: [500, 1000) with
  context [450, 1050)).  Reading: a chunk is ready once its right context
  has arrived, i.e. (k + 1) chunk + context <= frames so far; when the
  stream has finished, every remaining chunk is ready, its core and its
  context clipped at the stream's last frame.
"""
from __future__ import annotations

import numpy as np


def encoder_chunks(frame_offsets, chunk_frames: int = 3000, quantum: int = 3000) -> np.ndarray:
    """Rows (utt, row, frames, padded): utterance u's rows frame_offsets[u]
    .. frame_offsets[u + 1] cut into chunks of at most chunk_frames rows,
    each padded to a multiple of quantum rows (at most chunk_frames)."""
    if chunk_frames < 1 or quantum < 1:
        raise ValueError("chunk_frames and quantum must be positive")
    fo = [int(v) for v in frame_offsets]
    if any(b < a for a, b in zip(fo[:-1], fo[1:])):
        raise ValueError("frame offsets must not decrease")
    rows = []
    for u in range(len(fo) - 1):
        n = fo[u + 1] - fo[u]
        start = 0
        while start < n:
            frames = min(chunk_frames, n - start)
            padded = min(chunk_frames, -(-frames // quantum) * quantum)
            rows.append((u, fo[u] + start, frames, padded))
            start += chunk_frames
    return np.array(rows, dtype=np.int64).reshape(-1, 4)


def stream_windows(n_frames: int, finished: bool, chunk_frames: int = 500, context: int = 50) -> np.ndarray:
    """Rows (k, core_begin, core_end, ctx_begin, ctx_end) of the chunks of a
    stream that has emitted n_frames frames and whose right context has
    arrived (all remaining chunks once the stream has finished)."""
    if chunk_frames < 1 or context < 0 or n_frames < 0:
        raise ValueError("chunk_frames must be positive, context and n_frames non-negative")
    rows = []
    k = 0
    while k * chunk_frames < n_frames:
        core_begin = k * chunk_frames
        core_end = (k + 1) * chunk_frames
        if not finished and core_end + context > n_frames:
            break
        ctx_begin = max(0, core_begin - context)
        ctx_end = core_end + context
        if finished:
            core_end = min(core_end, n_frames)
            ctx_end = min(ctx_end, n_frames)
        rows.append((k, core_begin, core_end, ctx_begin, ctx_end))
        k += 1
    return np.array(rows, dtype=np.int64).reshape(-1, 5)
