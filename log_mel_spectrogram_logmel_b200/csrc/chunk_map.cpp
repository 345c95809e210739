// Encoder-ready index maps over the log-mel rows (host only, no copies).
//
// Offline chunks: the preprocessor configuration of "从零理解 ASR：音频基础、
// Qwen3-ASR 架构，以及离线 vs 流式推理原理" (section 2.3) sets chunk_length =
// 30 s, i.e. 3000 frames per encoder input; "Qwen3-ASR详解transcribe.cpp中
// audio-LLM token注入架构原理" (section "4. Padding 浪费") has the encoder pad
// every input to 3000 frames and suggests length buckets against the waste.
// Streaming windows: section 5.2 of the first page processes chunk k, frames
// [500 k, 500 (k + 1)), with n_window = 50 frames of context on each side.
#include <cstdint>

#include "logmel.h"

extern "C" {

int64_t logmel_encoder_chunk_count(const int64_t* frame_offsets, int64_t n_utt, int64_t chunk_frames) {
  if (!frame_offsets || n_utt < 0 || chunk_frames < 1) return -1;
  int64_t count = 0;
  for (int64_t u = 0; u < n_utt; ++u) {
    const int64_t n = frame_offsets[u + 1] - frame_offsets[u];
    if (n < 0) return -1;
    count += (n + chunk_frames - 1) / chunk_frames;
  }
  return count;
}

logmel_status logmel_encoder_chunks(const int64_t* frame_offsets, int64_t n_utt, int64_t chunk_frames,
                                    int64_t quantum, logmel_chunk* chunks, int64_t capacity, int64_t* n_chunks) {
  if (!n_chunks) return LOGMEL_ERR_INVALID_ARG;
  *n_chunks = 0;
  if (quantum < 1) return LOGMEL_ERR_INVALID_ARG;
  const int64_t need = logmel_encoder_chunk_count(frame_offsets, n_utt, chunk_frames);
  if (need < 0) return LOGMEL_ERR_INVALID_ARG;
  *n_chunks = need;
  if (need > capacity || (need > 0 && !chunks)) return LOGMEL_ERR_INVALID_ARG;
  int64_t i = 0;
  for (int64_t u = 0; u < n_utt; ++u) {
    const int64_t n = frame_offsets[u + 1] - frame_offsets[u];
    for (int64_t start = 0; start < n; start += chunk_frames) {
      const int64_t frames = n - start < chunk_frames ? n - start : chunk_frames;
      const int64_t up = (frames + quantum - 1) / quantum * quantum;   // next multiple of the quantum
      chunks[i].utt = u;
      chunks[i].row = frame_offsets[u] + start;
      chunks[i].frames = frames;
      chunks[i].padded = up < chunk_frames ? up : chunk_frames;
      ++i;
    }
  }
  return LOGMEL_OK;
}

logmel_status logmel_stream_windows(int64_t n_frames, int finished, int64_t chunk_frames, int64_t context,
                                    logmel_window* windows, int64_t capacity, int64_t* n_windows) {
  if (!n_windows) return LOGMEL_ERR_INVALID_ARG;
  *n_windows = 0;
  if (n_frames < 0 || chunk_frames < 1 || context < 0) return LOGMEL_ERR_INVALID_ARG;
  // chunks whose core has started; without the end of the stream, only those
  // whose right context has arrived
  int64_t ready = (n_frames + chunk_frames - 1) / chunk_frames;
  if (!finished) {
    const int64_t full = n_frames - context >= 0 ? (n_frames - context) / chunk_frames : 0;
    if (full < ready) ready = full;
  }
  *n_windows = ready;
  if (ready > capacity || (ready > 0 && !windows)) return LOGMEL_ERR_INVALID_ARG;
  for (int64_t k = 0; k < ready; ++k) {
    const int64_t core_begin = k * chunk_frames;
    int64_t core_end = core_begin + chunk_frames;
    int64_t ctx_end = core_end + context;
    if (finished) {
      if (core_end > n_frames) core_end = n_frames;
      if (ctx_end > n_frames) ctx_end = n_frames;
    }
    windows[k].chunk = k;
    windows[k].core_begin = core_begin;
    windows[k].core_end = core_end;
    windows[k].ctx_begin = core_begin - context > 0 ? core_begin - context : 0;
    windows[k].ctx_end = ctx_end;
  }
  return LOGMEL_OK;
}

}  // extern "C"
