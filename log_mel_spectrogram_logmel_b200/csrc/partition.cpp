// Data-parallel split of a log-mel batch over ranks (host only, no copies).
//
// Every frame of the front-end of "从零理解 ASR：音频基础、Qwen3-ASR 架构，以及
// 离线 vs 流式推理原理" (section 2.3) reads only its own 400 samples, so the
// utterances of a batch, or a set of streams, are split over GPUs with no
// data exchanged between them.  Each rank takes a contiguous run of whole
// utterances, so its rows are one contiguous slice of the batch's rows; the
// cut before rank r is the utterance boundary whose frame prefix sum lies
// nearest to r / G of the batch's frames (the smaller index on a tie).  A
// rank's frame count then differs from the mean by at most the frame count
// of the batch's longest utterance.
#include <cstdint>

#include "logmel.h"

extern "C" {

logmel_status logmel_partition_utterances(const int64_t* frame_offsets, int64_t n_utt, int n_parts,
                                          int64_t* utt_begin) {
  if (!frame_offsets || !utt_begin || n_utt < 0 || n_parts < 1) return LOGMEL_ERR_INVALID_ARG;
  for (int64_t u = 0; u < n_utt; ++u)
    if (frame_offsets[u + 1] < frame_offsets[u]) return LOGMEL_ERR_INVALID_ARG;
  const int64_t f0 = frame_offsets[0];
  const int64_t total = frame_offsets[n_utt] - f0;
  if (total > (INT64_MAX / 4) / n_parts) return LOGMEL_ERR_INPUT_TOO_LONG;
  const int64_t G = n_parts;
  utt_begin[0] = 0;
  for (int64_t r = 1; r < G; ++r) {
    // distances are scaled by G: boundary u sits at G (fo[u] - f0), the
    // target at r * total
    const int64_t target = r * total;
    int64_t a = 0, b = n_utt;   // first boundary at or past the target
    while (a < b) {
      const int64_t m = a + (b - a) / 2;
      if (G * (frame_offsets[m] - f0) >= target) b = m;
      else a = m + 1;
    }
    int64_t cut = a;
    if (a > 0) {
      int64_t v = a - 1;   // the last boundary below the target, at its first index
      while (v > 0 && frame_offsets[v - 1] == frame_offsets[v]) --v;
      const int64_t below = target - G * (frame_offsets[v] - f0);
      const int64_t above = G * (frame_offsets[a] - f0) - target;
      if (below <= above) cut = v;
    }
    utt_begin[r] = cut;
  }
  utt_begin[G] = n_utt;
  return LOGMEL_OK;
}

logmel_status logmel_partition_streams(int64_t n_streams, int n_parts, int64_t* stream_begin) {
  if (!stream_begin || n_streams < 0 || n_parts < 1) return LOGMEL_ERR_INVALID_ARG;
  if (n_streams > INT64_MAX / n_parts) return LOGMEL_ERR_INPUT_TOO_LONG;
  for (int64_t r = 0; r <= n_parts; ++r) stream_begin[r] = r * n_streams / n_parts;
  return LOGMEL_OK;
}

}  // extern "C"
