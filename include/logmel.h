/*
 * logmel.h -- C ABI of the B200 (sm_100a) batched log-mel spectrogram.
 *
 * The operation is the log-mel front-end that "从零理解 ASR：音频基础、
 * Qwen3-ASR 架构，以及离线 vs 流式推理原理" defines in section 2.3
 * ("Log-Mel Spectrogram 提取流水线", steps 1-5):
 *   16 kHz mono fp32 PCM -> frames of n_fft = 400 samples every hop = 160
 *   samples, no padding, floor((N - 400) / 160) + 1 frames (step 1)
 *   -> symmetric Hamming window 0.54 - 0.46 cos(2 pi n / 399) (step 2)
 *   -> real DFT to 201 bins, power |X|^2 (step 3)
 *   -> 128 triangular filters uniform on mel = 2595 log10(1 + f / 700)
 *      over fmin..fmax, linear in Hz, unnormalised (step 4)
 *   -> ln(max(mel_energy, 1e-10)) (step 5)
 * Output is fp32, frames-major [frames, n_mels] (the section's shape flow
 * [3000, 400] -> [3000, 201] -> [3000, 128]).
 *
 * Accuracy: the transform runs in fp32, whose rounding leaves each bin with
 * an error near 1e-7 of the frame's RMS bin amplitude.  A band whose energy
 * lies below about 3e-7 of the frame's windowed energy (a spectral null far
 * below the frame's level) is therefore recomputed in float64 by a direct DFT
 * of the frame, inside the same kernel, so every band with energy above 1e-8
 * stays within 2e-3 of the float64 definition in log units.
 *
 * Streaming follows the chunked input of section 6 of the same page and
 * the 80 / 120 / 160 ms audio clocks of the "Audio8-ASR-Infinite" page:
 * after each push the stream emits every frame that the audio received so
 * far completes, and carries the unconsumed samples (240..399 of them once
 * 400 samples have arrived) to the next push.  Streaming output equals the
 * offline output on the concatenated audio bit for bit.
 *
 * Conventions (all entry points):
 *   - Every pointer documented "device" must be memory of the plan's device;
 *     "host" pointers are ordinary host memory.  All work is enqueued on the
 *     caller's `stream` (a cudaStream_t, passed as void*; NULL = the legacy
 *     default stream); no entry point synchronises the device unless its
 *     comment says so.
 *   - The caller owns every input and output buffer.  A plan owns its
 *     constant tables and scratch; a logmel_stream owns its carry state.
 *   - A plan or stream object must not be used from two host threads at the
 *     same time.  Calls on one object must be ordered on the GPU (one CUDA
 *     stream, or explicit synchronisation between streams).
 *   - Errors are returned as logmel_status; nothing is truncated silently:
 *     sizes the kernels cannot index return LOGMEL_ERR_INPUT_TOO_LONG.
 *     On an error return nothing has been enqueued.
 */
#ifndef LOGMEL_H_
#define LOGMEL_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LOGMEL_OK = 0,
  LOGMEL_ERR_INVALID_ARG = 1,    /* null pointer, bad offsets, bad size      */
  LOGMEL_ERR_UNSUPPORTED = 2,    /* parameters outside what the kernels do   */
  LOGMEL_ERR_CUDA = 3,           /* a CUDA runtime call failed               */
  LOGMEL_ERR_OOM = 4,            /* device or pinned allocation failed       */
  LOGMEL_ERR_INPUT_TOO_LONG = 5, /* a count exceeds the kernels' index range */
  LOGMEL_ERR_DEVICE_STATUS = 6,  /* a kernel flagged an inconsistency        */
  LOGMEL_ERR_NOALLOC_LIMIT = 7   /* batch beyond logmel_compute_noalloc's fixed scratch */
} logmel_status;

typedef struct logmel_plan logmel_plan;
typedef struct logmel_stream logmel_stream;

/* Human-readable name of a status code (static string, never NULL). */
const char* logmel_status_string(logmel_status s);

/* The CUDA error behind the last LOGMEL_ERR_CUDA returned on this host
 * thread: error name, message and the failing call ("" if none).  The
 * string is thread-local and valid until the next failing call. */
const char* logmel_last_error(void);

/* Creates a plan on the current CUDA device: builds the Hamming window,
 * FFT twiddles and the mel filterbank in float64 on the host, rounds them
 * to fp32 and uploads them (section 2.3, steps 2-4; preprocessor config
 * n_mels 128, n_fft 400, hop 160).
 *   sr      sample rate in Hz (> 0); it places bin k at k * sr / n_fft Hz
 *   n_fft   must be 400          (else LOGMEL_ERR_UNSUPPORTED)
 *   hop     must be 160          (else LOGMEL_ERR_UNSUPPORTED)
 *   n_mels  1..201               (else LOGMEL_ERR_UNSUPPORTED)
 *   fmin, fmax  0 <= fmin < fmax <= sr / 2 (else LOGMEL_ERR_INVALID_ARG)
 * On success *out owns device memory until logmel_plan_destroy. */
logmel_status logmel_plan_create(int sr, int n_fft, int hop, int n_mels, float fmin, float fmax,
                                 logmel_plan** out);

/* Frees the plan (synchronises the plan's device first).  NULL is a no-op. */
void logmel_plan_destroy(logmel_plan* plan);

/* floor((n_samples - n_fft) / hop) + 1, or 0 if n_samples < n_fft
 * (section 2.3 step 1; no padding).  Returns -1 for a NULL plan. */
int64_t logmel_num_frames(const logmel_plan* plan, int64_t n_samples);

/* Frame offsets of a ragged batch: offsets (host, n_utt + 1 entries, CSR,
 * non-decreasing, offsets[0] may be non-zero) -> frame_offsets (host,
 * n_utt + 1 entries, frame_offsets[0] = 0, exclusive prefix sum of the
 * per-utterance frame counts).  Pure host function. */
logmel_status logmel_frame_offsets(const logmel_plan* plan, const int64_t* offsets, int64_t n_utt,
                                   int64_t* frame_offsets);

/* Offline ragged batch.  Utterance u is pcm[offsets[u] .. offsets[u+1]).
 *   pcm      device, fp32, at least offsets[n_utt] samples
 *   offsets  host, int64, n_utt + 1 entries, non-decreasing, offsets[0] >= 0
 *   out      device, fp32 [total_frames, n_mels] row-major, where
 *            total_frames = sum of logmel_num_frames over utterances; the
 *            rows of utterance u start at frame_offsets[u]
 * Utterances shorter than n_fft contribute no rows and no error.  The call
 * launches one kernel.  For n_utt <= 256 the per-utterance offsets travel in
 * the launch parameters; larger batches first copy them host->device on
 * `stream` (from a pinned ring owned by the plan).  It does not synchronise
 * unless the plan's scratch must grow (the first call with more 32-frame
 * tiles, or more than 256 utterances, than any call before it), which
 * synchronises the device.  The kernel writes the plan's device scratch (tile
 * descriptors, and the queue of frames whose bands it recomputes in float64),
 * so calls on one plan whose work could overlap on the GPU (two streams) must
 * be ordered, for example on one stream.  n_utt == 0 or total_frames == 0 is
 * a no-op. */
logmel_status logmel_compute(logmel_plan* plan, const float* pcm, const int64_t* offsets,
                             int64_t n_utt, float* out, void* stream);

/* Total output rows logmel_compute writes for these offsets (host). */
int64_t logmel_total_frames(const logmel_plan* plan, const int64_t* offsets, int64_t n_utt);

/* Streaming state for n_streams independent streams (device carry of up to
 * n_fft - 1 samples per stream; zero-initialised: every stream is empty).
 * The call synchronises the device once, so that the zeroed state is in
 * place before it returns. */
logmel_status logmel_stream_create(logmel_plan* plan, int n_streams, logmel_stream** out);
void logmel_stream_destroy(logmel_stream* st);

/* Frames the next push of `len` samples to stream `stream_id` will emit
 * (host bookkeeping only; -1 on a bad argument). */
int64_t logmel_stream_frames_for_push(const logmel_stream* st, int stream_id, int64_t len);

/* Pushes `len` samples (device, fp32) to one stream.  Emits n frames into
 * out (device, fp32 [out_capacity, n_mels]); *n_frames_out (host) receives
 * n, computed on the host, so no synchronisation is needed.  Returns
 * LOGMEL_ERR_INVALID_ARG if n > out_capacity (nothing enqueued). */
logmel_status logmel_stream_push(logmel_stream* st, int stream_id, const float* chunk, int64_t len,
                                 float* out, int64_t out_capacity, int64_t* n_frames_out,
                                 void* stream);

/* Pushes one chunk to every stream at once.
 *   chunks         device, fp32 [n_streams, chunk_stride], row s = stream s,
 *                  the first `len` samples of each row are pushed
 *   out            device, fp32 [n_streams, out_capacity, n_mels]; stream s
 *                  writes its n_frames_out[s] rows at out + s*out_capacity*n_mels
 *   n_frames_out   host, int64 [n_streams], filled before the call returns
 * All streams advance by `len` samples.  Returns LOGMEL_ERR_INVALID_ARG if
 * any stream would emit more than out_capacity frames. */
logmel_status logmel_stream_push_batch(logmel_stream* st, const float* chunks, int64_t chunk_stride,
                                       int64_t len, float* out, int64_t out_capacity,
                                       int64_t* n_frames_out, void* stream);

/* Pushes a chunk of its own length to every stream at once, in one launch
 * (chunked streaming input arriving as it comes: section 6 of the first
 * page; the 80 / 120 / 160 ms audio clocks of the "Audio8-ASR-Infinite" page
 * with streams whose pieces differ in size).
 *   chunks         device, fp32, the pushed samples of all streams packed:
 *                  stream s's chunk is chunks[chunk_offsets[s] ..
 *                  chunk_offsets[s + 1]) (may be empty: the stream is left
 *                  as it is)
 *   chunk_offsets  host, int64 [n_streams + 1], non-decreasing, >= 0
 *   out            device, fp32 [n_streams, out_capacity, n_mels]; stream s
 *                  writes its n_frames_out[s] rows at out + s*out_capacity*n_mels
 *   n_frames_out   host, int64 [n_streams], filled before the call returns
 * Every stream s advances by its own chunk_offsets[s + 1] - chunk_offsets[s]
 * samples; its output equals the offline log-mel of its concatenated audio
 * bit for bit, as for the other pushes.  The offsets are copied
 * host->device on `stream` through a pinned ring owned by the stream object
 * (allocated on the first ragged push; the host thread waits only when it
 * reuses a ring slot whose copy, four pushes earlier, is still pending).
 * Returns LOGMEL_ERR_INVALID_ARG if any stream would emit more than
 * out_capacity frames or the offsets are bad (nothing enqueued). */
logmel_status logmel_stream_push_batch_ragged(logmel_stream* st, const float* chunks,
                                              const int64_t* chunk_offsets, float* out,
                                              int64_t out_capacity, int64_t* n_frames_out, void* stream);

/* Largest per-stream frame count the next push_batch_ragged with these
 * chunk_offsets (host, int64 [n_streams + 1]) emits; -1 on a bad argument. */
int64_t logmel_stream_max_frames_ragged(const logmel_stream* st, const int64_t* chunk_offsets);

/* Largest per-stream frame count the next push_batch of `len` samples emits.
 * It depends on the carries' current lengths (it grows as they fill); a
 * carry never holds more than n_fft - 1 samples, so (len - 1) / hop + 1
 * (integer division, len >= 1) bounds the count in every state, which is
 * the size for an output buffer reused across pushes. */
int64_t logmel_stream_max_frames(const logmel_stream* st, int64_t len);

/* Checkpoint / resume of the carry state.  logmel_stream_state_bytes gives
 * the size of the opaque blob; get_state synchronises `stream` and copies
 * the state into host memory; set_state uploads a blob written by
 * get_state for the same n_streams (else LOGMEL_ERR_INVALID_ARG).  A
 * resumed stream produces output bit-identical to an uninterrupted one. */
int64_t logmel_stream_state_bytes(const logmel_stream* st);
logmel_status logmel_stream_get_state(logmel_stream* st, void* host_blob, int64_t bytes, void* stream);
logmel_status logmel_stream_set_state(logmel_stream* st, const void* host_blob, int64_t bytes,
                                      void* stream);

/* Empties one stream (or all streams if stream_id < 0), enqueued on `stream`. */
logmel_status logmel_stream_reset(logmel_stream* st, int stream_id, void* stream);

/* Offline ragged batch that allocates nothing.  (The paper has no
 * counterpart: this is a deployment variant of logmel_compute.)
 *
 * Who needs it: callers that cannot call cudaMalloc -- a process whose
 * device memory belongs to another allocator (a serving runtime or host
 * application that reserves the GPU's memory at start-up and hands out
 * buffers, so a raw cudaMalloc fails or escapes its accounting), and
 * real-time audio code for which cudaMalloc / cudaFree would block the
 * thread or synchronise the device.  Creating a plan allocates, so this
 * entry point takes none: it computes the default front-end (sr 16000,
 * n_fft 400, hop 160, 128 mels over 0-8000 Hz), the configuration
 * logmel_plan_create(16000, 400, 160, 128, 0, 8000) describes, with the same
 * kernel, and its output equals that plan's logmel_compute output.
 *
 * Arguments as logmel_compute, without the plan:
 *   pcm, offsets, n_utt, out   as logmel_compute (out holds sum over u of
 *                  floor((len_u - 400) / 160) + 1 rows of 128 floats, 0 rows
 *                  for len_u < 400)
 *   device_status  device, one int, or NULL: set to 0 on `stream` before the
 *                  kernel, which stores a nonzero code there if it flags an
 *                  inconsistency (NULL: a word inside the scratch, unread)
 * All of pcm, out and device_status must be memory of the current device.
 *
 * Scratch and limits: the FFT tables, the status word, the ragged metadata
 * and the tile descriptors live in one fixed array in device memory (about
 * 740 KB, held by every GPU that loads this library until the process
 * exits).  A call takes at most 4096 utterances and 32768 tiles, where
 * utterance u needs ceil(frames_u / 32) tiles (for example 4096 utterances
 * of up to 2.5 s, 64 of 30 s, or one of up to 2.9 h); beyond either limit it
 * returns LOGMEL_ERR_NOALLOC_LIMIT and enqueues nothing.
 *
 * Calls and set-up: the first call on each device does a one-time set-up
 * with that device current -- it looks up the scratch address, uploads the
 * tables with a synchronous copy and sets the kernel's shared-memory limit
 * -- so make that first call before any stream capture begins.  Every call
 * on a device shares the one scratch array, which keeps the last call's
 * contents: calls whose work overlaps on the GPU (two streams, or two host
 * threads without ordering) race on it and may return wrong output; order
 * them on one stream or with events.  Host-side, calls are serialised by a
 * lock.  Each call clears the status word and launches one kernel; batches
 * of more than 256 utterances first copy their metadata host->device from a
 * static host buffer with cudaMemcpyAsync.  That buffer is pageable host
 * memory, so such a call may block the calling thread until `stream` has
 * reached the copy (a copy from pageable memory returns once its source has
 * been consumed), and the next call rewrites the buffer.  Batches of up to
 * 256 utterances carry their metadata in the kernel launch and do not block.
 * Only those calls may be captured into a CUDA graph: a captured call of
 * more than 256 utterances would replay a copy of whatever the host buffer
 * holds at replay time.  No device or pinned memory is allocated or freed. */
logmel_status logmel_compute_noalloc(const float* pcm, const int64_t* offsets, int64_t n_utt,
                                     float* out, int* device_status, void* stream);

/* Output rows logmel_compute_noalloc writes for these offsets: the sum over
 * utterances of floor((len_u - 400) / 160) + 1 (0 for len_u < 400), the frame
 * count of section 2.3 step 1 for the default front-end.  Host only, needs
 * no plan and no device; -1 for NULL offsets, n_utt < 0 or decreasing
 * offsets. */
int64_t logmel_noalloc_total_frames(const int64_t* offsets, int64_t n_utt);

/* ---- Encoder-ready index maps over the log-mel rows (host only) ----------
 * The steps right after the log-mel front-end cut its rows into encoder
 * inputs.  These calls only compute row ranges: the encoder takes views of
 * the rows logmel_compute (or a stream's pushes) wrote; nothing is copied. */

/* One offline encoder chunk: rows [row, row + frames) of the output,
 * belonging to utterance utt, fed to the encoder padded to `padded` rows. */
typedef struct {
  int64_t utt;
  int64_t row;
  int64_t frames;
  int64_t padded;
} logmel_chunk;

/* Offline chunks: "从零理解 ASR：音频基础、Qwen3-ASR 架构，以及离线 vs 流式推理原理",
 * section 2.3 (preprocessor config chunk_length = 30 s = 3000 frames), and
 * "Qwen3-ASR详解transcribe.cpp中audio-LLM token注入架构原理", section
 * "4. Padding 浪费" (the encoder pads every input to 3000 frames; length
 * buckets reduce the waste).  Utterance u's rows frame_offsets[u] ..
 * frame_offsets[u + 1] (host, n_utt + 1 entries, as logmel_frame_offsets
 * returns them) are cut into consecutive chunks of at most chunk_frames rows
 * (3000); each is padded up to a multiple of quantum rows, at most
 * chunk_frames (quantum = chunk_frames: pad every chunk to 3000; smaller:
 * buckets).  Utterances without rows give no chunks.
 *   logmel_encoder_chunk_count: the number of chunks, or -1 on a bad
 *     argument (NULL offsets, n_utt < 0, chunk_frames < 1, decreasing offsets).
 *   logmel_encoder_chunks: writes them in utterance order into chunks (host,
 *     capacity entries).  *n_chunks (host) always receives the count; if it
 *     exceeds capacity, or an argument is bad (also quantum < 1), nothing is
 *     written and LOGMEL_ERR_INVALID_ARG is returned. */
int64_t logmel_encoder_chunk_count(const int64_t* frame_offsets, int64_t n_utt, int64_t chunk_frames);
logmel_status logmel_encoder_chunks(const int64_t* frame_offsets, int64_t n_utt, int64_t chunk_frames,
                                    int64_t quantum, logmel_chunk* chunks, int64_t capacity, int64_t* n_chunks);

/* One streaming encoder window: the encoder processes frames
 * [ctx_begin, ctx_end) of the stream and keeps the results of its core
 * frames [core_begin, core_end) (frame indices count the stream's frames
 * from its first push). */
typedef struct {
  int64_t chunk;
  int64_t core_begin;
  int64_t core_end;
  int64_t ctx_begin;
  int64_t ctx_end;
} logmel_window;

/* Streaming windows: the first page, section 5.2 ("流式模式的滑动窗口机制"):
 * chunk k covers frames [k * chunk_frames, (k + 1) * chunk_frames) (500) and
 * is processed with `context` frames (n_window = 50) on each side, clipped at
 * frame 0.  For a stream that has emitted n_frames frames, the windows are
 * those whose right context has arrived ((k + 1) * chunk_frames + context <=
 * n_frames); once the stream has finished (finished != 0), every chunk that
 * holds a frame, with its core and context clipped at n_frames.  Writes them
 * in order into windows (host, capacity entries); *n_windows (host) always
 * receives the count; if it exceeds capacity, or n_frames < 0,
 * chunk_frames < 1 or context < 0, nothing is written and
 * LOGMEL_ERR_INVALID_ARG is returned. */
logmel_status logmel_stream_windows(int64_t n_frames, int finished, int64_t chunk_frames, int64_t context,
                                    logmel_window* windows, int64_t capacity, int64_t* n_windows);

/* ---- Data-parallel split over ranks (host only) ----------------------------
 * Every frame reads only its own 400 samples (section 2.3 step 1), so the
 * utterances of one batch, or a set of streams, are split over GPUs with no
 * data exchanged between them: each rank runs logmel_compute (or its pushes)
 * on its own part, on its own device.
 *
 * logmel_partition_utterances: frame_offsets (host, n_utt + 1 entries, as
 * logmel_frame_offsets returns them, non-decreasing) -> utt_begin (host,
 * n_parts + 1 entries).  Rank r takes the contiguous utterances
 * utt_begin[r] .. utt_begin[r + 1] - 1, i.e. samples offsets[utt_begin[r]] ..
 * offsets[utt_begin[r + 1]] and output rows frame_offsets[utt_begin[r]] ..
 * frame_offsets[utt_begin[r + 1]] of the whole batch.  The cut before rank r
 * is the utterance boundary whose frame prefix sum is nearest to r / n_parts
 * of the batch's frames (the smaller index on a tie), so each rank's frame
 * count is within one utterance's frames of the mean.  Ranks may be empty.
 * LOGMEL_ERR_INVALID_ARG on NULL pointers, n_utt < 0, n_parts < 1 or
 * decreasing offsets; LOGMEL_ERR_INPUT_TOO_LONG if n_parts times the frame
 * count overflows.
 *
 * logmel_partition_streams: stream ids 0 .. n_streams - 1 -> stream_begin
 * (host, n_parts + 1 entries): rank r takes ids floor(r S / G) ..
 * floor((r + 1) S / G) - 1, runs whose sizes differ by at most one. */
logmel_status logmel_partition_utterances(const int64_t* frame_offsets, int64_t n_utt, int n_parts,
                                          int64_t* utt_begin);
logmel_status logmel_partition_streams(int64_t n_streams, int n_parts, int64_t* stream_begin);

/* Test hook for the bounded wait on a tile's span copies (not for normal
 * use; no page defines it).  Offline tiles staged by bulk copies wait on a
 * shared-memory barrier, polling at most poll_limit times (0: the default
 * 65536 polls, about 65 ms); a wait that runs out stores
 * LOGMEL_DEVICE_COPY_TIMEOUT (3) in the plan's device status word, waits once
 * more (again bounded) for the copies still in flight, and ends that tile
 * group's work, so the call returns and the context stays usable (the
 * group's remaining rows are not written).  extra_tx_bytes (a multiple of 16,
 * at most 1 MiB) is added to the bytes each tile's barrier expects: every
 * real copy is still issued and lands, but the barrier never completes, so
 * the wait runs out.  (0, 0) restores normal operation.  Host only. */
#define LOGMEL_DEVICE_COPY_TIMEOUT 3
logmel_status logmel_plan_set_wait_test(logmel_plan* plan, int extra_tx_bytes, int poll_limit);

/* Reads and clears the plan's device status word (synchronises `stream`).
 * *code = 0 when no kernel has flagged an inconsistency since the last read. */
logmel_status logmel_plan_device_status(logmel_plan* plan, int* code, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LOGMEL_H_ */
