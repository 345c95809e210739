// C ABI of the batched log-mel spectrogram (declared in include/logmel.h).
//
// Host side: plan creation (window, FFT twiddles and the mel filterbank of
// "从零理解 ASR：音频基础、Qwen3-ASR 架构，以及离线 vs 流式推理原理" section 2.3,
// built in float64 and rounded to fp32), the ragged-batch index map (frame
// and tile prefix sums), the streaming carry state and its checkpoint blob.
// Device side: logmel_kernel.cuh.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "logmel.h"
#include "logmel_kernel.cuh"

using namespace logmel;

namespace {

constexpr int RING = 4;
constexpr uint32_t STATE_MAGIC = 0x314d4c53u;   // "SLM1"

struct PinnedSlot {
  unsigned char* host = nullptr;
  cudaEvent_t done = nullptr;
  bool used = false;
};

struct MetaView {
  int64_t* sample_off;
  int64_t* frame_off;
  int* tile_off;
};

size_t meta_bytes(int64_t n_utt) {
  const size_t n = (size_t)n_utt + 1;
  size_t b = 16 * n;                 // two int64 arrays
  b += (4 * n + 15) & ~size_t(15);   // int32 tile offsets
  return b;
}

MetaView meta_view(unsigned char* base, int64_t n_utt) {
  const size_t n = (size_t)n_utt + 1;
  MetaView v;
  v.sample_off = reinterpret_cast<int64_t*>(base);
  v.frame_off = reinterpret_cast<int64_t*>(base + 8 * n);
  v.tile_off = reinterpret_cast<int*>(base + 16 * n);
  return v;
}

// cos and sin of 2 pi num / den, exact at multiples of pi / 2.
void cos_sin_2pi(long num, long den, double* c, double* s) {
  num %= den;
  if (num < 0) num += den;
  if (4 * num % den == 0) {
    const int q = (int)(4 * num / den);
    const double cs[4] = {1, 0, -1, 0}, sn[4] = {0, 1, 0, -1};
    *c = cs[q];
    *s = sn[q];
    return;
  }
  const double a = 2.0 * M_PI * (double)num / (double)den;
  *c = std::cos(a);
  *s = std::sin(a);
}

double hz_to_mel(double f) { return 2595.0 * std::log10(1.0 + f / 700.0); }
double mel_to_hz(double m) { return 700.0 * (std::pow(10.0, m / 2595.0) - 1.0); }

int64_t frames_of(int64_t n) { return n < NFFT ? 0 : (n - NFFT) / HOP + 1; }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    cudaGetLastError();
  }
  return fn;
}

// Offline spans land as their even and their odd 160-sample hop blocks in
// two regions, one box each: the tensor views below take every other row of
// the buffer, starting at row q (0 or 1), so a tile's hop blocks b, b + 2, ...
// are consecutive z-rows of one view.
constexpr int EO_BOX_ROWS = OFFLINE_SPAN_BLOCKS / 2;   // 17 hop blocks per region

// The rows 2 z + q of the PCM as a 3-D tensor [z][40][w] whose element
// (x, y, z) is pcm[160 q + 320 z + 4 y + x]: rows of w samples start at every
// 16-byte boundary (for w = 164 the strides overlap on purpose), so one
// 164 x 1 x 17 box lands the even or the odd hop blocks of any tile's span,
// from the boundary at or before it, in their slots.  Rows are counted so
// that every row of every start class lies inside the first `total` samples.
// Returns the rows, or 0 when no map can be made.
int encode_pcm_map(CUtensorMap* m, const float* pcm, int64_t total, int q, int w = BLK) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  const int64_t last = total - (int64_t)HOP * q - 4 * (HOP / 4 - 1) - w;   // start of the last full row, z = 0 based
  const int64_t rows = last >= 0 ? last / (2 * HOP) + 1 : 0;
  if (!enc || (reinterpret_cast<uintptr_t>(pcm) & 15) || rows < 1 || rows >= INT32_MAX) return 0;
  cuuint64_t dims[3] = {(cuuint64_t)w, (cuuint64_t)(HOP / 4), (cuuint64_t)rows};
  cuuint64_t strides[2] = {4 * sizeof(float), (cuuint64_t)(2 * HOP) * sizeof(float)};
  cuuint32_t box[3] = {(cuuint32_t)BLK, 1, (cuuint32_t)EO_BOX_ROWS};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(pcm + (int64_t)HOP * q), dims, strides, box,
             estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
             ? (int)rows
             : 0;
}

// The 160-sample rows 2 z + q of the PCM as a 2-D tensor [z][160] for the
// copies of spans that start on a row; the box is 164 x 17 and its columns
// 160..163 lie outside the tensor (zeros).  Returns the rows, or 0.
int encode_pcm_rows(CUtensorMap* m, const float* pcm, int64_t total, int q) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  const int64_t all = total / HOP;                  // whole 160-sample rows of the buffer
  const int64_t rows = all > q ? (all - q + 1) / 2 : 0;
  if (!enc || (reinterpret_cast<uintptr_t>(pcm) & 15) || rows < 1 || rows >= INT32_MAX) return 0;
  cuuint64_t dims[2] = {(cuuint64_t)HOP, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(2 * HOP) * sizeof(float)};
  cuuint32_t box[2] = {(cuuint32_t)BLK, (cuuint32_t)EO_BOX_ROWS};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(pcm + (int64_t)HOP * q), dims, strides, box,
             estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
             ? (int)rows
             : 0;
}

// The output rows as a 2-D tensor [rows][n_mels] for one-box stores of full
// tiles: the box is orow_floats(n_mels) x 32, matching the staged rows in
// shared memory; its pad columns lie outside the tensor and are not written.
// Returns the tensor's rows, or 0 when no map can be made (unaligned base,
// row size not a multiple of 16 bytes, no encoder).
int encode_out_map(CUtensorMap* m, float* out, int64_t rows, int n_mels) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc || (reinterpret_cast<uintptr_t>(out) & 15) || rows < 1 || rows >= INT32_MAX || (n_mels * 4) % 16)
    return 0;
  cuuint64_t dims[2] = {(cuuint64_t)n_mels, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)n_mels * sizeof(float)};
  cuuint32_t box[2] = {(cuuint32_t)orow_floats(n_mels), (cuuint32_t)TILE};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, out, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
             ? (int)rows
             : 0;
}

// True when some utterance with frames starts at an odd float offset from a
// 16-byte boundary (every tile of an utterance shares its start's parity).
bool has_odd_spans(const float* pcm, const int64_t* off, int64_t n_utt) {
  const uint64_t base = reinterpret_cast<uintptr_t>(pcm) >> 2;
  for (int64_t u = 0; u < n_utt; ++u)
    if (frames_of(off[u + 1] - off[u]) > 0 && ((base + (uint64_t)off[u]) & 1)) return true;
  return false;
}

}  // namespace

struct LaunchCfg {
  int groups = 0;        // tile groups (of 160 threads) per CTA
  int group_bytes = 0;   // shared memory per tile group
  int ybuf_bytes = 0;    // pass buffer per tile group
  int span_blocks = 0;
  size_t smem = 0;       // dynamic shared memory per CTA
  int max_ctas = 0;      // resident CTAs on the device
};

struct logmel_plan {
  int sr = 0, n_fft = 0, hop = 0, n_mels = 0;
  float fmin = 0.f, fmax = 0.f;
  int device = 0;
  LaunchCfg off{}, str{};    // offline and streaming launch shapes
  Tables* d_tables = nullptr;
  double* d_fix = nullptr;        // float64 window [400] and (cos, sin) [400] of the accuracy guard
  FixItem* d_fixq = nullptr;      // deferred accuracy-guard frames, FIXQ_CAP per offline tile group
  int fixq_groups = 0;            // tile groups d_fixq holds (0: none; recompute inside the tile)
  int* d_status = nullptr;
  unsigned char* d_meta = nullptr;
  size_t meta_cap = 0;
  TileDesc* d_tiles = nullptr;    // offline tile descriptors (kernel-written scratch)
  size_t tiles_cap = 0;
  PinnedSlot ring[RING];
  size_t ring_cap = 0;
  int ring_next = 0;
  Args mel{};               // filterbank fields copied into every launch
  bool default_mel = false; // structure equals the compiled default layout
  // tensor maps of the last offline PCM buffer (re-encoded when it changes)
  CUtensorMap tmap[2]{}, tmap_s[2]{};
  const float* tmap_pcm = nullptr;
  int64_t tmap_len = -1;
  int tmap_rows[2]{}, tmap_s_rows[2]{};
  // bounded span waits (test hook; 0, 0 in normal operation)
  int wait_polls = 0, tx_extra = 0;
  // tensor map of the last offline output buffer (full-tile row stores)
  CUtensorMap otmap{};
  const float* otmap_out = nullptr;
  int64_t otmap_len = -1;
  int otmap_rows = 0;
};

struct logmel_stream {
  logmel_plan* plan = nullptr;
  int n_streams = 0;
  float* d_carry = nullptr;
  int* d_carry_len = nullptr;
  std::vector<int64_t> total;    // samples received per stream
  std::vector<int> carry_len;    // host mirror of d_carry_len
  // ragged pushes: per-stream chunk offsets, staged in a pinned ring and
  // copied to the device ahead of the kernel (allocated on first use)
  int64_t* d_push_off = nullptr;
  PinnedSlot off_ring[RING];
  int off_next = 0;
};

// ---------------------------------------------------------------------------
// small kernels
// ---------------------------------------------------------------------------
namespace {

// New carry after a push whose frames were computed with the carry left in
// place (pushes emitting more than one tile per stream): one CTA per stream.
// push_off (ragged pushes): stream sl's chunk is chunks[push_off[sl] ..
// push_off[sl + 1]); else len samples at chunks + sl * chunk_stride.
__global__ void carry_update_kernel(float* carry, int* carry_len, const float* chunks,
                                    int64_t chunk_stride, int64_t len, int stream_base,
                                    const int64_t* push_off) {
  __shared__ float buf[CARRY_CAP];
  const int sl = blockIdx.x;
  const int s = stream_base + sl;
  float* cs = carry + (int64_t)s * CARRY_CAP;
  const float* ch = chunks + (int64_t)sl * chunk_stride;
  if (push_off != nullptr) {
    ch = chunks + push_off[sl];
    len = push_off[sl + 1] - push_off[sl];
  }
  const int c = carry_len[s];            // read by every thread before the barrier
  const int64_t B = c + len;
  const int64_t nf = B >= NFFT ? (B - NFFT) / HOP + 1 : 0;
  const int L = (int)(B - nf * HOP);     // < 400
  const int64_t from = nf * HOP;
  for (int i = threadIdx.x; i < L; i += blockDim.x) {
    const int64_t q = from + i;
    buf[i] = q < c ? cs[q] : ch[q - c];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < L; i += blockDim.x) cs[i] = buf[i];
  if (threadIdx.x == 0) carry_len[s] = L;
}

}  // namespace

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
// Text of the last failed CUDA call on this host thread (logmel_last_error).
static thread_local char g_last_error[256] = "";

static logmel_status cuda_fail(cudaError_t e, const char* call, int line) {
  snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s, logmel.cu:%d)", cudaGetErrorName(e),
           cudaGetErrorString(e), call, line);
  return LOGMEL_ERR_CUDA;
}

#define CK(call)                                           \
  do {                                                     \
    cudaError_t e_ = (call);                               \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call, __LINE__); \
  } while (0)

extern "C" {

const char* logmel_last_error(void) { return g_last_error; }

const char* logmel_status_string(logmel_status s) {
  switch (s) {
    case LOGMEL_OK: return "ok";
    case LOGMEL_ERR_INVALID_ARG: return "invalid argument";
    case LOGMEL_ERR_UNSUPPORTED: return "unsupported parameters";
    case LOGMEL_ERR_CUDA: return "CUDA runtime error";
    case LOGMEL_ERR_OOM: return "out of memory";
    case LOGMEL_ERR_INPUT_TOO_LONG: return "input too long for the kernels' index range";
    case LOGMEL_ERR_DEVICE_STATUS: return "a kernel flagged an inconsistency";
    case LOGMEL_ERR_NOALLOC_LIMIT:
      return "batch larger than the fixed scratch of logmel_compute_noalloc "
             "(at most 4096 utterances and 32768 tiles of 32 frames)";
  }
  return "unknown status";
}

// Float64 tables of the accuracy guard's recomputation: the window w[n]
// (n < 400), then (cos, sin)(2 pi j / 400) (j < 400).
constexpr int FIX_DOUBLES = NFFT + 2 * NFFT;
static void build_fix_tables(double* t) {
  for (int n = 0; n < NFFT; ++n) t[n] = 0.54 - 0.46 * std::cos(2.0 * M_PI * n / (NFFT - 1));
  for (int j = 0; j < NFFT; ++j) cos_sin_2pi(j, NFFT, &t[NFFT + 2 * j], &t[NFFT + 2 * j + 1]);
}

static logmel_status build_tables(Tables* t) {
  std::memset(t, 0, sizeof(Tables));
  // e^{-2 pi i k / 400} = c - i s, k = 0..399, as (c, c, s, s): the pass-A
  // twiddle e^{-2 pi i m2 k1 / 200} is entry 2 m2 k1; the real split uses
  // u_k = -i e^{-2 pi i k / 400}
  for (int k = 0; k < NFFT; ++k) {
    double c, s;
    cos_sin_2pi(k, NFFT, &c, &s);
    t->w400[k] = make_float4((float)c, (float)c, (float)s, (float)s);
  }
  // window pairs for pass A: sample n = 20 m1 + 2 m2 and n + 1
  for (int m2 = 0; m2 < N2; ++m2)
    for (int m1 = 0; m1 < N1; ++m1) {
      const int n = 2 * (N2 * m1 + m2);
      const double w0 = 0.54 - 0.46 * std::cos(2.0 * M_PI * n / (NFFT - 1));
      const double w1 = 0.54 - 0.46 * std::cos(2.0 * M_PI * (n + 1) / (NFFT - 1));
      t->win[m2][m1] = make_float2((float)w0, (float)w1);
    }
  return LOGMEL_OK;
}

}  // extern "C"

// Triangular filters, linear in Hz between mel-spaced edges, unnormalised
// (section 2.3 step 4), stored as contiguous nonzero runs per band; weights
// carry the factor 1/4 of the real split (which yields |2 X|^2).  Also the
// split of the bands over the mel warps (cost per band = nonzeros + 3, bands
// taken four at a time).
static logmel_status build_mel(logmel_plan* p) {
  Args& a = p->mel;
  const int nm = p->n_mels;
  std::vector<double> edge(nm + 2);
  const double m_lo = hz_to_mel(p->fmin), m_hi = hz_to_mel(p->fmax);
  for (int j = 0; j < nm + 2; ++j) edge[j] = mel_to_hz(m_lo + (m_hi - m_lo) * j / (nm + 1));
  edge[0] = p->fmin;          // the end edges are fmin and fmax exactly
  edge[nm + 1] = p->fmax;
  int woff = 0;
  std::vector<int> cost(nm);
  for (int m = 0; m < nm; ++m) {
    int lo = -1, cnt = 0;
    for (int k = 0; k < NBINS; ++k) {
      const double f = (double)k * p->sr / NFFT;
      const double rise = (f - edge[m]) / (edge[m + 1] - edge[m]);
      const double fall = (edge[m + 2] - f) / (edge[m + 2] - edge[m + 1]);
      const double h = std::max(0.0, std::min(rise, fall));
      if (h > 0.0) {
        if (k == 0 || k == NBINS - 1) return LOGMEL_ERR_UNSUPPORTED;   // edge bins never weigh
        if (lo < 0) lo = k;
        if (k != lo + cnt) return LOGMEL_ERR_UNSUPPORTED;              // not contiguous
        if (woff + cnt >= MAX_WEIGHTS) return LOGMEL_ERR_UNSUPPORTED;
        a.mel_w[woff + cnt] = (float)h * 0.25f;
        ++cnt;
      }
    }
    a.mel_lo[m] = (short)(lo < 0 ? 1 : lo);
    a.mel_cnt[m] = (short)cnt;
    a.mel_woff[m] = (short)woff;
    woff += cnt;
    cost[m] = cnt + 3;
  }
  long total = 0;
  for (int m = 0; m < nm; ++m) total += cost[m];
  a.warp_band[0] = 0;
  long run = 0;
  int m = 0;
  for (int w = 1; w < MEL_WARPS; ++w) {   // four bands at a time
    const long target = total * w / MEL_WARPS;
    while (m < nm) {
      long c4 = 0;
      for (int i = m; i < std::min(m + 4, nm); ++i) c4 += cost[i];
      if (run + c4 / 2 >= target) break;
      run += c4;
      m += 4;
    }
    a.warp_band[w] = (short)std::min(m, nm);
  }
  a.warp_band[MEL_WARPS] = (short)nm;
  // the unrolled path applies when the structure equals the compiled one
  bool same = nm == mel_default::N_MELS && woff == mel_default::NNZ;
  for (int i = 0; same && i < nm; ++i)
    same = (mel_default::CNT[i] == a.mel_cnt[i]) && (mel_default::WOFF[i] == a.mel_woff[i]) &&
           (mel_default::CNT[i] == 0 || mel_default::LO[i] == a.mel_lo[i]);
  for (int w = 0; same && w <= MEL_WARPS; ++w) same = mel_default::WARP_BAND[w] == a.warp_band[w];
  for (int i = 0; same && i < mel_default::NNZ; ++i)   // compiled weights, bit for bit
    same = std::memcmp(&mel_default::W[i], &a.mel_w[i], sizeof(float)) == 0;
  p->default_mel = same;
  return LOGMEL_OK;
}

static void shape_launch(LaunchCfg& c, int span_blocks, int n_mels, int max_smem) {
  c.span_blocks = span_blocks;
  c.ybuf_bytes = ybuf_bytes_for(n_mels);
  c.group_bytes = group_bytes_for(span_blocks, n_mels);
  c.groups = MAX_TILE_GROUPS;
  while (c.groups > 1 && TAB_BYTES + (size_t)c.groups * c.group_bytes + FIXN_BYTES > (size_t)max_smem) --c.groups;
  c.smem = TAB_BYTES + (size_t)c.groups * c.group_bytes + FIXN_BYTES;
}

template <bool kDefault>
static logmel_status setup_kernel(logmel_plan* p, int sms) {
  if (cudaFuncSetAttribute(logmel_fused_kernel<kDefault, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)p->off.smem) != cudaSuccess ||
      cudaFuncSetAttribute(logmel_fused_kernel<kDefault, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)p->off.smem) != cudaSuccess ||
      cudaFuncSetAttribute(logmel_fused_kernel<kDefault, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)p->str.smem) != cudaSuccess)
    return LOGMEL_ERR_CUDA;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, logmel_fused_kernel<kDefault, false, false>,
                                                    p->off.groups * GROUP_THREADS, p->off.smem) != cudaSuccess ||
      occ < 1)
    return LOGMEL_ERR_CUDA;
  p->off.max_ctas = sms * occ;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, logmel_fused_kernel<kDefault, false, true>,
                                                    p->str.groups * GROUP_THREADS, p->str.smem) != cudaSuccess ||
      occ < 1)
    return LOGMEL_ERR_CUDA;
  p->str.max_ctas = sms * occ;
  return LOGMEL_OK;
}

// odd: some utterance of this offline batch starts at an odd float offset
// from a 16-byte boundary (launch the kernel that can read such spans).
static cudaError_t launch(const logmel_plan* p, Args& a, int64_t tiles, cudaStream_t s, bool odd = false) {
  const LaunchCfg& c = a.mode == 0 ? p->off : p->str;
  {
    const cudaError_t pending = cudaGetLastError();
    if (pending != cudaSuccess) {
      cuda_fail(pending, "error pending before the launch", __LINE__);
      return pending;
    }
  }
  a.tables = p->d_tables;
  a.fix_win = p->d_fix;
  a.fix_cs = reinterpret_cast<const double2*>(p->d_fix + NFFT);
  a.wait_polls = p->wait_polls;
  a.tx_extra = p->tx_extra;
  a.span_blocks = c.span_blocks;
  a.eo_off = eo_off_for(c.span_blocks);
  a.group_bytes = c.group_bytes;
  a.ybuf_bytes = c.ybuf_bytes;
  a.bulk_store = p->default_mel && (reinterpret_cast<uintptr_t>(a.out) & 15) == 0;
  std::memcpy(a.mel_w, p->mel.mel_w, sizeof a.mel_w);
  std::memcpy(a.mel_lo, p->mel.mel_lo, sizeof a.mel_lo);
  std::memcpy(a.mel_cnt, p->mel.mel_cnt, sizeof a.mel_cnt);
  std::memcpy(a.mel_woff, p->mel.mel_woff, sizeof a.mel_woff);
  std::memcpy(a.warp_band, p->mel.warp_band, sizeof a.warp_band);
  // one CTA per tile up to the resident limit: a batch of fewer tiles than
  // the device has SMs runs one tile group per SM (the others idle)
  const int grid = (int)std::min<int64_t>(tiles, c.max_ctas);
  const int block = c.groups * GROUP_THREADS;
  // offline: each tile group queues its flagged frames (when the queue
  // covers every group of the grid)
  const bool fixq = a.mode == 0 && p->d_fixq != nullptr && (int64_t)grid * c.groups <= p->fixq_groups;
  a.fixq = fixq ? p->d_fixq : nullptr;
  a.fixq_cap = fixq ? FIXQ_CAP : 0;
  if (a.mode == 1) {
    if (p->default_mel) logmel_fused_kernel<true, false, true><<<grid, block, c.smem, s>>>(a);
    else logmel_fused_kernel<false, false, true><<<grid, block, c.smem, s>>>(a);
  } else if (p->default_mel) {
    if (odd) logmel_fused_kernel<true, true, false><<<grid, block, c.smem, s>>>(a);
    else logmel_fused_kernel<true, false, false><<<grid, block, c.smem, s>>>(a);
  } else {
    if (odd) logmel_fused_kernel<false, true, false><<<grid, block, c.smem, s>>>(a);
    else logmel_fused_kernel<false, false, false><<<grid, block, c.smem, s>>>(a);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    char what[96];
    snprintf(what, sizeof what, "launch grid %d block %d smem %zu tiles %lld", grid, block, c.smem,
             (long long)tiles);
    cuda_fail(e, what, __LINE__);
  }
  return e;
}

extern "C" {

logmel_status logmel_plan_create(int sr, int n_fft, int hop, int n_mels, float fmin, float fmax,
                                 logmel_plan** out) {
  if (!out) return LOGMEL_ERR_INVALID_ARG;
  *out = nullptr;
  if (sr <= 0 || !(fmin >= 0.f) || !(fmax > fmin) || (double)fmax > sr / 2.0)
    return LOGMEL_ERR_INVALID_ARG;
  if (n_fft != NFFT || hop != HOP || n_mels < 1 || n_mels > MAX_MELS) return LOGMEL_ERR_UNSUPPORTED;
  logmel_plan* p = new (std::nothrow) logmel_plan();
  if (!p) return LOGMEL_ERR_OOM;
  p->sr = sr;
  p->n_fft = n_fft;
  p->hop = hop;
  p->n_mels = n_mels;
  p->fmin = fmin;
  p->fmax = fmax;
  Tables* t = new (std::nothrow) Tables();
  if (!t) {
    delete p;
    return LOGMEL_ERR_OOM;
  }
  logmel_status st = build_tables(t);
  if (st == LOGMEL_OK) st = build_mel(p);
  if (st != LOGMEL_OK) {
    delete t;
    delete p;
    return st;
  }
  auto fail = [&](logmel_status s) {
    delete t;
    logmel_plan_destroy(p);
    return s;
  };
  if (cudaGetDevice(&p->device) != cudaSuccess) return fail(LOGMEL_ERR_CUDA);
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess)
    return fail(LOGMEL_ERR_CUDA);
  int max_smem = 0;
  if (cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, p->device) != cudaSuccess)
    return fail(LOGMEL_ERR_CUDA);
  shape_launch(p->off, OFFLINE_SPAN_BLOCKS, p->n_mels, max_smem);
  shape_launch(p->str, STREAM_SPAN_BLOCKS, p->n_mels, max_smem);
  st = p->default_mel ? setup_kernel<true>(p, sms) : setup_kernel<false>(p, sms);
  if (st != LOGMEL_OK) return fail(st);
  if (cudaMalloc(&p->d_tables, sizeof(Tables)) != cudaSuccess) return fail(LOGMEL_ERR_OOM);
  if (cudaMalloc(&p->d_fix, sizeof(double) * FIX_DOUBLES) != cudaSuccess) return fail(LOGMEL_ERR_OOM);
  if (cudaMalloc(&p->d_status, sizeof(int)) != cudaSuccess) return fail(LOGMEL_ERR_OOM);
  p->fixq_groups = p->off.max_ctas * p->off.groups;
  if (cudaMalloc(&p->d_fixq, sizeof(FixItem) * FIXQ_CAP * (size_t)p->fixq_groups) != cudaSuccess)
    return fail(LOGMEL_ERR_OOM);
  if (cudaMemcpy(p->d_tables, t, sizeof(Tables), cudaMemcpyHostToDevice) != cudaSuccess)
    return fail(LOGMEL_ERR_CUDA);
  {
    std::vector<double> fix(FIX_DOUBLES);
    build_fix_tables(fix.data());
    if (cudaMemcpy(p->d_fix, fix.data(), sizeof(double) * FIX_DOUBLES, cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(LOGMEL_ERR_CUDA);
  }
  if (cudaMemset(p->d_status, 0, sizeof(int)) != cudaSuccess) return fail(LOGMEL_ERR_CUDA);
  for (int i = 0; i < RING; ++i)
    if (cudaEventCreateWithFlags(&p->ring[i].done, cudaEventDisableTiming) != cudaSuccess)
      return fail(LOGMEL_ERR_CUDA);
  delete t;
  *out = p;
  return LOGMEL_OK;
}

void logmel_plan_destroy(logmel_plan* p) {
  if (!p) return;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(p->device);
  cudaDeviceSynchronize();
  cudaFree(p->d_tables);
  cudaFree(p->d_fix);
  cudaFree(p->d_fixq);
  cudaFree(p->d_status);
  cudaFree(p->d_meta);
  cudaFree(p->d_tiles);
  for (int i = 0; i < RING; ++i) {
    if (p->ring[i].host) cudaFreeHost(p->ring[i].host);
    if (p->ring[i].done) cudaEventDestroy(p->ring[i].done);
  }
  if (prev >= 0) cudaSetDevice(prev);
  delete p;
}

int64_t logmel_num_frames(const logmel_plan* p, int64_t n) {
  if (!p) return -1;
  return n < 0 ? 0 : frames_of(n);
}

static logmel_status check_offsets(const int64_t* off, int64_t n_utt) {
  if (!off || n_utt < 0) return LOGMEL_ERR_INVALID_ARG;
  if (n_utt == 0) return LOGMEL_OK;
  if (off[0] < 0) return LOGMEL_ERR_INVALID_ARG;
  for (int64_t u = 0; u < n_utt; ++u)
    if (off[u + 1] < off[u]) return LOGMEL_ERR_INVALID_ARG;
  return LOGMEL_OK;
}

logmel_status logmel_frame_offsets(const logmel_plan* p, const int64_t* off, int64_t n_utt,
                                   int64_t* fo) {
  if (!p || !fo) return LOGMEL_ERR_INVALID_ARG;
  logmel_status st = check_offsets(off, n_utt);
  if (st != LOGMEL_OK) return st;
  fo[0] = 0;
  for (int64_t u = 0; u < n_utt; ++u) fo[u + 1] = fo[u] + frames_of(off[u + 1] - off[u]);
  return LOGMEL_OK;
}

int64_t logmel_total_frames(const logmel_plan* p, const int64_t* off, int64_t n_utt) {
  if (!p || check_offsets(off, n_utt) != LOGMEL_OK) return -1;
  int64_t t = 0;
  for (int64_t u = 0; u < n_utt; ++u) t += frames_of(off[u + 1] - off[u]);
  return t;
}

static logmel_status ensure_meta(logmel_plan* p, size_t bytes) {
  if (bytes > p->ring_cap) {
    for (int i = 0; i < RING; ++i) {
      if (p->ring[i].used) CK(cudaEventSynchronize(p->ring[i].done));
      if (p->ring[i].host) CK(cudaFreeHost(p->ring[i].host));
      p->ring[i].host = nullptr;
      p->ring[i].used = false;
    }
    size_t cap = std::max<size_t>(bytes, 4096);
    for (int i = 0; i < RING; ++i)
      if (cudaHostAlloc(&p->ring[i].host, cap, cudaHostAllocDefault) != cudaSuccess) {
        p->ring_cap = 0;
        return LOGMEL_ERR_OOM;
      }
    p->ring_cap = cap;
  }
  if (bytes > p->meta_cap) {
    CK(cudaDeviceSynchronize());
    CK(cudaFree(p->d_meta));
    p->d_meta = nullptr;
    size_t cap = std::max<size_t>(bytes, 4096);
    if (cudaMalloc(&p->d_meta, cap) != cudaSuccess) {
      p->meta_cap = 0;
      return LOGMEL_ERR_OOM;
    }
    p->meta_cap = cap;
  }
  return LOGMEL_OK;
}

logmel_status logmel_compute(logmel_plan* p, const float* pcm, const int64_t* off, int64_t n_utt,
                             float* out, void* stream) {
  if (!p) return LOGMEL_ERR_INVALID_ARG;
  logmel_status st = check_offsets(off, n_utt);
  if (st != LOGMEL_OK) return st;
  if (n_utt == 0) return LOGMEL_OK;
  if (n_utt >= INT32_MAX) return LOGMEL_ERR_INPUT_TOO_LONG;
  // frames and tiles per utterance (the ragged index map)
  int64_t frames = 0, tiles = 0;
  for (int64_t u = 0; u < n_utt; ++u) {
    const int64_t f = frames_of(off[u + 1] - off[u]);
    frames += f;
    tiles += (f + TILE - 1) / TILE;
  }
  if (frames == 0) return LOGMEL_OK;
  if (!pcm || !out) return LOGMEL_ERR_INVALID_ARG;
  if (tiles >= INT32_MAX || frames >= INT32_MAX) return LOGMEL_ERR_INPUT_TOO_LONG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Args a{};
  // the tile descriptors, which the kernel's prologue writes and its tile
  // loop reads
  if ((size_t)tiles > p->tiles_cap) {
    CK(cudaDeviceSynchronize());
    CK(cudaFree(p->d_tiles));
    p->d_tiles = nullptr;
    const size_t cap = std::max<size_t>((size_t)tiles, 1024);
    if (cudaMalloc(&p->d_tiles, cap * sizeof(TileDesc)) != cudaSuccess) {
      p->tiles_cap = 0;
      return LOGMEL_ERR_OOM;
    }
    p->tiles_cap = cap;
  }
  a.tiles = p->d_tiles;
  if (n_utt <= INLINE_UTT) {
    // small batches: the ragged index map travels in the launch parameters,
    // and the kernel finds each tile's utterance there (no metadata copy)
    a.meta_inline = 1;
    a.im_frame_off[0] = 0;
    a.im_tile_off[0] = 0;
    for (int64_t u = 0; u <= n_utt; ++u) a.im_sample_off[u] = off[u];
    for (int64_t u = 0; u < n_utt; ++u) {
      const int64_t f = frames_of(off[u + 1] - off[u]);
      a.im_frame_off[u + 1] = a.im_frame_off[u] + (int)f;
      a.im_tile_off[u + 1] = a.im_tile_off[u] + (int)((f + TILE - 1) / TILE);
    }
  } else {
    const size_t bytes = meta_bytes(n_utt);
    st = ensure_meta(p, bytes);
    if (st != LOGMEL_OK) return st;
    PinnedSlot& slot = p->ring[p->ring_next];
    p->ring_next = (p->ring_next + 1) % RING;
    if (slot.used) CK(cudaEventSynchronize(slot.done));
    MetaView hv = meta_view(slot.host, n_utt);
    hv.frame_off[0] = 0;
    hv.tile_off[0] = 0;
    for (int64_t u = 0; u <= n_utt; ++u) hv.sample_off[u] = off[u];
    for (int64_t u = 0; u < n_utt; ++u) {
      const int64_t f = frames_of(off[u + 1] - off[u]);
      hv.frame_off[u + 1] = hv.frame_off[u] + f;
      hv.tile_off[u + 1] = hv.tile_off[u] + (int)((f + TILE - 1) / TILE);
    }
    CK(cudaMemcpyAsync(p->d_meta, slot.host, bytes, cudaMemcpyHostToDevice, s));
    CK(cudaEventRecord(slot.done, s));
    slot.used = true;
    MetaView dv = meta_view(p->d_meta, n_utt);
    a.sample_off = dv.sample_off;
    a.frame_off = dv.frame_off;
    a.tile_off = dv.tile_off;
  }
  a.out = out;
  a.status = p->d_status;
  a.mode = 0;
  // the PCM as a tensor for one-box tile copies (re-encoded when the buffer
  // or its length changes)
  const int64_t total = off[n_utt];
  if (pcm != p->tmap_pcm || total != p->tmap_len) {
    p->tmap_pcm = pcm;
    p->tmap_len = total;
    for (int q = 0; q < 2; ++q) {
      p->tmap_rows[q] = encode_pcm_rows(&p->tmap[q], pcm, total, q);
      p->tmap_s_rows[q] = encode_pcm_map(&p->tmap_s[q], pcm, total, q, BLK);
    }
  }
  for (int q = 0; q < 2; ++q) {
    a.tmap[q] = p->tmap[q];
    a.tmap_rows[q] = p->tmap_rows[q];
    a.tmap_s[q] = p->tmap_s[q];
    a.tmap_s_rows[q] = p->tmap_s_rows[q];
  }
  if (p->default_mel) {
    if (out != p->otmap_out || frames != p->otmap_len) {
      p->otmap_out = out;
      p->otmap_len = frames;
      p->otmap_rows = encode_out_map(&p->otmap, out, frames, p->n_mels);
    }
    a.otmap = p->otmap;
    a.otmap_rows = p->otmap_rows;
  }
  a.num_tiles = (int)tiles;
  a.n_mels = p->n_mels;
  a.pcm = pcm;
  a.pcm_len = off[n_utt];
  a.n_utt = (int)n_utt;
  if (launch(p, a, tiles, s, has_odd_spans(pcm, off, n_utt)) != cudaSuccess) return LOGMEL_ERR_CUDA;
  return LOGMEL_OK;
}

// ---------------------------------------------------------------------------
// streaming
// ---------------------------------------------------------------------------
logmel_status logmel_stream_create(logmel_plan* p, int n_streams, logmel_stream** out) {
  if (!p || !out || n_streams < 1) return LOGMEL_ERR_INVALID_ARG;
  *out = nullptr;
  logmel_stream* st = new (std::nothrow) logmel_stream();
  if (!st) return LOGMEL_ERR_OOM;
  st->plan = p;
  st->n_streams = n_streams;
  st->total.assign(n_streams, 0);
  st->carry_len.assign(n_streams, 0);
  if (cudaMalloc(&st->d_carry, sizeof(float) * (size_t)n_streams * CARRY_CAP) != cudaSuccess ||
      cudaMalloc(&st->d_carry_len, sizeof(int) * (size_t)n_streams) != cudaSuccess) {
    logmel_stream_destroy(st);
    return LOGMEL_ERR_OOM;
  }
  if (cudaMemset(st->d_carry, 0, sizeof(float) * (size_t)n_streams * CARRY_CAP) != cudaSuccess ||
      cudaMemset(st->d_carry_len, 0, sizeof(int) * (size_t)n_streams) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    logmel_stream_destroy(st);
    return LOGMEL_ERR_CUDA;
  }
  *out = st;
  return LOGMEL_OK;
}

void logmel_stream_destroy(logmel_stream* st) {
  if (!st) return;
  cudaDeviceSynchronize();
  cudaFree(st->d_carry);
  cudaFree(st->d_carry_len);
  cudaFree(st->d_push_off);
  for (int i = 0; i < RING; ++i) {
    if (st->off_ring[i].host) cudaFreeHost(st->off_ring[i].host);
    if (st->off_ring[i].done) cudaEventDestroy(st->off_ring[i].done);
  }
  delete st;
}

int64_t logmel_stream_frames_for_push(const logmel_stream* st, int id, int64_t len) {
  if (!st || id < 0 || id >= st->n_streams || len < 0) return -1;
  return frames_of(st->carry_len[id] + len);
}

int64_t logmel_stream_max_frames(const logmel_stream* st, int64_t len) {
  if (!st || len < 0) return -1;
  int64_t mx = 0;
  for (int s = 0; s < st->n_streams; ++s) mx = std::max(mx, frames_of(st->carry_len[s] + len));
  return mx;
}

// Pinned staging of a ragged push's chunk offsets and their device copy.
static logmel_status stage_push_offsets(logmel_stream* st, const int64_t* off, int count,
                                        cudaStream_t s, const int64_t** d_off) {
  const size_t bytes = sizeof(int64_t) * ((size_t)st->n_streams + 1);
  if (!st->d_push_off) {
    if (cudaMalloc(&st->d_push_off, bytes) != cudaSuccess) {
      st->d_push_off = nullptr;
      return LOGMEL_ERR_OOM;
    }
    for (int i = 0; i < RING; ++i) {
      if (cudaHostAlloc(&st->off_ring[i].host, bytes, cudaHostAllocDefault) != cudaSuccess) {
        st->off_ring[i].host = nullptr;
        return LOGMEL_ERR_OOM;
      }
      CK(cudaEventCreateWithFlags(&st->off_ring[i].done, cudaEventDisableTiming));
    }
  }
  PinnedSlot& slot = st->off_ring[st->off_next];
  st->off_next = (st->off_next + 1) % RING;
  if (slot.used) CK(cudaEventSynchronize(slot.done));
  std::memcpy(slot.host, off, sizeof(int64_t) * ((size_t)count + 1));
  CK(cudaMemcpyAsync(st->d_push_off, slot.host, sizeof(int64_t) * ((size_t)count + 1),
                     cudaMemcpyHostToDevice, s));
  CK(cudaEventRecord(slot.done, s));
  slot.used = true;
  *d_off = st->d_push_off;
  return LOGMEL_OK;
}

// One push to streams base .. base + count - 1: either every stream takes
// len samples at chunks + i * chunk_stride (h_off == nullptr), or stream
// base + i takes chunks[h_off[i] .. h_off[i + 1]) (h_off: host, count + 1
// entries, non-decreasing).
int64_t logmel_stream_max_frames_ragged(const logmel_stream* st, const int64_t* off) {
  if (!st || !off || off[0] < 0) return -1;
  int64_t mx = 0;
  for (int s = 0; s < st->n_streams; ++s) {
    if (off[s + 1] < off[s]) return -1;
    mx = std::max(mx, frames_of(st->carry_len[s] + (off[s + 1] - off[s])));
  }
  return mx;
}

static logmel_status push_impl(logmel_stream* st, int base, int count, const float* chunks,
                               int64_t chunk_stride, int64_t len, float* out, int64_t cap,
                               int64_t* n_out, void* stream, const int64_t* h_off = nullptr) {
  logmel_plan* p = st->plan;
  if (cap < 0 || !n_out) return LOGMEL_ERR_INVALID_ARG;
  auto len_of = [&](int i) { return h_off ? h_off[i + 1] - h_off[i] : len; };
  if (h_off) {
    if (h_off[0] < 0) return LOGMEL_ERR_INVALID_ARG;
    len = 0;
    for (int i = 0; i < count; ++i) {
      if (h_off[i + 1] < h_off[i]) return LOGMEL_ERR_INVALID_ARG;
      len = std::max(len, h_off[i + 1] - h_off[i]);
    }
    if (h_off[count] >= (int64_t)INT32_MAX * 64) return LOGMEL_ERR_INPUT_TOO_LONG;
  }
  if (len < 0) return LOGMEL_ERR_INVALID_ARG;
  if (len > (int64_t)INT32_MAX / 2) return LOGMEL_ERR_INPUT_TOO_LONG;
  int64_t max_n = 0;
  for (int i = 0; i < count; ++i) max_n = std::max(max_n, frames_of(st->carry_len[base + i] + len_of(i)));
  if (max_n > cap) return LOGMEL_ERR_INVALID_ARG;
  if (len > 0 && !chunks) return LOGMEL_ERR_INVALID_ARG;
  if (max_n > 0 && !out) return LOGMEL_ERR_INVALID_ARG;
  if (!h_off && count > 1 && chunk_stride < len) return LOGMEL_ERR_INVALID_ARG;
  const int spt = max_n <= TILE / 4 ? 4 : (max_n <= TILE / 2 ? 2 : 1);
  const int64_t tps = max_n <= TILE ? 1 : (max_n + TILE - 1) / TILE;
  const int64_t tiles = (int64_t)((count + spt - 1) / spt) * tps;
  if (tiles >= INT32_MAX || (int64_t)count * cap >= INT32_MAX) return LOGMEL_ERR_INPUT_TOO_LONG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (len > 0) {
    const int64_t* d_off = nullptr;
    if (h_off) {
      const logmel_status so = stage_push_offsets(st, h_off, count, s, &d_off);
      if (so != LOGMEL_OK) return so;
    }
    Args a{};
    a.out = out;
    a.status = p->d_status;
    a.mode = 1;
    a.num_tiles = (int)tiles;
    a.n_mels = p->n_mels;
    a.carry = st->d_carry;
    a.carry_len = st->d_carry_len;
    a.chunks = chunks;
    a.chunk_stride = chunk_stride;
    a.push_len = len;
    a.push_off = d_off;
    a.stream_base = base;
    a.n_push_streams = count;
    a.spt = spt;
    a.tps = (int)tps;
    a.update_carry = tps == 1 ? 1 : 0;
    a.out_cap = cap;
    if (launch(p, a, tiles, s) != cudaSuccess) return LOGMEL_ERR_CUDA;
    if (tps > 1) {
      carry_update_kernel<<<count, 128, 0, s>>>(st->d_carry, st->d_carry_len, chunks, chunk_stride,
                                                len, base, d_off);
      CK(cudaGetLastError());
    }
  }
  for (int i = 0; i < count; ++i) {
    const int id = base + i;
    const int64_t B = st->carry_len[id] + len_of(i);
    const int64_t n = frames_of(B);
    n_out[i] = n;
    st->carry_len[id] = (int)(B - n * HOP);
    st->total[id] += len_of(i);
  }
  return LOGMEL_OK;
}

logmel_status logmel_stream_push(logmel_stream* st, int id, const float* chunk, int64_t len,
                                 float* out, int64_t cap, int64_t* n_out, void* stream) {
  if (!st || id < 0 || id >= st->n_streams) return LOGMEL_ERR_INVALID_ARG;
  return push_impl(st, id, 1, chunk, len, len, out, cap, n_out, stream);
}

logmel_status logmel_stream_push_batch(logmel_stream* st, const float* chunks, int64_t stride,
                                       int64_t len, float* out, int64_t cap, int64_t* n_out,
                                       void* stream) {
  if (!st) return LOGMEL_ERR_INVALID_ARG;
  return push_impl(st, 0, st->n_streams, chunks, stride, len, out, cap, n_out, stream);
}

logmel_status logmel_stream_push_batch_ragged(logmel_stream* st, const float* chunks,
                                              const int64_t* chunk_offsets, float* out, int64_t cap,
                                              int64_t* n_out, void* stream) {
  if (!st || !chunk_offsets) return LOGMEL_ERR_INVALID_ARG;
  return push_impl(st, 0, st->n_streams, chunks, 0, 0, out, cap, n_out, stream, chunk_offsets);
}

struct StateHeader {
  uint32_t magic;
  int32_t n_streams;
  int32_t carry_cap;
  int32_t reserved;
};

int64_t logmel_stream_state_bytes(const logmel_stream* st) {
  if (!st) return -1;
  return (int64_t)sizeof(StateHeader) +
         (int64_t)st->n_streams * (int64_t)(sizeof(int64_t) + sizeof(int32_t) + 4 * CARRY_CAP);
}

logmel_status logmel_stream_get_state(logmel_stream* st, void* blob, int64_t bytes, void* stream) {
  if (!st || !blob || bytes != logmel_stream_state_bytes(st)) return LOGMEL_ERR_INVALID_ARG;
  const int S = st->n_streams;
  std::vector<float> carry((size_t)S * CARRY_CAP);
  std::vector<int> lens(S);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CK(cudaMemcpyAsync(carry.data(), st->d_carry, carry.size() * 4, cudaMemcpyDeviceToHost, s));
  CK(cudaMemcpyAsync(lens.data(), st->d_carry_len, (size_t)S * 4, cudaMemcpyDeviceToHost, s));
  CK(cudaStreamSynchronize(s));
  for (int i = 0; i < S; ++i)
    if (lens[i] != st->carry_len[i]) return LOGMEL_ERR_DEVICE_STATUS;
  unsigned char* b = static_cast<unsigned char*>(blob);
  StateHeader h{STATE_MAGIC, S, CARRY_CAP, 0};
  std::memcpy(b, &h, sizeof h);
  b += sizeof h;
  for (int i = 0; i < S; ++i) {
    std::memcpy(b, &st->total[i], 8);
    std::memcpy(b + 8, &lens[i], 4);
    std::memcpy(b + 12, &carry[(size_t)i * CARRY_CAP], 4 * CARRY_CAP);
    b += 12 + 4 * CARRY_CAP;
  }
  return LOGMEL_OK;
}

logmel_status logmel_stream_set_state(logmel_stream* st, const void* blob, int64_t bytes,
                                      void* stream) {
  if (!st || !blob || bytes != logmel_stream_state_bytes(st)) return LOGMEL_ERR_INVALID_ARG;
  const unsigned char* b = static_cast<const unsigned char*>(blob);
  StateHeader h;
  std::memcpy(&h, b, sizeof h);
  if (h.magic != STATE_MAGIC || h.n_streams != st->n_streams || h.carry_cap != CARRY_CAP)
    return LOGMEL_ERR_INVALID_ARG;
  b += sizeof h;
  const int S = st->n_streams;
  std::vector<float> carry((size_t)S * CARRY_CAP);
  std::vector<int> lens(S);
  std::vector<int64_t> total(S);
  for (int i = 0; i < S; ++i) {
    std::memcpy(&total[i], b, 8);
    std::memcpy(&lens[i], b + 8, 4);
    std::memcpy(&carry[(size_t)i * CARRY_CAP], b + 12, 4 * CARRY_CAP);
    b += 12 + 4 * CARRY_CAP;
    const int64_t expect = total[i] - frames_of(total[i]) * HOP;
    if (total[i] < 0 || lens[i] != expect) return LOGMEL_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CK(cudaMemcpyAsync(st->d_carry, carry.data(), carry.size() * 4, cudaMemcpyHostToDevice, s));
  CK(cudaMemcpyAsync(st->d_carry_len, lens.data(), (size_t)S * 4, cudaMemcpyHostToDevice, s));
  CK(cudaStreamSynchronize(s));
  st->total = total;
  st->carry_len = lens;
  return LOGMEL_OK;
}

logmel_status logmel_stream_reset(logmel_stream* st, int id, void* stream) {
  if (!st || id >= st->n_streams) return LOGMEL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (id < 0) {
    CK(cudaMemsetAsync(st->d_carry_len, 0, sizeof(int) * (size_t)st->n_streams, s));
    std::fill(st->total.begin(), st->total.end(), 0);
    std::fill(st->carry_len.begin(), st->carry_len.end(), 0);
  } else {
    CK(cudaMemsetAsync(st->d_carry_len + id, 0, sizeof(int), s));
    st->total[id] = 0;
    st->carry_len[id] = 0;
  }
  return LOGMEL_OK;
}

logmel_status logmel_plan_set_wait_test(logmel_plan* p, int extra_tx_bytes, int poll_limit) {
  if (!p || extra_tx_bytes < 0 || extra_tx_bytes > (1 << 20) || extra_tx_bytes % 16 || poll_limit < 0)
    return LOGMEL_ERR_INVALID_ARG;
  p->tx_extra = extra_tx_bytes;
  p->wait_polls = poll_limit;
  return LOGMEL_OK;
}

logmel_status logmel_plan_device_status(logmel_plan* p, int* code, void* stream) {
  if (!p || !code) return LOGMEL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  CK(cudaMemcpyAsync(&v, p->d_status, sizeof(int), cudaMemcpyDeviceToHost, s));
  CK(cudaMemsetAsync(p->d_status, 0, sizeof(int), s));
  CK(cudaStreamSynchronize(s));
  *code = v;
  return LOGMEL_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free offline entry point: logmel_compute_noalloc
//
// For callers that cannot call cudaMalloc: a process whose device memory is
// owned by another allocator (a serving runtime or a host application that
// reserves the GPU's memory at start-up and hands out buffers, so a raw
// cudaMalloc fails or escapes its accounting), and a real-time audio path on
// which cudaMalloc / cudaFree would block the host thread or synchronise the
// device.  The caller still owns pcm and out; everything else the offline
// kernel needs lives in one fixed array in device memory.
// ---------------------------------------------------------------------------
namespace {

constexpr int64_t NOALLOC_MAX_UTT = 4096;     // utterances per call
constexpr int64_t NOALLOC_MAX_TILES = 32768;  // 32-frame tiles per call (1,048,576 frames)
constexpr int NOALLOC_MAX_DEVICES = 64;

// Scratch layout: FFT tables | float64 guard tables | status word | ragged
// metadata | tile descriptors | deferred guard frames.
constexpr size_t NA_TABLES_OFF = 0;
constexpr size_t NA_FIX_OFF = (sizeof(Tables) + 255) / 256 * 256;
constexpr size_t NA_STATUS_OFF = NA_FIX_OFF + (sizeof(double) * FIX_DOUBLES + 255) / 256 * 256;
constexpr size_t NA_META_OFF = NA_STATUS_OFF + 256;
constexpr size_t NA_META_CAP =   // meta_bytes(NOALLOC_MAX_UTT), rounded up to 256
    (16 * (NOALLOC_MAX_UTT + 1) + ((4 * (NOALLOC_MAX_UTT + 1) + 15) & ~15) + 255) / 256 * 256;
constexpr size_t NA_TILES_OFF = NA_META_OFF + NA_META_CAP;
constexpr int NA_FIXQ_GROUPS = 512;   // tile groups with a deferred-frame queue (148 SMs x 3 on a B200)
constexpr size_t NA_FIXQ_OFF = NA_TILES_OFF + NOALLOC_MAX_TILES * sizeof(TileDesc);
constexpr size_t NA_SCRATCH_BYTES = NA_FIXQ_OFF + (size_t)NA_FIXQ_GROUPS * FIXQ_CAP * sizeof(FixItem);
static_assert(NA_SCRATCH_BYTES < 768 * 1024, "no-alloc scratch is meant to stay modest");

}  // namespace

// The fixed device scratch (about 740 KB; every GPU that loads this library
// holds one copy until the process exits).  In host code this name is only
// a stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress, once per device, in noalloc_setup.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NA_SCRATCH_BYTES];

namespace {

struct NoAllocDevice {
  bool ready = false;
  unsigned char* scratch = nullptr;   // device address of g_noalloc_scratch on this device
  logmel_plan plan;                   // default front-end; tables and status word point into scratch
};

NoAllocDevice g_noalloc[NOALLOC_MAX_DEVICES];
std::mutex g_noalloc_mu;                                  // set-up and the host metadata buffer
alignas(16) unsigned char g_noalloc_meta[NA_META_CAP];    // host side of the metadata copy

}  // namespace

// Once per device, with that device current: look up the scratch address,
// build the default tables and filterbank on the host, upload the tables
// with a synchronous copy and set the kernel's shared-memory attribute.
static logmel_status noalloc_setup(int dev, NoAllocDevice& d) {
  void* sym = nullptr;
  CK(cudaGetSymbolAddress(&sym, g_noalloc_scratch));
  logmel_plan& p = d.plan;
  p.sr = 16000;
  p.n_fft = NFFT;
  p.hop = HOP;
  p.n_mels = 128;
  p.fmin = 0.f;
  p.fmax = 8000.f;
  p.device = dev;
  Tables t;
  logmel_status st = build_tables(&t);
  if (st == LOGMEL_OK) st = build_mel(&p);
  if (st != LOGMEL_OK) return st;
  if (!p.default_mel) return LOGMEL_ERR_UNSUPPORTED;   // the compiled layout is this filterbank
  int sms = 0, max_smem = 0;
  CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  CK(cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
  shape_launch(p.off, OFFLINE_SPAN_BLOCKS, p.n_mels, max_smem);
  shape_launch(p.str, STREAM_SPAN_BLOCKS, p.n_mels, max_smem);
  st = setup_kernel<true>(&p, sms);
  if (st != LOGMEL_OK) return st;
  unsigned char* base = static_cast<unsigned char*>(sym);
  CK(cudaMemcpy(base + NA_TABLES_OFF, &t, sizeof(Tables), cudaMemcpyHostToDevice));
  {
    double fix[FIX_DOUBLES];
    build_fix_tables(fix);
    CK(cudaMemcpy(base + NA_FIX_OFF, fix, sizeof fix, cudaMemcpyHostToDevice));
  }
  p.d_tables = reinterpret_cast<Tables*>(base + NA_TABLES_OFF);
  p.d_fix = reinterpret_cast<double*>(base + NA_FIX_OFF);
  p.d_status = reinterpret_cast<int*>(base + NA_STATUS_OFF);
  p.d_fixq = reinterpret_cast<FixItem*>(base + NA_FIXQ_OFF);
  p.fixq_groups = NA_FIXQ_GROUPS;
  d.scratch = base;
  d.ready = true;
  return LOGMEL_OK;
}

extern "C" int64_t logmel_noalloc_total_frames(const int64_t* off, int64_t n_utt) {
  if (check_offsets(off, n_utt) != LOGMEL_OK) return -1;
  int64_t t = 0;
  for (int64_t u = 0; u < n_utt; ++u) t += frames_of(off[u + 1] - off[u]);
  return t;
}

extern "C" logmel_status logmel_compute_noalloc(const float* pcm, const int64_t* off, int64_t n_utt,
                                                 float* out, int* device_status, void* stream) {
  logmel_status st = check_offsets(off, n_utt);
  if (st != LOGMEL_OK) return st;
  if (n_utt == 0) return LOGMEL_OK;
  if (n_utt > NOALLOC_MAX_UTT) return LOGMEL_ERR_NOALLOC_LIMIT;
  int64_t frames = 0, tiles = 0;
  for (int64_t u = 0; u < n_utt; ++u) {
    const int64_t f = frames_of(off[u + 1] - off[u]);
    frames += f;
    tiles += (f + TILE - 1) / TILE;
  }
  if (frames == 0) return LOGMEL_OK;
  if (!pcm || !out) return LOGMEL_ERR_INVALID_ARG;
  if (tiles > NOALLOC_MAX_TILES) return LOGMEL_ERR_NOALLOC_LIMIT;
  int dev = -1;
  CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return LOGMEL_ERR_UNSUPPORTED;

  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice& d = g_noalloc[dev];
  if (!d.ready) {
    st = noalloc_setup(dev, d);
    if (st != LOGMEL_OK) return st;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Args a{};
  if (n_utt <= INLINE_UTT) {
    // the ragged index map in the launch parameters, as logmel_compute does
    a.meta_inline = 1;
    a.im_frame_off[0] = 0;
    a.im_tile_off[0] = 0;
    for (int64_t u = 0; u <= n_utt; ++u) a.im_sample_off[u] = off[u];
    for (int64_t u = 0; u < n_utt; ++u) {
      const int64_t f = frames_of(off[u + 1] - off[u]);
      a.im_frame_off[u + 1] = a.im_frame_off[u] + (int)f;
      a.im_tile_off[u + 1] = a.im_tile_off[u] + (int)((f + TILE - 1) / TILE);
    }
  } else {
    // larger batches: the index map in the static host buffer, copied into
    // the scratch (a copy from pageable memory has consumed its source when
    // it returns)
    const size_t bytes = meta_bytes(n_utt);
    MetaView hv = meta_view(g_noalloc_meta, n_utt);
    hv.frame_off[0] = 0;
    hv.tile_off[0] = 0;
    for (int64_t u = 0; u <= n_utt; ++u) hv.sample_off[u] = off[u];
    for (int64_t u = 0; u < n_utt; ++u) {
      const int64_t f = frames_of(off[u + 1] - off[u]);
      hv.frame_off[u + 1] = hv.frame_off[u] + f;
      hv.tile_off[u + 1] = hv.tile_off[u] + (int)((f + TILE - 1) / TILE);
    }
    unsigned char* dmeta = d.scratch + NA_META_OFF;
    CK(cudaMemcpyAsync(dmeta, g_noalloc_meta, bytes, cudaMemcpyHostToDevice, s));
    MetaView dv = meta_view(dmeta, n_utt);
    a.sample_off = dv.sample_off;
    a.frame_off = dv.frame_off;
    a.tile_off = dv.tile_off;
  }
  a.tiles = reinterpret_cast<TileDesc*>(d.scratch + NA_TILES_OFF);
  // the status word starts at zero on every call; the tile descriptors are
  // rewritten by the kernel before it reads them, so they need no clearing
  int* status = device_status ? device_status : d.plan.d_status;
  CK(cudaMemsetAsync(status, 0, sizeof(int), s));
  a.out = out;
  a.status = status;
  a.mode = 0;
  // the PCM as a tensor for one-box tile copies, as in logmel_compute
  for (int q = 0; q < 2; ++q) {
    a.tmap_rows[q] = encode_pcm_rows(&a.tmap[q], pcm, off[n_utt], q);
    a.tmap_s_rows[q] = encode_pcm_map(&a.tmap_s[q], pcm, off[n_utt], q, BLK);
  }
  a.otmap_rows = encode_out_map(&a.otmap, out, frames, d.plan.n_mels);
  a.num_tiles = (int)tiles;
  a.n_mels = d.plan.n_mels;
  a.pcm = pcm;
  a.pcm_len = off[n_utt];
  a.n_utt = (int)n_utt;
  if (launch(&d.plan, a, tiles, s, has_odd_spans(pcm, off, n_utt)) != cudaSuccess) return LOGMEL_ERR_CUDA;
  return LOGMEL_OK;
}
