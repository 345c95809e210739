// FP32 FMA-pipe probe (declared in include/fp32_peak.h): the FP32 peak that
// the log-mel kernel's arithmetic is measured against, taken on the device
// itself rather than from a nominal clock and lane count.
#include <cuda_runtime.h>

#include "fp32_peak.h"

namespace {

constexpr int CHAINS = 16;   // independent accumulators per thread (f32x2: 32 lanes of work)

__global__ void fma_scalar(float* out, int iters, float a, float b) {
  float acc[2 * CHAINS];
#pragma unroll
  for (int i = 0; i < 2 * CHAINS; ++i) acc[i] = threadIdx.x * 1e-7f + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 2 * CHAINS; ++i) acc[i] = fmaf(acc[i], a, b);
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 2 * CHAINS; ++i) s += acc[i];
  if (s == 12345.678f) out[threadIdx.x] = s;   // keeps the chains live
}

__global__ void fma_packed(float* out, int iters, float a, float b) {
  float2 acc[CHAINS];
  const float2 va = make_float2(a, a), vb = make_float2(b, b);
#pragma unroll
  for (int i = 0; i < CHAINS; ++i) acc[i] = make_float2(threadIdx.x * 1e-7f + i, i + 0.5f);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < CHAINS; ++i) acc[i] = __ffma2_rn(acc[i], va, vb);
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < CHAINS; ++i) s += acc[i].x + acc[i].y;
  if (s == 12345.678f) out[threadIdx.x] = s;
}

}  // namespace

extern "C" int fp32_fma_probe(int packed, int blocks_per_sm, int iters, double* fma_per_s) {
  if (!fma_per_s || blocks_per_sm < 1 || iters < 1) return (int)cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  float* out = nullptr;
  if (e == cudaSuccess) e = cudaMalloc(&out, 256 * sizeof(float));
  cudaEvent_t t0 = nullptr, t1 = nullptr;
  if (e == cudaSuccess) e = cudaEventCreate(&t0);
  if (e == cudaSuccess) e = cudaEventCreate(&t1);
  const int threads = 256, blocks = sms * blocks_per_sm;
  float ms = 0.f;
  for (int rep = 0; e == cudaSuccess && rep < 2; ++rep) {   // the first launch warms up
    e = cudaEventRecord(t0);
    if (packed) fma_packed<<<blocks, threads>>>(out, iters, 0.999999f, 1e-6f);
    else fma_scalar<<<blocks, threads>>>(out, iters, 0.999999f, 1e-6f);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaEventRecord(t1);
    if (e == cudaSuccess) e = cudaEventSynchronize(t1);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, t0, t1);
  }
  if (e == cudaSuccess)
    *fma_per_s = (double)blocks * threads * iters * (2.0 * CHAINS) / (ms * 1e-3);
  if (t0) cudaEventDestroy(t0);
  if (t1) cudaEventDestroy(t1);
  if (out) cudaFree(out);
  return (int)e;
}
