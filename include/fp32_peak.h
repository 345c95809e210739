/*
 * fp32_peak.h -- measurement helper beside the log-mel library (not part of
 * the log-mel method; no page defines it).
 *
 * The log-mel kernel's roofline is the slower of its bytes over HBM and its
 * FFT + mel arithmetic over the FP32 pipe.  The HBM peak comes from a copy
 * measured on the device; this probe measures the FP32 side the same way:
 * a kernel of independent fused multiply-adds, 32 chains per thread, on
 * every SM, timed with CUDA events.
 */
#ifndef FP32_PEAK_H_
#define FP32_PEAK_H_

#ifdef __cplusplus
extern "C" {
#endif

/* Runs the FMA probe on the current device and returns the achieved rate in
 * FP32 FMA lane-operations per second (one fused multiply-add on one fp32
 * value; two flops) in *fma_per_s, for the packed two-lane form (packed != 0:
 * fma.rn.f32x2) or the scalar form.  blocks_per_sm x 256 threads per SM,
 * `iters` loop trips of 32 dependent-chain steps each.  Synchronises the
 * device.  Returns 0 on success, else the cudaError_t of the failing call. */
int fp32_fma_probe(int packed, int blocks_per_sm, int iters, double* fma_per_s);

#ifdef __cplusplus
}
#endif

#endif /* FP32_PEAK_H_ */
