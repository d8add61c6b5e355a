// 128-point radix-2 decimation-in-time FFT of one row held by one warp in registers, shared by
// the rFFT codecs' append and the polar decode's query transform.
//
// The input is loaded in bit-reversed order; lane l holds elements 4l .. 4l + 3 (element
// 4l + r is x[bitrev5(l) + 32 bitrev2(r)]).  Spans 2 and 4 pair elements inside a lane, spans
// 8 .. 128 pair lane l with lane l ^ (span / 8); every butterfly forms t = w b with separately
// rounded products and (a, b) <- (a + t, a - t), and both lanes of a pair form the same t from
// the same operands, so every element takes exactly the operations of the sequential transform.
// Afterwards lane l holds X_4l .. X_4l+3.  Twiddles: twr[k] + i twi[k] = exp(-2 pi i k / 128),
// k < 64, in shared memory (the lanes' indices diverge).
#pragma once

#include <cuda_runtime.h>

namespace kvq {

// One butterfly stage with half-span `half` >= 4 across lanes (partner lane ^ half / 4).
__device__ __forceinline__ void fft_stage_x(float (&re)[4], float (&im)[4], int half, int lane, const float* twr,
                                            const float* twi) {
  const int m = half >> 2, step = 64 / half;
  const bool up = (lane & m) != 0;  // this lane holds the i1 = i0 + half side
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int j = (4 * lane + r) & (half - 1);
    const float wr = twr[j * step], wi = twi[j * step];
    const float ore = __shfl_xor_sync(0xffffffffu, re[r], m), oim = __shfl_xor_sync(0xffffffffu, im[r], m);
    const float br = up ? re[r] : ore, bi = up ? im[r] : oim;
    const float ar = up ? ore : re[r], ai = up ? oim : im[r];
    const float tr = __fsub_rn(__fmul_rn(wr, br), __fmul_rn(wi, bi));
    const float ti = __fadd_rn(__fmul_rn(wr, bi), __fmul_rn(wi, br));
    re[r] = up ? __fsub_rn(ar, tr) : __fadd_rn(ar, tr);
    im[r] = up ? __fsub_rn(ai, ti) : __fadd_rn(ai, ti);
  }
}

// In-lane butterfly of elements (p, q = p + half) with twiddle index j * step.
__device__ __forceinline__ void fft_bfly(float (&re)[4], float (&im)[4], int p, int q, int tw, const float* twr,
                                         const float* twi) {
  const float wr = twr[tw], wi = twi[tw];
  const float br = re[q], bi = im[q];
  const float tr = __fsub_rn(__fmul_rn(wr, br), __fmul_rn(wi, bi));
  const float ti = __fadd_rn(__fmul_rn(wr, bi), __fmul_rn(wi, br));
  const float ar = re[p], ai = im[p];
  re[p] = __fadd_rn(ar, tr);
  im[p] = __fadd_rn(ai, ti);
  re[q] = __fsub_rn(ar, tr);
  im[q] = __fsub_rn(ai, ti);
}

// The whole transform (spans 2 .. 128) of a row loaded in bit-reversed order.
__device__ __forceinline__ void fft128_warp(float (&re)[4], float (&im)[4], int lane, const float* twr,
                                            const float* twi) {
  // spans 2 and 4 inside the lane (element index 4 lane + r: j = r mod half)
  fft_bfly(re, im, 0, 1, 0, twr, twi);
  fft_bfly(re, im, 2, 3, 0, twr, twi);
  fft_bfly(re, im, 0, 2, 0, twr, twi);
  fft_bfly(re, im, 1, 3, 32, twr, twi);
#pragma unroll
  for (int half = 4; half <= 64; half <<= 1) fft_stage_x(re, im, half, lane, twr, twi);
}

}  // namespace kvq
