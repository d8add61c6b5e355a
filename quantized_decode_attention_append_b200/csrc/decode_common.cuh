// Device helpers shared by the decode and dequantize kernels: read one stored-domain value (or a
// polar slot) of a packed row.  Stored domain = code x scale (+ zero); polar slots are
// m (cos phi, sin phi) with m = code x scale and phi = -pi + 2 pi k / 2^bp.
#pragma once

#include "kvq_internal.h"

namespace kvq {

// b-bit field starting at bit `bit` of a byte row (b <= 8: at most two bytes).
__device__ __forceinline__ uint32_t get_bits(const uint8_t* __restrict__ row, int bit, int b) {
  const int byte = bit >> 3, off = bit & 7;
  uint32_t v = row[byte];
  if (off + b > 8) v |= (uint32_t)row[byte + 1] << 8;
  return (v >> off) & ((1u << b) - 1u);
}

// Ternary digit (0, 1, 2 <-> -1, 0, +1) of element j: byte j/5 holds sum_m d_m 3^m.
__device__ __forceinline__ int get_trit(const uint8_t* __restrict__ row, int j) {
  int v = row[j / 5];
  switch (j % 5) {
    case 4: v /= 81; break;
    case 3: v /= 27; break;
    case 2: v /= 9; break;
    case 1: v /= 3; break;
    default: break;
  }
  return v % 3;
}

// Stored-domain value of element j of a non-polar quantized row.
//   row: packed codes; sc/zr: the row's fp16 scales / zero points; nf4: 16 levels; lloyd: the
//   2^bits Gaussian Lloyd-Max levels of the side's width.
__device__ __forceinline__ float stored_value(const SideDev& S, const uint8_t* __restrict__ row,
                                              const __half* __restrict__ sc, const __half* __restrict__ zr,
                                              int j, const float* nf4, const float* lloyd) {
  switch (S.fmt) {
    case KVQ_FMT_FP16:
      return __half2float(reinterpret_cast<const __half*>(row)[j]);
    case KVQ_FMT_INT: {
      const int g = j / S.group;
      const float d = __half2float(sc[g]);
      const int c = (int)get_bits(row, j * S.bits, S.bits);
      if (S.scale_mode == KVQ_SCALE_MINMAX) return __fadd_rn(__half2float(zr[g]), (float)c * d);
      if (S.scale_mode == KVQ_SCALE_SYMMETRIC) return ((float)c - 0.5f * (float)((1 << S.bits) - 1)) * d;
      return (float)(c - (1 << (S.bits - 1))) * d;
    }
    case KVQ_FMT_LLOYD:
      return lloyd[get_bits(row, j * S.bits, S.bits)] * __half2float(sc[j / S.group]);
    case KVQ_FMT_SORTED: {  // channel j's rank p (after the codes), then code p of its sorted group
      const int D = S.n_groups * S.group, rb = 32 - __clz(D - 1);
      const int p = (int)get_bits(row, D * S.bits + j * rb, rb), g = p / S.group;
      const int c = (int)get_bits(row, p * S.bits, S.bits);
      return __fadd_rn(__half2float(zr[g]), (float)c * __half2float(sc[g]));
    }
    case KVQ_FMT_NF4: {
      const float s = __half2float(sc[j / S.group]);
      return nf4[get_bits(row, j * 4, 4)] * s;
    }
    case KVQ_FMT_TERNARY: {
      const float s = __half2float(sc[j / S.group]);
      return (float)(get_trit(row, j) - 1) * s;
    }
    case KVQ_FMT_SIGN: {
      const float s = __half2float(sc[j / S.group]);
      return get_bits(row, j, 1) ? s : -s;
    }
    case KVQ_FMT_CART: {
      const int half = 1 << (S.bits - 1);
      return (float)((int)get_bits(row, j * S.bits, S.bits) - half) * __half2float(sc[0]);
    }
  }
  return 0.0f;
}

// Value j of anchor row `arow` (= unit x anchor_rows + slot) of a side, original domain: the fp16
// row, or an int8/int4 anchor's code times its group-of-32 scale.
__device__ __forceinline__ float anchor_value(const LayerDev& L, const SideDev& S, long long arow, int j) {
  if (L.anchor_bits == 16) return __half2float(S.anchors[arow * L.D + j]);
  const uint8_t* row = reinterpret_cast<const uint8_t*>(S.anchors) + arow * L.anchor_rb;
  const float d = __half2float(S.anchor_scales[arow * (L.D / 32) + j / 32]);
  return (float)((int)get_bits(row, j * L.anchor_bits, L.anchor_bits) - (1 << (L.anchor_bits - 1))) * d;
}

// Polar slot f of a row: (m cos phi, m sin phi); cs/sn: cos/sin tables for the row's phase bits.
__device__ __forceinline__ float2 polar_slot(const SideDev& S, const uint8_t* __restrict__ row,
                                             const __half* __restrict__ sc, int f, const float* cs,
                                             const float* sn) {
  const int bm = S.bits, bp = S.bits2;
  const float m = (float)get_bits(row, f * bm, bm) * __half2float(sc[0]);
  const int k = (int)get_bits(row, 64 * bm + f * bp, bp);
  return make_float2(__fmul_rn(m, cs[k]), __fmul_rn(m, sn[k]));
}

}  // namespace kvq
