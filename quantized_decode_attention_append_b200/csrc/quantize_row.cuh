// Quantization of appended rows, shared by the append kernels and the fused append + decode
// kernel: exact-rounded grid codes, group scales, bit-tight packing and anchor copies of one row
// slice (see quantize_slice).
//
// Every code is the nearest grid level in exact arithmetic, ties toward the larger code.  A fast
// fp32 estimate is corrected by comparisons against thresholds that are exact (fp32 for the
// absmax grids, whose thresholds are small odd integers times an fp16 scale; fp64 for min-max,
// whose thresholds add an fp16 zero point), so no rounding in a division can flip a code.
//
// Each translation unit that includes this header holds its own copy of the threshold tables and
// uploads it with upload_row_tables.
#pragma once

#include <math.h>

#include "kvq_internal.h"

namespace kvq {

static __constant__ float q_nf4_mid[15];
static __constant__ float q_lloyd_mid[3][15];

static inline cudaError_t upload_row_tables(const HostTables& t) {
  cudaError_t e = cudaMemcpyToSymbol(q_nf4_mid, t.nf4_mid, sizeof(t.nf4_mid));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(q_lloyd_mid, t.lloyd_mid, sizeof(t.lloyd_mid));
}

// Bitwise choice: bits of a where m is set, of b elsewhere (one 3-input logic op).
__device__ __forceinline__ uint32_t bsel(uint32_t m, uint32_t a, uint32_t b) { return (a & m) | (b & ~m); }

enum Fam { FAM_ABSMAX = 0, FAM_MINMAX = 1, FAM_NF4 = 2, FAM_TERNARY = 3, FAM_SIGN = 4, FAM_SYM = 5, FAM_LLOYD = 6 };

// Exact k = floor(x/d + 1/2) for fp16 d != 0 (absmax grids, zero point 0), in fp32.
// (2k +- 1) d is exact in fp32 for |k| <= 2^9, and 2x is exact, so the comparisons are exact.
__device__ __forceinline__ float round_exact_absmax(float x, float d, float inv) {
  float k = floorf(__fadd_rn(__fmul_rn(x, inv), 0.5f));
  const float t2 = __fmul_rn(2.0f, x);
  const float lo = __fmul_rn(__fsub_rn(__fmul_rn(2.0f, k), 1.0f), d);
  const float hi = __fmul_rn(__fadd_rn(__fmul_rn(2.0f, k), 1.0f), d);
  if (d > 0.0f) {
    if (t2 < lo) k -= 1.0f;
    else if (t2 >= hi) k += 1.0f;
  } else {
    if (t2 > lo) k -= 1.0f;
    else if (t2 <= hi) k += 1.0f;
  }
  return k;
}

// Pack 32 codes of `bits` bits (LSB-first) into bits words at out (skipped unless ok).
template <int B>
__device__ __forceinline__ void pack32(const uint32_t* code, uint32_t* out, bool ok) {
  uint32_t w[B];
#pragma unroll
  for (int k = 0; k < B; ++k) w[k] = 0u;
#pragma unroll
  for (int v = 0; v < 32; ++v) {  // fields are disjoint, so adding the shifted code is an OR
    const int bit = v * B, wi = bit >> 5, sh = bit & 31;
    w[wi] += code[v] << sh;
    if (sh + B > 32) w[wi + 1] |= code[v] >> (32 - sh);
  }
  if (ok) {
#pragma unroll
    for (int k = 0; k < B; ++k) out[k] = w[k];
  }
}

// Same, for codes held as fp32 bit patterns 1.5 * 2^23 + code (B divides 32, so no field crosses a
// word): the patterns' constant parts are added with the codes and taken off once per word.
template <int B>
__device__ __forceinline__ void pack32_biased(const uint32_t* code, uint32_t* out, bool ok) {
  static_assert(32 % B == 0, "fields must not cross words");
  constexpr int PW = 32 / B;
  constexpr uint32_t bias = [] {
    uint32_t t = 0u;
    for (int j = 0; j < PW; ++j) t += 0x4B400000u << (j * B);
    return t;
  }();
  uint32_t w[B];
#pragma unroll
  for (int k = 0; k < B; ++k) w[k] = 0u - bias;
#pragma unroll
  for (int v = 0; v < 32; ++v) w[v / PW] += code[v] << ((v % PW) * B);
  if (ok) {
#pragma unroll
    for (int k = 0; k < B; ++k) out[k] = w[k];
  }
}

__device__ __forceinline__ void pack32_bits(const uint32_t* code, int bits, uint32_t* out, bool ok) {
  switch (bits) {
    case 1: pack32<1>(code, out, ok); break;
    case 2: pack32<2>(code, out, ok); break;
    case 3: pack32<3>(code, out, ok); break;
    case 4: pack32<4>(code, out, ok); break;
    case 5: pack32<5>(code, out, ok); break;
    case 6: pack32<6>(code, out, ok); break;
    case 7: pack32<7>(code, out, ok); break;
    default: pack32<8>(code, out, ok); break;
  }
}

// The exact code from an estimate k within one of it: the midpoints z + (k -+ 1/2) d, exact in
// fp64 (fp16 values are multiples of 2^-25 below 2^25), decide (ties toward the larger code).
__device__ __forceinline__ float settle_minmax(float x, float z, float d, float k) {
  const double X = x, Z = z, Dd = d;
  if (X < fma((double)k - 0.5, Dd, Z)) return k - 1.0f;
  if (X >= fma((double)k + 0.5, Dd, Z)) return k + 1.0f;
  return k;
}

// Exact k = floor((x - z)/d + 1/2), d > 0, z and d fp16.  Far from a tie the fp32 estimate is
// exact (its error is < 2^-14); near one it is within one, and settle_minmax decides.
__device__ __forceinline__ float round_exact_minmax(float x, float z, float d, float inv) {
  const float r = __fmul_rn(__fsub_rn(x, z), inv);
  float k = floorf(__fadd_rn(r, 0.5f));
  const float fr = __fsub_rn(__fadd_rn(r, 0.5f), k);
  if (fr < (1.0f / 1024.0f) || fr > (1.0f - 1.0f / 1024.0f)) k = settle_minmax(x, z, d, k);
  return k;
}

__device__ __forceinline__ bool in_anchor(const LayerDev& L, int pos, int len_after) {
  if (!L.anchored) return false;
  if (L.anchor_rule == KVQ_ANCHOR_FIRST_N) return pos < L.anchor_n;
  if (L.anchor_rule == KVQ_ANCHOR_WINDOW) return pos >= len_after - L.anchor_n;
  if (L.anchor_rule == KVQ_ANCHOR_ALL) return true;
  return false;
}

__device__ __forceinline__ int anchor_slot(const LayerDev& L, int pos) {
  return (L.anchor_rule == KVQ_ANCHOR_WINDOW) ? (pos % L.anchor_n) : pos;
}

// NF4 code of x: number of thresholds th[0..14] (ascending) that x reaches, by a 4-step binary
// search whose thresholds are picked by multiplexers on the decisions taken so far.
__device__ __forceinline__ uint32_t nf4_code(float x, const float* th) {
  const bool b3 = x >= th[7];
  const bool b2 = x >= (b3 ? th[11] : th[3]);
  const bool b1 = x >= (b3 ? (b2 ? th[13] : th[9]) : (b2 ? th[5] : th[1]));
  const float t0 = b3 ? (b2 ? (b1 ? th[14] : th[12]) : (b1 ? th[10] : th[8]))
                      : (b2 ? (b1 ? th[6] : th[4]) : (b1 ? th[2] : th[0]));
  const bool b0 = x >= t0;
  return (b3 ? 8u : 0u) + (b2 ? 4u : 0u) + (b1 ? 2u : 0u) + (b0 ? 1u : 0u);
}

// An int8/int4 anchor row's group `li` (channels 32 li .. 32 li + 31, the lane's own slice): the
// signed absmax grid of the int format on the raw fp16 values (largest magnitude, first on ties,
// at -2^(b-1)), one fp16 scale (anchored rows are rare: a branch the row kernels seldom take).
__device__ __forceinline__ void anchor_quant32(const LayerDev& L, const SideDev& S, long long arow, int li, uint4 c0,
                                            uint4 c1, uint4 c2, uint4 c3) {
  const int b = L.anchor_bits, half = 1 << (b - 1);
  const uint4 cw[4] = {c0, c1, c2, c3};  // the 32 fp16 values, by value (no address of the caller's registers)
  float x[32];
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {
    const __half2* h2 = reinterpret_cast<const __half2*>(&cw[c4]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h2[e]);
      x[8 * c4 + 2 * e] = f.x;
      x[8 * c4 + 2 * e + 1] = f.y;
    }
  }
  float best = -1.0f, m = 0.0f;
#pragma unroll
  for (int v = 0; v < 32; ++v)
    if (fabsf(x[v]) > best) {
      best = fabsf(x[v]);
      m = x[v];
    }
  const __half sh = __float2half_rn(__fmul_rn(m, -1.0f / (float)half));
  const float d = __half2float(sh), inv = d != 0.0f ? __frcp_rn(d) : 0.0f;
  uint32_t code[32];
#pragma unroll
  for (int v = 0; v < 32; ++v) {
    const float k = d != 0.0f ? fminf(fmaxf(round_exact_absmax(x[v], d, inv), (float)(-half)), (float)(half - 1)) : 0.0f;
    code[v] = (uint32_t)((int)k + half);
  }
  uint32_t* out = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(S.anchors) + arow * L.anchor_rb) + li * b;
  if (b == 8) pack32<8>(code, out, true);
  else pack32<4>(code, out, true);
  S.anchor_scales[arow * (L.D / 32) + li] = sh;
}

// One appended row slice: lane li = lane % (head_dim / 32) of the row's lanes holds the row's
// values 32 li .. 32 li + 31 (cw, fp16).  Writes the anchor copy if the row is anchored, then the
// pre-transforms (key mean, channel scale, Hadamard), group scales, codes and packed words of the
// row at (unit u, position pos).  Every lane of the warp calls it (the shuffles span the warp);
// lanes with ok = false compute on zeros and store nothing.  EXT = false compiles out the key
// mean, int anchors and head-group input mapping.
template <int FAM, int G, int BITS, bool EXT>
__device__ __forceinline__ void quantize_slice(const LayerDev& L, const SideDev& S, const uint4 (&cw)[4], bool ok,
                                               int u, int pos, int len_after) {
  const int D = L.D, lpr = D >> 5;                    // lanes per row
  const int lane = threadIdx.x & 31;
  const int li = lane % lpr;                          // this lane's 32-value slice of its row
  constexpr int LG = G > 32 ? G / 32 : 1;             // lanes per group
  constexpr int GPL = G > 32 ? 1 : 32 / G;            // groups per lane
  // code bits: fixed by the family, by the instance (BITS > 0), or read from the side
  const int bits = FAM == FAM_SIGN ? 1 : (FAM == FAM_NF4 ? 4 : (BITS > 0 ? BITS : S.bits));
  // the grid sees the fp16 input itself (no key mean, channel scale or rotation in between)
  const bool raw = !S.rot && !S.chan_scale && !(EXT && S.mean_sub);
  float x[32];
  __half2 raw2[16];  // the lane's 32 input values as stored (fp16 pairs)
  if (ok) {
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      const __half2* h2 = reinterpret_cast<const __half2*>(&cw[c4]);
#pragma unroll
      for (int e = 0; e < 4; ++e) raw2[c4 * 4 + e] = h2[e];
    }
    if (!(FAM == FAM_NF4 && raw)) {  // NF4 on untransformed rows reads raw2 only
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 f = __half22float2(raw2[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
      }
    }
    if (in_anchor(L, pos, len_after)) {
      const long long arow = (long long)u * L.anchor_rows + anchor_slot(L, pos);
      if (!EXT || L.anchor_bits == 16) {
        __half* ap = S.anchors + arow * D + li * 32;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) reinterpret_cast<uint4*>(ap)[c4] = cw[c4];
      } else {
        anchor_quant32(L, S, arow, li, cw[0], cw[1], cw[2], cw[3]);
      }
    }
    if (EXT && S.mean_sub) {
      const __half* mp = S.kmean + (long long)u * D + li * 32;
#pragma unroll
      for (int v = 0; v < 32; ++v) x[v] = __fsub_rn(x[v], __half2float(mp[v]));
    }
    if (S.chan_scale) {
      const __half* cp = S.chan + (u % L.Hkv) * D + li * 32;
#pragma unroll
      for (int v = 0; v < 32; ++v) x[v] = __fdiv_rn(x[v], __half2float(cp[v]));
    }
  } else {
#pragma unroll
    for (int v = 0; v < 32; ++v) x[v] = 0.0f;
#pragma unroll
    for (int v = 0; v < 16; ++v) raw2[v] = __float2half2_rn(0.0f);
  }
  if (S.rot) {  // stages h = 1 .. rot/2 (warp-uniform: every lane takes part in the shuffles)
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
      for (int v = 0; v < 32; ++v)
        if ((v & h) == 0) {
          const float a = x[v], b = x[v + h];
          x[v] = __fadd_rn(a, b);
          x[v + h] = __fsub_rn(a, b);
        }
    }
    for (int h = 32; h < S.rot; h <<= 1) {
      const int lm = h >> 5;
      const bool upper = (li & lm) != 0;
#pragma unroll
      for (int v = 0; v < 32; ++v) {
        const float o = __shfl_xor_sync(0xffffffffu, x[v], lm);
        x[v] = upper ? __fsub_rn(o, x[v]) : __fadd_rn(x[v], o);
      }
    }
    const float rn = S.rot == 256 ? 0.0625f : __fdiv_rn(__fsqrt_rn(2.0f), 16.0f);
#pragma unroll
    for (int v = 0; v < 32; ++v) x[v] = __fmul_rn(x[v], rn);
  }
  const long long rix = (long long)u * L.Tcap + pos;
  uint32_t* wout = reinterpret_cast<uint32_t*>(S.codes + rix * S.row_bytes) + li * bits;  // this lane's words
  uint32_t code[32];
#pragma unroll
  for (int gl = 0; gl < GPL; ++gl) {
    const float* xg = x + gl * (G > 32 ? 32 : G);
    constexpr int NV = G > 32 ? 32 : G;
    __half sh, zh = __float2half_rn(0.0f);
    float d = 0.0f, z = 0.0f, inv = 0.0f;
    if (FAM == FAM_ABSMAX) {
      // signed value of largest magnitude, first channel on ties: the group's maximum or minimum,
      // whichever is larger in magnitude; only a group holding both +a and -a (or only zeros)
      // needs the earliest channel reaching a, found by a backward scan
      float mx, mn;
      if (NV >= 2 && raw) {  // x is the fp16 input: max and min two at a time
        const __half2* rg = raw2 + (gl * NV) / 2;
        __half2 hx = rg[0], hn = rg[0];
#pragma unroll
        for (int p2 = 1; p2 < NV / 2; ++p2) { hx = __hmax2(hx, rg[p2]); hn = __hmin2(hn, rg[p2]); }
        mx = fmaxf(__low2float(hx), __high2float(hx));
        mn = fminf(__low2float(hn), __high2float(hn));
      } else {
        mx = xg[0];
        mn = xg[0];
#pragma unroll
        for (int v = 1; v < NV; ++v) { mx = fmaxf(mx, xg[v]); mn = fminf(mn, xg[v]); }
      }
#pragma unroll
      for (int o = 1; o < LG; o <<= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      }
      float m = mx > -mn ? mx : mn;
      const bool tie = !(mx > -mn) && !(-mn > mx);
      if (__any_sync(0xffffffffu, tie)) {  // warp-uniform, so the shuffles below see every lane
        float am = 0.0f;
#pragma unroll
        for (int v = 0; v < NV; ++v) am = fmaxf(am, fabsf(xg[v]));
        float me = 0.0f;
#pragma unroll
        for (int v = NV - 1; v >= 0; --v) me = fabsf(xg[v]) == am ? xg[v] : me;
#pragma unroll
        for (int o = 1; o < LG; o <<= 1) {  // the lane with the lower channels wins ties
          const float oam = __shfl_xor_sync(0xffffffffu, am, o), om = __shfl_xor_sync(0xffffffffu, me, o);
          if (oam > am || (oam == am && (li & o))) { am = oam; me = om; }
        }
        if (tie) m = me;
      }
      const int half = 1 << (bits - 1);
      sh = __float2half_rn(__fmul_rn(m, -1.0f / (float)half));
      d = __half2float(sh);
      inv = d != 0.0f ? __frcp_rn(d) : 0.0f;
      // code = floor(x/d + 1/2) + half.  x * inv + half + 1.5 * 2^23, rounded once by the fma,
      // is 1.5 * 2^23 + the integer nearest to the estimate x * inv + half (error below 2^-17,
      // as |x/d| <= half <= 2^7), so the code sits in the low mantissa bits with no conversion
      // instruction.  A remainder within 2^-16 of +-1/2 sends the lane's group through the
      // exact comparisons instead.
      // With BIASED the codes stay as the fp32 patterns (pack32_biased removes the constant).
      constexpr bool BIASED = BITS == 2 || BITS == 4 || BITS == 8;
      constexpr float kMagic = 12582912.0f;
      const float c1 = (float)half + kMagic;
      const uint32_t top = 2u * half - 1u;
      const float ctop = kMagic + (float)top;
      bool near = false;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const float t = fmaf(xg[v], inv, c1);
        const float fr = fmaf(xg[v], inv, c1 - t);  // c1 - t = half - k exactly
        near |= fabsf(fr) > 0.5f - 1.0f / 65536.0f;
        code[gl * NV + v] = BIASED ? __float_as_uint(fminf(t, ctop)) : min(__float_as_uint(t) - 0x4B400000u, top);
      }
      if (near && d != 0.0f) {
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const float k = fminf(fmaxf(round_exact_absmax(xg[v], d, inv), (float)(-half)), (float)(half - 1));
          code[gl * NV + v] = (uint32_t)((int)k + half) + (BIASED ? 0x4B400000u : 0u);
        }
      }
    } else if (FAM == FAM_MINMAX) {
      float mn = xg[0], mx = xg[0];
#pragma unroll
      for (int v = 1; v < NV; ++v) { mn = fminf(mn, xg[v]); mx = fmaxf(mx, xg[v]); }
#pragma unroll
      for (int o = 1; o < LG; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (__any_sync(0xffffffffu, mn == 0.0f)) {  // a zero minimum is -0 iff the group holds a -0
        bool negz = false;
#pragma unroll
        for (int v = 0; v < NV; ++v) negz |= __float_as_uint(xg[v]) == 0x80000000u;
#pragma unroll
        for (int o = 1; o < LG; o <<= 1) negz |= __shfl_xor_sync(0xffffffffu, (int)negz, o) != 0;
        if (mn == 0.0f) mn = negz ? -0.0f : 0.0f;
      }
      const int top = (1 << bits) - 1;
      zh = __float2half_rn(mn);
      sh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)top));
      z = __half2float(zh);
      d = __half2float(sh);
      inv = d != 0.0f ? __frcp_rn(d) : 0.0f;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float k = 0.0f;
        if (d != 0.0f) k = fminf(fmaxf(round_exact_minmax(xg[v], z, d, inv), 0.0f), (float)top);
        code[gl * NV + v] = (uint32_t)(int)k;
      }
    } else if (FAM == FAM_SYM) {
      // levels (q - (2^b - 1)/2) d with the outermost at the group's largest magnitude:
      // d = fp16(m / (2^(b-1) - 1/2)), q = floor(x/d) + 2^(b-1) clamped; floor(x/d) from an fp32
      // estimate corrected by the exact products k d and (k + 1) d
      float am = fabsf(xg[0]);
#pragma unroll
      for (int v = 1; v < NV; ++v) am = fmaxf(am, fabsf(xg[v]));
#pragma unroll
      for (int o = 1; o < LG; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      const int half = 1 << (bits - 1);
      sh = __float2half_rn(__fdiv_rn(am, (float)half - 0.5f));
      d = __half2float(sh);
      inv = d != 0.0f ? __frcp_rn(d) : 0.0f;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float k = floorf(__fmul_rn(xg[v], inv));
        if (xg[v] < __fmul_rn(k, d)) k -= 1.0f;
        else if (xg[v] >= __fmul_rn(k + 1.0f, d)) k += 1.0f;
        const float q = fminf(fmaxf(k + (float)half, 0.0f), (float)(2 * half - 1));
        code[gl * NV + v] = d != 0.0f ? (uint32_t)(int)q : (uint32_t)half;
      }
    } else if (FAM == FAM_LLOYD) {
      // Gaussian Lloyd-Max levels times the group RMS: s = fp16(sqrt(fp32(sum of rounded
      // squares in channel order) / g)); the code counts the thresholds (level midpoints times s,
      // exact in fp32) that x reaches
      float sum = 0.0f;
      if (LG == 1) {
#pragma unroll
        for (int v = 0; v < NV; ++v) sum = __fadd_rn(sum, __fmul_rn(xg[v], xg[v]));
      } else {
        const int base = lane - (li % LG);
#pragma unroll
        for (int k = 0; k < LG; ++k) {
          if ((li % LG) == k) {
#pragma unroll
            for (int v = 0; v < NV; ++v) sum = __fadd_rn(sum, __fmul_rn(xg[v], xg[v]));
          }
          sum = __shfl_sync(0xffffffffu, sum, base + k);
        }
      }
      sh = __float2half_rn(__fsqrt_rn(__fdiv_rn(sum, (float)G)));
      d = __half2float(sh);
      const int nl = 1 << bits;
      const float* mid = q_lloyd_mid[bits - 2];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        uint32_t c = 0u;
        for (int k = 0; k < nl - 1; ++k) c += xg[v] >= __fmul_rn(mid[k], d) ? 1u : 0u;
        code[gl * NV + v] = d != 0.0f ? c : (uint32_t)(nl >> 1);
      }
    } else if (FAM == FAM_SIGN) {
      float sum = 0.0f;  // fp32 sum of |x| in channel order, lane by lane across the group
      if (LG == 1) {
#pragma unroll
        for (int v = 0; v < NV; ++v) sum = __fadd_rn(sum, fabsf(xg[v]));
      } else {
        const int base = lane - (li % LG);
#pragma unroll
        for (int k = 0; k < LG; ++k) {
          if ((li % LG) == k) {
#pragma unroll
            for (int v = 0; v < NV; ++v) sum = __fadd_rn(sum, fabsf(xg[v]));
          }
          sum = __shfl_sync(0xffffffffu, sum, base + k);
        }
      }
      sh = __float2half_rn(__fmul_rn(sum, 1.0f / (float)G));
#pragma unroll
      for (int v = 0; v < NV; ++v) code[gl * NV + v] = xg[v] >= 0.0f ? 1u : 0u;
    } else {  // NF4 and ternary: absmax magnitude scale
      float am;
      if (FAM == FAM_NF4 && NV >= 2 && raw) {  // from the fp16 input pairs
        const __half2* rg = raw2 + (gl * NV) / 2;
        __half2 hx = rg[0], hn = rg[0];
#pragma unroll
        for (int p2 = 1; p2 < NV / 2; ++p2) { hx = __hmax2(hx, rg[p2]); hn = __hmin2(hn, rg[p2]); }
        am = fabsf(fmaxf(fmaxf(__low2float(hx), __high2float(hx)), -fminf(__low2float(hn), __high2float(hn))));
      } else {
        am = fabsf(xg[0]);
#pragma unroll
        for (int v = 1; v < NV; ++v) am = fmaxf(am, fabsf(xg[v]));
      }
#pragma unroll
      for (int o = 1; o < LG; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      sh = __float2half_rn(am);
      d = __half2float(sh);
      if (FAM == FAM_NF4) {
        if (raw) {
          // x is the fp16 input itself, so x >= th <=> x >= th rounded up to fp16: count the
          // thresholds reached two values at a time in fp16 (1024 + count keeps the count in
          // the low mantissa bits)
          __half2 t2[15];
#pragma unroll
          for (int k = 0; k < 15; ++k) t2[k] = __half2half2(__float2half_ru(__fmul_rn(q_nf4_mid[k], d)));
          uint32_t tw[15];
#pragma unroll
          for (int k = 0; k < 15; ++k) tw[k] = h2u(t2[k]);
#pragma unroll
          for (int p2 = 0; p2 < NV / 2; ++p2) {
            // the thresholds reached form a prefix, so its length comes from a 4-step binary
            // search, run on both halves at once: each step compares with the threshold that
            // the decisions so far select (bit masks, one 3-input logic op per 2-way choice)
            const __half2 xv = raw2[(gl * NV) / 2 + p2];
            const uint32_t m3 = __hge2_mask(xv, t2[7]);
            const uint32_t m2 = __hge2_mask(xv, u2h(bsel(m3, tw[11], tw[3])));
            const uint32_t m1 = __hge2_mask(
                xv, u2h(bsel(m3, bsel(m2, tw[13], tw[9]), bsel(m2, tw[5], tw[1]))));
            const uint32_t m0 = __hge2_mask(
                xv, u2h(bsel(m3, bsel(m2, bsel(m1, tw[14], tw[12]), bsel(m1, tw[10], tw[8])),
                             bsel(m2, bsel(m1, tw[6], tw[4]), bsel(m1, tw[2], tw[0])))));
            const uint32_t b = (m3 & 0x00080008u) | (m2 & 0x00040004u) | (m1 & 0x00020002u) | (m0 & 0x00010001u);
            code[gl * NV + 2 * p2] = b & 0xFu;
            code[gl * NV + 2 * p2 + 1] = b >> 16;
          }
        } else {
          float th[15];
#pragma unroll
          for (int k = 0; k < 15; ++k) th[k] = __fmul_rn(q_nf4_mid[k], d);  // exact (<= 24 bits)
#pragma unroll
          for (int v = 0; v < NV; ++v) code[gl * NV + v] = nf4_code(xg[v], th);
        }
        if (d == 0.0f) {  // all-zero group: the zero level
#pragma unroll
          for (int v = 0; v < NV; ++v) code[gl * NV + v] = 7u;
        }
      } else {  // ternary digits t + 1 (packed into bytes after the groups)
        const float hh = __fmul_rn(d, 0.5f);
#pragma unroll
        for (int v = 0; v < NV; ++v)
          code[gl * NV + v] = d != 0.0f ? ((xg[v] >= hh) ? 2u : ((xg[v] < -hh) ? 0u : 1u)) : 1u;
      }
    }
    if (ok && (LG == 1 || (li % LG) == 0)) {
      const int gi = (li * 32 + gl * NV) / G;
      S.scales[rix * S.n_groups + gi] = sh;
      if (FAM == FAM_MINMAX) S.zeros[rix * S.n_groups + gi] = zh;
    }
  }
  if (FAM != FAM_TERNARY) {
    if (FAM == FAM_SIGN) pack32<1>(code, wout, ok);
    else if (FAM == FAM_NF4) pack32<4>(code, wout, ok);
    else if (FAM == FAM_ABSMAX && (BITS == 2 || BITS == 4 || BITS == 8))
      pack32_biased<(BITS == 2 || BITS == 4 || BITS == 8) ? BITS : 8>(code, wout, ok);
    else if (BITS > 0) pack32<(BITS > 0 ? BITS : 8)>(code, wout, ok);
    else pack32_bits(code, bits, wout, ok);
  }
  if (FAM == FAM_TERNARY) {
    // Bytes hold 5 digits (byte = sum d_m 3^m), so they straddle lanes.  A lane writes the
    // bytes whose first digit is its own: [ceil(32 li / 5), ceil(32 (li + 1) / 5)); the last
    // one may need up to 4 digits of the next lane (zero past the row's end).
    uint32_t dlo = 0u, dhi = 0u;  // the lane's 32 digits as 2-bit fields
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      dlo += code[v] << (2 * v);
      dhi += code[16 + v] << (2 * v);
    }
    uint32_t nlo = __shfl_down_sync(0xffffffffu, dlo, 1);
    if (li == lpr - 1) nlo = 0u;
    const int b0 = (32 * li + 4) / 5, nb = (32 * li + 36) / 5 - b0;
    const int o2 = 2 * (5 * b0 - 32 * li);  // bit of the first owned digit in the lane's stream
    const uint32_t s0 = __funnelshift_r(dlo, dhi, o2), s1 = __funnelshift_r(dhi, nlo, o2), s2 = nlo >> o2;
    uint8_t* op = S.codes + rix * S.row_bytes + b0;
#pragma unroll
    for (int j = 0; j < 7; ++j) {
      const int bit = 10 * j;
      const uint32_t f = bit <= 22 ? (s0 >> bit)
                                  : (bit < 32 ? __funnelshift_r(s0, s1, bit)
                                              : (bit <= 54 ? (s1 >> (bit - 32)) : __funnelshift_r(s1, s2, bit - 32)));
      uint32_t t = (f >> 8) & 3u;
      t = t * 3u + ((f >> 6) & 3u);
      t = t * 3u + ((f >> 4) & 3u);
      t = t * 3u + ((f >> 2) & 3u);
      t = t * 3u + (f & 3u);
      if (ok && j < nb) op[j] = (uint8_t)t;
    }
  }
}

}  // namespace kvq
