// kvq_quantize_append: pre-transform, group scales, exact-rounded codes, bit-tight packing and
// anchor copies for each appended K/V row.
//
// Format sources (page title, section):
//   signed absmax int ("E22L" "What I tested"/"Result": ggml signed grid -2..1 x scale; llama.cpp
//   #21385 "Finding 1": q4_0), per-token min-max ("E21W" "What I tested", variant A), NF4 /
//   ternary / sign and fp16 anchors ("Fourier Magnitude KV Cache Quantization" post 6,
//   "Corrected semantics", "Milestone", "Minimal recipe"), 256-wide Walsh-Hadamard rotation and
//   per-channel K scale ("E21W" variants B, C, D; "E22L" "What I tested"), rFFT polar and
//   Cartesian codecs (same thread, reply: "The finite-phase implementation and the physical codec
//   may be worth separating", "The three controls I would try first").
//
// Every code is the nearest grid level in exact arithmetic, ties toward the larger code.  A fast
// fp32 estimate is corrected by comparisons against thresholds that are exact (fp32 for the
// absmax grids, whose thresholds are small odd integers times an fp16 scale; fp64 for min-max,
// whose thresholds add an fp16 zero point), so no rounding in a division can flip a code.
//
// Work mapping: one thread per row (two for head_dim 256), the whole row in registers so the
// Hadamard butterflies run without shuffles (one xor-shuffle stage for the 256-wide transform).
// The polar/Cartesian codecs run one warp per row with the FFT in shared memory.
#include <math.h>
#include <stdio.h>

#include "kvq_internal.h"

namespace kvq {

__constant__ float q_nf4_mid[15];
__constant__ float q_tw_re[64];
__constant__ float q_tw_im[64];

cudaError_t upload_tables_quant(const HostTables& t) {
  cudaError_t e = cudaMemcpyToSymbol(q_nf4_mid, t.nf4_mid, sizeof(t.nf4_mid));
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(q_tw_re, t.tw_re, sizeof(t.tw_re));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(q_tw_im, t.tw_im, sizeof(t.tw_im));
}

enum Fam { FAM_ABSMAX = 0, FAM_MINMAX = 1, FAM_NF4 = 2, FAM_TERNARY = 3, FAM_SIGN = 4 };

// ------------------------------------------------------------------------------------------
// Bit packer: LSB-first stream of b-bit codes into 32-bit words (row chunks are whole words).
struct Packer {
  uint32_t* out;
  uint64_t acc;
  int nb;
  int w;
  __device__ __forceinline__ void put(uint32_t code, int b) {
    acc |= (uint64_t)code << nb;
    nb += b;
    if (nb >= 32) {
      out[w++] = (uint32_t)acc;
      acc >>= 32;
      nb -= 32;
    }
  }
};

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

// Exact k = floor((x - z)/d + 1/2), d > 0, z and d fp16.  Far from a tie the fp32 estimate is
// exact (its error is < 2^-14); near one, fp64 thresholds z + (k +- 1/2) d are exact (fp16
// values are multiples of 2^-25 below 2^25) and decide.
__device__ __forceinline__ float round_exact_minmax(float x, float z, float d, float inv) {
  const float r = __fmul_rn(__fsub_rn(x, z), inv);
  float k = floorf(__fadd_rn(r, 0.5f));
  const float fr = __fsub_rn(__fadd_rn(r, 0.5f), k);
  if (fr < (1.0f / 1024.0f) || fr > (1.0f - 1.0f / 1024.0f)) {
    const double X = x, Z = z, Dd = d;
    double kk = floor(__dadd_rn(__ddiv_rn(__dsub_rn(X, Z), Dd), 0.5));
    const double lo = __dadd_rn(Z, __dmul_rn(__dsub_rn(kk, 0.5), Dd));
    if (X < lo) {
      kk -= 1.0;
    } else {
      const double hi = __dadd_rn(Z, __dmul_rn(__dadd_rn(kk, 0.5), Dd));
      if (X >= hi) kk += 1.0;
    }
    k = (float)kk;
  }
  return k;
}

// ------------------------------------------------------------------------------------------
// In-register orthonormal Walsh-Hadamard over 128 values: stages h = 1 .. 64, then x fp32(1/sqrt n).
template <int N>
__device__ __forceinline__ void fwht_local(float* x) {
#pragma unroll
  for (int h = 1; h < N; h <<= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if ((i & h) == 0) {
        const float a = x[i], b = x[i + h];
        x[i] = __fadd_rn(a, b);
        x[i + h] = __fsub_rn(a, b);
      }
    }
  }
}

template <int DH>
__device__ __forceinline__ void scale_all(float* x, float r) {
#pragma unroll
  for (int i = 0; i < DH; ++i) x[i] = __fmul_rn(x[i], r);
}

// Quantize one group of G values x[0..G) of family FAM; packs codes, returns scale (and zero).
template <int G, int FAM>
__device__ __forceinline__ void quant_group(const float* x, int bits, Packer& pk, uint8_t* trit_bytes,
                                            int jbase, __half& s_out, __half& z_out) {
  if (FAM == FAM_ABSMAX) {
    float m = x[0], am = fabsf(x[0]);
#pragma unroll
    for (int j = 1; j < G; ++j) {
      const float a = fabsf(x[j]);
      if (a > am) { am = a; m = x[j]; }
    }
    const int half = 1 << (bits - 1);
    const __half dh = __float2half_rn(__fmul_rn(m, -1.0f / (float)half));
    const float d = __half2float(dh);
    s_out = dh;
    const float inv = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
#pragma unroll
    for (int j = 0; j < G; ++j) {
      float k = 0.0f;
      if (d != 0.0f) {
        k = round_exact_absmax(x[j], d, inv);
        k = fminf(fmaxf(k, (float)(-half)), (float)(half - 1));
      }
      pk.put((uint32_t)((int)k + half), bits);
    }
  } else if (FAM == FAM_MINMAX) {
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int j = 1; j < G; ++j) { mn = fminf(mn, x[j]); mx = fmaxf(mx, x[j]); }
    const int top = (1 << bits) - 1;
    const __half zh = __float2half_rn(mn);
    const __half dh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)top));
    const float z = __half2float(zh), d = __half2float(dh);
    s_out = dh;
    z_out = zh;
    const float inv = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
#pragma unroll
    for (int j = 0; j < G; ++j) {
      float k = 0.0f;
      if (d != 0.0f) {
        k = round_exact_minmax(x[j], z, d, inv);
        k = fminf(fmaxf(k, 0.0f), (float)top);
      }
      pk.put((uint32_t)(int)k, bits);
    }
  } else if (FAM == FAM_NF4) {
    float am = fabsf(x[0]);
#pragma unroll
    for (int j = 1; j < G; ++j) am = fmaxf(am, fabsf(x[j]));
    const __half sh = __float2half_rn(am);
    const float s = __half2float(sh);
    s_out = sh;
    float t[15];
#pragma unroll
    for (int i = 0; i < 15; ++i) t[i] = __fmul_rn(q_nf4_mid[i], s);  // exact (<= 24 bits)
#pragma unroll
    for (int j = 0; j < G; ++j) {
      int c = 7;
      if (s != 0.0f) {
        c = 0;
#pragma unroll
        for (int i = 0; i < 15; ++i) c += (x[j] >= t[i]) ? 1 : 0;
      }
      pk.put((uint32_t)c, 4);
    }
  } else if (FAM == FAM_TERNARY) {
    float am = fabsf(x[0]);
#pragma unroll
    for (int j = 1; j < G; ++j) am = fmaxf(am, fabsf(x[j]));
    const __half sh = __float2half_rn(am);
    const float s = __half2float(sh);
    s_out = sh;
    const float h = __fmul_rn(s, 0.5f);
#pragma unroll
    for (int j = 0; j < G; ++j) {
      int dgt = 1;
      if (s != 0.0f) dgt = (x[j] >= h) ? 2 : ((x[j] < -h) ? 0 : 1);
      const int e = jbase + j;  // static element index
      const int p3 = (e % 5 == 0) ? 1 : (e % 5 == 1) ? 3 : (e % 5 == 2) ? 9 : (e % 5 == 3) ? 27 : 81;
      trit_bytes[e / 5] = (uint8_t)(trit_bytes[e / 5] + dgt * p3);
    }
  } else {  // FAM_SIGN
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < G; ++j) acc = __fadd_rn(acc, fabsf(x[j]));
    const __half sh = __float2half_rn(__fmul_rn(acc, 1.0f / (float)G));
    s_out = sh;
#pragma unroll
    for (int j = 0; j < G; ++j) pk.put(x[j] >= 0.0f ? 1u : 0u, 1);
  }
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

// Completion ticket: the last CTA of an append (over all its launches) advances seq_len.
// Every CTA read seq_len before it takes its ticket, so the update cannot race a reader.
__device__ __forceinline__ void finish_append(const LayerDev& L, int n_new, unsigned total_ctas) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned t = atomicAdd(L.ticket, 1u);
    if (t == total_ctas - 1) {
      for (int b = 0; b < L.B; ++b) {
        const int nl = L.seq_len[b] + n_new;
        L.seq_len[b] = nl < L.Tcap ? nl : L.Tcap;
      }
      *L.ticket = 0u;
      __threadfence();
    }
  }
}

template <int DH, int TPR, int G, int FAM>
__device__ __forceinline__ void quantize_row(const LayerDev& L, const SideDev& S, const float* x, int u, int pos,
                                             int part);

// ------------------------------------------------------------------------------------------
// Row kernel: DH values per thread, TPR threads per row (head_dim = DH * TPR).
template <int DH, int TPR, int G, int FAM>
__global__ void __launch_bounds__(128) append_rows_kernel(LayerDev L, int side, const __half* __restrict__ src,
                                                          int n_new, unsigned total_ctas) {
  const SideDev& S = L.s[side];
  const int D = DH * TPR;
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long R = (long long)L.B * L.Hkv * n_new;
  const long long row = gt / TPR;
  const int part = (int)(gt % TPR);
  const bool active = row < R;
  int pos = 0, len_after = 0, u = 0, i = 0, b = 0;
  if (active) {
    i = (int)(row % n_new);
    u = (int)(row / n_new);
    b = u / L.Hkv;
    const int len0 = L.seq_len[b];
    pos = len0 + i;
    len_after = len0 + n_new;
  }
  const bool ok = active && pos < L.Tcap;
  if (active && !ok && part == 0 && i == 0) atomicOr(L.err, (unsigned)KVQ_ERRF_CAPACITY);

  // TPR = 2 rows must keep both lanes of the pair converged for the shuffle stage.
  float x[DH];
  const __half* rp = src + ((long long)u * n_new + i) * D + part * DH;
  if (ok) {
#pragma unroll
    for (int c = 0; c < DH / 8; ++c) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(rp) + c);
      const __half2* h2 = reinterpret_cast<const __half2*>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h2[e]);
        x[c * 8 + 2 * e] = f.x;
        x[c * 8 + 2 * e + 1] = f.y;
      }
    }
    if (in_anchor(L, pos, len_after)) {
      __half* ap = S.anchors + ((long long)u * L.anchor_rows + anchor_slot(L, pos)) * D + part * DH;
#pragma unroll
      for (int c = 0; c < DH / 8; ++c)
        reinterpret_cast<uint4*>(ap)[c] = __ldg(reinterpret_cast<const uint4*>(rp) + c);
    }
    if (S.chan_scale) {
      const __half* cp = S.chan + (u % L.Hkv) * D + part * DH;
#pragma unroll
      for (int j = 0; j < DH; ++j) x[j] = __fdiv_rn(x[j], __half2float(cp[j]));
    }
  } else {
#pragma unroll
    for (int j = 0; j < DH; ++j) x[j] = 0.0f;
  }

  if (S.rot == 128 && DH == 128) {
    fwht_local<128>(x);
    scale_all<DH>(x, __fdiv_rn(__fsqrt_rn(2.0f), 16.0f));
  } else if (S.rot == 256 && DH == 128 && TPR == 2) {
    fwht_local<128>(x);
    // stage h = 128 pairs element j of the first half with element j of the second half
#pragma unroll
    for (int j = 0; j < DH; ++j) {
      const float other = __shfl_xor_sync(0xffffffffu, x[j], 1);
      x[j] = part == 0 ? __fadd_rn(x[j], other) : __fsub_rn(other, x[j]);
    }
    scale_all<DH>(x, 0.0625f);
  }
  if (ok) quantize_row<DH, TPR, G, FAM>(L, S, x, u, pos, part);
  // one barrier for every thread of the CTA (inactive rows included)
  finish_append(L, n_new, total_ctas);
}

template <int DH, int TPR, int G, int FAM>
__device__ __forceinline__ void quantize_row(const LayerDev& L, const SideDev& S, const float* x, int u, int pos,
                                             int part) {
  const int D = DH * TPR;
  const long long rix = (long long)u * L.Tcap + pos;
  const int ng = D / G;
  __half* sp = S.scales + rix * ng + part * (DH / G);
  __half* zp = S.zeros ? S.zeros + rix * ng + part * (DH / G) : nullptr;
  const int b_eff = (FAM == FAM_SIGN) ? 1 : (FAM == FAM_NF4) ? 4 : S.bits;
  Packer pk;
  pk.out = reinterpret_cast<uint32_t*>(S.codes + rix * S.row_bytes + (part * DH * b_eff) / 8);
  pk.acc = 0;
  pk.nb = 0;
  pk.w = 0;
  uint8_t tb[(DH + 4) / 5 + 1];
  if (FAM == FAM_TERNARY) {
#pragma unroll
    for (int j = 0; j < (DH + 4) / 5 + 1; ++j) tb[j] = 0;
  }
#pragma unroll
  for (int g = 0; g < DH / G; ++g) {
    __half s, z = __float2half_rn(0.0f);
    quant_group<G, FAM>(x + g * G, S.bits, pk, tb, g * G, s, z);
    sp[g] = s;
    if (FAM == FAM_MINMAX) zp[g] = z;
  }
  if (FAM == FAM_TERNARY) {
    uint8_t* op = S.codes + rix * S.row_bytes;
#pragma unroll
    for (int j = 0; j < (DH + 4) / 5; ++j) op[j] = tb[j];
  }
}

// ------------------------------------------------------------------------------------------
// rFFT polar / Cartesian codecs (head_dim 128): one warp per row, the radix-2 DIT FFT in shared
// memory in the evaluation order the format fixes (bit-reversed input; spans 2..128; t = w*b
// with separately rounded products; (a, b) <- (a + t, a - t)).
constexpr int kFftWarps = 4;

__device__ __forceinline__ int bitrev7(int i) { return (int)(__brev((unsigned)i) >> 25); }

__global__ void __launch_bounds__(128) append_fft_kernel(LayerDev L, int side, const __half* __restrict__ src,
                                                         int n_new, unsigned total_ctas) {
  const SideDev& S = L.s[side];
  __shared__ float sre[kFftWarps][128], sim[kFftWarps][128];
  __shared__ uint32_t scode[kFftWarps][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long R = (long long)L.B * L.Hkv * n_new;
  const long long row = (long long)blockIdx.x * kFftWarps + warp;
  bool ok = row < R;
  int pos = 0, len_after = 0, u = 0, i = 0;
  if (ok) {
    i = (int)(row % n_new);
    u = (int)(row / n_new);
    const int len0 = L.seq_len[u / L.Hkv];
    pos = len0 + i;
    len_after = len0 + n_new;
    if (pos >= L.Tcap) {
      if (lane == 0 && i == 0) atomicOr(L.err, (unsigned)KVQ_ERRF_CAPACITY);
      ok = false;
    }
  }
  if (ok) {
    const __half* rp = src + ((long long)u * n_new + i) * 128;
    float* re = sre[warp];
    float* im = sim[warp];
    for (int j = lane; j < 128; j += 32) {
      float v = __half2float(rp[j]);
      if (S.chan_scale) v = __fdiv_rn(v, __half2float(S.chan[(u % L.Hkv) * 128 + j]));
      re[bitrev7(j)] = v;
      im[bitrev7(j)] = 0.0f;
    }
    if (in_anchor(L, pos, len_after)) {
      __half* ap = S.anchors + ((long long)u * L.anchor_rows + anchor_slot(L, pos)) * 128;
      for (int j = lane; j < 128; j += 32) ap[j] = rp[j];
    }
    __syncwarp();
    for (int span = 2; span <= 128; span <<= 1) {
      const int half = span >> 1, step = 128 / span;
      for (int bf = lane; bf < 64; bf += 32) {
        const int grp = bf / half, j = bf % half;
        const int i0 = grp * span + j, i1 = i0 + half;
        const float wr = q_tw_re[j * step], wi = q_tw_im[j * step];
        const float br = re[i1], bi = im[i1];
        const float tr = __fsub_rn(__fmul_rn(wr, br), __fmul_rn(wi, bi));
        const float ti = __fadd_rn(__fmul_rn(wr, bi), __fmul_rn(wi, br));
        const float ar = re[i0], ai = im[i0];
        re[i0] = __fadd_rn(ar, tr);
        im[i0] = __fadd_rn(ai, ti);
        re[i1] = __fsub_rn(ar, tr);
        im[i1] = __fsub_rn(ai, ti);
      }
      __syncwarp();
    }
    // folded slots: slot 0 = (X_0, X_64), slot f = X_f
    float a[2], bb[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int f = lane + 32 * r;
      a[r] = re[f];
      bb[r] = (f == 0) ? re[64] : im[f];
    }
    const long long rix = (long long)u * L.Tcap + pos;
    uint32_t* codes_w = reinterpret_cast<uint32_t*>(S.codes + rix * S.row_bytes);
    if (S.fmt == KVQ_FMT_POLAR) {
      const int bm = S.bits, bp = S.bits2;
      float mag[2];
      float mmax = 0.0f;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mag[r] = __fsqrt_rn(__fadd_rn(__fmul_rn(a[r], a[r]), __fmul_rn(bb[r], bb[r])));
        mmax = fmaxf(mmax, mag[r]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
      const __half sh = __float2half_rn(__fdiv_rn(mmax, (float)((1 << bm) - 1)));
      const float s = __half2float(sh);
      const float inv = s != 0.0f ? __frcp_rn(s) : 0.0f;
      const float PIf = 3.14159265358979f;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int f = lane + 32 * r;
        float k = 0.0f;
        if (s != 0.0f) k = fminf(fmaxf(round_exact_absmax(mag[r], s, inv), 0.0f), (float)((1 << bm) - 1));
        scode[warp][f] = (uint32_t)(int)k;
        // phase code: round((atan2 + pi) 2^bp / 2pi) mod 2^bp; fp32 with a guard band, fp64 near ties
        int pc;
        if (a[r] == 0.0f && bb[r] == 0.0f) {
          pc = (1 << bp) >> 1;  // angle 0
        } else {
          const float th = atan2f(bb[r], a[r]);
          const float v = (th + PIf) * ((float)(1 << bp) / (2.0f * PIf));
          const float fl = floorf(v + 0.5f);
          const float fr = v + 0.5f - fl;
          if (fr > 1e-3f && fr < 1.0f - 1e-3f) {
            pc = (int)fl;
          } else {
            const double PI = 3.141592653589793;
            const double th64 = atan2((double)bb[r], (double)a[r]);
            const double v64 = ((th64 + PI) * (double)(1 << bp)) / (2.0 * PI);
            pc = (int)floor(v64 + 0.5);
          }
          pc &= (1 << bp) - 1;
        }
        scode[warp][64 + f] = (uint32_t)pc;
      }
      __syncwarp();
      // pack: magnitude stream (64 x bm bits) then phase stream (64 x bp bits); 24 words
      const int nwords = (64 * (bm + bp)) / 32;
      for (int w = lane; w < nwords; w += 32) {
        uint32_t word = 0;
        const int b0 = w * 32;
        // magnitude elements overlapping [b0, b0+32)
        for (int e = b0 / bm; e < 64 && e * bm < b0 + 32; ++e) {
          const int off = e * bm - b0;
          const uint64_t v = (uint64_t)scode[warp][e];
          word |= (uint32_t)(off >= 0 ? (v << off) : (v >> (-off)));
        }
        const int pb = 64 * bm;
        if (b0 + 32 > pb) {
          const int lo = b0 > pb ? b0 - pb : 0;
          for (int e = lo / bp; e < 64 && pb + e * bp < b0 + 32; ++e) {
            const int off = pb + e * bp - b0;
            const uint64_t v = (uint64_t)scode[warp][64 + e];
            word |= (uint32_t)(off >= 0 ? (v << off) : (v >> (-off)));
          }
        }
        codes_w[w] = word;
      }
      if (lane == 0) S.scales[rix] = sh;
    } else {  // Cartesian: reals [a0, b0, a1, b1, ...], signed absmax int-bits, one scale
      const int bits = S.bits, half = 1 << (bits - 1);
      // largest |y| with first index (y index 2f for a, 2f+1 for b)
      float best = -1.0f, bestv = 0.0f;
      int besti = 1 << 30;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int f = lane + 32 * r;
        const float ya = fabsf(a[r]), yb = fabsf(bb[r]);
        if (ya > best || (ya == best && 2 * f < besti)) { best = ya; bestv = a[r]; besti = 2 * f; }
        if (yb > best || (yb == best && 2 * f + 1 < besti)) { best = yb; bestv = bb[r]; besti = 2 * f + 1; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const float ov = __shfl_xor_sync(0xffffffffu, bestv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, besti, o);
        if (ob > best || (ob == best && oi < besti)) { best = ob; bestv = ov; besti = oi; }
      }
      const __half dh = __float2half_rn(__fmul_rn(bestv, -1.0f / (float)half));
      const float d = __half2float(dh);
      const float inv = d != 0.0f ? __frcp_rn(d) : 0.0f;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int f = lane + 32 * r;
        float ka = 0.0f, kb = 0.0f;
        if (d != 0.0f) {
          ka = fminf(fmaxf(round_exact_absmax(a[r], d, inv), (float)(-half)), (float)(half - 1));
          kb = fminf(fmaxf(round_exact_absmax(bb[r], d, inv), (float)(-half)), (float)(half - 1));
        }
        scode[warp][2 * f] = (uint32_t)((int)ka + half);
        scode[warp][2 * f + 1] = (uint32_t)((int)kb + half);
      }
      __syncwarp();
      const int nwords = (128 * bits) / 32;
      for (int w = lane; w < nwords; w += 32) {
        uint32_t word = 0;
        const int b0 = w * 32;
        for (int e = b0 / bits; e < 128 && e * bits < b0 + 32; ++e) {
          const int off = e * bits - b0;
          const uint64_t v = (uint64_t)scode[warp][e];
          word |= (uint32_t)(off >= 0 ? (v << off) : (v >> (-off)));
        }
        codes_w[w] = word;
      }
      if (lane == 0) S.scales[rix] = dh;
    }
  }
  finish_append(L, n_new, total_ctas);
}

// ------------------------------------------------------------------------------------------
// Small appends (decode-time, a few hundred rows): one warp per row, V = D/32 contiguous values per
// lane, compact loops over runtime format parameters.  The unrolled thread-per-row kernel above is
// tens of thousands of straight-line instructions; with only a few warps resident its instruction
// fetch, not its arithmetic, sets the time, so short appends take this path instead.  Every
// decision is the same exact arithmetic as the row kernel (same helpers, same evaluation order:
// Hadamard stages in order, sign sums in channel order), so codes are identical.
constexpr int kSmallWarps = 4;

template <int V>
__global__ void __launch_bounds__(32 * kSmallWarps) append_small_kernel(LayerDev L, int side,
                                                                         const __half* __restrict__ src, int n_new,
                                                                         unsigned total_ctas) {
  const SideDev& S = L.s[side];
  constexpr int D = 32 * V;
  __shared__ uint32_t words[kSmallWarps][D / 4];  // packed row (up to 8 bits per value)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long R = (long long)L.B * L.Hkv * n_new;
  const long long row = (long long)blockIdx.x * kSmallWarps + warp;
  bool ok = row < R;
  int i = 0, u = 0, pos = 0, len_after = 0;
  if (ok) {
    i = (int)(row % n_new);
    u = (int)(row / n_new);
    const int len0 = L.seq_len[u / L.Hkv];
    pos = len0 + i;
    len_after = len0 + n_new;
    if (pos >= L.Tcap) {
      if (lane == 0 && i == 0) atomicOr(L.err, (unsigned)KVQ_ERRF_CAPACITY);
      ok = false;
    }
  }
  if (ok) {
    const __half* rp = src + ((long long)u * n_new + i) * D + lane * V;
    float x[V];
#pragma unroll
    for (int v = 0; v < V; ++v) x[v] = __half2float(rp[v]);
    if (in_anchor(L, pos, len_after)) {
      __half* ap = S.anchors + ((long long)u * L.anchor_rows + anchor_slot(L, pos)) * D + lane * V;
#pragma unroll
      for (int v = 0; v < V; ++v) ap[v] = rp[v];
    }
    if (S.chan_scale) {
      const __half* cp = S.chan + (u % L.Hkv) * D + lane * V;
#pragma unroll
      for (int v = 0; v < V; ++v) x[v] = __fdiv_rn(x[v], __half2float(cp[v]));
    }
    if (S.rot) {  // stages h = 1 .. n/2 over element index j = lane*V + v
      for (int h = 1; h < S.rot; h <<= 1) {
        if (h < V) {
#pragma unroll
          for (int v = 0; v < V; ++v)
            if ((v & h) == 0) {
              const float a = x[v], b = x[v + h];
              x[v] = __fadd_rn(a, b);
              x[v + h] = __fsub_rn(a, b);
            }
        } else {
          const int lm = h / V;
          const bool upper = (lane & lm) != 0;
#pragma unroll
          for (int v = 0; v < V; ++v) {
            const float o = __shfl_xor_sync(0xffffffffu, x[v], lm);
            x[v] = upper ? __fsub_rn(o, x[v]) : __fadd_rn(x[v], o);
          }
        }
      }
      const float rn = S.rot == 256 ? 0.0625f : __fdiv_rn(__fsqrt_rn(2.0f), 16.0f);
#pragma unroll
      for (int v = 0; v < V; ++v) x[v] = __fmul_rn(x[v], rn);
    }
    // groups: a lane holds ngl groups of epl values; a group spans lpg lanes
    const int g = S.group;
    const int epl = g < V ? g : V, ngl = V / epl, lpg = g / epl;
    const int fam = (S.fmt == KVQ_FMT_INT) ? (S.scale_mode == KVQ_SCALE_MINMAX ? FAM_MINMAX : FAM_ABSMAX)
                                           : (S.fmt == KVQ_FMT_NF4 ? FAM_NF4 : (S.fmt == KVQ_FMT_TERNARY ? FAM_TERNARY : FAM_SIGN));
    const int bits = fam == FAM_SIGN ? 1 : (fam == FAM_NF4 ? 4 : S.bits);
    const long long rix = (long long)u * L.Tcap + pos;
    for (int w = lane; w < D / 4; w += 32) words[warp][w] = 0u;
    __syncwarp();
    uint32_t code[V];
#pragma unroll
    for (int gl = 0; gl < V; ++gl) {
      if (gl >= ngl) break;
      const int v0 = gl * epl;
      // per-lane partial statistics over x[v0 .. v0+epl)
      float m = 0.0f, am = -1.0f, mn = INFINITY, mx = -INFINITY, sum = 0.0f;
      int mi = 1 << 30;
#pragma unroll
      for (int v = 0; v < V; ++v) {
        if (v < v0 || v >= v0 + epl) continue;
        const float a = fabsf(x[v]);
        if (a > am) { am = a; m = x[v]; mi = lane * V + v; }
        mn = fminf(mn, x[v]);
        mx = fmaxf(mx, x[v]);
      }
      if (fam == FAM_SIGN) {  // fp32 sum of |x| in channel order across the group's lanes
        const int base = lane - (lane % lpg);
        for (int k = 0; k < lpg; ++k) {
          if (lane == base + k) {
#pragma unroll
            for (int v = 0; v < V; ++v)
              if (v >= v0 && v < v0 + epl) sum = __fadd_rn(sum, fabsf(x[v]));
          }
          sum = __shfl_sync(0xffffffffu, sum, base + k);
        }
      }
      for (int o = 1; o < lpg; o <<= 1) {  // reductions inside the group (first index on ties)
        const float oam = __shfl_xor_sync(0xffffffffu, am, o), om = __shfl_xor_sync(0xffffffffu, m, o);
        const int omi = __shfl_xor_sync(0xffffffffu, mi, o);
        if (oam > am || (oam == am && omi < mi)) { am = oam; m = om; mi = omi; }
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      __half sh, zh = __float2half_rn(0.0f);
      float d = 0.0f, z = 0.0f, inv = 0.0f;
      int half = 0, top = 0;
      float t[15];
      if (fam == FAM_ABSMAX) {
        half = 1 << (bits - 1);
        sh = __float2half_rn(__fmul_rn(m, -1.0f / (float)half));
        d = __half2float(sh);
        inv = d != 0.0f ? __frcp_rn(d) : 0.0f;
      } else if (fam == FAM_MINMAX) {
        top = (1 << bits) - 1;
        zh = __float2half_rn(mn);
        sh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)top));
        z = __half2float(zh);
        d = __half2float(sh);
        inv = d != 0.0f ? __frcp_rn(d) : 0.0f;
      } else if (fam == FAM_SIGN) {
        sh = __float2half_rn(__fmul_rn(sum, 1.0f / (float)g));
      } else {
        sh = __float2half_rn(am);
        d = __half2float(sh);
        if (fam == FAM_NF4) {
#pragma unroll
          for (int k = 0; k < 15; ++k) t[k] = __fmul_rn(q_nf4_mid[k], d);
        }
      }
#pragma unroll
      for (int v = 0; v < V; ++v) {
        if (v < v0 || v >= v0 + epl) continue;
        uint32_t cd;
        if (fam == FAM_ABSMAX) {
          float k = 0.0f;
          if (d != 0.0f) k = fminf(fmaxf(round_exact_absmax(x[v], d, inv), (float)(-half)), (float)(half - 1));
          cd = (uint32_t)((int)k + half);
        } else if (fam == FAM_MINMAX) {
          float k = 0.0f;
          if (d != 0.0f) k = fminf(fmaxf(round_exact_minmax(x[v], z, d, inv), 0.0f), (float)top);
          cd = (uint32_t)(int)k;
        } else if (fam == FAM_NF4) {
          int cc = 7;
          if (d != 0.0f) {
            cc = 0;
#pragma unroll
            for (int k = 0; k < 15; ++k) cc += (x[v] >= t[k]) ? 1 : 0;
          }
          cd = (uint32_t)cc;
        } else if (fam == FAM_TERNARY) {
          const float hh = __fmul_rn(d, 0.5f);
          cd = d != 0.0f ? ((x[v] >= hh) ? 2u : ((x[v] < -hh) ? 0u : 1u)) : 1u;
        } else {
          cd = x[v] >= 0.0f ? 1u : 0u;
        }
        code[v] = cd;
      }
      // one scale (and zero point) per group, written by the group's first lane
      if (lane % lpg == 0) {
        const int gi = (lane * V + v0) / g;
        S.scales[rix * S.n_groups + gi] = sh;
        if (fam == FAM_MINMAX) S.zeros[rix * S.n_groups + gi] = zh;
      }
    }
    // pack: LSB-first bit stream (ternary: 5 trits per byte) into shared words, then store
    if (fam == FAM_TERNARY) {
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int j = lane * V + v, byte = j / 5, m5 = j % 5;
        const uint32_t p3 = m5 == 0 ? 1u : m5 == 1 ? 3u : m5 == 2 ? 9u : m5 == 3 ? 27u : 81u;
        atomicAdd(&words[warp][byte >> 2], (code[v] * p3) << (8 * (byte & 3)));
      }
      __syncwarp();
      uint8_t* op = S.codes + rix * S.row_bytes;
      for (int b = lane; b < S.row_bytes; b += 32) op[b] = (uint8_t)(words[warp][b >> 2] >> (8 * (b & 3)));
    } else {
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int bit = (lane * V + v) * bits;
        const uint64_t f = (uint64_t)code[v] << (bit & 31);
        atomicOr(&words[warp][bit >> 5], (uint32_t)f);
        if ((f >> 32) != 0ull) atomicOr(&words[warp][(bit >> 5) + 1], (uint32_t)(f >> 32));
      }
      __syncwarp();
      uint32_t* op = reinterpret_cast<uint32_t*>(S.codes + rix * S.row_bytes);
      for (int w = lane; w < S.row_bytes / 4; w += 32) op[w] = words[warp][w];
    }
  }
  finish_append(L, n_new, total_ctas);
}

// ------------------------------------------------------------------------------------------
// Dispatch.
typedef void (*RowKernel)(LayerDev, int, const __half*, int, unsigned);

static int fam_of(const SideDev& s) {
  switch (s.fmt) {
    case KVQ_FMT_INT: return s.scale_mode == KVQ_SCALE_MINMAX ? FAM_MINMAX : FAM_ABSMAX;
    case KVQ_FMT_NF4: return FAM_NF4;
    case KVQ_FMT_TERNARY: return FAM_TERNARY;
    case KVQ_FMT_SIGN: return FAM_SIGN;
    default: return -1;
  }
}

template <int DH, int TPR, int G>
static RowKernel pick_fam(int fam) {
  switch (fam) {
    case FAM_ABSMAX: return append_rows_kernel<DH, TPR, G, FAM_ABSMAX>;
    case FAM_MINMAX: return append_rows_kernel<DH, TPR, G, FAM_MINMAX>;
    case FAM_NF4: return append_rows_kernel<DH, TPR, G, FAM_NF4>;
    case FAM_TERNARY: return TPR == 1 ? append_rows_kernel<DH, 1, G, FAM_TERNARY> : nullptr;
    case FAM_SIGN: return append_rows_kernel<DH, TPR, G, FAM_SIGN>;
  }
  return nullptr;
}

template <int DH, int TPR>
static RowKernel pick_group(int g, int fam) {
  switch (g) {
    case 4: return pick_fam<DH, TPR, 4>(fam);
    case 8: return pick_fam<DH, TPR, 8>(fam);
    case 16: return pick_fam<DH, TPR, 16>(fam);
    case 32: return pick_fam<DH, TPR, 32>(fam);
    case 64: return pick_fam<DH, TPR, 64>(fam);
    case 128: return DH >= 128 ? pick_fam<128, TPR, 128>(fam) : nullptr;
  }
  return nullptr;
}

static RowKernel pick_row_kernel(int D, int g, int fam, int* tpr) {
  if (D == 64) { *tpr = 1; return pick_group<64, 1>(g, fam); }
  if (D == 128) { *tpr = 1; return pick_group<128, 1>(g, fam); }
  if (D == 256) { *tpr = 2; return pick_group<128, 2>(g, fam); }
  return nullptr;
}

bool append_supported(int D, const kvq_side& s) {
  if (s.format == KVQ_FMT_FP16) return true;
  if (s.format == KVQ_FMT_POLAR || s.format == KVQ_FMT_CART) return D == 128 && s.rotation == 0;
  SideDev sd{};
  sd.fmt = s.format;
  sd.scale_mode = s.scale_mode;
  const int fam = fam_of(sd);
  if (fam < 0) return false;
  if (s.rotation == 128 && D == 64) return false;
  if (s.rotation == 256 && D != 256) return false;
  int tpr = 0;
  return pick_row_kernel(D, s.group, fam, &tpr) != nullptr;
}

// fp16 side: plain row copy (16-byte vectors), plus anchors are irrelevant (rows already fp16).
__global__ void append_fp16_kernel(LayerDev L, int side, const __half* __restrict__ src, int n_new,
                                   unsigned total_ctas) {
  const SideDev& S = L.s[side];
  const int vec_per_row = L.D / 8;
  const long long R = (long long)L.B * L.Hkv * n_new;
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gt / vec_per_row;
  const int c = (int)(gt % vec_per_row);
  if (row < R) {
    const int i = (int)(row % n_new), u = (int)(row / n_new);
    const int pos = L.seq_len[u / L.Hkv] + i;
    if (pos < L.Tcap) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + ((long long)u * n_new + i) * L.D) + c);
      reinterpret_cast<uint4*>(S.codes + ((long long)u * L.Tcap + pos) * S.row_bytes)[c] = w;
      if (in_anchor(L, pos, L.seq_len[u / L.Hkv] + n_new))
        reinterpret_cast<uint4*>(S.anchors + ((long long)u * L.anchor_rows + anchor_slot(L, pos)) * L.D)[c] = w;
    } else if (c == 0 && i == 0) {
      atomicOr(L.err, (unsigned)KVQ_ERRF_CAPACITY);
    }
  }
  finish_append(L, n_new, total_ctas);
}

// Appends of at most this many rows (per side) use the warp-per-row kernel.
constexpr long long kSmallRows = 8192;

struct SidePlan {
  void (*kern)(LayerDev, int, const __half*, int, unsigned);
  unsigned blocks;
};

static SidePlan plan_side(const LayerDev& L, int side, int n_new) {
  const SideDev& S = L.s[side];
  const long long R = (long long)L.B * L.Hkv * n_new;
  SidePlan p{nullptr, 0};
  if (S.fmt == KVQ_FMT_FP16) {
    p.kern = append_fp16_kernel;
    p.blocks = (unsigned)((R * (L.D / 8) + 127) / 128);
  } else if (S.fmt == KVQ_FMT_POLAR || S.fmt == KVQ_FMT_CART) {
    p.kern = append_fft_kernel;
    p.blocks = (unsigned)((R + kFftWarps - 1) / kFftWarps);
  } else if (R <= kSmallRows) {
    p.kern = L.D == 64 ? append_small_kernel<2> : (L.D == 128 ? append_small_kernel<4> : append_small_kernel<8>);
    p.blocks = (unsigned)((R + kSmallWarps - 1) / kSmallWarps);
  } else {
    int tpr = 1;
    p.kern = pick_row_kernel(L.D, S.group, fam_of(S), &tpr);
    p.blocks = (unsigned)((R * tpr + 127) / 128);
  }
  return p;
}

cudaError_t launch_append(const LayerDev& L, const __half* k, const __half* v, int n_new, int /*max_len_before*/,
                          cudaStream_t st, int* launches) {
  const SidePlan pk = plan_side(L, 0, n_new), pv = plan_side(L, 1, n_new);
  if (!pk.kern || !pv.kern) return cudaErrorInvalidValue;
  const unsigned total = pk.blocks + pv.blocks;
  pk.kern<<<pk.blocks, 128, 0, st>>>(L, 0, k, n_new, total);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pv.kern<<<pv.blocks, 128, 0, st>>>(L, 1, v, n_new, total);
  if (launches) *launches = 2;
  return cudaGetLastError();
}

}  // namespace kvq
