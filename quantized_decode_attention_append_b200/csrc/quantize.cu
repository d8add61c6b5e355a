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
// Work mapping: head_dim/32 lanes per row, 32 contiguous values per lane, so a warp covers
// 32*32/head_dim rows and the grid strides over rows.  The Hadamard stages run in-lane, then by
// xor-shuffles across the row's lanes; group statistics reduce inside the group's lanes; codes are
// packed at compile-time widths into 32-bit words.  The polar/Cartesian codecs run one warp per
// row with the FFT in shared memory.
#include <math.h>
#include <stdio.h>

#include "kvq_internal.h"

namespace kvq {

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
// Bitwise choice: bits of a where m is set, of b elsewhere (one 3-input logic op).
__device__ __forceinline__ uint32_t bsel(uint32_t m, uint32_t a, uint32_t b) { return (a & m) | (b & ~m); }

__constant__ float q_nf4_mid[15];
__constant__ float q_tw_re[64];
__constant__ float q_tw_im[64];
__constant__ float q_lloyd_mid[3][15];

cudaError_t upload_tables_quant(const HostTables& t) {
  cudaError_t e = cudaMemcpyToSymbol(q_nf4_mid, t.nf4_mid, sizeof(t.nf4_mid));
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(q_lloyd_mid, t.lloyd_mid, sizeof(t.lloyd_mid));
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(q_tw_re, t.tw_re, sizeof(t.tw_re));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(q_tw_im, t.tw_im, sizeof(t.tw_im));
}

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

// Where appended row `row` lands.  Input rows are ordered (listed sequence, kv-head, token);
// the listed sequence is L.app_ids[s] (or s when the list is null).  A sequence whose rows would
// pass the capacity, or an id outside [0, B), gets none of its rows written; `err` names why and
// `first` marks the row (token 0 of kv-head 0) that reports it.
struct RowDst {
  int u, pos, len_after;
  unsigned err;
  bool first;
};
// (rows per call < 2^31, checked on the host, so 32-bit index arithmetic suffices)
__device__ __forceinline__ RowDst row_dst(const LayerDev& L, int row, int n_new) {
  RowDst d{0, 0, 0, 0u, false};
  const int ul = row / n_new;
  const int i = row - ul * n_new;
  const int sl = ul / L.Hkv, h = ul - sl * L.Hkv;
  const int b = L.app_ids ? L.app_ids[sl] : sl;
  d.first = i == 0 && h == 0;
  if (b < 0 || b >= L.B) {
    d.err = KVQ_ERRF_SEQ_ID;
    return d;
  }
  const int len0 = L.seq_len[b];
  if (len0 + n_new > L.cap) {
    d.err = KVQ_ERRF_CAPACITY;
    return d;
  }
  d.u = b * L.Hkv + h;
  d.pos = len0 + i;
  d.len_after = len0 + n_new;
  return d;
}

// Completion ticket: the last CTA of an append (over all its launches) advances the lengths of
// the listed sequences that had room (the same test every row of theirs took).  Every CTA read
// seq_len before it takes its ticket, so the update cannot race a reader.
__device__ __forceinline__ void finish_append(const LayerDev& L, int n_new, unsigned total_ctas) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned t = atomicAdd(L.ticket, 1u);
    if (t == total_ctas - 1) {
      for (int s = 0; s < L.app_n; ++s) {
        const int b = L.app_ids ? L.app_ids[s] : s;
        if (b < 0 || b >= L.B) continue;
        const int nl = L.seq_len[b] + n_new;
        if (nl <= L.cap) L.seq_len[b] = nl;
      }
      *L.ticket = 0u;
      __threadfence();
    }
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
  const long long R = (long long)L.app_n * L.Hkv * n_new;
  for (long long row = (long long)blockIdx.x * kFftWarps + warp; row < R; row += (long long)gridDim.x * kFftWarps) {
  const RowDst dst = row_dst(L, (int)row, n_new);
  const bool ok = dst.err == 0;
  const int pos = dst.pos, len_after = dst.len_after, u = dst.u;
  if (!ok && dst.first && lane == 0) atomicOr(L.err, dst.err);
  if (ok) {
    const __half* rp = src + (long long)input_row(L, (int)row, n_new) * 128;
    float* re = sre[warp];
    float* im = sim[warp];
    for (int j = lane; j < 128; j += 32) {
      float v = __half2float(rp[j]);
      if (S.mean_sub) v = __fsub_rn(v, __half2float(S.kmean[(long long)u * 128 + j]));
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
  __syncwarp();  // scode/sre/sim are reused by this warp's next row
  }
  finish_append(L, n_new, total_ctas);
}

// ------------------------------------------------------------------------------------------
// Sorted groups: one warp per row, the row in shared memory.  A channel's rank (its position when
// the row is sorted descending, equal values in channel order) is counted against every other
// channel; values move to their ranks; consecutive groups of the sorted row take the min-max grid;
// codes (sorted order) then ranks (channel order) are packed LSB-first.  Pre-transforms run first,
// the Hadamard stages in the same butterfly order as the row kernel.
constexpr int kSortWarps = 4;

__global__ void __launch_bounds__(128) append_sorted_kernel(LayerDev L, int side, const __half* __restrict__ src,
                                                            int n_new, unsigned total_ctas) {
  const SideDev& S = L.s[side];
  const int D = L.D, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ float sx[kSortWarps][256], sv[kSortWarps][256];
  __shared__ uint32_t scode[kSortWarps][256], srank[kSortWarps][256];
  const long long R = (long long)L.app_n * L.Hkv * n_new;
  const int G = S.group, bits = S.bits, rb = 32 - __clz(D - 1), ng = D / G, top = (1 << bits) - 1;
  for (long long row = (long long)blockIdx.x * kSortWarps + warp; row < R; row += (long long)gridDim.x * kSortWarps) {
    const RowDst dst = row_dst(L, (int)row, n_new);
    if (dst.err) {  // warp-uniform: the whole warp holds this row
      if (dst.first && lane == 0) atomicOr(L.err, dst.err);
      continue;
    }
    const __half* rp = src + (long long)input_row(L, (int)row, n_new) * D;
    float* x = sx[warp];
    for (int j = lane; j < D; j += 32) {
      float v = __half2float(rp[j]);
      if (S.mean_sub) v = __fsub_rn(v, __half2float(S.kmean[(long long)dst.u * D + j]));
      if (S.chan_scale) v = __fdiv_rn(v, __half2float(S.chan[(dst.u % L.Hkv) * D + j]));
      x[j] = v;
    }
    if (in_anchor(L, dst.pos, dst.len_after)) {  // fp16 anchors (int anchors are refused on the host)
      __half* ap = S.anchors + ((long long)dst.u * L.anchor_rows + anchor_slot(L, dst.pos)) * D;
      for (int j = lane; j < D; j += 32) ap[j] = rp[j];
    }
    __syncwarp();
    if (S.rot) {  // stages h = 1 .. rot/2: (x_i, x_i+h) <- (x_i + x_i+h, x_i - x_i+h), bit h of i clear
      for (int h = 1; h < S.rot; h <<= 1) {
        for (int p = lane; p < D / 2; p += 32) {
          const int i = ((p >> (__ffs(h) - 1)) << __ffs(h)) | (p & (h - 1));
          const float a = x[i], b = x[i + h];
          x[i] = __fadd_rn(a, b);
          x[i + h] = __fsub_rn(a, b);
        }
        __syncwarp();
      }
      const float rn = S.rot == 256 ? 0.0625f : __fdiv_rn(__fsqrt_rn(2.0f), 16.0f);
      for (int j = lane; j < D; j += 32) x[j] = __fmul_rn(x[j], rn);
      __syncwarp();
    }
    float* v = sv[warp];
    for (int j = lane; j < D; j += 32) {
      const float xj = x[j];
      int r = 0;
      for (int k = 0; k < D; ++k) {
        const float xk = x[k];
        r += (xk > xj || (xk == xj && k < j)) ? 1 : 0;
      }
      srank[warp][j] = (uint32_t)r;
      v[r] = xj;
    }
    __syncwarp();
    const long long rix = (long long)dst.u * L.Tcap + dst.pos;
    for (int gi = lane; gi < ng; gi += 32) {  // sorted descending: the group's max leads, its min ends it
      const float* gv = v + gi * G;
      const float mx = gv[0];
      float mn = gv[G - 1];
      if (mn == 0.0f) {  // a zero minimum is -0 iff the group holds a -0 (the min-max rule)
        bool negz = false;
        for (int e = 0; e < G; ++e) negz |= __float_as_uint(gv[e]) == 0x80000000u;
        mn = negz ? -0.0f : 0.0f;
      }
      const __half zh = __float2half_rn(mn), sh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), (float)top));
      const float z = __half2float(zh), d = __half2float(sh), inv = d != 0.0f ? __frcp_rn(d) : 0.0f;
      for (int e = 0; e < G; ++e) {
        const float k = d != 0.0f ? fminf(fmaxf(round_exact_minmax(gv[e], z, d, inv), 0.0f), (float)top) : 0.0f;
        scode[warp][gi * G + e] = (uint32_t)(int)k;
      }
      S.scales[rix * ng + gi] = sh;
      S.zeros[rix * ng + gi] = zh;
    }
    __syncwarp();
    uint32_t* cw = reinterpret_cast<uint32_t*>(S.codes + rix * S.row_bytes);
    const int nwords = D * (bits + rb) / 32, cbits = D * bits;
    for (int w = lane; w < nwords; w += 32) {
      uint32_t word = 0u;
      const int b0 = w * 32;
      for (int e = b0 / bits; e < D && e * bits < b0 + 32; ++e) {
        const int off = e * bits - b0;
        const uint64_t c = scode[warp][e];
        word |= (uint32_t)(off >= 0 ? (c << off) : (c >> (-off)));
      }
      if (b0 + 32 > cbits) {
        const int lo = b0 > cbits ? b0 - cbits : 0;
        for (int e = lo / rb; e < D && cbits + e * rb < b0 + 32; ++e) {
          const int off = cbits + e * rb - b0;
          const uint64_t r = srank[warp][e];
          word |= (uint32_t)(off >= 0 ? (r << off) : (r >> (-off)));
        }
      }
      cw[w] = word;
    }
    __syncwarp();  // sx/sv/scode/srank are reused by this warp's next row
  }
  finish_append(L, n_new, total_ctas);
}

// ------------------------------------------------------------------------------------------
// Row formats (int, NF4, ternary, sign): each row is split over D/32 lanes, each lane holding 32
// contiguous values in registers; a warp covers 32/(D/32) consecutive rows, so loads are
// coalesced 64-byte pieces and a lane's codes fill whole 32-bit words of the packed row.  The
// kernel is grid-stride (a few hundred CTAs, so only a few hundred completion tickets) and is
// specialised on the grid family and group size only, which keeps it small.  Hadamard stages run
// in-lane (h < 32) and by xor-shuffles between the row's lanes (h >= 32); groups of 64/128 reduce
// across 2/4 lanes.  Evaluation order follows the format: Hadamard stages h = 1, 2, ..., n/2,
// sign sums in channel order.
constexpr int kRowThreads = 128;

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

// Rows of one side over blocks bid = 0 .. nblk - 1 (grid-stride).  EXT = false compiles out the key
// mean, int anchors and head-group input mapping (the fused K+V kernel's common case), which
// keeps the hot instances at 128 registers; callers needing them use the EXT instances.
template <int FAM, int G, int BITS = 0, bool EXT = true>
__device__ __forceinline__ void rows_body(const LayerDev& L, int side, const __half* __restrict__ src, int n_new,
                                          int bid, int nblk) {
  const SideDev& S = L.s[side];
  const int D = L.D, lpr = D >> 5;                    // lanes per row
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NW = kRowThreads / 32;
  const int rpw = 32 / lpr;                           // rows per warp
  const int li = lane % lpr;                          // this lane's 32-value slice of its row
  const int R = L.app_n * L.Hkv * n_new;              // < 2^31 (checked on the host)
  constexpr int LG = G > 32 ? G / 32 : 1;             // lanes per group
  constexpr int GPL = G > 32 ? 1 : 32 / G;            // groups per lane
  // code bits: fixed by the family, by the instance (BITS > 0), or read from the side
  const int bits = FAM == FAM_SIGN ? 1 : (FAM == FAM_NF4 ? 4 : (BITS > 0 ? BITS : S.bits));
  // the grid sees the fp16 input itself (no key mean, channel scale or rotation in between)
  const bool raw = !S.rot && !S.chan_scale && !(EXT && S.mean_sub);

  // The next pass's input slice is loaded before this pass's arithmetic, so each warp keeps its
  // loads in flight while it computes (the arithmetic per row is long).
  const int stride = nblk * NW * rpw;
  uint4 nx[4];
  {
    const long long r0 = (long long)(bid * NW + warp) * rpw + lane / lpr;
    if (r0 < R) {
      const uint4* p = reinterpret_cast<const uint4*>(src + (long long)(EXT ? input_row(L, (int)r0, n_new) : (int)r0) * D +
                                                      li * 32);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) nx[c4] = __ldg(p + c4);
    }
  }
  for (int rb = (bid * NW + warp) * rpw; rb < R; rb += stride) {
    const int row = rb + lane / lpr;
    uint4 cw[4];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) cw[c4] = nx[c4];
    {
      const long long rn = (long long)row + stride;
      if (rn < R) {
        const uint4* p = reinterpret_cast<const uint4*>(src + (long long)(EXT ? input_row(L, (int)rn, n_new) : (int)rn) * D +
                                                        li * 32);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) nx[c4] = __ldg(p + c4);
      }
    }
    int u = 0, pos = 0, len_after = 0;
    bool ok = row < R;
    if (ok) {
      const RowDst d = row_dst(L, row, n_new);
      if (d.err && d.first && li == 0) atomicOr(L.err, d.err);
      ok = d.err == 0;
      u = d.u;
      pos = d.pos;
      len_after = d.len_after;
    }
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
}

template <int FAM, int G>
__global__ void __launch_bounds__(kRowThreads) append_rows_kernel(LayerDev L, int side, const __half* __restrict__ src,
                                                                  int n_new, unsigned total_ctas) {
  rows_body<FAM, G>(L, side, src, n_new, blockIdx.x, gridDim.x);
  finish_append(L, n_new, total_ctas);
}

// K and V in one launch: blocks [0, kblocks) take the K rows, the rest the V rows.
template <int FK, int GK, int BK, int FV, int GV, int BV>
__global__ void __launch_bounds__(kRowThreads) append_kv_kernel(LayerDev L, const __half* __restrict__ k,
                                                                const __half* __restrict__ v, int n_new,
                                                                unsigned kblocks, unsigned total_ctas) {
  if (blockIdx.x < kblocks) rows_body<FK, GK, BK, false>(L, 0, k, n_new, blockIdx.x, kblocks);
  else rows_body<FV, GV, BV, false>(L, 1, v, n_new, blockIdx.x - kblocks, gridDim.x - kblocks);
  finish_append(L, n_new, total_ctas);
}

// ------------------------------------------------------------------------------------------
// Dispatch.
typedef void (*RowKernel)(LayerDev, int, const __half*, int, unsigned);

static int fam_of(const SideDev& s) {
  switch (s.fmt) {
    case KVQ_FMT_INT:
      return s.scale_mode == KVQ_SCALE_MINMAX ? FAM_MINMAX : (s.scale_mode == KVQ_SCALE_SYMMETRIC ? FAM_SYM : FAM_ABSMAX);
    case KVQ_FMT_NF4: return FAM_NF4;
    case KVQ_FMT_TERNARY: return FAM_TERNARY;
    case KVQ_FMT_LLOYD: return FAM_LLOYD;
    default: return FAM_SIGN;
  }
}

template <int FAM>
static RowKernel pick_rows_g(int g) {
  switch (g) {
    case 4: return append_rows_kernel<FAM, 4>;
    case 8: return append_rows_kernel<FAM, 8>;
    case 16: return append_rows_kernel<FAM, 16>;
    case 32: return append_rows_kernel<FAM, 32>;
    case 64: return append_rows_kernel<FAM, 64>;
    case 128: return append_rows_kernel<FAM, 128>;
  }
  return nullptr;
}

static RowKernel pick_rows_kernel(int fam, int g) {
  switch (fam) {
    case FAM_ABSMAX: return pick_rows_g<FAM_ABSMAX>(g);
    case FAM_MINMAX: return pick_rows_g<FAM_MINMAX>(g);
    case FAM_NF4: return pick_rows_g<FAM_NF4>(g);
    case FAM_TERNARY: return pick_rows_g<FAM_TERNARY>(g);
    case FAM_SIGN: return pick_rows_g<FAM_SIGN>(g);
    case FAM_SYM: return pick_rows_g<FAM_SYM>(g);
    case FAM_LLOYD: return pick_rows_g<FAM_LLOYD>(g);
  }
  return nullptr;
}

bool append_supported(int D, const kvq_side& s) {
  if (s.format == KVQ_FMT_FP16) return true;
  if (s.format == KVQ_FMT_POLAR || s.format == KVQ_FMT_CART) return D == 128 && s.rotation == 0;
  if (s.format == KVQ_FMT_SORTED)
    return (D == 64 || D == 128 || D == 256) && !(s.rotation > D || (s.rotation && D % s.rotation)) && s.group >= 4 &&
           s.group <= D;
  if (s.format != KVQ_FMT_INT && s.format != KVQ_FMT_NF4 && s.format != KVQ_FMT_TERNARY && s.format != KVQ_FMT_SIGN &&
      s.format != KVQ_FMT_LLOYD)
    return false;
  if (D != 64 && D != 128 && D != 256) return false;
  if (s.rotation > D || (s.rotation && D % s.rotation)) return false;
  return s.group >= 4 && s.group <= 128 && s.group <= D;
}

// fp16 side: plain row copy (16-byte vectors), plus anchors are irrelevant (rows already fp16).
__global__ void append_fp16_kernel(LayerDev L, int side, const __half* __restrict__ src, int n_new,
                                   unsigned total_ctas) {
  const SideDev& S = L.s[side];
  const int vec_per_row = L.D / 8;
  const long long R = (long long)L.app_n * L.Hkv * n_new;
  for (long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x; gt < R * vec_per_row;
       gt += (long long)gridDim.x * blockDim.x) {
  const long long row = gt / vec_per_row;
  const int c = (int)(gt % vec_per_row);
  const RowDst d = row_dst(L, (int)row, n_new);
  if (d.err == 0) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + (long long)input_row(L, (int)row, n_new) * L.D) + c);
    reinterpret_cast<uint4*>(S.codes + ((long long)d.u * L.Tcap + d.pos) * S.row_bytes)[c] = w;
    if (in_anchor(L, d.pos, d.len_after))
      reinterpret_cast<uint4*>(S.anchors + ((long long)d.u * L.anchor_rows + anchor_slot(L, d.pos)) * L.D)[c] = w;
  } else if (c == 0 && d.first) {
    atomicOr(L.err, d.err);
  }
  }
  finish_append(L, n_new, total_ctas);
}

// Key means (K with mean_sub) of the listed sequences this append starts (stored length 0): one
// CTA per (listed sequence, kv-head).  Each fp16 key times 2^24 is an integer, so the sum is exact
// in int64 in any order; the mean is rounded once through fp64 to fp16.  Runs before the append
// kernels on the same stream, which then subtract it.
constexpr int kMeanThreads = 256;

__global__ void __launch_bounds__(kMeanThreads) key_mean_kernel(LayerDev L, const __half* __restrict__ k, int n_new) {
  const int ul = blockIdx.x, sl = ul / L.Hkv, h = ul - sl * L.Hkv;
  const int b = L.app_ids ? L.app_ids[sl] : sl;
  if (b < 0 || b >= L.B || L.seq_len[b] != 0) return;  // not this sequence's first append
  const int D = L.D, j = threadIdx.x % D, r0 = threadIdx.x / D, nr = kMeanThreads / D;
  const __half* src = k + (long long)input_row(L, ul * n_new, n_new) * D;
  long long acc = 0;
  for (int i = r0; i < n_new; i += nr) acc += __float2ll_rn(__fmul_rn(__half2float(src[(long long)i * D + j]), 16777216.0f));
  __shared__ long long part[kMeanThreads];
  part[threadIdx.x] = acc;
  __syncthreads();
  if (r0 == 0) {
    long long S = 0;
    for (int r = 0; r < nr; ++r) S += part[r * D + j];
    const double m = __dmul_rn(__ddiv_rn(__ll2double_rn(S), (double)n_new), 5.9604644775390625e-08);  // x 2^-24
    L.s[0].kmean[((long long)b * L.Hkv + h) * D + j] = __double2half(m);
  }
}

cudaError_t launch_key_mean(const LayerDev& L, const __half* k, int n_new, cudaStream_t st) {
  key_mean_kernel<<<L.app_n * L.Hkv, kMeanThreads, 0, st>>>(L, k, n_new);
  return cudaGetLastError();
}

// Grid cap of the grid-stride append kernels (148 SMs x 8 CTAs of 8 warps).
constexpr long long kMaxAppendCtas = 148 * 8;

struct SidePlan {
  void (*kern)(LayerDev, int, const __half*, int, unsigned);
  unsigned blocks, threads;
};

static SidePlan plan_side(const LayerDev& L, int side, int n_new) {
  const SideDev& S = L.s[side];
  const long long R = (long long)L.app_n * L.Hkv * n_new;
  SidePlan p{nullptr, 0, 128};
  if (S.fmt == KVQ_FMT_FP16) {
    p.kern = append_fp16_kernel;
    const long long want = (R * (L.D / 8) + 127) / 128;
    p.blocks = (unsigned)(want < kMaxAppendCtas ? want : kMaxAppendCtas);
  } else if (S.fmt == KVQ_FMT_SORTED) {
    p.kern = append_sorted_kernel;
    const long long want = (R + kSortWarps - 1) / kSortWarps;
    p.blocks = (unsigned)(want < kMaxAppendCtas ? want : kMaxAppendCtas);
  } else if (S.fmt == KVQ_FMT_POLAR || S.fmt == KVQ_FMT_CART) {
    p.kern = append_fft_kernel;
    const long long want = (R + kFftWarps - 1) / kFftWarps;
    p.blocks = (unsigned)(want < kMaxAppendCtas ? want : kMaxAppendCtas);
  } else {
    p.kern = pick_rows_kernel(fam_of(S), S.group);
    const long long rpc = (long long)(kRowThreads / 32) * (32 / (L.D / 32));  // rows per CTA pass
    const long long want = (R + rpc - 1) / rpc;
    p.blocks = (unsigned)(want < kMaxAppendCtas ? want : kMaxAppendCtas);
    p.threads = kRowThreads;
  }
  return p;
}

typedef void (*KvKernel)(LayerDev, const __half*, const __half*, int, unsigned, unsigned);

// The (K, V) format pairs that have a single-launch append kernel.
static KvKernel pick_kv_kernel(const LayerDev& L) {
  const SideDev& K = L.s[0];
  const SideDev& V = L.s[1];
  if (K.fmt == KVQ_FMT_FP16 || V.fmt == KVQ_FMT_FP16 || K.fmt == KVQ_FMT_POLAR || K.fmt == KVQ_FMT_CART ||
      V.fmt == KVQ_FMT_POLAR || V.fmt == KVQ_FMT_CART || K.fmt == KVQ_FMT_SORTED || V.fmt == KVQ_FMT_SORTED)
    return nullptr;
  if (K.mean_sub || L.anchor_bits != 16 || L.Hkv != L.Hkv_all) return nullptr;  // the fused kernel has no extras
  const int fk = fam_of(K), fv = fam_of(V), gk = K.group, gv = V.group;
  // bits 0: fixed by the family (NF4, ternary, sign)
#define KVQ_KV(FK_, GK_, BK_, FV_, GV_, BV_)                                                      \
  if (fk == FK_ && gk == GK_ && (BK_ == 0 || K.bits == BK_) && fv == FV_ && gv == GV_ &&        \
      (BV_ == 0 || V.bits == BV_))                                                               \
    return append_kv_kernel<FK_, GK_, BK_, FV_, GV_, BV_>;
  KVQ_KV(FAM_NF4, 64, 0, FAM_ABSMAX, 64, 4)
  KVQ_KV(FAM_ABSMAX, 64, 4, FAM_ABSMAX, 64, 4)
  KVQ_KV(FAM_ABSMAX, 128, 4, FAM_ABSMAX, 128, 2)
  KVQ_KV(FAM_ABSMAX, 128, 4, FAM_ABSMAX, 128, 3)
  KVQ_KV(FAM_ABSMAX, 128, 4, FAM_ABSMAX, 128, 4)
  KVQ_KV(FAM_ABSMAX, 32, 4, FAM_ABSMAX, 32, 4)
  KVQ_KV(FAM_MINMAX, 32, 3, FAM_MINMAX, 32, 3)
  KVQ_KV(FAM_MINMAX, 32, 4, FAM_MINMAX, 32, 4)
  KVQ_KV(FAM_TERNARY, 8, 0, FAM_TERNARY, 8, 0)
  KVQ_KV(FAM_SIGN, 4, 0, FAM_SIGN, 4, 0)
#undef KVQ_KV
  return nullptr;
}

unsigned append_ctas(const LayerDev& L, int n_new) {
  return plan_side(L, 0, n_new).blocks + plan_side(L, 1, n_new).blocks;
}

cudaError_t launch_append(const LayerDev& L, const __half* k, const __half* v, int n_new, unsigned total,
                          cudaStream_t st, int* launches) {
  const SidePlan pk = plan_side(L, 0, n_new), pv = plan_side(L, 1, n_new);
  if (!pk.kern || !pv.kern) return cudaErrorInvalidValue;
  if (KvKernel kv = pick_kv_kernel(L)) {
    kv<<<pk.blocks + pv.blocks, kRowThreads, 0, st>>>(L, k, v, n_new, pk.blocks, total);
    if (launches) *launches = 1;
    return cudaGetLastError();
  }
  pk.kern<<<pk.blocks, pk.threads, 0, st>>>(L, 0, k, n_new, total);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pv.kern<<<pv.blocks, pv.threads, 0, st>>>(L, 1, v, n_new, total);
  if (launches) *launches = 2;
  return cudaGetLastError();
}

}  // namespace kvq
