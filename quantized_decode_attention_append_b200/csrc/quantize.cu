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
// row with the FFT in registers (butterflies across lanes by shuffles).  The per-row-slice
// quantization itself lives in quantize_row.cuh, shared with the fused append + decode kernel.
#include <math.h>
#include <stdio.h>

#include "kvq_internal.h"
#include "fft128.cuh"
#include "quantize_row.cuh"

namespace kvq {


__constant__ float q_tw_re[64];
__constant__ float q_tw_im[64];

cudaError_t upload_tables_quant(const HostTables& t) {
  cudaError_t e = upload_row_tables(t);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(q_tw_re, t.tw_re, sizeof(t.tw_re));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(q_tw_im, t.tw_im, sizeof(t.tw_im));
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
  const int ul = div_by(row, L.div_new);  // row / n_new
  const int i = row - ul * n_new;
  const int sl = div_by(ul, L.div_hkv), h = ul - sl * L.Hkv;
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
// seq_len before it takes its ticket, so the update cannot race a reader.  The listed sequences
// are distinct, so the last CTA's threads update them in parallel (one dependent global round
// trip instead of one per sequence).
__device__ __forceinline__ void finish_append(const LayerDev& L, int n_new, unsigned total_ctas) {
  __shared__ int last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(L.ticket, 1u) == total_ctas - 1;
  }
  __syncthreads();
  if (last) {
    __threadfence();  // the other CTAs' rows and seq_len reads happened before their tickets
    for (int s = threadIdx.x; s < L.app_n; s += blockDim.x) {
      const int b = L.app_ids ? L.app_ids[s] : s;
      if (b < 0 || b >= L.B) continue;
      const int nl = L.seq_len[b] + n_new;
      if (nl <= L.cap) L.seq_len[b] = nl;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      *L.ticket = 0u;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------------------------------------
// rFFT polar / Cartesian codecs (head_dim 128): one warp per row, the radix-2 DIT FFT in
// registers (fft128.cuh), in the evaluation order the format fixes.
constexpr int kFftWarps = 4;

// OR a field of `nb` (<= 32) bits at stream bit `bit` into the shared words w.
__device__ __forceinline__ void or_field(uint32_t* w, int bit, uint32_t v, int nb) {
  const int wi = bit >> 5, sh = bit & 31;
  atomicOr(w + wi, v << sh);
  if (sh + nb > 32) atomicOr(w + wi + 1, v >> (32 - sh));
}

__global__ void __launch_bounds__(128) append_fft_kernel(LayerDev L, int side, const __half* __restrict__ src,
                                                         int n_new, unsigned total_ctas) {
  const SideDev& S = L.s[side];
  __shared__ float twr[64], twi[64];
  __shared__ uint32_t sw[kFftWarps][32];  // the row's packed words (2 (bm + bp) or 4 bits of them)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int k = threadIdx.x; k < 64; k += blockDim.x) {  // divergent twiddle indices: shared, not constant
    twr[k] = q_tw_re[k];
    twi[k] = q_tw_im[k];
  }
  __syncthreads();
  const long long R = (long long)L.app_n * L.Hkv * n_new;
  const int brl = (int)(__brev((unsigned)lane) >> 27);  // bit-reversed lane (5 bits)
  for (long long row = (long long)blockIdx.x * kFftWarps + warp; row < R; row += (long long)gridDim.x * kFftWarps) {
    const RowDst dst = row_dst(L, (int)row, n_new);
    const bool ok = dst.err == 0;  // warp-uniform: one row per warp
    if (!ok) {
      if (dst.first && lane == 0) atomicOr(L.err, dst.err);
      continue;
    }
    const int pos = dst.pos, len_after = dst.len_after, u = dst.u;
    const __half* rp = src + (long long)input_row(L, (int)row, n_new) * 128;
    // element 4 lane + r of the bit-reversed input is x[bitrev7(4 lane + r)] = x[brl + 32 bitrev2(r)]
    float re[4], im[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = brl + 32 * (((r & 1) << 1) | (r >> 1));
      float v = __half2float(rp[j]);
      if (S.mean_sub) v = __fsub_rn(v, __half2float(S.kmean[(long long)u * 128 + j]));
      if (S.chan_scale) v = __fdiv_rn(v, __half2float(S.chan[(u % L.Hkv) * 128 + j]));
      re[r] = v;
      im[r] = 0.0f;
    }
    if (in_anchor(L, pos, len_after)) {
      __half* ap = S.anchors + ((long long)u * L.anchor_rows + anchor_slot(L, pos)) * 128;
#pragma unroll
      for (int r = 0; r < 4; ++r) ap[lane + 32 * r] = rp[lane + 32 * r];
    }
    fft128_warp(re, im, lane, twr, twi);
    // folded slots f = 2 lane, 2 lane + 1: slot f = X_f (slot 0: (X_0, X_64)); X_f is element f & 3
    // of lane f >> 2
    float a[2], bb[2];
    {
      const int srcl = lane >> 1;
      const bool odd = (lane & 1) != 0;
      const float r0 = __shfl_sync(0xffffffffu, re[0], srcl), r1 = __shfl_sync(0xffffffffu, re[1], srcl);
      const float r2 = __shfl_sync(0xffffffffu, re[2], srcl), r3 = __shfl_sync(0xffffffffu, re[3], srcl);
      const float i0 = __shfl_sync(0xffffffffu, im[0], srcl), i1 = __shfl_sync(0xffffffffu, im[1], srcl);
      const float i2 = __shfl_sync(0xffffffffu, im[2], srcl), i3 = __shfl_sync(0xffffffffu, im[3], srcl);
      const float x64 = __shfl_sync(0xffffffffu, re[0], 16);
      a[0] = odd ? r2 : r0;
      bb[0] = odd ? i2 : i0;
      a[1] = odd ? r3 : r1;
      bb[1] = odd ? i3 : i1;
      if (lane == 0) bb[0] = x64;
    }
    const long long rix = (long long)u * L.Tcap + pos;
    uint32_t* codes_w = reinterpret_cast<uint32_t*>(S.codes + rix * S.row_bytes);
    uint32_t* w = sw[warp];
    if (S.fmt == KVQ_FMT_POLAR) {
      const int bm = S.bits, bp = S.bits2, nwords = 2 * (bm + bp);
      if (lane < nwords) w[lane] = 0u;
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
      uint32_t mc = 0u, pcw = 0u;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float k = 0.0f;
        if (s != 0.0f) k = fminf(fmaxf(round_exact_absmax(mag[r], s, inv), 0.0f), (float)((1 << bm) - 1));
        mc |= (uint32_t)(int)k << (r * bm);
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
        pcw |= (uint32_t)pc << (r * bp);
      }
      __syncwarp();
      // magnitude stream (64 x bm bits), then phase stream (64 x bp bits), slots in order
      or_field(w, 2 * bm * lane, mc, 2 * bm);
      or_field(w, 64 * bm + 2 * bp * lane, pcw, 2 * bp);
      __syncwarp();
      if (lane < nwords) codes_w[lane] = w[lane];
      if (lane == 0) S.scales[rix] = sh;
    } else {  // Cartesian: reals [a0, b0, a1, b1, ...], signed absmax int-bits, one scale
      const int bits = S.bits, half = 1 << (bits - 1), nwords = 4 * bits;
      if (lane < nwords) w[lane] = 0u;
      // largest |y| with first index (y index 2f for a, 2f + 1 for b; this lane: 4 lane .. 4 lane + 3)
      float best = -1.0f, bestv = 0.0f;
      int besti = 1 << 30;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int f = 2 * lane + r;
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
      uint32_t cw = 0u;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float ka = 0.0f, kb = 0.0f;
        if (d != 0.0f) {
          ka = fminf(fmaxf(round_exact_absmax(a[r], d, inv), (float)(-half)), (float)(half - 1));
          kb = fminf(fmaxf(round_exact_absmax(bb[r], d, inv), (float)(-half)), (float)(half - 1));
        }
        cw |= (uint32_t)((int)ka + half) << (2 * r * bits);
        cw |= (uint32_t)((int)kb + half) << ((2 * r + 1) * bits);
      }
      __syncwarp();
      or_field(w, 4 * bits * lane, cw, 4 * bits);
      __syncwarp();
      if (lane < nwords) codes_w[lane] = w[lane];
      if (lane == 0) S.scales[rix] = dh;
    }
    __syncwarp();  // sw is reused by this warp's next row
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
    quantize_slice<FAM, G, BITS, EXT>(L, S, cw, ok, u, pos, len_after);
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
constexpr long long kMaxAppendCtas = 148 * 16;

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
