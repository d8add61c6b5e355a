// kvq_decode_attention: split-K flash decode over the packed cache, then a merge kernel.
//
// Sources (page title, section): attention over the dequantized cache and the proxy-query setup
// ("E21W" "What I tested": attention output, KL, causal proxy queries), the quantized-cache
// simulation it stands in for ("E22L" "What I tested": keys and values quantized on entry to
// the cache, the rotated variant being a 256-wide Hadamard), fp16 anchors ("Fourier Magnitude KV Cache
// Quantization" post 6 "Corrected semantics").
//
// Pass 1 (one CTA per query x kv-head x split): the query group is transformed once into the
// stored domain of K (q' = H(c . q), or the rFFT adjoint for polar/Cartesian K, pre-multiplied by
// sm_scale * log2 e), then each tile of keys is scored against q' without reconstructing K,
// online softmax runs in the log2 domain, and sum p * v is accumulated in V's stored domain.
// Anchor rows (fp16, original domain) get their own split with the raw query.
// Pass 2 (merge): log-sum-exp merge of the splits, V's inverse transform (Hadamard or inverse
// DFT) applied once to the merged vector, anchors added, normalised.
#include <math.h>

#include <mutex>

#include <vector>

#include "decode_common.cuh"
#include "fft128.cuh"
#include "kvq_internal.h"
#include "quantize_row.cuh"

namespace kvq {

__constant__ float d_nf4[16];
__constant__ float d_tw_re[64];
__constant__ float d_tw_im[64];
__constant__ float d_ph_cos[512];
__constant__ float d_ph_sin[512];
__constant__ float d_lloyd[3][16];

// The phase levels' (cos, sin) in the polar decode's layout: for phase width bp, level k, copy r
// at entry ((2^bp - 2) + k) x 16 + r (16 copies, one per shared-memory bank pair once staged).
__device__ __align__(16) float2 g_ph_rep[510 * 16];
// W_128^k = exp(-2 pi i k / 128), k < 64, as (re[k], im[k]) in global memory: the register FFT's
// lanes read divergent indices, which constant memory would serialise.
__device__ float g_tw[2][64];

cudaError_t upload_tables_decode(const HostTables& t) {
  cudaError_t e;
  {
    std::vector<float2> rep(510 * 16);
    for (int k = 0; k < 510; ++k)
      for (int r = 0; r < 16; ++r) rep[k * 16 + r] = make_float2(t.ph_cos[k], t.ph_sin[k]);
    if ((e = cudaMemcpyToSymbol(g_ph_rep, rep.data(), rep.size() * sizeof(float2))) != cudaSuccess) return e;
    float tw[2][64];
    for (int k = 0; k < 64; ++k) {
      tw[0][k] = t.tw_re[k];
      tw[1][k] = t.tw_im[k];
    }
    if ((e = cudaMemcpyToSymbol(g_tw, tw, sizeof(tw))) != cudaSuccess) return e;
  }
  if ((e = upload_row_tables(t)) != cudaSuccess) return e;  // thresholds of the fused append
  if ((e = cudaMemcpyToSymbol(d_nf4, t.nf4, sizeof(t.nf4))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_tw_re, t.tw_re, sizeof(t.tw_re))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_tw_im, t.tw_im, sizeof(t.tw_im))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_ph_cos, t.ph_cos, sizeof(t.ph_cos))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(d_lloyd, t.lloyd, sizeof(t.lloyd))) != cudaSuccess) return e;
  return cudaMemcpyToSymbol(d_ph_sin, t.ph_sin, sizeof(t.ph_sin));
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kGenThreads = 128;
constexpr int kGenTile = 128;
constexpr int kMaxG = 8;  // GQA group size handled by the generic kernel

struct QueryRange {
  int seq, kv_len, len;
  int qa, qb;  // quantized token range
  int aa, ab;  // anchored token range
  int fresh;   // fused append + decode: rows [len - fresh, len) are this call's new rows
};

// FUSED: honour a fused append + decode call (L.fuse_n); the plain decode instances compile it out.
template <bool FUSED = true>
__device__ __forceinline__ QueryRange query_range(const LayerDev& L, int qi, const int* seq_ids, const int* kv_len) {
  QueryRange r;
  r.seq = seq_ids ? seq_ids[qi] : qi;
  if (r.seq < 0 || r.seq >= L.B) {  // caller error: attend nothing, report it
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) atomicOr(L.err, (unsigned)KVQ_ERRF_SEQ_ID);
    r.seq = 0;
    r.len = 0;
    r.kv_len = 0;
    r.qa = r.qb = r.aa = r.ab = 0;
    r.fresh = 0;
    return r;
  }
  r.len = L.seq_len[r.seq];
  r.fresh = 0;
  if (FUSED && L.fuse_n > 0) {  // the stored length before the rows this call appends
    if (r.len + L.fuse_n <= L.cap) {
      r.fresh = L.fuse_n;
      r.len += L.fuse_n;
    } else if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) {
      atomicOr(L.err, (unsigned)KVQ_ERRF_CAPACITY);  // no room: none of its rows, attend the old ones
    }
  }
  int kl = kv_len ? kv_len[qi] : r.len;
  kl = kl < 0 ? 0 : (kl > r.len ? r.len : kl);
  r.kv_len = kl;
  r.aa = 0;
  r.ab = 0;
  r.qa = 0;
  r.qb = kl;
  if (L.anchored) {
    if (L.anchor_rule == KVQ_ANCHOR_FIRST_N) {
      r.ab = L.anchor_n < kl ? L.anchor_n : kl;
      r.qa = r.ab;
    } else if (L.anchor_rule == KVQ_ANCHOR_WINDOW) {
      int w0 = r.len - L.anchor_n;
      w0 = w0 < 0 ? 0 : w0;
      r.aa = w0 < kl ? w0 : kl;
      r.ab = kl;
      r.qb = r.aa;
    } else if (L.anchor_rule == KVQ_ANCHOR_ALL) {
      r.ab = kl;
      r.qb = 0;
    }
  }
  return r;
}

// (q . mu) x sm_scale log2 e for the G heads of kv-head kvh, into qmu[G]: the logit every
// quantized row of a key-mean-subtracted sequence gets back (the original-domain dot product of
// the raw query with the sequence's fp16 key mean).  Zero without a key mean.  Warps take heads
// in turn; the caller synchronizes before reading.
__device__ void query_mean_term(const LayerDev& L, const __half* __restrict__ q, int qi, int seq, int kvh, int G,
                                float* qmu) {
  const SideDev& K = L.s[0];
  const int lane = threadIdx.x & 31, D = L.D;
  for (int h = threadIdx.x >> 5; h < G; h += blockDim.x >> 5) {
    float acc = 0.0f;
    if (K.mean_sub) {
      const __half* qp = q + query_row(L, qi, kvh, G, h) * D;
      const __half* mp = K.kmean + ((long long)seq * L.Hkv + kvh) * D;
      for (int j = lane; j < D; j += 32) acc = fmaf(__half2float(qp[j]), __half2float(mp[j]), acc);
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    }
    if (lane == 0) qmu[h] = acc * (L.sm_scale * kLog2e);
  }
}

// q' for G heads into qs[G][D] (stored domain of K, x sm_scale log2 e) and qa[G][D] (raw, x same).
template <int D>
__device__ void prepare_query(const LayerDev& L, const __half* __restrict__ q, int qi, int kvh, int G,
                              float* qs, float* qa) {
  const SideDev& K = L.s[0];
  const float scl = L.sm_scale * kLog2e;
  const int tid = threadIdx.x;
  for (int e = tid; e < G * D; e += blockDim.x) {
    const int h = e / D, j = e % D;
    const float v = __half2float(q[query_row(L, qi, kvh, G, h) * D + j]);
    qa[e] = v * scl;
    qs[e] = K.chan_scale ? v * __half2float(K.chan[kvh * D + j]) : v;
  }
  __syncthreads();
  if (K.rot == 128 || K.rot == 256) {
    const int n = K.rot;
    for (int h = 1; h < n; h <<= 1) {
      for (int e = tid; e < G * D / 2; e += blockDim.x) {
        // e-th pair: block of (i & ~h), index with bit h clear
        const int row = e / (D / 2), p = e % (D / 2);
        const int lo = p & (h - 1), hi = p >> __ffs(h) - 1;
        const int i = (hi << (__ffs(h))) | lo;  // insert a 0 bit at position log2(h)
        float* r = qs + row * D;
        const float a = r[i], b = r[i + h];
        r[i] = a + b;
        r[i + h] = a - b;
      }
      __syncthreads();
    }
    const float rn = (n == 256) ? 0.0625f : 0.08838834764831845f;
    for (int e = tid; e < G * D; e += blockDim.x) qs[e] *= rn;
    __syncthreads();
  } else if (K.fmt == KVQ_FMT_POLAR || K.fmt == KVQ_FMT_CART) {
    // Parseval adjoint of the folded rFFT (N = 128): logit = sum_f alpha_f a_f + beta_f b_f,
    // alpha_0 = Q_0/N, beta_0 = Q_64/N, alpha_f = 2 Re Q_f/N, beta_f = 2 Im Q_f/N.
    // twiddles of all 128 angles in shared memory: the threads' indices (f n mod N) diverge,
    // which constant memory would serialise
    __shared__ float tmp[kMaxG * 128], tc[128], ts[128];
    for (int e = tid; e < G * 128; e += blockDim.x) tmp[e] = qs[e];
    for (int k = tid; k < 128; k += blockDim.x) {
      tc[k] = k < 64 ? d_tw_re[k] : -d_tw_re[k - 64];
      ts[k] = k < 64 ? d_tw_im[k] : -d_tw_im[k - 64];  // -sin
    }
    __syncthreads();
    for (int e = tid; e < G * 64; e += blockDim.x) {
      const int h = e / 64, f = e % 64;
      const float* x = tmp + h * 128;
      float re = 0.0f, im = 0.0f, re64 = 0.0f;
      for (int n = 0; n < 128; ++n) {
        const int k = (f * n) & 127;
        const float c = tc[k];
        const float s = ts[k];
        re += x[n] * c;
        im += x[n] * s;
        if (f == 0) re64 += (n & 1) ? -x[n] : x[n];
      }
      float* o = qs + h * 128;
      if (f == 0) {
        o[0] = re / 128.0f;
        o[1] = re64 / 128.0f;
      } else {
        o[2 * f] = 2.0f * re / 128.0f;
        o[2 * f + 1] = 2.0f * im / 128.0f;
      }
    }
    __syncthreads();
  }
  for (int e = tid; e < G * D; e += blockDim.x) qs[e] *= scl;
  __syncthreads();
}

#include "decode_tc.cuh"
#include "decode_mq.cuh"
#include "decode_polar.cuh"

// Generic pass 1: any format, any GQA group (<= 8), CUDA cores.  Thread-per-token scoring,
// thread-per-channel value accumulation.
template <int D>
__global__ void __launch_bounds__(kGenThreads) decode_generic_kernel(LayerDev L, const __half* __restrict__ q,
                                                                     const int* __restrict__ seq_ids,
                                                                     const int* __restrict__ kv_len, float* __restrict__ work,
                                                                     int n_split, int nsp, int split_base) {
  constexpr int NCH = D > kGenThreads ? D / kGenThreads : 1;     // channels per thread
  constexpr int TSUB = D < kGenThreads ? kGenThreads / D : 1;    // token subsets in PV
  const int s = blockIdx.x + split_base, kvh = blockIdx.y, qi = blockIdx.z;
  const int G = L.Hq / L.Hkv;
  const int tid = threadIdx.x;
  __shared__ float qs[kMaxG * D], qa[kMaxG * D];
  __shared__ float sp[kMaxG][kGenTile];
  __shared__ float m_run[kMaxG], l_run[kMaxG], alpha[kMaxG];
  __shared__ float nf4[16], klm[16], vlm[16], kcs[256], ksn[256], vcs[256], vsn[256];
  __shared__ float red[kGenThreads / 32][kMaxG];
  __shared__ float qmu[kMaxG];

  const QueryRange R = query_range(L, qi, seq_ids, kv_len);
  const SideDev& K = L.s[0];
  const SideDev& V = L.s[1];
  const bool anchor_split = (s == n_split);
  int t0, t1;
  if (anchor_split) {
    t0 = R.aa;
    t1 = R.ab;
  } else {
    const int n = R.qb - R.qa;
    int chunk = (n + n_split - 1) / n_split;
    chunk = ((chunk + kGenTile - 1) / kGenTile) * kGenTile;
    t0 = R.qa + s * chunk;
    t1 = t0 + chunk < R.qb ? t0 + chunk : R.qb;
  }

  if (tid < 16) nf4[tid] = d_nf4[tid];
  if (K.fmt == KVQ_FMT_LLOYD && tid < 16) klm[tid] = d_lloyd[K.bits - 2][tid];
  if (V.fmt == KVQ_FMT_LLOYD && tid < 16) vlm[tid] = d_lloyd[V.bits - 2][tid];
  if (K.fmt == KVQ_FMT_POLAR)
    for (int k = tid; k < (1 << K.bits2); k += blockDim.x) {
      kcs[k] = d_ph_cos[(1 << K.bits2) - 2 + k];
      ksn[k] = d_ph_sin[(1 << K.bits2) - 2 + k];
    }
  if (V.fmt == KVQ_FMT_POLAR)
    for (int k = tid; k < (1 << V.bits2); k += blockDim.x) {
      vcs[k] = d_ph_cos[(1 << V.bits2) - 2 + k];
      vsn[k] = d_ph_sin[(1 << V.bits2) - 2 + k];
    }
  if (tid < kMaxG) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.0f;
  }
  query_mean_term(L, q, qi, R.seq, kvh, G, qmu);
  prepare_query<D>(L, q, qi, kvh, G, qs, qa);

  const long long u = (long long)R.seq * L.Hkv + kvh;
  float o[kMaxG][NCH];
#pragma unroll
  for (int h = 0; h < kMaxG; ++h)
#pragma unroll
    for (int c = 0; c < NCH; ++c) o[h][c] = 0.0f;

  for (int tb = t0; tb < t1; tb += kGenTile) {
    const int nt = (t1 - tb) < kGenTile ? (t1 - tb) : kGenTile;
    // ---- scores: thread tid scores token tb + tid for all G heads
    if (tid < nt) {
      const int t = tb + tid;
      float acc[kMaxG];
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) acc[h] = 0.0f;
      if (anchor_split) {
        const long long arow = u * L.anchor_rows + (L.anchor_rule == KVQ_ANCHOR_WINDOW ? t % L.anchor_n : t);
        for (int j = 0; j < D; ++j) {
          const float kv = anchor_value(L, K, arow, j);
#pragma unroll
          for (int h = 0; h < kMaxG; ++h)
            if (h < G) acc[h] += qa[h * D + j] * kv;
        }
      } else {
        const uint8_t* row = K.codes + (u * L.Tcap + t) * K.row_bytes;
        const __half* sc = K.scales + (u * L.Tcap + t) * K.n_groups;
        const __half* zr = K.zeros ? K.zeros + (u * L.Tcap + t) * K.n_groups : nullptr;
        if (K.fmt == KVQ_FMT_POLAR) {
          for (int f = 0; f < 64; ++f) {
            const float2 ab = polar_slot(K, row, sc, f, kcs, ksn);
#pragma unroll
            for (int h = 0; h < kMaxG; ++h)
              if (h < G) acc[h] += qs[h * D + 2 * f] * ab.x + qs[h * D + 2 * f + 1] * ab.y;
          }
        } else {
          for (int j = 0; j < D; ++j) {
            const float kv = stored_value(K, row, sc, zr, j, nf4, klm);
#pragma unroll
            for (int h = 0; h < kMaxG; ++h)
              if (h < G) acc[h] += qs[h * D + j] * kv;
          }
        }
#pragma unroll
        for (int h = 0; h < kMaxG; ++h)
          if (h < G) acc[h] += qmu[h];
      }
#pragma unroll
      for (int h = 0; h < kMaxG; ++h)
        if (h < G) sp[h][tid] = acc[h];
    }
    __syncthreads();
    // ---- online softmax (log2 domain): per-head tile max, rescale factor, probabilities
    {
      const int warp = tid >> 5, lane = tid & 31;
      for (int h = 0; h < G; ++h) {
        float mx = -INFINITY;
        for (int t = tid; t < nt; t += blockDim.x) mx = fmaxf(mx, sp[h][t]);
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red[warp][h] = mx;
      }
      __syncthreads();
      if (tid < G) {
        float mx = red[0][tid];
        for (int w = 1; w < kGenThreads / 32; ++w) mx = fmaxf(mx, red[w][tid]);
        const float mn = fmaxf(m_run[tid], mx);
        alpha[tid] = exp2f(m_run[tid] - mn);  // m_run = -inf -> 0
        m_run[tid] = mn;
      }
      __syncthreads();
      for (int h = 0; h < G; ++h) {
        float sum = 0.0f;
        for (int t = tid; t < nt; t += blockDim.x) {
          const float p = exp2f(sp[h][t] - m_run[h]);
          sp[h][t] = p;
          sum += p;
        }
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) red[warp][h] = sum;
      }
      __syncthreads();
      if (tid < G) {
        float sum = 0.0f;
        for (int w = 0; w < kGenThreads / 32; ++w) sum += red[w][tid];
        l_run[tid] = l_run[tid] * alpha[tid] + sum;
      }
    }
    // ---- values: thread owns channels (tid % D) + 128 c, token subset tid / D
    {
#pragma unroll
      for (int h = 0; h < kMaxG; ++h)
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          if (h < G) o[h][c] *= alpha[h];
      const int ch0 = tid % (D < kGenThreads ? D : kGenThreads);
      const int sub = tid / (D < kGenThreads ? D : kGenThreads);
      for (int tt = sub; tt < nt; tt += TSUB) {
        const int t = tb + tt;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          const int j = ch0 + c * kGenThreads;
          float vv;
          if (anchor_split) {
            vv = anchor_value(L, V, u * L.anchor_rows + (L.anchor_rule == KVQ_ANCHOR_WINDOW ? t % L.anchor_n : t), j);
          } else {
            const uint8_t* row = V.codes + (u * L.Tcap + t) * V.row_bytes;
            const __half* sc = V.scales + (u * L.Tcap + t) * V.n_groups;
            const __half* zr = V.zeros ? V.zeros + (u * L.Tcap + t) * V.n_groups : nullptr;
            if (V.fmt == KVQ_FMT_POLAR) {
              const float2 ab = polar_slot(V, row, sc, j >> 1, vcs, vsn);
              vv = (j & 1) ? ab.y : ab.x;
            } else {
              vv = stored_value(V, row, sc, zr, j, nf4, vlm);
            }
          }
#pragma unroll
          for (int h = 0; h < kMaxG; ++h)
            if (h < G) o[h][c] += sp[h][tt] * vv;
        }
      }
    }
    __syncthreads();
  }
  // ---- write partials (combine token subsets through shared memory when TSUB > 1)
  __shared__ float ored[kMaxG * D];
  if (TSUB > 1) {
    for (int e = tid; e < G * D; e += blockDim.x) ored[e] = 0.0f;
    __syncthreads();
#pragma unroll
    for (int h = 0; h < kMaxG; ++h)
      if (h < G) atomicAdd(&ored[h * D + (tid % D)], o[h][0]);
    __syncthreads();
  }
#pragma unroll
  for (int h = 0; h < kMaxG; ++h) {
    if (h >= G) break;
    float* P = work + (((long long)qi * L.Hq + kvh * G + h) * nsp + s) * (D + kPartStride);
    if (tid == 0) {
      P[0] = m_run[h];
      P[1] = l_run[h];
    }
    if (TSUB > 1) {
      for (int j = tid; j < D; j += blockDim.x) P[kPartStride + j] = ored[h * D + j];
    } else {
#pragma unroll
      for (int c = 0; c < NCH; ++c) P[kPartStride + tid + c * kGenThreads] = o[h][c];
    }
  }
}

// Pass 2: merge the splits of one (query, head), undo V's transform, add anchors, normalise.
// D x SP threads: thread (group sg, channel j) sums the splits s = sg (mod SP) of channel j, so
// many splits (long sequences, few queries) are read with SP times more loads in flight; the
// split weights are computed in parallel first.
template <int D>
constexpr int merge_groups() { return D >= 256 ? 4 : 512 / D; }

template <int D>
__global__ void __launch_bounds__(D * merge_groups<D>()) merge_kernel(LayerDev L, const float* __restrict__ work,
                                                                     int n_split, int nsp, void* __restrict__ out,
                                                                     int out_fp32, float* __restrict__ lse,
                                                                     const int* __restrict__ seq_ids) {
  constexpr int SP = merge_groups<D>(), NT = D * SP, NWP = NT / 32;
  const int qh = blockIdx.x;  // qi * Hq + h (this view's heads)
  const int tid = threadIdx.x, j = tid % D, sg = tid / D;
  const long long orow = (long long)(qh / L.Hq) * L.Hkv_all * (L.Hq / L.Hkv) + L.h0 * (L.Hq / L.Hkv) + qh % L.Hq;
  const SideDev& V = L.s[1];
  const float* P = work + (long long)qh * nsp * (D + kPartStride);
  __shared__ float w[kMaxSplit + 1];
  __shared__ float rm[NWP], rl[NWP];
  __shared__ float po[SP][D];
  __shared__ float ov[D];
  const int warp = tid >> 5, lane = tid & 31;
  static_assert(NT >= kMaxSplit + 1, "one thread per split's (m, l)");
  // One round trip: every split's (m, l) (thread s takes split s) and this thread's first R
  // partial-output values, loaded before the weights they are scaled by are known.
  constexpr int R = 24;
  float mv = -INFINITY, lv = 0.0f;
  if (tid < nsp) {
    mv = P[tid * (D + kPartStride)];
    lv = P[tid * (D + kPartStride) + 1];
  }
  const float* pj = P + kPartStride + j;
  float pre[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int s = sg + r * SP;
    pre[r] = s < n_split ? pj[s * (D + kPartStride)] : 0.0f;
  }
  // max of the partial maxima
  float M = mv;
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) rm[warp] = M;
  __syncthreads();
  M = rm[0];
  for (int i = 1; i < NWP; ++i) M = fmaxf(M, rm[i]);
  // weights and the normaliser
  float ls = 0.0f;
  if (tid < nsp) {
    const float ws = (mv == -INFINITY) ? 0.0f : exp2f(mv - M);
    w[tid] = ws;
    ls = ws * lv;
  }
  for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  if (lane == 0) rl[warp] = ls;
  __syncthreads();
  float Ls = 0.0f;
  for (int i = 0; i < NWP; ++i) Ls += rl[i];
  {
    float acc = 0.0f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int s = sg + r * SP;
      if (s < n_split) acc += w[s] * pre[r];
    }
#pragma unroll 8
    for (int s = sg + R * SP; s < n_split; s += SP) acc += w[s] * pj[s * (D + kPartStride)];
    po[sg][j] = acc;
  }
  __syncthreads();
  if (tid < D) {
    float acc = 0.0f;
#pragma unroll
    for (int g = 0; g < SP; ++g) acc += po[g][tid];
    ov[tid] = acc;
  }
  __syncthreads();
  if (V.rot == 128 || V.rot == 256) {
    const int n = V.rot;
    if (tid < D) {  // stages h < 32 inside each warp (thread t holds channel t): same butterflies
      float v = ov[tid];
      for (int h = 1; h < 32; h <<= 1) {
        const float p = __shfl_xor_sync(0xffffffffu, v, h);
        v = (tid & h) ? p - v : v + p;
      }
      ov[tid] = v;
    }
    __syncthreads();
    for (int h = 32; h < n; h <<= 1) {
      for (int p = tid; p < D / 2; p += NT) {
        const int lo = p & (h - 1), hi = p >> (__ffs(h) - 1);
        const int i = (hi << __ffs(h)) | lo;
        const float a = ov[i], b = ov[i + h];
        ov[i] = a + b;
        ov[i + h] = a - b;
      }
      __syncthreads();
    }
    const float rn = (n == 256) ? 0.0625f : 0.08838834764831845f;
    if (tid < D) ov[tid] *= rn;
    __syncthreads();
  } else if (V.fmt == KVQ_FMT_POLAR || V.fmt == KVQ_FMT_CART) {
    // x_n = (1/N) [a_0 + b_0 (-1)^n + 2 sum_{f=1}^{63} (a_f cos(2 pi f n/N) - b_f sin(2 pi f n/N))]
    //     = (1/N) Re FFT(conj Y)_n for the Hermitian spectrum Y (Y_0 = a_0, Y_64 = b_0,
    //       Y_f = a_f + i b_f, Y_{N-f} = conj Y_f): one warp, the register FFT (bit-reversed input)
    if (tid < 32) {
      const int brl = (int)(__brev((unsigned)tid) >> 27);
      float re[4], im[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int f = brl + 32 * (((r & 1) << 1) | (r >> 1));  // spectrum index of element 4 tid + r
        if (f == 0 || f == 64) {
          re[r] = ov[f == 0 ? 0 : 1];
          im[r] = 0.0f;
        } else if (f < 64) {
          re[r] = ov[2 * f];
          im[r] = -ov[2 * f + 1];
        } else {
          re[r] = ov[2 * (128 - f)];
          im[r] = ov[2 * (128 - f) + 1];
        }
      }
      fft128_warp(re, im, tid, g_tw[0], g_tw[1]);  // its shuffles order every lane's reads first
#pragma unroll
      for (int r = 0; r < 4; ++r) ov[4 * tid + r] = re[r] / 128.0f;
    }
    __syncthreads();
  }
  if (tid < D) {
    const float inv = Ls > 0.0f ? 1.0f / Ls : 0.0f;
    float v = ov[tid];
    if (nsp > n_split) v += w[n_split] * P[n_split * (D + kPartStride) + kPartStride + tid];
    v *= inv;
    if (out_fp32) reinterpret_cast<float*>(out)[orow * D + tid] = v;
    else reinterpret_cast<__half*>(out)[orow * D + tid] = __float2half_rn(v);
    if (lse && tid == 0) lse[orow] = Ls > 0.0f ? (M + log2f(Ls)) * 0.6931471805599453f : -INFINITY;
  }
  // fused append + decode: every read of this call is done (the split pass ran before), so the
  // query's sequence takes its new length here (one CTA per query; sequences are distinct)
  if (L.fuse_n > 0 && tid == 0 && qh % L.Hq == 0) {
    const int qi = qh / L.Hq, b = seq_ids ? seq_ids[qi] : qi;
    if (b >= 0 && b < L.B) {
      const int nl = L.seq_len[b] + L.fuse_n;
      if (nl <= L.cap) L.seq_len[b] = nl;
    }
  }
}

// ----------------------------------------------------------------------------------------------
// Planning and launch.

// Tensor-core path: the split count that maximises (busy fraction of the resident-CTA slots over
// whole waves) x (balance of tiles across splits) x per / (per + F), where a CTA's fixed cost F
// (query transform and fragments, table build, warp combine, partial write) is about 0.75 tiles of
// streaming; ties go to fewer splits.
static int mma_split_count(long long units, int ntiles, int slots) {
  int best = 1;
  double best_score = -1.0;
  for (int n = 1; n <= kMaxSplit && n <= ntiles; ++n) {
    const long long ctas = units * n;
    const long long waves = (ctas + slots - 1) / slots;
    const double eff = (double)ctas / (double)(waves * slots);
    const int per = (ntiles + n - 1) / n;
    const double bal = (double)ntiles / (double)(per * n);
    const double score = eff * bal * (double)per / ((double)per + 0.75);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = n;
    }
  }
  return best;
}

typedef void (*MmaKernel)(LayerDev, const __half*, const int*, const int*, float*, int, int);

struct MmaPlan {
  MmaKernel kern;   // decode only
  MmaKernel fkern;  // fused append + decode (same tiles and splits)
  int smem, tile, threads;
};

template <int D, int G, int KF, int GK, int VF, int GV, int NW, int TPW, int ST, int MB>
static MmaPlan mma_plan_of() {
  using C = TcCfg<D, KF, GK, VF, GV, NW, TPW, ST>;
  return MmaPlan{decode_tc_kernel<D, G, KF, GK, VF, GV, NW, TPW, ST>,
                 decode_tc_fused_kernel<D, G, KF, GK, VF, GV, NW, TPW, ST, MB>, C::SMEM, C::TILE, C::NTH};
}

static int code_fmt(const SideDev& S, bool is_v) {
  if (S.fmt == KVQ_FMT_NF4 && !is_v) return CF_NF4;
  if (S.fmt == KVQ_FMT_FP16 && is_v) return CF_FP16;
  if (S.fmt == KVQ_FMT_SIGN) return CF_SIGN;
  if (S.fmt == KVQ_FMT_TERNARY) return CF_TERN;
  if (S.fmt == KVQ_FMT_INT && S.scale_mode == KVQ_SCALE_ABSMAX && (S.bits == 4 || S.bits == 2)) return S.bits;
  if (S.fmt == KVQ_FMT_INT && S.scale_mode == KVQ_SCALE_ABSMAX && S.bits == 3 && is_v) return CF_INT3;
  if (S.fmt == KVQ_FMT_INT && S.scale_mode == KVQ_SCALE_SYMMETRIC && S.bits == 2 && is_v) return CF_SYM2;
  return -1;
}

// The tensor-core instantiations (others use the generic kernel): warps per CTA, tokens per warp
// and tile, pipeline stages.  Measured on the 32K-token batch-16 workload: a warp's fixed cost per
// tile (barrier, wait, softmax reduction) is amortised best by 32-64 tokens per warp and tile, with
// two stages of 256 tokens; NF4's 32 KB per-lane table leaves room for 8 warps per CTA at most.
static bool pick_mma(const LayerDev& L, MmaPlan* out) {
  const int G = L.Hq / L.Hkv;
  const int kf = code_fmt(L.s[0], false), vf = code_fmt(L.s[1], true);
  if (kf < 0 || vf < 0) return false;
  const int gk = L.s[0].group, gv = vf == CF_FP16 ? 128 : L.s[1].group;
// Last argument: CTAs per SM of the plain instance (shared memory or registers), which its fused
// append + decode twin is held to.
#define KVQ_MMA(D_, G_, KF_, GK_, VF_, GV_, NW_, TPW_, ST_, MB_)                                \
  if (L.D == D_ && G == G_ && kf == KF_ && gk == GK_ && vf == VF_ && gv == GV_) {                \
    *out = mma_plan_of<D_, G_, KF_, GK_, VF_, GV_, NW_, TPW_, ST_, MB_>();                     \
    return true;                                                                              \
  }
  KVQ_MMA(128, 4, CF_NF4, 64, CF_INT4, 64, 8, 32, 2, 2)
  KVQ_MMA(128, 4, CF_INT4, 64, CF_INT4, 64, 4, 64, 2, 3)
  KVQ_MMA(128, 4, CF_INT4, 32, CF_INT4, 32, 8, 32, 2, 2)
  KVQ_MMA(128, 2, CF_INT4, 32, CF_INT4, 32, 8, 32, 2, 2)
  KVQ_MMA(128, 4, CF_SIGN, 4, CF_SIGN, 4, 8, 32, 2, 2)
  KVQ_MMA(128, 4, CF_TERN, 8, CF_TERN, 8, 8, 32, 2, 2)
  KVQ_MMA(256, 4, CF_INT4, 128, CF_INT2, 128, 4, 32, 3, 2)
  KVQ_MMA(256, 4, CF_INT4, 128, CF_SYM2, 128, 4, 32, 3, 2)
  KVQ_MMA(256, 4, CF_INT4, 128, CF_INT3, 128, 4, 32, 3, 2)
  KVQ_MMA(256, 4, CF_INT4, 128, CF_INT4, 128, 4, 16, 4, 3)
  KVQ_MMA(256, 4, CF_INT4, 128, CF_FP16, 128, 4, 16, 2, 2)
  KVQ_MMA(256, 4, CF_INT4, 32, CF_INT4, 32, 4, 16, 3, 2)
#undef KVQ_MMA
  return false;
}

static int mma_slots(const MmaPlan& p, int num_sms) {
  static MmaKernel cached_k = nullptr;
  static int cached_occ = 1;
  if (cached_k != p.kern) {
    cudaFuncSetAttribute(p.kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
    int occ = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, p.kern, p.threads, p.smem) != cudaSuccess || occ < 1)
      occ = 1;
    cudaGetLastError();
    cached_k = p.kern;
    cached_occ = occ;
  }
  return cached_occ * num_sms;
}

// The multi-query kernel (tiles decoded once per CTA into shared memory, any format) serves every
// quantized range that has no register-decode tensor-core instance, and GQA groups of 1 or 2 with
// more queries than sequences (some queries share a sequence, so a decoded tile serves several).
// The generic kernel is left with the anchor rows.
static bool use_mq(const LayerDev& L, int n_q) {
  MmaPlan p;
  return !pick_mma(L, &p) || (L.Hq / L.Hkv <= 2 && n_q > L.B);
}

// rFFT polar K and V with one query per sequence (GQA 1, 2 or 4): the CUDA-core polar kernel,
// whose lanes all work on the one live query row (the multi-query kernel's tiles would carry one
// row in 64).  Queries sharing a sequence (proxy queries) stay on the multi-query kernel.
static bool use_polar(const LayerDev& L, int n_q) {
  const int G = L.Hq / L.Hkv;
  return L.D == 128 && L.s[0].fmt == KVQ_FMT_POLAR && L.s[1].fmt == KVQ_FMT_POLAR && n_q <= L.B &&
         (G == 1 || G == 2 || G == 4);
}

typedef void (*PolarKernel)(const LayerDev, const __half*, const int*, const int*, float*, int, int);

template <int G>
static PolarKernel polar_kernel_g(const LayerDev& L) {
  const bool f48 = L.s[0].bits == 4 && L.s[0].bits2 == 8 && L.s[1].bits == 4 && L.s[1].bits2 == 8;
  return f48 ? decode_polar_kernel<G, 4, 8> : decode_polar_kernel<G, 0, 0>;
}
static PolarKernel polar_kernel(const LayerDev& L) {
  switch (L.Hq / L.Hkv) {
    case 1: return polar_kernel_g<1>(L);
    case 2: return polar_kernel_g<2>(L);
    default: return polar_kernel_g<4>(L);
  }
}
static int polar_smem(const LayerDev& L) {
  switch (L.Hq / L.Hkv) {
    case 1: return polar_smem_bytes<1>(L);
    case 2: return polar_smem_bytes<2>(L);
    default: return polar_smem_bytes<4>(L);
  }
}

// Resident CTAs of the polar kernel on L's formats x SMs.  Each instance's opt-in shared-memory
// limit is raised to the maximum once; occupancy is cached per (instance, bytes).
static int polar_slots(const LayerDev& L, int num_sms) {
  struct Occ {
    PolarKernel k;
    int smem, occ;
  };
  static PolarKernel raised[6] = {};
  static Occ occs[32] = {};
  static int n_occ = 0;
  const PolarKernel k = polar_kernel(L);
  const int smem = polar_smem(L);
  for (int i = 0; i < n_occ; ++i)
    if (occs[i].k == k && occs[i].smem == smem) return occs[i].occ * num_sms;
  bool seen = false;
  for (int i = 0; i < 6 && raised[i]; ++i) seen |= raised[i] == k;
  if (!seen) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, k) == cudaSuccess &&
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024 - (int)fa.sharedSizeBytes) == cudaSuccess)
      for (int i = 0; i < 6; ++i)
        if (!raised[i]) {
          raised[i] = k;
          break;
        }
    cudaGetLastError();
  }
  int occ = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, PolarCfg::NT, smem) != cudaSuccess || occ < 1) occ = 1;
  cudaGetLastError();
  if (n_occ < 32) occs[n_occ++] = Occ{k, smem, occ};
  return occ * num_sms;
}

// Splits of the polar kernel: one wave of resident CTAs (every CTA has the same work), at least
// one tile each.
static int polar_splits(const LayerDev& L, int n_q, int num_sms) {
  const long long units = (long long)L.Hkv * n_q;
  const long long tiles = L.Tcap / PolarCfg::TT;  // capacities are whole multiples of 256 tokens
  long long s = polar_slots(L, num_sms) / units;
  if (s > kMaxSplit) s = kMaxSplit;
  if (s > tiles) s = tiles;
  if (s < 1) s = 1;
  const long long per = (tiles + s - 1) / s;  // the same tiles over fewer splits: none left idle
  return (int)((tiles + per - 1) / per);
}

// Format class of a layer's (K, V) pair on the multi-query kernel (see MqFmtClass).
template <int D>
static int mq_class(const LayerDev& L) {
  auto mm_side = [](const SideDev& S) {
    return S.fmt == KVQ_FMT_INT && S.scale_mode == KVQ_SCALE_MINMAX && (S.bits == 3 || S.bits == 4) && S.group >= 8 &&
           S.zeros;
  };
  if (D == 256 && mm_side(L.s[0]) && mm_side(L.s[1])) return FC_MINMAX;
  if (D == 128 && L.s[0].fmt == KVQ_FMT_POLAR && L.s[1].fmt == KVQ_FMT_POLAR) return FC_POLAR;
  return FC_ANY;
}

// Splits of the multi-query kernel: about two waves of its CTAs, at least one tile each.
template <int D, int FC>
static int mq_split_count_fc(const LayerDev& L, int n_q, int num_sms) {
  using C = MqCfg<D, FC>;
  const int G = L.Hq / L.Hkv, qpb = C::QM / G;
  const long long units = (long long)L.Hkv * ((n_q + qpb - 1) / qpb);
  const int per_sm = (D >= 256 && FC != FC_MINMAX) ? 1 : 2;  // resident CTAs (shared memory)
  long long s = (2LL * per_sm * num_sms + units - 1) / units;
  const long long tiles = L.Tcap / C::TK;
  if (s > tiles) s = tiles;
  if (s > kMaxSplit) s = kMaxSplit;
  return s < 1 ? 1 : (int)s;
}

template <int D>
static int mq_split_count(const LayerDev& L, int n_q, int num_sms) {
  switch (mq_class<D>(L)) {
    case FC_MINMAX: return mq_split_count_fc<D, FC_MINMAX>(L, n_q, num_sms);
    case FC_POLAR: return mq_split_count_fc<D, FC_POLAR>(L, n_q, num_sms);
    default: return mq_split_count_fc<D, FC_ANY>(L, n_q, num_sms);
  }
}

static int mq_splits(const LayerDev& L, int n_q, int num_sms) {
  switch (L.D) {
    case 64: return mq_split_count<64>(L, n_q, num_sms);
    case 128: return mq_split_count<128>(L, n_q, num_sms);
    default: return mq_split_count<256>(L, n_q, num_sms);
  }
}

// Whether one decode launch can also append this call's rows (fused append + decode): a
// register-decode tensor-core instance serves the pair, and the append needs none of the extras
// (key mean, int anchors, head groups) that only the standalone append kernels carry.
// It is also worth it only when the split-K grid fits in one wave of resident CTAs: there the step
// is latency-bound and the saved launch shows (64K-token batch-1 step: +19 % steps/s), while on
// multi-wave grids the fused instances' split pass measured slower than the plain pass plus the
// one-token append (batch-16 NF4 + int4: 183 against 150 + 10 us per layer).
bool fused_decode_ok(const LayerDev& L, int n_q, int num_sms) {
  MmaPlan p;
  if (!pick_mma(L, &p) || use_mq(L, n_q) || L.s[0].mean_sub || L.s[1].mean_sub || L.anchor_bits != 16 ||
      L.Hkv != L.Hkv_all)
    return false;
  const int slots = mma_slots(p, num_sms);
  const long long units = (long long)n_q * L.Hkv;
  return (long long)mma_split_count(units, L.Tcap / p.tile, slots) * units <= slots;
}

// Partials per (query, head) the decode of `L` writes for n_q queries (the workspace bound).
int decode_partials(const LayerDev& L, int n_q, int num_sms) {
  if (use_mq(L, n_q))  // + anchor split (+ prepared queries on the multi-query kernel)
    return use_polar(L, n_q) ? polar_splits(L, n_q, num_sms) + 1 : mq_splits(L, n_q, num_sms) + 2;
  MmaPlan p;
  pick_mma(L, &p);
  const int ntiles = L.Tcap / p.tile;
  return mma_split_count((long long)n_q * L.Hkv, ntiles, mma_slots(p, num_sms)) + 1;
}

template <int D>
static cudaError_t launch_decode_d(const LayerDev& L, const __half* q, int n_q, const int* seq_ids, const int* kv_len,
                                   void* out, int out_fp32, float* lse, float* work, int num_sms, cudaStream_t st,
                                   int* launches) {
  int nl = 0;
  MmaPlan p;
  int n_quant;  // quantized partials per (query, head)
  if (D == 128 && use_mq(L, n_q) && use_polar(L, n_q)) {
    if (L.fuse_n > 0) return cudaErrorInvalidValue;  // the caller checks fused_decode_ok first
    const int n_split = polar_splits(L, n_q, num_sms);  // raises the kernel's shared-memory limit
    n_quant = n_split;
    const int nsp = n_quant + (L.anchored ? 1 : 0);
    polar_kernel(L)<<<dim3(n_split, L.Hkv, n_q), PolarCfg::NT, polar_smem(L), st>>>(L, q, seq_ids, kv_len, work,
                                                                                   n_split, nsp);
    ++nl;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (L.anchored) {  // anchor rows: the generic kernel's anchor split alone
      decode_generic_kernel<D><<<dim3(1, L.Hkv, n_q), kGenThreads, 0, st>>>(L, q, seq_ids, kv_len, work, n_quant, nsp,
                                                                           n_quant);
      ++nl;
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  } else if (use_mq(L, n_q)) {
    if (L.fuse_n > 0) return cudaErrorInvalidValue;  // the caller checks fused_decode_ok first
    // Tile decode without the format dispatch where both sides' class is known: min-max int codes
    // of 3 or 4 bits in groups of >= 8 (config 2, head_dim 256), rFFT polar (config 4, head_dim 128).
    const int fc = mq_class<D>(L);
    auto kern = decode_mq_kernel<D, FC_ANY>;
    int smem = mq_smem_bytes<D, FC_ANY>(L), nt = MqCfg<D, FC_ANY>::NT, qm = MqCfg<D, FC_ANY>::QM;
    if constexpr (D == 256) {
      if (fc == FC_MINMAX) {
        kern = decode_mq_kernel<D, FC_MINMAX>;
        smem = mq_smem_bytes<D, FC_MINMAX>(L);
        nt = MqCfg<D, FC_MINMAX>::NT;
        qm = MqCfg<D, FC_MINMAX>::QM;
      }
    } else if constexpr (D == 128) {
      if (fc == FC_POLAR) {
        kern = decode_mq_kernel<D, FC_POLAR>;
        smem = mq_smem_bytes<D, FC_POLAR>(L);
      }
    }
    static int dyn_max[3] = {-1, -1, -1};  // per instantiation (the attribute is per kernel)
    if (dyn_max[fc] < 0) {  // the opt-in limit covers static + dynamic shared memory
      cudaFuncAttributes fa;
      cudaError_t e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return e;
      const int lim = MqCfg<D>::SMEM_MAX - (int)fa.sharedSizeBytes;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
      if (e != cudaSuccess) return e;
      dyn_max[fc] = lim;
    }
    if (smem > dyn_max[fc]) return cudaErrorInvalidValue;  // staged rows of this format pair do not fit
    const int n_split = mq_split_count<D>(L, n_q, num_sms);
    n_quant = n_split;
    const int nsp = n_quant + (L.anchored ? 1 : 0);
    // the prepared queries take the workspace slot after the partials (decode_partials counts it)
    float* prep = work + (size_t)n_q * L.Hq * nsp * (D + kPartStride);
    mq_prep_kernel<D><<<dim3(L.Hkv, n_q), 256, 0, st>>>(L, q, seq_ids, kv_len, prep);
    ++nl;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int qpb = qm / (L.Hq / L.Hkv);
    kern<<<dim3(n_split, L.Hkv, (n_q + qpb - 1) / qpb), nt, smem, st>>>(L, prep, seq_ids, kv_len, work, n_split, nsp,
                                                                       n_q);
    ++nl;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (L.anchored) {  // anchor rows: the generic kernel's anchor split alone
      decode_generic_kernel<D><<<dim3(1, L.Hkv, n_q), kGenThreads, 0, st>>>(L, q, seq_ids, kv_len, work, n_quant, nsp,
                                                                           n_quant);
      ++nl;
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  } else {  // a register-decode tensor-core instance exists (use_mq said no)
    pick_mma(L, &p);
    const int slots = mma_slots(p, num_sms);
    const int n_split = mma_split_count((long long)n_q * L.Hkv, L.Tcap / p.tile, slots);
    n_quant = n_split;
    const int nsp = n_quant + (L.anchored ? 1 : 0);
    if (L.fuse_n > 0) {  // the fused instance: same tiles and splits, the new rows written first
      static MmaKernel fset[32] = {};
      bool seen = false;
      for (int i = 0; i < 32 && fset[i]; ++i) seen |= fset[i] == p.fkern;
      if (!seen) {
        cudaError_t e = cudaFuncSetAttribute(p.fkern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
        if (e != cudaSuccess) return e;
        for (int i = 0; i < 32; ++i)
          if (!fset[i]) {
            fset[i] = p.fkern;
            break;
          }
      }
      p.kern = p.fkern;
    }
    p.kern<<<dim3(n_split, L.Hkv, n_q), p.threads, p.smem, st>>>(L, q, seq_ids, kv_len, work, n_split, nsp);
    ++nl;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (L.anchored) {  // anchor rows: the generic kernel's anchor split alone
      decode_generic_kernel<D><<<dim3(1, L.Hkv, n_q), kGenThreads, 0, st>>>(L, q, seq_ids, kv_len, work, n_quant, nsp,
                                                                           n_quant);
      ++nl;
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  const int nsp = n_quant + (L.anchored ? 1 : 0);
  merge_kernel<D><<<n_q * L.Hq, D * merge_groups<D>(), 0, st>>>(L, work, n_quant, nsp, out, out_fp32, lse, seq_ids);
  ++nl;
  if (launches) *launches = nl;
  return cudaGetLastError();
}

cudaError_t launch_decode(const LayerDev& L, const __half* q, int n_q, const int* seq_ids, const int* kv_len, void* out,
                          int out_fp32, float* lse, float* work, int num_sms, int /*max_queries*/, cudaStream_t st,
                          int* launches) {
  switch (L.D) {
    case 64: return launch_decode_d<64>(L, q, n_q, seq_ids, kv_len, out, out_fp32, lse, work, num_sms, st, launches);
    case 128: return launch_decode_d<128>(L, q, n_q, seq_ids, kv_len, out, out_fp32, lse, work, num_sms, st, launches);
    case 256: return launch_decode_d<256>(L, q, n_q, seq_ids, kv_len, out, out_fp32, lse, work, num_sms, st, launches);
  }
  return cudaErrorInvalidValue;
}


// ----------------------------------------------------------------------------------------------
// Fixed scratch for kvq_decode_attention_noalloc: split-K partials live in this file-scope device
// array instead of a workspace from cudaMalloc.  Every GPU that loads the library holds it (8 MiB)
// until the process exits.  Host code must not pass `g_static_work` itself to a kernel (on the
// host that name is only a stand-in); its device address comes from cudaGetSymbolAddress, taken
// once per device with that device current.
constexpr size_t kStaticWorkFloats = size_t(2) << 20;
static __device__ __align__(256) float g_static_work[kStaticWorkFloats];

static std::mutex g_static_mu;
static float* g_static_ptr[128] = {};

size_t static_work_floats() { return kStaticWorkFloats; }

cudaError_t static_work_ptr(int dev, float** out) {
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[dev]) {
    float* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_static_work);
    if (e != cudaSuccess) return e;
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return cudaSuccess;
}

}  // namespace kvq
