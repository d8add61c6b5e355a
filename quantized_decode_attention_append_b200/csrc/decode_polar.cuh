// Pass 1 of the split-K decode for rFFT polar K and V with one query per sequence, on CUDA cores
// (included by decode.cu inside namespace kvq, after decode_tc.cuh and fft128.cuh: uses the
// mbarrier and bulk-copy primitives, the register FFT, the twiddles g_tw and the replicated phase
// table g_ph_rep).
//
// What it computes.  A polar row stores, for each of the 64 slots f of the folded spectrum of a
// 128-channel row ("Fourier Magnitude KV Cache Quantization", the reply on finite-phase codes), a
// magnitude code c_f (bits wide) and a phase code k_f (bits2 wide), with one fp16 scale s per
// row: the stored values are s c_f cos(phi_k) and s c_f sin(phi_k) at elements 2f and 2f + 1.
// The logit of a token is q' . k over those 128 stored values, q' being the Parseval adjoint of
// the folded rFFT applied to the query (x sm_scale log2 e), i.e. s sum_f c_f (q'_2f cos phi +
// q'_2f+1 sin phi); V is accumulated in the same stored domain and turned back into channels by
// the merge.
//
// Why a kernel of its own.  With one query per (sequence, kv-head) both products are
// matrix-vector ones: the multi-query kernel's 64-row tensor-core tiles would carry one live row,
// and its per-tile decode into shared memory would feed one warp's products.  Here every lane
// works on live data.
//
// Query.  Each CTA transforms its query heads itself, warp h head h, with the register FFT of the
// 128 channels (fft128.cuh): q'_0 = X_0 / 128, q'_1 = X_64 / 128, q'_2f = 2 Re X_f / 128,
// q'_2f+1 = 2 Im X_f / 128, through shared memory -- no separate launch.
//
// Lanes.  Eight lanes share a token; lane j of the group owns slots 8j .. 8j + 7.  Their
// magnitude fields are bytes [j bits, (j + 1) bits) of the row's magnitude stream and their phase
// fields bytes [j bits2, (j + 1) bits2) of the phase stream (8 fields of b bits = b bytes), so for
// every field width a lane reads whole bytes.  The magnitude code becomes a float by the exponent
// trick (2^23 + c as bits, minus 2^23); on the V side w c = fma(w, 2^23 + c, -w 2^23) is the
// exact product in one instruction.  (cos, sin) of the phase level come as one 64-bit load from a
// table held in 16 interleaved copies, copy r on bank pair r, lane l reading copy l % 16: a warp's
// 32 random lookups take the two wavefronts of any 64-bit access.
//
// Tokens.  The CTA's 32 groups take two tokens each of a 64-token tile, group g tokens g and
// g + 32 (consecutive groups of a warp then read rows on distinct banks for 96-byte rows).  The
// logit is reduced across the group by three shuffles; each group runs its own online softmax
// (log2 domain) and accumulates P V for its slots.  At the end the groups' states are combined
// (within the warp by shuffles, across warps in shared memory) into the split's (m, l, o).
//
// Copies.  One thread issues bulk copies (cp.async.bulk on an mbarrier): the phase table once, and
// per 64-token tile the K codes, K scales, V codes and V scales -- NSTAGE tiles at the start, each
// later tile into the stage of the tile NSTAGE before it once every warp is done with that one (a
// CTA with at most NSTAGE tiles takes no barrier in its loop).  Tiles start at multiples of 64
// tokens and capacities are whole multiples of 256, so every copy is 16-byte aligned and whole
// tiles stay inside the sequence's rows.  Tokens outside the query's quantized range get a zero
// scale and a -inf logit, so rows past the length never reach the sums.  Waits are bounded
// (KVQ_ERRF_WAIT_TIMEOUT); after one runs out the CTA waits, bounded again, for the copies it
// issued before it exits.
//
// GQA groups of 1, 2 and 4 heads share the decoded fields; queries and accumulators live in
// registers.  Field widths 4 + 8 (the common split) are compiled in; others are read at run time.

struct PolarCfg {
  static constexpr int D = 128;
  static constexpr int NT = 256;
  static constexpr int NW = NT / 32;
  static constexpr int LPT = 8;             // lanes per token
  static constexpr int SPL = 64 / LPT;      // slots per lane
  static constexpr int NG = NT / LPT;       // token groups per CTA
  static constexpr int TT = 2 * NG;         // tokens per tile
  static constexpr int NSTAGE = 3;          // staged tiles
  static constexpr int COPIES = 16;         // phase-table copies (one per bank pair)
  static constexpr int EP = D + 4;          // floats per (warp, head) in the combine: o[D], m, l
  static constexpr int OFF_TAB = 64;        // after the mbarriers (NSTAGE + 1 of 8 bytes)
};

// Bytes of one side's slice of a staged tile: codes, then the fp16 row scales.
__host__ __device__ __forceinline__ int polar_codes_bytes(const SideDev& S) { return PolarCfg::TT * S.row_bytes; }
__host__ __device__ __forceinline__ int polar_side_bytes(const SideDev& S) {
  return polar_codes_bytes(S) + PolarCfg::TT * 2;
}

// Dynamic shared memory of one decode_polar_kernel<G, ...> launch on `L`: barriers, the phase
// tables (one when both sides have the same phase width), then the staging ring, which the final
// combine reuses.
template <int G>
inline int polar_smem_bytes(const LayerDev& L) {
  using C = PolarCfg;
  const int tk = (1 << L.s[0].bits2) * C::COPIES * 8;
  const int tv = L.s[1].bits2 == L.s[0].bits2 ? 0 : (1 << L.s[1].bits2) * C::COPIES * 8;
  const int st = C::NSTAGE * (polar_side_bytes(L.s[0]) + polar_side_bytes(L.s[1]));
  const int ep = C::NW * G * C::EP * 4;  // the warps' combine
  return C::OFF_TAB + tk + tv + (st > ep ? st : ep) + 16;  // + 16: mq_bits64 reads past a field
}

// Shared-memory loads at 32-bit shared addresses (the table and field reads take one address add).
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds_u2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ float2 lds_f2(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];\n" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_h2f(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];\n" : "=h"(v) : "r"(a));
  return __half2float(__ushort_as_half(v));
}

// The eight magnitude codes of a lane as floats 2^23 + c, and its eight phase codes as byte
// offsets into a phase table (level k at k x 16 copies x 8 bytes).  row_s: the staged row's shared
// address; row: the same row (generic pointer, for the run-time field widths).
template <int BM, int BP>
__device__ __forceinline__ void polar_fields(uint32_t row_s, const uint8_t* row, int j, int bm, int bp, float* F,
                                             uint32_t* ko) {
  if constexpr (BM == 4 && BP == 8) {
    const uint32_t mw = lds_u32(row_s + 4 * j);
    const uint2 pw = lds_u2(row_s + 32 + 8 * j);
    const uint32_t ev = mw & 0x0F0F0F0Fu, od = (mw >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // byte i / 2 of the even or odd nibbles into the low byte of 0x4B000000
      F[i] = __uint_as_float(__byte_perm(i & 1 ? od : ev, 0x4B000000u, 0x7440u | (i >> 1)));
      ko[i] = __byte_perm(i < 4 ? pw.x : pw.y, 0u, 0x4440u | (i & 3)) << 7;
    }
  } else {
    const uint64_t mw = mq_bits64(row, j * 8 * bm), pw = mq_bits64(row, 64 * bm + j * 8 * bp);
    const uint32_t mm = (1u << bm) - 1u, pm = (1u << bp) - 1u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      F[i] = __uint_as_float(0x4B000000u | ((uint32_t)(mw >> (i * bm)) & mm));
      ko[i] = ((uint32_t)(pw >> (i * bp)) & pm) << 7;
    }
  }
}

// Query head h of a CTA's (query, kv-head) in one warp: the rFFT of its 128 channels (x the K
// channel scale when K has one) left in registers (lane l: X_4l .. X_4l+3), and the key-mean term
// (q . mu) sm_scale log2 e (zero without a key mean) on every lane.
__device__ __forceinline__ void polar_query_fft(const LayerDev& L, const __half* __restrict__ q, int qi, int kvh,
                                                int seq, int G, int h, int lane, float scl, float (&re)[4],
                                                float (&im)[4], float& mu) {
  constexpr int D = PolarCfg::D;
  const SideDev& K = L.s[0];
  const int brl = (int)(__brev((unsigned)lane) >> 27);
  const __half* qp = q + query_row(L, qi, kvh, G, h) * D;
  const __half* km = K.mean_sub ? K.kmean + ((long long)seq * L.Hkv + kvh) * D : nullptr;
  float dot = 0.0f;
#pragma unroll
  for (int r = 0; r < 4; ++r) {  // element 4 lane + r of the bit-reversed input
    const int n = brl + 32 * (((r & 1) << 1) | (r >> 1));
    const float x = __half2float(qp[n]);
    if (km) dot = fmaf(x, __half2float(km[n]), dot);
    re[r] = K.chan_scale ? x * __half2float(K.chan[kvh * D + n]) : x;
    im[r] = 0.0f;
  }
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  mu = dot * scl;
  fft128_warp(re, im, lane, g_tw[0], g_tw[1]);
}

template <int G, int BM, int BP>
__global__ void __launch_bounds__(PolarCfg::NT, G == 1 ? 3 : (G == 2 ? 2 : 1))
    decode_polar_kernel(const __grid_constant__ LayerDev L, const __half* __restrict__ q,
                        const int* __restrict__ seq_ids, const int* __restrict__ kv_len, float* __restrict__ work,
                        int n_split, int nsp_total) {
  using C = PolarCfg;
  constexpr int D = C::D;
  constexpr float kTwo23 = 8388608.0f;
  constexpr float kSlack = 8.0f;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(16) float qs[G][D], qmu[G];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, j = lane & (C::LPT - 1), gid = tid / C::LPT;
  const int split = blockIdx.x, kvh = blockIdx.y, qi = blockIdx.z;
  const SideDev& K = L.s[0];
  const SideDev& V = L.s[1];
  const int bmK = BM ? BM : K.bits, bpK = BP ? BP : K.bits2, bmV = BM ? BM : V.bits, bpV = BP ? BP : V.bits2;
  const int nK = 1 << bpK, nV = 1 << bpV;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);  // [0, NSTAGE): tiles; NSTAGE: phase tables
  float2* tabK = reinterpret_cast<float2*>(smem + C::OFF_TAB);
  float2* tabV = bpV == bpK ? tabK : tabK + nK * C::COPIES;
  uint8_t* raw = reinterpret_cast<uint8_t*>(tabK + nK * C::COPIES + (bpV == bpK ? 0 : nV * C::COPIES));
  const int sbK = polar_side_bytes(K), sbV = polar_side_bytes(V), stg = sbK + sbV;
  const int cbK = polar_codes_bytes(K), cbV = polar_codes_bytes(V);

  // ---- this split's tiles of the query's quantized range
  const QueryRange R = query_range<false>(L, qi, seq_ids, kv_len);
  const int qa = R.qa, qb = R.qb;
  const int tstart = (qa / C::TT) * C::TT;
  const int ntiles = qb > qa ? (qb - tstart + C::TT - 1) / C::TT : 0;
  const int per = (ntiles + n_split - 1) / n_split;
  const int it0 = split * per, nmy = max(0, min(ntiles, it0 + per) - it0);
  if (nmy == 0) {  // nothing to attend: an empty partial per head
    for (int e = tid; e < G * (D + kPartStride); e += C::NT) {
      const int h = e / (D + kPartStride), c = e % (D + kPartStride);
      work[(((long long)qi * L.Hq + kvh * G + h) * nsp_total + split) * (D + kPartStride) + c] =
          c == 0 ? -INFINITY : 0.0f;
    }
    return;
  }
  const long long u = (long long)R.seq * L.Hkv + kvh;
  const long long row0 = u * L.Tcap + tstart + (long long)it0 * C::TT;  // first row of tile 0
  auto issue = [&](int it, int s) {  // one thread: the four copies of tile it into stage s
    const long long r = row0 + (long long)it * C::TT;
    uint8_t* b = raw + s * stg;
    fence_proxy_async();
    mbar_expect_tx(bar + s, (uint32_t)stg);
    bulk_g2s(b, K.codes + r * K.row_bytes, cbK, bar + s);
    bulk_g2s(b + cbK, K.scales + r, C::TT * 2, bar + s);
    bulk_g2s(b + sbK, V.codes + r * V.row_bytes, cbV, bar + s);
    bulk_g2s(b + sbK + cbV, V.scales + r, C::TT * 2, bar + s);
  };
  int issued = 0;  // tiles issued (thread 0)
  if (tid == 0) {
    for (int s = 0; s <= C::NSTAGE; ++s) mbar_init(bar + s, 1);
    mbar_init_fence();
    const int tbytes = (nK + (bpV == bpK ? 0 : nV)) * C::COPIES * 8;
    mbar_expect_tx(bar + C::NSTAGE, (uint32_t)tbytes);
    bulk_g2s(tabK, g_ph_rep + (nK - 2) * C::COPIES, nK * C::COPIES * 8, bar + C::NSTAGE);
    if (bpV != bpK) bulk_g2s(tabV, g_ph_rep + (nV - 2) * C::COPIES, nV * C::COPIES * 8, bar + C::NSTAGE);
    for (; issued < C::NSTAGE && issued < nmy; ++issued) issue(issued, issued);
  }

  // ---- the query heads' transform (overlaps the first copies)
  const float scl = L.sm_scale * kLog2e;
  float q2[G][C::SPL][2], mu[G];
  if (warp < G) {  // warp h: head h
    const int h = warp;
    float re[4], im[4], m0;
    polar_query_fft(L, q, qi, kvh, R.seq, G, h, lane, scl, re, im, m0);
    if (lane == 0) qmu[h] = m0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {  // lane l holds X_4l+r
      const int f = 4 * lane + r;
      if (f == 0) {
        qs[h][0] = re[0] / 128.0f * scl;
      } else if (f < 64) {
        qs[h][2 * f] = 2.0f * re[r] / 128.0f * scl;
        qs[h][2 * f + 1] = 2.0f * im[r] / 128.0f * scl;
      } else if (f == 64) {
        qs[h][1] = re[0] / 128.0f * scl;
      }
    }
  }
  __syncthreads();  // also orders the barriers' initialisation before every wait
#pragma unroll
  for (int h = 0; h < G; ++h) {
    mu[h] = qmu[h];
#pragma unroll
    for (int i = 0; i < C::SPL; ++i) {
      const float2 v = *reinterpret_cast<const float2*>(&qs[h][2 * C::SPL * j + 2 * i]);
      q2[h][i][0] = v.x;
      q2[h][i][1] = v.y;
    }
  }

  float acc[G][C::SPL][2];
  float m[G], l[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.0f;
#pragma unroll
    for (int i = 0; i < C::SPL; ++i) acc[h][i][0] = acc[h][i][1] = 0.0f;
  }
  const uint32_t tk_s = smem_u32(tabK) + (lane & (C::COPIES - 1)) * 8;  // this lane's table copy
  const uint32_t tv_s = smem_u32(tabV) + (lane & (C::COPIES - 1)) * 8;
  const uint32_t raw_s = smem_u32(raw);
  bool timed_out = false;
  if (__any_sync(0xffffffffu, !mbar_wait(bar + C::NSTAGE, 0u))) {
    if (lane == 0) atomicOr(L.err, (unsigned)KVQ_ERRF_WAIT_TIMEOUT);
    timed_out = true;
  }

  for (int it = 0; it < nmy; ++it) {
    if (it >= 1 && it - 1 + C::NSTAGE < nmy) {  // refill the stage of tile it - 1 (CTA-uniform test)
      if (__syncthreads_or(timed_out)) break;  // every warp is done with tile it - 1
      if (tid == 0) {
        issue(it - 1 + C::NSTAGE, (it - 1) % C::NSTAGE);
        ++issued;
      }
    }
    if (timed_out) continue;  // this warp reads nothing more; it still meets every barrier
    const int s = it % C::NSTAGE;
    if (__any_sync(0xffffffffu, !mbar_wait(bar + s, (uint32_t)(it / C::NSTAGE) & 1u))) {
      if (lane == 0) atomicOr(L.err, (unsigned)KVQ_ERRF_WAIT_TIMEOUT);
      timed_out = true;
      continue;
    }
    const uint8_t* bk = raw + s * stg;
    const uint8_t* bv = bk + sbK;
    const uint32_t bk_s = raw_s + s * stg, bv_s = bk_s + sbK;
    const int t0 = tstart + (it0 + it) * C::TT;

    // ---- logits of the group's two tokens
    float sc[2][G], vsc[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int tt = gid + x * C::NG, t = t0 + tt;
      const bool ok = t >= qa && t < qb;
      const float ks = ok ? lds_h2f(bk_s + cbK + 2 * tt) : 0.0f;
      vsc[x] = ok ? lds_h2f(bv_s + cbV + 2 * tt) : 0.0f;
      float F[C::SPL];
      uint32_t ko[C::SPL];
      polar_fields<BM, BP>(bk_s + tt * K.row_bytes, bk + tt * K.row_bytes, j, bmK, bpK, F, ko);
      float d[G];
#pragma unroll
      for (int h = 0; h < G; ++h) d[h] = 0.0f;
#pragma unroll
      for (int i = 0; i < C::SPL; ++i) {
        const float c = F[i] - kTwo23;
        const float2 cs = lds_f2(tk_s + ko[i]);
#pragma unroll
        for (int h = 0; h < G; ++h) d[h] = fmaf(c, fmaf(q2[h][i][1], cs.y, q2[h][i][0] * cs.x), d[h]);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = d[h];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        sc[x][h] = ok ? fmaf(ks, v, mu[h]) : -INFINITY;
      }
    }

    // ---- online softmax per head over the two tokens.  The running maximum moves only when a
    // logit passes it by more than kSlack (log2 units): the weights stay below 2^kSlack, and the
    // accumulators are rescaled rarely.
    float w[2][G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mn = fmaxf(sc[0][h], sc[1][h]);
      const float m1 = mn > m[h] + kSlack ? mn : m[h];  // m = -inf: the first finite logit
      const float al = m1 == m[h] ? 1.0f : ex2(m[h] - m1);
      if (__any_sync(0xffffffffu, al != 1.0f)) {
#pragma unroll
        for (int i = 0; i < C::SPL; ++i) {
          acc[h][i][0] *= al;
          acc[h][i][1] *= al;
        }
        l[h] *= al;
      }
      m[h] = m1;
      const float mb = m1 == -INFINITY ? 0.0f : m1;
      const float p0 = ex2(sc[0][h] - mb), p1 = ex2(sc[1][h] - mb);
      l[h] += p0 + p1;
      w[0][h] = p0 * vsc[0];
      w[1][h] = p1 * vsc[1];
    }

    // ---- O += p s_v c_f (cos, sin) for the group's two tokens
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int tt = gid + x * C::NG;
      float F[C::SPL];
      uint32_t ko[C::SPL];
      polar_fields<BM, BP>(bv_s + tt * V.row_bytes, bv + tt * V.row_bytes, j, bmV, bpV, F, ko);
      float w23[G];
#pragma unroll
      for (int h = 0; h < G; ++h) w23[h] = -w[x][h] * kTwo23;
#pragma unroll
      for (int i = 0; i < C::SPL; ++i) {
        const float2 cs = lds_f2(tv_s + ko[i]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float wc = fmaf(w[x][h], F[i], w23[h]);  // = w c exactly: F = 2^23 + c
          acc[h][i][0] = fmaf(wc, cs.x, acc[h][i][0]);
          acc[h][i][1] = fmaf(wc, cs.y, acc[h][i][1]);
        }
      }
    }
  }

  // After a timed-out wait the tiles issued may still be landing (and the table): wait, bounded
  // again, for the last tile issued into each stage before the buffers are reused or the CTA exits.
  timed_out = __syncthreads_or(timed_out);
  if (timed_out && tid == 0) {
    mbar_wait(bar + C::NSTAGE, 0u);
    for (int s = 0; s < C::NSTAGE; ++s) {
      const int last = issued - 1 - ((issued - 1 - s) % C::NSTAGE + C::NSTAGE) % C::NSTAGE;
      if (last >= 0) mbar_wait(bar + s, (uint32_t)(last / C::NSTAGE) & 1u);
    }
  }
  __syncthreads();  // the staging ring becomes the combine buffer

  // ---- combine the groups: within the warp by shuffles, then across warps in shared memory
  float* cmb = reinterpret_cast<float*>(raw);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float M = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], 8));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 16));
    const float f = m[h] == -INFINITY ? 0.0f : ex2(m[h] - M);
    float lw = l[h] * f;
    lw += __shfl_xor_sync(0xffffffffu, lw, 8);
    lw += __shfl_xor_sync(0xffffffffu, lw, 16);
    float* dst = cmb + (warp * G + h) * C::EP;
#pragma unroll
    for (int i = 0; i < C::SPL; ++i) {
      float a0 = acc[h][i][0] * f, a1 = acc[h][i][1] * f;
      a0 += __shfl_xor_sync(0xffffffffu, a0, 8);
      a1 += __shfl_xor_sync(0xffffffffu, a1, 8);
      a0 += __shfl_xor_sync(0xffffffffu, a0, 16);
      a1 += __shfl_xor_sync(0xffffffffu, a1, 16);
      if (lane < C::LPT) *reinterpret_cast<float2*>(dst + 2 * C::SPL * j + 2 * i) = make_float2(a0, a1);
    }
    if (lane == 0) {
      dst[D] = M;
      dst[D + 1] = lw;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += C::NT) {
    const int h = e / D, ch = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int wi = 0; wi < C::NW; ++wi) M = fmaxf(M, cmb[(wi * G + h) * C::EP + D]);
    float o = 0.0f, lsum = 0.0f;
#pragma unroll
    for (int wi = 0; wi < C::NW; ++wi) {
      const float* src = cmb + (wi * G + h) * C::EP;
      const float f = src[D] == -INFINITY ? 0.0f : ex2(src[D] - M);
      o = fmaf(src[ch], f, o);
      lsum = fmaf(src[D + 1], f, lsum);
    }
    float* P = work + (((long long)qi * L.Hq + kvh * G + h) * nsp_total + split) * (D + kPartStride);
    P[kPartStride + ch] = o;
    if (ch == 0) {
      P[0] = M;
      P[1] = lsum;
    }
  }
}
