// Tensor-core pass 1 of kvq_decode_attention for many queries over few sequences (GQA groups of 1
// or 2 with more queries than sequences, as in the proxy-query setup: "E21W" "What I tested", the
// post-RoPE keys at many positions of one text, each attending the keys before it), and for every
// format that has no register-decode instance.  The queries of one (sequence, kv-head) form a
// real M dimension, so a tile of keys and values is decoded once per CTA and shared by all of its
// query rows.
//
// Included by decode.cu inside namespace kvq (uses QueryRange, query_range, prepare_query, kLog2e,
// kMaxG, d_nf4, d_lloyd, d_ph_cos, d_ph_sin).  Same contract as the other pass-1 kernels: one
// log2-domain partial (m, l, o[D] in V's stored domain) per (query, head) and split.
//
// Queries.  mq_prep_kernel transforms each (query, kv-head) once (q' x sm_scale log2 e, as the
// other kernels build it, and the key-mean term) into a workspace row; the CTAs of the main kernel
// load their rows from there instead of each transforming them again.
//
// Rows.  A CTA holds QM = 64 rows, row r = (query q0 + r / G, head r % G); each warp owns a 16-row
// block (with head_dim 256 two warps share one, each accumulating half of the channels).  The
// transformed queries are split into fp16 hi + lo halves in shared memory.  A warp none of whose
// rows attends the current sequence skips the products.
//
// Tiles.  The packed bytes of a tile of TK = 32 tokens (codes, scales, zero points: contiguous
// ranges of the cache) are copied into shared memory by cp.async one tile ahead of their use.
// Every thread then decodes 8-element chunks of the staged rows into fp16 hi + lo halves of the
// exact stored-domain value (any format: code x scale, + zero, levels, polar m (cos phi, sin phi),
// ...; rows past the sequence's length are zero), so no format logic remains in the products.
// Scores S[16 rows x 8 tokens] = Q . K^T take three mma per 16 channels (hi.hi + lo.hi + hi.lo,
// ~22-bit products), fragments loaded by ldmatrix; each row masks its own causal range; the online
// softmax runs per row across the quad that shares it; the score fragments are reused directly as
// the A operand of O += P . V (hi + lo again), with V's B fragments loaded transposed (ldmatrix
// .trans).  Queries of different sequences in one CTA are served by one pass per sequence over
// that sequence's tiles, other rows masked.

// Format class of both sides, decoded without the format dispatch when known: FC_ANY (any
// format), FC_MINMAX (min-max int codes of 3 or 4 bits in groups of at least 8), FC_POLAR (rFFT
// polar).
enum MqFmtClass { FC_ANY = 0, FC_MINMAX = 1, FC_POLAR = 2 };

// Tile shapes per head_dim and format class.  The min-max class needs no level or phase tables and
// takes 16-token tiles, which fits two CTAs per SM at head_dim 256.
template <int D, int FC = FC_ANY>
struct MqCfg {
  static constexpr int CS = D >= 256 ? 2 : 1;      // warps sharing a 16-row block (channel split)
  static constexpr int RB = 4;                     // 16-row blocks per CTA
  static constexpr int NW = RB * CS;
  static constexpr int NT = NW * 32;
  static constexpr int QM = 16 * RB;               // rows per CTA
  static constexpr int TK = FC == FC_MINMAX ? 16 : 32;  // tokens per tile
  static constexpr int LD = D + 8;                 // halves per shared row: ldmatrix rows on distinct banks
  static constexpr int DC = D / CS;                // O channels per warp
  static constexpr int NB = DC / 8;                // O n-blocks per warp
  static constexpr int OFF_QH = 0;
  static constexpr int OFF_QL = OFF_QH + QM * LD * 2;
  static constexpr int OFF_KH = OFF_QL + QM * LD * 2;
  static constexpr int OFF_KL = OFF_KH + TK * LD * 2;
  static constexpr int OFF_VH = OFF_KL + TK * LD * 2;
  static constexpr int OFF_VL = OFF_VH + TK * LD * 2;
  static constexpr int OFF_META = OFF_VL + TK * LD * 2;          // per row: seq, qa, qb, q.mu
  static constexpr int OFF_TAB = OFF_META + QM * 4 * 4;          // NF4 16, Lloyd-Max 2 x 16, phase cos/sin 2 x 2 x 256
  static constexpr int TAB_BYTES = FC == FC_MINMAX ? 0 : (16 + 32 + 1024) * 4;
  static constexpr int OFF_RAW = OFF_TAB + TAB_BYTES;  // two staging buffers of packed tile bytes
  static constexpr int SMEM_MAX = 227 * 1024;
  static_assert(OFF_RAW % 16 == 0, "staging buffers must start 16-byte aligned");
  static_assert((LD * 2) % 16 == 0, "ldmatrix rows must stay 16-byte aligned");
};

__host__ __device__ __forceinline__ int mq_up16(int x) { return (x + 15) & ~15; }

// Staged bytes of one side for one tile: codes, then scales, then zero points, each range
// starting 16-byte aligned.
template <int TK>
__host__ __device__ __forceinline__ int mq_stage_bytes(const SideDev& S) {
  const int sc = S.scales ? mq_up16(TK * S.n_groups * 2) : 0;
  return mq_up16(TK * S.row_bytes) + sc + (S.zeros ? sc : 0);
}

// Dynamic shared memory of one decode_mq_kernel<D, FC> launch on `L`.
template <int D, int FC>
inline int mq_smem_bytes(const LayerDev& L) {
  using C = MqCfg<D, FC>;
  return C::OFF_RAW + 2 * (mq_stage_bytes<C::TK>(L.s[0]) + mq_stage_bytes<C::TK>(L.s[1]));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(__cvta_generic_to_global(src))
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(__cvta_generic_to_global(src))
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// n bytes from global `src` to shared `dst` (16-byte aligned): asynchronous 16- or 4-byte copies
// where the source's alignment allows them, the remaining bytes by plain loads and stores.
__device__ __forceinline__ void mq_stage(uint8_t* dst, const uint8_t* src, int n, int tid, int nt) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(src);
  int done = 0;
  if ((a & 15) == 0) {
    const int n16 = n >> 4;
    for (int i = tid; i < n16; i += nt) cp_async16(smem_u32(dst + 16 * i), src + 16 * i);
    done = n16 << 4;
  } else if ((a & 3) == 0) {
    const int n4 = n >> 2;
    for (int i = tid; i < n4; i += nt) cp_async4(smem_u32(dst + 4 * i), src + 4 * i);
    done = n4 << 2;
  }
  for (int i = done + tid; i < n; i += nt) dst[i] = src[i];
}

// Rows [rix0, rix0 + nrow) of side S (codes, scales, zero points) into the staging buffer `buf`.
template <int TK>
__device__ __forceinline__ void mq_stage_side(const SideDev& S, long long rix0, int nrow, uint8_t* buf, int tid,
                                              int nt) {
  const int cb = mq_up16(TK * S.row_bytes), sb = S.scales ? mq_up16(TK * S.n_groups * 2) : 0;
  mq_stage(buf, S.codes + rix0 * S.row_bytes, nrow * S.row_bytes, tid, nt);
  if (S.scales)
    mq_stage(buf + cb, reinterpret_cast<const uint8_t*>(S.scales + rix0 * S.n_groups), nrow * S.n_groups * 2, tid, nt);
  if (S.zeros)
    mq_stage(buf + cb + sb, reinterpret_cast<const uint8_t*>(S.zeros + rix0 * S.n_groups), nrow * S.n_groups * 2,
             tid, nt);
}

// The n (<= 8) bytes at p as a little-endian word: one load when p is aligned for it.
__device__ __forceinline__ uint64_t mq_bytes(const uint8_t* p, int n) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  if (n == 4 && (a & 3) == 0) return *reinterpret_cast<const uint32_t*>(p);
  if (n == 2 && (a & 1) == 0) return *reinterpret_cast<const uint16_t*>(p);
  if (n == 8 && (a & 7) == 0) return *reinterpret_cast<const unsigned long long*>(p);
  uint64_t w = 0;
  for (int i = 0; i < n; ++i) w |= (uint64_t)p[i] << (8 * i);
  return w;
}

// The 64 bits that start at bit `bit` of the staged bytes at p (LSB-first), from three aligned
// 32-bit shared-memory words.  May read up to 11 bytes past the field: the staging buffers are
// followed by more staged data, so the reads stay inside the CTA's shared memory.
__device__ __forceinline__ uint64_t mq_bits64(const uint8_t* p, int bit) {
  const uint8_t* a = p + (bit >> 3);
  const uint32_t* w = reinterpret_cast<const uint32_t*>(reinterpret_cast<uintptr_t>(a) & ~uintptr_t(3));
  const int sh = (int)((reinterpret_cast<uintptr_t>(a) & 3) * 8) + (bit & 7);  // 0 .. 31
  const uint32_t w0 = w[0], w1 = w[1], w2 = w[2];
  const uint32_t lo = __funnelshift_r(w0, w1, sh), hi = __funnelshift_r(w1, w2, sh);
  return ((uint64_t)hi << 32) | lo;
}

// Polar slots j0 / 2 .. j0 / 2 + 3 of a staged row as (m cos phi, m sin phi) pairs, as polar_slot
// computes them: the magnitude fields, then the phase fields, read at once.
__device__ __forceinline__ void mq_chunk_polar(const SideDev& S, const uint8_t* row, const __half* sc, int j0,
                                               float* v, const float* cs, const float* sn) {
  const int bm = S.bits, bp = S.bits2, f0 = j0 >> 1;
  const uint64_t mw = mq_bits64(row, f0 * bm), pw = mq_bits64(row, 64 * bm + f0 * bp);
  const uint32_t mm = (1u << bm) - 1u, pm = (1u << bp) - 1u;
  const float s = __half2float(sc[0]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float m = (float)(uint32_t)((mw >> (i * bm)) & mm) * s;
    const int k = (int)((pw >> (i * bp)) & pm);
    v[2 * i] = __fmul_rn(m, cs[k]);
    v[2 * i + 1] = __fmul_rn(m, sn[k]);
  }
}

// Stored-domain values of elements j0 .. j0 + 7 (j0 % 8 == 0) of one staged row, with the same
// arithmetic as stored_value / polar_slot (polar: slots j0 / 2 .. j0 / 2 + 3, (cos, sin) parts).
__device__ __forceinline__ void mq_chunk(const SideDev& S, const uint8_t* row, const __half* sc, const __half* zr,
                                         int j0, float* v, const float* nf4, const float* lloyd, const float* cs,
                                         const float* sn) {
  const int f = S.fmt;
  if (f == KVQ_FMT_FP16) {
    const uint4 w = *reinterpret_cast<const uint4*>(row + 2 * j0);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __half22float2(u2h(u[i]));
      v[2 * i] = x.x;
      v[2 * i + 1] = x.y;
    }
    return;
  }
  if (f == KVQ_FMT_POLAR) {
    mq_chunk_polar(S, row, sc, j0, v, cs, sn);
    return;
  }
  if (f == KVQ_FMT_TERNARY || f == KVQ_FMT_SORTED) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = stored_value(S, row, sc, zr, j0 + i, nf4, lloyd);
    return;
  }
  const int b = f == KVQ_FMT_NF4 ? 4 : (f == KVQ_FMT_SIGN ? 1 : S.bits);
  const uint64_t w = mq_bytes(row + b * (j0 >> 3), b);
  const uint32_t M = (1u << b) - 1u;
  if (f == KVQ_FMT_CART) {
    const float d = __half2float(sc[0]);
    const int half = 1 << (b - 1);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (float)((int)((w >> (b * i)) & M) - half) * d;
    return;
  }
  const bool one = S.group >= 8;  // the chunk lies in one group
  const int g0 = j0 / S.group;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = (int)((w >> (b * i)) & M);
    const int g = one ? g0 : (j0 + i) / S.group;
    const float d = __half2float(sc[g]);
    float x;
    if (f == KVQ_FMT_INT) {
      if (S.scale_mode == KVQ_SCALE_MINMAX) x = __fadd_rn(__half2float(zr[g]), (float)c * d);
      else if (S.scale_mode == KVQ_SCALE_SYMMETRIC) x = ((float)c - 0.5f * (float)M) * d;
      else x = (float)(c - (1 << (b - 1))) * d;
    } else if (f == KVQ_FMT_LLOYD) {
      x = lloyd[c] * d;
    } else if (f == KVQ_FMT_NF4) {
      x = nf4[c] * d;
    } else {  // sign
      x = c ? d : -d;
    }
    v[i] = x;
  }
}

// mq_chunk for a side known to hold min-max int codes of 3 or 4 bits in groups of at least 8
// (the config-2 formats): the same arithmetic without the format dispatch.
__device__ __forceinline__ void mq_chunk_minmax(const SideDev& S, const uint8_t* row, const __half* sc,
                                                const __half* zr, int j0, float* v) {
  const int b = S.bits;
  const uint64_t w = mq_bytes(row + b * (j0 >> 3), b);
  const uint32_t M = (1u << b) - 1u;
  const int g = j0 / S.group;
  const float d = __half2float(sc[g]), z = __half2float(zr[g]);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __fadd_rn(z, (float)(int)((w >> (b * i)) & M) * d);
}

// 8 values as fp16 hi halves and the fp16 roundings of their remainders, 16 bytes each.
__device__ __forceinline__ void mq_store8(__half* hi, __half* lo, int idx, const float* v) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 a = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
    const float2 af = __half22float2(a);
    h[i] = h2u(a);
    l[i] = h2u(__floats2half2_rn(v[2 * i] - af.x, v[2 * i + 1] - af.y));
  }
  *reinterpret_cast<uint4*>(hi + idx) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(lo + idx) = make_uint4(l[0], l[1], l[2], l[3]);
}

// Transformed queries of one (query, kv-head): row (qi, kvh G + h) of `prep` holds the key-mean
// term (x sm_scale log2 e) at 0 and q'[D] from kPartStride on.
template <int D>
__global__ void __launch_bounds__(256) mq_prep_kernel(LayerDev L, const __half* __restrict__ q,
                                                      const int* __restrict__ seq_ids,
                                                      const int* __restrict__ kv_len, float* __restrict__ prep) {
  __shared__ float qt[kMaxG * D], qa[kMaxG * D];
  const int kvh = blockIdx.x, qi = blockIdx.y, G = L.Hq / L.Hkv, tid = threadIdx.x;
  const SideDev& K = L.s[0];
  if (tid == 0 && kvh == 0) {  // a sequence id out of range attends nothing; report it
    const int s = seq_ids ? seq_ids[qi] : qi;
    if (s < 0 || s >= L.B) atomicOr(L.err, (unsigned)KVQ_ERRF_SEQ_ID);
  }
  prepare_query<D>(L, q, qi, kvh, G, qt, qa);  // synchronizes internally
  float* dst = prep + ((long long)qi * L.Hq + kvh * G) * (D + kPartStride);
  for (int e = tid; e < G * D; e += blockDim.x) dst[(e / D) * (D + kPartStride) + kPartStride + e % D] = qt[e];
  if (tid < G) {
    float mu = 0.0f;
    if (K.mean_sub) {
      const QueryRange R = query_range<false>(L, qi, seq_ids, kv_len);
      const __half* qp = q + query_row(L, qi, kvh, G, tid) * D;
      const __half* mp = K.kmean + ((long long)R.seq * L.Hkv + kvh) * D;
      for (int j = 0; j < D; ++j) mu = fmaf(__half2float(qp[j]), __half2float(mp[j]), mu);
    }
    dst[tid * (D + kPartStride)] = mu * (L.sm_scale * kLog2e);
  }
}

template <int D, int FC = FC_ANY>
__global__ void __launch_bounds__(MqCfg<D, FC>::NT) decode_mq_kernel(LayerDev L, const float* __restrict__ prep,
                                                                 const int* __restrict__ seq_ids,
                                                                 const int* __restrict__ kv_len, float* __restrict__ work,
                                                                 int n_split, int nsp_total, int n_q) {
  using C = MqCfg<D, FC>;
  extern __shared__ __align__(128) unsigned char smem[];
  __half* Qh = reinterpret_cast<__half*>(smem + C::OFF_QH);
  __half* Ql = reinterpret_cast<__half*>(smem + C::OFF_QL);
  __half* Kh = reinterpret_cast<__half*>(smem + C::OFF_KH);
  __half* Kl = reinterpret_cast<__half*>(smem + C::OFF_KL);
  __half* Vh = reinterpret_cast<__half*>(smem + C::OFF_VH);
  __half* Vl = reinterpret_cast<__half*>(smem + C::OFF_VL);
  int* r_seq = reinterpret_cast<int*>(smem + C::OFF_META);
  int* r_qa = r_seq + C::QM;
  int* r_qb = r_qa + C::QM;
  float* r_mu = reinterpret_cast<float*>(r_qb + C::QM);
  float* t_nf4 = reinterpret_cast<float*>(smem + C::OFF_TAB);
  float* t_lk = t_nf4 + 16;
  float* t_lv = t_lk + 16;
  float* t_kc = t_lv + 16;
  float* t_ks = t_kc + 256;
  float* t_vc = t_ks + 256;
  float* t_vs = t_vc + 256;
  uint8_t* raw = smem + C::OFF_RAW;
  __shared__ int pass_seq[MqCfg<D, FC>::QM];
  __shared__ int n_pass;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int split = blockIdx.x, kvh = blockIdx.y;
  const int G = L.Hq / L.Hkv, QPB = C::QM / G;
  const int q0 = blockIdx.z * QPB;
  const SideDev& K = L.s[0];
  const SideDev& V = L.s[1];
  const int stK = mq_stage_bytes<C::TK>(K), stV = mq_stage_bytes<C::TK>(V);
  const int cbK = mq_up16(C::TK * K.row_bytes), sbK = K.scales ? mq_up16(C::TK * K.n_groups * 2) : 0;
  const int cbV = mq_up16(C::TK * V.row_bytes), sbV = V.scales ? mq_up16(C::TK * V.n_groups * 2) : 0;

  // ---- tables (none for the min-max class)
  if constexpr (FC != FC_MINMAX) {
  if (tid < 16) t_nf4[tid] = d_nf4[tid];
  if (K.fmt == KVQ_FMT_LLOYD && tid < 16) t_lk[tid] = d_lloyd[K.bits - 2][tid];
  if (V.fmt == KVQ_FMT_LLOYD && tid < 16) t_lv[tid] = d_lloyd[V.bits - 2][tid];
  if (K.fmt == KVQ_FMT_POLAR)
    for (int k = tid; k < (1 << K.bits2); k += C::NT) {
      t_kc[k] = d_ph_cos[(1 << K.bits2) - 2 + k];
      t_ks[k] = d_ph_sin[(1 << K.bits2) - 2 + k];
    }
  if (V.fmt == KVQ_FMT_POLAR)
    for (int k = tid; k < (1 << V.bits2); k += C::NT) {
      t_vc[k] = d_ph_cos[(1 << V.bits2) - 2 + k];
      t_vs[k] = d_ph_sin[(1 << V.bits2) - 2 + k];
    }
  }

  // ---- rows: the prepared queries as fp16 hi + lo; per-row sequence, causal range, key-mean term
  for (int e = tid; e < C::QM * (D / 4); e += C::NT) {
    const int r = e / (D / 4), j = (e % (D / 4)) * 4;
    const int qi = q0 + r / G, h = r % G;
    float4 x = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (qi < n_q)
      x = *reinterpret_cast<const float4*>(prep + ((long long)qi * L.Hq + kvh * G + h) * (D + kPartStride) +
                                           kPartStride + j);
    const __half2 a = __floats2half2_rn(x.x, x.y), b = __floats2half2_rn(x.z, x.w);
    const float2 af = __half22float2(a), bf = __half22float2(b);
    *reinterpret_cast<uint2*>(Qh + r * C::LD + j) = make_uint2(h2u(a), h2u(b));
    *reinterpret_cast<uint2*>(Ql + r * C::LD + j) =
        make_uint2(h2u(__floats2half2_rn(x.x - af.x, x.y - af.y)), h2u(__floats2half2_rn(x.z - bf.x, x.w - bf.y)));
  }
  if (tid < C::QM) {
    const int r = tid, qi = q0 + r / G, h = r % G;
    if (qi < n_q) {
      const QueryRange R = query_range<false>(L, qi, seq_ids, kv_len);
      r_seq[r] = R.qb > R.qa ? R.seq : -1;
      r_qa[r] = R.qa;
      r_qb[r] = R.qb;
      r_mu[r] = prep[((long long)qi * L.Hq + kvh * G + h) * (D + kPartStride)];
    } else {
      r_seq[r] = -1;
      r_qa[r] = r_qb[r] = 0;
      r_mu[r] = 0.0f;
    }
  }
  __syncthreads();
  // distinct sequences among the rows that attend anything (in row order)
  if (tid == 0) {
    int n = 0;
    for (int r = 0; r < C::QM; ++r) {
      const int s = r_seq[r];
      if (s < 0) continue;
      bool seen = false;
      for (int i = 0; i < n; ++i) seen |= pass_seq[i] == s;
      if (!seen) pass_seq[n++] = s;
    }
    n_pass = n;
  }
  __syncthreads();

  const int rb = warp / C::CS, chh = warp % C::CS;
  const int row0 = rb * 16 + g, row1 = row0 + 8;
  const int ch0 = chh * C::DC;
  const uint32_t qh_s = smem_u32(Qh), ql_s = smem_u32(Ql), kh_s = smem_u32(Kh), kl_s = smem_u32(Kl);
  const uint32_t vh_s = smem_u32(Vh), vl_s = smem_u32(Vl);
  // ldmatrix lane addresses (halves): A (rows, k), K B (token, k), V B transposed (token, channel)
  const int a_off = (rb * 16 + (lane & 15)) * C::LD + (lane >> 4) * 8;
  const int k_off = ((lane & 7) + (lane >> 4) * 8) * C::LD + ((lane >> 3) & 1) * 8;
  const int v_off = ((lane & 7) + ((lane >> 3) & 1) * 8) * C::LD + (lane >> 4) * 8;

  float o[C::NB][4];
#pragma unroll
  for (int i = 0; i < C::NB; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;
  const float mu0 = r_mu[row0], mu1 = r_mu[row1];

  for (int p = 0; p < n_pass; ++p) {
    const int seq = pass_seq[p];
    int lo = 1 << 30, hi = 0;
    for (int r = 0; r < C::QM; ++r)
      if (r_seq[r] == seq) {
        lo = min(lo, r_qa[r]);
        hi = max(hi, r_qb[r]);
      }
    const int len = L.seq_len[seq];
    const int tstart = (lo / C::TK) * C::TK;
    const int ntiles = (hi - tstart + C::TK - 1) / C::TK;
    const int per = (ntiles + n_split - 1) / n_split;
    const int it0 = split * per, it1 = min(ntiles, it0 + per);
    const bool a0 = r_seq[row0] == seq, a1 = r_seq[row1] == seq;
    const bool wact = __any_sync(0xffffffffu, a0 || a1);  // some row of this warp's block attends seq
    const int qa0 = r_qa[row0], qb0 = a0 ? r_qb[row0] : 0, qa1 = r_qa[row1], qb1 = a1 ? r_qb[row1] : 0;
    const long long u = (long long)seq * L.Hkv + kvh;
    // tile it's packed rows (those below the length) into staging buffer `buf`
    auto stage = [&](int it, int buf) {
      const int t0 = tstart + it * C::TK;
      const int nrow = min(C::TK, len - t0);
      uint8_t* bk = raw + buf * (stK + stV);
      mq_stage_side<C::TK>(K, u * L.Tcap + t0, nrow, bk, tid, C::NT);
      mq_stage_side<C::TK>(V, u * L.Tcap + t0, nrow, bk + stK, tid, C::NT);
      cp_async_commit();
    };
    if (it0 < it1) stage(it0, 0);
    for (int it = it0; it < it1; ++it) {
      const int cur = (it - it0) & 1;
      if (it + 1 < it1) {
        stage(it + 1, cur ^ 1);  // its buffer was last read by the decode of tile it - 1
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();  // tile it staged; every warp is done with the previous tile's K and V
      const int t0 = tstart + it * C::TK;
      // ---- decode the staged tile: exact stored values as fp16 hi + lo (rows past the length: 0)
      {
        const uint8_t* bk = raw + cur * (stK + stV);
        const uint8_t* bv = bk + stK;
        const __half* sk = reinterpret_cast<const __half*>(bk + cbK);
        const __half* zk = K.zeros ? reinterpret_cast<const __half*>(bk + cbK + sbK) : nullptr;
        const __half* sv = reinterpret_cast<const __half*>(bv + cbV);
        const __half* zv = V.zeros ? reinterpret_cast<const __half*>(bv + cbV + sbV) : nullptr;
        for (int e = tid; e < C::TK * (D / 8); e += C::NT) {
          const int t = e / (D / 8), j0 = (e % (D / 8)) * 8;
          float kv[8], vv[8];
          if (t0 + t < len) {
            if constexpr (FC == FC_MINMAX) {
              mq_chunk_minmax(K, bk + t * K.row_bytes, sk + t * K.n_groups, zk + t * K.n_groups, j0, kv);
              mq_chunk_minmax(V, bv + t * V.row_bytes, sv + t * V.n_groups, zv + t * V.n_groups, j0, vv);
            } else if constexpr (FC == FC_POLAR) {
              mq_chunk_polar(K, bk + t * K.row_bytes, sk + t * K.n_groups, j0, kv, t_kc, t_ks);
              mq_chunk_polar(V, bv + t * V.row_bytes, sv + t * V.n_groups, j0, vv, t_vc, t_vs);
            } else {
              mq_chunk(K, bk + t * K.row_bytes, sk + t * K.n_groups, zk ? zk + t * K.n_groups : nullptr, j0, kv,
                       t_nf4, t_lk, t_kc, t_ks);
              mq_chunk(V, bv + t * V.row_bytes, sv + t * V.n_groups, zv ? zv + t * V.n_groups : nullptr, j0, vv,
                       t_nf4, t_lv, t_vc, t_vs);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) kv[i] = vv[i] = 0.0f;
          }
          mq_store8(Kh, Kl, t * C::LD + j0, kv);
          mq_store8(Vh, Vl, t * C::LD + j0, vv);
        }
      }
      __syncthreads();
      if (wact) {
        // ---- scores for this warp's 16 rows x 32 tokens
        float s[C::TK / 8][4];
#pragma unroll
        for (int nb = 0; nb < C::TK / 8; ++nb) {
          s[nb][0] = s[nb][1] = mu0;
          s[nb][2] = s[nb][3] = mu1;
        }
#pragma unroll 4
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t ah[4], al[4];
          ldsm_x4(qh_s + 2 * (a_off + ks * 16), ah[0], ah[1], ah[2], ah[3]);
          ldsm_x4(ql_s + 2 * (a_off + ks * 16), al[0], al[1], al[2], al[3]);
#pragma unroll
          for (int nb = 0; nb < C::TK / 8; nb += 2) {
            uint32_t bh[4], bl[4];
            ldsm_x4(kh_s + 2 * (k_off + nb * 8 * C::LD + ks * 16), bh[0], bh[1], bh[2], bh[3]);
            ldsm_x4(kl_s + 2 * (k_off + nb * 8 * C::LD + ks * 16), bl[0], bl[1], bl[2], bl[3]);
            mma16816(s[nb], ah[0], ah[1], ah[2], ah[3], bh[0], bh[1]);
            mma16816(s[nb], al[0], al[1], al[2], al[3], bh[0], bh[1]);
            mma16816(s[nb], ah[0], ah[1], ah[2], ah[3], bl[0], bl[1]);
            mma16816(s[nb + 1], ah[0], ah[1], ah[2], ah[3], bh[2], bh[3]);
            mma16816(s[nb + 1], al[0], al[1], al[2], al[3], bh[2], bh[3]);
            mma16816(s[nb + 1], ah[0], ah[1], ah[2], ah[3], bl[2], bl[3]);
          }
        }
        // ---- causal masks per row, online softmax per row (the quad c = 0..3 shares a row)
        float tm0 = -INFINITY, tm1 = -INFINITY;
#pragma unroll
        for (int nb = 0; nb < C::TK / 8; ++nb) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tok = t0 + nb * 8 + 2 * c + e;
            if (!(tok >= qa0 && tok < qb0)) s[nb][e] = -INFINITY;
            if (!(tok >= qa1 && tok < qb1)) s[nb][2 + e] = -INFINITY;
            tm0 = fmaxf(tm0, s[nb][e]);
            tm1 = fmaxf(tm1, s[nb][2 + e]);
          }
        }
        tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, 1));
        tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, 2));
        tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, 1));
        tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, 2));
        const float n0 = fmaxf(m0, tm0), n1 = fmaxf(m1, tm1);
        const float al0 = n0 == -INFINITY ? 1.0f : ex2(m0 - n0), al1 = n1 == -INFINITY ? 1.0f : ex2(m1 - n1);
        m0 = n0;
        m1 = n1;
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int i = 0; i < C::NB; ++i) {
          o[i][0] *= al0;
          o[i][1] *= al0;
          o[i][2] *= al1;
          o[i][3] *= al1;
        }
#pragma unroll
        for (int nb = 0; nb < C::TK / 8; ++nb) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            s[nb][e] = m0 == -INFINITY ? 0.0f : ex2(s[nb][e] - m0);
            s[nb][2 + e] = m1 == -INFINITY ? 0.0f : ex2(s[nb][2 + e] - m1);
            l0 += s[nb][e];
            l1 += s[nb][2 + e];
          }
        }
        // ---- O += P . V: the score fragments of tokens [16 kk, 16 kk + 16) are P's A fragment
#pragma unroll
        for (int kk = 0; kk < C::TK / 16; ++kk) {
          uint32_t ph[4], pl[4];
          const float* f[4] = {&s[2 * kk][0], &s[2 * kk][2], &s[2 * kk + 1][0], &s[2 * kk + 1][2]};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const __half2 h = __floats2half2_rn(f[i][0], f[i][1]);
            const float2 hf = __half22float2(h);
            ph[i] = h2u(h);
            pl[i] = h2u(__floats2half2_rn(f[i][0] - hf.x, f[i][1] - hf.y));
          }
#pragma unroll
          for (int nb = 0; nb < C::NB; nb += 2) {
            uint32_t bh[4], bl[4];
            const int vo = v_off + kk * 16 * C::LD + ch0 + nb * 8;
            ldsm_x4_t(vh_s + 2 * vo, bh[0], bh[1], bh[2], bh[3]);
            ldsm_x4_t(vl_s + 2 * vo, bl[0], bl[1], bl[2], bl[3]);
            mma16816(o[nb], ph[0], ph[1], ph[2], ph[3], bh[0], bh[1]);
            mma16816(o[nb], pl[0], pl[1], pl[2], pl[3], bh[0], bh[1]);
            mma16816(o[nb], ph[0], ph[1], ph[2], ph[3], bl[0], bl[1]);
            mma16816(o[nb + 1], ph[0], ph[1], ph[2], ph[3], bh[2], bh[3]);
            mma16816(o[nb + 1], pl[0], pl[1], pl[2], pl[3], bh[2], bh[3]);
            mma16816(o[nb + 1], ph[0], ph[1], ph[2], ph[3], bl[2], bl[3]);
          }
        }
      }
    }
  }

  // ---- partials: (m, l, o) per row; the quad's l parts summed
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = half ? row1 : row0;
    const int qi = q0 + r / G, h = r % G;
    if (qi >= n_q) continue;
    float* P = work + (((long long)qi * L.Hq + kvh * G + h) * nsp_total + split) * (D + kPartStride);
    if (c == 0 && chh == 0) {
      P[0] = half ? m1 : m0;
      P[1] = half ? l1 : l0;
    }
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb)
      *reinterpret_cast<float2*>(P + kPartStride + ch0 + nb * 8 + 2 * c) =
          make_float2(o[nb][2 * half], o[nb][2 * half + 1]);
  }
}
