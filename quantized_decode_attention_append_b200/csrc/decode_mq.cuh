// Tensor-core pass 1 of kvq_decode_attention for many queries over few sequences: GQA groups of 1
// or 2 with more queries than sequences, as in the proxy-query setup ("E21W" "What I tested": the
// post-RoPE keys at many positions of one text, each attending the keys before it).  There the
// queries of one (sequence, kv-head) form a real M dimension, so a tile of keys and values is
// decoded once per CTA and shared by all of its query rows.
//
// Included by decode.cu inside namespace kvq (uses QueryRange, query_range, prepare_query, kLog2e,
// kMaxG, d_nf4, d_lloyd, d_ph_cos, d_ph_sin).  Same contract as the other pass-1 kernels: one
// log2-domain partial (m, l, o[D] in V's stored domain) per (query, head) and split.
//
// Rows.  A CTA holds QM = 64 rows, row r = (query q0 + r / G, head r % G); each warp owns a 16-row
// block (with head_dim 256 two warps share one, each accumulating half of the channels).  The
// transformed queries (q' x sm_scale log2 e, as the other kernels build them) are split into fp16
// hi + lo halves in shared memory.
//
// Tiles.  Per tile of TK = 32 tokens every thread decodes its share of the K and V rows into shared
// memory as fp16 hi + lo halves of the exact stored-domain value (any format: code x scale, + zero,
// levels, polar m (cos phi, sin phi), ...; rows past the sequence's length are zero), so no format
// logic remains in the products.  Scores S[16 rows x 8 tokens] = Q . K^T take three mma per 16
// channels (hi.hi + lo.hi + hi.lo, ~22-bit products), fragments loaded by ldmatrix; each row masks
// its own causal range; the online softmax runs per row across the quad that shares it; the score
// fragments are reused directly as the A operand of O += P . V (hi + lo again), with V's B
// fragments loaded transposed (ldmatrix .trans).  Queries of different sequences in one CTA are
// served by one pass per sequence over that sequence's tiles, other rows masked.

template <int D>
struct MqCfg {
  static constexpr int CS = D >= 256 ? 2 : 1;      // warps sharing a 16-row block (channel split)
  static constexpr int RB = 4;                     // 16-row blocks per CTA
  static constexpr int NW = RB * CS;
  static constexpr int NT = NW * 32;
  static constexpr int QM = 16 * RB;               // rows per CTA
  static constexpr int TK = 32;                    // tokens per tile
  static constexpr int LD = D + 8;                 // halves per shared row: ldmatrix rows on distinct banks
  static constexpr int DC = D / CS;                // O channels per warp
  static constexpr int NB = DC / 8;                // O n-blocks per warp
  static constexpr int OFF_QH = 0;
  static constexpr int OFF_QL = OFF_QH + QM * LD * 2;
  static constexpr int OFF_KH = OFF_QL + QM * LD * 2;
  static constexpr int OFF_KL = OFF_KH + TK * LD * 2;
  static constexpr int OFF_VH = OFF_KL + TK * LD * 2;
  static constexpr int OFF_VL = OFF_VH + TK * LD * 2;
  static constexpr int OFF_QT = OFF_VL + TK * LD * 2;         // fp32 [kMaxG][D] transformed query
  static constexpr int OFF_QA = OFF_QT + kMaxG * D * 4;       // fp32 [kMaxG][D] (prepare_query's raw copy)
  static constexpr int OFF_META = OFF_QA + kMaxG * D * 4;     // per row: seq, qa, qb, q.mu
  static constexpr int OFF_TAB = OFF_META + QM * 4 * 4;       // NF4 16, Lloyd-Max 2 x 16, phase cos/sin 2 x 2 x 256
  static constexpr int SMEM = OFF_TAB + (16 + 32 + 1024) * 4;
  static_assert(SMEM <= 227 * 1024, "multi-query tiles exceed one CTA's shared memory");
  static_assert((LD * 2) % 16 == 0, "ldmatrix rows must stay 16-byte aligned");
};

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

// Stored-domain value of element j of a row of any format (polar: slot j / 2, cos or sin part).
__device__ __forceinline__ float mq_value(const SideDev& S, const uint8_t* __restrict__ row, const __half* __restrict__ sc,
                                          const __half* __restrict__ zr, int j, const float* nf4, const float* lloyd,
                                          const float* cs, const float* sn) {
  if (S.fmt == KVQ_FMT_POLAR) {
    const float2 ab = polar_slot(S, row, sc, j >> 1, cs, sn);
    return (j & 1) ? ab.y : ab.x;
  }
  return stored_value(S, row, sc, zr, j, nf4, lloyd);
}

__device__ __forceinline__ void split_store(__half* hi, __half* lo, int idx, float v) {
  const __half h = __float2half_rn(v);
  hi[idx] = h;
  lo[idx] = __float2half_rn(v - __half2float(h));
}

template <int D>
__global__ void __launch_bounds__(MqCfg<D>::NT) decode_mq_kernel(LayerDev L, const __half* __restrict__ q,
                                                                 const int* __restrict__ seq_ids,
                                                                 const int* __restrict__ kv_len, float* __restrict__ work,
                                                                 int n_split, int nsp_total, int n_q) {
  using C = MqCfg<D>;
  extern __shared__ __align__(128) unsigned char smem[];
  __half* Qh = reinterpret_cast<__half*>(smem + C::OFF_QH);
  __half* Ql = reinterpret_cast<__half*>(smem + C::OFF_QL);
  __half* Kh = reinterpret_cast<__half*>(smem + C::OFF_KH);
  __half* Kl = reinterpret_cast<__half*>(smem + C::OFF_KL);
  __half* Vh = reinterpret_cast<__half*>(smem + C::OFF_VH);
  __half* Vl = reinterpret_cast<__half*>(smem + C::OFF_VL);
  float* qt = reinterpret_cast<float*>(smem + C::OFF_QT);
  float* qraw = reinterpret_cast<float*>(smem + C::OFF_QA);
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
  __shared__ int pass_seq[MqCfg<D>::QM];
  __shared__ int n_pass;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, c = lane & 3;
  const int split = blockIdx.x, kvh = blockIdx.y;
  const int G = L.Hq / L.Hkv, QPB = C::QM / G;
  const int q0 = blockIdx.z * QPB;
  const SideDev& K = L.s[0];
  const SideDev& V = L.s[1];

  // ---- tables
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

  // ---- rows: transformed queries as fp16 hi + lo; per-row sequence and causal range
  for (int qq = 0; qq < QPB; ++qq) {
    const int qi = q0 + qq;  // uniform over the CTA
    if (qi < n_q) {
      prepare_query<D>(L, q, qi, kvh, G, qt, qraw);  // synchronizes internally
      for (int e = tid; e < G * D; e += C::NT) {
        const int r = qq * G + e / D, j = e % D;
        split_store(Qh, Ql, r * C::LD + j, qt[e]);
      }
      if (tid < G) {
        const int r = qq * G + tid;
        const QueryRange R = query_range(L, qi, seq_ids, kv_len);
        r_seq[r] = R.qb > R.qa ? R.seq : -1;
        r_qa[r] = R.qa;
        r_qb[r] = R.qb;
        float mu = 0.0f;
        if (K.mean_sub) {
          const __half* qp = q + query_row(L, qi, kvh, G, tid) * D;
          const __half* mp = K.kmean + ((long long)R.seq * L.Hkv + kvh) * D;
          for (int j = 0; j < D; ++j) mu = fmaf(__half2float(qp[j]), __half2float(mp[j]), mu);
        }
        r_mu[r] = mu * (L.sm_scale * kLog2e);
      }
    } else {
      for (int e = tid; e < G * D; e += C::NT) {
        const int r = qq * G + e / D, j = e % D;
        split_store(Qh, Ql, r * C::LD + j, 0.0f);
      }
      if (tid < G) {
        const int r = qq * G + tid;
        r_seq[r] = -1;
        r_qa[r] = r_qb[r] = 0;
        r_mu[r] = 0.0f;
      }
    }
    __syncthreads();  // qt / qraw are reused for the next query
  }
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
    const int qa0 = r_qa[row0], qb0 = a0 ? r_qb[row0] : 0, qa1 = r_qa[row1], qb1 = a1 ? r_qb[row1] : 0;
    const long long u = (long long)seq * L.Hkv + kvh;
    for (int it = it0; it < it1; ++it) {
      const int t0 = tstart + it * C::TK;
      // ---- decode the tile: exact stored values as fp16 hi + lo (rows past the length: 0)
      for (int e = tid; e < C::TK * D; e += C::NT) {
        const int t = e / D, j = e % D, tok = t0 + t;
        float kv = 0.0f, vv = 0.0f;
        if (tok < len) {
          const long long rix = u * L.Tcap + tok;
          kv = mq_value(K, K.codes + rix * K.row_bytes, K.scales + rix * K.n_groups,
                        K.zeros ? K.zeros + rix * K.n_groups : nullptr, j, t_nf4, t_lk, t_kc, t_ks);
          vv = mq_value(V, V.codes + rix * V.row_bytes, V.scales + rix * V.n_groups,
                        V.zeros ? V.zeros + rix * V.n_groups : nullptr, j, t_nf4, t_lv, t_vc, t_vs);
        }
        split_store(Kh, Kl, t * C::LD + j, kv);
        split_store(Vh, Vl, t * C::LD + j, vv);
      }
      __syncthreads();
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
      __syncthreads();  // the next tile overwrites K and V
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
