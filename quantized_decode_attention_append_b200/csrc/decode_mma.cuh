// Tensor-core pass 1 of kvq_decode_attention for GQA groups of up to 4 query heads.
//
// Included by decode.cu.  Same contract as the generic pass: one CTA per (query, kv-head, split)
// writes one log2-domain partial (m, l, o[D] in V's stored domain); the four warps' partials are
// combined in shared memory first.
//
// Work mapping (mma.sync m16n8k16, fp16 operands, fp32 accumulate):
//   scores  S[16 tokens x 8] = K[16 x 16 ch] . Q'^T[16 ch x 8]; the 8 columns are 4 heads x
//           (hi, lo) fp16 halves of the pre-transformed query, so the logit keeps ~22 bits; one
//           accumulator per K group, scaled by the group's fp16 scale afterwards.
//   values  O^T[16 ch x 8] += V^T[16 ch x 16 tokens] . P'^T[16 tokens x 8]; columns are 4 heads x
//           (hi, lo) halves of p * d_v (the V group scale folded into the probability).
// K/V codes are turned into exact fp16 operands in registers: b-bit integer fields with the
// 0x6400 exponent trick (1024 + code, then - (1024 + 2^(b-1))), NF4 through a byte -> level-pair
// table in shared memory (a register-resident table read by byte permutes measured slower: it
// costs more instructions than the shared-memory lookups save), fp16 V by byte permutes.  Because a dot product does not depend on the order of its
// terms, each thread reads a contiguous chunk of a row and the query is permuted to match.
// Tiles of keys are staged with cp.async (16-byte copies) in a multi-stage pipeline.
//
// This fragment is included inside namespace kvq (it uses QueryRange, kLog2e and d_nf4).

enum CodeFmt { CF_INT2 = 2, CF_INT4 = 4, CF_NF4 = 16, CF_FP16 = 32 };

template <int F> struct CodeBits { static constexpr int v = F == CF_NF4 ? 4 : (F == CF_FP16 ? 16 : F); };

__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// (x & mask) | magic
__device__ __forceinline__ uint32_t and_or(uint32_t x, uint32_t mask, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(mask), "r"(magic));
  return r;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// b-bit field pair (element k, element k + 16/b) of a 32-bit word as signed fp16 values.
template <int B>
__device__ __forceinline__ uint32_t int_pair(uint32_t w, int k) {
  constexpr uint32_t mask = ((1u << B) - 1u) * 0x00010001u;
  const uint32_t h = and_or(w >> (B * k), mask, 0x64006400u);
  const __half off = __float2half_rn(1024.0f + (float)(1 << (B - 1)));
  return h2u(__hsub2(u2h(h), __halves2half2(off, off)));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ uint32_t pack_h2(float lo_part, float hi_part) {
  return h2u(__floats2half2_rn(lo_part, hi_part));
}

template <int D, int KF, int GK, int VF, int GV, int TPW, int STAGES>
struct MmaCfg {
  static constexpr int KB = CodeBits<KF>::v, VB = CodeBits<VF>::v;
  static constexpr int TILE = 4 * TPW;                 // tokens per stage (4 warps)
  static constexpr int NSB = TPW / 16;                 // 16-token sub-blocks per warp
  static constexpr int RBK = D * KB / 8, RBV = D * VB / 8;
  static constexpr int NGK = D / GK, NGV = D / GV;
  static constexpr bool VSCALE = VF != CF_FP16;
  static constexpr int KS_BYTES = TILE * NGK * 2, VS_BYTES = VSCALE ? TILE * NGV * 2 : 0;
  static constexpr int OFF_KC = 0, OFF_KS = TILE * RBK, OFF_VC = OFF_KS + KS_BYTES, OFF_VS = OFF_VC + TILE * RBV;
  static constexpr int STAGE_BYTES = OFF_VS + VS_BYTES;
  static constexpr int KCB = GK * KB / 32;             // bytes of a thread's K chunk per group
  static constexpr int KCW = KCB / 4;
  static constexpr int VCB = GV * VB / 64;             // bytes of a thread's V chunk per group
  static constexpr int VCW = VCB >= 4 ? VCB / 4 : 1;   // words (a 2-byte chunk sits in one word)
  static constexpr int VCH = VCB / 2;                  // 16-bit halves of the chunk
  static constexpr int KSTEPS = GK / 16;               // mma k-steps per K group
  static constexpr int MT = GV / 16;                   // M-tiles (16 channels) per V group
  static constexpr int SMEM = STAGES * STAGE_BYTES > 4 * 4 * (D + 2) * 4 ? STAGES * STAGE_BYTES : 4 * 4 * (D + 2) * 4;
  static_assert(KCB % 4 == 0 && (VCB % 4 == 0 || VCB == 2), "chunks must be whole words or one half");
  static_assert(STAGE_BYTES % 16 == 0, "stage must be 16-byte aligned");
  static_assert(SMEM + 8192 <= 227 * 1024, "stages exceed the shared memory of one CTA");
};

// Element pair (e1, e2) within a thread's K chunk consumed by pair index p.
template <int KF>
__device__ __forceinline__ void k_pair_elems(int p, int& e1, int& e2) {
  if (KF == CF_NF4) {
    e1 = 2 * p;
    e2 = 2 * p + 1;
  } else {
    constexpr int B = CodeBits<KF>::v;
    constexpr int PPW = 16 / B;  // pairs per word
    const int w = p / PPW, k = p % PPW;
    e1 = w * (32 / B) + k;
    e2 = e1 + PPW;
  }
}

// All element pairs of a thread's K chunk (pair p = the p-th mma half-pair of the chunk).
template <int KF, int KCW>
__device__ __forceinline__ void k_pairs(const uint32_t* kw, uint32_t* pr, const uint32_t* lut) {
  if (KF == CF_NF4) {  // byte -> (level of low nibble, level of high nibble) table in shared memory
#pragma unroll
    for (int w = 0; w < KCW; ++w)
#pragma unroll
      for (int b = 0; b < 4; ++b) pr[4 * w + b] = lut[(kw[w] >> (8 * b)) & 0xFFu];
  } else {
    constexpr int B = CodeBits<KF>::v;
    constexpr int PPW = 16 / B;
#pragma unroll
    for (int w = 0; w < KCW; ++w)
#pragma unroll
      for (int k = 0; k < PPW; ++k) pr[w * PPW + k] = int_pair<B>(kw[w], k);
  }
}

template <int D>
__device__ void prepare_query_rot(const LayerDev& L, const __half* __restrict__ q, int qi, int kvh, int G, float* qs) {
  const SideDev& K = L.s[0];
  const int tid = threadIdx.x;
  for (int e = tid; e < G * D; e += blockDim.x) {
    const int h = e / D, j = e % D;
    const float v = __half2float(q[((long long)qi * L.Hq + kvh * G + h) * D + j]);
    qs[e] = K.chan_scale ? v * __half2float(K.chan[kvh * D + j]) : v;
  }
  __syncthreads();
  if (K.rot == 128 || K.rot == 256) {
    for (int h = 1; h < K.rot; h <<= 1) {
      for (int e = tid; e < G * D / 2; e += blockDim.x) {
        const int row = e / (D / 2), p = e % (D / 2);
        const int lo = p & (h - 1), hi = p >> (__ffs(h) - 1);
        const int i = (hi << __ffs(h)) | lo;
        float* r = qs + row * D;
        const float a = r[i], b = r[i + h];
        r[i] = a + b;
        r[i + h] = a - b;
      }
      __syncthreads();
    }
  }
  const float rn = K.rot == 256 ? 0.0625f : (K.rot == 128 ? 0.08838834764831845f : 1.0f);
  const float scl = L.sm_scale * kLog2e * rn;
  for (int e = tid; e < G * D; e += blockDim.x) qs[e] *= scl;
  __syncthreads();
}

// Shared-memory XOR swizzle of 16-byte chunks within a staged row, chosen per row size and
// per-thread chunk size so that the rows a warp reads in one instruction fall in distinct banks
// (K: rows g = 0..7 of a 16-token block; V: rows c, c+4, c+8, c+12 of the permuted k order).
template <int RB, int CB>
__device__ __forceinline__ int swz_k(int r) {
  if (RB == 64 && CB == 8) return ((r >> 1) & 1) << 1;
  if (RB == 64 && CB == 4) return (r >> 1) & 3;
  if (RB == 128 && CB == 16) return (r & 1) << 2;
  if (RB == 128 && CB == 4) return r & 7;
  return 0;
}
template <int RB, int CB>
__device__ __forceinline__ int swz_v(int r) {
  if (RB == 64 && (CB == 4 || CB == 2)) return ((r >> 1) & 1) << 1;
  if (RB == 128 && CB == 8) return (r & 3) << 1;
  if (RB == 512 && CB == 32) return (r & 1) | ((r & 2) << 1);
  return 0;
}
template <int RB>
__device__ __forceinline__ int swz_off(int r, int off, int sw) {  // byte offset within a row
  return (((off >> 4) ^ sw) << 4) | (off & 15);
}

template <int D, int G, int KF, int GK, int VF, int GV, int TPW, int STAGES>
__global__ void __launch_bounds__(128) decode_mma_kernel(LayerDev L, const __half* __restrict__ q,
                                                         const int* __restrict__ seq_ids, const int* __restrict__ kv_len,
                                                         float* __restrict__ work, int n_split, int nsp_total) {
  using C = MmaCfg<D, KF, GK, VF, GV, TPW, STAGES>;
  extern __shared__ __align__(16) unsigned char smem[];
  // P' = p * d_v as fp16 (hi, lo) per V group, in mma k order: [warp][group][column n][16 k]
  __shared__ __half pk[4][C::NGV][8][16];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int split = blockIdx.x, kvh = blockIdx.y, qi = blockIdx.z;
  const QueryRange R = query_range(L, qi, seq_ids, kv_len);
  const SideDev& K = L.s[0];
  const SideDev& V = L.s[1];
  const long long u = (long long)R.seq * L.Hkv + kvh;

  __shared__ uint32_t lut[KF == CF_NF4 ? 256 : 1];
  if (KF == CF_NF4) {
    for (int b = tid; b < 256; b += 128) lut[b] = pack_h2(d_nf4[b & 15], d_nf4[b >> 4]);
  }
  // ---- query: stored domain of K, x sm_scale log2 e; fragments hold (hi, lo) halves
  float* qs = reinterpret_cast<float*>(smem);
  prepare_query_rot<D>(L, q, qi, kvh, G, qs);
  uint32_t qreg[D / 16][2];
  {
    const int h = g >> 1, part = g & 1;
#pragma unroll
    for (int gk = 0; gk < C::NGK; ++gk) {
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          int e1, e2;
          k_pair_elems<KF>(2 * ks + r, e1, e2);
          const int cb = gk * GK + c * (GK / 4);
          float v1 = 0.0f, v2 = 0.0f;
          if (h < G) {
            v1 = qs[h * D + cb + e1];
            v2 = qs[h * D + cb + e2];
          }
          const float h1 = __half2float(__float2half_rn(v1)), h2 = __half2float(__float2half_rn(v2));
          qreg[gk * C::KSTEPS + ks][r] = part ? pack_h2(v1 - h1, v2 - h2) : pack_h2(h1, h2);
        }
      }
    }
  }
  __syncthreads();  // qs aliases the stage buffers

  // ---- token range of this split, in whole tiles
  const int tstart = (R.qa / C::TILE) * C::TILE;
  const int ntiles = R.qb > tstart ? (R.qb - tstart + C::TILE - 1) / C::TILE : 0;
  const int per = (ntiles + n_split - 1) / n_split;
  const int it0 = split * per;
  const int it1 = min(ntiles, it0 + per);
  const int nmy = max(0, it1 - it0);

  const uint8_t* gK = K.codes + u * L.Tcap * C::RBK;
  const uint8_t* gKs = reinterpret_cast<const uint8_t*>(K.scales + u * L.Tcap * C::NGK);
  const uint8_t* gV = V.codes + u * L.Tcap * C::RBV;
  const uint8_t* gVs = C::VSCALE ? reinterpret_cast<const uint8_t*>(V.scales + u * L.Tcap * C::NGV) : nullptr;

  auto issue = [&](int tile_idx, int stage) {
    const int t0 = tstart + tile_idx * C::TILE;
    unsigned char* st = smem + stage * C::STAGE_BYTES;
    constexpr int NCK = C::RBK / 16, NCV = C::RBV / 16;
    constexpr int NKC = C::TILE * NCK, NKS = C::KS_BYTES / 16, NVC = C::TILE * NCV, NVS = C::VS_BYTES / 16;
    for (int i = tid; i < NKC + NKS + NVC + NVS; i += 128) {
      if (i < NKC) {
        const int r = i / NCK, j = i % NCK;
        cp_async16(st + C::OFF_KC + r * C::RBK + ((j ^ swz_k<C::RBK, C::KCB>(r)) << 4),
                   gK + (long long)t0 * C::RBK + i * 16);
      } else if (i < NKC + NKS) {
        cp_async16(st + C::OFF_KS + (i - NKC) * 16, gKs + (long long)t0 * C::NGK * 2 + (i - NKC) * 16);
      } else if (i < NKC + NKS + NVC) {
        const int iv = i - NKC - NKS, r = iv / NCV, j = iv % NCV;
        cp_async16(st + C::OFF_VC + r * C::RBV + ((j ^ swz_v<C::RBV, C::VCB>(r)) << 4),
                   gV + (long long)t0 * C::RBV + iv * 16);
      } else {
        cp_async16(st + C::OFF_VS + (i - NKC - NKS - NVC) * 16,
                   gVs + (long long)t0 * C::NGV * 2 + (i - NKC - NKS - NVC) * 16);
      }
    }
  };

  float oacc[D / 16][4];
#pragma unroll
  for (int i = 0; i < D / 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f;
  const bool head_ok = c < G;

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < nmy) issue(it0 + s, s);
    cp_async_commit();
  }

  for (int it = 0; it < nmy; ++it) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    if (it + STAGES - 1 < nmy) issue(it0 + it + STAGES - 1, (it + STAGES - 1) % STAGES);
    cp_async_commit();

    const unsigned char* st = smem + (it % STAGES) * C::STAGE_BYTES;
    const int tile_t0 = tstart + (it0 + it) * C::TILE;
    const int rb = warp * TPW;

    // ---- scores
    float sc[C::NSB][2];
#pragma unroll
    for (int sb = 0; sb < C::NSB; ++sb) {
      const int r0 = rb + sb * 16 + g, r1 = r0 + 8;
      float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
      for (int gk = 0; gk < C::NGK; ++gk) {
        uint32_t kw0[C::KCW], kw1[C::KCW];
        const int off = (gk * GK + c * (GK / 4)) * C::KB / 8;
        const uint32_t* p0 = reinterpret_cast<const uint32_t*>(
            st + C::OFF_KC + r0 * C::RBK + swz_off<C::RBK>(r0, off, swz_k<C::RBK, C::KCB>(r0)));
        const uint32_t* p1 = reinterpret_cast<const uint32_t*>(
            st + C::OFF_KC + r1 * C::RBK + swz_off<C::RBK>(r1, off, swz_k<C::RBK, C::KCB>(r1)));
#pragma unroll
        for (int w = 0; w < C::KCW; ++w) {
          kw0[w] = p0[w];
          kw1[w] = p1[w];
        }
        uint32_t kp0[2 * C::KSTEPS], kp1[2 * C::KSTEPS];
        k_pairs<KF, C::KCW>(kw0, kp0, lut);
        k_pairs<KF, C::KCW>(kw1, kp1, lut);
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks)
          mma16816(acc, kp0[2 * ks], kp1[2 * ks], kp0[2 * ks + 1], kp1[2 * ks + 1], qreg[gk * C::KSTEPS + ks][0],
                   qreg[gk * C::KSTEPS + ks][1]);
        const __half* ks_ = reinterpret_cast<const __half*>(st + C::OFF_KS);
        s0 += __half2float(ks_[r0 * C::NGK + gk]) * (acc[0] + acc[1]);
        s1 += __half2float(ks_[r1 * C::NGK + gk]) * (acc[2] + acc[3]);
      }
      const int t0 = tile_t0 + r0, t1 = t0 + 8;
      sc[sb][0] = (t0 >= R.qa && t0 < R.qb) ? s0 : -INFINITY;
      sc[sb][1] = (t1 >= R.qa && t1 < R.qb) ? s1 : -INFINITY;
    }
    // ---- online softmax (log2 domain), per head c over this warp's TPW tokens
    float tmax = -INFINITY;
#pragma unroll
    for (int sb = 0; sb < C::NSB; ++sb) tmax = fmaxf(tmax, fmaxf(sc[sb][0], sc[sb][1]));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
    const float m_new = fmaxf(m_run, tmax);
    float alpha = 1.0f;
    if (m_new != -INFINITY) {
      alpha = exp2f(m_run - m_new);
      l_run *= alpha;
#pragma unroll
      for (int sb = 0; sb < C::NSB; ++sb) {
        sc[sb][0] = exp2f(sc[sb][0] - m_new);
        sc[sb][1] = exp2f(sc[sb][1] - m_new);
        l_run += sc[sb][0] + sc[sb][1];
      }
      m_run = m_new;
    } else {
#pragma unroll
      for (int sb = 0; sb < C::NSB; ++sb) sc[sb][0] = sc[sb][1] = 0.0f;
    }
    if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        oacc[i][0] *= alpha;
        oacc[i][1] *= alpha;
        oacc[i][2] *= alpha;
        oacc[i][3] *= alpha;
      }
    }
    // ---- values, one 16-token sub-block at a time.  k order of a sub-block: slot 2c, 2c+1,
    // 2c+8, 2c+9 holds token c, c+4, c+8, c+12 (so the rows a warp loads together are adjacent).
#pragma unroll
    for (int sb = 0; sb < C::NSB; ++sb) {
      // P' (hi, lo) per V group from this thread's two tokens g, g+8 (head c)
      {
        const int tk[2] = {g, g + 8};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int t = tk[i];
          const int kslot = 2 * (t & 3) + ((t >> 2) & 1) + 8 * (t >> 3);
          const float p = head_ok ? sc[sb][i] : 0.0f;
#pragma unroll
          for (int gv = 0; gv < C::NGV; ++gv) {
            float d = 1.0f;
            if (C::VSCALE) d = __half2float(reinterpret_cast<const __half*>(st + C::OFF_VS)[(rb + sb * 16 + t) * C::NGV + gv]);
            const float x = p == 0.0f ? 0.0f : p * d;
            const __half hi = __float2half_rn(x);
            pk[warp][gv][2 * c][kslot] = hi;
            pk[warp][gv][2 * c + 1][kslot] = __float2half_rn(x - __half2float(hi));
          }
        }
      }
      __syncwarp();
      const int rr[4] = {rb + sb * 16 + c, rb + sb * 16 + c + 4, rb + sb * 16 + c + 8, rb + sb * 16 + c + 12};
      uint32_t vmask_a = 0xFFFFFFFFu, vmask_c = 0xFFFFFFFFu;
      if (VF == CF_FP16) {  // unwritten fp16 rows may hold NaN; zero them (p is 0 there)
        auto ok = [&](int r) { const int t = tile_t0 + r; return t >= R.qa && t < R.qb; };
        vmask_a = (ok(rr[0]) ? 0x0000FFFFu : 0u) | (ok(rr[1]) ? 0xFFFF0000u : 0u);
        vmask_c = (ok(rr[2]) ? 0x0000FFFFu : 0u) | (ok(rr[3]) ? 0xFFFF0000u : 0u);
      }
#pragma unroll
      for (int gv = 0; gv < C::NGV; ++gv) {
        const uint32_t* pkw = reinterpret_cast<const uint32_t*>(&pk[warp][gv][g][0]);
        const uint32_t b0 = pkw[c], b1 = pkw[c + 4];
        uint32_t vw[4][C::VCW];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int off = (gv * GV + g * (GV / 8)) * C::VB / 8;
          const int sw = swz_v<C::RBV, C::VCB>(rr[i]);
          const unsigned char* rowp = st + C::OFF_VC + rr[i] * C::RBV;
          if (C::VCB == 2) {
            vw[i][0] = *reinterpret_cast<const uint16_t*>(rowp + swz_off<C::RBV>(rr[i], off, sw));
          } else {
#pragma unroll
            for (int w = 0; w < C::VCW; ++w)
              vw[i][w] = *reinterpret_cast<const uint32_t*>(rowp + swz_off<C::RBV>(rr[i], off + 4 * w, sw));
          }
        }
        // (t, t') pairs of each chunk element; element e -> M-tile e/2, row g (+8 if odd)
        uint32_t pa[GV / 8], pc[GV / 8];
        if (VF == CF_FP16) {
#pragma unroll
          for (int w = 0; w < C::VCW; ++w) {
            pa[2 * w] = prmt(vw[0][w], vw[1][w], 0x5410) & vmask_a;
            pa[2 * w + 1] = prmt(vw[0][w], vw[1][w], 0x7632) & vmask_a;
            pc[2 * w] = prmt(vw[2][w], vw[3][w], 0x5410) & vmask_c;
            pc[2 * w + 1] = prmt(vw[2][w], vw[3][w], 0x7632) & vmask_c;
          }
        } else {
          constexpr int B = C::VB, PH = 16 / B;  // elements per 16-bit half
#pragma unroll
          for (int hh = 0; hh < C::VCH; ++hh) {
            const int w = hh >> 1, hf = hh & 1;
            const uint32_t xa = prmt(vw[0][w], vw[1][w], hf ? 0x7632 : 0x5410);
            const uint32_t xc = prmt(vw[2][w], vw[3][w], hf ? 0x7632 : 0x5410);
#pragma unroll
            for (int k = 0; k < PH; ++k) {
              const int e = hh * PH + k;
              pa[e] = int_pair<B>(xa, k);
              pc[e] = int_pair<B>(xc, k);
            }
          }
        }
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt)
          mma16816(oacc[gv * C::MT + mt], pa[2 * mt], pa[2 * mt + 1], pc[2 * mt], pc[2 * mt + 1], b0, b1);
      }
      __syncwarp();
    }
  }
  cp_async_wait<0>();
  __syncthreads();  // stage buffers are free: reuse them to combine the four warps

  // ---- combine the four warps' (m, l, o) into one partial per CTA
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 4);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
  float* red = reinterpret_cast<float*>(smem);             // [4 warps][4 heads][D]
  float* ml = red + 4 * 4 * D;                             // [4 warps][4 heads][2]
  if (head_ok) {
    if (g == 0) {
      ml[(warp * 4 + c) * 2] = m_run;
      ml[(warp * 4 + c) * 2 + 1] = l_run;
    }
#pragma unroll
    for (int gv = 0; gv < C::NGV; ++gv)
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) {
        const int ch = gv * GV + g * (GV / 8) + 2 * mt;
        const float* o = oacc[gv * C::MT + mt];
        *reinterpret_cast<float2*>(red + (warp * 4 + c) * D + ch) = make_float2(o[0] + o[1], o[2] + o[3]);
      }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += 128) {
    const int h = e / D, j = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, ml[(w * 4 + h) * 2]);
    float lsum = 0.0f, osum = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = ml[(w * 4 + h) * 2];
        const float sc = mw == -INFINITY ? 0.0f : exp2f(mw - M);
        lsum += sc * ml[(w * 4 + h) * 2 + 1];
        osum += sc * red[(w * 4 + h) * D + j];
      }
    }
    float* P = work + (((long long)qi * L.Hq + kvh * G + h) * nsp_total + split) * (D + kPartStride);
    if (j == 0) {
      P[0] = M;
      P[1] = lsum;
    }
    P[kPartStride + j] = osum;
  }
}
