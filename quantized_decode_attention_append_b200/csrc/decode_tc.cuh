// Tensor-core pass 1 of kvq_decode_attention for GQA groups of up to 4 query heads.
//
// Included by decode.cu inside namespace kvq (uses QueryRange, query_range, kLog2e and d_nf4).
// Same contract as the generic pass: one CTA per (query, kv-head, split) writes one log2-domain
// partial (m, l, o[D] in V's stored domain); the CTA's warps are combined in shared memory first.
//
// Staging.  A tile of TILE consecutive tokens of one (sequence, kv-head) is four contiguous byte
// ranges of the cache: K codes, K scales, V codes, V scales.  One thread moves each range with a
// bulk asynchronous copy (cp.async.bulk, the TMA engine's linear mode) into a stage of shared
// memory and the copies count their bytes on that stage's mbarrier; every thread waits on the
// barrier with a bounded poll.  STAGES - 1 tiles are in flight while one is consumed.  Stages are
// recycled behind one CTA barrier per tile.
//
// Work mapping (mma.sync m16n8k16, fp16 operands, fp32 accumulate):
//   scores  S[16 tokens x 8] = K[16 x 16 ch] . Q'^T[16 ch x 8]; the 8 columns are 4 heads x
//           (hi, lo) fp16 halves of the pre-transformed query, so a logit keeps ~22 bits; one
//           accumulator per K group, multiplied by the group's fp16 scale afterwards.
//   values  O^T[16 ch x 8] += V^T[16 ch x 16 tokens] . P'^T[16 tokens x 8]; the columns are 4
//           heads x (hi, lo) halves of p * d_v (the V group scale folded into the probability).
// Codes become exact fp16 operands in registers.  b-bit fields use the 0x6400 exponent trick:
// (field << s) | 0x6400 is 1024 + 2^s field, so one fused multiply-add by 2^-s with the offset
// -(1024 2^-s + 2^(b-1)) yields the signed code exactly; fields at shifts 0..7 of a 16-bit half
// need no shift instruction, only the upper byte does.  NF4 goes through a byte -> level-pair table
// in shared memory with one copy per bank (entry e of lane l at word 32 e + l), so the lanes of a
// warp never contend for a bank.  fp16 V is regrouped by byte permutes.
//
// Shared-memory banks.  Each of the four ranges of a tile is copied as two halves (tokens
// [0, TILE/2) and [TILE/2, TILE)), the second one behind a small pad, so rows of the two halves
// start on different banks.  A 16-token block takes 8 tokens from each half: score row rho is token
// (half R(rho), index k(rho)) with k(rho + 8) = k(rho) + 4, and R, k chosen per row size so that the
// rows one load phase touches fall on distinct banks (for 64-byte rows: R = bit 1 of rho,
// k = bit 0 + 2 * (rho >> 2); for 128-byte rows: R = bit 0, k = rho >> 1).  In the V product the k
// slots (2c, 2c+1) hold the two tokens of score row c and slots (2c+8, 2c+9) those of row c + 4, so
// the pair of probabilities a score thread owns is one 32-bit word of P'.  P' is staged per warp in
// rows of 12 words (16 halves + 4 pad), which keeps its stores and fragment loads conflict-free.

// CF_SYM2: 2-bit codes of the symmetric grid, value code - 3/2 (exact in fp16).
enum CodeFmt { CF_INT2 = 2, CF_INT3 = 3, CF_INT4 = 4, CF_NF4 = 16, CF_FP16 = 32, CF_SIGN = 64, CF_TERN = 128,
               CF_SYM2 = 256 };

template <int F> struct CodeBits {
  // bits per value in the layout the operands are built from (ternary: transcoded 2-bit digits)
  static constexpr int v =
      F == CF_NF4 ? 4 : (F == CF_FP16 ? 16 : (F == CF_SIGN ? 1 : (F == CF_TERN || F == CF_SYM2 ? 2 : (F == CF_INT3 ? 4 : F))));
};

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


__device__ __forceinline__ uint32_t pack_h2(float lo_part, float hi_part) {
  return h2u(__floats2half2_rn(lo_part, hi_part));
}

// fp16 pair (x, x) from its bit pattern
__device__ __forceinline__ __half2 h2c(unsigned short bits) {
  const __half h = __ushort_as_half(bits);
  return __halves2half2(h, h);
}

// The 16/B field pairs of a 32-bit word of B-bit offset-binary codes as signed fp16 pairs
// (field - ofs, exact while ofs is a multiple of 1/2 below 2^9):
// out[k] = (field k, field k + 16/B), i.e. field k of each 16-bit half.
// A half-integer offset needs every field at a shift of at least 1: the constant 2^(10-s) + ofs
// is then a multiple of 1/2 below 1024, an fp16 value; the word is pre-shifted left by one bit
// (fields of each byte at bits 1..8 of their 16-bit half, still inside the 10-bit mantissa).
template <int B>
__device__ __forceinline__ void code_pairs(uint32_t w, uint32_t* out, float ofs = (float)(1 << (B - 1))) {
  constexpr int PH = 16 / B;                 // fields per 16-bit half
  constexpr int PB = 8 / B;                  // fields per byte
  constexpr uint32_t M = ((1u << B) - 1u) * 0x00010001u;
  const bool half_ofs = ofs != floorf(ofs);  // folded at compile time (ofs is a constant)
  const int s0 = half_ofs ? 1 : 0;
  const uint32_t wl = half_ofs ? (w << 1) : w, w8 = half_ofs ? (w >> 7) : (w >> 8);
#pragma unroll
  for (int k = 0; k < PH; ++k) {
    const int s = B * (k % PB) + s0;         // shift of the field inside its 16-bit half
    const uint32_t x = and_or(k < PB ? wl : w8, M << s, 0x64006400u);  // 1024 + 2^s field
    // 2^-s and -(1024 2^-s + 2^(B-1)) as fp16 bit patterns
    const unsigned short scl = (unsigned short)((15 - s) << 10);
    const float off = -(1024.0f / (float)(1 << s) + ofs);
    const __half2 r = __hfma2(u2h(x), h2c(scl), __float2half2_rn(off));
    out[k] = h2u(r);
  }
}

// 2^x by the special-function unit (ex2.approx, subnormal results flushed to zero; 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Entry of byte `b` of `w` in the per-lane level-pair table at shared address `base` (lane's copy;
// entries 128 bytes apart): byte extraction by permute, address by multiply-add.
template <int b>
__device__ __forceinline__ uint32_t lut_pair(uint32_t base, uint32_t w) {
  uint32_t v;
  asm volatile(
      "{\n .reg .u32 i, a;\n prmt.b32 i, %1, 0, %3;\n mad.lo.u32 a, i, 128, %2;\n ld.shared.u32 %0, [a];\n}\n"
      : "=r"(v)
      : "r"(w), "r"(base), "n"(0x4440 | b));
  return v;
}

// Sign codes carry their scale in the operand: a value is +d (bit set) or -d, exact in fp16, so the
// sign bit of the duplicated fp16 scale is flipped per element.
// K: pairs (channels 2p, 2p+1) of one word of sign bits (LSB first) with the scales of its 8
// groups of 4 (sv: 4 words of fp16 pairs).  Odd bits are first moved 15 places up, so pair p's two
// signs sit 16 bits apart and one shift brings them to bits 15 and 31.
__device__ __forceinline__ void sign_pairs_k(uint32_t w, const uint32_t* sv, uint32_t* out) {
  const uint32_t t = ~w, th = t >> 16;
  const uint32_t lo = (t & 0x5555u) | ((t << 15) & 0x55550000u);
  const uint32_t hi = (th & 0x5555u) | ((th << 15) & 0x55550000u);
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const uint32_t dd = prmt(sv[p >> 2], sv[p >> 2], ((p >> 1) & 1) ? 0x3232u : 0x1010u);
    out[p] = (((p < 8 ? lo : hi) << (15 - 2 * (p & 7))) & 0x80008000u) ^ dd;
  }
}
// V: pairs (row A, row B) of element e of 16 sign bits per row (ab: row A's bits in the low half,
// row B's in the high half) with the rows' scales of 4 groups of 4 (sa, sb: 2 words each).
__device__ __forceinline__ void sign_pairs_v(uint32_t ab, const uint32_t* sa, const uint32_t* sb, uint32_t* out) {
  const uint32_t t = ~ab;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int k = e >> 2;
    const uint32_t dd = prmt(sa[k >> 1], sb[k >> 1], (k & 1) ? 0x7632u : 0x5410u);
    out[e] = ((t << (15 - e)) & 0x80008000u) ^ dd;
  }
}

// Ternary: digits d = t + 1 (2-bit fields after transcoding) -> (d - 1) x scale, exact in fp16;
// dd holds the scales of the two elements of each pair (low, high half).
__device__ __forceinline__ void tern_pairs(uint32_t w, uint32_t dd, uint32_t* out) {
  uint32_t r[8];
  code_pairs<2>(w, r, 1.0f);
#pragma unroll
  for (int k = 0; k < 8; ++k) out[k] = h2u(__hmul2(u2h(r[k]), u2h(dd)));
}

// ---- mbarrier and bulk-copy primitives

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// Global -> shared bulk copy completing `bytes` on `bar` (16-byte aligned ends, bytes % 16 == 0).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete; false after `limit` clock cycles of polling
// (by default about one second).
constexpr long long kWaitCycles = 2000000000LL;
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, long long limit) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > limit) return false;
  return true;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit = kWaitCycles) {
  return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, limit);
}

// N consecutive 32-bit words from 4N-byte aligned shared memory
template <int N>
__device__ __forceinline__ void lds_words(const unsigned char* p, uint32_t* w) {
  if constexpr (N == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (N == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (N == 1) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else {
#pragma unroll
    for (int i = 0; i < N; i += 4) lds_words<4>(p + 4 * i, w + i);
  }
}

template <int D, int KF, int GK, int VF, int GV, int NW, int TPW, int STAGES>
struct TcCfg {
  static constexpr int KB = CodeBits<KF>::v, VB = CodeBits<VF>::v;
  static constexpr int NT = NW * 32;                   // consumer threads
  // A dedicated producer warp recycles stages through per-stage "empty" barriers, so consumer
  // warps never meet at a CTA barrier.  Measured: faster for head_dim 256 (4 consumer warps),
  // slightly slower for the head_dim-128 instances, which keep one CTA barrier per tile.
  static constexpr bool PROD = D >= 256;
  static constexpr int NTH = NT + (PROD ? 32 : 0);
  static constexpr int TILE = NW * TPW;                // tokens per stage
  static constexpr int HALF = TILE / 2;                // tokens per half-tile range
  static constexpr int NSB = TPW / 16;                 // 16-token blocks per warp and tile
  static constexpr int RBK = D * KB / 8, RBV = D * VB / 8;
  static constexpr int NGK = D / GK, NGV = D / GV;       // scale groups per row (storage)
  static constexpr bool KSGN = KF == CF_SIGN, VSGN = VF == CF_SIGN;
  static constexpr bool KTRN = KF == CF_TERN, VTRN = VF == CF_TERN;  // ternary rows transcoded per warp
  static constexpr bool V3 = VF == CF_INT3;                          // int3 V rows transcoded to nibbles
  static constexpr bool VX = VTRN || V3;                             // V read from the transcode buffer
  static constexpr float VOFS = V3 ? 4.0f : (VF == CF_SYM2 ? 1.5f : (float)(1 << (VB - 1)));  // V code offset
  static constexpr bool KSCL = KSGN || KTRN, VSCL = VSGN || VTRN;    // scale inside the operand
  static constexpr bool VSCALE = VF != CF_FP16 && !VSCL;  // V scale folded into P'
  static constexpr bool VSROW = VF != CF_FP16;            // V rows carry scales
  static constexpr int GKM = KSCL ? D : GK, GVM = VSCL ? D : GV;  // channels per accumulation group
  static constexpr int NGKM = D / GKM, NGVM = D / GVM;
  static constexpr int NPV = VSCALE ? NGV : 1;         // distinct P' operands (one per V group)
  static constexpr int GKB = GKM * KB / 8, GVB = GVM * VB / 8;  // bytes of an accumulation group in a row
  static constexpr int KCB = GKB / 4, KCW = KCB / 4;   // a thread's K chunk of a group
  static constexpr int VCB = GVB / 8;                  // a thread's V chunk of a group (bytes)
  static constexpr int VCW = VCB >= 4 ? VCB / 4 : 1;
  static constexpr int VCH = VCB / 2;                  // 16-bit halves of the V chunk
  static constexpr int KSTEPS = GKM / 16, MT = GVM / 16;
  static constexpr int KCS = KSCL ? (D / 4 / GK) * 2 : 0;  // bytes of a K chunk's scales (scale in operand)
  static constexpr int VCS = VSCL ? (D / 8 / GV) * 2 : 0;  // bytes of a V chunk's scales (scale in operand)
  // stored row bytes (ternary: 5 digits per byte) and the per-warp transcode buffers
  static constexpr int RSK = KTRN ? (D + 4) / 5 : RBK, RSV = VTRN ? (D + 4) / 5 : (V3 ? D * 3 / 8 : RBV);
  // transcode buffers per warp: half A (TPW/2 rows), pad, half B, for K then V
  static constexpr int XKH = (TPW / 2) * RBK, XKB = XKH + (RBK == 64 ? 32 : 64), XKS = KTRN ? XKB + XKH : 0;
  static constexpr int XVH = (TPW / 2) * RBV, XVB = XVH + (RBV == 64 ? 32 : 64), XVS = VX ? XVB + XVH : 0;
  static constexpr int XW = XKS + XVS;  // per warp
  static constexpr bool ALT = RBK >= 128;              // row -> (half, index) mapping
  // log2 headroom of p over the running max: |d_v| <= 65504 / 2^(b-1) for b-bit absmax V, so
  // p <= 2^(b-1) keeps p * d_v finite in fp16; P' carries no scale for fp16 and sign V.
  // (symmetric 2-bit: |d_v| <= 65504 / 1.5, so p <= 1)
  static constexpr float SLACK = VSCALE ? (VF == CF_SYM2 ? 0.0f : (float)((V3 ? 3 : VB) - 1)) : 8.0f;
  static constexpr int PADK = RBK == 64 ? 32 : 64, PADV = RBV == 64 ? 32 : 64, PADS = 16;
  // stage: [K codes A | pad | K codes B][K scales A | pad | B][V codes A | pad | B][V scales A | pad | B]
  static constexpr int KC_H = HALF * RSK, KS_H = HALF * NGK * 2;
  static constexpr int VC_H = HALF * RSV, VS_H = VSROW ? HALF * NGV * 2 : 0;
  static constexpr int OFF_KA = 0, OFF_KB = OFF_KA + KC_H + PADK;
  static constexpr int OFF_KSA = OFF_KB + KC_H, OFF_KSB = OFF_KSA + KS_H + PADS;
  static constexpr int OFF_VA = OFF_KSB + KS_H, OFF_VB = OFF_VA + VC_H + PADV;
  static constexpr int OFF_VSA = OFF_VB + VC_H, OFF_VSB = OFF_VSA + VS_H + PADS;
  static constexpr int STAGE_RAW = OFF_VSB + VS_H;
  static constexpr int STAGE_BYTES = (STAGE_RAW + 127) / 128 * 128;
  static constexpr uint32_t TX_BYTES = 2 * (KC_H + KS_H + VC_H + VS_H);  // bytes one tile brings
  static constexpr int RED_BYTES = NW * 4 * (D + 2) * 4;  // epilogue: per-warp (o, m, l)
  static constexpr int RING_BYTES = STAGES * STAGE_BYTES > RED_BYTES ? STAGES * STAGE_BYTES : RED_BYTES;
  static constexpr int PKS = 12;                       // words per staged P' row
  static constexpr int PK_WORDS = NPV * 8 * PKS;       // per warp
  static constexpr int PK_BYTES_RAW = NW * PK_WORDS * 4;
  static constexpr int QS_BYTES = (4 * D + 4) * 4;     // query staging (+ q . mu per head) aliases the P' area
  static constexpr int PK_BYTES = PK_BYTES_RAW > QS_BYTES ? PK_BYTES_RAW : QS_BYTES;
  static constexpr int LUT_BYTES = (KF == CF_NF4 || KTRN || VTRN) ? 256 * 32 * 4 : 0;
  static constexpr int OFF_PK = RING_BYTES, OFF_LUT = OFF_PK + PK_BYTES, OFF_X = OFF_LUT + LUT_BYTES;
  static constexpr int OFF_BAR = OFF_X + NW * XW;
  static constexpr int SMEM = OFF_BAR + 2 * STAGES * 8 + 16;  // full and empty barriers, test barrier, abort flag

  static_assert(KCB % 4 == 0, "K chunks must be whole words");
  static_assert(!(KTRN || VTRN) || (D == 128 && TPW == 32 && GK == 8 && GV == 8), "ternary instance shape");
  static_assert(!V3 || (TPW == 32 && GV >= 16), "int3 V instance shape");
  static_assert(KF != CF_NF4 || !(VTRN), "one table per kernel");
  static_assert(VCB % 4 == 0 || VCB == 2, "V chunks must be whole words or one half");
  static_assert(KC_H % 128 == 0 && VC_H % 128 == 0 && KS_H % 128 == 0 && VS_H % 128 == 0,
                "half ranges keep the bank position of what follows them");
  static_assert(STAGE_BYTES % 16 == 0 && RING_BYTES % 16 == 0 && PK_BYTES % 16 == 0, "16-byte aligned areas");
  static_assert(TPW % 16 == 0 && 256 % TILE == 0, "tiles must divide the 256-token capacity unit");
  static_assert(SMEM <= 227 * 1024, "stages exceed the shared memory of one CTA");

  // Half and index (within this 16-token block's 8 tokens of that half) of score row rho.
  __device__ static __forceinline__ int row_half(int rho) { return ALT ? (rho & 1) : ((rho >> 1) & 1); }
  __device__ static __forceinline__ int row_index(int rho) { return ALT ? (rho >> 1) : ((rho & 1) + 2 * (rho >> 2)); }
};

// q' = H(c . q) x sm_scale log2 e for the G heads of kv-head kvh into qs[G][D].  Warp h < G takes
// head h with D/32 contiguous values per lane: Hadamard stages below D/32 run in-lane, the rest by
// xor-shuffles (same fp32 butterflies, same order h = 1, 2, ..., rot/2).
template <int D>
__device__ void prepare_query_rot(const LayerDev& L, const __half* __restrict__ q, int qi, int kvh, int G, float* qs) {
  const SideDev& K = L.s[0];
  constexpr int V = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < G) {
    const int h = warp, j0 = lane * V;
    float x[V];
    const __half* qp = q + query_row(L, qi, kvh, G, h) * D + j0;
#pragma unroll
    for (int v = 0; v < V; ++v) {
      x[v] = __half2float(qp[v]);
      if (K.chan_scale) x[v] = x[v] * __half2float(K.chan[kvh * D + j0 + v]);
    }
    if (K.rot == 128 || K.rot == 256) {
#pragma unroll
      for (int hh = 1; hh < V; hh <<= 1)
#pragma unroll
        for (int v = 0; v < V; ++v)
          if ((v & hh) == 0) {
            const float a = x[v], b = x[v + hh];
            x[v] = a + b;
            x[v + hh] = a - b;
          }
      for (int hh = V; hh < K.rot; hh <<= 1) {
        const int lm = hh / V;
        const bool upper = (lane & lm) != 0;
#pragma unroll
        for (int v = 0; v < V; ++v) {
          const float o = __shfl_xor_sync(0xffffffffu, x[v], lm);
          x[v] = upper ? o - x[v] : x[v] + o;
        }
      }
    }
    const float rn = K.rot == 256 ? 0.0625f : (K.rot == 128 ? 0.08838834764831845f : 1.0f);
    const float scl = L.sm_scale * kLog2e * rn;
#pragma unroll
    for (int v = 0; v < V; ++v) qs[h * D + j0 + v] = x[v] * scl;
  }
  __syncthreads();
}

// Element pair (e1, e2) of a thread's K chunk that pair index p covers.
template <int KF>
__device__ __forceinline__ void k_pair_elems(int p, int& e1, int& e2) {
  if (KF == CF_NF4 || KF == CF_SIGN) {
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

// One ternary row (26 bytes, 5 base-3 digits per byte, 2-byte aligned) -> 8 words of 2-bit digits
// (channel j at bits 2j) through the per-lane byte table at shared address `lutb`.
__device__ __forceinline__ void tern_transcode(const unsigned char* src, unsigned char* dst, uint32_t lutb) {
  uint32_t out[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) out[i] = 0u;
#pragma unroll
  for (int h = 0; h < 13; ++h) {
    const uint32_t two = *reinterpret_cast<const uint16_t*>(src + 2 * h);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int b = 2 * h + q, bit = 10 * b, w = bit >> 5, sh = bit & 31;
      const uint32_t dg = q ? lut_pair<1>(lutb, two) : lut_pair<0>(lutb, two);
      if (w < 8) out[w] |= dg << sh;
      if (sh > 22 && w + 1 < 8) out[w + 1] |= dg >> (32 - sh);
    }
  }
  uint4* o = reinterpret_cast<uint4*>(dst);
  o[0] = make_uint4(out[0], out[1], out[2], out[3]);
  o[1] = make_uint4(out[4], out[5], out[6], out[7]);
}

// One int3 row (D fields of 3 bits, LSB first, 16-byte aligned) -> D 4-bit fields (nibble j =
// field j).  Each output word takes 24 input bits (a funnel shift), splits them into two 12-bit
// halves at bits 0 and 16, and spreads 3-bit fields to nibbles in two shift-and-mask steps.
template <int D>
__device__ __forceinline__ void int3_transcode(const unsigned char* src, unsigned char* dst) {
  constexpr int NIN = D * 3 / 32, NOUT = D / 8;
  uint32_t in[NIN + 1];
#pragma unroll
  for (int i = 0; i < NIN; i += 4) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[i / 4];
    in[i] = v.x; in[i + 1] = v.y; in[i + 2] = v.z; in[i + 3] = v.w;
  }
  in[NIN] = 0u;
  uint32_t out[NOUT];
#pragma unroll
  for (int o = 0; o < NOUT; ++o) {
    const int bit = 24 * o, wi = bit >> 5, sh = bit & 31;
    const uint32_t g = __funnelshift_r(in[wi], in[wi + 1], sh);              // fields 8o .. 8o + 7 in bits 0..23
    const uint32_t t = (g & 0x00000FFFu) | ((g << 4) & 0x0FFF0000u);          // halves at bits 0 and 16
    const uint32_t x1 = (t & 0x003F003Fu) | ((t << 2) & 0x3F003F00u);         // fields 2, 3 up by 2
    out[o] = (x1 & 0x07070707u) | ((x1 << 1) & 0x70707070u);                  // fields 1, 3 up by 1
  }
#pragma unroll
  for (int o = 0; o < NOUT; o += 4)
    reinterpret_cast<uint4*>(dst)[o / 4] = make_uint4(out[o], out[o + 1], out[o + 2], out[o + 3]);
}

__device__ __forceinline__ bool head_ok_of(int c, int G) { return c < G; }

// Append family and code bits of a tensor-core code format (the grid its rows are written with).
template <int F> struct TcFam { static constexpr int fam = FAM_ABSMAX, bits = F; };  // CF_INT2 / CF_INT4
template <> struct TcFam<CF_INT3> { static constexpr int fam = FAM_ABSMAX, bits = 3; };
template <> struct TcFam<CF_SYM2> { static constexpr int fam = FAM_SYM, bits = 2; };
template <> struct TcFam<CF_NF4> { static constexpr int fam = FAM_NF4, bits = 0; };
template <> struct TcFam<CF_SIGN> { static constexpr int fam = FAM_SIGN, bits = 0; };
template <> struct TcFam<CF_TERN> { static constexpr int fam = FAM_TERNARY, bits = 0; };

// Fused append + decode: the new rows of (query qi's sequence, kv-head kvh) that this CTA owns
// are written by warp 0 before a tile copy reads them.  A new row inside the quantized range
// belongs to the CTA whose tiles cover it (the only reader of its codes in this launch); the
// others (anchored rows, read later from their anchor copies) to split 0.  One row per lane group
// of head_dim / 32 lanes, as in the append kernels, with the same arithmetic (quantize_slice).
// Not inlined (called once per CTA), so its working registers are not live in the decode loop;
// the fused kernel's LayerDev is a __grid_constant__ parameter, so the reference reads it in
// place.  Under the fused instances' register cap the call still makes the 8-warp loops spill,
// which is why multi-wave grids take the separate append and decode calls (kvq_append_decode).
template <int D, int KF, int GK, int VF, int GV>
__device__ __noinline__ void fused_append_rows(const LayerDev& L, const QueryRange& R, int qi, int kvh, int split,
                                               int t_lo, int t_hi) {
  constexpr int LPR = D / 32, RPW = 32 / LPR;
  const int lane = threadIdx.x & 31, li = lane % LPR;
  const int p0 = R.len - R.fresh;
  const int u = R.seq * L.Hkv + kvh;
  for (int base = 0; base < R.fresh; base += RPW) {
    const int i = base + lane / LPR, p = p0 + i;
    const bool in_q = p >= R.qa && p < R.qb;
    const bool mine = i < R.fresh && (in_q ? (p >= t_lo && p < t_hi) : split == 0);
    if (!__any_sync(0xffffffffu, mine)) continue;
    const long long in_row = ((long long)qi * L.Hkv_all + L.h0 + kvh) * L.fuse_n + (mine ? i : 0);
    uint4 cw[4];
    const uint4* pk = reinterpret_cast<const uint4*>(L.fuse_k + in_row * D) + li * 4;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) cw[c4] = mine ? __ldg(pk + c4) : make_uint4(0u, 0u, 0u, 0u);
    quantize_slice<TcFam<KF>::fam, GK, TcFam<KF>::bits, false>(L, L.s[0], cw, mine, u, p, R.len);
    const uint4* pv = reinterpret_cast<const uint4*>(L.fuse_v + in_row * D) + li * 4;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) cw[c4] = mine ? __ldg(pv + c4) : make_uint4(0u, 0u, 0u, 0u);
    if constexpr (VF == CF_FP16) {  // fp16 V: the row as it comes, and its anchor copy
      const SideDev& S = L.s[1];
      if (mine) {
        uint4* dst = reinterpret_cast<uint4*>(S.codes + ((long long)u * L.Tcap + p) * S.row_bytes) + li * 4;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) dst[c4] = cw[c4];
        if (in_anchor(L, p, R.len)) {
          uint4* ap = reinterpret_cast<uint4*>(S.anchors + ((long long)u * L.anchor_rows + anchor_slot(L, p)) * D) + li * 4;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) ap[c4] = cw[c4];
        }
      }
    } else {
      quantize_slice<TcFam<VF>::fam, GV, TcFam<VF>::bits, false>(L, L.s[1], cw, mine, u, p, R.len);
    }
  }
  // the rows were written through the generic proxy; the tile copies read them through the async one
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
}

// The split-K pass; FUSE: the fused append + decode step (see fused_append_rows).
template <int D, int G, int KF, int GK, int VF, int GV, int NW, int TPW, int STAGES, bool FUSE>
__device__ __forceinline__ void decode_tc_body(const LayerDev& L, const __half* __restrict__ q,
                                               const int* __restrict__ seq_ids, const int* __restrict__ kv_len,
                                               float* __restrict__ work, int n_split, int nsp_total) {
  using C = TcCfg<D, KF, GK, VF, GV, NW, TPW, STAGES>;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // full[s]: tile landed (bytes)
  uint64_t* ebar = bar + STAGES;                                      // empty[s]: every consumer warp done
  uint64_t* dummy = ebar + STAGES;                                    // never arrived on (test hook)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dummy + 1);  // a consumer gave up

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int split = blockIdx.x, kvh = blockIdx.y, qi = blockIdx.z;
  const QueryRange R = query_range<FUSE>(L, qi, seq_ids, kv_len);
  const SideDev& K = L.s[0];
  const SideDev& V = L.s[1];
  const long long u = (long long)R.seq * L.Hkv + kvh;

  // ---- token range of this split, in whole tiles
  const int tstart = (R.qa / C::TILE) * C::TILE;
  const int ntiles = R.qb > tstart ? (R.qb - tstart + C::TILE - 1) / C::TILE : 0;
  const int per = (ntiles + n_split - 1) / n_split;
  const int it0 = split * per;
  const int nmy = max(0, min(ntiles, it0 + per) - it0);

  const uint8_t* gK = K.codes + u * L.Tcap * C::RSK;
  const uint8_t* gKs = reinterpret_cast<const uint8_t*>(K.scales + u * L.Tcap * C::NGK);
  const uint8_t* gV = V.codes + u * L.Tcap * C::RSV;
  const uint8_t* gVs = C::VSROW ? reinterpret_cast<const uint8_t*>(V.scales + u * L.Tcap * C::NGV) : nullptr;

  auto issue = [&](int tile_idx, int stage) {  // one thread: eight bulk copies (six for fp16 V)
    const long long t0 = tstart + (long long)tile_idx * C::TILE, t1 = t0 + C::HALF;
    unsigned char* st = smem + stage * C::STAGE_BYTES;
    uint64_t* b = bar + stage;
    fence_proxy_async();
    mbar_expect_tx(b, C::TX_BYTES);
    bulk_g2s(st + C::OFF_KA, gK + t0 * C::RSK, C::KC_H, b);
    bulk_g2s(st + C::OFF_KB, gK + t1 * C::RSK, C::KC_H, b);
    bulk_g2s(st + C::OFF_KSA, gKs + t0 * C::NGK * 2, C::KS_H, b);
    bulk_g2s(st + C::OFF_KSB, gKs + t1 * C::NGK * 2, C::KS_H, b);
    bulk_g2s(st + C::OFF_VA, gV + t0 * C::RSV, C::VC_H, b);
    bulk_g2s(st + C::OFF_VB, gV + t1 * C::RSV, C::VC_H, b);
    if (C::VSROW) {
      bulk_g2s(st + C::OFF_VSA, gVs + t0 * C::NGV * 2, C::VS_H, b);
      bulk_g2s(st + C::OFF_VSB, gVs + t1 * C::NGV * 2, C::VS_H, b);
    }
  };

  const bool producer = C::PROD && warp == NW;  // lane 0 of the extra warp moves the tiles
  // Fused append + decode: this call's new rows that this CTA owns are written by warp 0 before a
  // copy reads them.  Without a producer warp, when the first copies hold none of them, those
  // copies go out first and the rows are written while they are in flight (the issuing thread is
  // in warp 0, and every later copy follows a CTA barrier).
  const int t_lo = tstart + it0 * C::TILE, t_hi = tstart + (it0 + nmy) * C::TILE;
  bool fuse_late = false;
  if constexpr (FUSE) {
    if (R.fresh > 0) {
      const int p0 = R.len - R.fresh, first_hi = min(t_hi, t_lo + (STAGES - 1) * C::TILE);
      const int a = max(p0, max(R.qa, t_lo)), b = min(R.len, min(R.qb, first_hi));  // owned rows in the first copies
      fuse_late = !C::PROD && a >= b;
      if (!fuse_late && warp == 0) fused_append_rows<D, KF, GK, VF, GV>(L, R, qi, kvh, split, t_lo, t_hi);
    }
  }
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar + s, 1);
      mbar_init(ebar + s, NW);
    }
    mbar_init(dummy, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();
  int issued = 0;  // tiles the producer has issued
  if constexpr (C::PROD) {
    if (producer && lane == 0)
      for (; issued < STAGES && issued < nmy; ++issued) issue(it0 + issued, issued);
  } else if (tid == 0) {
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s)
      if (s < nmy) issue(it0 + s, s);
  }
  if constexpr (FUSE) {
    if (fuse_late && warp == 0) fused_append_rows<D, KF, GK, VF, GV>(L, R, qi, kvh, split, t_lo, t_hi);
  }

  // ---- while the first tiles are in flight: NF4 table, query fragments
  const uint32_t lut = smem_u32(smem + C::OFF_LUT) + 4 * lane;
  if constexpr (C::LUT_BYTES > 0) {
    uint32_t* t = reinterpret_cast<uint32_t*>(smem + C::OFF_LUT);
    for (int b = warp * 32 + lane; b < 256; b += NW * 32) {
      uint32_t v;
      if constexpr (KF == CF_NF4) {
        v = pack_h2(d_nf4[b & 15], d_nf4[b >> 4]);
      } else {  // ternary byte -> its five digits as 2-bit fields (bytes above 242 do not occur)
        v = 0u;
        int r = b < 243 ? b : 0;
#pragma unroll
        for (int m = 0; m < 5; ++m) {
          v |= (uint32_t)(r % 3) << (2 * m);
          r /= 3;
        }
      }
#pragma unroll 8
      for (int i = 0; i < 32; ++i) t[b * 32 + ((lane + i) & 31)] = v;  // lanes write distinct banks
    }
  }
  float* qs = reinterpret_cast<float*>(smem + C::OFF_PK);
  query_mean_term(L, q, qi, R.seq, kvh, G, qs + 4 * D);
  prepare_query_rot<D>(L, q, qi, kvh, G, qs);
  // logit term of the sequence's key mean (0 without one): it starts every score accumulator
  const float kmu = head_ok_of(c, G) ? qs[4 * D + c] : 0.0f;
  uint32_t qreg[C::NGKM][C::KSTEPS][2];
  {
    const int h = g >> 1, part = g & 1;
#pragma unroll
    for (int j = 0; j < C::NGKM; ++j) {
      const int cb = j * C::GKM + c * (C::GKM / 4);
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          int e1, e2;
          k_pair_elems<KF>(2 * ks + r, e1, e2);
          float v1 = 0.0f, v2 = 0.0f;
          if (h < G) {
            v1 = qs[h * D + cb + e1];
            v2 = qs[h * D + cb + e2];
          }
          const float h1 = __half2float(__float2half_rn(v1)), h2 = __half2float(__float2half_rn(v2));
          qreg[j][ks][r] = part ? pack_h2(v1 - h1, v2 - h2) : pack_h2(h1, h2);
        }
      }
    }
  }
  __syncthreads();  // qs aliases the P' area; the table is complete

  float oacc[D / 16][4];
#pragma unroll
  for (int i = 0; i < D / 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.0f;
  float m_run = -INFINITY, l_run = 0.0f;
  const bool head_ok = c < G;
  uint32_t* pk = reinterpret_cast<uint32_t*>(smem + C::OFF_PK) + warp * C::PK_WORDS;
  // Score rows g and g + 8 are tokens (sh, si) and (sh, si + 4) of each block's 8 tokens per half;
  // V rows of lane c are tokens (vh, vi + {0, 4, 2, 6}).  Blocks of a warp start at index hb.
  const int sh = C::row_half(g), si = C::row_index(g);
  const int vh = C::row_half(c), vi = C::row_index(c);
  const int hb0 = warp * (TPW / 2);
  const int ks_off = (sh ? C::OFF_KSB : C::OFF_KSA) + (hb0 + si) * C::NGK * 2;   // K scales, row g
  // codes are read from the stage, or for ternary from this warp's transcoded rows (base `smem`)
  const int kc_off = C::KTRN ? C::OFF_X + warp * C::XW + (sh ? C::XKB : 0) + si * C::RBK + c * C::KCB
                             : (sh ? C::OFF_KB : C::OFF_KA) + (hb0 + si) * C::RBK + c * C::KCB;
  const int vs_off = (sh ? C::OFF_VSB : C::OFF_VSA) + (hb0 + si) * C::NGV * 2;
  const int vc_off = C::VX ? C::OFF_X + warp * C::XW + C::XKS + (vh ? C::XVB : 0) + vi * C::RBV +
                                   g * C::VCB
                             : (vh ? C::OFF_VB : C::OFF_VA) + (hb0 + vi) * C::RBV + g * C::VCB;
  const int vsc_off = (vh ? C::OFF_VSB : C::OFF_VSA) + (hb0 + vi) * C::NGV * 2 + g * C::VCS;  // sign V
  const int st_tok = sh * C::HALF + hb0 + si;  // tile-relative token of score row g, block 0
  const int vt_tok = vh * C::HALF + hb0 + vi;  // tile-relative token of V row c, block 0
  bool timed_out = false;
  int it = 0;

  if (producer) {  // refill a stage once every consumer warp has released it (bounded waits)
    if (lane == 0) {
      for (; issued < nmy; ++issued) {
        const int s = issued % STAGES;
        if (!mbar_wait(ebar + s, (uint32_t)(issued / STAGES - 1) & 1u)) {
          atomicOr(L.err, (unsigned)KVQ_ERRF_WAIT_TIMEOUT);
          timed_out = true;
          break;
        }
        if (*abort_flag) break;  // a consumer gave up: the stage may still be landing
        issue(it0 + issued, s);
      }
    }
  } else for (; it < nmy; ++it) {
    if constexpr (!C::PROD) {
      if (__syncthreads_or(timed_out)) break;  // every warp is done with tile it - 1: refill its stage
      if (tid == 0 && it + STAGES - 1 < nmy) issue(it0 + it + STAGES - 1, (it + STAGES - 1) % STAGES);
    }
    const int stage = it % STAGES;
    // (test hook: the first wait polls a barrier nothing arrives on, for L.test_stall cycles)
    const bool stall = L.test_stall > 0 && it == 0;
    if (!timed_out && __any_sync(0xffffffffu, !(stall ? mbar_wait(dummy, 0u, L.test_stall)
                                                      : mbar_wait(bar + stage, (uint32_t)(it / STAGES) & 1u)))) {
      if (lane == 0) atomicOr(L.err, (unsigned)KVQ_ERRF_WAIT_TIMEOUT);
      timed_out = true;
    }
    if (timed_out) {  // release the stage without reading it; the producer issues no more tiles
      if (C::PROD && lane == 0) {
        *abort_flag = 1;
        mbar_arrive(ebar + stage);
      }
      continue;
    }

    const unsigned char* st = smem + stage * C::STAGE_BYTES;
    const int tile_t0 = tstart + (it0 + it) * C::TILE;
    const bool full_tile = tile_t0 >= R.qa && tile_t0 + C::TILE <= R.qb;
    const unsigned char* kb_ = C::KTRN ? smem : st;  // base of K code reads
    const unsigned char* vb_ = C::VX ? smem : st;    // base of V code reads
    if constexpr (C::KTRN || C::VX) {  // lane l transcodes row (half l / 16, index l % 16) of this warp
      const int R2 = lane >> 4, li = lane & 15;
      unsigned char* xw = smem + C::OFF_X + warp * C::XW;
      if constexpr (C::KTRN)
        tern_transcode(st + (R2 ? C::OFF_KB : C::OFF_KA) + (hb0 + li) * C::RSK, xw + (R2 ? C::XKB : 0) + li * 32, lut);
      if constexpr (C::VTRN)
        tern_transcode(st + (R2 ? C::OFF_VB : C::OFF_VA) + (hb0 + li) * C::RSV,
                       xw + C::XKS + (R2 ? C::XVB : 0) + li * 32, lut);
      if constexpr (C::V3)
        int3_transcode<D>(st + (R2 ? C::OFF_VB : C::OFF_VA) + (hb0 + li) * C::RSV,
                           xw + C::XKS + (R2 ? C::XVB : 0) + li * C::RBV);
      __syncwarp();
    }

    // ---- scores: thread (g, c) gets head c's logits of score rows g and g + 8 of each block
    float sc[C::NSB][2];
#pragma unroll
    for (int sb = 0; sb < C::NSB; ++sb) {
      if constexpr (C::KSCL) {  // scale inside the operand: one accumulator over the row
        const unsigned char* k0p = kb_ + kc_off + sb * 8 * C::RBK;
        const unsigned char* s0p = st + ks_off + sb * 8 * C::NGK * 2 + c * C::KCS;
        uint32_t kw0[C::KCW], kw1[C::KCW], sv0[C::KCS / 4], sv1[C::KCS / 4];
        lds_words<C::KCW>(k0p, kw0);
        lds_words<C::KCW>(k0p + 4 * C::RBK, kw1);
        lds_words<C::KCS / 4>(s0p, sv0);
        lds_words<C::KCS / 4>(s0p + 4 * C::NGK * 2, sv1);
        uint32_t kp0[2 * C::KSTEPS], kp1[2 * C::KSTEPS];
        if constexpr (C::KSGN) {
#pragma unroll
          for (int w = 0; w < C::KCW; ++w) {
            sign_pairs_k(kw0[w], sv0 + 4 * w, kp0 + 16 * w);
            sign_pairs_k(kw1[w], sv1 + 4 * w, kp1 + 16 * w);
          }
        } else {  // ternary, groups of 8: word w of the chunk spans groups 2w, 2w + 1 (halves of sv[w])
#pragma unroll
          for (int w = 0; w < C::KCW; ++w) {
            tern_pairs(kw0[w], sv0[w], kp0 + 8 * w);
            tern_pairs(kw1[w], sv1[w], kp1 + 8 * w);
          }
        }
        float acc[4] = {kmu, 0.0f, kmu, 0.0f};
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks)
          mma16816(acc, kp0[2 * ks], kp1[2 * ks], kp0[2 * ks + 1], kp1[2 * ks + 1], qreg[0][ks][0], qreg[0][ks][1]);
        float s0 = acc[0] + acc[1], s1 = acc[2] + acc[3];
        if (!full_tile) {
          const int t0 = tile_t0 + st_tok + sb * 8, t1 = t0 + 4;
          s0 = (t0 >= R.qa && t0 < R.qb) ? s0 : -INFINITY;
          s1 = (t1 >= R.qa && t1 < R.qb) ? s1 : -INFINITY;
        }
        sc[sb][0] = s0;
        sc[sb][1] = s1;
      } else {
      float kd0[C::NGK], kd1[C::NGK];
      {
        const __half* s0p = reinterpret_cast<const __half*>(st + ks_off + sb * 8 * C::NGK * 2);
        const __half* s1p = s0p + 4 * C::NGK;
        if constexpr (C::NGK == 2) {
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(s0p));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(s1p));
          kd0[0] = a.x; kd0[1] = a.y; kd1[0] = b.x; kd1[1] = b.y;
        } else {
#pragma unroll
          for (int j = 0; j < C::NGK; ++j) {
            kd0[j] = __half2float(s0p[j]);
            kd1[j] = __half2float(s1p[j]);
          }
        }
      }
      const unsigned char* k0p = kb_ + kc_off + sb * 8 * C::RBK;
      const unsigned char* k1p = k0p + 4 * C::RBK;
      float s0 = kmu, s1 = kmu;
#pragma unroll
      for (int j = 0; j < C::NGK; ++j) {
        uint32_t kw0[C::KCW], kw1[C::KCW];
        lds_words<C::KCW>(k0p + j * C::GKB, kw0);
        lds_words<C::KCW>(k1p + j * C::GKB, kw1);
        uint32_t kp0[2 * C::KSTEPS], kp1[2 * C::KSTEPS];
        if constexpr (KF == CF_NF4) {
#pragma unroll
          for (int w = 0; w < C::KCW; ++w) {
              kp0[4 * w + 0] = lut_pair<0>(lut, kw0[w]);
              kp0[4 * w + 1] = lut_pair<1>(lut, kw0[w]);
              kp0[4 * w + 2] = lut_pair<2>(lut, kw0[w]);
              kp0[4 * w + 3] = lut_pair<3>(lut, kw0[w]);
              kp1[4 * w + 0] = lut_pair<0>(lut, kw1[w]);
              kp1[4 * w + 1] = lut_pair<1>(lut, kw1[w]);
              kp1[4 * w + 2] = lut_pair<2>(lut, kw1[w]);
              kp1[4 * w + 3] = lut_pair<3>(lut, kw1[w]);
            }
        } else {
          constexpr int PPW = 16 / C::KB;
#pragma unroll
          for (int w = 0; w < C::KCW; ++w) {
            code_pairs<C::KB>(kw0[w], kp0 + w * PPW);
            code_pairs<C::KB>(kw1[w], kp1 + w * PPW);
          }
        }
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks)
          mma16816(acc, kp0[2 * ks], kp1[2 * ks], kp0[2 * ks + 1], kp1[2 * ks + 1], qreg[j][ks][0], qreg[j][ks][1]);
        s0 = fmaf(kd0[j], acc[0] + acc[1], s0);
        s1 = fmaf(kd1[j], acc[2] + acc[3], s1);
      }
      if (!full_tile) {
        const int t0 = tile_t0 + st_tok + sb * 8, t1 = t0 + 4;
        s0 = (t0 >= R.qa && t0 < R.qb) ? s0 : -INFINITY;
        s1 = (t1 >= R.qa && t1 < R.qb) ? s1 : -INFINITY;
      }
      sc[sb][0] = s0;
      sc[sb][1] = s1;
      }
    }

    // ---- online softmax (log2 domain) for head c over this warp's TPW tokens.  The reference
    // max moves only when the tile's max exceeds it by more than C::SLACK, so p <= 2^SLACK and the
    // accumulators are rescaled rarely; p * d_v still fits fp16 for any stored V scale.
    float tmax = -INFINITY;
#pragma unroll
    for (int sb = 0; sb < C::NSB; ++sb) tmax = fmaxf(tmax, fmaxf(sc[sb][0], sc[sb][1]));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
    const bool move = tmax > m_run + C::SLACK;
    if (__any_sync(0xffffffffu, move)) {
      const float alpha = move ? ex2(m_run - tmax) : 1.0f;  // 0 when m_run = -inf
      const float m_new = move ? tmax : m_run;
      l_run *= alpha;
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        oacc[i][0] *= alpha;
        oacc[i][1] *= alpha;
        oacc[i][2] *= alpha;
        oacc[i][3] *= alpha;
      }
      m_run = m_new;
    }
    if (m_run != -INFINITY) {
#pragma unroll
      for (int sb = 0; sb < C::NSB; ++sb) {
        sc[sb][0] = ex2(sc[sb][0] - m_run);
        sc[sb][1] = ex2(sc[sb][1] - m_run);
        l_run += sc[sb][0] + sc[sb][1];
      }
    } else {
#pragma unroll
      for (int sb = 0; sb < C::NSB; ++sb) sc[sb][0] = sc[sb][1] = 0.0f;
    }

    // ---- values
#pragma unroll
    for (int sb = 0; sb < C::NSB; ++sb) {
      {  // P' (hi, lo) of score rows g and g + 8 for head c: word g of rows 2c and 2c + 1
        const float p0 = (G == 4 || head_ok) ? sc[sb][0] : 0.0f, p1 = (G == 4 || head_ok) ? sc[sb][1] : 0.0f;
        float dv0[C::NPV], dv1[C::NPV];
        if constexpr (C::VSCALE) {
          const __half* d0p = reinterpret_cast<const __half*>(st + vs_off + sb * 8 * C::NGV * 2);
          const __half* d1p = d0p + 4 * C::NGV;
          if constexpr (C::NGV == 2) {
            const float2 a = __half22float2(*reinterpret_cast<const __half2*>(d0p));
            const float2 b = __half22float2(*reinterpret_cast<const __half2*>(d1p));
            dv0[0] = a.x; dv0[1] = a.y; dv1[0] = b.x; dv1[1] = b.y;
          } else {
#pragma unroll
            for (int v = 0; v < C::NGV; ++v) {
              dv0[v] = __half2float(d0p[v]);
              dv1[v] = __half2float(d1p[v]);
            }
          }
        } else {
          dv0[0] = dv1[0] = 1.0f;
        }
#pragma unroll
        for (int v = 0; v < C::NPV; ++v) {
          float x0 = p0 * dv0[v], x1 = p1 * dv1[v];
          if (!full_tile) {  // masked tokens may carry unwritten (non-finite) scales
            x0 = p0 == 0.0f ? 0.0f : x0;
            x1 = p1 == 0.0f ? 0.0f : x1;
          }
          const __half2 hi = __floats2half2_rn(x0, x1);
          const float2 hf = __half22float2(hi);
          const __half2 lo = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
          pk[(v * 8 + 2 * c) * C::PKS + g] = h2u(hi);
          pk[(v * 8 + 2 * c + 1) * C::PKS + g] = h2u(lo);
        }
      }
      __syncwarp();
      uint32_t vmask_a = 0xFFFFFFFFu, vmask_c = 0xFFFFFFFFu;
      if ((VF == CF_FP16 || C::VSCL) && !full_tile) {  // unwritten rows may hold NaN (fp16 values or sign
                                                        // scales); zero them (p is 0 there)
        const int t = tile_t0 + vt_tok + sb * 8;
        auto ok = [&](int d) { return t + d >= R.qa && t + d < R.qb; };
        vmask_a = (ok(0) ? 0x0000FFFFu : 0u) | (ok(4) ? 0xFFFF0000u : 0u);
        vmask_c = (ok(2) ? 0x0000FFFFu : 0u) | (ok(6) ? 0xFFFF0000u : 0u);
      }
#pragma unroll
      for (int gv = 0; gv < C::NGVM; ++gv) {
        const uint32_t* pr = pk + ((C::VSCALE ? gv : 0) * 8 + g) * C::PKS;
        const uint32_t b0 = pr[c], b1 = pr[c + 4];
        const unsigned char* vp = vb_ + vc_off + sb * 8 * C::RBV + gv * C::GVB;
        uint32_t vw[4][C::VCW];
        constexpr int roff[4] = {0, 4, 2, 6};  // slots (2c, 2c+1) then (2c+8, 2c+9)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if constexpr (C::VCB == 2) {
            vw[i][0] = *reinterpret_cast<const uint16_t*>(vp + roff[i] * C::RBV);
          } else {
            lds_words<C::VCW>(vp + roff[i] * C::RBV, vw[i]);
          }
        }
        uint32_t pa[C::GVM / 8], pc[C::GVM / 8];
        if constexpr (C::VTRN) {  // rows (vi, vi+4) -> pa, (vi+2, vi+6) -> pc; half hh is group 2g + hh
          const unsigned char* sp = st + vsc_off + sb * 8 * C::NGV * 2;
          uint32_t s4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) s4[i] = *reinterpret_cast<const uint32_t*>(sp + roff[i] * C::NGV * 2);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint32_t sel = hh ? 0x7632u : 0x5410u;
            tern_pairs(prmt(vw[0][0], vw[1][0], sel), prmt(s4[0], s4[1], sel), pa + 8 * hh);
            tern_pairs(prmt(vw[2][0], vw[3][0], sel), prmt(s4[2], s4[3], sel), pc + 8 * hh);
          }
          if (!full_tile) {
#pragma unroll
            for (int e = 0; e < C::GVM / 8; ++e) {
              pa[e] &= vmask_a;
              pc[e] &= vmask_c;
            }
          }
        } else if constexpr (C::VSGN) {  // rows (vi, vi+4) -> pa, (vi+2, vi+6) -> pc, scales of each row's 4 groups per half
          const unsigned char* sp = st + vsc_off + sb * 8 * C::NGV * 2;
          uint32_t s4[4][C::VCS / 4];
#pragma unroll
          for (int i = 0; i < 4; ++i) lds_words<C::VCS / 4>(sp + roff[i] * C::NGV * 2, s4[i]);
#pragma unroll
          for (int hh = 0; hh < C::VCH; ++hh) {
            const int w = hh >> 1, hf = hh & 1;
            sign_pairs_v(prmt(vw[0][w], vw[1][w], hf ? 0x7632 : 0x5410), s4[0] + 2 * hh, s4[1] + 2 * hh, pa + 16 * hh);
            sign_pairs_v(prmt(vw[2][w], vw[3][w], hf ? 0x7632 : 0x5410), s4[2] + 2 * hh, s4[3] + 2 * hh, pc + 16 * hh);
          }
          if (!full_tile) {
#pragma unroll
            for (int e = 0; e < C::GVM / 8; ++e) {
              pa[e] &= vmask_a;
              pc[e] &= vmask_c;
            }
          }
        } else if constexpr (VF == CF_FP16) {
#pragma unroll
          for (int w = 0; w < C::VCW; ++w) {
            pa[2 * w] = prmt(vw[0][w], vw[1][w], 0x5410) & vmask_a;
            pa[2 * w + 1] = prmt(vw[0][w], vw[1][w], 0x7632) & vmask_a;
            pc[2 * w] = prmt(vw[2][w], vw[3][w], 0x5410) & vmask_c;
            pc[2 * w + 1] = prmt(vw[2][w], vw[3][w], 0x7632) & vmask_c;
          }
        } else {
          constexpr int PH = 16 / C::VB;  // elements per 16-bit half
#pragma unroll
          for (int hh = 0; hh < C::VCH; ++hh) {
            const int w = hh >> 1, hf = hh & 1;
            code_pairs<C::VB>(prmt(vw[0][w], vw[1][w], hf ? 0x7632 : 0x5410), pa + hh * PH, C::VOFS);
            code_pairs<C::VB>(prmt(vw[2][w], vw[3][w], hf ? 0x7632 : 0x5410), pc + hh * PH, C::VOFS);
          }
        }
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt)
          mma16816(oacc[gv * C::MT + mt], pa[2 * mt], pa[2 * mt + 1], pc[2 * mt], pc[2 * mt + 1], b0, b1);
      }
      __syncwarp();
    }
    if (C::PROD && lane == 0) mbar_arrive(ebar + stage);  // this warp no longer reads the stage
  }

  // After a timed-out wait the last tile issued into each stage may still be landing: the
  // producer waits for them (bounded again) before the stage buffers are reused or the CTA exits.
  timed_out = __syncthreads_or(timed_out);
  if constexpr (C::PROD) {
    if (timed_out && producer && lane == 0) {
      for (int s = 0; s < STAGES; ++s) {
        const int last = issued - 1 - ((issued - 1 - s) % STAGES + STAGES) % STAGES;  // last tile issued into s
        if (last >= 0) mbar_wait(bar + s, (uint32_t)(last / STAGES) & 1u);
      }
    }
  } else if (timed_out && tid == 0) {
    const int iss = min(nmy, it + STAGES - 1);
    for (int i = max(it - 1, 0); i < iss; ++i) mbar_wait(bar + i % STAGES, (uint32_t)(i / STAGES) & 1u);
  }
  __syncthreads();  // stage buffers are free: reuse them to combine the warps

  // ---- combine the warps' (m, l, o) into one partial per CTA
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 4);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
  float* red = reinterpret_cast<float*>(smem);  // [NW][4 heads][D]
  float* ml = red + NW * 4 * D;                 // [NW][4 heads][2]
  if (timed_out) {
    m_run = -INFINITY;
    l_run = 0.0f;
  }
  if (head_ok && !producer) {
    if (g == 0) {
      ml[(warp * 4 + c) * 2] = m_run;
      ml[(warp * 4 + c) * 2 + 1] = l_run;
    }
#pragma unroll
    for (int gv = 0; gv < C::NGVM; ++gv)
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) {
        const int ch = gv * C::GVM + g * (C::GVM / 8) + 2 * mt;
        const float* o = oacc[gv * C::MT + mt];
        *reinterpret_cast<float2*>(red + (warp * 4 + c) * D + ch) =
            timed_out ? make_float2(0.0f, 0.0f) : make_float2(o[0] + o[1], o[2] + o[3]);
      }
  }
  __syncthreads();
  for (int e = tid; e < G * D && tid < C::NT; e += C::NT) {
    const int h = e / D, j = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, ml[(w * 4 + h) * 2]);
    float lsum = 0.0f, osum = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = ml[(w * 4 + h) * 2];
        const float sc = mw == -INFINITY ? 0.0f : ex2(mw - M);
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

template <int D, int G, int KF, int GK, int VF, int GV, int NW, int TPW, int STAGES>
__global__ void __launch_bounds__(TcCfg<D, KF, GK, VF, GV, NW, TPW, STAGES>::NTH)
    decode_tc_kernel(LayerDev L, const __half* __restrict__ q, const int* __restrict__ seq_ids,
                     const int* __restrict__ kv_len, float* __restrict__ work, int n_split, int nsp_total) {
  decode_tc_body<D, G, KF, GK, VF, GV, NW, TPW, STAGES, false>(L, q, seq_ids, kv_len, work, n_split, nsp_total);
}

// The fused append + decode instance: held to MINB CTAs per SM (the plain instance's occupancy),
// so that the once-per-CTA row quantization may spill but never costs residency; LayerDev is a
// __grid_constant__ parameter, so the non-inlined row quantization reads it in place.
template <int D, int G, int KF, int GK, int VF, int GV, int NW, int TPW, int STAGES, int MINB>
__global__ void __launch_bounds__(TcCfg<D, KF, GK, VF, GV, NW, TPW, STAGES>::NTH, MINB)
    decode_tc_fused_kernel(const __grid_constant__ LayerDev L, const __half* __restrict__ q,
                           const int* __restrict__ seq_ids, const int* __restrict__ kv_len,
                           float* __restrict__ work, int n_split, int nsp_total) {
  decode_tc_body<D, G, KF, GK, VF, GV, NW, TPW, STAGES, true>(L, q, seq_ids, kv_len, work, n_split, nsp_total);
}
