// kvq_dequantize: packed rows back to values, in the stored domain (code x scale (+ zero); polar
// m cos phi, m sin phi) or the original domain (inverse DFT, inverse Hadamard, x channel scale,
// anchored rows replaced by their fp16 copy).  One warp per row; not on the decode hot path.
#include "decode_common.cuh"
#include "kvq_internal.h"

namespace kvq {

__constant__ float dq_nf4[16];
__constant__ float dq_tw_re[64];
__constant__ float dq_tw_im[64];
__constant__ float dq_ph_cos[512];
__constant__ float dq_ph_sin[512];
__constant__ float dq_lloyd[3][16];

cudaError_t upload_tables_dequant(const HostTables& t) {
  cudaError_t e;
  if ((e = cudaMemcpyToSymbol(dq_nf4, t.nf4, sizeof(t.nf4))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(dq_tw_re, t.tw_re, sizeof(t.tw_re))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(dq_tw_im, t.tw_im, sizeof(t.tw_im))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(dq_ph_cos, t.ph_cos, sizeof(t.ph_cos))) != cudaSuccess) return e;
  if ((e = cudaMemcpyToSymbol(dq_lloyd, t.lloyd, sizeof(t.lloyd))) != cudaSuccess) return e;
  return cudaMemcpyToSymbol(dq_ph_sin, t.ph_sin, sizeof(t.ph_sin));
}

constexpr int kDqWarps = 4;

__global__ void __launch_bounds__(128) dequant_kernel(LayerDev L, int side, int domain, int t0, int nt,
                                                      void* __restrict__ out, int out_fp32) {
  const SideDev& S = L.s[side];
  const int D = L.D;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float buf[kDqWarps][256], tmp[kDqWarps][256];
  __shared__ float nf4[16], lloyd[16], cs[256], sn[256];
  if (threadIdx.x < 16) nf4[threadIdx.x] = dq_nf4[threadIdx.x];
  if (S.fmt == KVQ_FMT_LLOYD && threadIdx.x < 16) lloyd[threadIdx.x] = dq_lloyd[S.bits - 2][threadIdx.x];
  if (S.fmt == KVQ_FMT_POLAR)
    for (int k = threadIdx.x; k < (1 << S.bits2); k += blockDim.x) {
      cs[k] = dq_ph_cos[(1 << S.bits2) - 2 + k];
      sn[k] = dq_ph_sin[(1 << S.bits2) - 2 + k];
    }
  __syncthreads();
  const long long R = (long long)L.B * L.Hkv * nt;
  const long long row = (long long)blockIdx.x * kDqWarps + warp;
  if (row >= R) return;
  const int i = (int)(row % nt);
  const long long u = row / nt;
  const int t = t0 + i;
  const long long rix = u * L.Tcap + t;
  const uint8_t* cr = S.codes + rix * S.row_bytes;
  const __half* sc = S.scales + rix * S.n_groups;
  const __half* zr = S.zeros ? S.zeros + rix * S.n_groups : nullptr;
  float* x = buf[warp];
  if (S.fmt == KVQ_FMT_POLAR) {
    for (int f = lane; f < 64; f += 32) {
      const float2 ab = polar_slot(S, cr, sc, f, cs, sn);
      x[2 * f] = ab.x;
      x[2 * f + 1] = ab.y;
    }
  } else {
    for (int j = lane; j < D; j += 32) x[j] = stored_value(S, cr, sc, zr, j, nf4, lloyd);
  }
  __syncwarp();
  if (domain == KVQ_DOMAIN_ORIGINAL) {
    if (S.fmt == KVQ_FMT_POLAR || S.fmt == KVQ_FMT_CART) {
      float* y = tmp[warp];
      for (int j = lane; j < 128; j += 32) y[j] = x[j];
      __syncwarp();
      for (int n = lane; n < 128; n += 32) {
        float acc = y[0] + ((n & 1) ? -y[1] : y[1]);
        float sacc = 0.0f;
        for (int f = 1; f < 64; ++f) {
          const int k = (f * n) & 127;
          const float c = k < 64 ? dq_tw_re[k] : -dq_tw_re[k - 64];
          const float s = k < 64 ? -dq_tw_im[k] : dq_tw_im[k - 64];
          sacc += y[2 * f] * c - y[2 * f + 1] * s;
        }
        x[n] = (acc + 2.0f * sacc) / 128.0f;
      }
      __syncwarp();
    }
    if (S.rot == 128 || S.rot == 256) {
      for (int h = 1; h < S.rot; h <<= 1) {
        for (int p = lane; p < D / 2; p += 32) {
          const int lo = p & (h - 1), hi = p >> (__ffs(h) - 1);
          const int ii = (hi << __ffs(h)) | lo;
          const float a = x[ii], b = x[ii + h];
          x[ii] = a + b;
          x[ii + h] = a - b;
        }
        __syncwarp();
      }
      const float rn = (S.rot == 256) ? 0.0625f : 0.08838834764831845f;
      for (int j = lane; j < D; j += 32) x[j] *= rn;
      __syncwarp();
    }
    if (S.chan_scale)
      for (int j = lane; j < D; j += 32) x[j] *= __half2float(S.chan[(u % L.Hkv) * D + j]);
    if (S.mean_sub)
      for (int j = lane; j < D; j += 32) x[j] += __half2float(S.kmean[u * D + j]);
    // anchored rows: attention reads the fp16 copy
    bool anc = false;
    if (L.anchored) {
      const int len = L.seq_len[u / L.Hkv];
      if (L.anchor_rule == KVQ_ANCHOR_FIRST_N) anc = t < L.anchor_n;
      else if (L.anchor_rule == KVQ_ANCHOR_WINDOW) anc = t >= len - L.anchor_n && t < len;
      else if (L.anchor_rule == KVQ_ANCHOR_ALL) anc = true;
    }
    if (anc) {
      const int slot = L.anchor_rule == KVQ_ANCHOR_WINDOW ? t % L.anchor_n : t;
      for (int j = lane; j < D; j += 32) x[j] = anchor_value(L, S, u * L.anchor_rows + slot, j);
    }
    __syncwarp();
  }
  const long long ob = (((u / L.Hkv) * L.Hkv_all + L.h0 + u % L.Hkv) * nt + i) * D;  // caller's [B][Hkv_all][nt]
  for (int j = lane; j < D; j += 32) {
    if (out_fp32) reinterpret_cast<float*>(out)[ob + j] = x[j];
    else reinterpret_cast<__half*>(out)[ob + j] = __float2half_rn(x[j]);
  }
}

cudaError_t launch_dequant(const LayerDev& L, int side, int domain, int t0, int nt, void* out, int out_fp32,
                           cudaStream_t st) {
  const long long R = (long long)L.B * L.Hkv * nt;
  const unsigned blocks = (unsigned)((R + kDqWarps - 1) / kDqWarps);
  dequant_kernel<<<blocks, 128, 0, st>>>(L, side, domain, t0, nt, out, out_fp32);
  return cudaGetLastError();
}

__global__ void fill_kernel(int* p, int n, int v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

cudaError_t launch_fill_len(int* lens, int n, int value, cudaStream_t st) {
  fill_kernel<<<(n + 127) / 128, 128, 0, st>>>(lens, n, value);
  return cudaGetLastError();
}

}  // namespace kvq
