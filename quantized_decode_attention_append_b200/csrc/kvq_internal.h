// Internal definitions shared by the translation units of libkvq (not part of the C ABI).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvq.h"

namespace kvq {

// fp16 pairs as 32-bit words and back
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

constexpr int kMaxSplit = 256;     // split-K partitions per (query, kv-head)
constexpr int kPartStride = 4;     // floats of (m, l, pad, pad) before o[D] in a partial

// Division of n < 2^31 by a fixed d >= 1 as a multiply and a shift: m = ceil(2^(31 + l) / d),
// l = ceil(log2 d), so 2^(31 + l) <= m d < 2^(31 + l) + 2^l, which makes floor(n m / 2^(31 + l))
// equal floor(n / d) for every n < 2^31 (Granlund and Montgomery, "Division by invariant integers
// using multiplication", PLDI 1994, Theorem 4.2).
struct FastDiv {
  unsigned long long m;
  int sh;
};
inline FastDiv fast_div(unsigned d) {
  if (d == 0) d = 1;  // callers pass counts >= 1; never divide by zero on the host
  int l = 0;
  while ((1ull << l) < d) ++l;
  const int sh = 31 + l;
  return FastDiv{((1ull << sh) + d - 1) / d, sh};
}
__device__ __forceinline__ int div_by(int n, const FastDiv& f) {
  return (int)(((unsigned long long)(unsigned)n * f.m) >> f.sh);
}

// Device view of one (layer, side).
struct SideDev {
  uint8_t* codes;        // [B*Hkv][Tcap][row_bytes]
  __half* scales;        // [B*Hkv][Tcap][n_groups]
  __half* zeros;         // [B*Hkv][Tcap][n_groups] (MINMAX) or null
  __half* anchors;       // [B*Hkv][anchor_rows][D] fp16, or [..][anchor_rb] codes (int anchors), or null
  __half* anchor_scales; // int anchors: [B*Hkv][anchor_rows][D/32] or null
  const __half* chan;    // [Hkv][D] (K with chan_scale) or null
  __half* kmean;         // [B*Hkv][D] key means (K with mean_sub) or null
  int fmt, bits, bits2, scale_mode, group, rot, chan_scale, mean_sub;
  int row_bytes, n_groups;
};

// Device view of the kv-heads [h0, h0 + Hkv) of one layer that share one (K, V) format pair (all of
// its heads unless the layer has per-head formats).  Arena regions are the view's own: unit
// u = b * Hkv + local head.  The caller's arrays (queries, outputs, append inputs, dequantized
// rows) hold all Hkv_all heads of the layer.
struct LayerDev {
  SideDev s[2];
  int B, Hkv, Hq, D, Tcap;
  int Hkv_all, h0;       // kv-heads of the layer; first kv-head of this view
  int cap;               // configured capacity (tokens per sequence); appends never pass it
  int anchored;          // this layer keeps anchor rows
  int anchor_rule, anchor_n, anchor_rows;
  int anchor_bits, anchor_rb;  // 16 (fp16 rows) or 8/4 (code bytes per anchor row: anchor_rb)
  int* seq_len;          // [B] stored lengths of this layer
  unsigned* ticket;      // append completion counter of this layer
  unsigned* err;         // error word (KVQ_ERRF_*)
  float sm_scale;
  // append call: sequences that receive rows (null: every sequence, in order) and how many
  const int* app_ids;
  int app_n;
  FastDiv div_new, div_hkv;  // by the call's rows per sequence and by Hkv (row -> destination)
  long long test_stall;  // test hook (0 = off): the decode's first stage wait polls a barrier nothing
                         // arrives on for this many clock cycles, then gives up
  // fused append + decode (fuse_n > 0): query i's sequence also receives fuse_n new rows, input
  // rows [n_q][Hkv_all][fuse_n][D] fp16 of K (fuse_k) and V (fuse_v); the decode kernel writes
  // them before it reads them and the merge advances the stored length
  const __half* fuse_k;
  const __half* fuse_v;
  int fuse_n;
};

// Row of query head h (of kv-head kvh of the view, G query heads per kv-head) of query qi in the
// caller's [n_q][Hq_all][..] arrays.
__device__ __forceinline__ long long query_row(const LayerDev& L, int qi, int kvh, int G, int h) {
  return ((long long)qi * L.Hkv_all + L.h0 + kvh) * G + h;
}

// Caller row ([n_seqs][Hkv_all][n_new] order) of the view's append row `row` ([n_seqs][Hkv][n_new]);
// rows of one call are fewer than 2^31 (checked on the host), so 32-bit arithmetic suffices.
__device__ __forceinline__ int input_row(const LayerDev& L, int row, int n_new) {
  if (L.Hkv == L.Hkv_all) return row;
  const int ul = row / n_new, sl = ul / L.Hkv;
  return (sl * L.Hkv_all + L.h0 + (ul - sl * L.Hkv)) * n_new + (row - ul * n_new);
}

// Tables the host builds once (NF4 levels, FFT twiddles, phase cos/sin) and every
// translation unit uploads into its own constant memory.
struct HostTables {
  float nf4[16];
  float nf4_mid[15];
  float tw_re[64], tw_im[64];     // W_128^k = exp(-2 pi i k/128), k < 64
  float ph_cos[512], ph_sin[512]; // phase angle -pi + 2 pi k / 2^bp at offset 2^bp - 2
  float lloyd[3][16];             // Gaussian Lloyd-Max levels for 2, 3, 4 bits (2^b used)
  float lloyd_mid[3][15];         // their midpoints
};

const HostTables& host_tables();

// Per-TU uploaders (called once per device by kvq_create).
cudaError_t upload_tables_quant(const HostTables& t);
cudaError_t upload_tables_decode(const HostTables& t);
cudaError_t upload_tables_dequant(const HostTables& t);

// Launchers (host side, validate nothing; the API validates first).
// CTAs launch_append starts for `L` (the completion ticket of one append counts the CTAs of every
// view of the layer: total_ctas).
unsigned append_ctas(const LayerDev& L, int n_new);
cudaError_t launch_append(const LayerDev& L, const __half* k, const __half* v, int n_new, unsigned total_ctas,
                          cudaStream_t st, int* launches);
cudaError_t launch_dequant(const LayerDev& L, int side, int domain, int t0, int nt, void* out,
                           int out_fp32, cudaStream_t st);
cudaError_t launch_decode(const LayerDev& L, const __half* q, int n_q, const int* seq_ids,
                          const int* kv_len, void* out, int out_fp32, float* lse, float* work,
                          int num_sms, int max_queries, cudaStream_t st, int* launches);
cudaError_t launch_fill_len(int* lens, int n, int value, cudaStream_t st);
// Key means of the listed sequences whose first append this is (K side with mean_sub).
cudaError_t launch_key_mean(const LayerDev& L, const __half* k, int n_new, cudaStream_t st);

// Split-K partials per (query, head) one decode call on `L` writes (workspace sizing).
int decode_partials(const LayerDev& L, int n_q, int num_sms);
// Fused append + decode is available and chosen for this view and query count (see decode.cu).
bool fused_decode_ok(const LayerDev& L, int n_q, int num_sms);

// Fixed device scratch for the no-allocation decode entry point (decode.cu).
size_t static_work_floats();
cudaError_t static_work_ptr(int dev, float** out);

// Which append kernels exist for a side (the API reports KVQ_ERR_UNSUPPORTED otherwise).
bool append_supported(int D, const kvq_side& s);

}  // namespace kvq
