// C ABI of libkvq: configuration checks, arena layout, handle lifetime, launch wrappers.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <new>
#include <set>
#include <vector>

#include "kvq_internal.h"

using namespace kvq;

// Arena offsets of one side of one head group.
struct SideOff {
  int64_t codes, scales, zeros, anchors, anchor_scales;
  int row_bytes, n_groups;
};

// Consecutive kv-heads [h0, h0 + nh) of a layer with one (K, V) format pair: they share arena
// regions (unit = b * nh + local head) and are appended, decoded and dequantized by one set of
// launches.  A layer without per-head formats is one group.
struct HeadGroup {
  int h0, nh;
  kvq_side side[2];
  SideOff off[2];
  int64_t kmean;  // K key means [B * nh][D] fp16, or -1
};

struct kvq_cache {
  kvq_config cfg;
  std::vector<HeadGroup> grp[64];  // per layer
  int Tcap;
  char* arena;
  uint64_t arena_bytes;
  int64_t chan[64];      // per layer [Hkv][D] fp16 channel scales (some K side of the layer has them), or -1
  int64_t lens, tickets, err;
  int anchor_rows;
  int max_len[64];       // host-side bound on every sequence's length (exact while len_exact)
  bool len_exact[64];    // false once a per-sequence append made the bound inexact
  bool chan_set[64];
  long long test_stall;  // decode test hook, from KVQ_TEST_STALL_FIRST_WAIT (0 = off)
  float* work;
  size_t work_floats;
  int device, num_sms;
  int last_launches;
};

namespace {

constexpr uint64_t kAlign = 256;

uint64_t align_up(uint64_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool is_pow2_group(int g) { return g == 4 || g == 8 || g == 16 || g == 32 || g == 64 || g == 128; }

kvq_status check_side(const kvq_config& c, const kvq_side& s, bool is_k) {
  const int D = c.head_dim;
  if (!is_k && (s.chan_scale || s.mean_sub)) return KVQ_ERR_INVALID_ARG;
  if (s.chan_scale != 0 && s.chan_scale != 1) return KVQ_ERR_INVALID_ARG;
  if (s.mean_sub != 0 && s.mean_sub != 1) return KVQ_ERR_INVALID_ARG;
  if (s.mean_sub && s.format == KVQ_FMT_FP16) return KVQ_ERR_INVALID_ARG;
  if (s.rotation != KVQ_ROT_NONE && s.rotation != KVQ_ROT_H128 && s.rotation != KVQ_ROT_H256)
    return KVQ_ERR_INVALID_ARG;
  if (s.rotation > D) return KVQ_ERR_INVALID_ARG;
  switch (s.format) {
    case KVQ_FMT_FP16:
      if (s.rotation != KVQ_ROT_NONE || s.chan_scale) return KVQ_ERR_INVALID_ARG;
      return KVQ_OK;
    case KVQ_FMT_INT:
      if (s.bits < 2 || s.bits > 8) return KVQ_ERR_INVALID_ARG;
      if (s.scale_mode != KVQ_SCALE_ABSMAX && s.scale_mode != KVQ_SCALE_MINMAX && s.scale_mode != KVQ_SCALE_SYMMETRIC)
        return KVQ_ERR_INVALID_ARG;
      break;
    case KVQ_FMT_LLOYD:
    case KVQ_FMT_SORTED:
      if (s.bits < 2 || s.bits > 4) return KVQ_ERR_INVALID_ARG;
      if (s.scale_mode != KVQ_SCALE_ABSMAX) return KVQ_ERR_INVALID_ARG;
      break;
    case KVQ_FMT_NF4:
    case KVQ_FMT_TERNARY:
    case KVQ_FMT_SIGN:
      if (s.scale_mode != KVQ_SCALE_ABSMAX) return KVQ_ERR_INVALID_ARG;
      break;
    case KVQ_FMT_POLAR:
      if (s.bits < 1 || s.bits > 8 || s.bits2 < 1 || s.bits2 > 8) return KVQ_ERR_INVALID_ARG;
      if (s.scale_mode != KVQ_SCALE_ABSMAX || s.rotation != KVQ_ROT_NONE) return KVQ_ERR_INVALID_ARG;
      if (D != 128) return KVQ_ERR_UNSUPPORTED;
      return KVQ_OK;
    case KVQ_FMT_CART:
      if (s.bits < 2 || s.bits > 8) return KVQ_ERR_INVALID_ARG;
      if (s.scale_mode != KVQ_SCALE_ABSMAX || s.rotation != KVQ_ROT_NONE) return KVQ_ERR_INVALID_ARG;
      if (D != 128) return KVQ_ERR_UNSUPPORTED;
      return KVQ_OK;
    default:
      return KVQ_ERR_INVALID_ARG;
  }
  if (!is_pow2_group(s.group) || s.group > D) return KVQ_ERR_INVALID_ARG;
  if (!append_supported(D, s)) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

// The (layer, kv-head, side) formats of a cache: per-head arrays where given, else per-layer
// arrays, else cfg.k / cfg.v.
struct HeadSides {
  std::vector<kvq_side> k, v;  // [n_layers * n_kv_heads]
  const kvq_side& at(int side, int l, int h, int H) const { return (side ? v : k)[(size_t)l * H + h]; }
};

bool fill_sides(const kvq_config* c, const kvq_side* lk, const kvq_side* lv, const kvq_side* hk, const kvq_side* hv,
                HeadSides* out) {
  if (!c || c->n_layers < 1 || c->n_layers > 64 || c->n_kv_heads < 1 || c->n_kv_heads > 4096) return false;
  const int L = c->n_layers, H = c->n_kv_heads;
  out->k.resize((size_t)L * H);
  out->v.resize((size_t)L * H);
  for (int l = 0; l < L; ++l)
    for (int h = 0; h < H; ++h) {
      const size_t i = (size_t)l * H + h;
      out->k[i] = hk ? hk[i] : (lk ? lk[l] : c->k);
      out->v[i] = hv ? hv[i] : (lv ? lv[l] : c->v);
    }
  return true;
}

bool same_side(const kvq_side& a, const kvq_side& b) { return memcmp(&a, &b, sizeof(kvq_side)) == 0; }

kvq_status check_config(const kvq_config* c, const HeadSides& sides) {
  if (!c) return KVQ_ERR_INVALID_ARG;
  if (c->n_layers < 1 || c->n_layers > 64) return KVQ_ERR_INVALID_ARG;
  if (c->batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1) return KVQ_ERR_INVALID_ARG;
  if (c->n_q_heads % c->n_kv_heads) return KVQ_ERR_INVALID_ARG;
  if (c->n_q_heads / c->n_kv_heads > 8) return KVQ_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256) return KVQ_ERR_UNSUPPORTED;
  if (c->capacity < 1 || c->capacity > (1 << 26)) return KVQ_ERR_INVALID_ARG;
  if (c->max_queries < 1) return KVQ_ERR_INVALID_ARG;
  if (!(c->sm_scale >= 0.0f) || isinf(c->sm_scale)) return KVQ_ERR_INVALID_ARG;
  const int H = c->n_kv_heads;
  for (int sd = 0; sd < 2; ++sd)
    for (int l = 0; l < c->n_layers; ++l)
      for (int h = 0; h < H; ++h) {
        const kvq_status st = check_side(*c, sides.at(sd, l, h, H), sd == 0);
        if (st != KVQ_OK) return st;
      }
  if (c->anchor_rule < KVQ_ANCHOR_NONE || c->anchor_rule > KVQ_ANCHOR_ALL) return KVQ_ERR_INVALID_ARG;
  if (c->n_layers < 64 && (c->anchor_layer_mask >> c->n_layers)) return KVQ_ERR_INVALID_ARG;
  if (c->anchor_rule == KVQ_ANCHOR_FIRST_N || c->anchor_rule == KVQ_ANCHOR_WINDOW) {
    if (c->anchor_n < 1 || c->anchor_n > c->capacity) return KVQ_ERR_INVALID_ARG;
  }
  if (c->anchor_bits != 0 && c->anchor_bits != 16 && c->anchor_bits != 8 && c->anchor_bits != 4)
    return KVQ_ERR_INVALID_ARG;
  if (c->anchor_bits == 8 || c->anchor_bits == 4) {  // anchors are quantized by the row kernels
    for (int l = 0; l < c->n_layers; ++l) {
      if (c->anchor_rule == KVQ_ANCHOR_NONE || !((c->anchor_layer_mask >> l) & 1ULL)) continue;
      for (int sd = 0; sd < 2; ++sd)
        for (int h = 0; h < H; ++h) {
          const kvq_side& x = sides.at(sd, l, h, H);
          if (x.format == KVQ_FMT_FP16 || x.format == KVQ_FMT_POLAR || x.format == KVQ_FMT_CART ||
              x.format == KVQ_FMT_SORTED)
            return KVQ_ERR_UNSUPPORTED;
        }
    }
  }
  return KVQ_OK;
}

int anchor_bits_of(const kvq_config& c) { return (c.anchor_bits == 8 || c.anchor_bits == 4) ? c.anchor_bits : 16; }

int rank_bits(int D) { return 32 - __builtin_clz((unsigned)(D - 1)); }  // ceil(log2 D), D >= 2

bool has_zero_points(const kvq_side& s) {
  return (s.format == KVQ_FMT_INT && s.scale_mode == KVQ_SCALE_MINMAX) || s.format == KVQ_FMT_SORTED;
}

void side_geometry(int D, const kvq_side& s, int* row_bytes, int* n_groups) {
  switch (s.format) {
    case KVQ_FMT_FP16: *row_bytes = 2 * D; *n_groups = 0; return;
    case KVQ_FMT_INT:
    case KVQ_FMT_LLOYD: *row_bytes = D * s.bits / 8; *n_groups = D / s.group; return;
    case KVQ_FMT_SORTED: *row_bytes = D * (s.bits + rank_bits(D)) / 8; *n_groups = D / s.group; return;
    case KVQ_FMT_NF4: *row_bytes = D / 2; *n_groups = D / s.group; return;
    case KVQ_FMT_TERNARY: *row_bytes = (D + 4) / 5; *n_groups = D / s.group; return;
    case KVQ_FMT_SIGN: *row_bytes = D / 8; *n_groups = D / s.group; return;
    case KVQ_FMT_POLAR: *row_bytes = (D / 2) * (s.bits + s.bits2) / 8; *n_groups = 1; return;
    case KVQ_FMT_CART: *row_bytes = D * s.bits / 8; *n_groups = 1; return;
  }
  *row_bytes = 0;
  *n_groups = 0;
}

bool layer_anchored(const kvq_config& c, int l) {
  return c.anchor_rule != KVQ_ANCHOR_NONE && ((c.anchor_layer_mask >> l) & 1ULL);
}

// Lay out the arena; fills `h` (head groups and offsets) if non-null.  Returns total bytes.
uint64_t layout(const kvq_config& c, const HeadSides& sides, kvq_cache* h) {
  const int D = c.head_dim, H = c.n_kv_heads;
  const int Tcap = (c.capacity + 255) / 256 * 256;  // whole 256-token decode tiles
  const int anchor_rows = c.anchor_rule == KVQ_ANCHOR_ALL ? Tcap : c.anchor_n;
  uint64_t off = 0;
  for (int l = 0; l < c.n_layers; ++l) {
    std::vector<HeadGroup> groups;
    for (int hh = 0; hh < H;) {  // maximal runs of heads with equal (K, V) formats
      HeadGroup g{};
      g.h0 = hh;
      g.side[0] = sides.at(0, l, hh, H);
      g.side[1] = sides.at(1, l, hh, H);
      int e = hh + 1;
      while (e < H && same_side(sides.at(0, l, e, H), g.side[0]) && same_side(sides.at(1, l, e, H), g.side[1])) ++e;
      g.nh = e - hh;
      hh = e;
      const uint64_t units = (uint64_t)c.batch * g.nh;
      for (int s = 0; s < 2; ++s) {
        const kvq_side& sd = g.side[s];
        int rb, ng;
        side_geometry(D, sd, &rb, &ng);
        SideOff& so = g.off[s];
        so.row_bytes = rb;
        so.n_groups = ng;
        so.codes = (int64_t)off;
        off = align_up(off + units * Tcap * (uint64_t)rb);
        so.scales = -1;
        if (ng) {
          so.scales = (int64_t)off;
          off = align_up(off + units * Tcap * (uint64_t)ng * 2);
        }
        so.zeros = -1;
        if (has_zero_points(sd)) {
          so.zeros = (int64_t)off;
          off = align_up(off + units * Tcap * (uint64_t)ng * 2);
        }
        so.anchors = -1;
        so.anchor_scales = -1;
        if (layer_anchored(c, l)) {
          const int ab = anchor_bits_of(c);
          so.anchors = (int64_t)off;
          off = align_up(off + units * (uint64_t)anchor_rows * D * ab / 8);
          if (ab != 16) {
            so.anchor_scales = (int64_t)off;
            off = align_up(off + units * (uint64_t)anchor_rows * (D / 32) * 2);
          }
        }
      }
      g.kmean = -1;
      if (g.side[0].mean_sub) {
        g.kmean = (int64_t)off;
        off = align_up(off + units * D * 2);
      }
      groups.push_back(g);
    }
    bool any_chan = false;
    for (const HeadGroup& g : groups) any_chan |= g.side[0].chan_scale != 0;
    int64_t ch = -1;
    if (any_chan) {
      ch = (int64_t)off;
      off = align_up(off + (uint64_t)H * D * 2);
    }
    if (h) {
      h->grp[l] = groups;
      h->chan[l] = ch;
    }
  }
  const int64_t lens = (int64_t)off;
  off = align_up(off + (uint64_t)c.n_layers * c.batch * 4);
  const int64_t tickets = (int64_t)off;
  off = align_up(off + (uint64_t)c.n_layers * 4);
  const int64_t err = (int64_t)off;
  off = align_up(off + 4);
  if (h) {
    h->Tcap = Tcap;
    h->anchor_rows = anchor_rows;
    h->lens = lens;
    h->tickets = tickets;
    h->err = err;
  }
  return off;
}

// Device view of head group gi of layer l.
LayerDev layer_dev(const kvq_cache* h, int l, int gi) {
  LayerDev L{};
  const kvq_config& c = h->cfg;
  const HeadGroup& g = h->grp[l][gi];
  const int D = c.head_dim;
  for (int s = 0; s < 2; ++s) {
    const kvq_side& sd = g.side[s];
    const SideOff& so = g.off[s];
    SideDev& S = L.s[s];
    S.codes = reinterpret_cast<uint8_t*>(h->arena + so.codes);
    S.scales = so.scales >= 0 ? reinterpret_cast<__half*>(h->arena + so.scales) : nullptr;
    S.zeros = so.zeros >= 0 ? reinterpret_cast<__half*>(h->arena + so.zeros) : nullptr;
    S.anchors = so.anchors >= 0 ? reinterpret_cast<__half*>(h->arena + so.anchors) : nullptr;
    S.anchor_scales = so.anchor_scales >= 0 ? reinterpret_cast<__half*>(h->arena + so.anchor_scales) : nullptr;
    S.chan = (s == 0 && sd.chan_scale && h->chan[l] >= 0)
                 ? reinterpret_cast<const __half*>(h->arena + h->chan[l]) + (size_t)g.h0 * D
                 : nullptr;
    S.kmean = (s == 0 && g.kmean >= 0) ? reinterpret_cast<__half*>(h->arena + g.kmean) : nullptr;
    S.mean_sub = s == 0 ? sd.mean_sub : 0;
    S.fmt = sd.format;
    S.bits = sd.bits;
    S.bits2 = sd.bits2;
    S.scale_mode = sd.scale_mode;
    S.group = sd.group;
    S.rot = sd.rotation;
    S.chan_scale = s == 0 ? sd.chan_scale : 0;
    S.row_bytes = so.row_bytes;
    S.n_groups = so.n_groups;
  }
  const int G = c.n_q_heads / c.n_kv_heads;
  L.B = c.batch;
  L.cap = c.capacity;
  L.app_ids = nullptr;
  L.app_n = c.batch;
  L.div_new = fast_div(1u);
  L.test_stall = h->test_stall;
  L.Hkv = g.nh;
  L.div_hkv = fast_div((unsigned)L.Hkv);
  L.Hq = g.nh * G;
  L.Hkv_all = c.n_kv_heads;
  L.h0 = g.h0;
  L.D = D;
  L.Tcap = h->Tcap;
  L.anchored = layer_anchored(c, l) ? 1 : 0;
  L.anchor_rule = c.anchor_rule;
  L.anchor_n = c.anchor_n;
  L.anchor_rows = h->anchor_rows;
  L.anchor_bits = anchor_bits_of(c);
  L.anchor_rb = c.head_dim * L.anchor_bits / 8;
  L.seq_len = reinterpret_cast<int*>(h->arena + h->lens) + (size_t)l * c.batch;
  L.ticket = reinterpret_cast<unsigned*>(h->arena + h->tickets) + l;
  L.err = reinterpret_cast<unsigned*>(h->arena + h->err);
  L.sm_scale = c.sm_scale > 0.0f ? c.sm_scale : (float)(1.0 / sqrt((double)c.head_dim));
  return L;
}

bool layer_needs_chan(const kvq_cache* h, int l) {
  for (const HeadGroup& g : h->grp[l])
    if (g.side[0].chan_scale) return true;
  return false;
}

// ----------------------------------------------------------------------------- host tables
// Inverse of the standard normal CDF by bisection on Phi(x) = erfc(-x / sqrt 2) / 2.
double inv_norm_cdf(double p) {
  double lo = -40.0, hi = 40.0;
  for (int it = 0; it < 400; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    const double ph = 0.5 * erfc(-mid / sqrt(2.0));
    if (ph < p) lo = mid;
    else hi = mid;
  }
  return 0.5 * (lo + hi);
}

HostTables build_tables() {
  HostTables t{};
  // NF4 (NormalFloat) construction: 8 quantiles above zero, 7 below, exact 0, ends at +-1.
  const double delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
  double vals[16];
  int n = 0;
  const double step_p = (0.5 - delta) / 8.0, step_n = (0.5 - delta) / 7.0;
  for (int i = 0; i < 8; ++i) vals[n++] = inv_norm_cdf((double)i * step_p + delta);
  for (int i = 0; i < 7; ++i) vals[n++] = -inv_norm_cdf((double)i * step_n + delta);
  vals[n++] = 0.0;
  double mx = 0.0;
  for (int i = 0; i < 16; ++i) mx = fabs(vals[i]) > mx ? fabs(vals[i]) : mx;
  for (int i = 0; i < 16; ++i)
    for (int j = i + 1; j < 16; ++j)
      if (vals[j] < vals[i]) {
        const double tmp = vals[i];
        vals[i] = vals[j];
        vals[j] = tmp;
      }
  for (int i = 0; i < 16; ++i) t.nf4[i] = __half2float(__double2half(vals[i] / mx));
  for (int i = 0; i < 15; ++i) t.nf4_mid[i] = 0.5f * (t.nf4[i] + t.nf4[i + 1]);
  for (int k = 0; k < 64; ++k) {
    t.tw_re[k] = (float)cos(2.0 * M_PI * k / 128.0);
    t.tw_im[k] = (float)(-sin(2.0 * M_PI * k / 128.0));
  }
  // Gaussian Lloyd-Max levels: thresholds at midpoints, levels at the centroids of their cells
  // (standard normal: (phi(a) - phi(b)) / (Phi(b) - Phi(a))), alternated from evenly spaced levels
  // until they stop moving; stored at fp16 precision.
  for (int bi = 0; bi < 3; ++bi) {
    const int n = 4 << bi;
    double lv[16], nx[16];
    for (int k = 0; k < n; ++k) lv[k] = -2.0 + 4.0 * k / (n - 1);
    for (int it = 0; it < 200000; ++it) {
      double delta = 0.0;
      for (int k = 0; k < n; ++k) {
        const double a = k == 0 ? -INFINITY : 0.5 * (lv[k - 1] + lv[k]);
        const double b = k == n - 1 ? INFINITY : 0.5 * (lv[k] + lv[k + 1]);
        const double pa = isinf(a) ? 0.0 : exp(-0.5 * a * a) / sqrt(2.0 * M_PI);
        const double pb = isinf(b) ? 0.0 : exp(-0.5 * b * b) / sqrt(2.0 * M_PI);
        const double Pa = isinf(a) ? 0.0 : 0.5 * erfc(-a / sqrt(2.0));
        const double Pb = isinf(b) ? 1.0 : 0.5 * erfc(-b / sqrt(2.0));
        nx[k] = (pa - pb) / (Pb - Pa);
        delta = fmax(delta, fabs(nx[k] - lv[k]));
      }
      for (int k = 0; k < n; ++k) lv[k] = nx[k];
      if (delta < 1e-12) break;
    }
    for (int k = 0; k < n; ++k) t.lloyd[bi][k] = __half2float(__double2half(lv[k]));
    for (int k = 0; k + 1 < n; ++k) t.lloyd_mid[bi][k] = 0.5f * (t.lloyd[bi][k] + t.lloyd[bi][k + 1]);
  }
  for (int bp = 1; bp <= 8; ++bp) {
    const int nb = 1 << bp;
    for (int k = 0; k < nb; ++k) {
      const double phi = -M_PI + 2.0 * M_PI * k / (double)nb;
      t.ph_cos[nb - 2 + k] = (float)cos(phi);
      t.ph_sin[nb - 2 + k] = (float)sin(phi);
    }
  }
  return t;
}

std::mutex g_mu;
std::set<int> g_ready_devices;

cudaError_t ensure_tables(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_ready_devices.count(dev)) return cudaSuccess;
  const HostTables& t = host_tables();
  cudaError_t e = upload_tables_quant(t);
  if (e == cudaSuccess) e = upload_tables_decode(t);
  if (e == cudaSuccess) e = upload_tables_dequant(t);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) g_ready_devices.insert(dev);
  return e;
}

}  // namespace

namespace kvq {
const HostTables& host_tables() {
  static const HostTables t = build_tables();
  return t;
}
}  // namespace kvq

extern "C" {

const char* kvq_status_str(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "capacity exceeded";
    case KVQ_ERR_CUDA: return "CUDA error";
    case KVQ_ERR_ALLOC: return "allocation failed or arena too small";
    case KVQ_ERR_STATE: return "invalid call order";
  }
  return "unknown status";
}

kvq_status kvq_nf4_levels(float out[16]) {
  if (!out) return KVQ_ERR_INVALID_ARG;
  memcpy(out, host_tables().nf4, sizeof(float) * 16);
  return KVQ_OK;
}

kvq_status kvq_lloyd_levels(int32_t bits, float* out) {
  if (!out || bits < 2 || bits > 4) return KVQ_ERR_INVALID_ARG;
  memcpy(out, host_tables().lloyd[bits - 2], sizeof(float) << bits);
  return KVQ_OK;
}

kvq_status kvq_arena_bytes_heads(const kvq_config* cfg, const kvq_side* head_k, const kvq_side* head_v,
                                 uint64_t* bytes) {
  if (!bytes) return KVQ_ERR_INVALID_ARG;
  HeadSides sides;
  if (!fill_sides(cfg, nullptr, nullptr, head_k, head_v, &sides)) return KVQ_ERR_INVALID_ARG;
  const kvq_status st = check_config(cfg, sides);
  if (st != KVQ_OK) return st;
  *bytes = layout(*cfg, sides, nullptr);
  return KVQ_OK;
}

kvq_status kvq_arena_bytes_layers(const kvq_config* cfg, const kvq_side* layer_k, const kvq_side* layer_v,
                                  uint64_t* bytes) {
  if (!bytes) return KVQ_ERR_INVALID_ARG;
  HeadSides sides;
  if (!fill_sides(cfg, layer_k, layer_v, nullptr, nullptr, &sides)) return KVQ_ERR_INVALID_ARG;
  const kvq_status st = check_config(cfg, sides);
  if (st != KVQ_OK) return st;
  *bytes = layout(*cfg, sides, nullptr);
  return KVQ_OK;
}

kvq_status kvq_arena_bytes(const kvq_config* cfg, uint64_t* bytes) {
  return kvq_arena_bytes_layers(cfg, nullptr, nullptr, bytes);
}

static kvq_status create_impl(const kvq_config* cfg, const HeadSides& sides, void* arena, uint64_t arena_bytes,
                              kvq_cache** out) {
  kvq_status st = check_config(cfg, sides);
  if (st != KVQ_OK) return st;
  if (!arena || (reinterpret_cast<uintptr_t>(arena) % kAlign)) return KVQ_ERR_INVALID_ARG;
  const uint64_t need = layout(*cfg, sides, nullptr);
  if (arena_bytes < need) return KVQ_ERR_ALLOC;
  kvq_cache* h = new (std::nothrow) kvq_cache();
  if (!h) return KVQ_ERR_ALLOC;
  h->cfg = *cfg;
  h->arena = reinterpret_cast<char*>(arena);
  h->arena_bytes = arena_bytes;
  layout(*cfg, sides, h);
  for (int l = 0; l < 64; ++l) {
    h->max_len[l] = 0;
    h->len_exact[l] = true;
    h->chan_set[l] = false;
  }
  // Test hook: with KVQ_TEST_STALL_FIRST_WAIT=<cycles> set when the handle is created, the first
  // staged-tile wait of every tensor-core decode CTA polls a barrier that nothing arrives on, for
  // that many clock cycles, then takes the give-up path (KVQ_ERRF_WAIT_TIMEOUT, empty partial,
  // copies already issued drained).  Unset or 0: off.
  h->test_stall = 0;
  if (const char* w = getenv("KVQ_TEST_STALL_FIRST_WAIT")) {
    char* end = nullptr;
    const long long v = strtoll(w, &end, 10);
    if (end != w && v > 0 && v <= 2000000000LL) h->test_stall = v;
  }
  if (cudaGetDevice(&h->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
    delete h;
    return KVQ_ERR_CUDA;
  }
  if (ensure_tables(h->device) != cudaSuccess) {
    delete h;
    return KVQ_ERR_CUDA;
  }
  // workspace for the largest split-K grid any head group and any n_q <= max_queries can use
  size_t wf = 0;
  for (int l = 0; l < cfg->n_layers; ++l)
    for (int gi = 0; gi < (int)h->grp[l].size(); ++gi) {
      const LayerDev L = layer_dev(h, l, gi);
      for (int nq = 1; nq <= cfg->max_queries; ++nq) {
        const size_t f = (size_t)nq * L.Hq * decode_partials(L, nq, h->num_sms) * (cfg->head_dim + kPartStride);
        wf = f > wf ? f : wf;
      }
    }
  h->work_floats = wf;
  if (cudaMalloc(&h->work, wf * sizeof(float)) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return KVQ_ERR_ALLOC;
  }
  // zero lengths, tickets and the error word
  if (cudaMemset(h->arena + h->lens, 0, (size_t)(need - (uint64_t)h->lens)) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(h->work);
    delete h;
    return KVQ_ERR_CUDA;
  }
  *out = h;
  return KVQ_OK;
}

kvq_status kvq_create_heads(const kvq_config* cfg, const kvq_side* head_k, const kvq_side* head_v, void* arena,
                            uint64_t arena_bytes, kvq_cache** out) {
  if (!out) return KVQ_ERR_INVALID_ARG;
  *out = nullptr;
  HeadSides sides;
  if (!fill_sides(cfg, nullptr, nullptr, head_k, head_v, &sides)) return KVQ_ERR_INVALID_ARG;
  return create_impl(cfg, sides, arena, arena_bytes, out);
}

kvq_status kvq_create_layers(const kvq_config* cfg, const kvq_side* layer_k, const kvq_side* layer_v, void* arena,
                             uint64_t arena_bytes, kvq_cache** out) {
  if (!out) return KVQ_ERR_INVALID_ARG;
  *out = nullptr;
  HeadSides sides;
  if (!fill_sides(cfg, layer_k, layer_v, nullptr, nullptr, &sides)) return KVQ_ERR_INVALID_ARG;
  return create_impl(cfg, sides, arena, arena_bytes, out);
}

kvq_status kvq_create(const kvq_config* cfg, void* arena, uint64_t arena_bytes, kvq_cache** out) {
  return kvq_create_layers(cfg, nullptr, nullptr, arena, arena_bytes, out);
}

void kvq_free(kvq_cache* h) {
  if (!h) return;
  if (h->work) cudaFree(h->work);
  delete h;
}

kvq_status kvq_get_layout_head(const kvq_cache* h, int32_t layer, int32_t side, int32_t head, kvq_layout* out) {
  if (!h || !out || layer < 0 || layer >= h->cfg.n_layers || (side != 0 && side != 1) || head < 0 ||
      head >= h->cfg.n_kv_heads)
    return KVQ_ERR_INVALID_ARG;
  const HeadGroup* g = nullptr;
  for (const HeadGroup& x : h->grp[layer])
    if (head >= x.h0 && head < x.h0 + x.nh) g = &x;
  const SideOff& so = g->off[side];
  out->codes = so.codes;
  out->scales = so.scales;
  out->zeros = so.zeros;
  out->anchors = so.anchors;
  out->chan_scale = side == 0 ? h->chan[layer] : -1;
  out->seq_len = h->lens + (int64_t)layer * h->cfg.batch * 4;
  out->key_mean = side == 0 ? g->kmean : -1;
  out->anchor_scales = so.anchor_scales;
  out->row_bytes = so.row_bytes;
  out->n_groups = so.n_groups;
  out->row_stride_tokens = h->Tcap;
  out->anchor_rows = so.anchors >= 0 ? h->anchor_rows : 0;
  out->head0 = g->h0;
  out->n_heads = g->nh;
  return KVQ_OK;
}

kvq_status kvq_get_layout(const kvq_cache* h, int32_t layer, int32_t side, kvq_layout* out) {
  return kvq_get_layout_head(h, layer, side, 0, out);
}

kvq_status kvq_set_chan_scale(kvq_cache* h, int32_t layer, const void* c, void* stream) {
  if (!h || !c || layer < 0 || layer >= h->cfg.n_layers) return KVQ_ERR_INVALID_ARG;
  if (h->chan[layer] < 0) return KVQ_ERR_STATE;
  const size_t bytes = (size_t)h->cfg.n_kv_heads * h->cfg.head_dim * 2;
  if (cudaMemcpyAsync(h->arena + h->chan[layer], c, bytes, cudaMemcpyDeviceToDevice,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KVQ_ERR_CUDA;
  h->chan_set[layer] = true;
  return KVQ_OK;
}

kvq_status kvq_set_seq_len(kvq_cache* h, int32_t layer, int32_t len, void* stream) {
  if (!h || layer < -1 || layer >= h->cfg.n_layers || len < 0 || len > h->cfg.capacity) return KVQ_ERR_INVALID_ARG;
  int* lens = reinterpret_cast<int*>(h->arena + h->lens);
  const int B = h->cfg.batch;
  cudaError_t e;
  if (layer < 0) {
    e = launch_fill_len(lens, B * h->cfg.n_layers, len, reinterpret_cast<cudaStream_t>(stream));
    for (int l = 0; l < h->cfg.n_layers; ++l) {
      h->max_len[l] = len;
      h->len_exact[l] = true;
    }
  } else {
    e = launch_fill_len(lens + (size_t)layer * B, B, len, reinterpret_cast<cudaStream_t>(stream));
    h->max_len[layer] = len;
    h->len_exact[layer] = true;
  }
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_quantize_append(kvq_cache* h, int32_t layer, const void* k, const void* v, const int32_t* seq_ids,
                               int32_t n_seqs, int32_t n_new, void* stream) {
  if (!h || !k || !v || layer < 0 || layer >= h->cfg.n_layers || n_new < 1) return KVQ_ERR_INVALID_ARG;
  if (seq_ids ? (n_seqs < 1 || n_seqs > h->cfg.batch) : n_seqs != h->cfg.batch) return KVQ_ERR_INVALID_ARG;
  if (layer_needs_chan(h, layer) && !h->chan_set[layer]) return KVQ_ERR_STATE;
  if ((uintptr_t)k % 16 || (uintptr_t)v % 16) return KVQ_ERR_INVALID_ARG;
  if (n_new > h->cfg.capacity) return KVQ_ERR_CAPACITY;
  // every sequence advances together: the host bound is exact and decides; otherwise the device
  // checks each listed sequence
  if (!seq_ids && h->len_exact[layer] && (int64_t)h->max_len[layer] + n_new > h->cfg.capacity) return KVQ_ERR_CAPACITY;
  if ((int64_t)n_seqs * h->cfg.n_kv_heads * n_new >= (int64_t)1 << 31) return KVQ_ERR_INVALID_ARG;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int ng = (int)h->grp[layer].size();
  std::vector<LayerDev> views(ng);
  unsigned total = 0;  // every view's CTAs take a ticket; the last one advances the lengths
  for (int gi = 0; gi < ng; ++gi) {
    views[gi] = layer_dev(h, layer, gi);
    views[gi].app_ids = seq_ids;
    views[gi].app_n = n_seqs;
    views[gi].div_new = fast_div((unsigned)n_new);
    total += append_ctas(views[gi], n_new);
  }
  int launches = 0;
  cudaError_t e = cudaSuccess;
  for (int gi = 0; gi < ng && e == cudaSuccess; ++gi) {
    const LayerDev& L = views[gi];
    if (L.s[0].mean_sub) {  // key means of the sequences this append starts, before their rows
      e = launch_key_mean(L, reinterpret_cast<const __half*>(k), n_new, st);
      ++launches;
    }
    if (e == cudaSuccess) {
      int n = 0;
      e = launch_append(L, reinterpret_cast<const __half*>(k), reinterpret_cast<const __half*>(v), n_new, total, st, &n);
      launches += n;
    }
  }
  h->last_launches = launches;
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  const int64_t nl = (int64_t)h->max_len[layer] + n_new;
  h->max_len[layer] = (int)(nl < h->cfg.capacity ? nl : h->cfg.capacity);
  if (seq_ids) h->len_exact[layer] = false;
  return KVQ_OK;
}

kvq_status kvq_dequantize(const kvq_cache* h, int32_t layer, int32_t side, int32_t domain, int32_t t0, int32_t nt,
                          void* out, int32_t out_fp32, void* stream) {
  if (!h || !out || layer < 0 || layer >= h->cfg.n_layers || (side != 0 && side != 1)) return KVQ_ERR_INVALID_ARG;
  if (domain != KVQ_DOMAIN_STORED && domain != KVQ_DOMAIN_ORIGINAL) return KVQ_ERR_INVALID_ARG;
  if (t0 < 0 || nt < 1 || (int64_t)t0 + nt > h->cfg.capacity) return KVQ_ERR_INVALID_ARG;
  for (int gi = 0; gi < (int)h->grp[layer].size(); ++gi) {
    const LayerDev L = layer_dev(h, layer, gi);
    const cudaError_t e =
        launch_dequant(L, side, domain, t0, nt, out, out_fp32 ? 1 : 0, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return KVQ_ERR_CUDA;
  }
  return KVQ_OK;
}

// Decode every head group of `layer` with `work` as the split-K scratch (the groups run one after
// another on the stream, so they share it).
static kvq_status decode_groups(kvq_cache* h, int32_t layer, const void* q, int32_t n_q, const int32_t* seq_ids,
                                const int32_t* kv_len, void* out, int32_t out_fp32, float* lse, float* work,
                                void* stream) {
  int launches = 0;
  for (int gi = 0; gi < (int)h->grp[layer].size(); ++gi) {
    const LayerDev L = layer_dev(h, layer, gi);
    int n = 0;
    const cudaError_t e = launch_decode(L, reinterpret_cast<const __half*>(q), n_q, seq_ids, kv_len, out,
                                        out_fp32 ? 1 : 0, lse, work, h->num_sms, h->cfg.max_queries,
                                        reinterpret_cast<cudaStream_t>(stream), &n);
    launches += n;
    if (e != cudaSuccess) {
      h->last_launches = launches;
      return KVQ_ERR_CUDA;
    }
  }
  h->last_launches = launches;
  return KVQ_OK;
}

kvq_status kvq_decode_attention(kvq_cache* h, int32_t layer, const void* q, int32_t n_q, const int32_t* seq_ids,
                                const int32_t* kv_len, void* out, int32_t out_fp32, float* lse, void* stream) {
  if (!h || !q || !out || layer < 0 || layer >= h->cfg.n_layers || n_q < 1) return KVQ_ERR_INVALID_ARG;
  if (n_q > h->cfg.max_queries) return KVQ_ERR_CAPACITY;
  if (!seq_ids && n_q > h->cfg.batch) return KVQ_ERR_INVALID_ARG;
  return decode_groups(h, layer, q, n_q, seq_ids, kv_len, out, out_fp32, lse, h->work, stream);
}

// Same computation as kvq_decode_attention; the split-K partials go to the library's fixed
// device scratch instead of the handle's workspace, and nothing is allocated.
kvq_status kvq_decode_attention_noalloc(kvq_cache* h, int32_t layer, const void* q, int32_t n_q,
                                        const int32_t* seq_ids, const int32_t* kv_len, void* out, int32_t out_fp32,
                                        float* lse, void* stream) {
  if (!h || !q || !out || layer < 0 || layer >= h->cfg.n_layers || n_q < 1) return KVQ_ERR_INVALID_ARG;
  if (n_q > h->cfg.max_queries) return KVQ_ERR_CAPACITY;
  if (!seq_ids && n_q > h->cfg.batch) return KVQ_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
  if (dev != h->device) return KVQ_ERR_INVALID_ARG;
  size_t need = 0;
  for (int gi = 0; gi < (int)h->grp[layer].size(); ++gi) {
    const LayerDev L = layer_dev(h, layer, gi);
    const size_t f = (size_t)n_q * L.Hq * decode_partials(L, n_q, h->num_sms) * (h->cfg.head_dim + kPartStride);
    need = f > need ? f : need;
  }
  if (need > static_work_floats()) return KVQ_ERR_CAPACITY;
  float* ws = nullptr;
  if (static_work_ptr(dev, &ws) != cudaSuccess) return KVQ_ERR_CUDA;
  return decode_groups(h, layer, q, n_q, seq_ids, kv_len, out, out_fp32, lse, ws, stream);
}

// Append then decode in one split-K launch (plus the merge) where the layer allows it; otherwise
// the two calls in turn.  Query i belongs to listed sequence i and attends its whole new length.
kvq_status kvq_append_decode(kvq_cache* h, int32_t layer, const void* k, const void* v, const int32_t* seq_ids,
                             int32_t n_seqs, int32_t n_new, const void* q, void* out, int32_t out_fp32, float* lse,
                             void* stream) {
  if (!h || !k || !v || !q || !out || layer < 0 || layer >= h->cfg.n_layers || n_new < 1) return KVQ_ERR_INVALID_ARG;
  if (seq_ids ? (n_seqs < 1 || n_seqs > h->cfg.batch) : n_seqs != h->cfg.batch) return KVQ_ERR_INVALID_ARG;
  if (n_seqs > h->cfg.max_queries) return KVQ_ERR_CAPACITY;
  if (layer_needs_chan(h, layer) && !h->chan_set[layer]) return KVQ_ERR_STATE;
  if ((uintptr_t)k % 16 || (uintptr_t)v % 16) return KVQ_ERR_INVALID_ARG;
  if (n_new > h->cfg.capacity) return KVQ_ERR_CAPACITY;
  if (!seq_ids && h->len_exact[layer] && (int64_t)h->max_len[layer] + n_new > h->cfg.capacity) return KVQ_ERR_CAPACITY;
  if ((int64_t)n_seqs * h->cfg.n_kv_heads * n_new >= (int64_t)1 << 31) return KVQ_ERR_INVALID_ARG;
  LayerDev L = layer_dev(h, layer, 0);
  if (h->grp[layer].size() != 1 || !fused_decode_ok(L, n_seqs, h->num_sms)) {
    kvq_status s = kvq_quantize_append(h, layer, k, v, seq_ids, n_seqs, n_new, stream);
    if (s != KVQ_OK) return s;
    const int na = h->last_launches;
    s = decode_groups(h, layer, q, n_seqs, seq_ids, nullptr, out, out_fp32, lse, h->work, stream);
    h->last_launches += na;
    return s;
  }
  L.fuse_k = reinterpret_cast<const __half*>(k);
  L.fuse_v = reinterpret_cast<const __half*>(v);
  L.fuse_n = n_new;
  int n = 0;
  const cudaError_t e = launch_decode(L, reinterpret_cast<const __half*>(q), n_seqs, seq_ids, nullptr, out,
                                      out_fp32 ? 1 : 0, lse, h->work, h->num_sms, h->cfg.max_queries,
                                      reinterpret_cast<cudaStream_t>(stream), &n);
  h->last_launches = n;
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  const int64_t nl = (int64_t)h->max_len[layer] + n_new;
  h->max_len[layer] = (int)(nl < h->cfg.capacity ? nl : h->cfg.capacity);
  if (seq_ids) h->len_exact[layer] = false;
  return KVQ_OK;
}

kvq_status kvq_error_flags(kvq_cache* h, int32_t* flags) {
  if (!h || !flags) return KVQ_ERR_INVALID_ARG;
  unsigned v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return KVQ_ERR_CUDA;
  if (cudaMemcpy(&v, h->arena + h->err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return KVQ_ERR_CUDA;
  if (cudaMemset(h->arena + h->err, 0, 4) != cudaSuccess) return KVQ_ERR_CUDA;
  *flags = (int32_t)v;
  return KVQ_OK;
}

int32_t kvq_last_launch_count(const kvq_cache* h) { return h ? h->last_launches : 0; }

}  // extern "C"
