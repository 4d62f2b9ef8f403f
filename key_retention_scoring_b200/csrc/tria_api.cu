// Host entry points of the C ABI declared in include/tria.h.
//
// Load time (tria_load_stats) folds the future-offset average into the query
// centers, in fp64 on the host: W_f = (1/|D|) sum_{delta in D} e^{i omega_f delta}
// (academ.us article 2607.13051, Eq. 6) and mu'_f = E[q_f] W_f (Eq. 7); the
// norm-term weight is w_f = E|q_f| - |E q_f| = (1 - R_f) E|q_f| (ghidav.me,
// "TriAttention, or: what a rotating query already knows", "The Method").
// Every other entry point validates its arguments on the host and enqueues
// kernels on the caller's stream; none allocates device memory.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <vector>

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cuda_runtime.h>

#include "tria_internal.h"

struct tria_stats {
  tria::StatsDev dev;
};

namespace tria {
namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tria_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TRIA_OK : TRIA_ERR_CUDA; }

// Validate the arguments shared by the per-pass entry points and derive the
// call geometry.
tria_status make_geom(const tria_stats *stats, const tria_cache_view *cache,
                      const tria_params *params, int layer0, int layer1, Geom *geo) {
  if (stats == nullptr || cache == nullptr || params == nullptr || geo == nullptr)
    return TRIA_ERR_INVALID_ARG;
  const tria_model_desc &d = stats->dev.desc;
  if (layer0 < 0 || layer1 <= layer0 || layer1 > d.n_layers) return TRIA_ERR_INVALID_ARG;
  if (cache->n_seq < 1 || cache->n_seq > TRIA_MAX_SEQS) return TRIA_ERR_INVALID_ARG;
  if (cache->max_seq_len < 1) return TRIA_ERR_INVALID_ARG;
  if (params->window < 0 || params->sinks < 0 || params->interval < 0 || params->wait_limit_ns < 0)
    return TRIA_ERR_INVALID_ARG;
  const double pct = params->budget_pct;  // the fp32 value, exactly
  if (!std::isfinite(pct) || pct < 0.0 || pct > 100.0) return TRIA_ERR_INVALID_ARG;
  if (cache->layout != TRIA_LAYOUT_CONTIGUOUS && cache->layout != TRIA_LAYOUT_PAGED)
    return TRIA_ERR_INVALID_ARG;
  const bool layer_lens = cache->layer_seq_lens != nullptr;
  if (cache->k_layers == nullptr || cache->query_pos == nullptr ||
      (!layer_lens && cache->seq_lens == nullptr))
    return TRIA_ERR_INVALID_ARG;
  for (int l = layer0; l < layer1; ++l)
    if (cache->k_layers[l] == nullptr || !aligned16(cache->k_layers[l])) return TRIA_ERR_INVALID_ARG;
  if (cache->stride_head < 0 || cache->stride_token <= 0 || cache->stride_seq < 0 ||
      cache->stride_block < 0)
    return TRIA_ERR_INVALID_ARG;
  if ((cache->stride_head % 8) || (cache->stride_token % 8) || (cache->stride_seq % 8) ||
      (cache->stride_block % 8))
    return TRIA_ERR_INVALID_ARG;
  if (cache->layout == TRIA_LAYOUT_PAGED) {
    const int bs = cache->block_size;
    if (cache->block_table == nullptr || cache->max_blocks_per_seq < 1 || cache->num_blocks < 1 ||
        !(bs == 8 || bs == 16 || bs == 32 || bs == 64 || bs == 128))
      return TRIA_ERR_INVALID_ARG;
    if ((int64_t)cache->max_blocks_per_seq * cache->block_size < cache->max_seq_len)
      return TRIA_ERR_INVALID_ARG;
  }
  if (cache->positions != nullptr && (reinterpret_cast<uintptr_t>(cache->positions) & 3u))
    return TRIA_ERR_INVALID_ARG;
  Geom g{};
  g.n_seq = cache->n_seq;
  g.nl = layer1 - layer0;
  g.layer0 = layer0;
  g.n_layers = d.n_layers;
  g.hkv = d.n_kv_heads;
  g.hq = d.n_q_heads;
  g.g = d.n_q_heads / d.n_kv_heads;
  // budget of every layer: base = the absolute budget, or pct % of the
  // capacity; B_l = round-half-up(base * scale_l); B_max sizes the kept rows
  const double base = pct > 0.0 ? std::floor(pct * (double)cache->max_seq_len / 100.0)
                                 : (double)params->budget;
  int bmax = 0, b_first = 0;
  bool uniform = true;
  for (int l = 0; l < d.n_layers; ++l) {
    double sc = 1.0;
    if (params->layer_budget_scales != nullptr) {
      sc = params->layer_budget_scales[l];
      if (!std::isfinite(sc) || !(sc > 0.0)) return TRIA_ERR_INVALID_ARG;
    }
    const double b = std::floor(base * sc + 0.5);
    if (!(b >= 1.0) || b > (double)(INT32_MAX / 4)) return TRIA_ERR_INVALID_ARG;
    const int bl = (int)b;
    if (bl < params->window + params->sinks) return TRIA_ERR_INVALID_ARG;
    if (l == 0) b_first = bl;
    uniform = uniform && bl == b_first;
    bmax = bl > bmax ? bl : bmax;
    if (l >= layer0 && l < layer1) g.lbudget[l - layer0] = bl;
  }
  // one length per sequence cannot describe layers kept at different budgets
  if (!uniform && !layer_lens) return TRIA_ERR_INVALID_ARG;
  g.budget = bmax;
  g.trigger = params->interval > 1 ? params->interval : 1;
  g.per_layer = layer_lens ? 1 : 0;
  if (layer_lens) {
    g.lens = cache->layer_seq_lens + layer0;
    g.lens_s = d.n_layers;
    g.lens_l = 1;
  } else {
    g.lens = cache->seq_lens;
    g.lens_s = 1;
    g.lens_l = 0;
  }
  g.window = params->window;
  g.sinks = params->sinks;
  g.max_seq_len = cache->max_seq_len;
  const int cm = cache->max_seq_len - params->window - params->sinks;
  g.c_max = cm > 1 ? cm : 1;
  // scheduling tiles are aligned to kTileKeys slots and cover [sinks, N - window)
  const int hi = cache->max_seq_len - params->window - 1;
  g.tiles_max = hi >= params->sinks ? hi / kTileKeys - params->sinks / kTileKeys + 1 : 1;
  g.pairing = d.pairing;
  g.ncol = (2 * g.g < 16) ? 16 : 2 * g.g;
  g.n_units = (int64_t)g.n_seq * g.nl * g.hkv;
  g.mode = params->offset_reduce;
  if (g.mode != TRIA_OFFSET_MEAN && g.mode != TRIA_OFFSET_MAX) return TRIA_ERR_INVALID_ARG;
  g.n_off = d.offset_log2_max + 1;
  g.ncol_t = ((g.n_off * g.g + 15) / 16) * 16;
  g.ncol_n = g.ncol;
  if (g.mode == TRIA_OFFSET_MAX) {
    // the max-over-offsets kernel is built for G <= 8
    if (g.g > 8 || g.n_off > kMaxOffsets || 2 * g.n_off * g.g > kMaxOffCols) return TRIA_ERR_UNSUPPORTED;
    // trig hi and lo parts (two 64-wide K blocks of 128-byte rows each), norm
    g.b_bytes = (2 * g.ncol_t + g.ncol_n) * 256;
  } else {
    g.b_bytes = g.ncol * kCoefK * 2;
  }
  if (g.n_units * (int64_t)g.tiles_max > INT32_MAX) return TRIA_ERR_UNSUPPORTED;
  // paged offset-mean scoring reads whole blocks when one block of every KV
  // head is a 128-row tile; the heads' 2G coefficient columns each, side by
  // side, are the MMA's N (16 <= N <= 128)
  g.grouped = (cache->layout == TRIA_LAYOUT_PAGED && g.mode == TRIA_OFFSET_MEAN &&
               (g.hkv == 2 || g.hkv == 4 || g.hkv == 8) && cache->block_size * g.hkv == 128 &&
               g.g <= 8 && g.hkv * 2 * g.g >= 16) ? 1 : 0;
  *geo = g;
  return TRIA_OK;
}

// ---------------------------------------------------------------------------
// TMA tensor maps of the K cache (encoded on the host, cached by pointer and
// geometry; entries are 128 bytes).
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

struct MapKey {
  const void *ptr;
  int layout;
  uint64_t dims[4];
  uint64_t strides[3];
  uint32_t box[4];
  bool operator<(const MapKey &o) const { return std::memcmp(this, &o, sizeof(MapKey)) < 0; }
};

tria_status k_tensor_map(const tria_cache_view *c, int hkv, bool all_heads, const void *base,
                        CUtensorMap *out) {
  MapKey key;
  std::memset(&key, 0, sizeof(key));
  key.ptr = base;
  key.layout = c->layout;
  if (c->layout == TRIA_LAYOUT_CONTIGUOUS) {
    // [n_seq][hkv][max_seq_len][128] by strides; box = 128 rows x 64 dims
    key.dims[0] = 128;
    key.dims[1] = (uint64_t)c->max_seq_len;
    key.dims[2] = (uint64_t)hkv;
    key.dims[3] = (uint64_t)c->n_seq;
    key.strides[0] = (uint64_t)c->stride_token * 2;
    key.strides[1] = (uint64_t)c->stride_head * 2;
    key.strides[2] = (uint64_t)c->stride_seq * 2;
    key.box[0] = 64; key.box[1] = 128; key.box[2] = 1; key.box[3] = 1;
  } else if (all_heads) {
    // [num_blocks][block_size][hkv][128] by strides, dimensions ordered (dim,
    // token, head, block): box = one block of every head x 64 dims, rows
    // head-major (head block_size + token)
    key.dims[0] = 128;
    key.dims[1] = (uint64_t)c->block_size;
    key.dims[2] = (uint64_t)hkv;
    key.dims[3] = (uint64_t)c->num_blocks;
    key.strides[0] = (uint64_t)c->stride_token * 2;
    key.strides[1] = (uint64_t)c->stride_head * 2;
    key.strides[2] = (uint64_t)c->stride_block * 2;
    key.box[0] = 64; key.box[1] = (uint32_t)c->block_size; key.box[2] = (uint32_t)hkv; key.box[3] = 1;
  } else {
    // [num_blocks][block_size][hkv][128] by strides; box = one block of one
    // head x 64 dims
    key.dims[0] = 128;
    key.dims[1] = (uint64_t)hkv;
    key.dims[2] = (uint64_t)c->block_size;
    key.dims[3] = (uint64_t)c->num_blocks;
    key.strides[0] = (uint64_t)c->stride_head * 2;
    key.strides[1] = (uint64_t)c->stride_token * 2;
    key.strides[2] = (uint64_t)c->stride_block * 2;
    key.box[0] = 64; key.box[1] = 1; key.box[2] = (uint32_t)c->block_size; key.box[3] = 1;
  }
  // a dimension of extent 1 never advances: give it a stride the encoder accepts
  for (int i = 0; i < 3; ++i)
    if (key.dims[i + 1] == 1 && key.strides[i] == 0)
      key.strides[i] = (i == 0 ? 256 : key.strides[i - 1] * key.dims[i]);
  static std::mutex mu;
  static std::map<MapKey, CUtensorMap> cache;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *out = it->second;
    return TRIA_OK;
  }
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return TRIA_ERR_CUDA;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUtensorMap m;
  const CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base),
                         key.dims, key.strides, key.box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return TRIA_ERR_UNSUPPORTED;
  if (cache.size() > 4096) cache.clear();
  cache.emplace(key, m);
  *out = m;
  return TRIA_OK;
}

CacheDev make_cache_dev(const tria_cache_view *c, int layer0, int layer1) {
  CacheDev cd{};
  cd.layout = c->layout;
  cd.block_size = c->layout == TRIA_LAYOUT_PAGED ? c->block_size : 1;
  cd.max_blocks = c->layout == TRIA_LAYOUT_PAGED ? c->max_blocks_per_seq : 0;
  cd.s_seq = c->stride_seq;
  cd.s_head = c->stride_head;
  cd.s_tok = c->stride_token;
  cd.s_blk = c->stride_block;
  cd.block_table = c->block_table;
  cd.seq_lens = c->seq_lens;
  cd.query_pos = c->query_pos;
  cd.positions = c->positions;
  cd.pos_unit_stride = c->max_seq_len;
  for (int l = layer0; l < layer1; ++l) {
    cd.k[l - layer0] = static_cast<const uint16_t *>(c->k_layers[l]);
    cd.v[l - layer0] = c->v_layers ? static_cast<uint16_t *>(c->v_layers[l]) : nullptr;
  }
  return cd;
}

tria_status check_workspace(const Geom &g, void *ws, size_t bytes, WsLayout *wl) {
  *wl = ws_layout(g);
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return TRIA_ERR_WORKSPACE;
  if (bytes < wl->total) return TRIA_ERR_WORKSPACE;
  return TRIA_OK;
}

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<unsigned char *>(ws) + off);
}

CoefParams make_coef(const tria_stats *st, const Geom &g, const tria_cache_view *c, void *ws,
                     const WsLayout &wl, int32_t *kept, bool with_hist) {
  CoefParams cp{};
  cp.geo = g;
  cp.mu_fold = st->dev.mu_fold;
  cp.mu_raw = st->dev.mu_raw;
  cp.w_norm = st->dev.w_norm;
  cp.omega = st->dev.omega;
  cp.rot_off = st->dev.rot_off;
  cp.query_pos = c->query_pos;
  cp.btile = at<uint16_t>(ws, wl.btile);
  cp.item_counter = at<uint32_t>(ws, wl.hdr);
  cp.status = at<int32_t>(ws, wl.hdr + 4);
  cp.unit_done = at<uint32_t>(ws, wl.unit_done);
  cp.seq_items = at<int32_t>(ws, wl.seq_items);
  cp.row_items = at<int32_t>(ws, wl.row_items);
  cp.kept = kept;
  cp.hist = with_hist ? at<uint32_t>(ws, wl.hist) : nullptr;
  return cp;
}

tria_status make_score(const Geom &g, const tria_cache_view *c, const tria_params *prm, int layer0,
                       int layer1, void *ws, const WsLayout &wl, ScoreParams &sp) {
  std::memset(&sp, 0, sizeof(sp));
  for (int l = layer0; l < layer1; ++l) {
    const tria_status st = k_tensor_map(c, g.hkv, g.grouped != 0, c->k_layers[l], &sp.kmap[l - layer0]);
    if (st != TRIA_OK) return st;
  }
  sp.geo = g;
  sp.cache = make_cache_dev(c, layer0, layer1);
  sp.btile = at<uint16_t>(ws, wl.btile);
  sp.item_counter = at<uint32_t>(ws, wl.hdr);
  sp.status = at<int32_t>(ws, wl.hdr + 4);
  sp.seq_items = at<int32_t>(ws, wl.seq_items);
  sp.row_items = at<int32_t>(ws, wl.row_items);
  sp.moments = at<double>(ws, wl.moments);
  sp.raw = at<float>(ws, wl.raw);
  sp.raw_stride = wl.raw_stride;
  sp.wait_ns = (uint64_t)prm->wait_limit_ns;
  return TRIA_OK;
}

TailParams make_tail(const Geom &g, const tria_cache_view *c, void *ws, const WsLayout &wl) {
  TailParams tp{};
  tp.geo = g;
  tp.status = at<int32_t>(ws, wl.hdr + 4);
  tp.moments = at<double>(ws, wl.moments);
  tp.raw = at<float>(ws, wl.raw);
  tp.raw_stride = wl.raw_stride;
  tp.agg = at<float>(ws, wl.agg);
  tp.agg_stride = wl.agg_stride;
  tp.kept = nullptr;
  tp.hist = at<uint32_t>(ws, wl.hist);
  tp.unit_done = at<uint32_t>(ws, wl.unit_done);
  // dropping dead scratch lines from L2 saves their write-back only while the
  // scratch still fits in L2; beyond that they are long written back
  const bool small = (int64_t)g.n_units * wl.raw_stride * 4 <= (int64_t)48 << 20;
  tp.discard_raw = small ? 1 : 0;
  tp.discard_agg = small ? 1 : 0;
  return tp;
}

LensParams make_lens(const Geom &g, const tria_cache_view *c, int layer0, int layer1,
                     int32_t *freed_blocks, int32_t *n_freed) {
  LensParams lp{};
  lp.geo = g;
  lp.layer_lens = c->layer_seq_lens;
  lp.paged = c->layout == TRIA_LAYOUT_PAGED ? 1 : 0;
  lp.block_table = c->block_table;
  lp.max_blocks = c->max_blocks_per_seq;
  lp.block_size = c->block_size;
  lp.all_layers = (layer0 == 0 && layer1 == g.n_layers) ? 1 : 0;
  lp.freed_blocks = freed_blocks;
  lp.n_freed = n_freed;
  return lp;
}

}  // namespace

WsLayout ws_layout(const Geom &g) {
  WsLayout w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  w.raw_stride = (int64_t)align_up((size_t)g.c_max * g.g, 32);
  w.agg_stride = (int64_t)align_up((size_t)g.c_max, 32);
  w.hdr = take(256);
  w.unit_done = take((size_t)g.n_units * 4);
  w.seq_items = take((size_t)(g.n_seq + 1) * 4);
  w.row_items = take(((size_t)g.n_seq * g.nl + 1) * 4);
  w.btile = take((size_t)g.n_units * g.b_bytes);
  w.moments = take((size_t)g.n_units * g.tiles_max * kRowGroups * g.g * 2 * 8);
  w.hist = take((size_t)g.n_units * kAggHistBins * 4);
  w.raw = take((size_t)g.n_units * w.raw_stride * 4);
  w.agg = take((size_t)g.n_units * w.agg_stride * 4);
  w.kept = take((size_t)g.n_units * g.budget * 4);
  w.total = off;
  return w;
}

}  // namespace tria

using namespace tria;

extern "C" {

const char *tria_status_string(tria_status s) {
  switch (s) {
    case TRIA_OK: return "TRIA_OK";
    case TRIA_ERR_INVALID_ARG: return "TRIA_ERR_INVALID_ARG: invalid argument";
    case TRIA_ERR_UNSUPPORTED: return "TRIA_ERR_UNSUPPORTED: configuration not built";
    case TRIA_ERR_WORKSPACE: return "TRIA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case TRIA_ERR_CUDA: return "TRIA_ERR_CUDA: CUDA runtime error";
    case TRIA_ERR_OOM: return "TRIA_ERR_OOM: device allocation failed";
    case TRIA_ERR_IO: return "TRIA_ERR_IO: stats file missing, unreadable or not in this format";
  }
  return "unknown tria_status";
}

const char *tria_version(void) { return "tria 0.1 (sm_100a)"; }

tria_status tria_load_stats(const tria_model_desc *desc, const float *q_mean_re,
                            const float *q_mean_im, const float *q_abs_mean,
                            const float *band_mask, tria_stream_t stream, tria_stats **out) {
  if (desc == nullptr || q_mean_re == nullptr || q_mean_im == nullptr || q_abs_mean == nullptr ||
      out == nullptr)
    return TRIA_ERR_INVALID_ARG;
  *out = nullptr;
  const tria_model_desc d = *desc;
  if (d.n_layers < 1 || d.n_layers > TRIA_MAX_LAYERS || d.n_kv_heads < 1 || d.n_q_heads < 1 ||
      d.n_q_heads % d.n_kv_heads != 0)
    return TRIA_ERR_INVALID_ARG;
  if (d.pairing != TRIA_PAIR_NEOX && d.pairing != TRIA_PAIR_INTERLEAVED) return TRIA_ERR_INVALID_ARG;
  if (!(d.rope_theta > 1.0) || !std::isfinite(d.rope_theta)) return TRIA_ERR_INVALID_ARG;
  if (d.offset_log2_max < 0 || d.offset_log2_max > 30) return TRIA_ERR_INVALID_ARG;
  if (d.head_dim != TRIA_HEAD_DIM) return TRIA_ERR_UNSUPPORTED;
  const int G = d.n_q_heads / d.n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return TRIA_ERR_UNSUPPORTED;

  const int F = d.head_dim / 2;
  const size_t n = (size_t)d.n_layers * d.n_q_heads * F;
  std::vector<double> omega(F);
  std::vector<double> wre(F), wim(F);
  std::vector<double2> rot_off((size_t)F * kMaxOffsets, double2{0.0, 0.0});
  const int nd = d.offset_log2_max + 1;
  for (int f = 0; f < F; ++f) {
    omega[f] = std::pow(d.rope_theta, -2.0 * f / (double)d.head_dim);
    double sr = 0.0, si = 0.0;
    double delta = 1.0;
    for (int j = 0; j < nd; ++j) {
      const double c = std::cos(omega[f] * delta), sn = std::sin(omega[f] * delta);
      sr += c;
      si += sn;
      if (j < kMaxOffsets) rot_off[(size_t)f * kMaxOffsets + j] = double2{c, sn};
      delta *= 2.0;
    }
    wre[f] = sr / nd;
    wim[f] = si / nd;
  }
  std::vector<double2> mu(n), mu_raw(n);
  std::vector<double> wn(n);
  for (size_t i = 0; i < n; ++i) {
    const int f = (int)(i % F);
    const double re = q_mean_re[i], im = q_mean_im[i], am = q_abs_mean[i];
    if (!std::isfinite(re) || !std::isfinite(im) || !std::isfinite(am)) return TRIA_ERR_INVALID_ARG;
    double m = 1.0;
    if (band_mask != nullptr) {
      m = band_mask[f];
      if (!std::isfinite(m)) return TRIA_ERR_INVALID_ARG;
    }
    mu[i].x = (re * wre[f] - im * wim[f]) * m;
    mu[i].y = (re * wim[f] + im * wre[f]) * m;
    mu_raw[i].x = re * m;
    mu_raw[i].y = im * m;
    wn[i] = am - std::hypot(re, im);
  }

  tria_stats *st = new (std::nothrow) tria_stats();
  if (st == nullptr) return TRIA_ERR_OOM;
  st->dev.desc = d;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMalloc(&st->dev.mu_fold, n * sizeof(double2)) != cudaSuccess ||
      cudaMalloc(&st->dev.mu_raw, n * sizeof(double2)) != cudaSuccess ||
      cudaMalloc(&st->dev.w_norm, n * sizeof(double)) != cudaSuccess ||
      cudaMalloc(&st->dev.omega, F * sizeof(double)) != cudaSuccess ||
      cudaMalloc(&st->dev.rot_off, rot_off.size() * sizeof(double2)) != cudaSuccess) {
    cudaFree(st->dev.mu_fold);
    cudaFree(st->dev.mu_raw);
    cudaFree(st->dev.w_norm);
    cudaFree(st->dev.omega);
    cudaFree(st->dev.rot_off);
    delete st;
    cudaGetLastError();
    return TRIA_ERR_OOM;
  }
  cudaError_t e = cudaMemcpyAsync(st->dev.mu_fold, mu.data(), n * sizeof(double2),
                                  cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->dev.mu_raw, mu_raw.data(), n * sizeof(double2), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->dev.w_norm, wn.data(), n * sizeof(double), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->dev.omega, omega.data(), F * sizeof(double), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->dev.rot_off, rot_off.data(), rot_off.size() * sizeof(double2),
                        cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    tria_free_stats(st);
    return TRIA_ERR_CUDA;
  }
  *out = st;
  return TRIA_OK;
}

tria_status tria_free_stats(tria_stats *st) {
  if (st == nullptr) return TRIA_OK;
  cudaError_t e = cudaDeviceSynchronize();
  cudaFree(st->dev.mu_fold);
  cudaFree(st->dev.mu_raw);
  cudaFree(st->dev.w_norm);
  cudaFree(st->dev.omega);
  cudaFree(st->dev.rot_off);
  delete st;
  return cuda_status(e);
}

tria_status tria_stats_desc(const tria_stats *st, tria_model_desc *out) {
  if (st == nullptr || out == nullptr) return TRIA_ERR_INVALID_ARG;
  *out = st->dev.desc;
  return TRIA_OK;
}

tria_status tria_layer_budgets(const tria_stats *stats, const tria_cache_view *cache,
                               const tria_params *params, int *budgets, int *row_len) {
  if (stats == nullptr) return TRIA_ERR_INVALID_ARG;
  const int L = stats->dev.desc.n_layers;
  Geom g;
  const tria_status st = make_geom(stats, cache, params, 0, L, &g);
  if (st != TRIA_OK) return st;
  if (budgets != nullptr)
    for (int l = 0; l < L; ++l) budgets[l] = g.lbudget[l];
  if (row_len != nullptr) *row_len = g.budget;
  return TRIA_OK;
}

tria_status tria_workspace_size(const tria_stats *stats, const tria_cache_view *cache,
                                const tria_params *params, int layer0, int layer1,
                                size_t *bytes) {
  if (bytes == nullptr) return TRIA_ERR_INVALID_ARG;
  Geom g;
  tria_status st = make_geom(stats, cache, params, layer0, layer1, &g);
  if (st != TRIA_OK) return st;
  *bytes = ws_layout(g).total;
  return TRIA_OK;
}

tria_status tria_score(const tria_stats *stats, const tria_cache_view *cache,
                       const tria_params *params, int layer0, int layer1, float *agg_out,
                       float *scores_out, void *ws, size_t ws_bytes, tria_stream_t stream) {
  Geom g;
  tria_status st = make_geom(stats, cache, params, layer0, layer1, &g);
  if (st != TRIA_OK) return st;
  if (agg_out == nullptr || !aligned16(agg_out)) return TRIA_ERR_INVALID_ARG;
  if (scores_out != nullptr && !aligned16(scores_out)) return TRIA_ERR_INVALID_ARG;
  WsLayout wl;
  if ((st = check_workspace(g, ws, ws_bytes, &wl)) != TRIA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  static thread_local ScoreParams sp;
  if ((st = make_score(g, cache, params, layer0, layer1, ws, wl, sp)) != TRIA_OK) return st;
  TailParams tp = make_tail(g, cache, ws, wl);
  if (scores_out != nullptr) {
    sp.raw = scores_out;
    sp.raw_stride = (int64_t)g.c_max * g.g;
    tp.raw = scores_out;
    tp.raw_stride = sp.raw_stride;
    tp.discard_raw = 0;
  }
  tp.agg = agg_out;
  tp.agg_stride = g.c_max;
  tp.discard_agg = 0;
  if (launch_coef(make_coef(stats, g, cache, ws, wl, nullptr, false), s) != cudaSuccess)
    return TRIA_ERR_CUDA;
  if (launch_score(sp, s) != cudaSuccess) return TRIA_ERR_CUDA;
  return cuda_status(launch_tail(tp, s));
}

tria_status tria_select(const tria_stats *stats, const tria_cache_view *cache,
                        const tria_params *params, const float *agg, int layer0, int layer1,
                        int32_t *kept_idx, void *ws, size_t ws_bytes, tria_stream_t stream) {
  Geom g;
  tria_status st = make_geom(stats, cache, params, layer0, layer1, &g);
  if (st != TRIA_OK) return st;
  if (agg == nullptr || kept_idx == nullptr || !aligned16(agg)) return TRIA_ERR_INVALID_ARG;
  WsLayout wl;
  if ((st = check_workspace(g, ws, ws_bytes, &wl)) != TRIA_OK) return st;
  SelectParams p{};
  p.geo = g;
  p.status = at<int32_t>(ws, wl.hdr + 4);
  p.agg = agg;
  p.agg_stride = g.c_max;
  p.kept = kept_idx;
  return cuda_status(launch_select(p, reinterpret_cast<cudaStream_t>(stream)));
}

tria_status tria_compact(const tria_stats *stats, const tria_cache_view *cache,
                         const tria_params *params, const int32_t *kept_idx, int layer0,
                         int layer1, int32_t *freed_blocks, int32_t *n_freed,
                         tria_stream_t stream) {
  Geom g;
  tria_status st = make_geom(stats, cache, params, layer0, layer1, &g);
  if (st != TRIA_OK) return st;
  if (kept_idx == nullptr || cache->v_layers == nullptr) return TRIA_ERR_INVALID_ARG;
  for (int l = layer0; l < layer1; ++l)
    if (cache->v_layers[l] == nullptr || !aligned16(cache->v_layers[l])) return TRIA_ERR_INVALID_ARG;
  CompactParams p{};
  p.geo = g;
  p.cache = make_cache_dev(cache, layer0, layer1);
  p.kept = kept_idx;
  p.update_lens = (!g.per_layer && layer1 == g.n_layers) ? 1 : 0;
  p.freed_blocks = freed_blocks;
  p.n_freed = n_freed;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (launch_compact(p, s) != cudaSuccess) return TRIA_ERR_CUDA;
  if (!g.per_layer) return TRIA_OK;
  return cuda_status(launch_layer_lens(make_lens(g, cache, layer0, layer1, freed_blocks, n_freed), s));
}

static thread_local cudaEvent_t g_pass_events[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};

tria_status tria_set_pass_events(void *const *events) {
  for (int i = 0; i < 5; ++i)
    g_pass_events[i] = events ? static_cast<cudaEvent_t>(events[i]) : nullptr;
  return TRIA_OK;
}

static inline cudaError_t mark(int i, cudaStream_t s) {
  return g_pass_events[i] ? cudaEventRecord(g_pass_events[i], s) : cudaSuccess;
}

tria_status tria_compress_pass(const tria_stats *stats, const tria_cache_view *cache,
                               const tria_params *params, int32_t *kept_idx,
                               int32_t *freed_blocks, int32_t *n_freed, void *ws,
                               size_t ws_bytes, tria_stream_t stream) {
  Geom g;
  if (stats == nullptr) return TRIA_ERR_INVALID_ARG;
  const int L = stats->dev.desc.n_layers;
  tria_status st = make_geom(stats, cache, params, 0, L, &g);
  if (st != TRIA_OK) return st;
  if (cache->v_layers == nullptr) return TRIA_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l)
    if (cache->v_layers[l] == nullptr || !aligned16(cache->v_layers[l])) return TRIA_ERR_INVALID_ARG;
  WsLayout wl;
  if ((st = check_workspace(g, ws, ws_bytes, &wl)) != TRIA_OK) return st;
  int32_t *kept = kept_idx != nullptr ? kept_idx : at<int32_t>(ws, wl.kept);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  static thread_local ScoreParams sp;
  if ((st = make_score(g, cache, params, 0, L, ws, wl, sp)) != TRIA_OK) return st;
  TailParams tp = make_tail(g, cache, ws, wl);
  tp.kept = kept;
  // one block per unit when its candidates' keys fit in shared memory, else
  // blocks over candidate chunks with a histogram in the workspace
  const bool per_unit = unit_tail_fits(g);
  if (mark(0, s) != cudaSuccess) return TRIA_ERR_CUDA;
  if (launch_coef(make_coef(stats, g, cache, ws, wl, kept, !per_unit), s) != cudaSuccess)
    return TRIA_ERR_CUDA;
  if (mark(1, s) != cudaSuccess) return TRIA_ERR_CUDA;
  if (launch_score(sp, s) != cudaSuccess) return TRIA_ERR_CUDA;
  if (mark(2, s) != cudaSuccess) return TRIA_ERR_CUDA;
  if ((per_unit ? launch_unit_tail(tp, s) : launch_tail(tp, s)) != cudaSuccess) return TRIA_ERR_CUDA;
  if (mark(3, s) != cudaSuccess) return TRIA_ERR_CUDA;
  CompactParams cp{};
  cp.geo = g;
  cp.cache = make_cache_dev(cache, 0, L);
  cp.kept = kept;
  cp.update_lens = g.per_layer ? 0 : 1;
  cp.freed_blocks = freed_blocks;
  cp.n_freed = n_freed;
  if (launch_compact(cp, s) != cudaSuccess) return TRIA_ERR_CUDA;
  if (g.per_layer &&
      launch_layer_lens(make_lens(g, cache, 0, L, freed_blocks, n_freed), s) != cudaSuccess)
    return TRIA_ERR_CUDA;
  return cuda_status(mark(4, s));
}

tria_status tria_read_device_status(void *ws, tria_stream_t stream, int32_t *flags_out) {
  if (ws == nullptr || flags_out == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0)
    return TRIA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t *dflag = reinterpret_cast<int32_t *>(static_cast<unsigned char *>(ws) + 4);
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, dflag, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(dflag, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return TRIA_ERR_CUDA;
  *flags_out = h;
  return TRIA_OK;
}

}  // extern "C"
