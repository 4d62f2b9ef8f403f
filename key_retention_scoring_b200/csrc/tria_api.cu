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
#include <new>
#include <vector>

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
  if (params->window < 0 || params->sinks < 0 || params->budget < 1 ||
      params->budget < params->window + params->sinks)
    return TRIA_ERR_INVALID_ARG;
  if (cache->layout != TRIA_LAYOUT_CONTIGUOUS && cache->layout != TRIA_LAYOUT_PAGED)
    return TRIA_ERR_INVALID_ARG;
  if (cache->k_layers == nullptr || cache->seq_lens == nullptr || cache->query_pos == nullptr)
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
    if (cache->block_table == nullptr || cache->block_size < 1 || cache->block_size > 1024 ||
        cache->max_blocks_per_seq < 1)
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
  g.budget = params->budget;
  g.window = params->window;
  g.sinks = params->sinks;
  g.max_seq_len = cache->max_seq_len;
  const int cm = cache->max_seq_len - params->window - params->sinks;
  g.c_max = cm > 1 ? cm : 1;
  g.tiles_max = (g.c_max + kTileKeys - 1) / kTileKeys;
  g.pairing = d.pairing;
  g.n_units = (int64_t)g.n_seq * g.nl * g.hkv;
  if (g.n_units * (int64_t)g.tiles_max > INT32_MAX) return TRIA_ERR_UNSUPPORTED;
  *geo = g;
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
                     const WsLayout &wl, int32_t *kept) {
  CoefParams cp{};
  cp.geo = g;
  cp.mu_fold = st->dev.mu_fold;
  cp.w_norm = st->dev.w_norm;
  cp.omega = st->dev.omega;
  cp.query_pos = c->query_pos;
  cp.seq_lens = c->seq_lens;
  cp.coef = at<float>(ws, wl.coef);
  cp.item_counter = at<uint32_t>(ws, wl.hdr);
  cp.status = at<int32_t>(ws, wl.hdr + 4);
  cp.unit_done = at<uint32_t>(ws, wl.unit_done);
  cp.seq_items = at<int32_t>(ws, wl.seq_items);
  cp.kept = kept;
  return cp;
}

ScoreParams make_score(const Geom &g, const tria_cache_view *c, int layer0, int layer1, void *ws,
                       const WsLayout &wl) {
  ScoreParams sp{};
  sp.geo = g;
  sp.cache = make_cache_dev(c, layer0, layer1);
  sp.coef = at<float>(ws, wl.coef);
  sp.item_counter = at<uint32_t>(ws, wl.hdr);
  sp.status = at<int32_t>(ws, wl.hdr + 4);
  sp.unit_done = at<uint32_t>(ws, wl.unit_done);
  sp.seq_items = at<int32_t>(ws, wl.seq_items);
  sp.moments = at<double>(ws, wl.moments);
  sp.raw = at<float>(ws, wl.raw);
  sp.raw_stride = wl.raw_stride;
  sp.agg = at<float>(ws, wl.agg);
  sp.agg_stride = wl.agg_stride;
  sp.kept = nullptr;
  sp.discard_raw = 1;
  sp.discard_agg = 1;
  return sp;
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
  w.coef = take((size_t)g.n_seq * g.nl * g.hq * kCoefPerHead * 4);
  w.moments = take((size_t)g.n_units * g.tiles_max * g.g * 2 * 8);
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
  const int nd = d.offset_log2_max + 1;
  for (int f = 0; f < F; ++f) {
    omega[f] = std::pow(d.rope_theta, -2.0 * f / (double)d.head_dim);
    double sr = 0.0, si = 0.0;
    double delta = 1.0;
    for (int j = 0; j < nd; ++j) {
      sr += std::cos(omega[f] * delta);
      si += std::sin(omega[f] * delta);
      delta *= 2.0;
    }
    wre[f] = sr / nd;
    wim[f] = si / nd;
  }
  std::vector<double2> mu(n);
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
    wn[i] = am - std::hypot(re, im);
  }

  tria_stats *st = new (std::nothrow) tria_stats();
  if (st == nullptr) return TRIA_ERR_OOM;
  st->dev.desc = d;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMalloc(&st->dev.mu_fold, n * sizeof(double2)) != cudaSuccess ||
      cudaMalloc(&st->dev.w_norm, n * sizeof(double)) != cudaSuccess ||
      cudaMalloc(&st->dev.omega, F * sizeof(double)) != cudaSuccess) {
    cudaFree(st->dev.mu_fold);
    cudaFree(st->dev.w_norm);
    cudaFree(st->dev.omega);
    delete st;
    cudaGetLastError();
    return TRIA_ERR_OOM;
  }
  cudaError_t e = cudaMemcpyAsync(st->dev.mu_fold, mu.data(), n * sizeof(double2),
                                  cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->dev.w_norm, wn.data(), n * sizeof(double), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->dev.omega, omega.data(), F * sizeof(double), cudaMemcpyHostToDevice, s);
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
  cudaFree(st->dev.w_norm);
  cudaFree(st->dev.omega);
  delete st;
  return cuda_status(e);
}

tria_status tria_stats_desc(const tria_stats *st, tria_model_desc *out) {
  if (st == nullptr || out == nullptr) return TRIA_ERR_INVALID_ARG;
  *out = st->dev.desc;
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
  cudaError_t e = launch_coef(make_coef(stats, g, cache, ws, wl, nullptr), s);
  if (e != cudaSuccess) return TRIA_ERR_CUDA;
  ScoreParams sp = make_score(g, cache, layer0, layer1, ws, wl);
  if (scores_out != nullptr) {
    sp.raw = scores_out;
    sp.raw_stride = (int64_t)g.c_max * g.g;
    sp.discard_raw = 0;
  }
  sp.agg = agg_out;
  sp.agg_stride = g.c_max;
  sp.discard_agg = 0;
  return cuda_status(launch_score(sp, s));
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
  p.seq_lens = cache->seq_lens;
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
  p.update_lens = (layer1 == g.n_layers) ? 1 : 0;
  p.freed_blocks = freed_blocks;
  p.n_freed = n_freed;
  return cuda_status(launch_compact(p, reinterpret_cast<cudaStream_t>(stream)));
}

static thread_local cudaEvent_t g_pass_events[4] = {nullptr, nullptr, nullptr, nullptr};

tria_status tria_set_pass_events(void *const *events) {
  for (int i = 0; i < 4; ++i)
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
  if (mark(0, s) != cudaSuccess) return TRIA_ERR_CUDA;
  if (launch_coef(make_coef(stats, g, cache, ws, wl, kept), s) != cudaSuccess) return TRIA_ERR_CUDA;
  if (mark(1, s) != cudaSuccess) return TRIA_ERR_CUDA;
  ScoreParams sp = make_score(g, cache, 0, L, ws, wl);
  sp.kept = kept;
  if (launch_score(sp, s) != cudaSuccess) return TRIA_ERR_CUDA;
  if (mark(2, s) != cudaSuccess) return TRIA_ERR_CUDA;
  CompactParams cp{};
  cp.geo = g;
  cp.cache = make_cache_dev(cache, 0, L);
  cp.kept = kept;
  cp.update_lens = 1;
  cp.freed_blocks = freed_blocks;
  cp.n_freed = n_freed;
  if (launch_compact(cp, s) != cudaSuccess) return TRIA_ERR_CUDA;
  return cuda_status(mark(3, s));
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
