// Kernels of the TriAttention compression pass for sm_100a.
//
//   coef_kernel     per (sequence, layer, query head): the per-pass scoring
//                   coefficients c_f = mu'_f e^{i omega_f p_q} (fp64 -> fp32)
//                   and w_f; resets the scheduling counters; lays out the
//                   work items of every sequence.
//   score_kernel    persistent; dynamic items of kTileKeys keys of one unit.
//                   S~_g(k) = sum_f Re(c_gf conj(ktilde_f)) + w_gf |ktilde_f|
//                   from the post-RoPE key ktilde (the key position cancels:
//                   conj(k_f) e^{i omega_f (p_q - p_k)} = conj(ktilde_f) e^{i omega_f p_q}).
//                   The CTA that finishes a unit's last item z-normalises,
//                   takes the GQA max and (in the fused pass) selects.
//   select_kernel   one CTA per unit: radix top-K of agg + ascending kept list.
//   compact_kernel  in-place gather of kept K/V rows (and positions).
//
// Sources: academ.us article 2607.13051 (Eqs. 2, 3, 4, 6, 7 and sec. 4),
// ghidav.me "TriAttention, or: what a rotating query already knows" ("The
// Method"), GitHub issue #10 of the llama.cpp TurboQuant HIP fork (RoPE
// pairing, window/sink conventions).
#include <cstddef>

#include <cuda_runtime.h>

#include "tria_internal.h"

namespace tria {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint4 ld_stream_v4(const void *ptr, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr), "l"(pol));
  return r;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void *ptr, uint64_t pol) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0,%1}, [%2], %3;"
               : "=r"(r.x), "=r"(r.y)
               : "l"(ptr), "l"(pol));
  return r;
}

// Drop a 128-byte L2 line without writing it back (scratch that is dead).
__device__ __forceinline__ void discard_line(const void *ptr) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(ptr) : "memory");
}

// Order-preserving unsigned key of an fp32 score: larger score -> larger
// key; -0.0 and +0.0 share a key; NaN gets the smallest key of all.
__device__ __forceinline__ uint32_t order_key(float a) {
  if (a != a) return 0u;
  uint32_t u = __float_as_uint(a);
  if (a == 0.0f) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan over the block (kThreads threads); *total receives the sum.
__device__ __forceinline__ int block_excl_scan(int v, int *s_warp, int *total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[w] = x;
  __syncthreads();
  int before = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) {
    int t = s_warp[i];
    before += (i < w) ? t : 0;
    tot += t;
  }
  __syncthreads();
  *total = tot;
  return before + x - v;
}

// Row pointer of slot t of (sequence s, layer index lrel, KV head h).
template <int LAYOUT>
__device__ __forceinline__ const uint16_t *k_row(const CacheDev &c, int lrel, int s, int h, int t) {
  int64_t off;
  if (LAYOUT == TRIA_LAYOUT_CONTIGUOUS) {
    off = (int64_t)s * c.s_seq + (int64_t)h * c.s_head + (int64_t)t * c.s_tok;
  } else {
    const int blk = c.block_table[(int64_t)s * c.max_blocks + t / c.block_size];
    off = (int64_t)blk * c.s_blk + (int64_t)(t % c.block_size) * c.s_tok + (int64_t)h * c.s_head;
  }
  return c.k[lrel] + off;
}

__device__ __forceinline__ int64_t row_off(const CacheDev &c, int s, int h, int t) {
  if (c.layout == TRIA_LAYOUT_CONTIGUOUS)
    return (int64_t)s * c.s_seq + (int64_t)h * c.s_head + (int64_t)t * c.s_tok;
  const int blk = c.block_table[(int64_t)s * c.max_blocks + t / c.block_size];
  return (int64_t)blk * c.s_blk + (int64_t)(t % c.block_size) * c.s_tok + (int64_t)h * c.s_head;
}

// ---------------------------------------------------------------------------
// Selection of one unit (shared by the fused tail and select_kernel).
// ---------------------------------------------------------------------------
struct SelectSmem {
  uint32_t hist[kWarps][256];
  int warp_tmp[kWarps];
  uint32_t prefix;
  int remaining;
  int digit;
  int above;
};

// Combine the per-warp histograms and pick the digit that holds the
// `remaining`-th largest key.  Updates prefix / remaining.
__device__ void pick_digit(SelectSmem &sm, int shift) {
  const int t = threadIdx.x;
  __syncthreads();
  const int d = 255 - t;  // thread t looks at bin d (descending order)
  int v = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) v += (int)sm.hist[w][d];
  int total;
  const int excl = block_excl_scan(v, sm.warp_tmp, &total);
  const int rem = sm.remaining;
  if (excl < rem && rem <= excl + v) {
    sm.digit = d;
    sm.above = excl;
  }
  __syncthreads();
  if (t == 0) {
    sm.prefix |= (uint32_t)sm.digit << shift;
    sm.remaining = rem - sm.above;
  }
  __syncthreads();
}

__device__ __forceinline__ void clear_hist(SelectSmem &sm) {
  for (int i = threadIdx.x; i < kWarps * 256; i += kThreads) (&sm.hist[0][0])[i] = 0u;
}

// Radix passes 1..3 (pass 0's histogram is already in sm.hist), then the
// ascending emission of kept slots.  agg: the unit's C candidate scores.
__device__ void select_finish(SelectSmem &sm, const float *agg, int C, int K, int N, int B,
                              int W, int S, int32_t *kept) {
  const int t = threadIdx.x, warp = t >> 5;
  // sinks and window are always kept
  for (int j = t; j < S; j += kThreads) kept[j] = j;
  for (int j = t; j < W; j += kThreads) kept[B - W + j] = N - W + j;
  if (K <= 0) return;
  if (t == 0) {
    sm.prefix = 0u;
    sm.remaining = K;
  }
  pick_digit(sm, 24);
  for (int shift = 16; shift >= 0; shift -= 8) {
    clear_hist(sm);
    __syncthreads();
    const uint32_t pmask = 0xffffffffu << (shift + 8);
    const uint32_t pre = sm.prefix;
    for (int c = t; c < C; c += kThreads) {
      const uint32_t key = order_key(__ldcg(agg + c));
      if ((key & pmask) == pre) atomicAdd(&sm.hist[warp][(key >> shift) & 255u], 1u);
    }
    pick_digit(sm, shift);
  }
  const uint32_t T = sm.prefix;
  const int need_ties = sm.remaining;  // keys equal to T still to take (>= 1)
  int run_ties = 0, run_keep = 0;
  constexpr int E = 8;
  for (int base = 0; base < C && run_keep < K; base += kThreads * E) {
    uint32_t keys[E];
    int nt = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = base + t * E + e;
      keys[e] = (c < C) ? order_key(__ldcg(agg + c)) : 0u;
      nt += (c < C && keys[e] == T) ? 1 : 0;
    }
    int tot_t;
    const int ex_t = block_excl_scan(nt, sm.warp_tmp, &tot_t);
    int tie = run_ties + ex_t, nk = 0;
    bool keep[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = base + t * E + e;
      bool k = false;
      if (c < C) {
        if (keys[e] > T) {
          k = true;
        } else if (keys[e] == T) {
          k = tie < need_ties;
          ++tie;
        }
      }
      keep[e] = k;
      nk += k ? 1 : 0;
    }
    int tot_k;
    int pos = run_keep + block_excl_scan(nk, sm.warp_tmp, &tot_k);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (keep[e] && pos < K) kept[S + pos] = S + base + t * E + e;
      pos += keep[e] ? 1 : 0;
    }
    run_ties += tot_t;
    run_keep += tot_k;
  }
}

// ---------------------------------------------------------------------------
// coef_kernel: grid (n_seq * nl * hq), block 64
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(64) coef_kernel(const __grid_constant__ CoefParams p) {
  const Geom &g = p.geo;
  const int f = threadIdx.x;
  const int64_t blk = blockIdx.x;
  const int qh = (int)(blk % g.hq);
  const int lrel = (int)((blk / g.hq) % g.nl);
  const int s = (int)(blk / ((int64_t)g.hq * g.nl));
  const int l = g.layer0 + lrel;
  const int N = p.seq_lens[s];
  const bool bad = (N < 0 || N > g.max_seq_len);

  if (blk == 0) {
    if (f == 0) *p.item_counter = 0u;
    // items per sequence, prefix over sequences (n_seq <= 1024: <= 16 per thread)
    __shared__ int s_part[64];
    const int per = (g.n_seq + 63) / 64;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int sq = f * per + i;
      if (sq < g.n_seq) {
        const int n = p.seq_lens[sq];
        int items = 0;
        if (n >= 0 && n <= g.max_seq_len && n > g.budget) {
          const int C = n - g.window - g.sinks;
          items = ((C + kTileKeys - 1) / kTileKeys) * g.nl * g.hkv;
        }
        local += items;
      }
    }
    s_part[f] = local;
    __syncthreads();
    if (f == 0) {
      int run = 0;
      for (int i = 0; i < 64; ++i) {
        const int v = s_part[i];
        s_part[i] = run;
        run += v;
      }
    }
    __syncthreads();
    int run = s_part[f];
    for (int i = 0; i < per; ++i) {
      const int sq = f * per + i;
      if (sq < g.n_seq) {
        p.seq_items[sq] = run;
        const int n = p.seq_lens[sq];
        if (n >= 0 && n <= g.max_seq_len && n > g.budget) {
          const int C = n - g.window - g.sinks;
          run += ((C + kTileKeys - 1) / kTileKeys) * g.nl * g.hkv;
        }
      }
    }
    if (f == 63) p.seq_items[g.n_seq] = run;
  }

  if (qh % g.g == 0) {
    const int h = qh / g.g;
    const int64_t u = ((int64_t)s * g.nl + lrel) * g.hkv + h;
    if (f == 0) {
      p.unit_done[u] = 0u;
      if (bad && lrel == 0 && h == 0) atomicOr(p.status, 1);
    }
    if (p.kept != nullptr && (bad || N <= g.budget)) {
      int32_t *kr = p.kept + u * g.budget;
      for (int j = f; j < g.budget; j += 64) kr[j] = (!bad && j < N) ? j : -1;
    }
  }

  // c_f = mu'_f e^{i omega_f p_q} in fp64, rounded to fp32
  const double2 mu = p.mu_fold[((int64_t)l * g.hq + qh) * kBands + f];
  const double ang = p.omega[f] * (double)p.query_pos[s];
  double sn, cs;
  sincos(ang, &sn, &cs);
  float *dst = p.coef + (((int64_t)s * g.nl + lrel) * g.hq + qh) * kCoefPerHead;
  dst[f] = (float)(mu.x * cs - mu.y * sn);
  dst[kBands + f] = (float)(mu.x * sn + mu.y * cs);
  dst[2 * kBands + f] = (float)p.w_norm[((int64_t)l * g.hq + qh) * kBands + f];
}

// ---------------------------------------------------------------------------
// score_kernel (CUDA cores): half-warp per key, each lane owns 4 bands.
// ---------------------------------------------------------------------------
template <int G>
__device__ __forceinline__ float halfwarp_reduce(float (&a)[G], int hl) {
  // Reduce-scatter of G partial sums over the 16 lanes of a half-warp; lane
  // hl ends with the total of head hl >> log2(16 / G).
  if constexpr (G >= 16) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool up = hl & 8;
      float keep = up ? a[8 + i] : a[i], give = up ? a[i] : a[8 + i];
      a[i] = keep + __shfl_xor_sync(kFull, give, 8);
    }
  }
  if constexpr (G >= 8) {
    constexpr int o = (G >= 16) ? 4 : 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool up = hl & o;
      float keep = up ? a[4 + i] : a[i], give = up ? a[i] : a[4 + i];
      a[i] = keep + __shfl_xor_sync(kFull, give, o);
    }
  }
  if constexpr (G >= 4) {
    constexpr int o = (G >= 16) ? 2 : (G >= 8) ? 4 : 8;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const bool up = hl & o;
      float keep = up ? a[2 + i] : a[i], give = up ? a[i] : a[2 + i];
      a[i] = keep + __shfl_xor_sync(kFull, give, o);
    }
  }
  if constexpr (G >= 2) {
    constexpr int o = (G >= 16) ? 1 : (G >= 8) ? 2 : (G >= 4) ? 4 : 8;
    const bool up = hl & o;
    float keep = up ? a[1] : a[0], give = up ? a[0] : a[1];
    a[0] = keep + __shfl_xor_sync(kFull, give, o);
  }
  // remaining offsets: plain sums (all lanes of the group end equal)
  constexpr int done = (G >= 16) ? 4 : (G >= 8) ? 3 : (G >= 4) ? 2 : (G >= 2) ? 1 : 0;
#pragma unroll
  for (int st = done; st < 4; ++st) a[0] += __shfl_xor_sync(kFull, a[0], 8 >> st);
  return a[0];
}

struct ScoreSmem {
  alignas(16) float coef[TRIA_MAX_GROUP * kCoefPerHead];  // read as float4
  alignas(16) double mom[16][TRIA_MAX_GROUP][2];
  alignas(16) int seq_items[kMaxSeqTable];
  float mean[TRIA_MAX_GROUP];
  float inv[TRIA_MAX_GROUP];
  int item;
  int last;
  SelectSmem sel;
};
static_assert(offsetof(ScoreSmem, coef) % 16 == 0, "coef is read as float4");

template <int G>
__device__ void unit_tail(const ScoreParams &p, ScoreSmem &sm, int64_t u, int C, int ntiles,
                          int N) {
  const Geom &geo = p.geo;
  const int t = threadIdx.x, warp = t >> 5;
  // population mean / std of each head over the C candidates
  if (t < G) {
    const double *m = p.moments + (u * geo.tiles_max) * G * 2;
    double s1 = 0.0, s2 = 0.0;
    for (int i = 0; i < ntiles; ++i) {
      s1 += __ldcg(m + (int64_t)i * G * 2 + t * 2);
      s2 += __ldcg(m + (int64_t)i * G * 2 + t * 2 + 1);
    }
    const double mean = s1 / C;
    double var = s2 / C - mean * mean;
    var = var > 0.0 ? var : 0.0;
    sm.mean[t] = (float)mean;
    sm.inv[t] = (float)(1.0 / (sqrt(var) + 1e-6));
  }
  const bool do_sel = p.kept != nullptr;
  if (do_sel) clear_hist(sm.sel);
  __syncthreads();
  float mean[G], inv[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    mean[g] = sm.mean[g];
    inv[g] = sm.inv[g];
  }
  const float *raw = p.raw + u * p.raw_stride;
  float *agg = p.agg + u * p.agg_stride;
  for (int c = t; c < C; c += kThreads) {
    float a = 0.0f;
    bool nan = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float z = __fmul_rn(__fsub_rn(__ldcg(raw + (int64_t)c * G + g), mean[g]), inv[g]);
      a = (g == 0) ? z : fmaxf(a, z);
      nan |= (z != z);
    }
    if (nan) a = __int_as_float(0x7fc00000);
    agg[c] = a;
    if (do_sel) atomicAdd(&sm.sel.hist[warp][order_key(a) >> 24], 1u);
  }
  __syncthreads();
  if (p.discard_raw) {
    const int64_t lines = ((int64_t)C * G * 4 + 127) / 128;
    for (int64_t i = t; i < lines; i += kThreads) discard_line(raw + i * 32);
  }
  if (!do_sel) return;
  __threadfence_block();
  const int K = geo.budget - geo.window - geo.sinks;
  select_finish(sm.sel, agg, C, K, N, geo.budget, geo.window, geo.sinks,
                p.kept + u * geo.budget);
  __syncthreads();
  if (p.discard_agg) {
    const int64_t lines = ((int64_t)C * 4 + 127) / 128;
    for (int64_t i = t; i < lines; i += kThreads) discard_line(agg + i * 32);
  }
}

template <int G, int PAIR, int LAYOUT>
__global__ void __launch_bounds__(kThreads, (G >= 8) ? 1 : 2)
    score_kernel(const __grid_constant__ ScoreParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ScoreSmem &sm = *reinterpret_cast<ScoreSmem *>(smem_raw);
  const Geom &geo = p.geo;
  const int t = threadIdx.x;
  const int hl = t & 15, hw = t >> 4;
  constexpr int SPLIT = 16 / G;
  const int my_head = hl / SPLIT;
  const bool owner = (hl % SPLIT) == 0;
  const uint64_t pol = evict_first_policy();

  for (int i = t; i <= geo.n_seq; i += kThreads) sm.seq_items[i] = p.seq_items[i];
  __syncthreads();
  const int n_items = sm.seq_items[geo.n_seq];
  const int units_per_seq = geo.nl * geo.hkv;

  for (;;) {
    if (t == 0) sm.item = (int)atomicAdd(p.item_counter, 1u);
    __syncthreads();
    const int item = sm.item;
    if (item >= n_items) break;
    // sequence: last s with seq_items[s] <= item
    int lo = 0, hi = geo.n_seq - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.seq_items[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int ntiles = (sm.seq_items[s + 1] - sm.seq_items[s]) / units_per_seq;
    const int rem = item - sm.seq_items[s];
    const int ul = rem / ntiles, tile = rem % ntiles;
    const int lrel = ul / geo.hkv, h = ul % geo.hkv;
    const int64_t u = (int64_t)s * units_per_seq + ul;
    const int N = p.cache.seq_lens[s];
    const int C = N - geo.window - geo.sinks;
    const int c0 = tile * kTileKeys;
    const int c1 = min(C, c0 + kTileKeys);

    const float *cg = p.coef + (((int64_t)s * geo.nl + lrel) * geo.hq + h * G) * kCoefPerHead;
    for (int i = t; i < G * kCoefPerHead / 4; i += kThreads)
      reinterpret_cast<float4 *>(sm.coef)[i] = __ldcg(reinterpret_cast<const float4 *>(cg) + i);
    __syncthreads();
    float cre[G][4], cim[G][4], cw[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float4 a = *reinterpret_cast<const float4 *>(sm.coef + g * kCoefPerHead + 4 * hl);
      const float4 b = *reinterpret_cast<const float4 *>(sm.coef + g * kCoefPerHead + kBands + 4 * hl);
      const float4 w = *reinterpret_cast<const float4 *>(sm.coef + g * kCoefPerHead + 2 * kBands + 4 * hl);
      cre[g][0] = a.x; cre[g][1] = a.y; cre[g][2] = a.z; cre[g][3] = a.w;
      cim[g][0] = b.x; cim[g][1] = b.y; cim[g][2] = b.z; cim[g][3] = b.w;
      cw[g][0] = w.x; cw[g][1] = w.y; cw[g][2] = w.z; cw[g][3] = w.w;
    }
    double msum = 0.0, msq = 0.0;
    float *raw = p.raw + u * p.raw_stride;

    // both half-warps of a warp iterate together (full-warp shuffles below)
    for (int cb = c0 + 2 * (hw >> 1); cb < c1; cb += 16) {
      const int c = cb + (hw & 1);
      const bool valid = c < c1;
      const uint16_t *row = k_row<LAYOUT>(p.cache, lrel, s, h, geo.sinks + (valid ? c : cb));
      float xr[4], xi[4];
      if (PAIR == TRIA_PAIR_NEOX) {
        uint2 a = make_uint2(0u, 0u), b = make_uint2(0u, 0u);
        if (valid) {
          a = ld_stream_v2(row + 4 * hl, pol);
          b = ld_stream_v2(row + kBands + 4 * hl, pol);
        }
        xr[0] = bf_lo(a.x); xr[1] = bf_hi(a.x); xr[2] = bf_lo(a.y); xr[3] = bf_hi(a.y);
        xi[0] = bf_lo(b.x); xi[1] = bf_hi(b.x); xi[2] = bf_lo(b.y); xi[3] = bf_hi(b.y);
      } else {
        uint4 a = make_uint4(0u, 0u, 0u, 0u);
        if (valid) a = ld_stream_v4(row + 8 * hl, pol);
        xr[0] = bf_lo(a.x); xi[0] = bf_hi(a.x);
        xr[1] = bf_lo(a.y); xi[1] = bf_hi(a.y);
        xr[2] = bf_lo(a.z); xi[2] = bf_hi(a.z);
        xr[3] = bf_lo(a.w); xi[3] = bf_hi(a.w);
      }
      float acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = 0.0f;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float m = sqrt_approx(fmaf(xr[b], xr[b], xi[b] * xi[b]));
#pragma unroll
        for (int g = 0; g < G; ++g) {
          acc[g] = fmaf(cre[g][b], xr[b], acc[g]);
          acc[g] = fmaf(cim[g][b], xi[b], acc[g]);
          acc[g] = fmaf(cw[g][b], m, acc[g]);
        }
      }
      const float sc = halfwarp_reduce<G>(acc, hl);
      if (owner && valid) {
        raw[(int64_t)c * G + my_head] = sc;
        msum += (double)sc;
        msq = fma((double)sc, (double)sc, msq);
      }
    }
    if (owner) {
      sm.mom[hw][my_head][0] = msum;
      sm.mom[hw][my_head][1] = msq;
    }
    __syncthreads();
    if (t < G) {
      double s1 = 0.0, s2 = 0.0;
      for (int i = 0; i < 16; ++i) {
        s1 += sm.mom[i][t][0];
        s2 += sm.mom[i][t][1];
      }
      double *m = p.moments + ((u * geo.tiles_max + tile) * G + t) * 2;
      m[0] = s1;
      m[1] = s2;
    }
    __threadfence();
    __syncthreads();
    if (t == 0) {
      const uint32_t done = atomicAdd(p.unit_done + u, 1u);
      sm.last = (done == (uint32_t)ntiles - 1u) ? 1 : 0;
    }
    __syncthreads();
    if (sm.last) {
      __threadfence();
      unit_tail<G>(p, sm, u, C, ntiles, N);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// select_kernel: one CTA per unit
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) select_kernel(const __grid_constant__ SelectParams p) {
  __shared__ SelectSmem sm;
  const Geom &geo = p.geo;
  const int64_t u = blockIdx.x;
  const int s = (int)(u / ((int64_t)geo.nl * geo.hkv));
  const int N = p.seq_lens[s];
  int32_t *kept = p.kept + u * geo.budget;
  const int t = threadIdx.x, warp = t >> 5;
  if (N < 0 || N > geo.max_seq_len || N <= geo.budget) {
    const bool bad = (N < 0 || N > geo.max_seq_len);
    if (bad && t == 0 && u == 0) atomicOr(p.status, 1);
    for (int j = t; j < geo.budget; j += kThreads) kept[j] = (!bad && j < N) ? j : -1;
    return;
  }
  const int C = N - geo.window - geo.sinks;
  const int K = geo.budget - geo.window - geo.sinks;
  const float *agg = p.agg + u * p.agg_stride;
  clear_hist(sm);
  __syncthreads();
  for (int c = t; c < C; c += kThreads)
    atomicAdd(&sm.hist[warp][order_key(__ldcg(agg + c)) >> 24], 1u);
  select_finish(sm, agg, C, K, N, geo.budget, geo.window, geo.sinks, kept);
}

// ---------------------------------------------------------------------------
// compact_kernel: items (unit, part) with part 0/1 = K bytes [0,128)/[128,256),
// part 2/3 = V.  Destination chunks are walked in ascending order; a chunk's
// sources are all read before any of its rows is written.  Because the kept
// list is ascending with kept[j] >= j, a chunk never overwrites a row that a
// later chunk still has to read.
// ---------------------------------------------------------------------------
constexpr int kCompactRowsPerChunk = 256;  // 8 threads x 16 B per half row

__global__ void __launch_bounds__(kThreads) compact_kernel(const __grid_constant__ CompactParams p) {
  const Geom &geo = p.geo;
  const int t = threadIdx.x;
  const int sub = t & 7;         // 16-byte piece of the 128-byte half row
  const int rsub = t >> 3;       // 0..31
  const int64_t n_items = geo.n_units * 4;
  for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x) {
    const int64_t u = it >> 2;
    const int part = (int)(it & 3);
    const int s = (int)(u / ((int64_t)geo.nl * geo.hkv));
    const int ul = (int)(u % ((int64_t)geo.nl * geo.hkv));
    const int lrel = ul / geo.hkv, h = ul % geo.hkv;
    const int32_t *kept = p.kept + u * geo.budget;
    uint16_t *base = (part < 2) ? const_cast<uint16_t *>(p.cache.k[lrel]) : p.cache.v[lrel];
    const int byte_off = (part & 1) * 128 + sub * 16;
    // positions are laid out over all layers of the model
    const int64_t pu = ((int64_t)s * geo.n_layers + geo.layer0 + lrel) * geo.hkv + h;
    int32_t *pos = (part == 0 && p.cache.positions != nullptr)
                       ? p.cache.positions + pu * p.cache.pos_unit_stride
                       : nullptr;
    for (int j0 = 0; j0 < geo.budget; j0 += kCompactRowsPerChunk) {
      uint4 vals[kCompactRowsPerChunk / 32];
      int32_t pv[kCompactRowsPerChunk / 32];
      int srcs[kCompactRowsPerChunk / 32];
#pragma unroll
      for (int r = 0; r < kCompactRowsPerChunk / 32; ++r) {
        const int j = j0 + r * 32 + rsub;
        int src = (j < geo.budget) ? kept[j] : -1;
        // only well-formed moves inside the cache capacity
        if (src == j || src < 0 || src >= geo.max_seq_len || j >= geo.max_seq_len) src = -1;
        srcs[r] = src;
        if (src >= 0) {
          const uint16_t *row = base + row_off(p.cache, s, h, src);
          vals[r] = *reinterpret_cast<const uint4 *>(reinterpret_cast<const unsigned char *>(row) + byte_off);
          if (pos != nullptr && sub == 0) pv[r] = pos[src];
        }
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < kCompactRowsPerChunk / 32; ++r) {
        const int j = j0 + r * 32 + rsub;
        if (srcs[r] >= 0) {
          uint16_t *row = base + row_off(p.cache, s, h, j);
          *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(row) + byte_off) = vals[r];
          if (pos != nullptr && sub == 0) pos[j] = pv[r];
        }
      }
      __syncthreads();
    }
    // sequence length / freed blocks: once per sequence, after the last layer
    if (p.update_lens && part == 0 && ul == 0 && t == 0) {
      const int N = p.cache.seq_lens[s];
      int newlen = geo.budget;
      if (kept[geo.budget - 1] < 0) {
        newlen = 0;
        while (newlen < geo.budget && kept[newlen] >= 0) ++newlen;
      }
      if (N > geo.budget && N <= geo.max_seq_len) {
        if (p.cache.layout == TRIA_LAYOUT_PAGED && p.n_freed != nullptr) {
          const int bs = p.cache.block_size;
          const int keep_blocks = (newlen + bs - 1) / bs;
          const int old_blocks = (N + bs - 1) / bs;
          int nf = 0;
          for (int b = keep_blocks; b < old_blocks; ++b) {
            if (p.freed_blocks != nullptr)
              p.freed_blocks[(int64_t)s * p.cache.max_blocks + nf] =
                  p.cache.block_table[(int64_t)s * p.cache.max_blocks + b];
            ++nf;
          }
          p.n_freed[s] = nf;
        }
        p.cache.seq_lens[s] = newlen;
      } else if (p.cache.layout == TRIA_LAYOUT_PAGED && p.n_freed != nullptr) {
        p.n_freed[s] = 0;
      }
    }
  }
}

template <int G, int PAIR, int LAYOUT>
cudaError_t launch_score_t(const ScoreParams &p, cudaStream_t st) {
  auto kern = score_kernel<G, PAIR, LAYOUT>;
  const int smem = (int)sizeof(ScoreSmem);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) != cudaSuccess)
    return e;
  if (per_sm < 1) per_sm = 1;
  kern<<<sms * per_sm, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int G>
cudaError_t launch_score_g(const ScoreParams &p, cudaStream_t st) {
  const bool paged = p.cache.layout == TRIA_LAYOUT_PAGED;
  if (p.geo.pairing == TRIA_PAIR_NEOX)
    return paged ? launch_score_t<G, TRIA_PAIR_NEOX, TRIA_LAYOUT_PAGED>(p, st)
                 : launch_score_t<G, TRIA_PAIR_NEOX, TRIA_LAYOUT_CONTIGUOUS>(p, st);
  return paged ? launch_score_t<G, TRIA_PAIR_INTERLEAVED, TRIA_LAYOUT_PAGED>(p, st)
               : launch_score_t<G, TRIA_PAIR_INTERLEAVED, TRIA_LAYOUT_CONTIGUOUS>(p, st);
}

}  // namespace

cudaError_t launch_coef(const CoefParams &p, cudaStream_t st) {
  const int64_t blocks = (int64_t)p.geo.n_seq * p.geo.nl * p.geo.hq;
  coef_kernel<<<(unsigned)blocks, 64, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_score(const ScoreParams &p, cudaStream_t st) {
  switch (p.geo.g) {
    case 1: return launch_score_g<1>(p, st);
    case 2: return launch_score_g<2>(p, st);
    case 4: return launch_score_g<4>(p, st);
    case 8: return launch_score_g<8>(p, st);
    case 16: return launch_score_g<16>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_select(const SelectParams &p, cudaStream_t st) {
  select_kernel<<<(unsigned)p.geo.n_units, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_compact(const CompactParams &p, cudaStream_t st) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t items = p.geo.n_units * 4;
  int64_t grid = (int64_t)sms * 8;
  if (grid > items) grid = items;
  compact_kernel<<<(unsigned)grid, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace tria
