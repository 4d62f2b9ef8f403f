// Device helpers shared by the kernels: bf16 unpacking, cache hints, the
// order-preserving score key, block scans, the radix top-K selection of one
// unit over agg in global memory and normalize-then-max.
//
// Everything that synchronises takes a barrier id BAR: 0 = __syncthreads of
// a kSelThreads-thread block, n > 0 = named barrier n over the first
// kSelThreads threads of a larger block.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "tria_internal.h"

namespace tria {
namespace dev {

constexpr int kSelThreads = 256;  // threads of the standalone selection block
constexpr uint32_t kFull = 0xffffffffu;

// Barrier over a group of NT threads: BAR 0 = __syncthreads (the group is the
// block), BAR n > 0 = named barrier n.
template <int BAR, int NT>
__device__ __forceinline__ void csync() {
  if constexpr (BAR == 0) {
    __syncthreads();
  } else {
    asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
  }
}

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

// Drop a 128-byte L2 line without writing it back (scratch that is dead).
__device__ __forceinline__ void discard_line(const void *ptr) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(ptr) : "memory");
}

// Maximum that returns NaN when either operand is NaN.
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Maximum of three that returns NaN when any operand is NaN (one instruction).
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Order-preserving unsigned key of an fp32 score: larger score -> larger
// key; -0.0 and +0.0 share a key; NaN gets the smallest key of all.
__device__ __forceinline__ uint32_t order_key(float a) {
  if (a != a) return 0u;
  uint32_t u = __float_as_uint(a);
  if (a == 0.0f) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan over a group of NT threads (tid = index in the group);
// *total receives the sum.
template <int BAR, int NT>
__device__ __forceinline__ int block_excl_scan(int v, int tid, int *s_warp, int *total) {
  const int lane = tid & 31, w = tid >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[w] = x;
  csync<BAR, NT>();
  int before = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) {
    int t = s_warp[i];
    before += (i < w) ? t : 0;
    tot += t;
  }
  csync<BAR, NT>();
  *total = tot;
  return before + x - v;
}

// Counter increment with acquire-release semantics at GPU scope.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Scheduling tiles of a unit with N rows: kTileKeys-slot aligned tiles that
// cover the candidate slots [S, N - W) (N > B >= W + S).
__device__ __forceinline__ int unit_tiles(int N, int W, int S) {
  return (N - W - 1) / kTileKeys - S / kTileKeys + 1;
}

// Slot t of (sequence s, KV head h): element offset from the layer base.
__device__ __forceinline__ int64_t row_off(const CacheDev &c, int s, int h, int t) {
  if (c.layout == TRIA_LAYOUT_CONTIGUOUS)
    return (int64_t)s * c.s_seq + (int64_t)h * c.s_head + (int64_t)t * c.s_tok;
  const int blk = c.block_table[(int64_t)s * c.max_blocks + t / c.block_size];
  return (int64_t)blk * c.s_blk + (int64_t)(t % c.block_size) * c.s_tok + (int64_t)h * c.s_head;
}

// ---------------------------------------------------------------------------
// Radix top-K of one unit.  Digits of the order key, most significant first:
// bits [31:20] (12 bits), [19:8] (12 bits), [7:0] (8 bits).  After a digit
// is fixed, when the bin that holds the K-th largest key has at most
// kListCap members they are gathered into a shared list and the remaining
// digits are resolved there; otherwise the next digit is histogrammed over
// all candidates.  The emission pass then keeps every key above the
// threshold key T and the first `need` keys equal to T in slot order.
// All functions run on a group of NT threads; tid is the index in the group.
// ---------------------------------------------------------------------------
constexpr int kListCap = 2048;
constexpr int kHistBins = 4096;

struct TailScratch {          // 32 KB of shared memory
  uint32_t hist[kHistBins];
  uint2 list[kListCap];       // (key, candidate index)
};

struct SelScalars {
  int warp_tmp[8];
  uint32_t prefix;
  int remaining;
  int digit;
  int above;
  int bin_count;
  int list_n;
  float mean[TRIA_MAX_GROUP];
  float inv[TRIA_MAX_GROUP];
};

// Histogram increment in shared memory: one atomic per key (merging equal
// bins across a warp first with __match_any_sync measured slower: the
// unit tail took 191 instead of 157 us per Qwen3-32B 32K pass).
__device__ __forceinline__ void hist_add(uint32_t *hist, uint32_t bin, bool valid) {
  if (valid) atomicAdd(hist + bin, 1u);
}

template <int NT>
__device__ __forceinline__ void clear_words(uint32_t *w, int n, int tid) {
  for (int i = tid; i < n; i += NT) w[i] = 0u;
}

// Pick the bin holding the `remaining`-th largest key among nbins bins
// (digit at `shift`); updates prefix, remaining, bin_count.
template <int BAR, int NT, class Sc>
__device__ void pick_bin(const uint32_t *hist, int nbins, Sc &sc, int shift, int tid) {
  const int per = nbins / NT;  // bins per thread, descending
  int v = 0;
  for (int e = 0; e < per; ++e) v += (int)hist[nbins - 1 - (tid * per + e)];
  int total;
  const int excl = block_excl_scan<BAR, NT>(v, tid, sc.warp_tmp, &total);
  const int rem = sc.remaining;
  int cum = excl;
  for (int e = 0; e < per; ++e) {
    const int d = nbins - 1 - (tid * per + e);
    const int c = (int)hist[d];
    if (cum < rem && rem <= cum + c) {
      sc.digit = d;
      sc.above = cum;
      sc.bin_count = c;
    }
    cum += c;
  }
  csync<BAR, NT>();
  if (tid == 0) {
    sc.prefix |= (uint32_t)sc.digit << shift;
    sc.remaining = rem - sc.above;
  }
  csync<BAR, NT>();
}

__device__ __forceinline__ bool aligned16p(const void *p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// One histogram pass over agg for the keys matching (prefix, pmask).
template <int NT>
__device__ void hist_pass(const float *agg, int C, uint32_t pmask, uint32_t prefix, int shift,
                          uint32_t dmask, uint32_t *hist, int tid) {
  if (aligned16p(agg)) {
    const int C4 = C >> 2;
    const float4 *a4 = reinterpret_cast<const float4 *>(agg);
    for (int b = 0; b < C4; b += NT * 4) {
      float4 v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = b + e * NT + tid;
        v[e] = (i < C4) ? __ldcg(a4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool in = (b + e * NT + tid) < C4;
        const float x[4] = {v[e].x, v[e].y, v[e].z, v[e].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t k = order_key(x[q]);
          hist_add(hist, (k >> shift) & dmask, in && (k & pmask) == prefix);
        }
      }
    }
    for (int c = (C4 << 2) + tid; c < C; c += NT) {
      const uint32_t k = order_key(__ldcg(agg + c));
      if ((k & pmask) == prefix) atomicAdd(hist + ((k >> shift) & dmask), 1u);
    }
  } else {
    for (int c = tid; c < C; c += NT) {
      const uint32_t k = order_key(__ldcg(agg + c));
      if ((k & pmask) == prefix) atomicAdd(hist + ((k >> shift) & dmask), 1u);
    }
  }
}

// Gather (key, c) of the keys matching (prefix, pmask) into the list.
template <int NT>
__device__ void gather_pass(const float *agg, int C, uint32_t pmask, uint32_t prefix,
                            TailScratch &ts, SelScalars &sc, int tid) {
  const int lane = tid & 31;
  if (aligned16p(agg)) {
    // 8 candidates per thread per round (2 float4 loads in flight); the
    // list order does not matter
    const int C4 = C >> 2;
    const float4 *a4 = reinterpret_cast<const float4 *>(agg);
    for (int b = 0; b < C4 + 1; b += NT * 2) {
      float4 v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = b + e * NT + tid;
        v[e] = (i < C4) ? __ldcg(a4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = b + e * NT + tid;
        const float x[4] = {v[e].x, v[e].y, v[e].z, v[e].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          // candidates past the float4s (at most 3) ride on index C4
          const int c = (i < C4) ? 4 * i + q : (i == C4 ? 4 * C4 + q : C);
          const float xv = (i < C4) ? x[q] : (c < C ? __ldcg(agg + c) : 0.f);
          const uint32_t k = order_key(xv);
          const bool m = c < C && (k & pmask) == prefix;
          const uint32_t bal = __ballot_sync(kFull, m);
          int base = 0;
          if (lane == 0 && bal) base = atomicAdd(&sc.list_n, __popc(bal));
          base = __shfl_sync(kFull, base, 0);
          if (m) {
            const int idx = base + __popc(bal & ((1u << lane) - 1u));
            if (idx < kListCap) ts.list[idx] = make_uint2(k, (uint32_t)c);
          }
        }
      }
    }
    return;
  }
  for (int c0 = 0; c0 < C; c0 += NT * 4) {
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = c0 + e * NT + tid;
      x[e] = (c < C) ? __ldcg(agg + c) : 0.0f;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = c0 + e * NT + tid;
      const uint32_t k = order_key(x[e]);
      const bool m = (c < C) && (k & pmask) == prefix;
      const uint32_t bal = __ballot_sync(kFull, m);
      int base = 0;
      if (lane == 0 && bal) base = atomicAdd(&sc.list_n, __popc(bal));
      base = __shfl_sync(kFull, base, 0);
      if (m) {
        const int idx = base + __popc(bal & ((1u << lane) - 1u));
        if (idx < kListCap) ts.list[idx] = make_uint2(k, (uint32_t)c);
      }
    }
  }
}

// Selection of one unit from its C aggregated scores.  hist0_ready: the
// caller already holds the histogram of bits [31:20] of every key in ts.hist.
template <int BAR, int NT>
__device__ void select_unit(const float *agg, int C, int K, int N, int B, int W, int S,
                            int32_t *kept, TailScratch &ts, SelScalars &sc, bool hist0_ready,
                            int tid) {
  for (int j = tid; j < S; j += NT) kept[j] = j;
  for (int j = tid; j < W; j += NT) kept[B - W + j] = N - W + j;
  if (K <= 0) return;
  if (!hist0_ready) {
    clear_words<NT>(ts.hist, kHistBins, tid);
    csync<BAR, NT>();
    hist_pass<NT>(agg, C, 0u, 0u, 20, 0xfffu, ts.hist, tid);
    csync<BAR, NT>();
  }
  if (tid == 0) {
    sc.prefix = 0u;
    sc.remaining = K;
  }
  csync<BAR, NT>();
  pick_bin<BAR, NT>(ts.hist, kHistBins, sc, 20, tid);
  int level = 0;
  bool in_list = false;
  while (level < 2) {
    const int cur_shift = level == 0 ? 20 : 8;
    if (!in_list && sc.bin_count <= kListCap) {
      if (tid == 0) sc.list_n = 0;
      csync<BAR, NT>();
      gather_pass<NT>(agg, C, 0xffffffffu << cur_shift, sc.prefix, ts, sc, tid);
      csync<BAR, NT>();
      in_list = true;
    }
    ++level;
    const int sh = level == 1 ? 8 : 0;
    const int width = level == 1 ? 12 : 8;
    const uint32_t dmask = (1u << width) - 1u;
    const int nb = 1 << width;
    clear_words<NT>(ts.hist, nb, tid);
    csync<BAR, NT>();
    const uint32_t pm = 0xffffffffu << (sh + width);
    const uint32_t pre = sc.prefix;
    if (in_list) {
      const int n = sc.list_n;
      for (int i = tid; i < n; i += NT) {
        const uint32_t k = ts.list[i].x;
        if ((k & pm) == pre) atomicAdd(ts.hist + ((k >> sh) & dmask), 1u);
      }
    } else {
      hist_pass<NT>(agg, C, pm, pre, sh, dmask, ts.hist, tid);
    }
    csync<BAR, NT>();
    pick_bin<BAR, NT>(ts.hist, nb, sc, sh, tid);
  }
  const uint32_t T = sc.prefix;
  const int need_ties = sc.remaining;  // keys equal to T still to take (>= 1)

  // emission in slot order: 8 consecutive candidates per thread per chunk,
  // the next chunk's loads issued before the current chunk is scanned
  constexpr int E = 8;
  const bool vec = aligned16p(agg);
  auto load8 = [&](int base, uint32_t (&k)[E]) {
    const int c = base + tid * E;
    if (vec && c + E <= C) {
      const float4 a = __ldcg(reinterpret_cast<const float4 *>(agg + c));
      const float4 b = __ldcg(reinterpret_cast<const float4 *>(agg + c + 4));
      k[0] = order_key(a.x); k[1] = order_key(a.y); k[2] = order_key(a.z); k[3] = order_key(a.w);
      k[4] = order_key(b.x); k[5] = order_key(b.y); k[6] = order_key(b.z); k[7] = order_key(b.w);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) k[e] = (c + e < C) ? order_key(__ldcg(agg + c + e)) : 0u;
    }
  };
  int run_ties = 0, run_keep = 0;
  uint32_t cur[E], nxt[E];
  load8(0, cur);
  for (int base = 0; base < C && run_keep < K; base += NT * E) {
    if (base + NT * E < C) load8(base + NT * E, nxt);
    int nt = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) nt += (base + tid * E + e < C && cur[e] == T) ? 1 : 0;
    int tot_t;
    const int ex_t = block_excl_scan<BAR, NT>(nt, tid, sc.warp_tmp, &tot_t);
    int tie = run_ties + ex_t, nk = 0;
    uint32_t keepm = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      bool k = false;
      if (base + tid * E + e < C) {
        if (cur[e] > T) {
          k = true;
        } else if (cur[e] == T) {
          k = tie < need_ties;
          ++tie;
        }
      }
      keepm |= (k ? 1u : 0u) << e;
      nk += k ? 1 : 0;
    }
    int tot_k;
    int pos = run_keep + block_excl_scan<BAR, NT>(nk, tid, sc.warp_tmp, &tot_k);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if (((keepm >> e) & 1u) && pos < K) kept[S + pos] = S + base + tid * E + e;
      pos += (keepm >> e) & 1u;
    }
    run_ties += tot_t;
    run_keep += tot_k;
#pragma unroll
    for (int e = 0; e < E; ++e) cur[e] = nxt[e];
  }
}

// ---------------------------------------------------------------------------
// Normalize-then-max of a range of candidates of one unit.
// unit_norm: population mean and 1/(std + eps) of every head over the C
// candidates, from the fp64 moment partials of each (item, 32-row group).
// agg_range: agg[c] = max_g (S_g[c] - mean_g) * inv_g for c in [c0, c1), with
// the histogram of the top 12 key bits added into hist when it is non-null.
// ---------------------------------------------------------------------------
template <int G, int BAR, int NT, class Sc>
__device__ void unit_norm(const double *mom_unit, int ntiles, int C, int tid, Sc &sc) {
  // head g is summed by warp g % (NT / 32): lane l adds the head's partials
  // l, l + 32, ... in order, then a butterfly over the lanes (every lane ends
  // with the same sums).  The order depends on neither NT nor the caller,
  // so every kernel that normalizes a unit gets bit-identical mean and std.
  // No barrier inside: the caller syncs before reading sc.mean / sc.inv.
  static_assert(NT % 32 == 0, "whole warps");
  constexpr int NW = NT / 32;
  const int lane = tid & 31, w = tid >> 5;
  const int n = ntiles * kRowGroups;
  const double2 *m2 = reinterpret_cast<const double2 *>(mom_unit);
  for (int g = w; g < G; g += NW) {
    double s1 = 0.0, s2 = 0.0;
    int i = lane;
    // eight loads in flight, added in the same order as one at a time
    for (; i + 7 * 32 < n; i += 8 * 32) {
      double2 v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = __ldcg(m2 + (int64_t)(i + 32 * e) * G + g);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        s1 += v[e].x;
        s2 += v[e].y;
      }
    }
    for (; i < n; i += 32) {
      const double2 v = __ldcg(m2 + (int64_t)i * G + g);
      s1 += v.x;
      s2 += v.y;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      s1 += __shfl_xor_sync(kFull, s1, o);
      s2 += __shfl_xor_sync(kFull, s2, o);
    }
    if (lane == 0) {
      const double mean = s1 / C;
      double var = s2 / C - mean * mean;
      var = var > 0.0 ? var : 0.0;
      sc.mean[g] = (float)mean;
      sc.inv[g] = (float)(1.0 / (sqrt(var) + 1e-6));
    }
  }
}

template <int G, int NT>
__device__ void agg_range(const float *__restrict__ raw, float *agg, int c0, int c1,
                          const float *s_mean, const float *s_inv, uint32_t *hist, int tid) {
  float mean[G], inv[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    mean[g] = s_mean[g];
    inv[g] = s_inv[g];
  }
  auto agg_of = [&](const float *sv) {
    float a = 0.0f;
    bool nan = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float z = __fmul_rn(__fsub_rn(sv[g], mean[g]), inv[g]);
      a = (g == 0) ? z : fmaxf(a, z);
      nan |= (z != z);
    }
    return nan ? __int_as_float(0x7fc00000) : a;
  };
  // E consecutive candidates per thread per step: E*G/4 float4 loads in
  // flight (through L1: the two halves of a 32-byte sector hit it once)
  constexpr int E = (G >= 8) ? 16 / G * 2 : 8;
  int c = c0;
  if (aligned16p(raw + (int64_t)c0 * G)) {
    for (; c + NT * E <= c1; c += NT * E) {
      const int cc = c + tid * E;
      float v[E * G];
      const float4 *src = reinterpret_cast<const float4 *>(raw + (int64_t)cc * G);
#pragma unroll
      for (int i = 0; i < (E * G) / 4; ++i) {
        const float4 x = __ldg(src + i);
        v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
      }
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float a = agg_of(v + e * G);
        agg[cc + e] = a;
        if (hist != nullptr) hist_add(hist, order_key(a) >> 20, true);
      }
    }
  }
  for (int cc = c + tid; cc < c1; cc += NT) {
    float v[G];
#pragma unroll
    for (int g = 0; g < G; ++g) v[g] = __ldg(raw + (int64_t)cc * G + g);
    const float a = agg_of(v);
    agg[cc] = a;
    if (hist != nullptr) atomicAdd(hist + (order_key(a) >> 20), 1u);
  }
}

// Warp-wide inclusive scan of v (lane order).
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

}  // namespace dev
}  // namespace tria
