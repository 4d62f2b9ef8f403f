// Unit tail of the compression pass: normalize-then-max and top-K selection
// with the candidates' agg keys in shared memory, one thread-block cluster of
// 1 to 8 blocks per unit (sequence, layer, KV head).
//
// Per unit (academ.us article 2607.13051, Eq. 8 and sec. 4; ghidav.me
// "TriAttention, or: what a rotating query already knows", "The Method"):
//   agg(k) = max_g (S~_g(k) - mean_g) / (std_g + 1e-6)
// over the G query heads of the KV head (population mean and std over the
// unit's candidates), then the K = B - W - S candidates of largest agg are
// kept, ties to the lower slot, and the kept list is written in ascending slot
// order: the S sinks, the kept candidates, the W window slots.
//
// Layout.  Block r of a unit's cluster takes the candidate slice
// [r P, r P + P) (P a multiple of 128); thread t of a block owns the KPT
// consecutive candidates [t KPT, (t + 1) KPT) of the slice.  Its keys sit in
// shared memory in 16-byte chunks rotated per thread (chunk q of thread t at
// chunk (q + t NQ / 8) mod NQ of the thread's row, NQ = KPT / 4), so that the
// eight threads of a quarter warp read eight different bank groups when they
// walk their chunks in slot order.
//
// Steps.  One coalesced pass over the slice's raw scores [P][G] writes the
// order keys (order_key of agg; NaN lowest) and the histogram of their top 12
// bits.  The radix selection then takes three digits (12, 12, 8 bits): each
// digit's histogram is summed over the cluster through distributed shared
// memory, and every block picks the same bin (the K-th largest key's).  Each
// further digit is one pass of every thread over its own keys.  Finally
// every thread counts its keys above the threshold key T and equal to it,
// one block scan plus the cluster's block totals give its first position in
// the kept list and its first tie rank, and it writes its kept slots in order.
#include <cooperative_groups.h>

#include "tria_device.cuh"

namespace tria {
namespace {

namespace cg = cooperative_groups;
using namespace dev;

constexpr int kTailThreads = 1024;
constexpr int kTailWarps = kTailThreads / 32;

struct alignas(16) TailShared {
  float mean[TRIA_MAX_GROUP];
  float inv[TRIA_MAX_GROUP];
  uint32_t wsum[kTailWarps];  // per-warp totals / exclusive prefixes of the block scans
  uint32_t prefix;       // digits of T fixed so far
  int remaining;         // rank of T among the keys matching prefix
  int cta_gt, cta_eq;    // this block's keys > T and == T (read by the cluster)
  int pre_gt, pre_eq;    // the same summed over the cluster's lower blocks
  uint32_t total;        // block sum of the last scan
  int pad[1];
};
static_assert(sizeof(TailShared) % 16 == 0, "the histogram after TailShared stays 16-byte aligned");

// Word offset of chunk q (4 keys) of thread t.
template <int KPT>
__device__ __forceinline__ int chunk_word(int t, int q) {
  constexpr int NQ = KPT / 4;
  return t * KPT + 4 * ((q + (t * NQ) / 8) % NQ);
}

// Shared-memory word of local candidate c.
template <int KPT>
__device__ __forceinline__ int key_word(int c) {
  return chunk_word<KPT>(c / KPT, (c % KPT) >> 2) + (c & 3);
}

// Eight consecutive floats from a 32-byte-aligned address with one 256-bit
// streaming load (read once: evict first).
__device__ __forceinline__ void ld_cs_v8(const float *p, float (&x)[8]) {
  asm volatile("ld.global.cs.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=f"(x[0]), "=f"(x[1]), "=f"(x[2]), "=f"(x[3]), "=f"(x[4]), "=f"(x[5]),
                 "=f"(x[6]), "=f"(x[7])
               : "l"(p));
}

// Raw-score pass over a slice of P candidates: keys (order keys of agg) into
// the rotated layout and the histogram of their top 12 bits.
template <int G, int KPT>
__device__ void slice_keys(const float *raw, int P, const float *s_mean, const float *s_inv,
                           uint32_t *keys, uint32_t *hist, int tid) {
  constexpr int NT = kTailThreads;
  constexpr int U = 8;  // float4 loads in flight per thread
  const float4 *src = reinterpret_cast<const float4 *>(raw);
  if constexpr (G >= 8) {
    // LPC lanes per candidate, each loading 8 of its G heads with one
    // 256-bit load (the slice starts on a 32-byte boundary: checked at launch)
    constexpr int LPC = G / 8, U8 = 4;
    const int h0 = (tid % LPC) * 8;
    float m[8], iv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      m[k] = s_mean[h0 + k];
      iv[k] = s_inv[h0 + k];
    }
    const int n8 = P * LPC;
    for (int j0 = 0; j0 < n8; j0 += NT * U8) {
      float x[U8][8];
#pragma unroll
      for (int u = 0; u < U8; ++u) {
        const int j = j0 + u * NT + tid;
        if (j < n8) {
          ld_cs_v8(raw + (int64_t)j * 8, x[u]);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) x[u][k] = 0.0f;
        }
      }
#pragma unroll
      for (int u = 0; u < U8; ++u) {
        const int j = j0 + u * NT + tid;
        float z[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) z[k] = __fmul_rn(__fsub_rn(x[u][k], m[k]), iv[k]);
        // NaN in any head makes agg NaN, whose key is 0
        float a = max3_nan(max3_nan(z[0], z[1], z[2]), max3_nan(z[3], z[4], z[5]), max_nan(z[6], z[7]));
#pragma unroll
        for (int o = 1; o < LPC; o <<= 1) a = max_nan(a, __shfl_xor_sync(kFull, a, o));
        const uint32_t k = order_key(a);
        const bool lead = (j < n8) && (tid % LPC) == 0;
        if (lead) keys[key_word<KPT>(j / LPC)] = k;
        hist_add(hist, k >> 20, lead);
      }
    }
  } else if constexpr (G >= 4) {
    // LPC lanes per candidate, each with 4 of its G heads
    constexpr int LPC = G / 4;
    const int h0 = (tid % LPC) * 4;
    float m[4], iv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      m[k] = s_mean[h0 + k];
      iv[k] = s_inv[h0 + k];
    }
    const int n4 = P * LPC;
    for (int j0 = 0; j0 < n4; j0 += NT * U) {
      float4 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u * NT + tid;
        x[u] = (j < n4) ? __ldcs(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u * NT + tid;
        const float z0 = __fmul_rn(__fsub_rn(x[u].x, m[0]), iv[0]);
        const float z1 = __fmul_rn(__fsub_rn(x[u].y, m[1]), iv[1]);
        const float z2 = __fmul_rn(__fsub_rn(x[u].z, m[2]), iv[2]);
        const float z3 = __fmul_rn(__fsub_rn(x[u].w, m[3]), iv[3]);
        // NaN in any head makes agg NaN, whose key is 0
        float a = max_nan(max_nan(z0, z1), max_nan(z2, z3));
#pragma unroll
        for (int o = 1; o < LPC; o <<= 1) a = max_nan(a, __shfl_xor_sync(kFull, a, o));
        const uint32_t k = order_key(a);
        const bool lead = (j < n4) && (tid % LPC) == 0;
        if (lead) keys[key_word<KPT>(j / LPC)] = k;
        hist_add(hist, k >> 20, lead);
      }
    }
  } else {
    // a float4 holds CPF = 4 / G candidates
    constexpr int CPF = 4 / G;
    float m[G], iv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = s_mean[g];
      iv[g] = s_inv[g];
    }
    const int n4 = (P + CPF - 1) / CPF;
    for (int j0 = 0; j0 < n4; j0 += NT * U) {
      float4 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u * NT + tid;
        x[u] = (j < n4) ? __ldcs(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u * NT + tid;
        const float v[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
        for (int e = 0; e < CPF; ++e) {
          const int c = j * CPF + e;
          float a = 0.0f;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float z = __fmul_rn(__fsub_rn(v[e * G + g], m[g]), iv[g]);
            a = (g == 0) ? z : max_nan(a, z);
          }
          const uint32_t k = order_key(a);
          const bool in = (j < n4) && c < P;
          if (in) keys[key_word<KPT>(c)] = k;
          hist_add(hist, k >> 20, in);
        }
      }
    }
  }
}

// Block-wide exclusive scan (warp scans, then warp 0 over the warp totals) of
// non-negative counts, in unsigned 32-bit arithmetic; returns this thread's
// exclusive prefix, sc.total the block's sum.  Starts and ends with a
// barrier-separated use of sc.wsum.
__device__ __forceinline__ uint32_t tail_excl_scan_u(uint32_t v, TailShared &sc, int tid) {
  const int lane = tid & 31, warp = tid >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sc.wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = sc.wsum[lane];
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(kFull, xi, o);
      if (lane >= o) xi += y;
    }
    sc.wsum[lane] = xi - x;  // each lane reads and writes its own entry
    if (lane == 31) sc.total = xi;
  }
  __syncthreads();
  return sc.wsum[warp] + incl - v;
}

// The same for int counts (a block's sum stays below 2^31).
__device__ __forceinline__ int tail_excl_scan(int v, TailShared &sc, int tid) {
  return (int)tail_excl_scan_u((uint32_t)v, sc, tid);
}

// The bin holding the sc.remaining-th largest key among hist[0, nbins)
// (higher bins hold larger keys): sets sc.prefix |= bin << shift and
// sc.remaining -= the keys in higher bins.  1 <= sc.remaining <= the
// histogram's total on entry.
__device__ void pick_bin_desc(const uint32_t *hist, int nbins, TailShared &sc, int shift, int tid) {
  constexpr int NT = kTailThreads;
  const int per = nbins >= NT ? nbins / NT : 1;
  const int first = tid * per;  // positions in descending bin order
  int v = 0;
  if (first < nbins)
    for (int e = 0; e < per; ++e) v += (int)hist[nbins - 1 - (first + e)];
  const int rem = sc.remaining;  // read by every thread before the scan's barriers
  int cum = tail_excl_scan(v, sc, tid);
  if (v > 0 && cum < rem && rem <= cum + v) {
    // the one thread whose bins hold the rank: it alone updates the state
    for (int e = 0; e < per; ++e) {
      const int d = nbins - 1 - (first + e);
      const int c = (int)hist[d];
      if (cum < rem && rem <= cum + c) {
        sc.prefix |= (uint32_t)d << shift;
        sc.remaining = rem - cum;
      }
      cum += c;
    }
  }
  __syncthreads();
}

// Sum hist[0, nbins) over the cluster's blocks (every block ends with the
// sums); a plain barrier when the unit has one block.
__device__ void cluster_sum_hist(uint32_t *hist, int nbins, int cs, int tid) {
  constexpr int NT = kTailThreads, E = kHistBins / NT;
  if (cs == 1) {
    __syncthreads();
    return;
  }
  cg::cluster_group cl = cg::this_cluster();
  cl.sync();  // every block's histogram is complete
  uint32_t acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0u;
  for (int r = 0; r < cs; ++r) {
    const uint32_t *h = cl.map_shared_rank(hist, r);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int b = tid + e * NT;
      if (b < nbins) acc[e] += h[b];
    }
  }
  cl.sync();  // every block has read every histogram
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int b = tid + e * NT;
    if (b < nbins) hist[b] = acc[e];
  }
  __syncthreads();
}

template <int G, int KPT>
__global__ void __launch_bounds__(kTailThreads, 1) cluster_tail_kernel(const __grid_constant__ TailParams p) {
  constexpr int NT = kTailThreads, NQ = KPT / 4;
  extern __shared__ __align__(16) uint8_t smem_tail[];
  TailShared &sc = *reinterpret_cast<TailShared *>(smem_tail);
  uint32_t *hist = reinterpret_cast<uint32_t *>(smem_tail + sizeof(TailShared));
  uint32_t *keys = hist + kHistBins;
  const Geom &geo = p.geo;
  const int t = threadIdx.x;
  const int cs = p.cluster;
  // the last units first: the scoring kernel claims units in ascending
  // order, so the raw scores it wrote last may still be in L2 (154.4 against
  // 156.8 us per Qwen3-32B 32K pass)
  const int64_t u = p.geo.n_units - 1 - blockIdx.x / cs;
  const int rank = (int)(blockIdx.x % cs);  // clusters are cs consecutive blocks along x
  const int s = (int)(u / ((int64_t)geo.nl * geo.hkv));
  const int lrel = (int)((u / geo.hkv) % geo.nl);
  const int N = unit_len(geo, s, lrel);
  // invalid lengths and units left as they are: the coefficient kernel wrote
  // their kept rows and flagged the former (the same for every block of the
  // cluster, so no cluster barrier is left waiting)
  if (!compresses(geo, N, lrel)) return;
  const int W = geo.window, S = geo.sinks;
  const int B = geo.lbudget[lrel];
  const int K = B - W - S;
  const int C = N - W - S;
  int32_t *kept = p.kept + u * geo.budget;
  if (rank == 0) {
    for (int j = t; j < S; j += NT) kept[j] = j;
    for (int j = t; j < W; j += NT) kept[B - W + j] = N - W + j;
    for (int j = B + t; j < geo.budget; j += NT) kept[j] = -1;
  }
  if (K <= 0) return;
  const int c0 = rank * p.slice;
  const int P = max(0, min(C - c0, p.slice));
  unit_norm<G, 0, NT>(p.moments + u * geo.tiles_max * kRowGroups * G * 2,
                      unit_tiles(N, W, S), C, t, sc);
  clear_words<NT>(hist, kHistBins, t);
  if (t == 0) {
    sc.prefix = 0u;
    sc.remaining = K;
  }
  __syncthreads();
  const float *raw = p.raw + u * p.raw_stride + (int64_t)c0 * G;
  slice_keys<G, KPT>(raw, P, sc.mean, sc.inv, keys, hist, t);
  if (p.discard_raw) {
    // the slice starts and ends on 128-byte lines (P is a multiple of 128)
    __syncthreads();
    const int64_t lines = ((int64_t)P * G * 4 + 127) / 128;
    for (int64_t i = t; i < lines; i += NT) discard_line(raw + i * 32);
  }
  // this thread's keys: local candidates [t KPT, t KPT + KPT) ∩ [0, P)
  const int cb = t * KPT;
  const int nmine = max(0, min(P - cb, KPT));
  // digit 1: bits [31:20]
  cluster_sum_hist(hist, kHistBins, cs, t);
  pick_bin_desc(hist, kHistBins, sc, 20, t);
  // digit 2: bits [19:8] of the keys in the chosen bin
  clear_words<NT>(hist, kHistBins, t);
  __syncthreads();
  {
    const uint32_t d1 = sc.prefix >> 20;
    auto keys_q1 = [&](int q) {
      const uint4 k4 = *reinterpret_cast<const uint4 *>(keys + chunk_word<KPT>(t, q));
      const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (4 * q + i < nmine && (kk[i] >> 20) == d1) atomicAdd(hist + ((kk[i] >> 8) & 0xfffu), 1u);
    };
    if (nmine == KPT) {
#pragma unroll
      for (int q = 0; q < NQ; ++q) keys_q1(q);
    } else {
      for (int q = 0; 4 * q < nmine; ++q) keys_q1(q);
    }
  }
  cluster_sum_hist(hist, kHistBins, cs, t);
  pick_bin_desc(hist, kHistBins, sc, 8, t);
  // digit 3: bits [7:0]
  clear_words<NT>(hist, 256, t);
  __syncthreads();
  {
    const uint32_t d12 = sc.prefix >> 8;
    auto keys_q2 = [&](int q) {
      const uint4 k4 = *reinterpret_cast<const uint4 *>(keys + chunk_word<KPT>(t, q));
      const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (4 * q + i < nmine && (kk[i] >> 8) == d12) atomicAdd(hist + (kk[i] & 0xffu), 1u);
    };
    if (nmine == KPT) {
#pragma unroll
      for (int q = 0; q < NQ; ++q) keys_q2(q);
    } else {
      for (int q = 0; 4 * q < nmine; ++q) keys_q2(q);
    }
  }
  cluster_sum_hist(hist, 256, cs, t);
  pick_bin_desc(hist, 256, sc, 0, t);
  const uint32_t T = sc.prefix;
  const int need = sc.remaining;  // keys equal to T to keep, lowest slots first (>= 1)
  // this thread's keys above / equal to T; block prefixes (counts < 2^16 per block)
  int gt = 0, eq = 0;
  auto keys_q3 = [&](int q) {
    const uint4 k4 = *reinterpret_cast<const uint4 *>(keys + chunk_word<KPT>(t, q));
    const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool valid = 4 * q + i < nmine;
      gt += (valid && kk[i] > T) ? 1 : 0;
      eq += (valid && kk[i] == T) ? 1 : 0;
    }
  };
  if (nmine == KPT) {
#pragma unroll
    for (int q = 0; q < NQ; ++q) keys_q3(q);
  } else {
    for (int q = 0; 4 * q < nmine; ++q) keys_q3(q);
  }
  // gt and eq packed in the low and high halves of one unsigned word: a
  // block holds at most kTailThreads x 44 = 45056 < 2^16 candidates, so
  // neither half overflows (a signed word would, past 32767 ties)
  static_assert(kTailThreads * 44 < (1 << 16), "packed block counts");
  const uint32_t ex = tail_excl_scan_u((uint32_t)gt | ((uint32_t)eq << 16), sc, t);
  if (t == 0) {
    sc.cta_gt = (int)(sc.total & 0xffffu);
    sc.cta_eq = (int)(sc.total >> 16);
    sc.pre_gt = 0;
    sc.pre_eq = 0;
  }
  if (cs > 1) {
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();  // every block's totals are published
    if (t == 0) {
      int pg = 0, pe = 0;
      for (int r = 0; r < rank; ++r) {
        const TailShared *o = cl.map_shared_rank(&sc, r);
        pg += o->cta_gt;
        pe += o->cta_eq;
      }
      sc.pre_gt = pg;
      sc.pre_eq = pe;
    }
    cl.sync();  // no block reads another's shared memory after this
  } else {
    __syncthreads();
  }
  // emission in slot order
  int eqr = sc.pre_eq + (int)(ex >> 16);
  int pos = sc.pre_gt + (int)(ex & 0xffffu) + min(eqr, need);
  const int slot0 = S + c0 + cb;
  auto keys_q4 = [&](int q) {
    const uint4 k4 = *reinterpret_cast<const uint4 *>(keys + chunk_word<KPT>(t, q));
    const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = 4 * q + i;
      if (c < nmine) {
        bool keep = kk[i] > T;
        if (kk[i] == T) {
          keep = eqr < need;
          ++eqr;
        }
        if (keep) {
          if (pos < K) kept[S + pos] = slot0 + c;
          ++pos;
        }
      }
    }
  };
  if (nmine == KPT) {
#pragma unroll
    for (int q = 0; q < NQ; ++q) keys_q4(q);
  } else {
    for (int q = 0; 4 * q < nmine; ++q) keys_q4(q);
  }
}

// Candidates per thread for a slice of P candidates (0: too many).
int tail_kpt(int P) {
  if (P <= kTailThreads * 8) return 8;
  if (P <= kTailThreads * 16) return 16;
  if (P <= kTailThreads * 32) return 32;
  if (P <= kTailThreads * 44) return 44;
  return 0;
}

size_t tail_smem_bytes(int kpt) {
  return sizeof(TailShared) + (size_t)kHistBins * 4 + (size_t)kTailThreads * kpt * 4;
}

template <int G, int KPT>
cudaError_t launch_ct(TailParams p, size_t smem, cudaStream_t st) {
  auto kern = cluster_tail_kernel<G, KPT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.geo.n_units * p.cluster), 1, 1);
  cfg.blockDim = dim3(kTailThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int G>
cudaError_t launch_ct_g(const TailParams &p, int kpt, size_t smem, cudaStream_t st) {
  switch (kpt) {
    case 8: return launch_ct<G, 8>(p, smem, st);
    case 16: return launch_ct<G, 16>(p, smem, st);
    case 32: return launch_ct<G, 32>(p, smem, st);
    case 44: return launch_ct<G, 44>(p, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// The smallest cluster (1 to 8 blocks) whose slices of at most
// ceil(c_max / cs) candidates, rounded up to 128, fit a block's key area.
bool tail_shape(const Geom &g, int *cs, int *slice, int *kpt) {
  for (int c = 1; c <= kMaxTailCluster; ++c) {
    const int sl = ((g.c_max + c - 1) / c + 127) / 128 * 128;
    const int k = tail_kpt(sl);
    if (k != 0 && tail_smem_bytes(k) <= kMaxDynSmem) {
      *cs = c;
      *slice = sl;
      *kpt = k;
      return true;
    }
  }
  return false;
}

bool unit_tail_fits(const Geom &g) {
  int cs, sl, k;
  return tail_shape(g, &cs, &sl, &k);
}

cudaError_t launch_unit_tail(const TailParams &p0, cudaStream_t st) {
  TailParams p = p0;
  // G >= 8 reads a candidate's heads in 32-byte pieces: the raw scores of
  // every unit start on a 32-byte boundary (workspace layout)
  if (p.geo.g >= 8 && ((reinterpret_cast<uintptr_t>(p.raw) & 31u) != 0 || (p.raw_stride & 7) != 0))
    return cudaErrorInvalidValue;
  int kpt = 0;
  if (!tail_shape(p.geo, &p.cluster, &p.slice, &kpt)) return cudaErrorInvalidValue;
  const size_t smem = tail_smem_bytes(kpt);
  switch (p.geo.g) {
    case 1: return launch_ct_g<1>(p, kpt, smem, st);
    case 2: return launch_ct_g<2>(p, kpt, smem, st);
    case 4: return launch_ct_g<4>(p, kpt, smem, st);
    case 8: return launch_ct_g<8>(p, kpt, smem, st);
    case 16: return launch_ct_g<16>(p, kpt, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tria
