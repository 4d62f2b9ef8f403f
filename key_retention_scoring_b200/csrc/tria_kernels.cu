// Kernels of the TriAttention compression pass for sm_100a.
//
//   coef_kernel     per unit: the per-pass scoring coefficients
//                   c_f = mu'_f e^{i omega_f p_q} (fp64 -> fp32) and w_f as a
//                   bf16 hi/lo tensor-core operand; resets the scheduling
//                   counters; lays out the work items of every sequence.
//   (the scoring kernel is in tria_score_tc.cu)
//   tail_kernel     blocks over (unit, candidate chunk): normalize-then-max,
//                   histogram of the agg keys, selection by the last block.
//   select_kernel   one CTA per unit: radix top-K of agg + ascending kept list.
//   (the cluster unit tail of the pass is in tria_tail.cu)
//   (the compaction kernel is in tria_compact.cu)
//
// Sources: academ.us article 2607.13051 (Eqs. 2, 3, 4, 6, 7 and sec. 4),
// ghidav.me "TriAttention, or: what a rotating query already knows" ("The
// Method"), GitHub issue #10 of the llama.cpp TurboQuant HIP fork (RoPE
// pairing, window/sink conventions).
#include "tria_device.cuh"

namespace tria {
namespace {

using namespace dev;
constexpr int kThreads = kSelThreads;

// ---------------------------------------------------------------------------
// coef_kernel: one block of 256 threads per unit (sequence, layer, KV head).
//   c_gf = mu'_gf e^{i omega_f p_q} (fp64, then fp32) for the G query heads,
//   then the bf16 coefficient tile of the scoring contraction ([ncol][256]:
//   row 2g holds the hi parts, row 2g+1 the lo parts (x - hi) of head g's
//   coefficients), stored as the scoring kernel's shared-memory image: four
//   64-wide K blocks of ncol rows x 128 bytes, 16-byte chunks swizzled by the
//   row (chunk ^ (row & 7)), the 128-byte-swizzle K-major operand layout:
//     k in [0,128)   the key-dimension coefficients v (NEOX: v[f] = Re c_f,
//                    v[64+f] = Im c_f; interleaved: v[2f] = Re c_f, v[2f+1] = Im c_f)
//     k in [128,192) w_f = E|q_f| - |E q_f|      (multiplies |k_f| hi part)
//     k in [192,256) w_f in the hi row, 0 in the lo row (multiplies |k_f| lo part)
//   Block 0 also resets the item counter and lays out the work items.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint16_t bf16_rn_bits(float x) {
  uint32_t u = __float_as_uint(x);
  if (x != x) return 0x7FC0u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// e^{i omega_f p} for a query position p (fp64).
__device__ __forceinline__ double2 rot_at(const CoefParams &p, int f, int64_t pos) {
  double sn, cs;
  sincos(p.omega[f] * (double)pos, &sn, &cs);
  return make_double2(cs, sn);
}

__global__ void __launch_bounds__(kThreads) coef_kernel(const __grid_constant__ CoefParams p) {
  const Geom &g = p.geo;
  const int t = threadIdx.x;
  const int64_t u = blockIdx.x;
  const int h = (int)(u % g.hkv);
  const int lrel = (int)((u / g.hkv) % g.nl);
  const int s = (int)(u / ((int64_t)g.hkv * g.nl));
  const int l = g.layer0 + lrel;
  const int N = unit_len(g, s, lrel);
  const bool bad = !len_valid(g, N);
  const bool comp = compresses(g, N, lrel);
  __shared__ double2 rot[kBands];
  __shared__ float cf[TRIA_MAX_GROUP][3 * kBands];
  __shared__ int s_part[kThreads];

  // scheduling items per 1024-slot range of a (sequence, layer): one per KV
  // head, or one for all heads when the paged tiles hold every head
  const int ipu = g.grouped ? 1 : g.hkv;
  if (u == 0) {
    if (t == 0) *p.item_counter = 0u;
    if (!g.per_layer) {
      // one length per sequence: items per sequence, prefix over sequences
      // (n_seq <= 1024: <= 4 per thread)
      const int per = (g.n_seq + kThreads - 1) / kThreads;
      int local = 0;
      for (int i = 0; i < per; ++i) {
        const int sq = t * per + i;
        if (sq < g.n_seq) {
          const int n = unit_len(g, sq, 0);
          if (compresses(g, n, 0)) local += unit_tiles(n, g.window, g.sinks) * g.nl * ipu;
        }
      }
      int total;
      int run = block_excl_scan<0, kThreads>(local, t, s_part, &total);
      for (int i = 0; i < per; ++i) {
        const int sq = t * per + i;
        if (sq < g.n_seq) {
          p.seq_items[sq] = run;
          const int n = unit_len(g, sq, 0);
          if (compresses(g, n, 0)) run += unit_tiles(n, g.window, g.sinks) * g.nl * ipu;
        }
      }
      if (t == 0) p.seq_items[g.n_seq] = total;
    } else {
      // a length per (sequence, layer): items per row (s, lrel) = hkv x tiles
      // of the row's units; prefix over the rows, and over the sequences
      const int rows = g.n_seq * g.nl;
      const int per = (rows + kThreads - 1) / kThreads;
      auto row_n = [&](int r) {
        const int n = unit_len(g, r / g.nl, r % g.nl);
        return compresses(g, n, r % g.nl) ? unit_tiles(n, g.window, g.sinks) * ipu : 0;
      };
      int local = 0;
      for (int i = 0; i < per; ++i) {
        const int r = t * per + i;
        if (r < rows) local += row_n(r);
      }
      int total;
      int run = block_excl_scan<0, kThreads>(local, t, s_part, &total);
      for (int i = 0; i < per; ++i) {
        const int r = t * per + i;
        if (r < rows) {
          p.row_items[r] = run;
          if (r % g.nl == 0) p.seq_items[r / g.nl] = run;
          run += row_n(r);
        }
      }
      if (t == 0) {
        p.row_items[rows] = total;
        p.seq_items[g.n_seq] = total;
      }
    }
  }
  if (t == 0) {
    p.unit_done[u] = 0u;
    if (bad && h == 0 && (lrel == 0 || g.per_layer)) atomicOr(p.status, 1);
  }
  if (p.hist != nullptr)
    for (int j = t; j < kAggHistBins; j += kThreads) p.hist[u * kAggHistBins + j] = 0u;
  if (p.kept != nullptr && !comp) {
    int32_t *kr = p.kept + u * g.budget;
    for (int j = t; j < g.budget; j += kThreads) kr[j] = (!bad && j < N) ? j : -1;
  }
  if (!comp) return;

  if (g.mode == TRIA_OFFSET_MAX) {
    // max over the offsets: one coefficient vector per (head, offset delta_j)
    // with the unfolded center, c_gfj = E[q_gf] mask_f e^{i omega_f (p_q + delta_j)};
    // e^{i omega_f (p_q + 2^j)} = e^{i omega_f p_q} e^{i omega_f 2^j}, the
    // second factor from the table built with the statistics.  Band f sits
    // at f + f/8 in the shared tables so that the eight bands 8 apart that a
    // warp reads together fall in different banks.
    __shared__ double2 rotj[kMaxOffsets][kBands + kBands / 8];
    __shared__ double2 mu_s[8][kBands + kBands / 8];  // the form takes G <= 8
    const int nd = g.n_off;
    if (t < kBands) rot[t] = rot_at(p, t, p.query_pos[s]);
    // the unit's E[q_g] mask per head and band (read 17 x 2 times per value below)
    for (int i = t; i < g.g * kBands; i += kThreads) {
      const int f = i % kBands;
      mu_s[i / kBands][f + (f >> 3)] = p.mu_raw[((int64_t)l * g.hq + h * g.g) * kBands + i];
    }
    __syncthreads();
    for (int i = t; i < kBands * nd; i += kThreads) {
      const int f = i % kBands, j = i / kBands;
      const double2 a = rot[f], b = p.rot_off[f * kMaxOffsets + j];
      rotj[j][f + (f >> 3)] = make_double2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
    }
    __syncthreads();
    unsigned char *dst = reinterpret_cast<unsigned char *>(p.btile) + u * (int64_t)g.b_bytes;
    // trig rows n = gg nd + j over the 128 key dims: the hi parts in two
    // 64-wide blocks, then the lo parts in two more (each value computed once)
    for (int i = t; i < g.ncol_t * 16; i += kThreads) {
      const int n = i >> 4, ch = i & 15, kb = ch >> 3, c8 = ch & 7;
      const int gg = n / nd, j = n % nd;
      uint32_t whi[4], wlo[4];
      for (int e = 0; e < 8; e += 2) {
        uint16_t h2[2], l2[2];
        for (int q2 = 0; q2 < 2; ++q2) {
          const int k = ch * 8 + e + q2;  // key dim
          float x = 0.0f;
          if (gg < g.g) {
            const int f = (g.pairing == TRIA_PAIR_NEOX) ? (k & 63) : (k >> 1);
            const bool im = (g.pairing == TRIA_PAIR_NEOX) ? (k >= 64) : (k & 1);
            const double2 mu = mu_s[gg][f + (f >> 3)];
            const double2 r = rotj[j][f + (f >> 3)];
            x = im ? (float)(mu.x * r.y + mu.y * r.x) : (float)(mu.x * r.x - mu.y * r.y);
          }
          h2[q2] = bf16_rn_bits(x);
          l2[q2] = bf16_rn_bits(x - __uint_as_float((uint32_t)h2[q2] << 16));
        }
        whi[e >> 1] = (uint32_t)h2[0] | ((uint32_t)h2[1] << 16);
        wlo[e >> 1] = (uint32_t)l2[0] | ((uint32_t)l2[1] << 16);
      }
      const int64_t off = (int64_t)n * 128 + ((c8 ^ (n & 7)) << 4);
      *reinterpret_cast<uint4 *>(dst + kb * (g.ncol_t * 128) + off) =
          make_uint4(whi[0], whi[1], whi[2], whi[3]);
      *reinterpret_cast<uint4 *>(dst + (2 + kb) * (g.ncol_t * 128) + off) =
          make_uint4(wlo[0], wlo[1], wlo[2], wlo[3]);
    }
    // norm rows n = 2 gg + part over the magnitude dims: block 0 multiplies
    // |k_f| hi (w_f split hi/lo over the rows), block 1 |k_f| lo (w_f hi, 0)
    unsigned char *dn = dst + 4 * g.ncol_t * 128;
    for (int i = t; i < g.ncol_n * 16; i += kThreads) {
      const int n = i >> 4, ch = i & 15, kb = ch >> 3, c8 = ch & 7;
      const int gg = n >> 1, part = n & 1;
      uint32_t w[4];
      for (int e = 0; e < 8; e += 2) {
        uint16_t b2[2];
        for (int q2 = 0; q2 < 2; ++q2) {
          const int f = (ch & 7) * 8 + e + q2;
          float x = 0.0f;
          if (gg < g.g) x = (float)p.w_norm[((int64_t)l * g.hq + h * g.g + gg) * kBands + f];
          const uint16_t hi = bf16_rn_bits(x);
          const uint16_t lo = bf16_rn_bits(x - __uint_as_float((uint32_t)hi << 16));
          b2[q2] = (kb == 0) ? (part == 0 ? hi : lo) : (part == 0 ? hi : (uint16_t)0);
        }
        w[e >> 1] = (uint32_t)b2[0] | ((uint32_t)b2[1] << 16);
      }
      *reinterpret_cast<uint4 *>(dn + kb * (g.ncol_n * 128) + n * 128 + ((c8 ^ (n & 7)) << 4)) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
    return;
  }

  if (t < kBands) rot[t] = rot_at(p, t, p.query_pos[s]);
  __syncthreads();
  for (int i = t; i < g.g * kBands; i += kThreads) {
    const int gg = i / kBands, f = i % kBands;
    const int64_t qi = ((int64_t)l * g.hq + h * g.g + gg) * kBands + f;
    const double2 mu = p.mu_fold[qi];
    const double2 r = rot[f];
    cf[gg][f] = (float)(mu.x * r.x - mu.y * r.y);
    cf[gg][kBands + f] = (float)(mu.x * r.y + mu.y * r.x);
    cf[gg][2 * kBands + f] = (float)p.w_norm[qi];
  }
  __syncthreads();
  // grouped paged tiles: the hkv units of a (sequence, layer) share one image
  // with their 2G columns side by side (unit h at rows 2G h .. 2G h + 2G - 1
  // of every K block; no padding columns)
  const int64_t gu = g.grouped ? u - h : u;
  const int ucols = g.grouped ? 2 * g.g : g.ncol;
  const int rows = g.grouped ? g.hkv * ucols : g.ncol, row0 = g.grouped ? h * ucols : 0;
  unsigned char *dst = reinterpret_cast<unsigned char *>(p.btile) + gu * (int64_t)g.b_bytes;
  for (int i = t; i < ucols * (kCoefK / 8); i += kThreads) {
    const int n = i / (kCoefK / 8), ch = i % (kCoefK / 8), k0 = ch * 8;
    const int gg = n >> 1, part = n & 1;
    uint32_t w[4];
    for (int e = 0; e < 8; e += 2) {
      uint16_t b2[2];
      for (int q = 0; q < 2; ++q) {
        const int k = k0 + e + q;
        float x = 0.0f;
        if (gg < g.g) {
          if (k < 128) {
            x = (g.pairing == TRIA_PAIR_NEOX) ? cf[gg][k]
                                              : ((k & 1) ? cf[gg][kBands + (k >> 1)] : cf[gg][k >> 1]);
          } else if (k < 192) {
            x = cf[gg][2 * kBands + (k - 128)];
          } else {
            x = (part == 0) ? cf[gg][2 * kBands + (k - 192)] : 0.0f;
          }
        }
        const uint16_t hi = bf16_rn_bits(x);
        const uint16_t lo = bf16_rn_bits(x - __uint_as_float((uint32_t)hi << 16));
        b2[q] = (part == 0) ? hi : lo;
      }
      w[e >> 1] = (uint32_t)b2[0] | ((uint32_t)b2[1] << 16);
    }
    const int kb = ch >> 3, c8 = ch & 7, row = row0 + n;
    *reinterpret_cast<uint4 *>(dst + kb * (rows * 128) + row * 128 + ((c8 ^ (row & 7)) << 4)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ---------------------------------------------------------------------------
// tail_kernel: normalize-then-max over blocks of (unit, chunk of kAggChunk
// candidates); with selection, every block adds its chunk's histogram of the
// top 12 agg-key bits into the unit's, and the block that finishes the
// unit's last chunk runs the radix selection.
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(kThreads) tail_kernel(const __grid_constant__ TailParams p) {
  __shared__ TailScratch ts;
  __shared__ SelScalars sc;
  __shared__ int s_last;
  const Geom &geo = p.geo;
  const int nch_max = (geo.c_max + kAggChunk - 1) / kAggChunk;
  const int64_t u = blockIdx.x / nch_max;
  const int chunk = (int)(blockIdx.x % nch_max);
  const int s = (int)(u / ((int64_t)geo.nl * geo.hkv));
  const int lrel = (int)((u / geo.hkv) % geo.nl);
  const int N = unit_len(geo, s, lrel);
  if (!compresses(geo, N, lrel)) return;
  const int C = N - geo.window - geo.sinks;
  const int nch = (C + kAggChunk - 1) / kAggChunk;
  if (chunk >= nch) return;
  const int t = threadIdx.x;
  unit_norm<G, 0, kThreads>(p.moments + u * geo.tiles_max * kRowGroups * G * 2,
                            unit_tiles(N, geo.window, geo.sinks), C, t, sc);
  const bool sel = p.kept != nullptr;
  if (sel) clear_words<kThreads>(ts.hist, kAggHistBins, t);
  __syncthreads();
  const int c0 = chunk * kAggChunk, c1 = min(C, c0 + kAggChunk);
  const float *raw = p.raw + u * p.raw_stride;
  float *agg = p.agg + u * p.agg_stride;
  agg_range<G, kThreads>(raw, agg, c0, c1, sc.mean, sc.inv, sel ? ts.hist : nullptr, t);
  __syncthreads();
  if (p.discard_raw) {
    const int64_t l0 = (int64_t)c0 * G * 4 / 128, l1 = ((int64_t)c1 * G * 4 + 127) / 128;
    for (int64_t i = l0 + t; i < l1; i += kThreads) discard_line(raw + i * 32);
  }
  if (!sel) return;
  uint32_t *gh = p.hist + u * kAggHistBins;
  for (int i = t; i < kAggHistBins; i += kThreads) {
    const uint32_t v = ts.hist[i];
    if (v) atomicAdd(gh + i, v);
  }
  __syncthreads();
  if (t == 0) s_last = (atom_add_acq_rel(p.unit_done + u, 1u) == (uint32_t)nch - 1u) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  for (int i = t; i < kAggHistBins; i += kThreads) ts.hist[i] = __ldcg(gh + i);
  __syncthreads();
  const int B = geo.lbudget[lrel];
  int32_t *kept = p.kept + u * geo.budget;
  select_unit<0, kThreads>(agg, C, B - geo.window - geo.sinks, N, B, geo.window, geo.sinks, kept,
                           ts, sc, true, t);
  for (int j = B + t; j < geo.budget; j += kThreads) kept[j] = -1;
  __syncthreads();
  if (p.discard_agg) {
    const int64_t lines = ((int64_t)C * 4 + 127) / 128;
    for (int64_t i = t; i < lines; i += kThreads) discard_line(agg + i * 32);
  }
}

// ---------------------------------------------------------------------------
// select_kernel: one CTA per unit
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) select_kernel(const __grid_constant__ SelectParams p) {
  __shared__ TailScratch ts;
  __shared__ SelScalars sc;
  const Geom &geo = p.geo;
  const int64_t u = blockIdx.x;
  const int s = (int)(u / ((int64_t)geo.nl * geo.hkv));
  const int lrel = (int)((u / geo.hkv) % geo.nl);
  const int N = unit_len(geo, s, lrel);
  int32_t *kept = p.kept + u * geo.budget;
  const int t = threadIdx.x;
  if (!compresses(geo, N, lrel)) {
    const bool bad = !len_valid(geo, N);
    if (bad && t == 0) atomicOr(p.status, 1);
    for (int j = t; j < geo.budget; j += kThreads) kept[j] = (!bad && j < N) ? j : -1;
    return;
  }
  const int C = N - geo.window - geo.sinks;
  const int B = geo.lbudget[lrel];
  select_unit<0, kThreads>(p.agg + u * p.agg_stride, C, B - geo.window - geo.sinks, N, B,
                           geo.window, geo.sinks, kept, ts, sc, false, t);
  for (int j = B + t; j < geo.budget; j += kThreads) kept[j] = -1;
}

}  // namespace

cudaError_t launch_coef(const CoefParams &p, cudaStream_t st) {
  coef_kernel<<<(unsigned)p.geo.n_units, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_tail(const TailParams &p, cudaStream_t st) {
  const int64_t blocks = p.geo.n_units * ((p.geo.c_max + kAggChunk - 1) / kAggChunk);
  switch (p.geo.g) {
    case 1: tail_kernel<1><<<(unsigned)blocks, kThreads, 0, st>>>(p); break;
    case 2: tail_kernel<2><<<(unsigned)blocks, kThreads, 0, st>>>(p); break;
    case 4: tail_kernel<4><<<(unsigned)blocks, kThreads, 0, st>>>(p); break;
    case 8: tail_kernel<8><<<(unsigned)blocks, kThreads, 0, st>>>(p); break;
    case 16: tail_kernel<16><<<(unsigned)blocks, kThreads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectParams &p, cudaStream_t st) {
  select_kernel<<<(unsigned)p.geo.n_units, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}


}  // namespace tria
