// Scoring kernel of the max-over-offsets mode (tria_params.offset_reduce =
// TRIA_OFFSET_MAX), the non-default variant named at the end of sec. 4 of
// the academ.us article 2607.13051: the trigonometric term takes the
// maximum over the future offsets delta_j in D instead of their mean.
//
// S_g(k) = max_j S_trig,g(k, Delta + delta_j) + S_norm,g(k).  The maximum is
// not linear, so nothing folds: per (head g, offset delta_j) the coefficient
// vector c_gj = E[q_g] mask e^{i omega (p_q + delta_j)} is its own column of
// the trig operand (|D| G columns, padded to a multiple of 16: NTH), split
// into bf16 hi and lo parts that sit in two K halves, and the norm weights
// a separate 2G-column operand.  Per tile two contractions:
//   [k | k] (128 x 256) . [Bhi ; Blo] (256 x NTH)  -> trig accumulator
//   [m_hi | m_lo] (128 x 128) . Bnorm (128 x 2G)   -> norm accumulator
// (the K tile is read twice from shared memory, once per part), then a max
// over the |D| offset columns of each head in the epilogue.  With one column
// per (head, offset) a tile needs NTH <= 144 trig columns, so tensor memory
// holds two buffers of everything (trig 0..143 | 144..287, norm 288.. |
// 304.., magnitudes 320.. | 384..): the epilogue of tile i - 1 runs while
// the MMAs of tile i do.
//
// Roles as in the offset-mean kernel (tria_score_tc.cu): warps 0-7 compute
// (magnitudes of tile i, then the epilogue of tile i - 1), warp 8 producer
// (TMA), warp 9 MMA issuer.  Bounded waits and the abort path as described
// in tria_tc.cuh.
#include "tria_tc.cuh"

namespace tria {
namespace {

using namespace dev;
using namespace tc;

constexpr int kBandGroups = 2;
constexpr int kBandsPerThread = kBands / kBandGroups;
constexpr int kComputeWarps = 4 * kBandGroups;
constexpr int kProducerWarp = kComputeWarps;
constexpr int kMmaWarp = kComputeWarps + 1;
constexpr int kThreads = 32 * (kComputeWarps + 2);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTrigCols = 144;                 // one trig buffer: |D| G <= 136, padded
constexpr uint32_t kMaxNormCol = 2 * kTrigCols;     // norm buffers: 288.., 304..
constexpr uint32_t kNormCols = 16;
constexpr uint32_t kMaxMagCol = kMaxNormCol + 2 * kNormCols;  // magnitude buffers: 320.., 384..
static_assert(kMaxMagCol + 2 * 64 <= kTmemCols, "tensor memory columns of the max-mode kernel");

template <int G>
struct MaxCfg {
  static constexpr int NN = (2 * G < 16) ? 16 : 2 * G;                  // norm columns
  static constexpr int NTH_MAX = ((17 * G + 15) / 16) * 16;             // trig columns at |D| = 17
  static constexpr int STAGES = (G >= 8) ? 2 : 4;
  static constexpr int BMAX = (2 * NTH_MAX + NN) * 256;                  // coefficient image bytes
  static constexpr int GQ = (G >= kBandGroups) ? G / kBandGroups : 1;
  static_assert(NN == (int)kNormCols && NTH_MAX <= (int)kTrigCols, "max-mode operand columns");
};

template <int G>
struct MaxSmem {
  alignas(1024) uint8_t k[MaxCfg<G>::STAGES][2][kHalfBlock];
  alignas(1024) uint8_t b[2][MaxCfg<G>::BMAX];
  alignas(8) uint64_t full[MaxCfg<G>::STAGES];
  alignas(8) uint64_t kempty[MaxCfg<G>::STAGES];
  alignas(8) uint64_t aready[2];
  alignas(8) uint64_t accfull[2];
  alignas(8) uint64_t bempty[2];
  SubRec rec[MaxCfg<G>::STAGES];
  alignas(16) int seq_items[kMaxSeqTable];
  int seq_len[kMaxSeqTable];
  uint32_t tmem_base;
  volatile int abort_flag;
  __device__ __forceinline__ uint8_t *bbuf(int i) { return &b[i][0]; }
};

template <int G>
__device__ void mma_issuer_max(const ScoreParams &p, MaxSmem<G> &sm, uint32_t tmem,
                               const WaitCtl wc) {
  using Cfg = MaxCfg<G>;
  constexpr int ST = Cfg::STAGES, NN = Cfg::NN;
  const int NTH = p.geo.ncol_t;
  const uint32_t idt = idesc_bf16_m128_n(NTH);
  constexpr uint32_t idn = idesc_bf16_m128_n(NN);
  const uint64_t da0 = sw128_desc(smem_u32(&sm.k[0][0][0]));
  const uint64_t db0 = sw128_desc(smem_u32(&sm.b[0][0]));
  constexpr uint32_t kStageBytes = 2 * kHalfBlock;
  const uint32_t tblk = (uint32_t)NTH * 128u;  // one 64-wide K block of the trig image
  const uint32_t nbase = 4u * tblk;            // norm image after the trig hi and lo parts
  int i = 0;
  for (;; ++i) {
    const int ab = i & 1;
    if (!mbar_wait(&sm.aready[ab], (i >> 1) & 1, wc)) break;
    tc_fence_after();
    const int stage = i % ST;
    const SubRec &rec = sm.rec[stage];
    const int flags = rec.flags, bpar = rec.bpar;
    if (flags & kFlagEnd) break;
    const uint64_t da = da0 + (uint64_t)((stage * kStageBytes) >> 4);
    const uint64_t db = db0 + (uint64_t)(((uint32_t)bpar * (uint32_t)Cfg::BMAX) >> 4);
    const uint32_t dt = tmem + (uint32_t)ab * kTrigCols;
    // trig: K = 128 key dims against the hi part, then again against the lo part
#pragma unroll
    for (int s = 0; s < 16; ++s) {
      const int k = s & 7;
      const uint32_t ao = (k >> 2) * kHalfBlock + (k & 3) * 32;
      const uint32_t bo = (uint32_t)(s >> 2) * tblk + (k & 3) * 32;
      mma_bf16(dt, da + (ao >> 4), db + (bo >> 4), idt, s > 0 ? 1u : 0u);
    }
    mma_commit(&sm.kempty[stage]);  // the K tile is consumed
    const uint32_t dn = tmem + kMaxNormCol + (uint32_t)ab * kNormCols;
    const uint32_t ta = tmem + kMaxMagCol + (uint32_t)ab * 64u;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t bo = nbase + (uint32_t)(s >> 2) * NN * 128u + (s & 3) * 32;
      mma_bf16_ta(dn, ta + (uint32_t)(s * 8), db + (bo >> 4), idn, s > 0 ? 1u : 0u);
    }
    if (flags & kFlagLast) mma_commit(&sm.bempty[bpar]);
    mma_commit(&sm.accfull[ab]);  // issued last: it covers every MMA before it
  }
  if (i > 0) mbar_drain(&sm.accfull[(i - 1) & 1], ((i - 1) >> 1) & 1, wc.status);
}

// Raw scores, fp64 moment sums and the item's moment partials of one tile.
template <int G>
__device__ __forceinline__ void emit_scores(const ScoreParams &p, const EpRec &pr,
                                            const float (&sc)[MaxCfg<G>::GQ], bool active, int q,
                                            int rg, int lane, double (&msum)[MaxCfg<G>::GQ],
                                            double (&msq)[MaxCfg<G>::GQ]) {
  constexpr int GQ = MaxCfg<G>::GQ;
  const Geom &geo = p.geo;
  if (pr.flags & kFlagFirst) {
#pragma unroll
    for (int g = 0; g < GQ; ++g) msum[g] = msq[g] = 0.0;
  }
  if (active) {
    const int slot = pr.slot0 + rg * 32 + lane;
    if (slot >= geo.sinks && slot < pr.N - geo.window) {
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        msum[g] += (double)sc[g];
        msq[g] = fma((double)sc[g], (double)sc[g], msq[g]);
      }
      float *dst = ep_raw(p, pr) + (slot - geo.sinks) * G + q * GQ;
      if constexpr (GQ == 4) {
        *reinterpret_cast<float4 *>(dst) = make_float4(sc[0], sc[1], sc[2], sc[3]);
      } else if constexpr (GQ == 2) {
        *reinterpret_cast<float2 *>(dst) = make_float2(sc[0], sc[1]);
      } else {
#pragma unroll
        for (int g = 0; g < GQ; ++g) dst[g] = sc[g];
      }
    }
  }
  if ((pr.flags & kFlagLast) && active) {
#pragma unroll
    for (int g = 0; g < GQ; ++g) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        msum[g] += __shfl_xor_sync(kFull, msum[g], o);
        msq[g] += __shfl_xor_sync(kFull, msq[g], o);
      }
    }
    if (lane == 0) {
      double *m = ep_mom(p, pr) + (rg * G + q * GQ) * 2;
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        m[2 * g] = msum[g];
        m[2 * g + 1] = msq[g];
      }
    }
  }
}

// Epilogue of tile j (buffer j & 1): per head of this thread's band group,
// S = max_j trig_j + (norm hi + norm lo).
template <int G>
__device__ __forceinline__ void epilogue_max(const ScoreParams &p, uint32_t tmem, int buf,
                                             const EpRec &pr, int q, int rg, int lane,
                                             double (&msum)[MaxCfg<G>::GQ],
                                             double (&msq)[MaxCfg<G>::GQ]) {
  constexpr int GQ = MaxCfg<G>::GQ;
  const bool active = (G >= kBandGroups) || q < G;
  const int nd = p.geo.n_off;
  float sc[GQ];
  if (active) {
    const uint32_t lb = tmem + ((uint32_t)(32 * rg) << 16);
    const uint32_t tb = lb + (uint32_t)buf * kTrigCols;
    const uint32_t nb = lb + kMaxNormCol + (uint32_t)buf * kNormCols;
    // two heads per tensor-memory round trip (one wait per pair instead of
    // per head: 1916 -> 1704 us per Qwen3-32B 32K score launch; all four
    // heads at once measured 1773 us): a head's nd columns are one 16-column
    // load (offsets 0..15; past nd it reads the next head's columns, unused)
    // and, at nd = 17, a 2-column load for offset 16 (its second column unused)
    constexpr int HP = (GQ >= 2) ? 2 : 1;
    if (GQ >= 2 && nd == kMaxOffsets) {
      // |D| = 17: a head pair's 34 trig columns are adjacent (one 32-column
      // and one 2-column load) and so are its 4 norm columns (one load)
#pragma unroll
      for (int g0 = 0; g0 < GQ; g0 += 2) {
        uint32_t t[32], t2[2], nv[4];
        const int g = q * GQ + g0;
        const uint32_t c0 = tb + (uint32_t)(g * kMaxOffsets);
        tmem_ld_nowait<32>(c0, t);
        tmem_ld_nowait<2>(c0 + 32, t2);
        tmem_ld_nowait<4>(nb + (uint32_t)(2 * g), nv);
        tmem_wait_ld();
        float m0 = __uint_as_float(t[0]), m1 = __uint_as_float(t[17]);
#pragma unroll
        for (int j = 1; j < 17; ++j) m0 = max_nan(m0, __uint_as_float(t[j]));
#pragma unroll
        for (int j = 18; j < 32; ++j) m1 = max_nan(m1, __uint_as_float(t[j]));
        m1 = max_nan(m1, max_nan(__uint_as_float(t2[0]), __uint_as_float(t2[1])));
        sc[g0] = m0 + (__uint_as_float(nv[0]) + __uint_as_float(nv[1]));
        sc[g0 + 1] = m1 + (__uint_as_float(nv[2]) + __uint_as_float(nv[3]));
      }
    } else {
#pragma unroll
    for (int g0 = 0; g0 < GQ; g0 += HP) {
      uint32_t t[HP][16], t16[HP][2], nv[HP][2];
#pragma unroll
      for (int a = 0; a < HP; ++a) {
        const int g = q * GQ + g0 + a;
        const uint32_t c0 = tb + (uint32_t)(g * nd);
        tmem_ld_nowait<16>(c0, t[a]);
        if (nd == 17) tmem_ld_nowait<2>(c0 + 16, t16[a]);
        tmem_ld_nowait<2>(nb + (uint32_t)(2 * g), nv[a]);
      }
      tmem_wait_ld();
#pragma unroll
      for (int a = 0; a < HP; ++a) {
        // offsets past |D| read as -inf; a pairwise tree of NaN-propagating maxes
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (j >= nd) t[a][j] = __float_as_uint(-INFINITY);
#pragma unroll
        for (int w = 1; w < 16; w *= 2) {
#pragma unroll
          for (int j = 0; j + w < 16; j += 2 * w)
            t[a][j] = __float_as_uint(max_nan(__uint_as_float(t[a][j]), __uint_as_float(t[a][j + w])));
        }
        const float v16 = (nd == 17) ? __uint_as_float(t16[a][0]) : -INFINITY;
        const float m = max_nan(__uint_as_float(t[a][0]), v16);
        sc[g0 + a] = m + (__uint_as_float(nv[a][0]) + __uint_as_float(nv[a][1]));
      }
    }
    }
  } else {
#pragma unroll
    for (int gi = 0; gi < GQ; ++gi) sc[gi] = 0.0f;
  }
  tc_fence_before();
  emit_scores<G>(p, pr, sc, active, q, rg, lane, msum, msq);
}

// Tile i: magnitudes of tile i into buffer i & 1 (its previous reader, the
// MMAs of tile i - 2, finished before this warp's epilogue of tile i - 2),
// then the epilogue of tile i - 1 while the MMAs of tile i run.
template <int G, int PAIR>
__device__ void compute_max(const ScoreParams &p, MaxSmem<G> &sm, uint32_t tmem, int tid,
                            const WaitCtl wc) {
  constexpr int ST = MaxCfg<G>::STAGES, GQ = MaxCfg<G>::GQ, W = kBandsPerThread / 2;
  const int warp = tid >> 5, lane = tid & 31;
  const int q = warp >> 2, rg = warp & 3, r = rg * 32 + lane;
  const uint32_t mag = tmem + ((uint32_t)(32 * rg) << 16) + kMaxMagCol;
  double msum[GQ], msq[GQ];
#pragma unroll
  for (int g = 0; g < GQ; ++g) msum[g] = msq[g] = 0.0;
  EpRec prev{};
  for (int i = 0;; ++i) {
    const int stage = i % ST;
    if (!warp_wait(&sm.full[stage], (i / ST) & 1, wc, lane)) return;
    const SubRec &rc = sm.rec[stage];
    const int flags = rc.flags;
    const bool end = (flags & kFlagEnd) != 0;
    EpRec cur{};
    if (!end) {
      cur = ep_of(rc);
      uint32_t hi[W], lo[W];
      mags_regs<PAIR, kBandsPerThread>(&sm.k[stage][0][0], r, q, hi, lo);
      const uint32_t mb = mag + (uint32_t)((i & 1) * 64);
      tmem_st<W>(mb + (uint32_t)(W * q), hi);
      tmem_st<W>(mb + (uint32_t)(32 + W * q), lo);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.aready[i & 1]);
    if (i >= 1) {
      const int j = i - 1;
      if (!warp_wait(&sm.accfull[j & 1], (j >> 1) & 1, wc, lane)) return;
      tc_fence_after();
      epilogue_max<G>(p, tmem, j & 1, prev, q, rg, lane, msum, msq);
    }
    if (end) return;
    prev = cur;
  }
}

template <int G, int PAIR, int LAYOUT>
__global__ void __launch_bounds__(kThreads, 1) score_max_kernel(const __grid_constant__ ScoreParams p) {
  using Cfg = MaxCfg<G>;
  extern __shared__ uint8_t smem_dyn[];
  MaxSmem<G> &sm = *reinterpret_cast<MaxSmem<G> *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  const Geom &geo = p.geo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int i = tid; i <= geo.n_seq; i += kThreads) sm.seq_items[i] = p.seq_items[i];
  for (int i = tid; i < geo.n_seq; i += kThreads) sm.seq_len[i] = unit_len(geo, i, 0);
  if (tid == 0) {
    for (int i = 0; i < Cfg::STAGES; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.kempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.aready[i], kComputeWarps);
      mbar_init(&sm.accfull[i], 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&sm.bempty[i], 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int n_items = sm.seq_items[geo.n_seq];
  const WaitCtl wc = wait_ctl(&sm.abort_flag, p.status, p.wait_ns);

  if (warp < kComputeWarps) {
    compute_max<G, PAIR>(p, sm, tmem, tid, wc);
  } else if (warp == kProducerWarp) {
    producer<Cfg::STAGES, LAYOUT>(p, sm, n_items, lane, wc);
  } else if (warp == kMmaWarp) {
    if (lane == 0) mma_issuer_max<G>(p, sm, tmem, wc);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int G, int PAIR, int LAYOUT>
cudaError_t launch_max_t(const ScoreParams &p, cudaStream_t st) {
  auto kern = score_max_kernel<G, PAIR, LAYOUT>;
  const int smem = (int)sizeof(MaxSmem<G>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  kern<<<sms, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int G>
cudaError_t launch_max_g(const ScoreParams &p, cudaStream_t st) {
  const bool paged = p.cache.layout == TRIA_LAYOUT_PAGED;
  if (p.geo.pairing == TRIA_PAIR_NEOX)
    return paged ? launch_max_t<G, TRIA_PAIR_NEOX, TRIA_LAYOUT_PAGED>(p, st)
                 : launch_max_t<G, TRIA_PAIR_NEOX, TRIA_LAYOUT_CONTIGUOUS>(p, st);
  return paged ? launch_max_t<G, TRIA_PAIR_INTERLEAVED, TRIA_LAYOUT_PAGED>(p, st)
               : launch_max_t<G, TRIA_PAIR_INTERLEAVED, TRIA_LAYOUT_CONTIGUOUS>(p, st);
}

static_assert(sizeof(MaxSmem<8>) + 1024 <= 232448, "shared memory of the G=8 max-mode kernel");
static_assert(sizeof(MaxSmem<4>) + 1024 <= 232448, "shared memory of the G=4 max-mode kernel");


}  // namespace

cudaError_t launch_score_max(const ScoreParams &p, cudaStream_t st) {
  switch (p.geo.g) {
    case 1: return launch_max_g<1>(p, st);
    case 2: return launch_max_g<2>(p, st);
    case 4: return launch_max_g<4>(p, st);
    case 8: return launch_max_g<8>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tria
