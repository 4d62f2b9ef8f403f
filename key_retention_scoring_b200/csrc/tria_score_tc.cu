// Scoring kernel of the compression pass on the sm_100a tensor cores, with
// the unit tail (normalize-then-max and selection) optionally fused.
//
// Per unit (sequence, layer, KV head) the averaged score of G query heads is
//   S~_g(k) = sum_f Re(c_gf conj(ktilde_f)) + w_gf |ktilde_f|
// with ktilde the post-RoPE key, c_gf = mu'_gf e^{i omega_f p_q} the folded
// center turned to the query position (academ.us article 2607.13051, Eqs. 3,
// 6, 7: the key position cancels because conj(k_f) e^{i omega_f (p_q - p_k)}
// = conj(ktilde_f) e^{i omega_f p_q}) and w_gf = E|q_f| - |E q_f| the norm-term
// weight.  Over a tile of 128 keys both sums are one dense contraction
//   D[128 x 2G] = [ktilde | m_hi | m_lo] (128 x 256) . Bcoef (256 x 2G)
// where m = |ktilde_f| is split into bf16 hi + lo parts and every fp32
// coefficient x into bf16 hi + lo columns (D[:,2g] + D[:,2g+1] = S~_g up to a
// relative 2^-16 of the terms).  The keys are bf16 already, so the product is
// exact and accumulates in fp32 in tensor memory.
//
// Roles (one CTA per SM, persistent, dynamic items of kTileKeys slots):
//   warps 0-7   band magnitudes -> tensor memory (tcgen05.st; warp w takes
//               rows 32(w%4).. and bands 32(w/4)..), then, two tiles later,
//               the epilogue (tcgen05.ld, raw scores, fp64 moment partials).
//               Magnitude tiles and accumulators rotate through kNB
//               tensor-memory buffers, so two MMA chains stay in flight;
//   warp 8      producer: TMA tensor loads of 128-slot K tiles (two 64-dim
//               boxes, or one box per paged block) into a ring of 128-byte-
//               swizzled K-major tiles, plus the unit's coefficient image
//               (one bulk copy per item); completion as mbarrier tx bytes;
//   warp 9      one lane issues tcgen05.mma (M=128, N=16|32, K=16): 8 steps
//               with A = the K tile in shared memory (then the K stage is
//               released), 8 steps with A = the magnitude tile in tensor
//               memory, and tcgen05.commit.
// Normalize-then-max and the selection run in the next kernel (the unit tail
// in tria_kernels.cu).  Every wait is bounded (ScoreParams::wait_ns); on
// expiry the kernel flags status bit 1, lets its own loads and MMAs land,
// frees its tensor memory and returns.
#include "tria_tc.cuh"

namespace tria {
namespace {

using namespace dev;
using namespace tc;

constexpr int kBandGroups = 2;              // compute warps per 32-row quadrant of a tile
constexpr int kBandsPerThread = kBands / kBandGroups;
constexpr int kComputeWarps = 4 * kBandGroups;
constexpr int kProducerWarp = kComputeWarps;
constexpr int kMmaWarp = kComputeWarps + 1;
constexpr int kTcThreads = 32 * (kComputeWarps + 2);
// The epilogue of tile i runs after the magnitudes of tile i + 2, so two MMA
// chains are in flight while the compute warps work; magnitude tiles and
// accumulators rotate through kNB tensor-memory buffers (tile i uses i % kNB,
// whose previous user, tile i - kNB, finished its epilogue before the
// magnitudes of tile i - 1).
constexpr int kNB = 4;
constexpr uint32_t kTmemCols = 512;         // [0, 256): accumulators; [256, 512): magnitude tiles
constexpr uint32_t kTmemMag = 256;

template <int G>
struct TcCfg {
  static constexpr int NCOL = (2 * G < 16) ? 16 : 2 * G;   // MMA N
  static constexpr int STAGES = (G <= 8) ? 6 : 5;
  static constexpr int GQ = (G >= kBandGroups) ? G / kBandGroups : 1;  // heads per band group
  static constexpr int BBLK = NCOL * 128;                  // bytes per 64-wide K block of B
  // K-steps of a tile may accumulate into NACC partial accumulators (summed
  // by the epilogue) so that consecutive MMAs do not wait on each other's
  // results; with two tiles of slack between a tile's MMAs and its epilogue
  // the single chain of 16 measured fastest (931 us per Qwen3-32B 32K pass,
  // against 936 with two chains and 960 with four)
  static constexpr int NACC = 1;
  static_assert(kNB * NACC * NCOL <= 256, "accumulator columns");
};

template <int G>
struct TcSmem {
  alignas(1024) uint8_t k[TcCfg<G>::STAGES][2][kHalfBlock];
  alignas(1024) uint8_t b[2][4][TcCfg<G>::BBLK];
  alignas(8) uint64_t full[TcCfg<G>::STAGES];
  alignas(8) uint64_t kempty[TcCfg<G>::STAGES];
  alignas(8) uint64_t aready[kNB];
  alignas(8) uint64_t accfull[kNB];
  alignas(8) uint64_t bempty[2];
  SubRec rec[TcCfg<G>::STAGES];
  alignas(16) int seq_items[kMaxSeqTable];
  int seq_len[kMaxSeqTable];
  uint32_t tmem_base;
  volatile int abort_flag;
  __device__ __forceinline__ uint8_t *bbuf(int i) { return &b[i][0][0]; }
};

// ---------------------------------------------------------------------------
// MMA issuer (one lane)
// ---------------------------------------------------------------------------
template <int G>
__device__ void mma_issuer(const ScoreParams &p, TcSmem<G> &sm, uint32_t tmem, const WaitCtl wc) {
  using Cfg = TcCfg<G>;
  constexpr int ST = Cfg::STAGES, NCOL = Cfg::NCOL, BBLK = Cfg::BBLK, NACC = Cfg::NACC;
  constexpr uint32_t idesc = idesc_bf16_m128_n(NCOL);
  // descriptors of stage 0 / coefficient buffer 0; an operand at byte offset
  // o from there is the descriptor plus o >> 4 (shared addresses < 256 KB)
  const uint64_t da0 = sw128_desc(smem_u32(&sm.k[0][0][0]));
  const uint64_t db0 = sw128_desc(smem_u32(&sm.b[0][0][0]));
  constexpr uint32_t kStageBytes = 2 * kHalfBlock;
  int i = 0;
  for (;; ++i) {
    if (!mbar_wait(&sm.aready[i % kNB], (i / kNB) & 1, wc)) break;
    tc_fence_after();
    const int stage = i % ST, ab = i % kNB;
    const SubRec &rec = sm.rec[stage];
    const int flags = rec.flags, bpar = rec.bpar;
    if (flags & kFlagEnd) break;
    const uint32_t d = tmem + (uint32_t)(ab * NACC * NCOL);
    const uint32_t ta = tmem + kTmemMag + (uint32_t)(ab * 64);
    const uint64_t da = da0 + (uint64_t)((stage * kStageBytes) >> 4);
    const uint64_t db = db0 + (uint64_t)((bpar * 4 * BBLK) >> 4);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t ao = (s >> 2) * kHalfBlock + (s & 3) * 32;
      const uint32_t bo = (s >> 2) * BBLK + (s & 3) * 32;
      mma_bf16(d + (uint32_t)((s % NACC) * NCOL), da + (ao >> 4), db + (bo >> 4), idesc,
               s >= NACC ? 1u : 0u);
    }
    mma_commit(&sm.kempty[stage]);  // the K tile is consumed: the producer may refill it
#pragma unroll
    for (int s = 8; s < 16; ++s) {
      const uint32_t bo = (s >> 2) * BBLK + (s & 3) * 32;
      mma_bf16_ta(d + (uint32_t)((s % NACC) * NCOL), ta + (uint32_t)((s - 8) * 8), db + (bo >> 4),
                  idesc, 1u);
    }
    if (flags & kFlagLast) mma_commit(&sm.bempty[bpar]);
    mma_commit(&sm.accfull[ab]);  // issued last: it covers every MMA before it
  }
  // the MMAs already issued must land before the tensor memory is freed
  if (i > 0) mbar_drain(&sm.accfull[(i - 1) % kNB], ((i - 1) / kNB) & 1, wc.status);
}

// ---------------------------------------------------------------------------
// compute warps
// ---------------------------------------------------------------------------
template <int PAIR>
__device__ __forceinline__ void mags(const uint8_t *kt, uint32_t tcol, int r, int q) {
  constexpr int W = kBandsPerThread / 2;
  uint32_t hi[W], lo[W];
  mags_regs<PAIR, kBandsPerThread>(kt, r, q, hi, lo);
  tmem_st<W>(tcol + (uint32_t)(W * q), hi);
  tmem_st<W>(tcol + (uint32_t)(32 + W * q), lo);
}

// Epilogue of tile j (record pr): raw scores of this warp's 32 rows and GQ
// heads, fp64 moment sums, and the item's moment partials after its last tile.
template <int G>
__device__ __forceinline__ bool epilogue(const ScoreParams &p, TcSmem<G> &sm, uint32_t tmem, int j,
                                         const EpRec &pr, int q, int rg, int lane,
                                         double (&msum)[TcCfg<G>::GQ], double (&msq)[TcCfg<G>::GQ],
                                         const WaitCtl wc) {
  constexpr int NCOL = TcCfg<G>::NCOL, GQ = TcCfg<G>::GQ, NACC = TcCfg<G>::NACC;
  const Geom &geo = p.geo;
  const bool active = (G >= kBandGroups) || q < G;  // group q scores heads [q GQ, (q + 1) GQ)
  if (!warp_wait(&sm.accfull[j % kNB], (j / kNB) & 1, wc, lane)) return false;
  tc_fence_after();
  if (pr.flags & kFlagFirst) {
#pragma unroll
    for (int g = 0; g < GQ; ++g) msum[g] = msq[g] = 0.0;
  }
  if (active) {
    // this thread's 2 GQ columns ((hi, lo) per head) of each partial
    // accumulator, summed in a fixed order
    uint32_t pa[NACC][2 * GQ];
    const uint32_t col = tmem + ((uint32_t)(32 * rg) << 16) +
                         (uint32_t)((j % kNB) * NACC * NCOL + q * 2 * GQ);
#pragma unroll
    for (int a = 0; a < NACC; ++a) tmem_ld_nowait<2 * GQ>(col + (uint32_t)(a * NCOL), pa[a]);
    tmem_wait_ld();
    float v[2 * GQ];
#pragma unroll
    for (int c = 0; c < 2 * GQ; ++c) {
      float x = __uint_as_float(pa[0][c]);
#pragma unroll
      for (int a = 1; a < NACC; ++a) x += __uint_as_float(pa[a][c]);
      v[c] = x;
    }
    const int slot = pr.slot0 + rg * 32 + lane;
    if (slot >= geo.sinks && slot < pr.N - geo.window) {
      float sc[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        sc[g] = v[2 * g] + v[2 * g + 1];
        msum[g] += (double)sc[g];
        msq[g] = fma((double)sc[g], (double)sc[g], msq[g]);
      }
      float *dst = ep_raw(p, pr) + (slot - geo.sinks) * G + q * GQ;
      if constexpr (GQ == 8) {
        reinterpret_cast<float4 *>(dst)[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
        reinterpret_cast<float4 *>(dst)[1] = make_float4(sc[4], sc[5], sc[6], sc[7]);
      } else if constexpr (GQ == 4) {
        *reinterpret_cast<float4 *>(dst) = make_float4(sc[0], sc[1], sc[2], sc[3]);
      } else if constexpr (GQ == 2) {
        *reinterpret_cast<float2 *>(dst) = make_float2(sc[0], sc[1]);
      } else {
        dst[0] = sc[0];
      }
    }
  }
  tc_fence_before();
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
  return true;
}

template <int G, int PAIR>
__device__ void compute(const ScoreParams &p, TcSmem<G> &sm, uint32_t tmem, int tid, const WaitCtl wc) {
  constexpr int ST = TcCfg<G>::STAGES, GQ = TcCfg<G>::GQ;
  const int warp = tid >> 5, lane = tid & 31;
  const int q = warp >> 2, rg = warp & 3, r = rg * 32 + lane;  // band group, quadrant, row
  const uint32_t mag_base = tmem + ((uint32_t)(32 * rg) << 16) + kTmemMag;
  double msum[GQ], msq[GQ];
#pragma unroll
  for (int g = 0; g < GQ; ++g) msum[g] = msq[g] = 0.0;
  // Tile i: magnitudes of tile i, then the epilogue of tile i - 2 (record
  // `older`, replaced by tile i's record); after the end marker also the
  // epilogue of tile i - 1 (record `other`).  0: go on, 1: done, -1: abort.
  auto step = [&](int i, EpRec &older, EpRec &other) -> int {
    const int stage = i % ST;
    if (!warp_wait(&sm.full[stage], (i / ST) & 1, wc, lane)) return -1;
    const SubRec &rc = sm.rec[stage];
    const int flags = rc.flags;
    const bool end = (flags & kFlagEnd) != 0;
    EpRec cur;
    if (!end) {
      cur = ep_of(rc);
      mags<PAIR>(&sm.k[stage][0][0], mag_base + (uint32_t)((i % kNB) * 64), r, q);
      tmem_wait_st();
      tc_fence_before();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.aready[i % kNB]);
    if (i >= 2 && !epilogue<G>(p, sm, tmem, i - 2, older, q, rg, lane, msum, msq, wc)) return -1;
    if (end) {
      if (i >= 1 && !epilogue<G>(p, sm, tmem, i - 1, other, q, rg, lane, msum, msq, wc)) return -1;
      return 1;
    }
    older = cur;
    return 0;
  };
  EpRec ra{}, rb{};
  for (int i = 0;; i += 2) {
    if (step(i, ra, rb)) return;
    if (step(i + 1, rb, ra)) return;
  }
}

template <int G, int PAIR, int LAYOUT>
__global__ void __launch_bounds__(kTcThreads, 1) score_tc_kernel(const __grid_constant__ ScoreParams p) {
  using Cfg = TcCfg<G>;
  extern __shared__ uint8_t smem_dyn[];
  TcSmem<G> &sm = *reinterpret_cast<TcSmem<G> *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  const Geom &geo = p.geo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int i = tid; i <= geo.n_seq; i += kTcThreads) sm.seq_items[i] = p.seq_items[i];
  for (int i = tid; i < geo.n_seq; i += kTcThreads) sm.seq_len[i] = unit_len(geo, i, 0);
  if (tid == 0) {
    for (int i = 0; i < Cfg::STAGES; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.kempty[i], 1);
    }
    for (int i = 0; i < kNB; ++i) {
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
    compute<G, PAIR>(p, sm, tmem, tid, wc);
  } else if (warp == kProducerWarp) {
    producer<Cfg::STAGES, LAYOUT>(p, sm, n_items, lane, wc);
  } else if (warp == kMmaWarp) {
    if (lane == 0) mma_issuer<G>(p, sm, tmem, wc);
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
cudaError_t launch_t(const ScoreParams &p, cudaStream_t st) {
  auto kern = score_tc_kernel<G, PAIR, LAYOUT>;
  const int smem = (int)sizeof(TcSmem<G>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  kern<<<sms, kTcThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int G>
cudaError_t launch_g(const ScoreParams &p, cudaStream_t st) {
  const bool paged = p.cache.layout == TRIA_LAYOUT_PAGED;
  if (p.geo.pairing == TRIA_PAIR_NEOX)
    return paged ? launch_t<G, TRIA_PAIR_NEOX, TRIA_LAYOUT_PAGED>(p, st)
                 : launch_t<G, TRIA_PAIR_NEOX, TRIA_LAYOUT_CONTIGUOUS>(p, st);
  return paged ? launch_t<G, TRIA_PAIR_INTERLEAVED, TRIA_LAYOUT_PAGED>(p, st)
               : launch_t<G, TRIA_PAIR_INTERLEAVED, TRIA_LAYOUT_CONTIGUOUS>(p, st);
}

static_assert(sizeof(TcSmem<8>) + 1024 <= 232448, "shared memory of the G=8 kernel");
static_assert(sizeof(TcSmem<16>) + 1024 <= 232448, "shared memory of the G=16 kernel");

}  // namespace

cudaError_t launch_score(const ScoreParams &p, cudaStream_t st) {
  if (p.geo.mode == TRIA_OFFSET_MAX) return launch_score_max(p, st);
  if (p.geo.grouped) return launch_score_grouped(p, st);
  switch (p.geo.g) {
    case 1: return launch_g<1>(p, st);
    case 2: return launch_g<2>(p, st);
    case 4: return launch_g<4>(p, st);
    case 8: return launch_g<8>(p, st);
    case 16: return launch_g<16>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tria
