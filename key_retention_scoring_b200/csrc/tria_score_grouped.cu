// Offset-mean scoring for paged caches in whole blocks: one 128-row tile is
// one paged block of every KV head of a (sequence, layer), BS = 128 / HKV
// tokens x HKV heads.
//
// In the NHD paged layout the heads of a token are adjacent (256 bytes
// each), so a tile of one head (tria_score_tc.cu) reads 128-byte pieces
// 256 HKV bytes apart; here each tile is the block's full BS x HKV x 256
// bytes, two TMA boxes of {64 dims, BS tokens, HKV heads}.  Rows are
// head-major (row = head BS + token).  Each row must meet its own head's
// coefficients, so the B operand holds the HKV units' coefficient columns
// side by side (2G each, no padding: N = 2 G HKV, 16 <= N <= 128, written so
// by the coefficient kernel):
//   D[128 x N] = [ktilde | m_hi | m_lo] (128 x 256) . [B_0 | ... | B_{HKV-1}]
// and row r keeps the block of columns of head r / BS (the other blocks
// are computed and ignored: the tensor pipe has the room).  The score of a
// row is the same sum as in the one-head kernel (academ.us article
// 2607.13051, Eqs. 3, 6, 7; the norm-term reading of the ghidav.me blog,
// "The Method").
//
// Roles as in the one-head kernel: warps 0-7 compute (magnitudes of tile i,
// then the epilogue of tile i - 1), warp 8 producer (TMA), warp 9 MMA issuer.
// Tensor memory holds two buffers of N accumulator and 64 magnitude columns.
// A scheduling item is a 1024-slot range of a (sequence, layer), all heads;
// the coefficient image (one buffer) is reloaded when an item's (sequence,
// layer) differs from the one it holds, once the previous item's MMAs are
// done.  Waits and the abort path as in tria_tc.cuh.
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

template <int G, int HKV>
struct GrpCfg {
  static constexpr int NCOL = 2 * G;                        // one unit's columns (hi, lo per head)
  static constexpr int N = HKV * NCOL;                      // MMA N
  static constexpr int BS = kRows / HKV;                    // tokens per tile (the block size)
  static constexpr int STAGES = (N <= 64) ? 5 : 4;
  static constexpr int GQ = (G >= kBandGroups) ? G / kBandGroups : 1;
  static constexpr int BBLK = N * 128;                      // bytes per 64-wide K block of B
  static constexpr uint32_t MAG0 = 2 * N;                   // magnitude buffers after two accumulators
  static_assert(N % 16 == 0 && N >= 16 && N <= 128, "MMA N of the grouped kernel");
  static_assert(MAG0 + 2 * 64 <= kTmemCols, "tensor memory of the grouped kernel");
};

template <int G, int HKV>
struct GrpSmem {
  alignas(1024) uint8_t k[GrpCfg<G, HKV>::STAGES][2][kHalfBlock];
  alignas(1024) uint8_t b[4][GrpCfg<G, HKV>::BBLK];
  alignas(8) uint64_t full[GrpCfg<G, HKV>::STAGES];
  alignas(8) uint64_t kempty[GrpCfg<G, HKV>::STAGES];
  alignas(8) uint64_t aready[2];
  alignas(8) uint64_t accfull[2];
  alignas(8) uint64_t bempty[2];
  SubRec rec[GrpCfg<G, HKV>::STAGES];
  alignas(16) int seq_items[kMaxSeqTable];
  int seq_len[kMaxSeqTable];
  uint32_t tmem_base;
  volatile int abort_flag;
};

// ---------------------------------------------------------------------------
// producer: items (sequence, layer, 1024-slot range) in claim order; per
// tile one paged block, two TMA boxes of every head.  Item m's MMAs are done
// when phase m >> 1 of bempty[m & 1] completes; at every item start the
// producer waits for the item two back (never more than one phase behind
// either barrier), and before reloading the coefficient image for the
// previous item.
// ---------------------------------------------------------------------------
template <int G, int HKV>
__device__ void producer_grp(const ScoreParams &p, GrpSmem<G, HKV> &sm, int n_items, int lane,
                             const WaitCtl wc) {
  using Cfg = GrpCfg<G, HKV>;
  constexpr int ST = Cfg::STAGES, BS = Cfg::BS;
  constexpr uint32_t kImg = (uint32_t)Cfg::N * 512u;  // the (sequence, layer)'s image: N x 256 bf16
  const Geom &geo = p.geo;
  const uint64_t pol = evict_first_policy();
  const int W = geo.window, S = geo.sinks;
  int i = 0, items = 0, sub = 0, sub_first = 0, sub_end = 0;
  int s = 0, lrel = 0, tile = 0, N = 0, tbase = 0;
  long long u0 = 0, b_unit = -1;
  bool ok = true;
  uint32_t nxt = 0;
  if (lane == 0) nxt = atomicAdd(p.item_counter, 1u);
  for (;;) {
    if (sub == sub_end) {
      const int it = (int)__shfl_sync(kFull, nxt, 0);
      if (it >= n_items) break;
      if (lane == 0) nxt = atomicAdd(p.item_counter, 1u);
      int lo = 0, hi = geo.n_seq - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sm.seq_items[mid] <= it) lo = mid; else hi = mid - 1;
      }
      s = lo;
      if (!geo.per_layer) {
        const int ntiles = (sm.seq_items[s + 1] - sm.seq_items[s]) / geo.nl;
        const int rem = it - sm.seq_items[s];
        lrel = rem / ntiles;
        tile = rem % ntiles;
        N = sm.seq_len[s];
      } else {
        const int32_t *ri = p.row_items + (int64_t)s * geo.nl;
        int cnt = 0;
        for (int l0 = 0; l0 < geo.nl; l0 += 32) {
          const int l = l0 + lane;
          cnt += __popc(__ballot_sync(kFull, l < geo.nl && __ldcg(ri + l) <= it));
        }
        lrel = cnt - 1;
        N = unit_len(geo, s, lrel);
        tile = it - __ldcg(ri + lrel);
      }
      u0 = ((long long)s * geo.nl + lrel) * HKV;
      tbase = (S / kTileKeys + tile) * kTileKeys;
      const int c_lo = max(S, tbase), c_hi = min(N - W, tbase + kTileKeys);
      sub_first = (c_lo - tbase) / BS;
      sub = sub_first;
      sub_end = (c_hi - tbase + BS - 1) / BS;
      ++items;
    }
    const int stage = i % ST;
    if (i >= ST) {
      if (lane == 0) ok = mbar_wait(&sm.kempty[stage], ((i / ST) - 1) & 1, wc);
      ok = __shfl_sync(kFull, ok, 0);
      if (!ok) break;
    }
    const int bpar = (items - 1) & 1;  // this item's completion barrier
    const bool first = (sub == sub_first);
    if (first && items > 2) {
      if (lane == 0) ok = mbar_wait(&sm.bempty[bpar], ((items - 3) >> 1) & 1, wc);
      ok = __shfl_sync(kFull, ok, 0);
      if (!ok) break;
    }
    const bool load_b = first && u0 != b_unit;
    if (load_b && items > 1) {
      if (lane == 0) ok = mbar_wait(&sm.bempty[bpar ^ 1], ((items - 2) >> 1) & 1, wc);
      ok = __shfl_sync(kFull, ok, 0);
      if (!ok) break;
    }
    if (load_b) b_unit = u0;
    const int slot0 = tbase + sub * BS;
    int blk = 0;
    if (lane == 0) blk = p.cache.block_table[(int64_t)s * p.cache.max_blocks + slot0 / BS];
    blk = __shfl_sync(kFull, blk, 0);
    const uint32_t bytes = 2u * kHalfBlock + (load_b ? kImg : 0u);
    if (lane == 0) {
      SubRec &r = sm.rec[stage];
      r.u = u0; r.tile = tile; r.N = N; r.slot0 = slot0;
      r.flags = (first ? kFlagFirst : 0) | (sub == sub_end - 1 ? kFlagLast : 0);
      r.bpar = bpar;
      mbar_arrive_expect_tx(&sm.full[stage], bytes);
      if (load_b)
        bulk_load(smem_u32(&sm.b[0][0]), reinterpret_cast<const uint8_t *>(p.btile) + u0 * p.geo.b_bytes,
                  kImg, &sm.full[stage]);
    }
    const uint32_t kdst = smem_u32(&sm.k[stage][0][0]);
    if (lane < 2)
      tma_load_4d(kdst + lane * kHalfBlock, &p.kmap[lrel], lane * 64, 0, 0, blk, &sm.full[stage], pol);
    ++sub;
    ++i;
  }
  if (ok) {
    const int stage = i % ST;
    if (i >= ST) {
      if (lane == 0) ok = mbar_wait(&sm.kempty[stage], ((i / ST) - 1) & 1, wc);
      ok = __shfl_sync(kFull, ok, 0);
    }
    if (ok && lane == 0) {
      sm.rec[stage].flags = kFlagEnd;
      mbar_arrive(&sm.full[stage]);
    }
    if (ok) ++i;
  }
  if (!ok && lane == 0) {
    for (int j = (i > ST ? i - ST : 0); j < i; ++j) mbar_drain(&sm.full[j % ST], (j / ST) & 1, wc.status);
  }
}

// ---------------------------------------------------------------------------
// MMA issuer (one lane): 8 K-steps with A = the K tile in shared memory, 8
// with A = the magnitude tile in tensor memory, into accumulator i & 1
// ---------------------------------------------------------------------------
template <int G, int HKV>
__device__ void mma_issuer_grp(GrpSmem<G, HKV> &sm, uint32_t tmem, const WaitCtl wc) {
  using Cfg = GrpCfg<G, HKV>;
  constexpr int ST = Cfg::STAGES, N = Cfg::N, BBLK = Cfg::BBLK;
  constexpr uint32_t idesc = idesc_bf16_m128_n(N);
  const uint64_t da0 = sw128_desc(smem_u32(&sm.k[0][0][0]));
  const uint64_t db = sw128_desc(smem_u32(&sm.b[0][0]));
  constexpr uint32_t kStageBytes = 2 * kHalfBlock;
  int i = 0;
  for (;; ++i) {
    const int ab = i & 1;
    if (!mbar_wait(&sm.aready[ab], (i >> 1) & 1, wc)) break;
    tc_fence_after();
    const int stage = i % ST;
    const SubRec &rec = sm.rec[stage];
    const int flags = rec.flags, bpar = rec.bpar;
    if (flags & kFlagEnd) break;
    const uint32_t d = tmem + (uint32_t)(ab * N);
    const uint32_t ta = tmem + Cfg::MAG0 + (uint32_t)(ab * 64);
    const uint64_t da = da0 + (uint64_t)((stage * kStageBytes) >> 4);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t ao = (s >> 2) * kHalfBlock + (s & 3) * 32;
      const uint32_t bo = (s >> 2) * BBLK + (s & 3) * 32;
      mma_bf16(d, da + (ao >> 4), db + (bo >> 4), idesc, s > 0 ? 1u : 0u);
    }
    mma_commit(&sm.kempty[stage]);
#pragma unroll
    for (int s = 8; s < 16; ++s) {
      const uint32_t bo = (s >> 2) * BBLK + (s & 3) * 32;
      mma_bf16_ta(d, ta + (uint32_t)((s - 8) * 8), db + (bo >> 4), idesc, 1u);
    }
    if (flags & kFlagLast) mma_commit(&sm.bempty[bpar]);
    mma_commit(&sm.accfull[ab]);
  }
  if (i > 0) mbar_drain(&sm.accfull[(i - 1) & 1], ((i - 1) >> 1) & 1, wc.status);
}

// ---------------------------------------------------------------------------
// compute warps
// ---------------------------------------------------------------------------
template <int PAIR>
__device__ __forceinline__ void mags_grp(const uint8_t *kt, uint32_t tcol, int r, int q) {
  constexpr int W = kBandsPerThread / 2;
  uint32_t hi[W], lo[W];
  mags_regs<PAIR, kBandsPerThread>(kt, r, q, hi, lo);
  tmem_st<W>(tcol + (uint32_t)(W * q), hi);
  tmem_st<W>(tcol + (uint32_t)(32 + W * q), lo);
}

// Epilogue of tile j (record pr): this thread's row r = 32 rg + lane is token
// r % BS of head r / BS (a warp holds 32 / BS heads, or part of one); its GQ
// heads of band group q are the columns head NCOL + q 2 GQ .. of the
// accumulator.  Raw scores, fp64 moment sums per head, and each head's item
// partial (row group rg) after the item's last tile.
template <int G, int HKV>
__device__ __forceinline__ bool epilogue_grp(const ScoreParams &p, GrpSmem<G, HKV> &sm, uint32_t tmem,
                                             int j, const EpRec &pr, int q, int rg, int lane,
                                             double (&msum)[GrpCfg<G, HKV>::GQ],
                                             double (&msq)[GrpCfg<G, HKV>::GQ], const WaitCtl wc) {
  using Cfg = GrpCfg<G, HKV>;
  constexpr int NCOL = Cfg::NCOL, N = Cfg::N, GQ = Cfg::GQ, BS = Cfg::BS;
  // rows are head-major (row = head BS + token): a warp's 32 rows hold HW heads
  constexpr int HW = (BS >= 32) ? 1 : 32 / BS;
  const Geom &geo = p.geo;
  const bool active = (G >= kBandGroups) || q < G;
  const int r = 32 * rg + lane, myh = r / BS, h_first = (32 * rg) / BS;
  if (!warp_wait(&sm.accfull[j & 1], (j >> 1) & 1, wc, lane)) return false;
  tc_fence_after();
  if (pr.flags & kFlagFirst) {
#pragma unroll
    for (int g = 0; g < GQ; ++g) msum[g] = msq[g] = 0.0;
  }
  if (active) {
    uint32_t v[2 * GQ];
    const uint32_t col = tmem + ((uint32_t)(32 * rg) << 16) + (uint32_t)((j & 1) * N + q * 2 * GQ);
    {
      uint32_t t[HW][2 * GQ];
#pragma unroll
      for (int a = 0; a < HW; ++a) tmem_ld_nowait<2 * GQ>(col + (uint32_t)((h_first + a) * NCOL), t[a]);
      tmem_wait_ld();
#pragma unroll
      for (int a = 0; a < HW; ++a)
        if (h_first + a == myh) {
#pragma unroll
          for (int c = 0; c < 2 * GQ; ++c) v[c] = t[a][c];
        }
    }
    const int slot = pr.slot0 + r % BS;
    if (slot >= geo.sinks && slot < pr.N - geo.window) {
      float sc[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        sc[g] = __uint_as_float(v[2 * g]) + __uint_as_float(v[2 * g + 1]);
        msum[g] += (double)sc[g];
        msq[g] = fma((double)sc[g], (double)sc[g], msq[g]);
      }
      float *dst = p.raw + (pr.u + myh) * p.raw_stride + (int64_t)(slot - geo.sinks) * G + q * GQ;
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
  tc_fence_before();
  if ((pr.flags & kFlagLast) && active) {
    // the lanes of one head: a run of min(BS, 32) lanes
    constexpr int RUN = (BS >= 32) ? 32 : BS;
#pragma unroll
    for (int g = 0; g < GQ; ++g) {
#pragma unroll
      for (int o = RUN / 2; o >= 1; o >>= 1) {
        msum[g] += __shfl_xor_sync(kFull, msum[g], o);
        msq[g] += __shfl_xor_sync(kFull, msq[g], o);
      }
    }
    if (lane % RUN == 0) {
      // this warp's partial in its own row group; a head's row groups that
      // none of its warps covers (BS < 128) get zeros from its first warp
      const int h = myh;
      double *mu = p.moments + ((pr.u + h) * geo.tiles_max + pr.tile) * kRowGroups * G * 2;
      const int rg0 = (h * BS) / 32, rg1 = (h * BS + BS - 1) / 32;  // the head's warps
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        mu[(rg * G + q * GQ + g) * 2] = msum[g];
        mu[(rg * G + q * GQ + g) * 2 + 1] = msq[g];
      }
      if (rg == rg0) {
        for (int o = 0; o < kRowGroups; ++o) {
          if (o >= rg0 && o <= rg1) continue;
#pragma unroll
          for (int g = 0; g < GQ; ++g) {
            mu[(o * G + q * GQ + g) * 2] = 0.0;
            mu[(o * G + q * GQ + g) * 2 + 1] = 0.0;
          }
        }
      }
    }
  }
  return true;
}

template <int G, int HKV, int PAIR>
__device__ void compute_grp(const ScoreParams &p, GrpSmem<G, HKV> &sm, uint32_t tmem, int tid,
                            const WaitCtl wc) {
  using Cfg = GrpCfg<G, HKV>;
  constexpr int ST = Cfg::STAGES, GQ = Cfg::GQ;
  const int warp = tid >> 5, lane = tid & 31;
  const int q = warp >> 2, rg = warp & 3, r = rg * 32 + lane;
  const uint32_t mag = tmem + ((uint32_t)(32 * rg) << 16) + Cfg::MAG0;
  double msum[GQ], msq[GQ];
#pragma unroll
  for (int g = 0; g < GQ; ++g) msum[g] = msq[g] = 0.0;
  EpRec prev{};
  for (int i = 0;; ++i) {
    const int stage = i % ST;
    if (!warp_wait(&sm.full[stage], (i / ST) & 1, wc, lane)) return;
    const SubRec &rc = sm.rec[stage];
    const bool end = (rc.flags & kFlagEnd) != 0;
    EpRec cur{};
    if (!end) {
      cur = ep_of(rc);
      // magnitude buffer i & 1: its previous reader, the MMAs of tile i - 2,
      // finished before this warp's epilogue of tile i - 2
      mags_grp<PAIR>(&sm.k[stage][0][0], mag + (uint32_t)((i & 1) * 64), r, q);
      tmem_wait_st();
      tc_fence_before();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.aready[i & 1]);
    if (i >= 1 && !epilogue_grp<G, HKV>(p, sm, tmem, i - 1, prev, q, rg, lane, msum, msq, wc)) return;
    if (end) return;
    prev = cur;
  }
}

template <int G, int HKV, int PAIR>
__global__ void __launch_bounds__(kThreads, 1) score_grp_kernel(const __grid_constant__ ScoreParams p) {
  using Cfg = GrpCfg<G, HKV>;
  extern __shared__ uint8_t smem_dyn[];
  GrpSmem<G, HKV> &sm = *reinterpret_cast<GrpSmem<G, HKV> *>(
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
      mbar_init(&sm.bempty[i], 1);
    }
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
    compute_grp<G, HKV, PAIR>(p, sm, tmem, tid, wc);
  } else if (warp == kProducerWarp) {
    producer_grp<G, HKV>(p, sm, n_items, lane, wc);
  } else if (warp == kMmaWarp) {
    if (lane == 0) mma_issuer_grp<G, HKV>(sm, tmem, wc);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int G, int HKV, int PAIR>
cudaError_t launch_grp_t(const ScoreParams &p, cudaStream_t st) {
  auto kern = score_grp_kernel<G, HKV, PAIR>;
  const int smem = (int)sizeof(GrpSmem<G, HKV>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  kern<<<sms, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <int G, int HKV>
cudaError_t launch_grp_h(const ScoreParams &p, cudaStream_t st) {
  if constexpr (2 * G * HKV < 16) {
    return cudaErrorInvalidValue;  // N < 16: not selected by the geometry
  } else {
    if (p.geo.pairing == TRIA_PAIR_NEOX) return launch_grp_t<G, HKV, TRIA_PAIR_NEOX>(p, st);
    return launch_grp_t<G, HKV, TRIA_PAIR_INTERLEAVED>(p, st);
  }
}

template <int HKV>
cudaError_t launch_grp_g(const ScoreParams &p, cudaStream_t st) {
  switch (p.geo.g) {
    case 1: return launch_grp_h<1, HKV>(p, st);
    case 2: return launch_grp_h<2, HKV>(p, st);
    case 4: return launch_grp_h<4, HKV>(p, st);
    case 8: return launch_grp_h<8, HKV>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

static_assert(sizeof(GrpSmem<8, 8>) + 1024 <= 232448, "shared memory of the grouped kernel");

}  // namespace

cudaError_t launch_score_grouped(const ScoreParams &p, cudaStream_t st) {
  switch (p.geo.hkv) {
    case 2: return launch_grp_g<2>(p, st);
    case 4: return launch_grp_g<4>(p, st);
    case 8: return launch_grp_g<8>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tria
