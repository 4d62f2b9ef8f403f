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
//               memory, and tcgen05.commit.  Consecutive steps accumulate
//               into NACC different partial accumulators (summed by the
//               epilogue), so they do not wait on each other's results;
// and, in the fused pass (academ.us article 2607.13051, sec. 4: the
// normalize-then-max consumes the per-head scores of the whole unit, so it
// starts once the unit's last key is scored):
//   warp 10     item warp: when the compute warps finish an item (all its
//               raw scores and moment partials written) it counts the item
//               in the unit's device-wide counter; the block that completes
//               a unit appends it to a device-wide queue of due tails;
//   warps 11-14 tail warps: take the next due unit from that queue, whichever
//               block completed it, and run its tail: the mean and std of
//               each head from the moment partials, the aggregated order
//               keys (read from the raw scores, which are still in L2), and
//               the radix selection over the keys into the ascending kept
//               list.  They run next to the scoring roles, on the issue
//               slots those leave free.  Taking units from one queue keeps
//               the tails spread over the blocks: a block slowed by its
//               tails would otherwise finish the last items of more units
//               and draw still more tails.  The tail warps wait on other
//               blocks, so the kernel is launched cooperatively (every block
//               resident).
// The raw scores then never need to reach HBM: the tail reads them back
// from L2 within microseconds of their writing and drops the lines.
// Every wait is bounded (ScoreParams::wait_ns); on expiry the kernel flags
// status bit 1, lets its own loads and MMAs land, frees its tensor memory
// and returns.
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
constexpr int kItemWarp = kComputeWarps + 2;
constexpr int kTailWarp0 = kComputeWarps + 3;
constexpr int kTailWarps = 4;
constexpr int kTailThreads = 32 * kTailWarps;
constexpr int kTailBar = 2;                 // named barrier of the tail warps
constexpr int kTailLoads = 8;               // float4 raw-score loads in flight per tail thread
constexpr int kItemRing = 8;                // finished-item records in flight
template <bool FUSED>
__host__ __device__ constexpr int tc_threads() {
  return 32 * (kComputeWarps + 2 + (FUSED ? 1 + kTailWarps : 0));
}
// The epilogue of tile i runs after the magnitudes of tile i + 2, so two MMA
// chains are in flight while the compute warps work; magnitude tiles and
// accumulators rotate through kNB tensor-memory buffers (tile i uses i % kNB,
// whose previous user, tile i - kNB, finished its epilogue before the
// magnitudes of tile i - 1).
constexpr int kNB = 4;
constexpr uint32_t kTmemCols = 512;         // [0, 256): accumulators; [256, 512): magnitude tiles
constexpr uint32_t kTmemMag = 256;

template <int G, bool FUSED>
struct TcCfg {
  static constexpr int NCOL = (2 * G < 16) ? 16 : 2 * G;   // MMA N
  // K ring depth: the fused pass gives shared memory to the tail
  static constexpr int STAGES = FUSED ? ((G <= 8) ? 5 : 4) : ((G <= 8) ? 6 : 5);
  static constexpr int GQ = (G >= kBandGroups) ? G / kBandGroups : 1;  // heads per band group
  static constexpr int BBLK = NCOL * 128;                  // bytes per 64-wide K block of B
  // Consecutive K-steps of a tile accumulate into NACC partial accumulators
  // (summed by the epilogue): an N = 16 MMA is a few tensor-pipe cycles, far
  // below the latency of its result, so a single accumulator would chain the
  // tile's 16 MMAs on that latency
  static constexpr int NACC = (NCOL <= 16) ? 4 : 2;
  static_assert(kNB * NACC * NCOL <= 256, "accumulator columns");
};

// A finished item, from the compute warps to the item warp.
struct ItemPost {
  long long u;
  int N, end;
};

struct TailArea {
  uint32_t hist[kHistBins];
  uint2 list[kListCap];
  GroupScalars<kTailWarps> sc;
  ItemPost irec[kItemRing];
  int act[2];                               // the unit the tail group takes next (-1: none)
  alignas(8) uint64_t idone[kItemRing];
  alignas(8) uint64_t ifree[kItemRing];
};

template <bool FUSED>
struct TailPart {};
template <>
struct TailPart<true> {
  TailArea t;
};

template <int G, bool FUSED>
struct TcSmem {
  alignas(1024) uint8_t k[TcCfg<G, FUSED>::STAGES][2][kHalfBlock];
  alignas(1024) uint8_t b[2][4][TcCfg<G, FUSED>::BBLK];
  alignas(8) uint64_t full[TcCfg<G, FUSED>::STAGES];
  alignas(8) uint64_t kempty[TcCfg<G, FUSED>::STAGES];
  alignas(8) uint64_t aready[kNB];
  alignas(8) uint64_t accfull[kNB];
  alignas(8) uint64_t bempty[2];
  SubRec rec[TcCfg<G, FUSED>::STAGES];
  alignas(16) int seq_items[kMaxSeqTable];
  int seq_len[kMaxSeqTable];
  uint32_t tmem_base;
  volatile int abort_flag;
  TailPart<FUSED> tp;
  __device__ __forceinline__ uint8_t *bbuf(int i) { return &b[i][0][0]; }
};

// ---------------------------------------------------------------------------
// MMA issuer (one lane)
// ---------------------------------------------------------------------------
template <int G, bool FUSED>
__device__ void mma_issuer(const ScoreParams &p, TcSmem<G, FUSED> &sm, uint32_t tmem,
                           const WaitCtl &wc) {
  using Cfg = TcCfg<G, FUSED>;
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
template <int G, bool FUSED>
__device__ __forceinline__ bool epilogue(const ScoreParams &p, TcSmem<G, FUSED> &sm, uint32_t tmem,
                                         int j, const EpRec &pr, int q, int rg, int lane,
                                         double (&msum)[TcCfg<G, FUSED>::GQ],
                                         double (&msq)[TcCfg<G, FUSED>::GQ], const WaitCtl &wc) {
  constexpr int NCOL = TcCfg<G, FUSED>::NCOL, GQ = TcCfg<G, FUSED>::GQ;
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
    constexpr int NACC = TcCfg<G, FUSED>::NACC;
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

template <int G, int PAIR, bool FUSED>
__device__ void compute(const ScoreParams &p, TcSmem<G, FUSED> &sm, uint32_t tmem, int tid,
                        const WaitCtl &wc) {
  constexpr int ST = TcCfg<G, FUSED>::STAGES, GQ = TcCfg<G, FUSED>::GQ;
  const int warp = tid >> 5, lane = tid & 31;
  const int q = warp >> 2, rg = warp & 3, r = rg * 32 + lane;  // band group, quadrant, row
  const uint32_t mag_base = tmem + ((uint32_t)(32 * rg) << 16) + kTmemMag;
  double msum[GQ], msq[GQ];
#pragma unroll
  for (int g = 0; g < GQ; ++g) msum[g] = msq[g] = 0.0;
  int posted = 0;
  // fused pass: hand a finished item (or the end) to the item warp
  auto post = [&](const EpRec &e, int end) -> bool {
    if constexpr (FUSED) {
      TailArea &ta = sm.tp.t;
      const int slot = posted % kItemRing;
      if (posted >= kItemRing &&
          !warp_wait(&ta.ifree[slot], ((posted / kItemRing) - 1) & 1, wc, lane))
        return false;
      if (warp == 0 && lane == 0) {
        ItemPost &ip = ta.irec[slot];
        ip.u = e.u;
        ip.N = e.N;
        ip.end = end;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ta.idone[slot]);
      ++posted;
    }
    return true;
  };
  auto ep = [&](int j, const EpRec &e) -> bool {
    if (!epilogue<G, FUSED>(p, sm, tmem, j, e, q, rg, lane, msum, msq, wc)) return false;
    if (FUSED && (e.flags & kFlagLast)) return post(e, 0);
    return true;
  };
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
    if (i >= 2 && !ep(i - 2, older)) return -1;
    if (end) {
      if (i >= 1 && !ep(i - 1, other)) return -1;
      EpRec none{};
      return post(none, 1) ? 1 : -1;
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

// ---------------------------------------------------------------------------
// fused pass: item warp and tail warps
// ---------------------------------------------------------------------------
__device__ __forceinline__ int ld_acquire(const int32_t *a) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(int32_t *a, int v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}

template <int G>
__device__ void item_warp(const ScoreParams &p, TailArea &ta, int lane, const WaitCtl &wc) {
  const Geom &geo = p.geo;
  for (int j = 0;; ++j) {
    const int slot = j % kItemRing;
    if (!warp_wait(&ta.idone[slot], (j / kItemRing) & 1, wc, lane)) return;
    const ItemPost ip = ta.irec[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(&ta.ifree[slot]);  // the record is copied
    if (ip.end) return;
    // Count the item in the unit's device-wide counter.  The compute warps'
    // raw-score and moment writes precede their arrivals on idone (release,
    // block scope), this warp acquired them by its wait, and the fence
    // below (cumulative) orders them before the count at device scope; the
    // block that takes the last count fences again and publishes the unit
    // with a release store, which the tail warps that take it acquire.
    if (lane == 0) {
      const int ntiles = unit_tiles(ip.N, geo.window, geo.sinks);
      __threadfence();
      const uint32_t old = atomicAdd(p.unit_done + ip.u, 1u);
      if (old + 1u == (uint32_t)ntiles) {
        __threadfence();
        const uint32_t at = atomicAdd(p.tq, 1u);
        st_release(p.tailq + at, (int)ip.u);
      }
    }
    __syncwarp();
  }
}

// Tail warp 0: the next due unit (device-wide order), or -1 when every unit
// the pass compresses has been taken, or on abort or expiry.  Lane 0 claims
// the next queue position and waits (bounded) until a block publishes the
// unit that completes there.
__device__ int claim_tail(const ScoreParams &p, int lane, const WaitCtl &wc) {
  int u = -1;
  if (lane == 0) {
    const uint32_t at = atomicAdd(p.tq + 1, 1u);
    if (at < __ldcg(p.tq + 2)) {
      const uint64_t t0 = global_timer();
      for (;;) {
        u = ld_acquire(p.tailq + at);
        if (u >= 0) break;
        if (*wc.abort_flag) break;
        if (global_timer() - t0 > wc.limit_ns) {
          flag_expiry(wc);
          break;
        }
        __nanosleep(500);
      }
    }
  }
  return __shfl_sync(kFull, u, 0);
}

template <int G>
__device__ void run_tail(const ScoreParams &p, TailArea &ta, long long u, int tt) {
  const Geom &geo = p.geo;
  const int s = (int)(u / ((int64_t)geo.nl * geo.hkv));
  const int lrel = (int)((u / geo.hkv) % geo.nl);
  const int N = unit_len(geo, s, lrel);
  const int C = N - geo.window - geo.sinks;
  const int B = geo.lbudget[lrel];
  unit_norm<G, kTailBar, kTailThreads>(p.moments + u * geo.tiles_max * kRowGroups * G * 2,
                                       unit_tiles(N, geo.window, geo.sinks), C, tt, ta.sc);
  clear_words<kTailThreads>(ta.hist, kHistBins, tt);
  csync<kTailBar, kTailThreads>();
  const float *raw = p.raw + u * p.raw_stride;
  uint32_t *keys = p.keys + u * p.keys_stride;
  unit_keys<G, kTailThreads, kTailLoads, true>(raw, C, ta.sc.mean, ta.sc.inv, keys, ta.hist, tt);
  csync<kTailBar, kTailThreads>();
  int32_t *kept = p.kept + u * geo.budget;
  select_global<kTailBar, kTailThreads>(keys, C, B - geo.window - geo.sinks, N, B, geo.window,
                                        geo.sinks, kept, ta.hist, ta.list, ta.sc, tt);
  for (int j = B + tt; j < geo.budget; j += kTailThreads) kept[j] = -1;
  csync<kTailBar, kTailThreads>();
  if (p.discard) {
    // the unit's raw scores and keys are dead: drop their lines from L2
    // without writing them back
    const int64_t rl = ((int64_t)C * G * 4 + 127) / 128, kl = ((int64_t)C * 4 + 127) / 128;
    for (int64_t i = tt; i < rl; i += kTailThreads) discard_line(raw + i * 32);
    for (int64_t i = tt; i < kl; i += kTailThreads) discard_line(keys + i * 32);
  }
}

template <int G>
__device__ void tail_warps(const ScoreParams &p, TailArea &ta, int tt, const WaitCtl &wc) {
  const int lane = tt & 31;
  // tail warp 0 takes each due unit and hands it to the group through
  // shared memory (the other tail warps wait at the group barrier only, so
  // no tail warp is left waiting for one that stopped)
  for (int j = 0;; ++j) {
    if (tt < 32) {
      const int u = claim_tail(p, lane, wc);
      if (lane == 0) ta.act[j & 1] = u;
    }
    csync<kTailBar, kTailThreads>();
    const int u = ta.act[j & 1];
    if (u < 0) return;
    run_tail<G>(p, ta, u, tt);
  }
}

template <int G, int PAIR, int LAYOUT, bool FUSED>
__global__ void __launch_bounds__(tc_threads<FUSED>(), 1)
    score_tc_kernel(const __grid_constant__ ScoreParams p) {
  using Cfg = TcCfg<G, FUSED>;
  extern __shared__ uint8_t smem_dyn[];
  TcSmem<G, FUSED> &sm = *reinterpret_cast<TcSmem<G, FUSED> *>(
      (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
  const Geom &geo = p.geo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int NT = tc_threads<FUSED>();

  for (int i = tid; i <= geo.n_seq; i += NT) sm.seq_items[i] = p.seq_items[i];
  for (int i = tid; i < geo.n_seq; i += NT) sm.seq_len[i] = unit_len(geo, i, 0);
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
    if constexpr (FUSED) {
      TailArea &ta = sm.tp.t;
      for (int i = 0; i < kItemRing; ++i) {
        mbar_init(&ta.idone[i], kComputeWarps);
        mbar_init(&ta.ifree[i], 1);
      }
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
    compute<G, PAIR, FUSED>(p, sm, tmem, tid, wc);
  } else if (warp == kProducerWarp) {
    producer<Cfg::STAGES, LAYOUT>(p, sm, n_items, lane, wc);
  } else if (warp == kMmaWarp) {
    if (lane == 0) mma_issuer<G, FUSED>(p, sm, tmem, wc);
    __syncwarp();
  } else if constexpr (FUSED) {
    if (warp == kItemWarp) item_warp<G>(p, sm.tp.t, lane, wc);
    else tail_warps<G>(p, sm.tp.t, tid - 32 * kTailWarp0, wc);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int G, int PAIR, int LAYOUT, bool FUSED>
cudaError_t launch_t(const ScoreParams &p, cudaStream_t st) {
  auto kern = score_tc_kernel<G, PAIR, LAYOUT, FUSED>;
  const int smem = (int)sizeof(TcSmem<G, FUSED>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if constexpr (FUSED) {
    // the tail warps wait on other blocks: every block must be resident
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sms);
    cfg.blockDim = dim3((unsigned)tc_threads<FUSED>());
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
  } else {
    kern<<<sms, tc_threads<FUSED>(), smem, st>>>(p);
    return cudaGetLastError();
  }
}

template <int G, bool FUSED>
cudaError_t launch_g(const ScoreParams &p, cudaStream_t st) {
  const bool paged = p.cache.layout == TRIA_LAYOUT_PAGED;
  if (p.geo.pairing == TRIA_PAIR_NEOX)
    return paged ? launch_t<G, TRIA_PAIR_NEOX, TRIA_LAYOUT_PAGED, FUSED>(p, st)
                 : launch_t<G, TRIA_PAIR_NEOX, TRIA_LAYOUT_CONTIGUOUS, FUSED>(p, st);
  return paged ? launch_t<G, TRIA_PAIR_INTERLEAVED, TRIA_LAYOUT_PAGED, FUSED>(p, st)
               : launch_t<G, TRIA_PAIR_INTERLEAVED, TRIA_LAYOUT_CONTIGUOUS, FUSED>(p, st);
}

template <bool FUSED>
cudaError_t launch_f(const ScoreParams &p, cudaStream_t st) {
  switch (p.geo.g) {
    case 1: return launch_g<1, FUSED>(p, st);
    case 2: return launch_g<2, FUSED>(p, st);
    case 4: return launch_g<4, FUSED>(p, st);
    case 8: return launch_g<8, FUSED>(p, st);
    case 16: return launch_g<16, FUSED>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

static_assert(sizeof(TcSmem<8, false>) + 1024 <= 232448, "shared memory of the G=8 kernel");
static_assert(sizeof(TcSmem<16, false>) + 1024 <= 232448, "shared memory of the G=16 kernel");
static_assert(sizeof(TcSmem<8, true>) + 1024 <= 232448, "shared memory of the G=8 fused kernel");
static_assert(sizeof(TcSmem<16, true>) + 1024 <= 232448, "shared memory of the G=16 fused kernel");
static_assert(sizeof(GroupScalars<kTailWarps>) % 8 == 0, "tail scalars");

}  // namespace

cudaError_t launch_score(const ScoreParams &p, bool fused, cudaStream_t st) {
  if (p.geo.mode == TRIA_OFFSET_MAX) return launch_score_max(p, st);
  return fused ? launch_f<true>(p, st) : launch_f<false>(p, st);
}

}  // namespace tria
