// Scoring kernel of the compression pass on the sm_100a tensor cores.
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
//   warp 16     producer: TMA tensor loads of 128-slot K tiles (two 64-dim
//               boxes, or one box per paged block) into a ring of 128-byte-
//               swizzled K-major tiles, plus the unit's coefficient image
//               (one bulk copy per item); completion as mbarrier tx bytes;
//   warp 17     one lane issues tcgen05.mma (M=128, N=16|32, K=16): 8 steps
//               with A = the K tile in shared memory (then the K stage is
//               released), 8 steps with A = the magnitude tile in tensor
//               memory, and tcgen05.commit.  Consecutive steps accumulate
//               into NACC different partial accumulators (summed by the
//               epilogue), so they do not wait on each other's results;
//   warps 0-7   band magnitudes -> tensor memory (tcgen05.st; warp w takes
//               rows 32(w%4).. and bands 32(w/4)..), then, two tiles later,
//               the epilogue (tcgen05.ld, raw scores, fp64 moment partials).
//               Magnitude tiles and accumulators rotate through kNB
//               tensor-memory buffers, so two MMA chains stay in flight.
// Normalize-then-max and the selection run in the next kernel (tail_kernel).
// Every wait is bounded (2 s); on expiry the kernel flags status bit 1, lets
// its own loads and MMAs land, frees its tensor memory and returns.
#include <cuda_bf16.h>

#include "tria_device.cuh"

namespace tria {
namespace {

using namespace dev;

constexpr int kRows = 128;                  // keys per MMA tile (M)
constexpr int kBandGroups = 2;              // compute warps per 32-row quadrant of a tile
constexpr int kBandsPerThread = kBands / kBandGroups;
constexpr int kComputeWarps = 4 * kBandGroups;
constexpr int kProducerWarp = kComputeWarps;
constexpr int kMmaWarp = kComputeWarps + 1;
constexpr int kTcThreads = 32 * (kComputeWarps + 2);
constexpr int kHalfBlock = kRows * 128;     // 128 rows x 64 bf16, swizzled
constexpr int kFlagFirst = 1, kFlagLast = 2, kFlagEnd = 4;
// The epilogue of tile i runs after the magnitudes of tile i + 2, so two MMA
// chains are in flight while the compute warps work; magnitude tiles and
// accumulators rotate through kNB tensor-memory buffers (tile i uses i % kNB,
// whose previous user, tile i - kNB, finished its epilogue before the
// magnitudes of tile i - 1).
constexpr int kNB = 4;
constexpr uint32_t kTmemCols = 512;         // [0, 256): accumulators; [256, 512): magnitude tiles
constexpr uint32_t kTmemMag = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kSuspendNs = 1000000;    // a blocked try_wait sleeps up to 1 ms per call

struct SubRec {
  float *raw;      // the unit's raw scores, candidate 0
  double *mom;     // the item's moment partials
  long long u;
  int s, lrel, h, tile, N;
  int slot0, flags, bpar;  // first slot of the 128-row tile (a multiple of 128)
};

// What the epilogue of a tile needs from its record.
struct EpRec {
  float *raw;
  double *mom;
  int slot0, N, flags;
};

template <int G>
struct TcCfg {
  static constexpr int NCOL = (2 * G < 16) ? 16 : 2 * G;   // MMA N
  static constexpr int STAGES = (G <= 8) ? 6 : 5;
  static constexpr int GQ = (G >= kBandGroups) ? G / kBandGroups : 1;  // heads per band group
  static constexpr int BBLK = NCOL * 128;                  // bytes per 64-wide K block of B
  static constexpr int NACC = (NCOL <= 16) ? 4 : 2;        // partial accumulators per tile
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
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *b, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// try_wait that may suspend the thread (up to kSuspendNs) until the phase
// completes, instead of returning at once.
__device__ __forceinline__ bool mbar_try_sleep(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(addr), "r"(parity), "n"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Bounded wait (one thread) for the phase of `parity`; false on expiry or abort.
__device__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                          int32_t *status) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try(a, parity)) return true;
  const uint64_t t0 = global_timer();
  for (;;) {
    if (mbar_try_sleep(a, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(status, 2);
      return false;
    }
  }
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)),
               "r"(bytes)
               : "memory");
}

// TMA tile load of a 4-D box into shared memory, completion as transaction
// bytes on `bar`.  x (the innermost coordinate) is 0 or 64 elements.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            int z, int w, uint64_t *bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::"
      "cache_hint [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar)),
      "l"(pol)
      : "memory");
}

// Contiguous bulk copy global -> shared (16-byte aligned, multiple of 16 bytes).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}


__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst, int ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, int ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Shared-memory matrix descriptor: 128-byte swizzle, K-major, 8-row groups
// 1024 bytes apart (the tile base is 1024-byte aligned).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(16u >> 4) << 16;    // leading-dimension byte offset (unused when swizzled)
  d |= (uint64_t)(1024u >> 4) << 32;  // stride byte offset
  d |= (uint64_t)1 << 46;             // descriptor version of sm_100
  d |= (uint64_t)2 << 61;             // SWIZZLE_128B
  return d;
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> f32, both K-major.
template <int NCOL>
__host__ __device__ constexpr uint32_t idesc_bf16_m128() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NCOL >> 3) << 17) |
         ((uint32_t)(kRows >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Store N (8 or 16) consecutive 32-bit columns of this thread's tensor-memory lane.
template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 8) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
  } else {
    static_assert(N == 16, "tmem_st width");
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
  }
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D (tmem) (+)= A (tmem, 128 lanes x 16 bf16 in 8 columns) . B (smem descriptor)
__device__ __forceinline__ void mma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Load N consecutive 32-bit columns of this thread's lane (no wait).
template <int N>
__device__ __forceinline__ void tmem_ld_nowait(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 2) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(taddr));
  } else if constexpr (N == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else if constexpr (N == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    static_assert(N == 32, "tmem_ld_nowait width");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
  }
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }

// Squared magnitude of a band from its bf16 parts (the low or high halves
// of re_w / im_w): re^2 (exact in fp32) + im^2 with one rounding.
template <bool HI>
__device__ __forceinline__ float band_sq(uint32_t re_w, uint32_t im_w) {
  float r;
  if constexpr (HI) {
    asm("{\n .reg .b16 a, b, c, d;\n mov.b32 {a, b}, %1;\n mov.b32 {c, d}, %2;\n"
        " fma.rn.f32.bf16 %0, b, b, 0f00000000;\n fma.rn.f32.bf16 %0, d, d, %0;\n}"
        : "=f"(r) : "r"(re_w), "r"(im_w));
  } else {
    asm("{\n .reg .b16 a, b, c, d;\n mov.b32 {a, b}, %1;\n mov.b32 {c, d}, %2;\n"
        " fma.rn.f32.bf16 %0, a, a, 0f00000000;\n fma.rn.f32.bf16 %0, c, c, %0;\n}"
        : "=f"(r) : "r"(re_w), "r"(im_w));
  }
  return r;
}

// Squared magnitude of a band held in one word (re low half, im high half).
__device__ __forceinline__ float band_sq_word(uint32_t w) {
  float r;
  asm("{\n .reg .b16 a, b;\n mov.b32 {a, b}, %1;\n"
      " fma.rn.f32.bf16 %0, a, a, 0f00000000;\n fma.rn.f32.bf16 %0, b, b, %0;\n}"
      : "=f"(r) : "r"(w));
  return r;
}

// Magnitudes of two bands from their squared magnitudes, split into bf16
// hi + lo parts (packed two per word, first band in the low half): hi = the
// top halves of the fp32 bit patterns (truncation), lo = bf16(x - hi)
// rounded to nearest.  |x - hi - lo| <= 2^-16 x.
__device__ __forceinline__ void mag_split(float sa, float sb, uint32_t &hi, uint32_t &lo) {
  const float ma = sqrt_approx(sa), mb = sqrt_approx(sb);
  const uint32_t ua = __float_as_uint(ma), ub = __float_as_uint(mb);
  hi = __byte_perm(ua, ub, 0x7632);
  const float xa = ma - __uint_as_float(ua & 0xffff0000u);
  const float xb = mb - __uint_as_float(ub & 0xffff0000u);
  const __nv_bfloat162 l = __floats2bfloat162_rn(xa, xb);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// ---------------------------------------------------------------------------
// producer warp
// ---------------------------------------------------------------------------
template <int ST, int LAYOUT, class Smem>
__device__ void producer(const ScoreParams &p, Smem &sm, int n_items, int lane) {
  const uint32_t kBBytes = (uint32_t)p.geo.b_bytes;  // one unit's coefficient image
  const Geom &geo = p.geo;
  const uint64_t pol = evict_first_policy();
  const int units_per_seq = geo.nl * geo.hkv;
  const int W = geo.window, S = geo.sinks;
  int i = 0, items = 0, sub = 0, sub_first = 0, sub_end = 0;
  int s = 0, lrel = 0, h = 0, tile = 0, ntiles = 1, N = 0, tbase = 0;
  long long u = 0;
  bool ok = true;
  // the next item index is claimed one item ahead
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
        ntiles = (sm.seq_items[s + 1] - sm.seq_items[s]) / units_per_seq;
        const int rem = it - sm.seq_items[s];
        const int ul = rem / ntiles;
        tile = rem % ntiles;
        lrel = ul / geo.hkv;
        h = ul % geo.hkv;
        N = sm.seq_len[s];
      } else {
        // a length per (sequence, layer): the layer is the last row of the
        // sequence whose first item is at or before this one (rows without
        // items share their successor's start)
        const int32_t *ri = p.row_items + (int64_t)s * geo.nl;
        int cnt = 0;
        for (int l0 = 0; l0 < geo.nl; l0 += 32) {
          const int l = l0 + lane;
          cnt += __popc(__ballot_sync(kFull, l < geo.nl && __ldcg(ri + l) <= it));
        }
        lrel = cnt - 1;
        N = unit_len(geo, s, lrel);
        ntiles = unit_tiles(N, W, S);
        const int rem = it - __ldcg(ri + lrel);
        h = rem / ntiles;
        tile = rem % ntiles;
      }
      u = (long long)s * units_per_seq + lrel * geo.hkv + h;
      tbase = (S / kTileKeys + tile) * kTileKeys;
      const int c_lo = max(S, tbase), c_hi = min(N - W, tbase + kTileKeys);
      sub_first = (c_lo - tbase) / kRows;
      sub = sub_first;
      sub_end = (c_hi - tbase + kRows - 1) / kRows;
      ++items;
    }
    const int stage = i % ST;
    if (i >= ST) {
      if (lane == 0) ok = mbar_wait(&sm.kempty[stage], ((i / ST) - 1) & 1, &sm.abort_flag, p.status);
      ok = __shfl_sync(kFull, ok, 0);
      if (!ok) break;
    }
    const int bpar = (items - 1) & 1;
    const bool first = (sub == sub_first);
    if (first && items > 2) {
      // the coefficient buffer is free once the MMAs of the item two back are done
      if (lane == 0) ok = mbar_wait(&sm.bempty[bpar], ((items - 3) >> 1) & 1, &sm.abort_flag, p.status);
      ok = __shfl_sync(kFull, ok, 0);
      if (!ok) break;
    }
    const int slot0 = tbase + sub * kRows;
    const uint32_t kdst = smem_u32(&sm.k[stage][0][0]);
    uint32_t bytes = first ? kBBytes : 0u;
    int blk = 0;
    bool bvalid = false;
    if (LAYOUT == TRIA_LAYOUT_CONTIGUOUS) {
      bytes += 2u * kHalfBlock;
    } else {
      // one box per block of this tile that holds a candidate row
      const int bs = p.cache.block_size;
      const int slot_b = slot0 + lane * bs;
      const int bidx = slot_b / bs;
      bvalid = lane < kRows / bs && slot_b < N - W && slot_b + bs > S && bidx < p.cache.max_blocks;
      if (bvalid) blk = p.cache.block_table[(int64_t)s * p.cache.max_blocks + bidx];
      bytes += (uint32_t)__popc(__ballot_sync(kFull, bvalid)) * (uint32_t)bs * 256u;
    }
    if (lane == 0) {
      SubRec &r = sm.rec[stage];
      r.u = u; r.s = s; r.lrel = lrel; r.h = h; r.tile = tile; r.N = N; r.slot0 = slot0;
      r.raw = p.raw + u * p.raw_stride;
      r.mom = p.moments + (u * geo.tiles_max + tile) * kRowGroups * geo.g * 2;
      r.flags = (first ? kFlagFirst : 0) | (sub == sub_end - 1 ? kFlagLast : 0);
      r.bpar = bpar;
      mbar_arrive_expect_tx(&sm.full[stage], bytes);
      if (first)
        bulk_load(smem_u32(sm.bbuf(bpar)), reinterpret_cast<const uint8_t *>(p.btile) + u * kBBytes,
                  kBBytes, &sm.full[stage]);
    }
    const CUtensorMap *map = &p.kmap[lrel];
    if (LAYOUT == TRIA_LAYOUT_CONTIGUOUS) {
      if (lane < 2)
        tma_load_4d(kdst + lane * kHalfBlock, map, lane * 64, slot0, h, s, &sm.full[stage], pol);
    } else if (bvalid) {
      const uint32_t off = (uint32_t)(lane * p.cache.block_size * 128);
      tma_load_4d(kdst + off, map, 0, h, 0, blk, &sm.full[stage], pol);
      tma_load_4d(kdst + kHalfBlock + off, map, 64, h, 0, blk, &sm.full[stage], pol);
    }
    ++sub;
    ++i;
  }
  // end marker, read by the compute warps and the MMA issuer
  if (ok) {
    const int stage = i % ST;
    if (i >= ST) {
      if (lane == 0) ok = mbar_wait(&sm.kempty[stage], ((i / ST) - 1) & 1, &sm.abort_flag, p.status);
      ok = __shfl_sync(kFull, ok, 0);
    }
    if (ok && lane == 0) {
      sm.rec[stage].flags = kFlagEnd;
      mbar_arrive(&sm.full[stage]);
    }
    ++i;
  }
  if (!ok && lane == 0) {
    // aborted: let the loads already issued land before the block exits
    for (int j = (i > ST ? i - ST : 0); j < i; ++j)
      mbar_wait(&sm.full[j % ST], (j / ST) & 1, &sm.abort_flag, p.status) ||
          mbar_try(smem_u32(&sm.full[j % ST]), (j / ST) & 1);
  }
}

// ---------------------------------------------------------------------------
// MMA issuer (one lane)
// ---------------------------------------------------------------------------
template <int G>
__device__ void mma_issuer(const ScoreParams &p, TcSmem<G> &sm, uint32_t tmem) {
  using Cfg = TcCfg<G>;
  constexpr int ST = Cfg::STAGES, NCOL = Cfg::NCOL, BBLK = Cfg::BBLK, NACC = Cfg::NACC;
  constexpr uint32_t idesc = idesc_bf16_m128<NCOL>();
  // descriptors of stage 0 / coefficient buffer 0; an operand at byte offset
  // o from there is the descriptor plus o >> 4 (shared addresses < 256 KB)
  const uint64_t da0 = sw128_desc(smem_u32(&sm.k[0][0][0]));
  const uint64_t db0 = sw128_desc(smem_u32(&sm.b[0][0][0]));
  constexpr uint32_t kStageBytes = 2 * kHalfBlock;
  int i = 0;
  for (;; ++i) {
    if (!mbar_wait(&sm.aready[i % kNB], (i / kNB) & 1, &sm.abort_flag, p.status)) break;
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
    mma_commit(&sm.accfull[ab]);  // issued last: the final wait below covers all
  }
  if (i > 0) mbar_wait(&sm.accfull[(i - 1) % kNB], ((i - 1) / kNB) & 1, &sm.abort_flag, p.status);
}

// ---------------------------------------------------------------------------
// compute warps
// ---------------------------------------------------------------------------
// Band magnitudes of row r, bands [B q, B q + B) with B = kBandsPerThread,
// stored to the row's tensor-memory lane: hi parts at columns
// [B q / 2, B q / 2 + B / 2), lo parts at 32 + the same (two bf16 per
// column, band order).
template <int PAIR>
__device__ __forceinline__ void mags_regs(const uint8_t *kt, int r, int q,
                                          uint32_t (&hi)[kBandsPerThread / 2],
                                          uint32_t (&lo)[kBandsPerThread / 2]) {
  constexpr int B = kBandsPerThread;
  const int sw = r & 7;
  if (PAIR == TRIA_PAIR_NEOX) {
    // band f: re at dim f, im at dim 64 + f; a word holds bands (2k, 2k + 1)
#pragma unroll
    for (int j = 0; j < B / 8; ++j) {
      const int cc = (B / 8) * q + j;
      const uint4 re = lds128(kt + r * 128 + ((cc ^ sw) << 4));
      const uint4 im = lds128(kt + kHalfBlock + r * 128 + ((cc ^ sw) << 4));
      const uint32_t rw[4] = {re.x, re.y, re.z, re.w}, iw[4] = {im.x, im.y, im.z, im.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        mag_split(band_sq<false>(rw[e], iw[e]), band_sq<true>(rw[e], iw[e]), hi[4 * j + e],
                  lo[4 * j + e]);
    }
  } else {
    // band f: re at dim 2f, im at dim 2f + 1; a word holds one band; bands
    // [32 h, 32 h + 32) are the half block h
    const int f0 = B * q;
    const uint8_t *kh = kt + (f0 / 32) * kHalfBlock;
    const int c0 = (f0 % 32) / 4;
#pragma unroll
    for (int j = 0; j < B / 4; ++j) {
      const int cc = c0 + j;
      const uint4 x = lds128(kh + r * 128 + ((cc ^ sw) << 4));
      mag_split(band_sq_word(x.x), band_sq_word(x.y), hi[2 * j], lo[2 * j]);
      mag_split(band_sq_word(x.z), band_sq_word(x.w), hi[2 * j + 1], lo[2 * j + 1]);
    }
  }
}

template <int PAIR>
__device__ __forceinline__ void mags(const uint8_t *kt, uint32_t tcol, int r, int q) {
  constexpr int W = kBandsPerThread / 2;
  uint32_t hi[W], lo[W];
  mags_regs<PAIR>(kt, r, q, hi, lo);
  tmem_st<W>(tcol + (uint32_t)(W * q), hi);
  tmem_st<W>(tcol + (uint32_t)(32 + W * q), lo);
}

// Bounded wait of a whole warp (every lane tests the barrier; the warp
// leaves together).  Returns false, uniformly over the warp, on expiry/abort.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *status, int lane) {
  const uint32_t a = smem_u32(bar);
  if (__all_sync(kFull, mbar_try(a, parity))) return true;
  const uint64_t t0 = global_timer();
  for (;;) {
    if (__all_sync(kFull, mbar_try_sleep(a, parity))) return true;
    if (__any_sync(kFull, *abort_flag != 0)) return false;
    if (__any_sync(kFull, global_timer() - t0 > kWaitLimitNs)) {
      if (lane == 0) {
        *abort_flag = 1;
        atomicOr(status, 2);
      }
      return false;
    }
  }
}

// Epilogue of tile j (record pr): raw scores of this warp's 32 rows and GQ
// heads, fp64 moment sums, and the item's moment partials after its last tile.
template <int G>
__device__ __forceinline__ bool epilogue(const ScoreParams &p, TcSmem<G> &sm, uint32_t tmem, int j,
                                         const EpRec &pr, int q, int rg, int lane,
                                         double (&msum)[TcCfg<G>::GQ], double (&msq)[TcCfg<G>::GQ]) {
  constexpr int NCOL = TcCfg<G>::NCOL, GQ = TcCfg<G>::GQ;
  const Geom &geo = p.geo;
  const bool active = (G >= kBandGroups) || q < G;  // group q scores heads [q GQ, (q + 1) GQ)
  if (!warp_wait(&sm.accfull[j % kNB], (j / kNB) & 1, &sm.abort_flag, p.status, lane)) return false;
  tc_fence_after();
  if (pr.flags & kFlagFirst) {
#pragma unroll
    for (int g = 0; g < GQ; ++g) msum[g] = msq[g] = 0.0;
  }
  if (active) {
    // this thread's 2 GQ columns of each partial accumulator, summed in order
    constexpr int NACC = TcCfg<G>::NACC;
    uint32_t pa[NACC][2 * GQ];
    const uint32_t col = tmem + ((uint32_t)(32 * rg) << 16) + (uint32_t)((j % kNB) * NACC * NCOL + q * 2 * GQ);
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
      float *dst = pr.raw + (slot - geo.sinks) * G + q * GQ;
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
      double *m = pr.mom + (rg * G + q * GQ) * 2;
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
__device__ void compute(const ScoreParams &p, TcSmem<G> &sm, uint32_t tmem, int tid) {
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
    if (!warp_wait(&sm.full[stage], (i / ST) & 1, &sm.abort_flag, p.status, lane)) return -1;
    const SubRec &rc = sm.rec[stage];
    const int flags = rc.flags;
    const bool end = (flags & kFlagEnd) != 0;
    EpRec cur;
    if (!end) {
      cur.raw = rc.raw;
      cur.mom = rc.mom;
      cur.slot0 = rc.slot0;
      cur.N = rc.N;
      cur.flags = flags;
      mags<PAIR>(&sm.k[stage][0][0], mag_base + (uint32_t)((i % kNB) * 64), r, q);
      tmem_wait_st();
      tc_fence_before();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.aready[i % kNB]);
    if (i >= 2 && !epilogue<G>(p, sm, tmem, i - 2, older, q, rg, lane, msum, msq)) return -1;
    if (end) {
      if (i >= 1 && !epilogue<G>(p, sm, tmem, i - 1, other, q, rg, lane, msum, msq)) return -1;
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

  if (warp < kComputeWarps) {
    compute<G, PAIR>(p, sm, tmem, tid);
  } else if (warp == kProducerWarp) {
    producer<Cfg::STAGES, LAYOUT>(p, sm, n_items, lane);
  } else if (warp == kMmaWarp) {
    if (lane == 0) mma_issuer<G>(p, sm, tmem);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Max-over-offsets mode (tria_params.offset_reduce = TRIA_OFFSET_MAX).
//
// S_g(k) = max_j S_trig,g(k, Delta + delta_j) + S_norm,g(k): per tile two
// contractions, [k] (128 x 128) . Btrig (128 x 2 |D| G) into the trig
// accumulator (column pair (hi, lo) per (head, offset); one or two MMAs per
// K-step, N <= 256 each) and [m_hi | m_lo] . Bnorm (128 x 2G) into the norm
// accumulator, then a max over the offset pairs in the epilogue.  Tensor
// memory holds one buffer of each (trig 0..271, norm 288.., magnitudes
// 320..383), so a tile's epilogue runs before the next tile's MMAs; the
// compute warps hide it behind the next tile's magnitude math (computed into
// registers first, stored to tensor memory after the epilogue).
// ---------------------------------------------------------------------------
constexpr uint32_t kMaxNormCol = 288, kMaxMagCol = 320;

template <int G>
struct MaxCfg {
  static constexpr int NN = (2 * G < 16) ? 16 : 2 * G;                  // norm columns
  static constexpr int NT_MAX = ((2 * 17 * G + 15) / 16) * 16;          // trig columns at |D| = 17
  static constexpr int STAGES = (G >= 8) ? 2 : 4;
  static constexpr int BMAX = (NT_MAX + NN) * 256;                       // coefficient image bytes
  static constexpr int GQ = (G >= kBandGroups) ? G / kBandGroups : 1;
};

template <int G>
struct MaxSmem {
  alignas(1024) uint8_t k[MaxCfg<G>::STAGES][2][kHalfBlock];
  alignas(1024) uint8_t b[2][MaxCfg<G>::BMAX];
  alignas(8) uint64_t full[MaxCfg<G>::STAGES];
  alignas(8) uint64_t kempty[MaxCfg<G>::STAGES];
  alignas(8) uint64_t aready;
  alignas(8) uint64_t accfull;
  alignas(8) uint64_t bempty[2];
  SubRec rec[MaxCfg<G>::STAGES];
  alignas(16) int seq_items[kMaxSeqTable];
  int seq_len[kMaxSeqTable];
  uint32_t tmem_base;
  volatile int abort_flag;
  __device__ __forceinline__ uint8_t *bbuf(int i) { return &b[i][0]; }
};

__host__ __device__ constexpr uint32_t idesc_bf16_m128_n(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(kRows >> 4) << 24);
}

template <int G>
__device__ void mma_issuer_max(const ScoreParams &p, MaxSmem<G> &sm, uint32_t tmem) {
  using Cfg = MaxCfg<G>;
  constexpr int ST = Cfg::STAGES, NN = Cfg::NN;
  const int NT = p.geo.ncol_t;
  const int N1 = NT < 256 ? NT : 256, N2 = NT - N1;
  const uint32_t id1 = idesc_bf16_m128_n(N1), id2 = idesc_bf16_m128_n(N2 > 0 ? N2 : 16);
  constexpr uint32_t idn = idesc_bf16_m128_n(NN);
  const uint64_t da0 = sw128_desc(smem_u32(&sm.k[0][0][0]));
  const uint64_t db0 = sw128_desc(smem_u32(&sm.b[0][0]));
  constexpr uint32_t kStageBytes = 2 * kHalfBlock;
  const uint32_t nbase = 2u * NT * 128u;  // norm image after the trig image
  int i = 0;
  for (;; ++i) {
    if (!mbar_wait(&sm.aready, i & 1, &sm.abort_flag, p.status)) break;
    tc_fence_after();
    const int stage = i % ST;
    const SubRec &rec = sm.rec[stage];
    const int flags = rec.flags, bpar = rec.bpar;
    if (flags & kFlagEnd) break;
    const uint64_t da = da0 + (uint64_t)((stage * kStageBytes) >> 4);
    const uint64_t db = db0 + (uint64_t)(((uint32_t)bpar * (uint32_t)Cfg::BMAX) >> 4);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t ao = (s >> 2) * kHalfBlock + (s & 3) * 32;
      const uint32_t bo = (uint32_t)(s >> 2) * (uint32_t)NT * 128u + (s & 3) * 32;
      mma_bf16(tmem, da + (ao >> 4), db + (bo >> 4), id1, s > 0 ? 1u : 0u);
      if (N2 > 0)
        mma_bf16(tmem + (uint32_t)N1, da + (ao >> 4), db + ((bo + (uint32_t)N1 * 128u) >> 4), id2,
                 s > 0 ? 1u : 0u);
    }
    mma_commit(&sm.kempty[stage]);  // the K tile is consumed
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t bo = nbase + (uint32_t)(s >> 2) * NN * 128u + (s & 3) * 32;
      mma_bf16_ta(tmem + kMaxNormCol, tmem + kMaxMagCol + (uint32_t)(s * 8), db + (bo >> 4), idn,
                  s > 0 ? 1u : 0u);
    }
    if (flags & kFlagLast) mma_commit(&sm.bempty[bpar]);
    mma_commit(&sm.accfull);
  }
  if (i > 0) mbar_wait(&sm.accfull, (i - 1) & 1, &sm.abort_flag, p.status);
}

// Raw scores, fp64 moment sums and the item's moment partials of one tile
// (shared by the max-mode epilogue).
template <int G>
__device__ __forceinline__ void emit_scores(const ScoreParams &p, const EpRec &pr,
                                            const float (&sc)[TcCfg<G>::GQ], bool active, int q,
                                            int rg, int lane, double (&msum)[TcCfg<G>::GQ],
                                            double (&msq)[TcCfg<G>::GQ]) {
  constexpr int GQ = TcCfg<G>::GQ;
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
      float *dst = pr.raw + (slot - geo.sinks) * G + q * GQ;
#pragma unroll
      for (int g = 0; g < GQ; ++g) dst[g] = sc[g];
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
      double *m = pr.mom + (rg * G + q * GQ) * 2;
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        m[2 * g] = msum[g];
        m[2 * g + 1] = msq[g];
      }
    }
  }
}

// Maximum that returns NaN when either operand is NaN.
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Epilogue of the previous tile in max mode: per head of this thread's band
// group, S = max_j (hi_j + lo_j) + (norm hi + norm lo).
template <int G>
__device__ __forceinline__ void epilogue_max(const ScoreParams &p, uint32_t tmem, const EpRec &pr,
                                             int q, int rg, int lane, double (&msum)[TcCfg<G>::GQ],
                                             double (&msq)[TcCfg<G>::GQ]) {
  constexpr int GQ = TcCfg<G>::GQ;
  const bool active = (G >= kBandGroups) || q < G;
  const int nd = p.geo.n_off;
  float sc[GQ];
  if (active) {
    const uint32_t lb = tmem + ((uint32_t)(32 * rg) << 16);
#pragma unroll
    for (int gi = 0; gi < GQ; ++gi) {
      const int g = q * GQ + gi;
      // the head's 2 nd columns: one 32-column load (offsets 0..15; beyond
      // 2 nd it reads the next head's columns, unused) and one 2-column load
      // for offset 16
      uint32_t t[32], t16[2], nv[2];
      const uint32_t c0 = lb + (uint32_t)(g * nd * 2);
      tmem_ld_nowait<32>(c0, t);
      if (nd == 17) tmem_ld_nowait<2>(c0 + 32, t16);
      tmem_ld_nowait<2>(lb + kMaxNormCol + (uint32_t)(2 * g), nv);
      tmem_wait_ld();
      // offsets past |D| read as -inf; a pairwise tree of NaN-propagating
      // maxes, built in place over the loaded words
#pragma unroll
      for (int j = 0; j < 16; ++j)
        t[j] = __float_as_uint((j < nd) ? __uint_as_float(t[2 * j]) + __uint_as_float(t[2 * j + 1])
                                        : -INFINITY);
      const float v16 = (nd == 17) ? __uint_as_float(t16[0]) + __uint_as_float(t16[1]) : -INFINITY;
#pragma unroll
      for (int w = 1; w < 16; w *= 2) {
#pragma unroll
        for (int j = 0; j + w < 16; j += 2 * w)
          t[j] = __float_as_uint(max_nan(__uint_as_float(t[j]), __uint_as_float(t[j + w])));
      }
      const float m = max_nan(__uint_as_float(t[0]), v16);
      sc[gi] = m + (__uint_as_float(nv[0]) + __uint_as_float(nv[1]));
    }
  } else {
#pragma unroll
    for (int gi = 0; gi < GQ; ++gi) sc[gi] = 0.0f;
  }
  tc_fence_before();
  emit_scores<G>(p, pr, sc, active, q, rg, lane, msum, msq);
}

template <int G, int PAIR>
__device__ void compute_max(const ScoreParams &p, MaxSmem<G> &sm, uint32_t tmem, int tid) {
  constexpr int ST = MaxCfg<G>::STAGES, GQ = TcCfg<G>::GQ, W = kBandsPerThread / 2;
  const int warp = tid >> 5, lane = tid & 31;
  const int q = warp >> 2, rg = warp & 3, r = rg * 32 + lane;
  const uint32_t mag = tmem + ((uint32_t)(32 * rg) << 16) + kMaxMagCol;
  double msum[GQ], msq[GQ];
#pragma unroll
  for (int g = 0; g < GQ; ++g) msum[g] = msq[g] = 0.0;
  EpRec prev{};
  for (int i = 0;; ++i) {
    const int stage = i % ST;
    if (!warp_wait(&sm.full[stage], (i / ST) & 1, &sm.abort_flag, p.status, lane)) return;
    const SubRec &rc = sm.rec[stage];
    const int flags = rc.flags;
    const bool end = (flags & kFlagEnd) != 0;
    EpRec cur{};
    uint32_t hi[W], lo[W];
    if (!end) {
      cur.raw = rc.raw;
      cur.mom = rc.mom;
      cur.slot0 = rc.slot0;
      cur.N = rc.N;
      cur.flags = flags;
      mags_regs<PAIR>(&sm.k[stage][0][0], r, q, hi, lo);
    }
    if (i >= 1) {
      // the previous tile's MMAs are done: its scores, and its magnitude
      // buffer may be overwritten
      if (!warp_wait(&sm.accfull, (i - 1) & 1, &sm.abort_flag, p.status, lane)) return;
      tc_fence_after();
      epilogue_max<G>(p, tmem, prev, q, rg, lane, msum, msq);
    }
    if (!end) {
      tmem_st<W>(mag + (uint32_t)(W * q), hi);
      tmem_st<W>(mag + (uint32_t)(32 + W * q), lo);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.aready);
    if (end) return;
    prev = cur;
  }
}

template <int G, int PAIR, int LAYOUT>
__global__ void __launch_bounds__(kTcThreads, 1) score_max_kernel(const __grid_constant__ ScoreParams p) {
  using Cfg = MaxCfg<G>;
  extern __shared__ uint8_t smem_dyn[];
  MaxSmem<G> &sm = *reinterpret_cast<MaxSmem<G> *>(
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
    mbar_init(&sm.aready, kComputeWarps);
    mbar_init(&sm.accfull, 1);
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

  if (warp < kComputeWarps) {
    compute_max<G, PAIR>(p, sm, tmem, tid);
  } else if (warp == kProducerWarp) {
    producer<Cfg::STAGES, LAYOUT>(p, sm, n_items, lane);
  } else if (warp == kMmaWarp) {
    if (lane == 0) mma_issuer_max<G>(p, sm, tmem);
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
  kern<<<sms, kTcThreads, smem, st>>>(p);
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
static_assert(MaxCfg<8>::NT_MAX <= 288 - 16, "max-mode trig columns");

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
  if (p.geo.mode == TRIA_OFFSET_MAX) {
    switch (p.geo.g) {
      case 1: return launch_max_g<1>(p, st);
      case 2: return launch_max_g<2>(p, st);
      case 4: return launch_max_g<4>(p, st);
      case 8: return launch_max_g<8>(p, st);
      default: return cudaErrorInvalidValue;
    }
  }
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
