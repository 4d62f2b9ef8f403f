// Pieces shared by the tensor-core scoring kernels (the offset-mean kernel in
// tria_score_tc.cu, the max-over-offsets kernel in tria_score_max.cu): inline
// PTX wrappers for mbarriers, TMA and tcgen05, bounded waits, the record a
// K tile carries through the ring, and the producer warp that streams the K
// tiles of the work items with TMA.
//
// Waits.  Every wait on an mbarrier is bounded by ScoreParams::wait_ns
// (%globaltimer).  A wait that runs out sets the block's abort flag and
// status bit 1; every role then leaves at its next wait.  Before the block
// exits, the producer waits for the loads it issued and the MMA issuer for
// its last commit (drain waits: bounded by kDrainNs, not cut short by the
// abort flag), so no copy or MMA into the block's shared or tensor memory is
// in flight when the tensor memory is freed.
#pragma once

#include <cuda_bf16.h>

#include "tria_device.cuh"

namespace tria {
namespace tc {

using namespace dev;

constexpr int kRows = 128;                  // keys per MMA tile (M)
constexpr int kHalfBlock = kRows * 128;     // 128 rows x 64 bf16, swizzled
constexpr int kFlagFirst = 1, kFlagLast = 2, kFlagEnd = 4;
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
constexpr uint64_t kDrainNs = 2000000000ull;
constexpr uint32_t kSuspendNs = 1000000;    // a blocked try_wait sleeps up to 1 ms per call

// Record of one 128-slot K tile, written by the producer next to the tile.
struct SubRec {
  long long u;     // unit
  int tile, N;     // scheduling item of the unit, the unit's length
  int slot0, flags, bpar;  // first slot of the 128-row tile (a multiple of 128)
};

// What the epilogue of a tile needs from its record (kept in registers
// for two tiles: the ring stage may be refilled before the epilogue).
struct EpRec {
  long long u;
  int tile, N, slot0, flags;
};

__device__ __forceinline__ EpRec ep_of(const SubRec &r) {
  EpRec e;
  e.u = r.u;
  e.tile = r.tile;
  e.N = r.N;
  e.slot0 = r.slot0;
  e.flags = r.flags;
  return e;
}

// The unit's raw scores (candidate 0) and the item's moment partials.
__device__ __forceinline__ float *ep_raw(const ScoreParams &p, const EpRec &e) {
  return p.raw + e.u * p.raw_stride;
}
__device__ __forceinline__ double *ep_mom(const ScoreParams &p, const EpRec &e) {
  return p.moments + (e.u * p.geo.tiles_max + e.tile) * kRowGroups * p.geo.g * 2;
}

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

// try_wait that may suspend the thread for up to hint_ns until the phase
// completes, instead of returning at once.
__device__ __forceinline__ bool mbar_try_sleep(uint32_t addr, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(addr), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// The limits of a block's waits and where an expiry is reported.
struct WaitCtl {
  volatile int *abort_flag;  // shared: set by the first wait that runs out
  int32_t *status;           // device status flags (bit 1: a wait ran out)
  uint64_t limit_ns;
  uint32_t hint_ns;          // suspend-time hint of one try_wait: min(limit, kSuspendNs)
};

__device__ __forceinline__ WaitCtl wait_ctl(volatile int *abort_flag, int32_t *status,
                                            uint64_t wait_ns) {
  WaitCtl w;
  w.abort_flag = abort_flag;
  w.status = status;
  w.limit_ns = wait_ns ? wait_ns : kDefaultWaitNs;
  w.hint_ns = (uint32_t)(w.limit_ns < kSuspendNs ? w.limit_ns : kSuspendNs);
  return w;
}

__device__ __forceinline__ void flag_expiry(const WaitCtl &w) {
  *w.abort_flag = 1;
  atomicOr(w.status, 2);
}

// Bounded wait (one thread) for the phase of `parity`; false on expiry or abort.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const WaitCtl &w) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try(a, parity)) return true;
  const uint64_t t0 = global_timer();
  for (;;) {
    if (mbar_try_sleep(a, parity, w.hint_ns)) return true;
    if (*w.abort_flag) return false;
    if (global_timer() - t0 > w.limit_ns) {
      flag_expiry(w);
      return false;
    }
  }
}

// Wait (one thread) on the abort path for work this block started (copies,
// MMA commits): not cut short by the abort flag; bounded by kDrainNs.
__device__ __forceinline__ bool mbar_drain(uint64_t *bar, uint32_t parity, int32_t *status) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = global_timer();
  for (;;) {
    if (mbar_try_sleep(a, parity, kSuspendNs)) return true;
    if (global_timer() - t0 > kDrainNs) {
      atomicOr(status, 2);
      return false;
    }
  }
}

// Bounded wait of a whole warp (every lane tests the barrier; the warp
// leaves together).  Returns false, uniformly over the warp, on expiry/abort.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const WaitCtl &w,
                                          int lane) {
  const uint32_t a = smem_u32(bar);
  if (__all_sync(kFull, mbar_try(a, parity))) return true;
  const uint64_t t0 = global_timer();
  for (;;) {
    if (__all_sync(kFull, mbar_try_sleep(a, parity, w.hint_ns))) return true;
    if (__any_sync(kFull, *w.abort_flag != 0)) return false;
    if (__any_sync(kFull, global_timer() - t0 > w.limit_ns)) {
      if (lane == 0) flag_expiry(w);
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

// Instruction descriptor of kind::f16: bf16 x bf16 -> f32, both K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16_m128_n(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(kRows >> 4) << 24);
}

// D (tmem) (+)= A (smem descriptor) . B (smem descriptor)
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
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

// ---------------------------------------------------------------------------
// Band magnitudes
// ---------------------------------------------------------------------------
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

// Band magnitudes of row r, bands [B q, B q + B) with B = BANDS, from the
// row's 128-byte-swizzled K tile: hi parts in hi[], lo parts in lo[] (two
// bf16 per word, band order).
template <int PAIR, int BANDS>
__device__ __forceinline__ void mags_regs(const uint8_t *kt, int r, int q, uint32_t (&hi)[BANDS / 2],
                                          uint32_t (&lo)[BANDS / 2]) {
  constexpr int B = BANDS;
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

// ---------------------------------------------------------------------------
// producer warp: claims work items (kTileKeys slots of one unit) in order and
// streams their 128-slot K tiles into the ring with TMA, plus each item's
// coefficient image (one bulk copy into one of two buffers).  SM is the
// kernel's shared-memory struct: k[ST][2][kHalfBlock], full/kempty[ST],
// bempty[2], rec[ST], seq_items, seq_len, bbuf(i).
// ---------------------------------------------------------------------------
template <int ST, int LAYOUT, class Smem>
__device__ void producer(const ScoreParams &p, Smem &sm, int n_items, int lane, const WaitCtl wc) {
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
      if (lane == 0) ok = mbar_wait(&sm.kempty[stage], ((i / ST) - 1) & 1, wc);
      ok = __shfl_sync(kFull, ok, 0);
      if (!ok) break;
    }
    const int bpar = (items - 1) & 1;
    const bool first = (sub == sub_first);
    if (first && items > 2) {
      // the coefficient buffer is free once the MMAs of the item two back are done
      if (lane == 0) ok = mbar_wait(&sm.bempty[bpar], ((items - 3) >> 1) & 1, wc);
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
      r.u = u; r.tile = tile; r.N = N; r.slot0 = slot0;
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
      if (lane == 0) ok = mbar_wait(&sm.kempty[stage], ((i / ST) - 1) & 1, wc);
      ok = __shfl_sync(kFull, ok, 0);
    }
    if (ok && lane == 0) {
      sm.rec[stage].flags = kFlagEnd;
      mbar_arrive(&sm.full[stage]);
    }
    if (ok) ++i;  // the marker's phase completes by this arrival
  }
  if (!ok && lane == 0) {
    // aborted: the loads of tiles [i - ST, i) may still be in flight (the
    // earlier ones completed before their stage was refilled); wait for each
    // to land before the block exits
    for (int j = (i > ST ? i - ST : 0); j < i; ++j) mbar_drain(&sm.full[j % ST], (j / ST) & 1, wc.status);
  }
}

}  // namespace tc
}  // namespace tria
