// compact_kernel: in-place gather of the kept K/V rows of every unit (and of
// the K positions), then the sequence lengths and freed paged blocks.
//
// The kept list of a unit is ascending with kept[j] >= j, so destination j
// never lies above its source.  Rows move in chunks of kCpRows destination
// rows, in ascending order, through a ring of shared-memory chunk buffers
// filled by cp.async (16 bytes per copy, no registers held while in flight):
//   * every row of chunk c is read before any row of chunk c is written, as a
//     destination of chunk c can be the source of another row of chunk c or
//     of an earlier chunk (one __syncthreads per chunk);
//   * chunk c + A is read before chunk c is written: its sources are at or
//     above its first destination, above every destination of chunk c.
// Each block (one per SM; two for paged caches) walks the chunks of its
// items (unit, K or V) as one stream, reading A = 2 chunks ahead of the chunk
// it writes; an item has ceil(B_l / kCpRows) chunks for the budget B_l of its
// layer.  A thread always
// handles the same rows and 16-byte pieces of a chunk: it loads their kept
// entries one chunk before it starts their copies, keeps their sources in
// shared memory for the write-back, and writes back exactly the pieces it
// read, so the only wait on the path is for copies started two chunks ago.
#include "tria_device.cuh"

namespace tria {
namespace {

using namespace dev;

constexpr int kCpDepth = 3;                               // chunk buffers
constexpr int kCpAhead = 2;                               // chunks read ahead
constexpr int kRowBytes = kHeadDim * 2;                   // 256
constexpr int kPieces = kRowBytes / 16;                   // 16-byte pieces per row
constexpr int kMinBlock = 8;                              // smallest paged block size

// Block shape per layout.  Contiguous: one block of 512 threads per SM with
// 256-row chunks.  Paged: four blocks of 128 threads per SM with 64-row
// chunks (the same bytes in flight per SM; its row addresses need block-table
// entries, and independent blocks hide that better: per 8-layer paged batch
// 2041 us with one block, 1903 with two of 256 threads and 128-row chunks,
// 1820 with four; the contiguous pass measured 215 -> 234 us with two).
template <bool PAGED>
struct CpCfg {
  static constexpr int THREADS = PAGED ? 128 : 512;
  static constexpr int ROWS = PAGED ? 64 : 256;           // destination rows per chunk
  static constexpr int BPS = PAGED ? 4 : 1;               // blocks per SM
  static constexpr int ROW_STEP = THREADS / kPieces;      // rows covered by one pass of the block
  static constexpr int ROWS_PER_THREAD = ROWS / ROW_STEP;  // 8
};

template <int ROWS>
struct CpSmem {
  alignas(16) uint8_t buf[kCpDepth][ROWS][kRowBytes];
  int32_t pos[kCpDepth][ROWS];
  int32_t src[kCpDepth][ROWS];   // source of each destination row (-1: stays)
  int32_t dblk[kCpDepth][ROWS / kMinBlock];  // paged: the chunk's destination blocks
};

struct ItemGeo {
  unsigned char *base;  // K or V of the layer
  int32_t *pos;         // positions of the unit (K items only; may be null)
  const int32_t *kept;
  int s, h, ul, part;
};

__device__ __forceinline__ ItemGeo item_geo(const CompactParams &p, int64_t it) {
  const Geom &geo = p.geo;
  ItemGeo g;
  const int64_t u = it >> 1;
  g.part = (int)(it & 1);
  g.s = (int)(u / ((int64_t)geo.nl * geo.hkv));
  g.ul = (int)(u % ((int64_t)geo.nl * geo.hkv));
  const int lrel = g.ul / geo.hkv;
  g.h = g.ul % geo.hkv;
  g.kept = p.kept + u * geo.budget;
  g.base = reinterpret_cast<unsigned char *>(g.part == 0 ? const_cast<uint16_t *>(p.cache.k[lrel])
                                                         : p.cache.v[lrel]);
  const int64_t pu = ((int64_t)g.s * geo.n_layers + geo.layer0 + lrel) * geo.hkv + g.h;
  g.pos = (g.part == 0 && p.cache.positions != nullptr)
              ? p.cache.positions + pu * p.cache.pos_unit_stride
              : nullptr;
  return g;
}

__device__ __forceinline__ void cp16(void *sdst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(sdst)),
               "l"(gsrc)
               : "memory");
}

__device__ __forceinline__ void cp4(void *sdst, const void *gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(sdst)),
               "l"(gsrc)
               : "memory");
}

__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Length and freed blocks of sequence s (one length for all its layers), from
// the kept list of its unit 0.
__device__ void update_len(const CompactParams &p, const ItemGeo &g) {
  const Geom &geo = p.geo;
  const int s = g.s;
  const int N = p.cache.seq_lens[s];
  int newlen = geo.budget;
  if (g.kept[geo.budget - 1] < 0) {
    newlen = 0;
    while (newlen < geo.budget && g.kept[newlen] >= 0) ++newlen;
  }
  if (compresses(geo, N, 0)) {
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

template <bool PAGED>
__global__ void __launch_bounds__(CpCfg<PAGED>::THREADS, CpCfg<PAGED>::BPS)
    compact_kernel(const __grid_constant__ CompactParams p) {
  constexpr int kCpRows = CpCfg<PAGED>::ROWS, kRowStep = CpCfg<PAGED>::ROW_STEP,
                kRowsPerThread = CpCfg<PAGED>::ROWS_PER_THREAD;
  extern __shared__ __align__(16) uint8_t smem_cp[];
  CpSmem<kCpRows> &sm = *reinterpret_cast<CpSmem<kCpRows> *>(smem_cp);
  const Geom &geo = p.geo;
  const int t = threadIdx.x;
  const int piece = t % kPieces, rr = t / kPieces;
  const int cap = geo.max_seq_len;
  const int64_t n_items = geo.n_units * 2;
  const int64_t my_items =
      (blockIdx.x < n_items) ? (n_items - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  // The block's items form one stream of chunks, item-major; an item has
  // ceil(B_l / kCpRows) chunks for the budget B_l of its layer.  A cursor is
  // a position in that stream.
  struct Cur {
    int64_t i;  // item ordinal within the block (>= my_items: past the end)
    int c, nch;
  };
  auto item_of = [&](int64_t i) { return (int64_t)blockIdx.x + i * gridDim.x; };
  auto chunks_of = [&](int64_t i) {
    const int64_t u = item_of(i) >> 1;
    const int lrel = (int)((u / geo.hkv) % geo.nl);
    return (geo.lbudget[lrel] + kCpRows - 1) / kCpRows;
  };
  auto start = [&]() {
    Cur q{0, 0, 0};
    if (my_items > 0) q.nch = chunks_of(0);
    return q;
  };
  auto advance = [&](Cur &q) {
    if (++q.c >= q.nch) {
      ++q.i;
      q.c = 0;
      q.nch = q.i < my_items ? chunks_of(q.i) : 0;
    }
  };

  constexpr bool paged = PAGED;
  const int bs = p.cache.block_size;  // a power of two (8 .. 128)
  const int bsh = __ffs(bs) - 1, bsm = bs - 1;
  // kept entries (raw) of this thread's rows of chunk q and, paged, the
  // block-table entries of their sources (both used one iteration later, so
  // the dependent table load is off the copy path)
  auto fetch = [&](const Cur &q, int (&kv)[kRowsPerThread], int (&kb)[kRowsPerThread]) {
    if (q.i < my_items) {
      const int64_t u = item_of(q.i) >> 1;
      const int32_t *kept = p.kept + u * geo.budget;
#pragma unroll
      for (int e = 0; e < kRowsPerThread; ++e) {
        const int j = q.c * kCpRows + rr + e * kRowStep;
        kv[e] = (j < geo.budget) ? __ldg(kept + j) : -1;
      }
      if constexpr (paged) {
        const int32_t *bt = p.cache.block_table +
                            (int64_t)(u / ((int64_t)geo.nl * geo.hkv)) * p.cache.max_blocks;
#pragma unroll
        for (int e = 0; e < kRowsPerThread; ++e) {
          const int j = q.c * kCpRows + rr + e * kRowStep, v = kv[e];
          const bool moves = j < geo.budget && v != j && v >= 0 && v < cap && j < cap;
          kb[e] = moves ? __ldg(bt + (v >> bsh)) : 0;
        }
      }
    }
  };
  // copies of this thread's pieces of chunk q into buffer b (one commit
  // group per chunk, empty past the end)
  auto issue = [&](const Cur &q, int b, const int (&kv)[kRowsPerThread],
                   const int (&kb)[kRowsPerThread]) {
    if (q.i < my_items) {
      const ItemGeo g = item_geo(p, item_of(q.i));
      if constexpr (paged) {
        // the chunk's destination blocks, for its write-back two iterations on
        // destination blocks of the chunk: one when a block holds more rows
        // than a chunk (the chunk's rows are then all in block b0)
        const int nb = max(1, kCpRows >> bsh), b0 = (q.c * kCpRows) >> bsh;
        if (t < nb)
          sm.dblk[b][t] = (b0 + t < p.cache.max_blocks)
                              ? __ldg(p.cache.block_table + (int64_t)g.s * p.cache.max_blocks + b0 + t)
                              : 0;
      }
#pragma unroll
      for (int e = 0; e < kRowsPerThread; ++e) {
        const int r = rr + e * kRowStep, j = q.c * kCpRows + r;
        const int v = kv[e];
        const int src = (j >= geo.budget || v == j || v < 0 || v >= cap || j >= cap) ? -1 : v;
        if (piece == 0) sm.src[b][r] = src;
        if (src >= 0) {
          const int64_t off = paged ? (int64_t)kb[e] * p.cache.s_blk + (int64_t)(src & bsm) * p.cache.s_tok +
                                          (int64_t)g.h * p.cache.s_head
                                    : row_off(p.cache, g.s, g.h, src);
          cp16(&sm.buf[b][r][piece * 16], g.base + off * 2 + piece * 16);
          if (g.pos != nullptr && piece == 0) cp4(&sm.pos[b][r], g.pos + src);
        }
      }
    }
    cp_commit();
  };

  int kv[kRowsPerThread], kb[kRowsPerThread];
  Cur fc = start();  // next chunk to fetch
  for (int k = 0; k < kCpAhead; ++k) {
    fetch(fc, kv, kb);
    issue(fc, k % kCpDepth, kv, kb);
    advance(fc);
  }
  Cur pend = fc;  // fetched, to be issued at the next iteration
  fetch(pend, kv, kb);
  advance(fc);
  Cur wc = start();  // chunk to write back
  for (int64_t k = 0; wc.i < my_items; ++k) {
    issue(pend, (int)((k + kCpAhead) % kCpDepth), kv, kb);
    pend = fc;
    fetch(pend, kv, kb);  // used at the next iteration
    advance(fc);
    cp_wait<kCpAhead>();  // this thread's copies of chunk k have landed
    __syncthreads();      // ... and every other thread's
    const ItemGeo g = item_geo(p, item_of(wc.i));
    const int b = (int)(k % kCpDepth);
#pragma unroll
    for (int e = 0; e < kRowsPerThread; ++e) {
      const int r = rr + e * kRowStep, j = wc.c * kCpRows + r;
      // the row's source, recorded (and now read) by the row's piece-0 thread
      const int mine = (piece == 0) ? sm.src[b][r] : 0;
      const int src = __shfl_sync(kFull, mine, (threadIdx.x & 31) & ~(kPieces - 1));
      if (src >= 0) {
        const uint4 v = *reinterpret_cast<const uint4 *>(&sm.buf[b][r][piece * 16]);
        const int64_t off = paged ? (int64_t)sm.dblk[b][r >> bsh] * p.cache.s_blk +
                                        (int64_t)(j & bsm) * p.cache.s_tok + (int64_t)g.h * p.cache.s_head
                                  : row_off(p.cache, g.s, g.h, j);
        *reinterpret_cast<uint4 *>(g.base + off * 2 + piece * 16) = v;
        if (g.pos != nullptr && piece == 0) g.pos[j] = sm.pos[b][r];
      }
    }
    // sequence length / freed blocks: once per sequence, after the last layer
    if (wc.c == wc.nch - 1 && p.update_lens && g.part == 0 && g.ul == 0 && t == 0) update_len(p, g);
    advance(wc);
  }
  cp_wait<0>();
}

// Per-(sequence, layer) lengths: every compressed (sequence, layer) of the
// call now holds B_l rows (C > K whenever N - B_l >= 1, so the selection
// always fills the budget).  The paged blocks are shared by the layers: a call
// over every layer frees the blocks past the longest new length that held
// rows of the longest old one.  One block of kLensThreads per sequence.
constexpr int kLensThreads = 128;

__global__ void __launch_bounds__(kLensThreads) layer_lens_kernel(const __grid_constant__ LensParams p) {
  const Geom &g = p.geo;
  const int s = blockIdx.x, t = threadIdx.x;
  int old_max = 0, new_max = 0, bad = 0;
  for (int lr = t; lr < g.nl; lr += kLensThreads) {
    const int n = unit_len(g, s, lr);
    if (!len_valid(g, n)) {
      bad = 1;
      continue;
    }
    const int nn = compresses(g, n, lr) ? g.lbudget[lr] : n;
    old_max = max(old_max, n);
    new_max = max(new_max, nn);
    if (nn != n) p.layer_lens[(int64_t)s * g.n_layers + g.layer0 + lr] = nn;
  }
  old_max = __reduce_max_sync(kFull, old_max);
  new_max = __reduce_max_sync(kFull, new_max);
  bad = __reduce_or_sync(kFull, bad);
  __shared__ int red[3][kLensThreads / 32];
  const int w = t >> 5;
  if ((t & 31) == 0) {
    red[0][w] = old_max;
    red[1][w] = new_max;
    red[2][w] = bad;
  }
  __syncthreads();
  if (t != 0 || !p.paged || p.n_freed == nullptr) return;
  for (int i = 1; i < kLensThreads / 32; ++i) {
    old_max = max(old_max, red[0][i]);
    new_max = max(new_max, red[1][i]);
    bad |= red[2][i];
  }
  int nf = 0;
  if (p.all_layers && !bad) {
    const int bs = p.block_size;
    for (int b = (new_max + bs - 1) / bs; b < (old_max + bs - 1) / bs; ++b) {
      if (p.freed_blocks != nullptr)
        p.freed_blocks[(int64_t)s * p.max_blocks + nf] = p.block_table[(int64_t)s * p.max_blocks + b];
      ++nf;
    }
  }
  p.n_freed[s] = nf;
}

}  // namespace

cudaError_t launch_layer_lens(const LensParams &p, cudaStream_t st) {
  layer_lens_kernel<<<(unsigned)p.geo.n_seq, kLensThreads, 0, st>>>(p);
  return cudaGetLastError();
}

template <bool PAGED>
cudaError_t launch_compact_t(const CompactParams &p, cudaStream_t st) {
  using Cfg = CpCfg<PAGED>;
  static_assert(sizeof(CpSmem<Cfg::ROWS>) * Cfg::BPS <= 232448, "shared memory of the compaction kernel");
  const int smem = (int)sizeof(CpSmem<Cfg::ROWS>);
  auto kern = compact_kernel<PAGED>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  int64_t grid = p.geo.n_units * 2;
  if (grid > (int64_t)sms * Cfg::BPS) grid = (int64_t)sms * Cfg::BPS;
  kern<<<(unsigned)grid, Cfg::THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_compact(const CompactParams &p, cudaStream_t st) {
  return p.cache.layout == TRIA_LAYOUT_PAGED ? launch_compact_t<true>(p, st)
                                             : launch_compact_t<false>(p, st);
}

}  // namespace tria
