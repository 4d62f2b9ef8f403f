// Decode attention over the cached rows of one layer: the attention that runs
// for every generated token, on the cache the compression pass pruned
// (academ.us article 2607.13051, sec. 8).  For sequence s and query head qh
// of KV head h = qh / G, over the rows j < N(s, layer) of unit (s, layer, h):
//   z_j = scale (q . k_j),   out = sum_j softmax(z)_j v_j,   lse = log sum_j e^{z_j}.
// A cached key carries its RoPE rotation, so a retained row keeps the logit
// it had in the full cache wherever compaction moved it (Eq. 3: the phase
// depends only on the rotations already applied to q and k).
//
// Split-K flash decoding.  The rows of every (sequence, KV head) are shared
// evenly by splits x 8 warps (about one block of 8 warps per SM in all); each
// warp streams its range through a 3-deep ring of 16-row K/V tiles (cp.async
// into XOR-swizzled shared memory, read with ldmatrix) and runs the two
// contractions on the tensor cores with warp-level mma.sync (m16n8k16, bf16
// inputs, fp32 accumulation), the 16 rows on the M side: S = K Q^T (heads as
// N), an online softmax in base 2 in registers, and O^T += V^T P^T (the 128
// dims as M) with each 8x8 block of P transposed in registers (movmatrix)
// and split into bf16 hi + lo.  The block's warps merge their (o, m, l) per
// head into the block's partial; the last block of each (sequence, KV head)
// to finish rescales the partials to their common maximum (an arrival count
// per unit in the workspace, reset by that block).  Decode attention at
// G <= 16 reads 512 bytes per row for 4 G multiply-adds per byte, well below
// the tensor cores' balance point, so the warp-level MMA (not the 128-row
// tcgen05 tile) is enough to leave the kernel bound by HBM.
#include <cmath>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tria_device.cuh"

namespace tria {
namespace {

using namespace dev;

constexpr int kDecWarps = 8;                   // warps per block
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kWTile = 16;                     // rows per warp tile
constexpr int kWStages = 3;                    // warp tiles in flight
constexpr int kTileBytes = kWTile * 256;       // one tile of K (or V)
constexpr int kWarpSmem = kWStages * 2 * kTileBytes;
constexpr int kDecSmem = kDecWarps * kWarpSmem;
constexpr int kMinSplitRows = kWTile * kDecWarps;
constexpr int kPart = 132;                     // per (head, partial): o[128], m, l, 2 pad floats
constexpr int kMaxSplits = 160;                // blocks per (sequence, KV head), at most
constexpr size_t kDecHeader = 256;
constexpr float kLn2 = 0.6931471805599453f;
// a head's running maximum (base 2) moves only when a tile exceeds it by more
// than this, so most tiles skip rescaling the accumulators; the weights then
// stay below 2^kRescale, well inside fp32 and bf16
constexpr float kRescale = 8.f;

struct DecodeParams {
  const uint16_t *k, *v;
  const uint16_t *q;
  const int32_t *block_table;
  const int32_t *lens;
  int64_t lens_s;
  int64_t s_seq, s_head, s_tok, s_blk, num_blocks;
  int layout, block_size, max_blocks;
  int max_seq_len, n_seq, hkv, hq;
  int splits;     // blocks (and partials) per (sequence, KV head)
  int nparts;     // warp ranges per (sequence, KV head): splits x kDecWarps
  float scale;    // natural-log logits
  float qscale;   // scale * log2(e): base-2 logits
  float *part;    // [n_seq * hq][splits][kPart]
  uint32_t *arrived;  // [n_seq * hkv] blocks done; the last one combines and resets it
  float *out, *lse, *logits;
  int32_t *status;
};

__device__ __forceinline__ int64_t dec_row(const DecodeParams &p, int s, int h, int t, bool &ok) {
  if (p.layout == TRIA_LAYOUT_CONTIGUOUS) {
    ok = true;
    return (int64_t)s * p.s_seq + (int64_t)h * p.s_head + (int64_t)t * p.s_tok;
  }
  const int blk = p.block_table[(int64_t)s * p.max_blocks + t / p.block_size];
  ok = blk >= 0 && blk < p.num_blocks;
  return (int64_t)blk * p.s_blk + (int64_t)(t % p.block_size) * p.s_tok + (int64_t)h * p.s_head;
}

// N of sequence s, or -1 when it lies outside [0, max_seq_len]
__device__ __forceinline__ int dec_len(const DecodeParams &p, int s) {
  const int n = p.lens[(int64_t)s * p.lens_s];
  return (n >= 0 && n <= p.max_seq_len) ? n : -1;
}

// rows per partial of a unit with n rows: the partials share them evenly
__host__ __device__ __forceinline__ int split_rows(int n, int parts) {
  return (n + parts - 1) / parts;
}

__device__ __forceinline__ void cp_async16(uint32_t sdst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sdst), "l"(gsrc) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A (16 x 16, bf16, rows) . B (16 x 8, bf16, columns), fp32 accumulate
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// transpose of an 8x8 b16 matrix held one row pair per lane (lane: row
// lane / 4, columns 2 (lane % 4), + 1)
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// two weights as bf16 pairs hi + lo (hi = bf16(x), lo = bf16(x - hi)): the
// product with a bf16 value then keeps ~16 bits of the weight
__device__ __forceinline__ void split2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// byte offset of 16-byte chunk c of tile row r (chunks XOR-swizzled by the
// row, so the 8 rows an ldmatrix reads hit 8 different bank groups)
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (uint32_t)(r * 256 + ((c ^ (r & 7)) << 4));
}

// Warp-level flash decoding on the tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate).  Each warp owns a contiguous range of the unit's rows,
// streamed through its own ring of 16-row K and V tiles (cp.async, 3 in
// flight).  Per tile and 8-head column tile: S = K Q^T with the 16 rows as
// M and the heads as N (K fragments straight from ldmatrix, Q^T fragments in
// registers); the online softmax in registers (a lane holds rows gid and
// gid + 8 of heads 2 tig and 2 tig + 1); then O^T += V^T P^T with the dims
// as M (V^T through ldmatrix.trans) and P^T as B, each 8x8 block of P
// transposed in registers by movmatrix and split into bf16 hi + lo.  The
// block's warps then merge their (o, m, l) in shared memory into the
// block's partial.
template <int G, int LAYOUT>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t sm_dec[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int u = blockIdx.x / p.splits, sp = blockIdx.x % p.splits;
  const int s = u / p.hkv, h = u % p.hkv;
  const int n = dec_len(p, s);
  const int qh0 = h * G;
  if (n <= 0) {
    // no rows (or a bad length, flagged): out = 0, lse = -inf
    if (sp == 0) {
      if (n < 0 && threadIdx.x == 0 && h == 0) atomicOr(p.status, 1);
      for (int i = threadIdx.x; i < G * 128; i += kDecThreads)
        p.out[((int64_t)s * p.hq + qh0) * 128 + i] = 0.f;
      if (p.lse != nullptr && threadIdx.x < G) p.lse[(int64_t)s * p.hq + qh0 + threadIdx.x] = -INFINITY;
    }
    return;
  }
  const int per = split_rows(n, p.nparts);
  const int r_begin = (sp * kDecWarps + warp) * per, r_end = min(n, r_begin + per);
  const int per_block = per * kDecWarps;
  if (sp * per_block >= n) return;  // the whole block is past the rows (uniform)
  const uint32_t ring = (uint32_t)__cvta_generic_to_shared(sm_dec + warp * kWarpSmem);
  constexpr int NT = (G + 7) / 8;  // 8-head column tiles

  // O^T accumulators: o[nt][mt] holds (dim 16 mt + gid, heads 8 nt + 2 tig,
  // + 1) and (dim 16 mt + gid + 8, the same heads)
  float o[NT][8][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
  // running maximum (base 2) and lane-partial sum of heads 8 nt + 2 tig + e
  float m[NT][2], l[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m[nt][0] = m[nt][1] = -INFINITY;
    l[nt][0] = l[nt][1] = 0.f;
  }

  if (r_begin < r_end) {
    // B fragments of the query per k-step: head 8 nt + gid (zero past G),
    // dims 16 ks + 2 tig, + 1 and 16 ks + 8 + 2 tig, + 1
    uint32_t qb[NT][8][2];
    {
      const uint32_t *q32 = reinterpret_cast<const uint32_t *>(p.q + ((int64_t)s * p.hq + qh0) * 128);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int hd = nt * 8 + gid;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          qb[nt][ks][0] = hd < G ? q32[hd * 64 + ks * 8 + tig] : 0u;
          qb[nt][ks][1] = hd < G ? q32[hd * 64 + ks * 8 + 4 + tig] : 0u;
        }
      }
    }
    // contiguous layout: this lane's first row of a tile, then a fixed stride
    const int64_t unit_off = (int64_t)s * p.s_seq + (int64_t)h * p.s_head + (lane & 15) * 8;
    // tile rows [r0, r0 + 16) of K and V into stage stg; rows past the range
    // and rows of invalid blocks are zero
    auto load_tile = [&](int r0, int stg) {
      const uint32_t kt = ring + (uint32_t)(stg * 2 * kTileBytes), vt = kt + kTileBytes;
      const bool full = r0 + kWTile <= r_end;
#pragma unroll
      for (int i = 0; i < kWTile / 2; ++i) {
        const int row = i * 2 + (lane >> 4), c = lane & 15;
        const int r = r0 + row;
        const uint32_t so = tile_off(row, c);
        bool ok;
        int64_t off;
        if (LAYOUT == TRIA_LAYOUT_CONTIGUOUS) {
          ok = full || r < r_end;
          off = unit_off + (int64_t)r * p.s_tok;
        } else {
          ok = false;
          off = 0;
          if (full || r < r_end) off = dec_row(p, s, h, r, ok) + c * 8;
        }
        if (ok) {
          cp_async16(kt + so, p.k + off);
          cp_async16(vt + so, p.v + off);
        } else {
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(kt + so), "r"(0u) : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vt + so), "r"(0u) : "memory");
        }
      }
    };

    const int ntiles = (r_end - r_begin + kWTile - 1) / kWTile;
#pragma unroll
    for (int i = 0; i < kWStages - 1; ++i) {
      if (i < ntiles) load_tile(r_begin + i * kWTile, i);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    const int mi = lane >> 3;  // the 8x8 matrix this lane addresses in an ldmatrix.x4
    for (int it = 0; it < ntiles; ++it) {
      const int r0 = r_begin + it * kWTile;
      if (it + kWStages - 1 < ntiles)
        load_tile(r0 + (kWStages - 1) * kWTile, (it + kWStages - 1) % kWStages);
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group %0;" ::"n"(kWStages - 1) : "memory");
      __syncwarp();
      const uint32_t kt = ring + (uint32_t)((it % kWStages) * 2 * kTileBytes), vt = kt + kTileBytes;

      // S = K Q^T: 16 rows x 8 heads per column tile, 8 k-steps; the K
      // fragments (rows gid, gid + 8) come straight from ldmatrix
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        ldsm_x4(kt + tile_off((lane & 7) + ((mi & 1) << 3), 2 * ks + (mi >> 1)), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma16816(sc[nt], a, qb[nt][ks][0], qb[nt][ks][1]);
      }
      // sc[nt][e]: row gid + 8 (e >> 1), head 8 nt + 2 tig + (e & 1)
      if (p.logits != nullptr) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int row = r0 + gid + 8 * (e >> 1);
            const int head = nt * 8 + 2 * tig + (e & 1);
            if (row < r_end && head < G)
              p.logits[((int64_t)s * p.hq + qh0 + head) * p.max_seq_len + row] = sc[nt][e] * p.scale;
          }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] *= p.qscale;
      if (r0 + kWTile > r_end) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (r0 + gid + 8 * (e >> 1) >= r_end) sc[nt][e] = -INFINITY;
      }
      // online softmax: the tile maximum of each head over its 16 rows (the
      // 8 lanes that share tig); the running maximum moves, and the
      // accumulators are rescaled, only when the tile exceeds it by more
      // than kRescale
      float t[NT][2];
      bool up = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float x = fmaxf(sc[nt][e], sc[nt][e + 2]);
          x = fmaxf(x, __shfl_xor_sync(kFull, x, 4));
          x = fmaxf(x, __shfl_xor_sync(kFull, x, 8));
          x = fmaxf(x, __shfl_xor_sync(kFull, x, 16));
          t[nt][e] = x;
          up = up || x > m[nt][e] + kRescale;  // always at the first tile
        }
      if (__any_sync(kFull, up)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float a[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float mn = t[nt][e] > m[nt][e] + kRescale ? t[nt][e] : m[nt][e];
            a[e] = exp2f(m[nt][e] - mn);  // 0 at the first tile
            m[nt][e] = mn;
            l[nt][e] *= a[e];
          }
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            o[nt][mt][0] *= a[0];
            o[nt][mt][1] *= a[1];
            o[nt][mt][2] *= a[0];
            o[nt][mt][3] *= a[1];
          }
        }
      }
      // weights; P^T as the B operand of O^T += V^T P^T: each 8x8 block of
      // P (rows x heads) transposed in registers (movmatrix), bf16 hi + lo
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sc[nt][e] = exp2f(sc[nt][e] - m[nt][e & 1]);
          l[nt][e & 1] += sc[nt][e];
        }
        uint32_t h0, l0, h1, l1;
        split2(sc[nt][0], sc[nt][1], h0, l0);  // rows 0..7
        split2(sc[nt][2], sc[nt][3], h1, l1);  // rows 8..15
        const uint32_t bh0 = movm_t(h0), bl0 = movm_t(l0), bh1 = movm_t(h1), bl1 = movm_t(l1);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          uint32_t a[4];
          // V^T fragments: dims 16 mt + gid (+ 8) x rows 2 tig (+ 8)
          ldsm_x4_t(vt + tile_off((lane & 7) + ((mi >> 1) << 3), 2 * mt + (mi & 1)), a[0], a[1], a[2], a[3]);
          mma16816(o[nt][mt], a, bh0, bh1);
          mma16816(o[nt][mt], a, bl0, bl1);
        }
      }
      __syncwarp();  // the stage is read: the next loads may overwrite it
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        l[nt][e] += __shfl_xor_sync(kFull, l[nt][e], 4);
        l[nt][e] += __shfl_xor_sync(kFull, l[nt][e], 8);
        l[nt][e] += __shfl_xor_sync(kFull, l[nt][e], 16);
      }
  }

  // merge the warps: (o, m, l) of every warp and head to shared memory (over
  // the rings), then O = sum_w 2^(m_w - M) o_w, L = sum_w 2^(m_w - M) l_w
  __syncthreads();
  float *wo = reinterpret_cast<float *>(sm_dec);          // [kDecWarps][G][128]
  float *wm = wo + kDecWarps * G * 128;                    // [kDecWarps][G]
  float *wl = wm + kDecWarps * G;                          // [kDecWarps][G]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int head = nt * 8 + 2 * tig + e;
      if (head < G) {
        float *dst = wo + (warp * G + head) * 128;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          dst[16 * mt + gid] = o[nt][mt][e];
          dst[16 * mt + gid + 8] = o[nt][mt][e + 2];
        }
        if (gid == 0) {
          wm[warp * G + head] = m[nt][e];
          wl[warp * G + head] = l[nt][e];
        }
      }
    }
  __syncthreads();
  for (int i = threadIdx.x; i < G * 128; i += kDecThreads) {
    const int g = i >> 7, d = i & 127;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wm[w * G + g]);
    float acc = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float a = wl[w * G + g] > 0.f ? exp2f(wm[w * G + g] - M) : 0.f;
      acc = fmaf(a, wo[(w * G + g) * 128 + d], acc);
      L = fmaf(a, wl[w * G + g], L);
    }
    float *pt = p.part + ((int64_t)(s * p.hq + qh0 + g) * p.splits + sp) * kPart;
    pt[d] = acc;
    if (d == 0) {
      pt[128] = M;
      pt[129] = L;
    }
  }

  // the last block of the unit to finish rescales the blocks' partials to
  // their common maximum (warp w: heads w, w + kDecWarps; lane l: dims
  // 4 l .. 4 l + 3) and resets the arrival count for the next call
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  const int ns = (n + per_block - 1) / per_block;  // blocks with rows
  if (threadIdx.x == 0) s_last = atomicAdd(p.arrived + u, 1u) == (uint32_t)(ns - 1) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x == 0) p.arrived[u] = 0u;
  for (int g = warp; g < G; g += kDecWarps) {
    const int64_t row = (int64_t)s * p.hq + qh0 + g;
    const float *pt = p.part + row * p.splits * kPart;
    constexpr int kMaxChunks = (kMaxSplits + 31) / 32;
    float mv[kMaxChunks], lv[kMaxChunks];
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int i = 32 * c + lane;
      mv[c] = i < ns ? __ldcg(pt + (int64_t)i * kPart + 128) : -INFINITY;
      lv[c] = i < ns ? __ldcg(pt + (int64_t)i * kPart + 129) : 0.f;
      M = fmaxf(M, mv[c]);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
    float L = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      mv[c] = lv[c] > 0.f ? exp2f(mv[c] - M) : 0.f;  // the partial's scale
      L = fmaf(lv[c], mv[c], L);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) L += __shfl_xor_sync(kFull, L, off);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) {
      const int cnt = min(32, ns - 32 * c);
      for (int b = 0; b < cnt; b += 8) {
        float4 x[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          x[k] = b + k < cnt ? __ldcg(reinterpret_cast<const float4 *>(pt + (int64_t)(32 * c + b + k) * kPart) + lane)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float a = __shfl_sync(kFull, mv[c], (b + k) & 31);
          acc.x = fmaf(a, x[k].x, acc.x);
          acc.y = fmaf(a, x[k].y, acc.y);
          acc.z = fmaf(a, x[k].z, acc.z);
          acc.w = fmaf(a, x[k].w, acc.w);
        }
      }
    }
    const float inv = 1.f / L;
    *reinterpret_cast<float4 *>(p.out + row * 128 + lane * 4) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (p.lse != nullptr && lane == 0) p.lse[row] = (M + log2f(L)) * kLn2;
  }
}

template <int G>
cudaError_t launch_decode_g(const DecodeParams &p, cudaStream_t st) {
  // the shared-memory opt-in once per device (it is a property of the kernel)
  static thread_local int attr_dev = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (attr_dev != dev) {
    e = cudaFuncSetAttribute(decode_kernel<G, TRIA_LAYOUT_CONTIGUOUS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<G, TRIA_LAYOUT_PAGED>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  const int64_t blocks = (int64_t)p.n_seq * p.hkv * p.splits;
  if (p.layout == TRIA_LAYOUT_CONTIGUOUS)
    decode_kernel<G, TRIA_LAYOUT_CONTIGUOUS><<<(unsigned)blocks, kDecThreads, kDecSmem, st>>>(p);
  else
    decode_kernel<G, TRIA_LAYOUT_PAGED><<<(unsigned)blocks, kDecThreads, kDecSmem, st>>>(p);
  return cudaGetLastError();
}

static_assert(kDecSmem <= 232448, "shared memory of the decode kernel");
static_assert(kDecWarps * 16 * 130 * 4 <= kDecSmem, "warp merge area over the rings (G = 16)");

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Host checks shared by both entry points; fills the model shape.
tria_status decode_check(const tria_stats *stats, const tria_cache_view *c, tria_model_desc *d,
                         int *splits) {
  if (stats == nullptr || c == nullptr) return TRIA_ERR_INVALID_ARG;
  tria_status st = tria_stats_desc(stats, d);
  if (st != TRIA_OK) return st;
  if (d->head_dim != TRIA_HEAD_DIM) return TRIA_ERR_UNSUPPORTED;
  if (c->n_seq < 1 || c->n_seq > TRIA_MAX_SEQS || c->max_seq_len < 1) return TRIA_ERR_INVALID_ARG;
  if (c->layout != TRIA_LAYOUT_CONTIGUOUS && c->layout != TRIA_LAYOUT_PAGED) return TRIA_ERR_INVALID_ARG;
  // blocks per (sequence, KV head): about one per SM over all units, no
  // more than one per kMinSplitRows rows of capacity
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return TRIA_ERR_CUDA;
  const int64_t units = (int64_t)c->n_seq * d->n_kv_heads;
  int64_t sp = (int64_t)sms / units;  // at most one wave of one block per SM
  if (sp > kMaxSplits) sp = kMaxSplits;
  const int64_t cap = (c->max_seq_len + kMinSplitRows - 1) / kMinSplitRows;
  if (sp > cap) sp = cap;
  if (sp < 1) sp = 1;
  if (units * sp > INT32_MAX) return TRIA_ERR_UNSUPPORTED;
  *splits = (int)sp;
  return TRIA_OK;
}

size_t decode_counters_bytes(const tria_cache_view *c, const tria_model_desc &d) {
  return ((size_t)c->n_seq * d.n_kv_heads * sizeof(uint32_t) + 255) / 256 * 256;
}

size_t decode_ws_bytes(const tria_cache_view *c, const tria_model_desc &d, int splits) {
  return kDecHeader + decode_counters_bytes(c, d) +
         (size_t)c->n_seq * d.n_q_heads * splits * kPart * sizeof(float);
}

}  // namespace
}  // namespace tria

using namespace tria;

extern "C" {

tria_status tria_decode_workspace_size(const tria_stats *stats, const tria_cache_view *cache,
                                       size_t *bytes) {
  if (bytes == nullptr) return TRIA_ERR_INVALID_ARG;
  tria_model_desc d;
  int splits = 0;
  const tria_status st = decode_check(stats, cache, &d, &splits);
  if (st != TRIA_OK) return st;
  *bytes = decode_ws_bytes(cache, d, splits);
  return TRIA_OK;
}

tria_status tria_decode_attention(const tria_stats *stats, const tria_cache_view *c, int layer,
                                  const void *q, float scale, float *out, float *lse,
                                  float *logits, void *ws, size_t ws_bytes, tria_stream_t stream) {
  tria_model_desc d;
  int splits = 0;
  tria_status st = decode_check(stats, c, &d, &splits);
  if (st != TRIA_OK) return st;
  if (layer < 0 || layer >= d.n_layers) return TRIA_ERR_INVALID_ARG;
  if (q == nullptr || out == nullptr || !aligned(q, 16) || !aligned(out, 16) || !std::isfinite(scale))
    return TRIA_ERR_INVALID_ARG;
  if ((lse != nullptr && !aligned(lse, 4)) || (logits != nullptr && !aligned(logits, 4)))
    return TRIA_ERR_INVALID_ARG;
  if (c->k_layers == nullptr || c->v_layers == nullptr) return TRIA_ERR_INVALID_ARG;
  const void *kb = c->k_layers[layer], *vb = c->v_layers[layer];
  if (kb == nullptr || vb == nullptr || !aligned(kb, 16) || !aligned(vb, 16)) return TRIA_ERR_INVALID_ARG;
  if (c->layer_seq_lens == nullptr && c->seq_lens == nullptr) return TRIA_ERR_INVALID_ARG;
  if (c->stride_head < 0 || c->stride_token <= 0 || c->stride_seq < 0 || c->stride_block < 0 ||
      (c->stride_head % 8) || (c->stride_token % 8) || (c->stride_seq % 8) || (c->stride_block % 8))
    return TRIA_ERR_INVALID_ARG;
  if (c->layout == TRIA_LAYOUT_PAGED) {
    const int bs = c->block_size;
    if (c->block_table == nullptr || c->max_blocks_per_seq < 1 || c->num_blocks < 1 ||
        !(bs == 8 || bs == 16 || bs == 32 || bs == 64 || bs == 128) ||
        (int64_t)c->max_blocks_per_seq * bs < c->max_seq_len)
      return TRIA_ERR_INVALID_ARG;
  }
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < decode_ws_bytes(c, d, splits))
    return TRIA_ERR_WORKSPACE;
  DecodeParams p{};
  p.k = static_cast<const uint16_t *>(kb);
  p.v = static_cast<const uint16_t *>(vb);
  p.q = static_cast<const uint16_t *>(q);
  p.block_table = c->block_table;
  if (c->layer_seq_lens != nullptr) {
    p.lens = c->layer_seq_lens + layer;
    p.lens_s = d.n_layers;
  } else {
    p.lens = c->seq_lens;
    p.lens_s = 1;
  }
  p.s_seq = c->stride_seq;
  p.s_head = c->stride_head;
  p.s_tok = c->stride_token;
  p.s_blk = c->stride_block;
  p.num_blocks = c->num_blocks;
  p.layout = c->layout;
  p.block_size = c->layout == TRIA_LAYOUT_PAGED ? c->block_size : 1;
  p.max_blocks = c->max_blocks_per_seq;
  p.max_seq_len = c->max_seq_len;
  p.n_seq = c->n_seq;
  p.hkv = d.n_kv_heads;
  p.hq = d.n_q_heads;
  p.splits = splits;
  p.nparts = splits * kDecWarps;
  p.scale = scale;
  p.qscale = (float)((double)scale * 1.4426950408889634);
  p.arrived = reinterpret_cast<uint32_t *>(static_cast<unsigned char *>(ws) + kDecHeader);
  p.part = reinterpret_cast<float *>(static_cast<unsigned char *>(ws) + kDecHeader +
                                     decode_counters_bytes(c, d));
  p.out = out;
  p.lse = lse;
  p.logits = logits;
  p.status = reinterpret_cast<int32_t *>(static_cast<unsigned char *>(ws) + 4);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (d.n_q_heads / d.n_kv_heads) {
    case 1: e = launch_decode_g<1>(p, s); break;
    case 2: e = launch_decode_g<2>(p, s); break;
    case 4: e = launch_decode_g<4>(p, s); break;
    case 8: e = launch_decode_g<8>(p, s); break;
    case 16: e = launch_decode_g<16>(p, s); break;
    default: return TRIA_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? TRIA_OK : TRIA_ERR_CUDA;
}

}  // extern "C"
