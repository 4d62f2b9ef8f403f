// Device-side seeded generator of synthetic KV caches (test and benchmark
// input only; not part of the compression library).
//
// Row recipe for (sequence s, layer l, KV head h, position p):
//   pre-RoPE key  x_j = center[h][j] + sigma * n_j,  n_j ~ N(0,1) from
//                 Philox4x32-10 counter (p, j/4 + 32h, l + 256s, 4), key (seed, "tria"),
//                 Box-Muller on the four uniforms (x+0.5)/2^32;
//   post-RoPE     band f = (x_a, x_b) turned by the angle omega_f * p, with
//                 omega_f = theta^(-2f/128), in fp64; pairs (a, b) = (f, f+64) (NEOX)
//                 or (2f, 2f+1) (interleaved); rounded fp64 -> fp32 -> bf16 (nearest even);
//   value         v_j ~ N(0,1) from counter (p, j/4 + 32h, l + 256s, 5).
// The Philox rounds follow the published definition (Salmon et al., SC'11).
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
constexpr uint32_t kKeyTag = 0x74726961u;

__device__ __forceinline__ uint4 philox(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(kM0, c.x), lo0 = kM0 * c.x;
    const uint32_t hi1 = __umulhi(kM1, c.z), lo1 = kM1 * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += kW0;
    k1 += kW1;
  }
  return c;
}

__device__ __forceinline__ double u01(uint32_t x) { return ((double)x + 0.5) * (1.0 / 4294967296.0); }

__device__ __forceinline__ void normals4(uint4 c, uint32_t seed, double out[4]) {
  const uint4 r = philox(c, seed, kKeyTag);
  const double ra = sqrt(-2.0 * log(u01(r.x))), rb = sqrt(-2.0 * log(u01(r.z)));
  const double two_pi = 6.283185307179586476925286766559;
  double s, co;
  sincos(two_pi * u01(r.y), &s, &co);
  out[0] = ra * co;
  out[1] = ra * s;
  sincos(two_pi * u01(r.w), &s, &co);
  out[2] = rb * co;
  out[3] = rb * s;
}

__device__ __forceinline__ uint16_t to_bf16(double v) {
  const float f = (float)v;
  uint32_t u = __float_as_uint(f);
  if (f != f) return 0x7FC0u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

struct FillArgs {
  uint16_t *k;
  uint16_t *v;
  int layout;  // 0 contiguous, 1 paged
  int64_t s_seq, s_head, s_tok, s_blk;
  const int32_t *block_table;
  int max_blocks, block_size;
  int n_seq, hkv;
  const int32_t *slot0;
  const int32_t *count;
  const int64_t *pos0;
  const float *centers;  // [hkv][128]
  int layer;
  uint32_t seed;
  int pairing;
  double theta;
  double sigma;
  int max_count;
  int32_t *positions;  // optional [n_seq][n_layers][hkv][pos_len]
  int n_layers;
  int pos_len;
};

__device__ __forceinline__ int64_t row_off(const FillArgs &a, int s, int h, int t) {
  if (a.layout == 0) return (int64_t)s * a.s_seq + (int64_t)h * a.s_head + (int64_t)t * a.s_tok;
  const int blk = a.block_table[(int64_t)s * a.max_blocks + t / a.block_size];
  return (int64_t)blk * a.s_blk + (int64_t)(t % a.block_size) * a.s_tok + (int64_t)h * a.s_head;
}

// one warp per row; grid.x over rows of (s, h), grid.y = n_seq * hkv
__global__ void __launch_bounds__(256) fill_kernel(const FillArgs a) {
  __shared__ double pre[8][128];
  __shared__ uint16_t post[8][128];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sh = blockIdx.y;
  const int s = sh / a.hkv, h = sh % a.hkv;
  const int r = blockIdx.x * 8 + w;
  const int cnt = a.count[s];
  if (r >= cnt) return;
  const int slot = a.slot0[s] + r;
  const int64_t p = a.pos0[s] + r;
  const uint32_t lz = (uint32_t)(a.layer + 256 * s);
  double n[4];
  normals4(make_uint4((uint32_t)p, (uint32_t)(lane + 32 * h), lz, 4u), a.seed, n);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    pre[w][4 * lane + i] = (double)a.centers[h * 128 + 4 * lane + i] + a.sigma * n[i];
  __syncwarp();
  // two bands per lane
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int f = 2 * lane + i;
    const int ia = a.pairing == 0 ? f : 2 * f;
    const int ib = a.pairing == 0 ? f + 64 : 2 * f + 1;
    const double om = pow(a.theta, -2.0 * f / 128.0);
    double sn, cs;
    sincos(om * (double)p, &sn, &cs);
    const double xa = pre[w][ia], xb = pre[w][ib];
    post[w][ia] = to_bf16(xa * cs - xb * sn);
    post[w][ib] = to_bf16(xa * sn + xb * cs);
  }
  __syncwarp();
  const int64_t off = row_off(a, s, h, slot);
  // 128 bf16 = 256 B: each lane writes 8 B
  uint2 kv;
  kv.x = (uint32_t)post[w][4 * lane] | ((uint32_t)post[w][4 * lane + 1] << 16);
  kv.y = (uint32_t)post[w][4 * lane + 2] | ((uint32_t)post[w][4 * lane + 3] << 16);
  *reinterpret_cast<uint2 *>(a.k + off + 4 * lane) = kv;
  if (a.v != nullptr) {
    normals4(make_uint4((uint32_t)p, (uint32_t)(lane + 32 * h), lz, 5u), a.seed, n);
    uint2 vv;
    vv.x = (uint32_t)to_bf16(n[0]) | ((uint32_t)to_bf16(n[1]) << 16);
    vv.y = (uint32_t)to_bf16(n[2]) | ((uint32_t)to_bf16(n[3]) << 16);
    *reinterpret_cast<uint2 *>(a.v + off + 4 * lane) = vv;
  }
  if (a.positions != nullptr && lane == 0) {
    const int64_t pu = ((int64_t)s * a.n_layers + a.layer) * a.hkv + h;
    a.positions[pu * a.pos_len + slot] = (int32_t)p;
  }
}

}  // namespace

extern "C" int synth_fill_layer(void *k, void *v, int layout, int64_t s_seq, int64_t s_head,
                                int64_t s_tok, int64_t s_blk, const int32_t *block_table,
                                int max_blocks, int block_size, int n_seq, int hkv,
                                const int32_t *slot0, const int32_t *count, const int64_t *pos0,
                                const float *centers, int layer, uint32_t seed, int pairing,
                                double theta, double sigma, int max_count, int32_t *positions,
                                int n_layers, int pos_len, cudaStream_t stream) {
  if (k == nullptr || centers == nullptr || slot0 == nullptr || count == nullptr ||
      pos0 == nullptr || n_seq < 1 || hkv < 1 || max_count < 0)
    return 1;
  if (max_count == 0) return 0;
  FillArgs a{};
  a.k = static_cast<uint16_t *>(k);
  a.v = static_cast<uint16_t *>(v);
  a.layout = layout;
  a.s_seq = s_seq;
  a.s_head = s_head;
  a.s_tok = s_tok;
  a.s_blk = s_blk;
  a.block_table = block_table;
  a.max_blocks = max_blocks;
  a.block_size = block_size > 0 ? block_size : 1;
  a.n_seq = n_seq;
  a.hkv = hkv;
  a.slot0 = slot0;
  a.count = count;
  a.pos0 = pos0;
  a.centers = centers;
  a.layer = layer;
  a.seed = seed;
  a.pairing = pairing;
  a.theta = theta;
  a.sigma = sigma;
  a.max_count = max_count;
  a.positions = positions;
  a.n_layers = n_layers;
  a.pos_len = pos_len;
  dim3 grid((unsigned)((max_count + 7) / 8), (unsigned)(n_seq * hkv));
  fill_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
