// Calibration reduction: the query statistics the scorer consumes, from a
// stream of pre-RoPE query vectors of one layer.  For every (query head h,
// band f) with the model's complex pairing (NEOX q_f = q[f] + i q[f + 64],
// interleaved q_f = q[2f] + i q[2f + 1]):
//   acc[h][f] += (sum_t Re q_f, sum_t Im q_f, sum_t |q_f|)
// and finalize divides by the token count: E[Re q_f], E[Im q_f], E|q_f|
// (GitHub issue #10 of the llama.cpp TurboQuant HIP fork, "Working
// calibration tool"; academ.us article 2607.13051 sec. 2: E[q_f] is the
// average of band-f queries over a calibration set).
//
// One warp reads one head's 256-byte query slice per token (lane l holds
// dims 4l..4l+3); blocks of 8 warps take one head and a range of tokens.  A
// lane sums 16 tokens in fp32 (|q_f| with sqrt.approx), folds that partial
// into fp64, the block reduces its warps in shared memory in a fixed order
// and adds its sums into acc with fp64 atomics.  HBM-bound: every query byte
// is read once.
#include <cuda_bf16.h>

#include "tria_device.cuh"

namespace tria {
namespace {

using namespace dev;

constexpr int kCalThreads = 256;
constexpr int kCalWarps = kCalThreads / 32;
constexpr int kCalUnroll = 16;  // tokens in flight per warp
constexpr int kCalChunk = 16;  // tokens per fp32 partial sum of a lane

struct CalParams {
  const uint16_t *q;
  int64_t n_tokens, s_tok, s_head;
  int hq, pairing;
  double *acc;  // [hq][64][3]
};

__device__ __forceinline__ float bfw_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bfw_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Lane sums for the bands this lane owns.  NEOX: lanes 0-15 own the real
// parts and |q_f| of bands 4l..4l+3 (the imaginary parts come from lane
// l + 16), lanes 16-31 the imaginary parts of bands 4(l-16)..; interleaved:
// lane l owns bands 2l and 2l + 1 entirely.
template <int PAIR>
__global__ void __launch_bounds__(kCalThreads) calib_kernel(const __grid_constant__ CalParams p) {
  const int h = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t per = (p.n_tokens + gridDim.y - 1) / gridDim.y;
  const int64_t t0 = (int64_t)blockIdx.y * per;
  const int64_t t1 = (t0 + per < p.n_tokens) ? t0 + per : p.n_tokens;
  const uint16_t *base = p.q + (int64_t)h * p.s_head + lane * 4;
  double a[4] = {0.0, 0.0, 0.0, 0.0};   // NEOX: Re or Im per band; interleaved: Re, Im of 2 bands
  double m[4] = {0.0, 0.0, 0.0, 0.0};   // |q_f| (NEOX lanes < 16: 4 bands; interleaved: 2 bands)
  // fp32 sums over kCalChunk consecutive tokens of this warp, folded into the
  // fp64 sums after each chunk
  for (int64_t c0 = t0 + warp; c0 < t1; c0 += (int64_t)kCalWarps * kCalChunk) {
    float a32[4] = {0.f, 0.f, 0.f, 0.f}, m32[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int g = 0; g < kCalChunk / kCalUnroll; ++g) {
      uint2 w[kCalUnroll];
#pragma unroll
      for (int u = 0; u < kCalUnroll; ++u) {
        const int64_t tt = c0 + (int64_t)(g * kCalUnroll + u) * kCalWarps;
        w[u] = (tt < t1) ? __ldcs(reinterpret_cast<const uint2 *>(base + tt * p.s_tok)) : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kCalUnroll; ++u) {
        const float x[4] = {bfw_lo(w[u].x), bfw_hi(w[u].x), bfw_lo(w[u].y), bfw_hi(w[u].y)};
        if (PAIR == TRIA_PAIR_NEOX) {
          float y[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) y[e] = __shfl_xor_sync(kFull, x[e], 16);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            a32[e] += x[e];
            m32[e] += sqrt_approx(fmaf(y[e], y[e], x[e] * x[e]));
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) a32[e] += x[e];
          m32[0] += sqrt_approx(fmaf(x[1], x[1], x[0] * x[0]));
          m32[1] += sqrt_approx(fmaf(x[3], x[3], x[2] * x[2]));
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      a[e] += (double)a32[e];
      m[e] += (double)m32[e];
    }
  }
  if (PAIR == TRIA_PAIR_NEOX && lane >= 16) {
#pragma unroll
    for (int e = 0; e < 4; ++e) m[e] = 0.0;  // the partner lane owns |q_f|
  }
  // reduce the block's warps in warp order, then one atomic add per value
  __shared__ double red[kCalWarps][32][8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    red[warp][lane][e] = a[e];
    red[warp][lane][4 + e] = m[e];
  }
  __syncthreads();
  if (warp == 0) {
    double s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      s[e] = 0.0;
      for (int w = 0; w < kCalWarps; ++w) s[e] += red[w][lane][e];
    }
    double *acc = p.acc + (int64_t)h * kBands * 3;
    if (PAIR == TRIA_PAIR_NEOX) {
      const int f0 = (lane & 15) * 4;
      const int comp = lane < 16 ? 0 : 1;  // Re or Im
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        atomicAdd(acc + (f0 + e) * 3 + comp, s[e]);
        if (lane < 16) atomicAdd(acc + (f0 + e) * 3 + 2, s[4 + e]);
      }
    } else {
      const int f0 = lane * 2;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        atomicAdd(acc + (f0 + b) * 3 + 0, s[2 * b]);
        atomicAdd(acc + (f0 + b) * 3 + 1, s[2 * b + 1]);
        atomicAdd(acc + (f0 + b) * 3 + 2, s[4 + b]);
      }
    }
  }
}

__global__ void calib_finalize_kernel(const double *acc, int n, double inv, float *re, float *im,
                                      float *ab) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  re[i] = (float)(acc[i * 3 + 0] * inv);
  im[i] = (float)(acc[i * 3 + 1] * inv);
  ab[i] = (float)(acc[i * 3 + 2] * inv);
}

}  // namespace
}  // namespace tria

using namespace tria;

extern "C" {

tria_status tria_calib_accumulate(const tria_model_desc *desc, const void *q, int64_t n_tokens,
                                  int64_t stride_token, int64_t stride_head, double *acc,
                                  tria_stream_t stream) {
  if (desc == nullptr || q == nullptr || acc == nullptr || n_tokens < 0) return TRIA_ERR_INVALID_ARG;
  if (desc->head_dim != TRIA_HEAD_DIM) return TRIA_ERR_UNSUPPORTED;
  if (desc->n_q_heads < 1 || desc->n_q_heads > 65535) return TRIA_ERR_INVALID_ARG;
  if (desc->pairing != TRIA_PAIR_NEOX && desc->pairing != TRIA_PAIR_INTERLEAVED)
    return TRIA_ERR_INVALID_ARG;
  if (stride_token < 0 || stride_head < 0 || (stride_token % 4) != 0 || (stride_head % 4) != 0 ||
      (reinterpret_cast<uintptr_t>(q) % 8) != 0 || (reinterpret_cast<uintptr_t>(acc) % 8) != 0)
    return TRIA_ERR_INVALID_ARG;
  if (n_tokens == 0) return TRIA_OK;
  CalParams p{};
  p.q = static_cast<const uint16_t *>(q);
  p.n_tokens = n_tokens;
  p.s_tok = stride_token;
  p.s_head = stride_head;
  p.hq = desc->n_q_heads;
  p.pairing = desc->pairing;
  p.acc = acc;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return TRIA_ERR_CUDA;
  // about 8 blocks per SM in total, at most one per 64 tokens of a head
  int64_t splits = ((int64_t)sms * 8 + p.hq - 1) / p.hq;
  const int64_t by_len = (n_tokens + 63) / 64;
  if (splits > by_len) splits = by_len;
  if (splits > 65535) splits = 65535;
  if (splits < 1) splits = 1;
  const dim3 grid((unsigned)p.hq, (unsigned)splits);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p.pairing == TRIA_PAIR_NEOX)
    calib_kernel<TRIA_PAIR_NEOX><<<grid, kCalThreads, 0, s>>>(p);
  else
    calib_kernel<TRIA_PAIR_INTERLEAVED><<<grid, kCalThreads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? TRIA_OK : TRIA_ERR_CUDA;
}

tria_status tria_calib_finalize(const tria_model_desc *desc, const double *acc, int64_t n_tokens,
                                float *q_mean_re, float *q_mean_im, float *q_abs_mean,
                                tria_stream_t stream) {
  if (desc == nullptr || acc == nullptr || q_mean_re == nullptr || q_mean_im == nullptr ||
      q_abs_mean == nullptr || n_tokens <= 0 || desc->n_q_heads < 1)
    return TRIA_ERR_INVALID_ARG;
  const int n = desc->n_q_heads * kBands;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  calib_finalize_kernel<<<(n + 255) / 256, 256, 0, s>>>(acc, n, 1.0 / (double)n_tokens, q_mean_re,
                                                         q_mean_im, q_abs_mean);
  return cudaGetLastError() == cudaSuccess ? TRIA_OK : TRIA_ERR_CUDA;
}

}  // extern "C"
