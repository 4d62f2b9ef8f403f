// Stats files: the calibrated query statistics (E[Re q_f], E[Im q_f], E|q_f|
// per layer, query head and band; GitHub issue #10 of the llama.cpp
// TurboQuant HIP fork, "Working calibration tool") with the model
// description, in this library's own little-endian format (layout in
// include/tria.h).  Host-only: no CUDA call.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <vector>

#include "../../include/tria.h"

namespace {

constexpr uint32_t kMagic = 0x54524941u;
constexpr uint32_t kVersion = 1u;
constexpr uint32_t kHasScales = 1u, kHasMask = 2u;

struct Header {
  uint32_t magic, version;
  int32_t n_layers, n_q_heads, n_kv_heads, head_dim, pairing, offset_log2_max;
  double rope_theta;
  uint32_t flags, reserved;
};
static_assert(sizeof(Header) == 48, "stats file header layout");

bool little_endian() {
  const uint32_t x = 1u;
  unsigned char b;
  std::memcpy(&b, &x, 1);
  return b == 1;
}

bool desc_ok(const tria_model_desc &d) {
  return d.n_layers >= 1 && d.n_layers <= TRIA_MAX_LAYERS && d.n_q_heads >= 1 && d.n_kv_heads >= 1 &&
         d.n_q_heads % d.n_kv_heads == 0 && d.head_dim >= 2 && d.head_dim % 2 == 0 &&
         (d.pairing == TRIA_PAIR_NEOX || d.pairing == TRIA_PAIR_INTERLEAVED) &&
         std::isfinite(d.rope_theta) && d.rope_theta > 1.0 && d.offset_log2_max >= 0 &&
         d.offset_log2_max <= 30;
}

size_t band_count(const tria_model_desc &d) {
  return (size_t)d.n_layers * d.n_q_heads * (d.head_dim / 2);
}

struct File {
  std::FILE *f;
  explicit File(std::FILE *p) : f(p) {}
  ~File() {
    if (f) std::fclose(f);
  }
};

}  // namespace

extern "C" {

tria_status tria_write_stats_file(const char *path, const tria_model_desc *desc,
                                  const float *q_mean_re, const float *q_mean_im,
                                  const float *q_abs_mean, const float *layer_budget_scales,
                                  const float *band_mask) {
  if (path == nullptr || desc == nullptr || q_mean_re == nullptr || q_mean_im == nullptr ||
      q_abs_mean == nullptr || !desc_ok(*desc))
    return TRIA_ERR_INVALID_ARG;
  if (!little_endian()) return TRIA_ERR_UNSUPPORTED;
  Header h{};
  h.magic = kMagic;
  h.version = kVersion;
  h.n_layers = desc->n_layers;
  h.n_q_heads = desc->n_q_heads;
  h.n_kv_heads = desc->n_kv_heads;
  h.head_dim = desc->head_dim;
  h.pairing = desc->pairing;
  h.offset_log2_max = desc->offset_log2_max;
  h.rope_theta = desc->rope_theta;
  h.flags = (layer_budget_scales ? kHasScales : 0u) | (band_mask ? kHasMask : 0u);
  File out(std::fopen(path, "wb"));
  if (out.f == nullptr) return TRIA_ERR_IO;
  const size_t n = band_count(*desc);
  bool ok = std::fwrite(&h, sizeof(h), 1, out.f) == 1 && std::fwrite(q_mean_re, 4, n, out.f) == n &&
            std::fwrite(q_mean_im, 4, n, out.f) == n && std::fwrite(q_abs_mean, 4, n, out.f) == n;
  if (ok && layer_budget_scales)
    ok = std::fwrite(layer_budget_scales, 4, (size_t)desc->n_layers, out.f) == (size_t)desc->n_layers;
  if (ok && band_mask)
    ok = std::fwrite(band_mask, 4, (size_t)desc->head_dim / 2, out.f) == (size_t)desc->head_dim / 2;
  ok = ok && std::fflush(out.f) == 0;
  return ok ? TRIA_OK : TRIA_ERR_IO;
}

tria_status tria_read_stats_file(const char *path, tria_model_desc *desc_out, int *has_scales,
                                 int *has_mask, float *q_mean_re, float *q_mean_im,
                                 float *q_abs_mean, float *layer_budget_scales,
                                 float *band_mask) {
  if (path == nullptr || desc_out == nullptr) return TRIA_ERR_INVALID_ARG;
  if (!little_endian()) return TRIA_ERR_UNSUPPORTED;
  File in(std::fopen(path, "rb"));
  if (in.f == nullptr) return TRIA_ERR_IO;
  Header h{};
  if (std::fread(&h, sizeof(h), 1, in.f) != 1 || h.magic != kMagic) return TRIA_ERR_IO;
  if (h.version != kVersion) return TRIA_ERR_UNSUPPORTED;
  tria_model_desc d{};
  d.n_layers = h.n_layers;
  d.n_q_heads = h.n_q_heads;
  d.n_kv_heads = h.n_kv_heads;
  d.head_dim = h.head_dim;
  d.pairing = h.pairing;
  d.rope_theta = h.rope_theta;
  d.offset_log2_max = h.offset_log2_max;
  if (!desc_ok(d) || (h.flags & ~(kHasScales | kHasMask)) != 0) return TRIA_ERR_IO;
  const bool sc = (h.flags & kHasScales) != 0, mk = (h.flags & kHasMask) != 0;
  if ((layer_budget_scales && !sc) || (band_mask && !mk)) return TRIA_ERR_INVALID_ARG;
  // the file must hold every array its header announces
  const size_t n = band_count(d);
  const size_t body = 3 * n + (sc ? (size_t)d.n_layers : 0) + (mk ? (size_t)d.head_dim / 2 : 0);
  if (std::fseek(in.f, 0, SEEK_END) != 0) return TRIA_ERR_IO;
  const long size = std::ftell(in.f);
  if (size < 0 || (size_t)size != sizeof(Header) + 4 * body) return TRIA_ERR_IO;
  // arrays in file order; a null pointer skips its array
  auto read = [&](float *dst, size_t count, size_t at) {
    if (dst == nullptr) return true;
    return std::fseek(in.f, (long)(sizeof(Header) + 4 * at), SEEK_SET) == 0 &&
           std::fread(dst, 4, count, in.f) == count;
  };
  const size_t at_scales = 3 * n, at_mask = 3 * n + (sc ? (size_t)d.n_layers : 0);
  if (!read(q_mean_re, n, 0) || !read(q_mean_im, n, n) || !read(q_abs_mean, n, 2 * n) ||
      !read(layer_budget_scales, (size_t)d.n_layers, at_scales) ||
      !read(band_mask, (size_t)d.head_dim / 2, at_mask))
    return TRIA_ERR_IO;
  *desc_out = d;
  if (has_scales) *has_scales = sc ? 1 : 0;
  if (has_mask) *has_mask = mk ? 1 : 0;
  return TRIA_OK;
}

}  // extern "C"
