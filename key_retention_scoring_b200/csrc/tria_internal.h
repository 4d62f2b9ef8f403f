// Internal declarations shared by the host entry points (tria_api.cu) and the
// kernels (tria_kernels.cu).  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/tria.h"

namespace tria {

constexpr int kHeadDim = 128;
constexpr int kBands = 64;          // d / 2 RoPE bands
constexpr int kCoefK = 256;         // K extent of the coefficient tile: 128 key dims + 2 x 64 bands
constexpr int kTileKeys = 1024;     // keys per scheduling item of the score kernel
constexpr int kRowGroups = 4;       // moment partials per item: one per 32-row group of a tile
constexpr int kMaxSeqTable = TRIA_MAX_SEQS + 1;
constexpr int kMaxOffsets = 17;     // |D| bound of the max-over-offsets form

// Device copy of the folded statistics.
struct StatsDev {
  tria_model_desc desc;
  double2 *mu_fold;   // [L][Hq][F]  mu'_f = E[q_f] W_f mask_f   (complex, fp64)
  double2 *mu_raw;    // [L][Hq][F]  E[q_f] mask_f (unfolded: the max-over-offsets form)
  double *w_norm;     // [L][Hq][F]  E|q_f| - |E q_f|            (fp64)
  double *omega;      // [F]         theta^(-2f/d)               (fp64)
  double2 *rot_off;   // [F][kMaxOffsets] e^{i omega_f 2^j}, j < min(|D|, kMaxOffsets) (fp64)
};

// Per-call geometry.
struct Geom {
  int ncol;      // coefficient tile rows: max(16, 2G)
  int n_seq;
  int nl;        // layers in [layer0, layer1)
  int layer0;
  int n_layers;  // of the model
  int hkv, hq, g;
  int budget;    // B_max: kept_idx row length (max over the model's layers)
  int window, sinks;
  int trigger;   // max(interval, 1): a unit is compressed when N - B_l >= trigger
  int per_layer; // lengths per (sequence, layer) (layer_seq_lens)
  // N of unit (s, lrel) = lens[s * lens_s + lrel * lens_l]
  const int32_t *lens;
  int64_t lens_s;
  int lens_l;
  int lbudget[TRIA_MAX_LAYERS];  // B_l of call layer lrel (layer0 + lrel)
  int max_seq_len;
  int c_max;     // max_seq_len - window - sinks (>= 1)
  int tiles_max; // upper bound of the scheduling tiles of one unit
  int pairing;
  int64_t n_units;  // n_seq * nl * hkv
  int mode;      // TRIA_OFFSET_MEAN / TRIA_OFFSET_MAX
  int n_off;     // |D| = offset_log2_max + 1
  int ncol_t;    // max mode: trig operand rows, |D| G rounded up to 16
  int ncol_n;    // max mode: norm operand rows, max(16, 2G)
  int b_bytes;   // bytes of one unit's coefficient image
  int grouped;   // paged scoring tiles of one block x all KV heads (tria_score_grouped.cu):
                 // the units of a (sequence, layer) share one image of 2G columns each
};

// Cache addressing (pointers indexed by layer - layer0).
struct CacheDev {
  int layout;
  int block_size;
  int max_blocks;
  int64_t s_seq, s_head, s_tok, s_blk;
  const int32_t *block_table;
  int32_t *seq_lens;
  const int64_t *query_pos;
  int32_t *positions;
  int64_t pos_unit_stride;  // max_seq_len
  const uint16_t *k[TRIA_MAX_LAYERS];
  uint16_t *v[TRIA_MAX_LAYERS];
};

// Workspace carve-up (byte offsets from the workspace base).
struct WsLayout {
  size_t hdr;         // 256 B: u32 item counter, i32 status flags
  size_t unit_done;   // n_units x u32: finished normalization chunks per unit
  size_t seq_items;   // (n_seq + 1) x i32 prefix of scheduling items per sequence
  size_t row_items;   // (n_seq x nl + 1) x i32 prefix per (sequence, layer) (per-layer lengths)
  size_t btile;       // n_units x ncol x kCoefK bf16 coefficient tiles
  size_t moments;     // n_units x tiles_max x kRowGroups x g x 2 fp64
  size_t hist;        // n_units x kAggHistBins u32: histogram of the top 12 bits of agg keys
  size_t raw;         // n_units x raw_stride fp32
  size_t agg;         // n_units x agg_stride fp32
  size_t kept;        // n_units x budget i32
  size_t total;
  int64_t raw_stride; // floats per unit, multiple of 32
  int64_t agg_stride; // floats per unit, multiple of 32
};

constexpr int kAggHistBins = 4096;
constexpr int kAggChunk = 4096;   // candidates per block of the normalization kernel
constexpr int kMaxTailCluster = 8;         // blocks per unit of the cluster tail (portable cluster size)
constexpr size_t kMaxDynSmem = 232448;     // opt-in shared memory per block (227 KB)

WsLayout ws_layout(const Geom &g);

// Max-over-offsets mode: columns of the trig accumulator and B-image rows.
constexpr int kMaxOffCols = 272;   // 2 |D| G <= 272 (|D| G <= 136)

// Score-kernel parameters.
struct ScoreParams {
  CUtensorMap kmap[TRIA_MAX_LAYERS];  // K of each layer in [layer0, layer1): 128B-swizzled boxes
  Geom geo;
  CacheDev cache;
  const uint16_t *btile;  // [unit][ncol][kCoefK] bf16, shared-memory image
  uint32_t *item_counter;
  int32_t *status;
  const int32_t *seq_items;
  const int32_t *row_items;  // per-layer lengths: prefix per (sequence, layer)
  double *moments;
  float *raw;           // [unit][raw_stride], per candidate G floats
  int64_t raw_stride;
  uint64_t wait_ns;     // bound of every wait in the kernel (0: 2 s)
};

// Normalize-then-max (and selection) kernel parameters.
struct TailParams {
  Geom geo;
  int32_t *status;
  const double *moments;
  float *raw;
  int64_t raw_stride;
  float *agg;
  int64_t agg_stride;
  int32_t *kept;        // null: agg only
  uint32_t *hist;       // [unit][kAggHistBins]
  uint32_t *unit_done;  // [unit]
  int discard_raw;      // raw is workspace scratch: drop its L2 lines after use
  int discard_agg;      // agg is workspace scratch
  int cluster;          // unit tail: blocks per unit (a thread-block cluster)
  int slice;            // unit tail: candidates per block (a multiple of 128)
};

struct CoefParams {
  Geom geo;
  const double2 *mu_fold;
  const double2 *mu_raw;
  const double *w_norm;
  const double *omega;
  const double2 *rot_off;
  const int64_t *query_pos;
  uint16_t *btile;
  uint32_t *item_counter;
  uint32_t *unit_done;
  int32_t *seq_items;
  int32_t *row_items;
  int32_t *status;
  int32_t *kept;      // identity rows for units that are not compressed (may be null)
  uint32_t *hist;     // zeroed per unit (may be null)
};

struct SelectParams {
  Geom geo;
  int32_t *status;
  const float *agg;
  int64_t agg_stride;
  int32_t *kept;
};

struct CompactParams {
  Geom geo;
  CacheDev cache;
  const int32_t *kept;
  int update_lens;      // layer1 == n_layers (one length per sequence)
  int32_t *freed_blocks;
  int32_t *n_freed;
};

// Per-(sequence, layer) lengths after compaction, and the freed blocks.
struct LensParams {
  Geom geo;
  int32_t *layer_lens;  // [n_seq][n_layers]
  const int32_t *block_table;
  int max_blocks, block_size, paged;
  int all_layers;       // the call covers every layer: blocks may be freed
  int32_t *freed_blocks;
  int32_t *n_freed;
};

// Launchers (tria_kernels.cu).  Return cudaGetLastError() of the launch.
cudaError_t launch_coef(const CoefParams &p, cudaStream_t st);
// Scoring (tria_score_tc.cu): raw scores and moment partials of every
// candidate; the max-over-offsets mode is launched by launch_score_max
// (tria_score_max.cu).
cudaError_t launch_score(const ScoreParams &p, cudaStream_t st);
cudaError_t launch_score_max(const ScoreParams &p, cudaStream_t st);
cudaError_t launch_score_grouped(const ScoreParams &p, cudaStream_t st);
cudaError_t launch_tail(const TailParams &p, cudaStream_t st);
cudaError_t launch_select(const SelectParams &p, cudaStream_t st);
// Normalize-then-max + selection with one thread-block cluster per unit and
// the agg keys in shared memory (kept != null; tria_tail.cu); only when
// unit_tail_fits(geo).
bool unit_tail_fits(const Geom &g);
cudaError_t launch_unit_tail(const TailParams &p, cudaStream_t st);
cudaError_t launch_compact(const CompactParams &p, cudaStream_t st);
cudaError_t launch_layer_lens(const LensParams &p, cudaStream_t st);

// Length N of unit (s, lrel) and whether the pass compresses it.
__host__ __device__ __forceinline__ int unit_len(const Geom &g, int s, int lrel) {
  return g.lens[(int64_t)s * g.lens_s + (int64_t)lrel * g.lens_l];
}
__host__ __device__ __forceinline__ bool len_valid(const Geom &g, int n) {
  return n >= 0 && n <= g.max_seq_len;
}
__host__ __device__ __forceinline__ bool compresses(const Geom &g, int n, int lrel) {
  return len_valid(g, n) && n - g.lbudget[lrel] >= g.trigger;
}

}  // namespace tria
