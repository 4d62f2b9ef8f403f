/*
 * tria.h - C ABI of the B200 (sm_100a) TriAttention KV-cache compression pass.
 *
 * The pass, for every cached key of every layer and KV head ("unit" =
 * (sequence, layer, KV head)):
 *   1. splits the 128-wide head into 64 RoPE bands (NEOX half split or
 *      interleaved pairs) and scores the key against calibrated query
 *      statistics:  S~(k) = S~_trig(k) + S_norm(k)
 *      - S~_trig is the trigonometric term of Eq. (2) of the academ.us article
 *        2607.13051 ("a small improvement to one step of TriAttention"),
 *        averaged over the future offsets D = {1, 2, 4, ..., 2^m} (Eq. 4),
 *        evaluated through the folded centers mu'_f = E[q_f] W_f of Eq. (7);
 *      - S_norm(k) = sum_f (E|q_f| - |E q_f|) |k_f|, the distance-independent
 *        term that weighs a key's own band magnitudes by (1 - R_f)
 *        (ghidav.me, "TriAttention, or: what a rotating query already knows",
 *        section "The Method");
 *   2. z-normalises the score of each query head over the unit's candidates
 *      and takes the max over the query heads sharing the KV head
 *      (article 2607.13051, sec. 4, "normalize-then-max");
 *   3. keeps the top-K candidates, always keeping the first `sinks` and the
 *      last `window` slots, `budget` rows in all (ghidav.me, "The Method":
 *      sort, keep the top B, drop the rest; GitHub issue #10 of the llama.cpp
 *      TurboQuant HIP fork, runtime log: window 256, interval 128, sink 0);
 *   4. gathers the kept K/V rows to the front of each unit, in place, in
 *      ascending slot order ("per-layer compaction path", triattention README).
 *
 * Conventions for every entry point:
 *   - Pointers documented "device" are CUDA device pointers owned by the
 *     caller; "host" pointers are read during the call only.
 *   - All work is enqueued on `stream` (NULL = legacy default stream) and is
 *     asynchronous; no entry point synchronises except tria_load_stats,
 *     tria_free_stats and tria_read_device_status.
 *   - Arguments are validated on the host before anything is enqueued; a
 *     validation failure returns an error and enqueues nothing.
 *   - Launch failures return TRIA_ERR_CUDA.
 *   - The library allocates device memory only in tria_load_stats (the stats
 *     object); scoring, selection and compaction never allocate.
 *   - bf16 K/V rows are 128 elements (256 bytes); row starts must be 16-byte
 *     aligned (strides multiples of 8 elements, 16-byte aligned bases).  The
 *     scoring kernel reads K through TMA tensor maps that the library encodes
 *     (and caches) per layer base pointer; a stride pattern the tensor-map
 *     encoder rejects returns TRIA_ERR_UNSUPPORTED.
 *   - A unit whose length N is at most its layer's budget B_l (plus the
 *     compression interval, see tria_params) is left unchanged.
 *   - Floating point decides the kept set only through the fp32 aggregated
 *     score agg (below); exactly equal agg go to the lower slot; -0.0 equals
 *     +0.0; NaN ranks below every number.
 */
#ifndef TRIA_H
#define TRIA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *tria_stream_t;

typedef enum {
  TRIA_OK = 0,
  TRIA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or range */
  TRIA_ERR_UNSUPPORTED = 2, /* valid but not built: head_dim != 128, G > 16 */
  TRIA_ERR_WORKSPACE = 3,   /* workspace null, not 256-byte aligned, or smaller than required */
  TRIA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  TRIA_ERR_OOM = 5,         /* device allocation failed (tria_load_stats) */
  TRIA_ERR_IO = 6           /* a stats file could not be opened, read or written,
                               or is not in this library's format */
} tria_status;

typedef enum {
  TRIA_PAIR_NEOX = 0,        /* band f = x[f] + i x[f + d/2]   (Qwen, NEOX)   */
  TRIA_PAIR_INTERLEAVED = 1  /* band f = x[2f] + i x[2f + 1]   (Llama, NORM)  */
} tria_pairing;

typedef enum {
  TRIA_LAYOUT_CONTIGUOUS = 0, /* row = k_layers[l] + s*stride_seq + h*stride_head + t*stride_token */
  TRIA_LAYOUT_PAGED = 1       /* row = k_layers[l] + block_table[s][t / block_size]*stride_block
                                       + (t % block_size)*stride_token + h*stride_head */
} tria_layout;

#define TRIA_HEAD_DIM 128
#define TRIA_MAX_LAYERS 128
#define TRIA_MAX_GROUP 16
#define TRIA_MAX_SEQS 1024

/* Model shape and RoPE convention. */
typedef struct {
  int n_layers;        /* 1 .. TRIA_MAX_LAYERS                                  */
  int n_q_heads;       /* Hq; a multiple of n_kv_heads                          */
  int n_kv_heads;      /* Hkv; G = Hq / Hkv in 1 .. TRIA_MAX_GROUP              */
  int head_dim;        /* d; only 128 is built                                  */
  int pairing;         /* tria_pairing                                          */
  double rope_theta;   /* theta of omega_f = theta^(-2f/d) (article 2607.13051,
                          sec. 2, list under Eq. 2); > 1                        */
  int offset_log2_max; /* m of D = {2^0 .. 2^m}; the published method uses 16
                          (article 2607.13051, Eq. 4); 0 .. 30                  */
} tria_model_desc;

/* Opaque, library-owned device copy of the folded statistics. */
typedef struct tria_stats tria_stats;

/* The caller's KV cache.  Every pointer stays owned by the caller.
 * Zero-initialise the struct: optional fields are off at zero (NULL). */
typedef struct {
  int layout;                /* tria_layout                                          */
  int n_seq;                 /* 1 .. TRIA_MAX_SEQS                                   */
  int max_seq_len;           /* host: upper bound of every seq_lens[s]; sizes the
                                candidate axis C_max = max_seq_len - window - sinks.
                                Contiguous layout: every (sequence, KV head) has room
                                for max_seq_len rows.                                */
  void *const *k_layers;     /* host array [n_layers] of device pointers, bf16 K     */
  void *const *v_layers;     /* host array [n_layers] of device pointers, bf16 V;
                                needed by compaction only                            */
  int64_t stride_seq;        /* elements between sequences (contiguous layout)       */
  int64_t stride_head;       /* elements between KV heads                            */
  int64_t stride_token;      /* elements between slots (contiguous) or between the
                                rows of one block (paged)                            */
  int64_t stride_block;      /* elements between blocks (paged)                      */
  const int32_t *block_table;/* device [n_seq][max_blocks_per_seq] (paged)           */
  int max_blocks_per_seq;    /* paged                                                */
  int block_size;            /* rows per block (paged): 8, 16, 32, 64 or 128         */
  int64_t num_blocks;        /* paged: blocks in each layer's K (and V) pool; block
                                ids outside [0, num_blocks) read as zero rows        */
  int32_t *seq_lens;         /* device [n_seq] cached tokens N per sequence; set to
                                the budget for every compressed sequence by
                                tria_compact when it covers the last layer           */
  const int64_t *query_pos;  /* device [n_seq] position p_q of the current query: the
                                position of the newest cached token (offsets
                                delta in D are added to it)                          */
  int32_t *positions;        /* optional device [n_seq][n_layers][n_kv_heads][max_seq_len]
                                token position of every slot; compacted with the
                                rows when non-null.  Scoring never reads it: the
                                post-RoPE key already carries its position.          */
  int32_t *layer_seq_lens;   /* optional device [n_seq][n_layers]: cached tokens N of
                                each (sequence, layer).  When non-null it replaces
                                seq_lens (which is then neither read nor written and
                                may be NULL) and tria_compact updates the entries of
                                the layers it covers.  Required when the per-layer
                                budgets differ (tria_params.layer_budget_scales),
                                since the layers then keep different lengths.        */
} tria_cache_view;

/* How the trigonometric term combines the future offsets delta in D. */
typedef enum {
  TRIA_OFFSET_MEAN = 0, /* the mean over D (academ.us article 2607.13051 Eq. 4), the
                           published default; computed folded (Eq. 7)               */
  TRIA_OFFSET_MAX = 1   /* the maximum over D instead (the non-default variant named
                           at the end of sec. 4 of the same article); not foldable:
                           |D| scores per head per key.  Needs G <= 8, |D| <= 17
                           and G * |D| <= 136, else UNSUPPORTED                    */
} tria_offset_reduce;

/* Retention parameters (one set for all units of a call).  Zero-initialise
 * the struct and set what is needed: every field past `sinks` is off at zero.
 *
 * Budget of layer l (rows kept per unit, window and sinks included):
 *   base = budget_pct > 0 ? floor(budget_pct * max_seq_len / 100) : budget
 *   B_l  = floor(base * scale_l + 1/2), scale_l = layer_budget_scales[l] (1 if NULL)
 * (the runtime of GitHub issue #10 of the llama.cpp TurboQuant HIP fork takes a
 * percentage budget, "budget=50%", and per-layer budget scales that default to
 * 1.0; the percentage is read as a share of the cache capacity max_seq_len).
 * Every B_l must be >= window + sinks, else INVALID_ARG.  A unit with N cached
 * rows is compressed only when N - B_l >= max(interval, 1): pruning runs once
 * per window of interval generated tokens (academ.us article 2607.13051, sec. 8,
 * beta = 128; the same issue's runtime log, "interval=128"); every other unit is
 * left as it is.  kept_idx rows have B_max = max_l B_l entries (over all layers
 * of the model; tria_layer_budgets returns it). */
typedef struct {
  int budget;  /* B: rows kept per unit, window and sinks included; >= window + sinks */
  int window;  /* W: the newest W slots are always kept                               */
  int sinks;   /* S: the oldest S slots are always kept                               */
  int offset_reduce;  /* tria_offset_reduce; 0 (mean) when zero-initialised           */
  float budget_pct;   /* > 0: percentage budget, replaces budget (see above); 0: off  */
  const float *layer_budget_scales;  /* optional host [n_layers], finite and > 0;
                                        NULL = 1.0 for every layer                   */
  int interval;       /* compression interval beta >= 0 (0 and 1: compress whenever
                         N > B_l)                                                   */
  int64_t wait_limit_ns; /* >= 0: bound, in ns, of every wait of the scoring kernel on
                            its pipeline (tile loads, MMA results, hand-offs between
                            its warps); 0 = 2 s.  A wait that runs out sets status
                            bit 1 (tria_read_device_status), the kernel lets its own
                            loads and MMAs land and returns; the call's results are
                            then undefined.  A limit far below a kernel's run time
                            makes that happen on purpose (tests of the abort path). */
} tria_params;

/* Human-readable name of a status code (static string). */
const char *tria_status_string(tria_status status);

/* Library version string (static). */
const char *tria_version(void);

/*
 * tria_load_stats - fold calibrated query statistics into a device object.
 *
 * Inputs (host, fp32, [n_layers][n_q_heads][head_dim/2], band f innermost):
 *   q_mean_re, q_mean_im : E[Re q_f], E[Im q_f] of the pre-RoPE query bands;
 *   q_abs_mean           : E|q_f|
 *   (the three statistics of the calibration tool in GitHub issue #10 of the
 *   llama.cpp TurboQuant HIP fork, paired as desc->pairing says);
 *   band_mask            : optional host [head_dim/2] per-band multiplier of
 *                          |mu'_f| (the high-frequency mask of article
 *                          2607.13051, sec. 7); NULL = all ones.
 * On the host, in fp64: W_f = (1/|D|) sum_{delta in D} e^{i omega_f delta}
 * (Eq. 6), mu'_f = E[q_f] W_f mask_f (Eq. 7), w_f = E|q_f| - |E q_f|.
 * The result is copied to the device (stream-ordered, then synchronised).
 * *out receives a new object; free it with tria_free_stats.
 * Errors: INVALID_ARG (null pointer, non-finite input, bad desc),
 * UNSUPPORTED (head_dim != 128, G > TRIA_MAX_GROUP), OOM, CUDA.
 */
tria_status tria_load_stats(const tria_model_desc *desc, const float *q_mean_re,
                            const float *q_mean_im, const float *q_abs_mean,
                            const float *band_mask, tria_stream_t stream,
                            tria_stats **out);

/*
 * Stats files: this library's own format for the calibrated statistics (the
 * llama.cpp port's stats.bin layout is not documented, so it is not read).
 * Little-endian, no padding:
 *   offset  size  field
 *   0       4     uint32 magic 0x54524941
 *   4       4     uint32 version 1
 *   8       24    int32 n_layers, n_q_heads, n_kv_heads, head_dim, pairing,
 *                 offset_log2_max
 *   32      8     float64 rope_theta
 *   40      4     uint32 flags: bit 0 per-layer budget scales present, bit 1
 *                 band mask present
 *   44      4     uint32 0
 *   48            float32 q_mean_re [n_layers][n_q_heads][head_dim/2], then
 *                 q_mean_im and q_abs_mean (the same shape), then the
 *                 per-layer budget scales [n_layers] and the band mask
 *                 [head_dim/2] when their flags are set.
 *
 * tria_write_stats_file - write the statistics (host arrays, layouts as in
 *   tria_load_stats; scales and mask nullable) to `path` (created or
 *   truncated).  Errors: INVALID_ARG (null pointer, bad desc), IO.
 * tria_read_stats_file - read the header into *desc_out and the flags into
 *   *has_scales / *has_mask (each nullable), and, for every non-null array
 *   pointer, the array (host memory the caller sized from *desc_out; asking
 *   for scales or mask the file does not hold is INVALID_ARG).  Calling it
 *   first with every array NULL gives the sizes.  Errors: INVALID_ARG, IO
 *   (missing, short or foreign file), UNSUPPORTED (another version).
 * Both are host-only: they make no CUDA call.
 */
tria_status tria_write_stats_file(const char *path, const tria_model_desc *desc,
                                  const float *q_mean_re, const float *q_mean_im,
                                  const float *q_abs_mean, const float *layer_budget_scales,
                                  const float *band_mask);
tria_status tria_read_stats_file(const char *path, tria_model_desc *desc_out, int *has_scales,
                                 int *has_mask, float *q_mean_re, float *q_mean_im,
                                 float *q_abs_mean, float *layer_budget_scales,
                                 float *band_mask);

/* Free a stats object (synchronises the device first).  NULL is allowed. */
tria_status tria_free_stats(tria_stats *stats);

/* Copy of the model description a stats object was built with. */
tria_status tria_stats_desc(const tria_stats *stats, tria_model_desc *desc_out);

/*
 * tria_layer_budgets - the budget B_l of every layer of the model under these
 * parameters (formula at tria_params) and the kept_idx row length B_max.
 *   budgets : optional host int [n_layers] (NULL: not written)
 *   row_len : optional host int, B_max = max_l B_l
 * Errors: INVALID_ARG (the same parameter checks as the pass entry points).
 */
tria_status tria_layer_budgets(const tria_stats *stats, const tria_cache_view *cache,
                               const tria_params *params, int *budgets, int *row_len);

/*
 * tria_workspace_size - device workspace bytes that tria_score, tria_select
 * and tria_compress_pass need for this cache view, these parameters and the
 * layer range [layer0, layer1).  The workspace is scratch: no state is kept
 * between calls, and concurrent calls need separate workspaces.  Its base
 * must be 256-byte aligned (cudaMalloc's are); the entry points that take it
 * return TRIA_ERR_WORKSPACE otherwise.
 * Errors: INVALID_ARG.
 */
tria_status tria_workspace_size(const tria_stats *stats, const tria_cache_view *cache,
                                const tria_params *params, int layer0, int layer1,
                                size_t *bytes);

/*
 * tria_score - averaged scores and the aggregated (normalize-then-max) score
 * of every candidate slot of layers [layer0, layer1).
 *
 * Candidates of a unit with N cached rows are slots [sinks, N - window);
 * C = N - window - sinks of them.  Outputs (device, fp32):
 *   agg_out    [n_seq][layer1 - layer0][n_kv_heads][C_max]:
 *              agg[c] = max_g (S~_g[c] - mean_g) / (std_g + 1e-6), mean and
 *              population std of head g over the unit's C candidates;
 *   scores_out optional [n_seq][layer1 - layer0][n_kv_heads][C_max][G]:
 *              S~_g of candidate c for the G query heads of the KV head.
 * Entries c >= C, and units that are not compressed (N - B_l < max(interval,
 * 1)), are not written.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
tria_status tria_score(const tria_stats *stats, const tria_cache_view *cache,
                       const tria_params *params, int layer0, int layer1,
                       float *agg_out, float *scores_out,
                       void *workspace, size_t workspace_bytes, tria_stream_t stream);

/*
 * tria_select - kept slots of every unit of layers [layer0, layer1) from
 * agg (layout of tria_score's agg_out).
 *   kept_idx (device int32 [n_seq][layer1 - layer0][n_kv_heads][B_max]):
 *   ascending slots: 0 .. sinks-1, then the top K = B_l - window - sinks
 *   candidates by agg (ties: lower slot), then N-window .. N-1, then -1 up to
 *   B_max.  A unit that is not compressed gets j at entry j < min(N, B_max)
 *   and -1 after it (nothing moves).
 * Errors: INVALID_ARG, WORKSPACE, CUDA.
 */
tria_status tria_select(const tria_stats *stats, const tria_cache_view *cache,
                        const tria_params *params, const float *agg, int layer0,
                        int layer1, int32_t *kept_idx, void *workspace,
                        size_t workspace_bytes, tria_stream_t stream);

/*
 * tria_compact - in-place gather of the kept K and V rows (and positions, if
 * the view has them) of layers [layer0, layer1): row j of each unit becomes
 * the old row kept_idx[j] (kept_idx as tria_select writes it; -1 entries and
 * entries equal to j move nothing).  kept_idx must be strictly ascending
 * with kept_idx[j] >= j (tria_select guarantees it); rows are byte-copied.
 * Without layer_seq_lens: when layer1 == n_layers, seq_lens[s] becomes B
 * for every compressed sequence and, for the paged layout, the blocks of each
 * sequence past ceil(B / block_size) that held rows are listed in freed_blocks
 * (device int32 [n_seq][max_blocks_per_seq], nullable) with their count in
 * n_freed (device int32 [n_seq], nullable); the block table itself is not
 * modified.  With layer_seq_lens: the length of every compressed (sequence,
 * layer) of [layer0, layer1) becomes B_l; blocks are shared by the layers, so
 * a call over every layer lists the blocks past ceil(max_l new N / block_size)
 * up to ceil(max_l old N / block_size), and a call over part of the layers
 * frees none (n_freed[s] = 0).
 * Errors: INVALID_ARG, CUDA.
 */
tria_status tria_compact(const tria_stats *stats, const tria_cache_view *cache,
                         const tria_params *params, const int32_t *kept_idx,
                         int layer0, int layer1, int32_t *freed_blocks,
                         int32_t *n_freed, tria_stream_t stream);

/*
 * tria_compress_pass - the whole pass over every layer: score, select and
 * compact, with scores and agg kept in the workspace.  kept_idx: optional
 * device [n_seq][n_layers][n_kv_heads][B_max] copy of the kept slots (NULL:
 * kept in the workspace only).  freed_blocks / n_freed as in tria_compact.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 */
tria_status tria_compress_pass(const tria_stats *stats, const tria_cache_view *cache,
                               const tria_params *params, int32_t *kept_idx,
                               int32_t *freed_blocks, int32_t *n_freed,
                               void *workspace, size_t workspace_bytes,
                               tria_stream_t stream);

/*
 * tria_compress_pass_static - tria_compress_pass without a workspace
 * argument: the scratch is a fixed device array inside this library.  The
 * paper has no counterpart of this call; it serves callers that cannot give
 * the library a workspace allocation, such as a serving engine that reserves
 * all free device memory for its KV-cache block pool at start-up (a later
 * cudaMalloc would fail or eat into the pool), or a decode loop that must not
 * stall other streams (cudaMalloc and cudaFree may synchronise the device).
 * The call allocates nothing: no cudaMalloc, cudaFree or allocating library
 * routine.  On `stream` it enqueues a memset of the scratch header, the
 * pass's kernels and, with device_status, one device-to-device copy.
 *
 * Scratch: TRIA_STATIC_SCRATCH_BYTES (32 MiB, 256-byte aligned) of device
 * memory per device, held for as long as the library is loaded.  The first
 * call made in a given CUDA context (per device; the context that follows a
 * cudaDeviceReset counts as a new one) looks up that context's address of
 * the array (cudaGetSymbolAddress, which may load the library's device code
 * on that device) and keeps it, keyed by the context's id; make that first
 * call on each device, and again after a reset, before any stream capture
 * begins.  The current device's array is used: `stream` must belong to the
 * current device.
 * Limit: the pass over all layers must need at most TRIA_STATIC_SCRATCH_BYTES
 * of workspace (tria_workspace_size with layers [0, n_layers)); a larger one
 * returns TRIA_ERR_WORKSPACE with nothing enqueued.  32 MiB holds, for
 * example, one 32K-token sequence of 8 KV heads x 8 query heads per KV head
 * for up to 3 layers.
 * Zeroing: each call clears the scratch header (work counter and status
 * flags) on `stream` before its kernels; the kernels rewrite every other
 * scratch region before reading it, so nothing carries over between calls.
 * Races: every call on a device uses the same array.  Calls ordered on one
 * stream are safe; calls that may overlap on the device (other streams or
 * host threads with no ordering between them) race on the scratch and give
 * undefined results.
 * device_status: optional device int32; receives this call's status flags
 * (bits as in tria_read_device_status) after the compaction.
 * kept_idx, freed_blocks, n_freed, results and errors as in
 * tria_compress_pass; also UNSUPPORTED when the current device ordinal is 64
 * or more.
 */
#define TRIA_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)

tria_status tria_compress_pass_static(const tria_stats *stats, const tria_cache_view *cache,
                                      const tria_params *params, int32_t *kept_idx,
                                      int32_t *freed_blocks, int32_t *n_freed,
                                      int32_t *device_status, tria_stream_t stream);

/*
 * tria_calib_accumulate - the calibration reduction that produces the query
 * statistics tria_load_stats takes (GitHub issue #10 of the llama.cpp
 * TurboQuant HIP fork, "Working calibration tool": q_mean_real[f] =
 * E[Re q_f], q_mean_imag[f] = E[Im q_f], q_abs_mean[f] = E[|q_f|] over the
 * post-norm, pre-RoPE queries, with the model's complex pairing; academ.us
 * article 2607.13051 sec. 2: E[q_f] is the average of band-f queries over a
 * calibration set).  One layer per call; batches of one layer add up.
 *   q    device bf16 pre-RoPE queries of one layer, element (t, h, i) at
 *        q[t * stride_token + h * stride_head + i], i < 128 contiguous;
 *        8-byte aligned, strides multiples of 4 elements;
 *   acc  device fp64 [n_q_heads][64][3] = (sum Re q_f, sum Im q_f,
 *        sum |q_f|) per (head, band); the caller zeroes it before the first
 *        batch and keeps it between batches.  The sums are added with fp64
 *        atomics (the order of additions, so the last bits, may vary).
 * Reads desc->n_q_heads, head_dim (128) and pairing.  Stream-ordered, no
 * allocation.  Errors: INVALID_ARG, UNSUPPORTED (head_dim), CUDA.
 */
tria_status tria_calib_accumulate(const tria_model_desc *desc, const void *q, int64_t n_tokens,
                                  int64_t stride_token, int64_t stride_head, double *acc,
                                  tria_stream_t stream);

/*
 * tria_calib_finalize - statistics from the sums of tria_calib_accumulate
 * over n_tokens tokens in total: device fp32 [n_q_heads][64] arrays
 * q_mean_re = sum Re / n_tokens, q_mean_im = sum Im / n_tokens,
 * q_abs_mean = sum |q_f| / n_tokens (one layer's slice of the host arrays
 * tria_load_stats takes).  Errors: INVALID_ARG (n_tokens <= 0), CUDA.
 */
tria_status tria_calib_finalize(const tria_model_desc *desc, const double *acc, int64_t n_tokens,
                                float *q_mean_re, float *q_mean_im, float *q_abs_mean,
                                tria_stream_t stream);

/*
 * tria_read_device_status - errors the kernels found during the calls that
 * used this workspace, then clears them.  Bit 0: a seq_lens entry outside
 * [0, max_seq_len] (such a unit is skipped and its kept row is all -1).
 * Bit 1: a wait of the scoring kernel ran out (tria_params.wait_limit_ns);
 * the kernel stopped early and the call's scores, kept rows and compaction
 * are undefined.  Synchronises `stream`.  *flags_out = 0 means none.
 * The flags start undefined in a fresh workspace: read (and so clear) them
 * once before the first call.
 */
tria_status tria_read_device_status(void *workspace, tria_stream_t stream,
                                    int32_t *flags_out);

/*
 * tria_set_pass_events - kernel timing hook for tria_compress_pass (tracing).
 * events: NULL to disable, or a host array of 5 cudaEvent_t created by the
 * caller; the next tria_compress_pass calls made from this host thread record
 * events[0] before the coefficient kernel, events[1] before the scoring
 * kernel, events[2] before the normalize-then-max / selection kernel,
 * events[3] before the compaction kernel and events[4] after it, on the
 * pass's stream.  The array is copied; the events stay owned by the caller.
 */
tria_status tria_set_pass_events(void *const *events);

/*
 * tria_decode_attention - the attention of one decode step over the cached
 * rows of one layer: the kernel that runs for every generated token, on the
 * cache that the pass pruned (academ.us article 2607.13051, sec. 8).  For
 * sequence s, query head qh and its KV head h = qh / G, over the rows
 * j < N(s, layer) of unit (s, layer, h):
 *   z_j  = scale * (q . k_j)
 *   out  = sum_j softmax(z)_j v_j,      lse = log sum_j exp(z_j)
 * The cached keys carry their rotation already (RoPE at the key's position),
 * so a row keeps its logit when compaction moves it: the retained rows
 * reproduce the full-cache logits of the keys they hold (Eq. 3: the phase
 * depends only on the rotations already applied to q and k).
 *   q       device bf16 [n_seq][n_q_heads][128], the post-RoPE decode query
 *           (16-byte aligned, contiguous)
 *   scale   softmax scale (1/sqrt(128) for standard attention); finite
 *   out     device fp32 [n_seq][n_q_heads][128]
 *   lse     optional device fp32 [n_seq][n_q_heads] (natural log; -inf when
 *           N = 0, with out = 0)
 *   logits  optional device fp32 [n_seq][n_q_heads][max_seq_len]: z_j at
 *           j < N (entries j >= N are not written)
 * N comes from layer_seq_lens when the view has it, else seq_lens; a length
 * outside [0, max_seq_len] sets status bit 0 and is read as 0.  Paged block
 * ids outside [0, num_blocks) read as zero rows.  The cache is only read.
 * Workspace: tria_decode_workspace_size bytes (256-byte aligned), all zero
 * before its first use (it holds per-unit arrival counts that every call
 * leaves at zero); its first 256 bytes hold the status flags read by
 * tria_read_device_status.  Calls that may overlap need separate workspaces.
 * Errors: INVALID_ARG, UNSUPPORTED (head_dim != 128), WORKSPACE, CUDA.
 */
tria_status tria_decode_workspace_size(const tria_stats *stats, const tria_cache_view *cache,
                                       size_t *bytes);
tria_status tria_decode_attention(const tria_stats *stats, const tria_cache_view *cache,
                                  int layer, const void *q, float scale, float *out,
                                  float *lse, float *logits, void *workspace,
                                  size_t workspace_bytes, tria_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TRIA_H */
