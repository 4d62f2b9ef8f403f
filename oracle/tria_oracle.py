"""fp64 CPU oracle for the TriAttention KV-cache compression pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference leg may use it.  It shares no code, constants or
helpers with the CUDA library under ``key_retention_scoring_b200/``.

Everything is plain numpy in float64 (complex128 for the band phasors).  Each
function follows one statement of the sources, cited by page and
section/equation:

* [P5]  academ.us article 2607.13051 ("a small improvement to one step of
        TriAttention"): sec. 2 Eqs. (1)-(3), sec. 3 Eqs. (4)-(7), sec. 4,
        sec. 7 Eq. (8) and its "Numerical confirmation" paragraph.
* [P3]  ghidav.me, "TriAttention, or: what a rotating query already knows":
        sections "The Intuition", "The Solution", "The Method".
* [P4]  GitHub issue #10 on the llama.cpp TurboQuant HIP fork, "Request:
        publish TriAttention calibration script": the calibration-tool comment
        (statistics fields, RoPE complex pairing, runtime log lines).
* [P1]  triattention project README (shadowgraph.io mirror): budget defaults.

Readings taken where the sources are silent (each is also listed in the
design notes of the repository):

* S_norm = sum_f (E|q_f| - |E[q_f]|) * |k_f|, i.e. (1 - R_f) E|q_f| |k_f| with
  the concentration R_f = |E[q_f]| / E|q_f|.  [P3] "The Method" says the term
  scores a key by its own magnitudes and weighs in proportionally to
  (1 - R_f); [P5] sec. 2 says it does not depend on the distance; the
  calibration statistics of [P4] hold exactly E[q_f] and E|q_f|.
  PARITY UNPINNED beyond this reading: the sources print no S_norm value.
* The current query sits at the position of the newest cached token (p_q);
  the future offsets start at delta = 1 ([P5] Eq. 4).
* GQA: z-normalise each query head over the scored candidates (population
  standard deviation, eps = 1e-6 added to it), then take the max over the
  heads sharing a KV head ([P5] sec. 4 "normalize-then-max").
* Budget B counts every kept row, window W and sinks S included; candidates
  are slots [S, N - W) ([P4] log line n_old = n_kv - window).
* Budget variants ([P4] runtime: a percentage budget and per-layer budget
  scales that default to 1.0; [P5] sec. 8: pruning once per window of beta
  generated tokens): a percentage is of the cache capacity (the rows a
  sequence can hold); layer l keeps B_l = floor(base * scale_l + 1/2) rows;
  a unit is compressed only when N - B_l >= max(beta, 1).
* Exact ties on the aggregated score go to the lower slot; the kept list is in
  ascending slot order; NaN ranks below every number and -0.0 equals +0.0.
* The optional high-frequency band mask multiplies |mu'_f| only ([P5] sec. 7,
  last paragraph).
"""
from __future__ import annotations

import numpy as np

PAIR_NEOX = 0
PAIR_INTERLEAVED = 1
NORM_EPS = 1e-6


# ----------------------------------------------------------------------------
# RoPE bands
# ----------------------------------------------------------------------------
def band_frequencies(head_dim: int, theta: float) -> np.ndarray:
    """omega_f = theta^(-2f/d) for f = 0 .. d/2-1 ([P5] sec. 2, list under Eq. 2)."""
    f = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * f / float(head_dim))


def to_bands(x: np.ndarray, pairing: int) -> np.ndarray:
    """Real head_dim vectors (last axis) -> complex bands (last axis d/2).

    NEOX pairing: band f = x[f] + i*x[f + d/2]; interleaved (NORM) pairing:
    band f = x[2f] + i*x[2f+1] ([P4] calibration-tool comment, "RoPE complex
    pairing matches the model's rope_type")."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    if pairing == PAIR_NEOX:
        re, im = x[..., : d // 2], x[..., d // 2:]
    elif pairing == PAIR_INTERLEAVED:
        re, im = x[..., 0::2], x[..., 1::2]
    else:
        raise ValueError("unknown pairing")
    return re + 1j * im


def from_bands(z: np.ndarray, pairing: int) -> np.ndarray:
    """Inverse of :func:`to_bands`."""
    z = np.asarray(z, dtype=np.complex128)
    F = z.shape[-1]
    out = np.empty(z.shape[:-1] + (2 * F,), dtype=np.float64)
    if pairing == PAIR_NEOX:
        out[..., :F], out[..., F:] = z.real, z.imag
    elif pairing == PAIR_INTERLEAVED:
        out[..., 0::2], out[..., 1::2] = z.real, z.imag
    else:
        raise ValueError("unknown pairing")
    return out


def derotate(k_bands: np.ndarray, positions: np.ndarray, omega: np.ndarray) -> np.ndarray:
    """Pre-RoPE band components of cached (post-RoPE) keys.

    RoPE turns band f of a token at position p by multiplying it with
    e^{i omega_f p} ([P5] sec. 2.0.0.3, fact 3), so the pre-rotation component
    is k_f = ktilde_f * e^{-i omega_f p_k}."""
    p = np.asarray(positions, dtype=np.float64)[..., None]
    return k_bands * np.exp(-1j * omega * p)


# ----------------------------------------------------------------------------
# Trigonometric term, single distance
# ----------------------------------------------------------------------------
def s_trig_polar(q_center: np.ndarray, k_pre: np.ndarray, omega: np.ndarray,
                 delta) -> np.ndarray:
    """[P5] Eq. (2): sum_f |E q_f| |k_f| cos(omega_f Delta + phi_f), with
    phi_f = arg E[q_f] - arg k_f.  q_center: [F]; k_pre: [..., F];
    delta broadcastable to k_pre[..., 0]."""
    mag = np.abs(q_center) * np.abs(k_pre)
    phi = np.angle(q_center) - np.angle(k_pre)
    d = np.asarray(delta, dtype=np.float64)[..., None]
    return np.sum(mag * np.cos(omega * d + phi), axis=-1)


def s_trig_phasor(q_center: np.ndarray, k_pre: np.ndarray, omega: np.ndarray,
                  delta) -> np.ndarray:
    """[P5] Eq. (3): Re sum_f E[q_f] conj(k_f) e^{i omega_f Delta}."""
    d = np.asarray(delta, dtype=np.float64)[..., None]
    return np.real(np.sum(q_center * np.conj(k_pre) * np.exp(1j * omega * d), axis=-1))


# ----------------------------------------------------------------------------
# Future-offset average
# ----------------------------------------------------------------------------
def offset_set(log2_max: int = 16) -> np.ndarray:
    """D = {1, 2, 4, ..., 2^m}; the published method uses m = 16, |D| = 17
    ([P5] Eq. 4)."""
    return np.power(2.0, np.arange(int(log2_max) + 1, dtype=np.float64))


def s_trig_direct_average(q_center: np.ndarray, k_pre: np.ndarray, omega: np.ndarray,
                          delta, offsets: np.ndarray) -> np.ndarray:
    """[P5] Eq. (4) done as written, the way the reference scorer does it:
    materialise a [keys x offsets x bands] table of band cosines of Eq. (2)
    and average it over the offset axis."""
    mag = np.abs(q_center) * np.abs(k_pre)                     # [..., F]
    phi = np.angle(q_center) - np.angle(k_pre)                 # [..., F]
    d = np.asarray(delta, dtype=np.float64)[..., None, None]   # [..., 1, 1]
    ang = omega * (d + offsets[:, None]) + phi[..., None, :]   # [..., |D|, F]
    table = mag[..., None, :] * np.cos(ang)
    return np.mean(np.sum(table, axis=-1), axis=-1)


def s_trig_direct_max(q_center: np.ndarray, k_pre: np.ndarray, omega: np.ndarray,
                      delta, offsets: np.ndarray) -> np.ndarray:
    """The non-default variant named at the end of [P5] sec. 4: the maximum of
    Eq. (2) over the future offsets delta in D instead of their mean.  It is
    not linear in the phasors, so it does not fold (Eqs. 6-7 do not apply);
    it is evaluated offset by offset on the same [keys x offsets x bands]
    table as :func:`s_trig_direct_average`."""
    mag = np.abs(q_center) * np.abs(k_pre)
    phi = np.angle(q_center) - np.angle(k_pre)
    d = np.asarray(delta, dtype=np.float64)[..., None, None]
    ang = omega * (d + offsets[:, None]) + phi[..., None, :]
    table = mag[..., None, :] * np.cos(ang)
    return np.max(np.sum(table, axis=-1), axis=-1)


def offset_weight(omega: np.ndarray, offsets: np.ndarray) -> np.ndarray:
    """W_f = (1/|D|) sum_{delta in D} e^{i omega_f delta} ([P5] Eq. 6)."""
    return np.mean(np.exp(1j * np.outer(offsets, omega)), axis=0)


def folded_center(q_center: np.ndarray, W: np.ndarray,
                  band_mask: np.ndarray | None = None) -> np.ndarray:
    """mu'_f = E[q_f] W_f ([P5] Eq. 7).  The optional per-band high-frequency
    mask rescales |mu'_f| ([P5] sec. 7, last paragraph)."""
    mu = q_center * W
    if band_mask is not None:
        mu = mu * np.asarray(band_mask, dtype=np.float64)
    return mu


def s_trig_folded(mu_folded: np.ndarray, k_pre: np.ndarray, omega: np.ndarray,
                  delta) -> np.ndarray:
    """[P5] Eq. (7): sum_f |mu'_f| |k_f| cos(omega_f Delta + phi'_f) with
    phi'_f = arg mu'_f - arg k_f.  (Eq. 2 evaluated once, on mu'.)"""
    return s_trig_polar(mu_folded, k_pre, omega, delta)


def s_trig_real_map(q_center: np.ndarray, k_pre: np.ndarray, omega: np.ndarray,
                    delta, W: np.ndarray) -> np.ndarray:
    """[P5] sec. 7, Eq. (8): real coefficients a_f = |Eq||k| cos(phi),
    b_f = -|Eq||k| sin(phi), mapped by [[A, B], [-B, A]] with A = Re W,
    B = Im W, then sum_f a'_f cos(omega_f Delta) + b'_f sin(omega_f Delta)."""
    mag = np.abs(q_center) * np.abs(k_pre)
    phi = np.angle(q_center) - np.angle(k_pre)
    a = mag * np.cos(phi)
    b = -mag * np.sin(phi)
    A, B = W.real, W.imag
    a2 = A * a + B * b
    b2 = -B * a + A * b
    d = np.asarray(delta, dtype=np.float64)[..., None]
    return np.sum(a2 * np.cos(omega * d) + b2 * np.sin(omega * d), axis=-1)


# ----------------------------------------------------------------------------
# Norm term and total score
# ----------------------------------------------------------------------------
def concentration(q_center: np.ndarray, q_abs_mean: np.ndarray) -> np.ndarray:
    """R_f = |E[q_f]| / E|q_f| in [0, 1] (mean resultant length, [P3] "The
    Intuition"), from the two statistics the calibration stores ([P4])."""
    return np.abs(q_center) / np.asarray(q_abs_mean, dtype=np.float64)


def s_norm(q_center: np.ndarray, q_abs_mean: np.ndarray, k_pre: np.ndarray) -> np.ndarray:
    """Distance-independent norm term (reading, see module docstring):
    sum_f (1 - R_f) E|q_f| |k_f| = sum_f (E|q_f| - |E q_f|) |k_f|."""
    w = np.asarray(q_abs_mean, dtype=np.float64) - np.abs(q_center)
    return np.sum(w * np.abs(k_pre), axis=-1)


def unit_scores(k_post: np.ndarray, positions: np.ndarray, p_q: int,
                q_center: np.ndarray, q_abs_mean: np.ndarray, omega: np.ndarray,
                pairing: int, log2_max: int = 16, band_mask=None,
                form: str = "folded") -> np.ndarray:
    """Averaged score S~(k) = S~_trig(k) + S_norm(k) ([P5] Eq. 1 with Eq. 4,
    written as Eq. 7) of every cached key of one (layer, KV head), for each
    of the G query heads sharing it.

    k_post: [N, d] post-RoPE keys; positions: [N] token positions p_k;
    q_center: [G, F] complex E[q_f]; q_abs_mean: [G, F] E|q_f|.
    form: "folded" (Eq. 7), "direct" (Eq. 4, the 17-offset table) or "max"
    (the maximum over the offsets instead of the mean, see
    :func:`s_trig_direct_max`).
    Returns [G, N] float64."""
    kb = to_bands(k_post, pairing)
    k_pre = derotate(kb, positions, omega)
    delta = float(p_q) - np.asarray(positions, dtype=np.float64)
    D = offset_set(log2_max)
    W = offset_weight(omega, D)
    G = q_center.shape[0]
    out = np.empty((G, k_pre.shape[0]), dtype=np.float64)
    for h in range(G):
        if form == "folded":
            trig = s_trig_folded(folded_center(q_center[h], W, band_mask), k_pre, omega, delta)
        elif form in ("direct", "max"):
            qc = q_center[h] if band_mask is None else q_center[h] * np.asarray(band_mask)
            fn = s_trig_direct_average if form == "direct" else s_trig_direct_max
            trig = np.empty(k_pre.shape[0])
            step = 4096
            for s in range(0, k_pre.shape[0], step):
                trig[s:s + step] = fn(qc, k_pre[s:s + step], omega, delta[s:s + step], D)
        else:
            raise ValueError(form)
        out[h] = trig + s_norm(q_center[h], q_abs_mean[h], k_pre)
    return out


# ----------------------------------------------------------------------------
# GQA aggregation, selection, compaction
# ----------------------------------------------------------------------------
def gqa_znorm_max(scores: np.ndarray, eps: float = NORM_EPS):
    """Grouped-query normalize-then-max ([P5] sec. 4): z-normalise each query
    head over the candidates (population mean and standard deviation), then
    take the max over the heads of the group.  scores: [G, C].
    Returns (agg [C], mean [G], std [G])."""
    S = np.asarray(scores, dtype=np.float64)
    m = S.mean(axis=1)
    sd = np.sqrt(((S - m[:, None]) ** 2).mean(axis=1))
    z = (S - m[:, None]) / (sd[:, None] + eps)
    return z.max(axis=0), m, sd


def rank_order(agg: np.ndarray) -> np.ndarray:
    """Candidate indices by descending score; equal scores keep ascending
    index order; NaN below every number (-inf included); -0.0 == +0.0.
    Sorted by (is NaN, -score, index)."""
    a = np.asarray(agg, dtype=np.float64)
    nan = np.isnan(a)
    return np.lexsort((np.arange(a.size), np.where(nan, 0.0, -a), nan))


def select_kept(agg: np.ndarray, n_tokens: int, budget: int, window: int,
                sinks: int) -> np.ndarray:
    """Top-K retention ([P3] "The Method": sort, keep the top B, drop the
    rest), always keeping the first `sinks` slots and the last `window` slots
    ([P4] runtime log: window 256, sink 0, n_old = n_kv - window).

    agg: [C] scores of candidate slots sinks .. n_tokens-window-1.
    Returns the kept slots in ascending order, length min(n_tokens, budget)."""
    N, B, W, S = int(n_tokens), int(budget), int(window), int(sinks)
    if N <= B:
        return np.arange(N, dtype=np.int64)
    C = N - W - S
    K = B - W - S
    assert len(agg) == C and K >= 0
    top = rank_order(agg)[:K] + S
    kept = np.concatenate([np.arange(S), np.sort(top), np.arange(N - W, N)])
    return kept.astype(np.int64)


def compact_rows(rows: np.ndarray, kept: np.ndarray) -> np.ndarray:
    """Per-layer compaction: row j of the result is row kept[j] of the input
    (the kept rows, in ascending slot order, moved to the front)."""
    return np.asarray(rows)[np.asarray(kept)]


def layer_budgets(n_layers: int, budget: int, capacity: int, budget_pct: float = 0.0,
                  scales=None) -> np.ndarray:
    """Budget of every layer.  [P4]'s runtime takes the budget as a
    percentage ("budget=50%") and per-layer budget scales that default to 1.0
    (uniform); [P1] gives absolute budgets (2048, 12000).  Readings: the
    percentage is of the cache capacity `capacity` (the rows one sequence can
    hold), base = floor(pct * capacity / 100); layer l keeps
    B_l = floor(base * scale_l + 1/2).  pct and the scales enter as the fp32
    values a caller passes."""
    pct = float(np.float32(budget_pct))
    base = np.floor(pct * float(capacity) / 100.0) if pct > 0.0 else float(budget)
    out = np.empty(int(n_layers), dtype=np.int64)
    for l in range(int(n_layers)):
        sc = 1.0 if scales is None else float(np.float32(scales[l]))
        out[l] = int(np.floor(base * sc + 0.5))
    return out


def is_compressed(n_tokens: int, budget: int, interval: int = 0) -> bool:
    """Pruning runs once per window of beta generated tokens ([P5] sec. 8,
    beta = 128; [P4] runtime log, interval 128): a unit is compressed once it
    holds at least max(beta, 1) rows more than its budget, else left as is."""
    return int(n_tokens) - int(budget) >= max(int(interval), 1)


def pass_lengths(lens: np.ndarray, budgets: np.ndarray, interval: int = 0) -> np.ndarray:
    """Lengths [n_seq][n_layers] after one pass: a compressed (sequence,
    layer) keeps its budget's rows, every other one its length."""
    lens = np.asarray(lens, dtype=np.int64)
    out = lens.copy()
    for s in range(lens.shape[0]):
        for l in range(lens.shape[1]):
            if is_compressed(lens[s, l], budgets[l], interval):
                out[s, l] = budgets[l]
    return out


def freed_block_range(old_lens: np.ndarray, new_lens: np.ndarray, block_size: int):
    """Paged cache whose blocks hold the rows of every layer: after a pass
    over all layers of a sequence, the blocks [first, end) are no longer used
    by any layer: first = ceil(max_l new / bs), end = ceil(max_l old / bs)."""
    bs = int(block_size)
    first = -(-int(np.max(new_lens)) // bs)
    end = -(-int(np.max(old_lens)) // bs)
    return first, max(first, end)


def compress_unit(k_post, positions, p_q, q_center, q_abs_mean, omega, pairing,
                  budget, window, sinks, log2_max=16, band_mask=None, form="folded",
                  interval=0):
    """One (sequence, layer, KV head) through the whole pass: scores of the
    candidate slots, normalize-then-max, selection.  Returns a dict with
    'scores' [G, C], 'agg' [C], 'mean', 'std', 'kept' [B] (all N rows when the
    unit is not compressed)."""
    N = k_post.shape[0]
    if not is_compressed(N, budget, interval):
        return {"scores": None, "agg": None, "mean": None, "std": None,
                "kept": np.arange(N, dtype=np.int64)}
    S_all = unit_scores(k_post, positions, p_q, q_center, q_abs_mean, omega, pairing,
                        log2_max, band_mask, form)
    cand = slice(sinks, N - window)
    sc = S_all[:, cand]
    agg, m, sd = gqa_znorm_max(sc)
    kept = select_kept(agg, N, budget, window, sinks)
    return {"scores": sc, "agg": agg, "mean": m, "std": sd, "kept": kept}


# ----------------------------------------------------------------------------
# Decode attention over the (pruned) cache
# ----------------------------------------------------------------------------
def decode_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Attention of one decode query per head over a unit's cached rows, the
    kernel that runs for every generated token on the pruned cache ([P5]
    sec. 8).  q: [G, d] post-RoPE queries; k, v: [N, d] cached rows (keys
    carry their RoPE rotation, so no position enters here: [P5] Eq. 3).
    Returns (out [G, d], lse [G], logits [G, N]) with logits = scale q.k_j,
    out = sum_j softmax(logits)_j v_j, lse = log sum_j exp(logits_j); N = 0
    gives out = 0 and lse = -inf."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    z = float(scale) * (q @ k.T)                       # [G, N]
    if z.shape[1] == 0:
        return np.zeros((q.shape[0], v.shape[1])), np.full(q.shape[0], -np.inf), z
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    tot = e.sum(axis=1, keepdims=True)
    out = (e / tot) @ v
    lse = (m + np.log(tot))[:, 0]
    return out, lse, z


def attention_recall(logits: np.ndarray, kept) -> np.ndarray:
    """Share of each head's full-cache attention mass that falls on the kept
    rows: sum_{j in kept} softmax(logits)_j, per head ([G, N] logits)."""
    z = np.asarray(logits, dtype=np.float64)
    e = np.exp(z - z.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    return p[:, np.asarray(kept, dtype=np.int64)].sum(axis=1)


# ----------------------------------------------------------------------------
# Helpers used by the parity tests
# ----------------------------------------------------------------------------
def score_l1_scale(k_post, positions, q_center, q_abs_mean, omega, pairing,
                   log2_max=16, band_mask=None, form="folded") -> np.ndarray:
    """Sum of the absolute sizes of the terms of the score of every key,
    sum_f (|mu'_f| + E|q_f| - |E q_f|) |k_f|, per head: [G, N] (with
    form="max", |E q_f| (masked) in place of |mu'_f|: the terms of one
    offset).  Used to scale the score tolerance (a plain relative error is
    meaningless where the score crosses zero)."""
    kb = to_bands(k_post, pairing)
    k_abs = np.abs(kb)
    W = offset_weight(omega, offset_set(log2_max))
    out = []
    for h in range(q_center.shape[0]):
        if form == "max":
            mu = q_center[h] if band_mask is None else q_center[h] * np.asarray(band_mask)
        else:
            mu = folded_center(q_center[h], W, band_mask)
        w = np.asarray(q_abs_mean[h]) - np.abs(q_center[h])
        out.append(np.sum((np.abs(mu) + w) * k_abs, axis=-1))
    return np.stack(out)


def calibration_stats(q_pre: np.ndarray, pairing: int):
    """Query statistics of the calibration step, from pre-RoPE queries
    q_pre [tokens..., Hq, d] (every axis before the head axis is averaged
    over): per (head, band) E[Re q_f], E[Im q_f] and E|q_f| ([P4]
    calibration-tool comment: q_mean_real, q_mean_imag and q_abs_mean over
    the post-norm, pre-RoPE queries, with the model's complex pairing; [P5]
    sec. 2: E[q_f] is the average of band-f queries over a calibration set).
    Returns three [Hq, d/2] float64 arrays."""
    z = to_bands(q_pre, pairing)
    z = z.reshape((-1,) + z.shape[-2:])
    return z.real.mean(axis=0), z.imag.mean(axis=0), np.abs(z).mean(axis=0)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 numbers given as their uint16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
