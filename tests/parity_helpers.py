"""Comparison of the CUDA pass with the fp64 oracle.

Tolerances (a score error is meaningless relative to a score that crosses
zero, so it is measured against the sum of the absolute sizes of the score's
terms):
* scores:  |S_gpu - S_oracle| <= 1e-4 * L1_k, L1_k = sum_f (|mu'_f| + w_f) |k_f|;
* agg:     |agg_gpu - agg_oracle| <= tau(k) = max over heads of
           1e-4 * (max_k L1_k / std_h) * (2 + |z|) + 1e-6 * (1 + |agg|);
* kept:    the kept set equals the oracle's own selection on the GPU's fp32
           agg bit for bit (same precision decides); against the fp64 oracle
           it agrees outside the tie band |agg_oracle - a_K| <= 2 tau, a_K the
           K-th largest oracle agg; |kept| = budget;
* compacted rows: byte-equal to the oracle's compaction of the GPU's kept set.
"""
from __future__ import annotations

import numpy as np

from oracle import tria_oracle as O

SCORE_RTOL = 1e-4


def unit_oracle(w, s: int, layer: int, h: int, k_bits=None, positions=None, form="folded",
                budget=None, interval=0, n=None, band_mask=None):
    """Oracle of one unit of a synth.Workload (reads K rows back unless given).
    budget: the unit's budget (default: the configuration's); n: its length
    (default: the sequence's)."""
    cfg = w.cfg
    B = cfg.budget if budget is None else int(budget)
    if k_bits is None:
        k_bits = w.unit_rows("k", s, layer, h, n)
    if positions is None:
        positions = w.unit_positions(s, layer, h, len(k_bits))
    k = O.bf16_bits_to_f64(k_bits)
    G = cfg.group
    re, im, am = w.stats
    qc = (re[layer, h * G:(h + 1) * G].astype(np.float64)
          + 1j * im[layer, h * G:(h + 1) * G].astype(np.float64))
    qa = am[layer, h * G:(h + 1) * G].astype(np.float64)
    omega = O.band_frequencies(cfg.head_dim, cfg.theta)
    p_q = int(w.query_pos[s].item())
    mask = None if band_mask is None else np.asarray(band_mask, np.float32).astype(np.float64)
    res = O.compress_unit(k, positions, p_q, qc, qa, omega, cfg.pairing, B, cfg.window,
                          cfg.sinks, cfg.offset_log2_max, band_mask=mask, form=form,
                          interval=interval)
    N = len(k)
    res["B"] = B
    res["compressed"] = O.is_compressed(N, B, interval)
    if res["scores"] is not None:
        l1 = O.score_l1_scale(k, positions, qc, qa, omega, cfg.pairing, cfg.offset_log2_max,
                              band_mask=mask, form="max" if form == "max" else "folded")
        res["l1"] = l1[:, cfg.sinks:N - cfg.window]
    res["N"] = N
    return res


def check_direct_sample(gpu_scores: np.ndarray, w, s: int, layer: int, h: int, k_bits, positions,
                        ora: dict, frac: float = 0.01, seed: int = 0, where=""):
    """The GPU scores of a seeded sample (frac) of the unit's candidates
    against the direct 17-offset form (Eq. 4 evaluated offset by offset),
    within the same 1e-4 * L1 bound as the folded comparison."""
    cfg = w.cfg
    C = gpu_scores.shape[0]
    n = max(1, int(round(frac * C)))
    cand = np.sort(np.random.default_rng(seed + 7919 * (layer * 64 + h)).choice(C, n, replace=False))
    slots = cand + cfg.sinks
    k = O.bf16_bits_to_f64(np.asarray(k_bits)[slots])
    G = cfg.group
    re, im, am = w.stats
    qc = (re[layer, h * G:(h + 1) * G].astype(np.float64)
          + 1j * im[layer, h * G:(h + 1) * G].astype(np.float64))
    qa = am[layer, h * G:(h + 1) * G].astype(np.float64)
    omega = O.band_frequencies(cfg.head_dim, cfg.theta)
    p_q = int(w.query_pos[s].item())
    direct = O.unit_scores(k, np.asarray(positions)[slots], p_q, qc, qa, omega, cfg.pairing,
                           cfg.offset_log2_max, form="direct")
    err = np.abs(np.asarray(gpu_scores, dtype=np.float64)[cand].T - direct)
    bound = SCORE_RTOL * ora["l1"][:, cand]
    assert np.all(err <= bound), (f"{where}: {np.sum(err > bound)} sampled scores off the direct "
                                  f"form; worst ratio {np.max(err / bound):.3g}")
    return n


def check_scores(gpu_scores: np.ndarray, ora: dict, where=""):
    """gpu_scores: [C, G] fp32."""
    S = np.asarray(gpu_scores, dtype=np.float64).T
    err = np.abs(S - ora["scores"])
    bound = SCORE_RTOL * ora["l1"]
    bad = err > bound
    assert not bad.any(), (f"{where}: {bad.sum()} scores outside 1e-4*L1; worst ratio "
                           f"{np.max(err / bound):.3g}")
    return float(np.max(err / ora["l1"]))


def agg_tolerance(ora: dict) -> np.ndarray:
    z_abs = np.abs(ora["agg"])
    l1max = ora["l1"].max(axis=1)              # [G]
    per_head = SCORE_RTOL * (l1max / np.maximum(ora["std"], 1e-30))
    return per_head.max() * (2.0 + z_abs) + 1e-6 * (1.0 + z_abs)


def check_agg(gpu_agg: np.ndarray, ora: dict, where=""):
    a = np.asarray(gpu_agg, dtype=np.float64)
    tau = agg_tolerance(ora)
    err = np.abs(a - ora["agg"])
    bad = err > tau
    assert not bad.any(), f"{where}: {bad.sum()} agg outside tolerance; worst {np.max(err / tau):.3g}"
    return tau


def check_kept_same_precision(gpu_kept: np.ndarray, gpu_agg: np.ndarray, N: int, cfg, where="",
                              budget=None):
    """The GPU's kept set equals the oracle's selection applied to the GPU's
    own fp32 agg (the floating point that decides is the same)."""
    B = cfg.budget if budget is None else int(budget)
    ref = O.select_kept(np.asarray(gpu_agg, dtype=np.float32).astype(np.float64), N, B,
                        cfg.window, cfg.sinks)
    got = np.asarray(gpu_kept[: len(ref)])
    assert np.array_equal(got, ref), f"{where}: kept set differs from select(gpu agg)"
    assert np.all(np.asarray(gpu_kept[len(ref):]) == -1)


def check_kept_vs_oracle(gpu_kept: np.ndarray, ora: dict, cfg, where=""):
    """Outside the tie band the kept sets agree; inside it any choice with
    |kept| = budget is valid."""
    N, B, W, S = ora["N"], ora.get("B", cfg.budget), cfg.window, cfg.sinks
    kept = np.asarray(gpu_kept)
    if not ora.get("compressed", N > B):
        n = min(N, len(kept))
        assert np.array_equal(kept[:n], np.arange(n)) and np.all(kept[n:] == -1), where
        return 0
    assert np.all(kept[B:] == -1), f"{where}: entries past the unit's budget"
    kept = kept[:B]
    assert np.all(np.diff(kept) > 0), f"{where}: kept not strictly ascending"
    assert set(range(S)) <= set(kept.tolist()) and set(range(N - W, N)) <= set(kept.tolist())
    K = B - W - S
    if K == 0:
        return 0
    agg = ora["agg"]
    tau = agg_tolerance(ora)
    aK = np.sort(agg)[::-1][K - 1]
    sel = np.zeros(len(agg), dtype=bool)
    cand = kept[(kept >= S) & (kept < N - W)] - S
    sel[cand] = True
    must = agg > aK + 2 * tau
    never = agg < aK - 2 * tau
    assert not np.any(must & ~sel), f"{where}: {np.sum(must & ~sel)} clear winners dropped"
    assert not np.any(never & sel), f"{where}: {np.sum(never & sel)} clear losers kept"
    return int(np.sum(~must & ~never))


def compact_host(rows: np.ndarray, kept: np.ndarray, N: int, budget: int) -> np.ndarray:
    """Oracle compaction of a unit's rows by a kept list (uint16 bits)."""
    out = rows.copy()
    k = np.asarray(kept)
    n = min(N, budget)
    valid = k[:n]
    out[:n] = O.compact_rows(rows, valid)
    return out
