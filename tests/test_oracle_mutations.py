"""Planted mistakes in the oracle must each trip at least one pin.

Every mutation below replaces one oracle function (on the CPU, for the
duration of one test) with a plausible wrong version: a dropped term, a
flipped sign, a wrong index or pairing, a transposed operand.  The pins of
``oracle_pins.py`` are then run; the test passes only if at least one of them
fails.  This is the evidence that the pins constrain the oracle rather than
restate it.
"""
import numpy as np
import pytest

from oracle import tria_oracle as O
from tests import oracle_pins as P


def _swap_pairing(x, pairing):
    return _orig["to_bands"](x, 1 - pairing)


def _derotate_wrong_sign(kb, positions, omega):
    p = np.asarray(positions, dtype=np.float64)[..., None]
    return kb * np.exp(+1j * omega * p)


def _omega_missing_two(head_dim, theta):
    f = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(theta), -f / float(head_dim))


def _omega_off_by_one(head_dim, theta):
    f = np.arange(1, head_dim // 2 + 1, dtype=np.float64)
    return np.power(float(theta), -2.0 * f / float(head_dim))


def _offsets_from_zero(log2_max=16):
    return np.concatenate([[0.0], np.power(2.0, np.arange(int(log2_max), dtype=np.float64))])


def _offsets_one_short(log2_max=16):
    return np.power(2.0, np.arange(int(log2_max), dtype=np.float64))


def _weight_conj(omega, offsets):
    return np.conj(_orig["offset_weight"](omega, offsets))


def _weight_sum_not_mean(omega, offsets):
    return np.sum(np.exp(1j * np.outer(offsets, omega)), axis=0)


def _folded_divides(q_center, W, band_mask=None):
    return q_center / W


def _polar_phase_flipped(q_center, k_pre, omega, delta):
    mag = np.abs(q_center) * np.abs(k_pre)
    phi = np.angle(k_pre) - np.angle(q_center)
    d = np.asarray(delta, dtype=np.float64)[..., None]
    return np.sum(mag * np.cos(omega * d + phi), axis=-1)


def _polar_sin(q_center, k_pre, omega, delta):
    mag = np.abs(q_center) * np.abs(k_pre)
    phi = np.angle(q_center) - np.angle(k_pre)
    d = np.asarray(delta, dtype=np.float64)[..., None]
    return np.sum(mag * np.sin(omega * d + phi), axis=-1)


def _phasor_no_conj(q_center, k_pre, omega, delta):
    d = np.asarray(delta, dtype=np.float64)[..., None]
    return np.real(np.sum(q_center * k_pre * np.exp(1j * omega * d), axis=-1))


def _realmap_b_sign(q_center, k_pre, omega, delta, W):
    return _orig["s_trig_real_map"](q_center, k_pre, omega, delta, np.conj(W))


def _norm_dropped(q_center, q_abs_mean, k_pre):
    return np.zeros(k_pre.shape[:-1])


def _norm_uses_abs_mean_only(q_center, q_abs_mean, k_pre):
    return np.sum(np.asarray(q_abs_mean) * np.abs(k_pre), axis=-1)


def _norm_uses_r_not_one_minus_r(q_center, q_abs_mean, k_pre):
    return np.sum(np.abs(q_center) * np.abs(k_pre), axis=-1)


def _znorm_sample_std(scores, eps=O.NORM_EPS):
    S = np.asarray(scores, dtype=np.float64)
    m = S.mean(axis=1)
    sd = S.std(axis=1, ddof=1)
    z = (S - m[:, None]) / (sd[:, None] + eps)
    return z.max(axis=0), m, sd


def _znorm_mean_not_max(scores, eps=O.NORM_EPS):
    agg, m, sd = _orig["gqa_znorm_max"](scores, eps)
    S = np.asarray(scores, dtype=np.float64)
    z = (S - m[:, None]) / (sd[:, None] + eps)
    return z.mean(axis=0), m, sd


def _znorm_max_before_norm(scores, eps=O.NORM_EPS):
    S = np.asarray(scores, dtype=np.float64)
    mx = S.max(axis=0)
    return (mx - mx.mean()) / (mx.std() + eps), S.mean(axis=1), S.std(axis=1)


def _rank_ties_high(agg):
    a = np.asarray(agg, dtype=np.float64)
    n = len(a)
    rev = np.argsort(np.where(np.isnan(a), np.inf, -a)[::-1], kind="stable")
    return (n - 1 - rev)


def _rank_ascending(agg):
    return np.argsort(np.asarray(agg, dtype=np.float64), kind="stable")


def _select_no_window(agg, n_tokens, budget, window, sinks):
    N, B, S = int(n_tokens), int(budget), int(sinks)
    if N <= B:
        return np.arange(N)
    K = B - S
    top = O.rank_order(agg)[:K] + S
    return np.sort(np.concatenate([np.arange(S), top]))


def _compact_off_by_one(rows, kept):
    return np.asarray(rows)[np.minimum(np.asarray(kept) + 1, len(rows) - 1)]


def _calib_abs_of_mean(q_pre, pairing):
    z = O.to_bands(q_pre, pairing).reshape((-1,) + O.to_bands(q_pre, pairing).shape[-2:])
    return z.real.mean(axis=0), z.imag.mean(axis=0), np.abs(z.mean(axis=0))


def _calib_sum_not_mean(q_pre, pairing):
    z = O.to_bands(q_pre, pairing).reshape((-1,) + O.to_bands(q_pre, pairing).shape[-2:])
    return z.real.sum(axis=0), z.imag.sum(axis=0), np.abs(z).sum(axis=0)


def _calib_re_im_swapped(q_pre, pairing):
    re, im, ab = _orig["calibration_stats"](q_pre, pairing)
    return im, re, ab


def _max_is_mean(q_center, k_pre, omega, delta, offsets):
    return _orig["s_trig_direct_average"](q_center, k_pre, omega, delta, offsets)


def _max_is_min(q_center, k_pre, omega, delta, offsets):
    mag = np.abs(q_center) * np.abs(k_pre)
    phi = np.angle(q_center) - np.angle(k_pre)
    d = np.asarray(delta, dtype=np.float64)[..., None, None]
    ang = omega * (d + offsets[:, None]) + phi[..., None, :]
    return np.min(np.sum(mag[..., None, :] * np.cos(ang), axis=-1), axis=-1)


def _budget_pct_of_fraction(n_layers, budget, capacity, budget_pct=0.0, scales=None):
    pct = float(budget_pct)
    if pct > 0:
        return _orig["layer_budgets"](n_layers, budget, capacity, 0.0, scales) * 0 + int(pct * capacity)
    return _orig["layer_budgets"](n_layers, budget, capacity, budget_pct, scales)


def _budget_floor_not_round(n_layers, budget, capacity, budget_pct=0.0, scales=None):
    base = np.floor(float(budget_pct) * capacity / 100.0) if budget_pct > 0 else float(budget)
    sc = np.ones(n_layers) if scales is None else np.asarray(scales, dtype=np.float32)
    return np.floor(base * sc).astype(np.int64)


def _budget_scales_ignored(n_layers, budget, capacity, budget_pct=0.0, scales=None):
    return _orig["layer_budgets"](n_layers, budget, capacity, budget_pct, None)


def _interval_strict(n_tokens, budget, interval=0):
    return int(n_tokens) - int(budget) > max(int(interval), 1)


def _interval_ignored(n_tokens, budget, interval=0):
    return int(n_tokens) > int(budget)


def _freed_from_shortest_layer(old_lens, new_lens, block_size):
    bs = int(block_size)
    return -(-int(np.min(new_lens)) // bs), -(-int(np.max(old_lens)) // bs)


def _attn_no_scale(q, k, v, scale):
    return _orig["decode_attention"](q, k, v, 1.0)


def _attn_keys_as_values(q, k, v, scale):
    return _orig["decode_attention"](q, k, k, scale)


def _attn_softmax_over_heads(q, k, v, scale):
    q = np.asarray(q, dtype=np.float64)
    z = float(scale) * (q @ np.asarray(k, dtype=np.float64).T)
    if z.shape[1] == 0:
        return _orig["decode_attention"](q, k, v, scale)
    e = np.exp(z - z.max(axis=0, keepdims=True))
    p = e / e.sum(axis=0, keepdims=True)
    m = z.max(axis=1, keepdims=True)
    return p @ np.asarray(v, dtype=np.float64), (m + np.log(np.exp(z - m).sum(axis=1, keepdims=True)))[:, 0], z


def _attn_lse_without_max(q, k, v, scale):
    out, lse, z = _orig["decode_attention"](q, k, v, scale)
    if z.shape[1] == 0:
        return out, lse, z
    return out, np.log(np.exp(z - z.max(axis=1, keepdims=True)).sum(axis=1)), z


def _recall_of_dropped(logits, kept):
    z = np.asarray(logits, dtype=np.float64)
    drop = np.setdiff1d(np.arange(z.shape[1]), np.asarray(kept, dtype=np.int64))
    return _orig["attention_recall"](logits, drop)


def _freed_floor(old_lens, new_lens, block_size):
    bs = int(block_size)
    first = int(np.max(new_lens)) // bs
    return first, max(first, int(np.max(old_lens)) // bs)


def _budget_pct_rounded_up(n_layers, budget, capacity, budget_pct=0.0, scales=None):
    pct = float(np.float32(budget_pct))
    base = np.ceil(pct * float(capacity) / 100.0) if pct > 0.0 else float(budget)
    sc = np.ones(int(n_layers)) if scales is None else np.asarray(scales, np.float32).astype(np.float64)
    return np.floor(base * sc + 0.5).astype(np.int64)


def _rank_negative_zero_below(agg):
    a = np.asarray(agg, dtype=np.float64)
    key = -a - np.where((a == 0) & np.signbit(a), 1e-300, 0.0)
    return np.argsort(np.where(np.isnan(a), np.inf, key), kind="stable")


def _mask_dropped(q_center, W, band_mask=None):
    return q_center * W


_orig = {name: getattr(O, name) for name in dir(O) if callable(getattr(O, name))}

MUTATIONS = {
    "pairing swapped": ("to_bands", _swap_pairing),
    "de-rotation sign": ("derotate", _derotate_wrong_sign),
    "omega exponent missing factor 2": ("band_frequencies", _omega_missing_two),
    "omega index off by one": ("band_frequencies", _omega_off_by_one),
    "offset set starts at 0": ("offset_set", _offsets_from_zero),
    "offset set one short": ("offset_set", _offsets_one_short),
    "offset weight conjugated": ("offset_weight", _weight_conj),
    "offset weight summed not averaged": ("offset_weight", _weight_sum_not_mean),
    "folded center divides by W": ("folded_center", _folded_divides),
    "phase difference reversed": ("s_trig_polar", _polar_phase_flipped),
    "cosine replaced by sine": ("s_trig_polar", _polar_sin),
    "phasor without conjugate": ("s_trig_phasor", _phasor_no_conj),
    "real map B sign": ("s_trig_real_map", _realmap_b_sign),
    "norm term dropped": ("s_norm", _norm_dropped),
    "norm term without (1 - R)": ("s_norm", _norm_uses_abs_mean_only),
    "norm term with R instead of (1 - R)": ("s_norm", _norm_uses_r_not_one_minus_r),
    "sample std": ("gqa_znorm_max", _znorm_sample_std),
    "mean over heads": ("gqa_znorm_max", _znorm_mean_not_max),
    "max before normalising": ("gqa_znorm_max", _znorm_max_before_norm),
    "ties go to the higher slot": ("rank_order", _rank_ties_high),
    "keeps the lowest scores": ("rank_order", _rank_ascending),
    "window not forced in": ("select_kept", _select_no_window),
    "compaction off by one": ("compact_rows", _compact_off_by_one),
    "calibration |E q| for E|q|": ("calibration_stats", _calib_abs_of_mean),
    "calibration sums not means": ("calibration_stats", _calib_sum_not_mean),
    "calibration Re and Im swapped": ("calibration_stats", _calib_re_im_swapped),
    "offset max taken as the mean": ("s_trig_direct_max", _max_is_mean),
    "offset max taken as the min": ("s_trig_direct_max", _max_is_min),
    "percentage taken as a fraction": ("layer_budgets", _budget_pct_of_fraction),
    "layer budget rounded down": ("layer_budgets", _budget_floor_not_round),
    "layer budget scales ignored": ("layer_budgets", _budget_scales_ignored),
    "interval needs one row more": ("is_compressed", _interval_strict),
    "interval ignored": ("is_compressed", _interval_ignored),
    "freed blocks from the shortest layer": ("freed_block_range", _freed_from_shortest_layer),
    "attention without the scale": ("decode_attention", _attn_no_scale),
    "attention returns keys": ("decode_attention", _attn_keys_as_values),
    "softmax over the heads": ("decode_attention", _attn_softmax_over_heads),
    "lse without the max": ("decode_attention", _attn_lse_without_max),
    "recall of the dropped rows": ("attention_recall", _recall_of_dropped),
    "freed blocks rounded down": ("freed_block_range", _freed_floor),
    "percentage budget rounded up": ("layer_budgets", _budget_pct_rounded_up),
    "-0.0 ranked below +0.0": ("rank_order", _rank_negative_zero_below),
    "band mask dropped": ("folded_center", _mask_dropped),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(O, attr, bad)
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"planted mistake '{name}' passed every pin"
