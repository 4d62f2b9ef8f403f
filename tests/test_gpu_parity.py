"""CUDA pass vs the fp64 oracle, through the C ABI (needs a B200)."""
from __future__ import annotations

import math

import numpy as np
import pytest

import synth
from tests import parity_helpers as PH

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import key_retention_scoring_b200 as T  # noqa: E402
from key_retention_scoring_b200 import build as tria_build  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _built():
    tria_build.build()
    synth.build()
    yield
    torch.cuda.empty_cache()


def load_stats(w):
    cfg = w.cfg
    desc = T.model_desc(cfg.n_layers, cfg.n_q_heads, cfg.n_kv_heads, cfg.pairing, cfg.theta,
                        cfg.offset_log2_max)
    return T.tria_load_stats(desc, *w.stats)


def score_layers(w, st, layer0, layer1, want_scores=True, offset_reduce=0):
    """tria_score + tria_select over [layer0, layer1); host copies."""
    cfg = w.cfg
    cache = T.Cache.from_workload(w)
    prm = T.params(cfg.budget, cfg.window, cfg.sinks, offset_reduce)
    ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm, layer0, layer1))
    T.tria_read_device_status(ws)
    nl = layer1 - layer0
    cmax = max(1, w.max_seq_len - cfg.window - cfg.sinks)
    agg = torch.full((cfg.n_seq, nl, cfg.n_kv_heads, cmax), float("nan"), device="cuda")
    sc = (torch.full((cfg.n_seq, nl, cfg.n_kv_heads, cmax, cfg.group), float("nan"), device="cuda")
          if want_scores else None)
    kept = torch.full((cfg.n_seq, nl, cfg.n_kv_heads, cfg.budget), -7, dtype=torch.int32,
                      device="cuda")
    T.tria_score(st, cache, prm, layer0, layer1, agg, sc, ws)
    T.tria_select(st, cache, prm, agg, layer0, layer1, kept, ws)
    torch.cuda.synchronize()
    assert T.tria_read_device_status(ws) == 0
    return (agg.cpu().numpy(), None if sc is None else sc.cpu().numpy(), kept.cpu().numpy())


def compress(w, st, offset_reduce=0):
    cfg = w.cfg
    cache = T.Cache.from_workload(w)
    prm = T.params(cfg.budget, cfg.window, cfg.sinks, offset_reduce)
    ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
    T.tria_read_device_status(ws)
    kept = torch.full((cfg.n_seq, cfg.n_layers, cfg.n_kv_heads, cfg.budget), -7, dtype=torch.int32,
                      device="cuda")
    freed = n_freed = None
    if cfg.layout == synth.LAYOUT_PAGED:
        freed = torch.full((cfg.n_seq, w.max_blocks), -1, dtype=torch.int32, device="cuda")
        n_freed = torch.full((cfg.n_seq,), -1, dtype=torch.int32, device="cuda")
    T.tria_compress_pass(st, cache, prm, kept, ws, freed, n_freed)
    torch.cuda.synchronize()
    assert T.tria_read_device_status(ws) == 0
    return kept.cpu().numpy(), freed, n_freed


def all_units(cfg):
    return [(s, l, h) for s in range(cfg.n_seq) for l in range(cfg.n_layers)
            for h in range(cfg.n_kv_heads)]


def full_check(cfg, units=None, score_layers_sel=None, direct_form=False, offset_reduce=0,
               direct_sample=0.0):
    """Score/select parity on `units` (default: all), then the fused pass:
    same kept set, compacted bytes, lengths, positions, freed blocks."""
    w = synth.Workload(cfg)
    st = load_stats(w)
    try:
        units = all_units(cfg) if units is None else units
        saved = {}
        for (s, l, h) in units:
            saved[(s, l, h)] = (w.unit_rows("k", s, l, h), w.unit_rows("v", s, l, h),
                                w.unit_positions(s, l, h))
        layers = sorted({l for (_, l, _) in units}) if score_layers_sel is None else score_layers_sel
        sel_kept = {}
        for l in layers:
            agg, sc, kept = score_layers(w, st, l, l + 1, offset_reduce=offset_reduce)
            for (s, ll, h) in units:
                if ll != l:
                    continue
                kb, _, pos = saved[(s, l, h)]
                ora = PH.unit_oracle(w, s, l, h, k_bits=kb, positions=pos,
                                     form="max" if offset_reduce else "folded")
                N = ora["N"]
                where = f"{cfg.name} s{s} l{l} h{h} N{N}"
                if ora["scores"] is not None:
                    C = N - cfg.window - cfg.sinks
                    PH.check_scores(sc[s, 0, h, :C], ora, where)
                    PH.check_agg(agg[s, 0, h, :C], ora, where)
                    PH.check_kept_same_precision(kept[s, 0, h], agg[s, 0, h, :C], N, cfg, where)
                    if direct_form:
                        ora_d = PH.unit_oracle(w, s, l, h, k_bits=kb, positions=pos, form="direct")
                        PH.check_scores(sc[s, 0, h, :C], ora_d, where + " direct")
                    elif direct_sample > 0 and not offset_reduce:
                        PH.check_direct_sample(sc[s, 0, h, :C], w, s, l, h, kb, pos, ora,
                                               frac=direct_sample, where=where + " direct sample")
                else:
                    PH.check_kept_same_precision(kept[s, 0, h], np.zeros(0), N, cfg, where)
                PH.check_kept_vs_oracle(kept[s, 0, h], ora, cfg, where)
                sel_kept[(s, l, h)] = kept[s, 0, h].copy()
        lens_before = w.lens.copy()
        kept_all, freed, n_freed = compress(w, st, offset_reduce)
        # the fused pass keeps exactly what score + select keep
        for key, k in sel_kept.items():
            s, l, h = key
            assert np.array_equal(kept_all[s, l, h], k), f"fused vs separate kept differ at {key}"
        # every unit: ascending, window and sinks kept, size
        for s in range(cfg.n_seq):
            N = int(lens_before[s])
            ks = kept_all[s].reshape(-1, cfg.budget)
            if N <= cfg.budget:
                assert np.all(ks[:, :N] == np.arange(N)) and np.all(ks[:, N:] == -1)
                continue
            assert np.all(np.diff(ks, axis=1) > 0)
            assert np.all(ks[:, :cfg.sinks] == np.arange(cfg.sinks))
            assert np.all(ks[:, cfg.budget - cfg.window:] == np.arange(N - cfg.window, N))
        # compaction bytes and positions of the sampled units
        new_lens = w.seq_lens.cpu().numpy()
        for (s, l, h), (kb, vb, pos) in saved.items():
            N = int(lens_before[s])
            k = kept_all[s, l, h]
            n_new = min(N, cfg.budget)
            assert new_lens[s] == n_new
            got_k = w.unit_rows("k", s, l, h, N)
            got_v = w.unit_rows("v", s, l, h, N)
            assert np.array_equal(got_k, PH.compact_host(kb, k, N, cfg.budget)), (s, l, h)
            assert np.array_equal(got_v, PH.compact_host(vb, k, N, cfg.budget)), (s, l, h)
            got_p = w.unit_positions(s, l, h, n_new)
            assert np.array_equal(got_p, pos[k[:n_new]]), (s, l, h)
        if freed is not None:
            nf = n_freed.cpu().numpy()
            fr = freed.cpu().numpy()
            bs = cfg.block_size
            for s in range(cfg.n_seq):
                N = int(lens_before[s])
                if N <= cfg.budget:
                    assert nf[s] == 0
                    continue
                keep_b = math.ceil(cfg.budget / bs)
                old_b = math.ceil(N / bs)
                assert nf[s] == old_b - keep_b
                assert np.array_equal(fr[s, :nf[s]], w.block_table_host[s, keep_b:old_b])
    finally:
        st.free()
        del w
        torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# small cases: every unit against the oracle
# ---------------------------------------------------------------------------
def test_pr1_tiny_all_units_direct_and_folded():
    full_check(synth.CONFIGS[0], direct_form=True)


def test_qwen3_8b_shape_small():
    cfg = synth.CONFIGS[1].scaled(n_layers=2, seq_len=3000)   # C = 2744: 2 tiles + ragged
    full_check(cfg)


def test_qwen3_32b_shape_small_gqa8():
    cfg = synth.CONFIGS[2].scaled(n_layers=2, seq_len=5133)
    full_check(cfg)


def test_llama3_paged_small_interleaved_sinks():
    cfg = synth.CONFIGS[3].scaled(n_layers=2, n_seq=6, len_range=(1900, 5000))
    full_check(cfg)


def test_contiguous_batch_of_mixed_lengths():
    # a contiguous cache of several sequences of different lengths, some at or
    # below the budget (left as they are) and some compressed
    cfg = synth.CONFIGS[2].scaled(n_layers=2, n_q_heads=32, n_seq=5, seq_len=0,
                                  len_range=(1200, 7000))
    full_check(cfg)


def test_paged_noop_and_minimal_units():
    # N <= budget (no-op), N = budget + 1, budget = window + sinks (K = 0)
    base = synth.CONFIGS[3].scaled(n_layers=1, n_seq=3, len_range=(2040, 2060))
    full_check(base)
    full_check(base.scaled(budget=260))


@pytest.mark.parametrize("block_size", [8, 64, 128])
def test_paged_block_sizes(block_size):
    # paged blocks smaller and larger than the scoring tile's slot groups and
    # the compaction's chunks (a 128-token block spans two 64-row chunks)
    cfg = synth.CONFIGS[3].scaled(n_layers=1, n_seq=3, len_range=(2300, 5000),
                                  block_size=block_size)
    full_check(cfg)


def test_long_context_small_nearzero_heads():
    cfg = synth.CONFIGS[4].scaled(n_layers=2, seq_len=14000, near_zero_frac=0.5)
    full_check(cfg)


def test_no_window_no_sinks_gqa1_and_gqa2():
    full_check(synth.CONFIGS[0].scaled(n_q_heads=2, window=0, budget=700, seq_len=1500))
    full_check(synth.CONFIGS[0].scaled(n_q_heads=4, window=0, sinks=3, budget=900, seq_len=2100,
                                       pairing=synth.PAIR_INTERLEAVED))


def test_gqa16():
    # G = 16: the scoring kernel's 32-column instance (5-stage ring) and the
    # tail's four-lanes-per-candidate path, with a ragged last tile
    full_check(synth.CONFIGS[0].scaled(n_q_heads=32, n_kv_heads=2, seq_len=3000))
    # and a unit long enough for a cluster of two tail blocks
    full_check(synth.CONFIGS[4].scaled(n_layers=1, n_q_heads=16, n_kv_heads=1, seq_len=50000))


def test_units_of_one_partial_tile():
    # fewer than 128 candidates (one ragged scoring tile), K close to C, with
    # and without sinks, both pairings
    full_check(synth.CONFIGS[0].scaled(seq_len=300, budget=290, window=256))
    full_check(synth.CONFIGS[0].scaled(seq_len=200, budget=190, window=64, sinks=5,
                                       pairing=synth.PAIR_INTERLEAVED))
    full_check(synth.CONFIGS[0].scaled(seq_len=130, budget=2, window=1, sinks=0))


@pytest.mark.parametrize("hkv,bs,hq", [(4, 32, 32), (2, 64, 8), (2, 64, 16), (8, 16, 16)],
                         ids=["hkv4_bs32_g8", "hkv2_bs64_g4", "hkv2_bs64_g8", "hkv8_bs16_g2"])
def test_paged_whole_block_shapes(hkv, bs, hq):
    # whole-block paged scoring (Hkv x block size = 128 rows per tile): a head
    # fills one warp (32-token blocks), two warps (64), or shares a warp with
    # another head (16), with 2G columns per head
    cfg = synth.CONFIGS[3].scaled(n_layers=1, n_q_heads=hq, n_kv_heads=hkv, block_size=bs,
                                  n_seq=3, len_range=(2300, 4500))
    full_check(cfg)


def test_paged_gqa16():
    # G = 16 on a paged cache (Hkv x block size = 32 rows: the one-head scoring
    # kernel; four lanes per candidate in the unit tail)
    full_check(synth.CONFIGS[3].scaled(n_layers=1, n_q_heads=32, n_kv_heads=2, n_seq=3,
                                       len_range=(2300, 4000)))


def test_offset_sets_and_theta():
    for m in (0, 7, 12):
        full_check(synth.CONFIGS[0].scaled(offset_log2_max=m, seq_len=1800, theta=5e5))


# ---------------------------------------------------------------------------
# long units: the pass's unit tail splits a unit's candidates over a cluster of
# up to 8 blocks (more than 32768 candidates per unit take 2 blocks or more;
# a block holds at most 45056)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("seq_len", [60000, 100000, 200000], ids=["2blocks", "3blocks", "5blocks"])
def test_cluster_tail_long_units(seq_len):
    cfg = synth.CONFIGS[4].scaled(n_layers=1, n_q_heads=16, n_kv_heads=2, seq_len=seq_len)
    full_check(cfg)


def test_pass_units_past_the_cluster_tail():
    # more than 8 x 45056 candidates per unit: the pass selects with the
    # chunked tail over global agg (workspace histogram) instead of a cluster
    cfg = synth.CONFIGS[4].scaled(n_layers=1, n_q_heads=16, n_kv_heads=2, seq_len=370000)
    assert cfg.seq_len - cfg.window - cfg.sinks > 8 * 45056
    full_check(cfg)


def test_cluster_tail_ragged_lengths_paged():
    # lengths per sequence from 20000 to 120000: the cluster is sized for the
    # longest, so the shorter units leave their trailing blocks without candidates
    cfg = synth.CONFIGS[3].scaled(n_layers=1, n_q_heads=8, n_kv_heads=2, n_seq=3, budget=9000,
                                  len_range=(20000, 120000))
    full_check(cfg)


@pytest.mark.parametrize("C", [32768, 32769, 45056, 45057])
def test_tail_sizing_boundaries(C):
    # candidate counts at the unit tail's sizing limits: 32 keys per thread
    # exactly full (32768), the first 44-keys-per-thread unit (32769), one
    # block exactly full (45056), and the first cluster of 2 (45057: slices
    # of 22656 and 22401 candidates)
    cfg = synth.CONFIGS[2].scaled(n_layers=1, n_q_heads=16, n_kv_heads=2, seq_len=C + 256)
    full_check(cfg)


def test_ties_past_32767_in_one_block():
    # one block of 44 keys per thread (32768 < C <= 45056) with every candidate
    # of unit h = 1 equal: all C keys tie at T, more than 2^15 of them in the
    # block (its tie count is packed in 16 bits of an unsigned word), and the
    # K lowest slots are kept.  Unit h = 0, whose kept row lies just before,
    # must come out as its own selection: no write strays outside a unit's row
    cfg = synth.CONFIGS[2].scaled(n_layers=1, n_q_heads=16, n_kv_heads=2, seq_len=40000)
    w = synth.Workload(cfg)
    st = load_stats(w)
    try:
        N, W, S, B = cfg.seq_len, cfg.window, cfg.sinks, cfg.budget
        C, K = N - W - S, B - W - S
        assert 32768 < C <= 45056
        k = w.k[0]
        k[0, 1, S:N - W] = k[0, 1, S:S + 1]
        agg, _, kept_sep = score_layers(w, st, 0, 1, want_scores=False)
        want1 = np.concatenate([np.arange(S), np.arange(S, S + K), np.arange(N - W, N)])
        assert np.array_equal(kept_sep[0, 0, 1], want1)
        PH.check_kept_same_precision(kept_sep[0, 0, 0], agg[0, 0, 0, :C], N, cfg, "h0")
        kept_all, _, _ = compress(w, st)
        for h in range(2):
            assert np.array_equal(kept_all[0, 0, h], kept_sep[0, 0, h]), f"h{h}"
    finally:
        st.free()
        del w
        torch.cuda.empty_cache()


def test_cluster_tail_ties_across_blocks():
    # unit h = 0: every candidate row equal, so every agg is equal and the K
    # lowest slots are kept; unit h = 1: rows repeat with period 3, so the
    # threshold falls on a value held by about C / 3 keys in every block of the
    # cluster (three blocks), and the kept ties run into the second block
    cfg = synth.CONFIGS[4].scaled(n_layers=1, n_q_heads=16, n_kv_heads=2, seq_len=100000)
    w = synth.Workload(cfg)
    st = load_stats(w)
    try:
        N, W, S, B = cfg.seq_len, cfg.window, cfg.sinks, cfg.budget
        k = w.k[0]
        k[0, 0, S:N - W] = k[0, 0, S:S + 1]
        base = k[0, 1, S:S + 3].clone()
        C = N - W - S
        k[0, 1, S:N - W] = base.repeat((C + 2) // 3, 1)[:C]
        agg, _, kept_sep = score_layers(w, st, 0, 1, want_scores=False)
        for h in range(2):
            PH.check_kept_same_precision(kept_sep[0, 0, h], agg[0, 0, h, :C], N, cfg, f"h{h}")
        K = B - W - S
        want0 = np.concatenate([np.arange(S), np.arange(S, S + K), np.arange(N - W, N)])
        assert np.array_equal(kept_sep[0, 0, 0], want0)
        kept_all, _, _ = compress(w, st)
        for h in range(2):
            assert np.array_equal(kept_all[0, 0, h], kept_sep[0, 0, h]), f"h{h}"
    finally:
        st.free()
        del w
        torch.cuda.empty_cache()


@pytest.mark.parametrize("shape", ["gqa8", "gqa16"])
def test_nan_key_row_poisons_its_unit(shape):
    # one candidate row holding NaN (every dim in unit h = 0, one dim in unit
    # h = 1) scores NaN for every head; the unit's moments, and so every agg
    # of the unit, are NaN (the oracle's mean propagates it too).  All keys tie
    # at the lowest rank: both the fused pass (raw scores -> unit tail) and
    # score + select keep the K lowest candidate slots; other units are as usual
    if shape == "gqa8":
        cfg = synth.CONFIGS[2].scaled(n_layers=1, seq_len=5133)
    else:
        cfg = synth.CONFIGS[0].scaled(n_q_heads=32, n_kv_heads=2, seq_len=3000)
    w = synth.Workload(cfg)
    st = load_stats(w)
    try:
        N, W, S, B = cfg.seq_len, cfg.window, cfg.sinks, cfg.budget
        C, K = N - W - S, B - W - S
        k = w.k[0]
        k[0, 0, S + C // 3] = float("nan")
        k[0, 1, S + 2 * C // 3, 37] = float("nan")
        oras = [PH.unit_oracle(w, 0, 0, h) for h in range(2)]
        agg, _, kept_sep = score_layers(w, st, 0, 1, want_scores=False)
        want = np.concatenate([np.arange(S), np.arange(S, S + K), np.arange(N - W, N)])
        for h in range(2):
            assert np.all(np.isnan(agg[0, 0, h, :C])), f"h{h}: agg not NaN"
            assert np.array_equal(kept_sep[0, 0, h], want), f"h{h}"
            PH.check_kept_vs_oracle(kept_sep[0, 0, h], oras[h], cfg, f"h{h} oracle")
        for h in range(2, cfg.n_kv_heads):
            PH.check_kept_same_precision(kept_sep[0, 0, h], agg[0, 0, h, :C], N, cfg, f"h{h}")
        kept_all, _, _ = compress(w, st)
        for h in range(cfg.n_kv_heads):
            assert np.array_equal(kept_all[0, 0, h], kept_sep[0, 0, h]), f"h{h}"
    finally:
        st.free()
        del w
        torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# multi-pass: positions are no longer slot indices after compaction
# ---------------------------------------------------------------------------
def test_multi_pass_with_appends():
    cfg = synth.CONFIGS[2].scaled(n_layers=2, seq_len=4096)
    w = synth.Workload(cfg, capacity=4096)
    st = load_stats(w)
    try:
        cache = T.Cache.from_workload(w)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks)
        ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
        kept = torch.empty((1, cfg.n_layers, cfg.n_kv_heads, cfg.budget), dtype=torch.int32,
                           device="cuda")
        for it in range(4):
            if it:
                w.append(128)
            units = [(0, l, h) for l in range(cfg.n_layers) for h in (0, 5)]
            oras = {u: PH.unit_oracle(w, *u) for u in units}
            saved = {u: w.unit_rows("k", *u) for u in units}
            T.tria_compress_pass(st, cache, prm, kept, ws)
            torch.cuda.synchronize()
            kh = kept.cpu().numpy()
            for u, ora in oras.items():
                s, l, h = u
                PH.check_kept_vs_oracle(kh[s, l, h], ora, cfg, f"pass {it} {u}")
                N = ora["N"]
                assert np.array_equal(w.unit_rows("k", s, l, h, cfg.budget),
                                      saved[u][kh[s, l, h]])
            assert int(w.seq_lens[0]) == cfg.budget
    finally:
        st.free()


# ---------------------------------------------------------------------------
# selection on adversarial agg: ties, signed zeros, infinities, NaN
# ---------------------------------------------------------------------------
def test_select_adversarial_agg():
    from oracle import tria_oracle as O

    cfg = synth.CONFIGS[3].scaled(n_layers=1, n_seq=4, len_range=(3000, 9000), n_kv_heads=2,
                                  n_q_heads=4)
    w = synth.Workload(cfg, with_values=False, with_positions=False)
    st = load_stats(w)
    try:
        cache = T.Cache.from_workload(w)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks)
        ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm, 0, 1))
        cmax = w.max_seq_len - cfg.window - cfg.sinks
        rng = np.random.default_rng(5)
        agg = np.zeros((cfg.n_seq, 1, cfg.n_kv_heads, cmax), dtype=np.float32)
        kinds = ["int_ties", "all_equal", "zeros", "specials", "normal", "nan_neginf"]
        for s in range(cfg.n_seq):
            for h in range(cfg.n_kv_heads):
                kind = kinds[(s * cfg.n_kv_heads + h) % len(kinds)]
                if kind == "int_ties":
                    a = rng.integers(-3, 4, size=cmax).astype(np.float32)
                elif kind == "all_equal":
                    a = np.full(cmax, 1.25, dtype=np.float32)
                elif kind == "zeros":
                    a = np.where(rng.random(cmax) < 0.5, -0.0, 0.0).astype(np.float32)
                    a[rng.random(cmax) < 0.1] = 1.0
                elif kind == "specials":
                    a = rng.normal(size=cmax).astype(np.float32)
                    r = rng.random(cmax)
                    a[r < 0.05] = np.inf
                    a[(r >= 0.05) & (r < 0.1)] = -np.inf
                    a[(r >= 0.1) & (r < 0.3)] = np.nan
                elif kind == "nan_neginf":
                    # only -inf and NaN: the K-th key falls among them, and
                    # -inf must rank above NaN
                    a = np.full(cmax, -np.inf, dtype=np.float32)
                    a[rng.random(cmax) < 0.6] = np.nan
                else:
                    a = rng.normal(size=cmax).astype(np.float32)
                agg[s, 0, h] = a
        d_agg = torch.from_numpy(agg).cuda()
        kept = torch.full((cfg.n_seq, 1, cfg.n_kv_heads, cfg.budget), -7, dtype=torch.int32,
                          device="cuda")
        T.tria_select(st, cache, prm, d_agg, 0, 1, kept, ws)
        kh = kept.cpu().numpy()
        for s in range(cfg.n_seq):
            N = int(w.lens[s])
            C = N - cfg.window - cfg.sinks
            for h in range(cfg.n_kv_heads):
                ref = O.select_kept(agg[s, 0, h, :C].astype(np.float64), N, cfg.budget, cfg.window,
                                    cfg.sinks)
                assert np.array_equal(kh[s, 0, h], ref), (s, h)
    finally:
        st.free()


# ---------------------------------------------------------------------------
# device-side input errors and host validation
# ---------------------------------------------------------------------------
def test_device_status_and_validation():
    cfg = synth.CONFIGS[0].scaled(seq_len=1500)
    w = synth.Workload(cfg)
    st = load_stats(w)
    try:
        cache = T.Cache.from_workload(w)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks)
        nbytes = T.tria_workspace_size(st, cache, prm)
        ws = T.alloc_workspace(nbytes)
        T.tria_read_device_status(ws)
        kept = torch.full((1, 1, cfg.n_kv_heads, cfg.budget), -7, dtype=torch.int32, device="cuda")
        # a length beyond max_seq_len: flagged, unit skipped, kept row all -1
        w.seq_lens.fill_(w.max_seq_len + 5)
        T.tria_compress_pass(st, cache, prm, kept, ws)
        assert T.tria_read_device_status(ws) == 1
        assert np.all(kept.cpu().numpy() == -1)
        assert T.tria_read_device_status(ws) == 0
        w.seq_lens.fill_(int(w.lens[0]))
        # host validation: nothing enqueued
        with pytest.raises(T.TriaError) as e:
            T.tria_compress_pass(st, cache, T.params(100, 256, 0), kept, ws)
        assert e.value.status == 1
        small = T.alloc_workspace(nbytes - 4096)
        with pytest.raises(T.TriaError) as e:
            T.tria_compress_pass(st, cache, prm, kept, small)
        assert e.value.status == 3
        with pytest.raises(T.TriaError) as e:
            T.tria_score(st, cache, prm, 0, 2, kept, None, ws)
        assert e.value.status == 1
        odd = torch.empty(nbytes + 512, dtype=torch.uint8, device="cuda")[16:]
        with pytest.raises(T.TriaError) as e:
            T.tria_compress_pass(st, cache, prm, kept, odd)
        assert e.value.status == 3
        bad = T.Cache(0, [w.k[0][..., 1:]], w.v, w.seq_lens, w.query_pos, w.max_seq_len,
                      stride_seq=w.strides["seq"], stride_head=w.strides["head"],
                      stride_token=w.strides["token"])
        with pytest.raises(T.TriaError) as e:
            T.tria_compress_pass(st, bad, prm, kept, ws)
        assert e.value.status == 1
    finally:
        st.free()


def test_generator_matches_host_recipe():
    for cfg in (synth.CONFIGS[0], synth.CONFIGS[3].scaled(n_layers=2, n_seq=3,
                                                            len_range=(500, 900))):
        w = synth.Workload(cfg)
        for (s, l, h) in [(0, 0, 0), (cfg.n_seq - 1, cfg.n_layers - 1, cfg.n_kv_heads - 1)]:
            dev = w.unit_rows("k", s, l, h)
            host = synth.host_key_rows(cfg, w.centers, s, l, h, np.arange(len(dev)))
            mism = np.mean(dev != host)
            assert mism < 1e-4, (cfg.name, s, l, h, mism)
        del w
        torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# full-size workloads: sampled units against the oracle
# ---------------------------------------------------------------------------
def _sample_units(cfg, n, seed):
    rng = np.random.default_rng(seed)
    out = set()
    while len(out) < n:
        out.add((int(rng.integers(cfg.n_seq)), int(rng.integers(cfg.n_layers)),
                 int(rng.integers(cfg.n_kv_heads))))
    return sorted(out)


# sampled units against the folded oracle on every key, and against the direct
# 17-offset form on a seeded 1 % of their keys
def test_full_size_qwen3_8b():
    cfg = synth.CONFIGS[1]
    full_check(cfg, units=_sample_units(cfg, 6, 1), direct_sample=0.01)


def test_full_size_qwen3_32b_32k():
    cfg = synth.CONFIGS[2]
    full_check(cfg, units=_sample_units(cfg, 4, 2), direct_sample=0.01)


def test_full_size_qwen3_32b_131k():
    cfg = synth.CONFIGS[4]
    full_check(cfg, units=_sample_units(cfg, 3, 4), direct_sample=0.01)


def test_full_size_llama3_batched_paged():
    cfg = synth.CONFIGS[3]
    free, total = torch.cuda.mem_get_info()
    need = 178e9
    if free < need:
        pytest.skip(f"needs ~{need / 1e9:.0f} GB free, {free / 1e9:.0f} GB available")
    full_check(cfg, units=_sample_units(cfg, 4, 3), direct_sample=0.01)


# ---------------------------------------------------------------------------
# max-over-offsets mode (tria_params.offset_reduce = TRIA_OFFSET_MAX)
# ---------------------------------------------------------------------------
def test_offset_max_pr1_tiny():
    full_check(synth.CONFIGS[0], offset_reduce=T.OFFSET_MAX)


def test_offset_max_qwen3_32b_shape_small():
    cfg = synth.CONFIGS[2].scaled(n_layers=2, seq_len=4096)
    units = [(0, l, h) for l in range(2) for h in (0, 3, 7)]
    full_check(cfg, units=units, offset_reduce=T.OFFSET_MAX)


def test_offset_max_paged_interleaved_sinks():
    cfg = synth.CONFIGS[3].scaled(n_layers=1, n_seq=3, len_range=(3000, 9000))
    units = [(s, 0, h) for s in range(3) for h in (0, 5)]
    full_check(cfg, units=units, offset_reduce=T.OFFSET_MAX)


def test_offset_max_eight_offsets():
    cfg = synth.CONFIGS[2].scaled(n_layers=1, seq_len=3000, offset_log2_max=7)
    units = [(0, 0, h) for h in (1, 6)]
    full_check(cfg, units=units, offset_reduce=T.OFFSET_MAX)


@pytest.mark.parametrize("m", [0, 15], ids=["one_offset", "sixteen_offsets"])
def test_offset_max_offset_count_limits(m):
    # |D| = 1 (every offset column past the first masked) and |D| = 16 (none
    # masked, no 17th column)
    cfg = synth.CONFIGS[2].scaled(n_layers=1, seq_len=3000, offset_log2_max=m)
    units = [(0, 0, h) for h in (0, 5)]
    full_check(cfg, units=units, offset_reduce=T.OFFSET_MAX)


def test_offset_max_unsupported_shapes():
    cfg = synth.CONFIGS[0].scaled(n_q_heads=32, n_kv_heads=2)  # G = 16
    w = synth.Workload(cfg, with_values=False, with_positions=False)
    st = load_stats(w)
    try:
        cache = T.Cache.from_workload(w)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks, T.OFFSET_MAX)
        with pytest.raises(T.TriaError) as ei:
            T.tria_workspace_size(st, cache, prm)
        assert ei.value.status == 2
        # G = 16 with few offsets (2 |D| G <= 272) is unsupported as well: the
        # max-over-offsets kernel is built for G <= 8
        st.free()
        cfg4 = cfg.scaled(offset_log2_max=3)
        w4 = synth.Workload(cfg4, with_values=False, with_positions=False)
        st = load_stats(w4)
        cache = T.Cache.from_workload(w4)
        with pytest.raises(T.TriaError) as ei:
            T.tria_workspace_size(st, cache, prm)
        assert ei.value.status == 2
        # the mean mode of the same shape is fine
        T.tria_workspace_size(st, cache, T.params(cfg.budget, cfg.window, cfg.sinks))
        with pytest.raises(T.TriaError) as ei:
            T.tria_workspace_size(st, cache, T.params(cfg.budget, cfg.window, cfg.sinks, 7))
        assert ei.value.status == 1
    finally:
        st.free()


# ---------------------------------------------------------------------------
# the high-frequency band mask (article 2607.13051 sec. 7), folded into the
# coefficients at load time
# ---------------------------------------------------------------------------
def test_band_mask_scores_and_selection():
    cfg = synth.CONFIGS[2].scaled(n_layers=1, seq_len=3000)
    w = synth.Workload(cfg)
    mask = np.linspace(0.2, 1.0, 64).astype(np.float32)
    desc = T.model_desc(cfg.n_layers, cfg.n_q_heads, cfg.n_kv_heads, cfg.pairing, cfg.theta,
                        cfg.offset_log2_max)
    st = T.tria_load_stats(desc, *w.stats, band_mask=mask)
    try:
        agg, sc, kept = score_layers(w, st, 0, 1)
        C = int(w.lens[0]) - cfg.window - cfg.sinks
        for h in (0, 3, 7):
            ora = PH.unit_oracle(w, 0, 0, h, band_mask=mask)
            where = f"{cfg.name} band mask h{h}"
            PH.check_scores(sc[0, 0, h, :C], ora, where)
            PH.check_agg(agg[0, 0, h, :C], ora, where)
            PH.check_kept_same_precision(kept[0, 0, h], agg[0, 0, h, :C], ora["N"], cfg, where)
            PH.check_kept_vs_oracle(kept[0, 0, h], ora, cfg, where)
    finally:
        st.free()
        del w
        torch.cuda.empty_cache()
