"""Budget variants on the GPU against the fp64 oracle, through the C ABI
(needs a B200): percentage budgets, per-layer budget scales with lengths per
(sequence, layer), and the compression interval."""
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
from oracle import tria_oracle as O  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _built():
    tria_build.build()
    synth.build()
    yield
    torch.cuda.empty_cache()


def _stats(w):
    cfg = w.cfg
    desc = T.model_desc(cfg.n_layers, cfg.n_q_heads, cfg.n_kv_heads, cfg.pairing, cfg.theta,
                        cfg.offset_log2_max)
    return T.tria_load_stats(desc, *w.stats)


def run_variant(cfg, layer_lens=None, scales=None, pct=0.0, interval=0, split_layers=None,
                offset_reduce=0):
    """One fused pass with the given budget variant; every unit checked
    against the oracle with its own budget and length: kept set, compacted
    K/V bytes and positions, the new lengths and the freed paged blocks.
    layer_lens: host int [n_seq][n_layers] (None: one length per sequence).
    split_layers: (l0, l1) also scored and selected on their own first."""
    w = synth.Workload(cfg)
    st = _stats(w)
    try:
        S, L, H = cfg.n_seq, cfg.n_layers, cfg.n_kv_heads
        d_ll = None
        if layer_lens is not None:
            lens = np.asarray(layer_lens, dtype=np.int64)
            d_ll = torch.from_numpy(lens.astype(np.int32)).cuda()
        else:
            lens = np.repeat(w.lens.astype(np.int64)[:, None], L, axis=1)
        cache = T.Cache.from_workload(w, layer_seq_lens=d_ll)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks, offset_reduce, budget_pct=pct,
                       layer_budget_scales=scales, interval=interval)
        budgets, bmax = T.tria_layer_budgets(st, cache, prm)
        want_b = O.layer_budgets(L, cfg.budget, w.max_seq_len, pct, scales)
        assert budgets == [int(b) for b in want_b] and bmax == int(want_b.max())
        saved, oras = {}, {}
        for s in range(S):
            for l in range(L):
                n = int(lens[s, l])
                for h in range(H):
                    kb = w.unit_rows("k", s, l, h, n)
                    pos = w.unit_positions(s, l, h, n)
                    saved[(s, l, h)] = (kb, w.unit_rows("v", s, l, h, n), pos)
                    oras[(s, l, h)] = PH.unit_oracle(w, s, l, h, k_bits=kb, positions=pos,
                                                     budget=budgets[l], interval=interval, n=n,
                                                     form="max" if offset_reduce else "folded")
        ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
        T.tria_read_device_status(ws)
        sep = {}
        if split_layers is not None:
            l0, l1 = split_layers
            cmax = max(1, w.max_seq_len - cfg.window - cfg.sinks)
            agg = torch.full((S, l1 - l0, H, cmax), float("nan"), device="cuda")
            sc = torch.full((S, l1 - l0, H, cmax, cfg.group), float("nan"), device="cuda")
            kp = torch.full((S, l1 - l0, H, bmax), -7, dtype=torch.int32, device="cuda")
            T.tria_score(st, cache, prm, l0, l1, agg, sc, ws)
            T.tria_select(st, cache, prm, agg, l0, l1, kp, ws)
            torch.cuda.synchronize()
            agg, sc, kp = agg.cpu().numpy(), sc.cpu().numpy(), kp.cpu().numpy()
            for (s, l, h), ora in oras.items():
                if not l0 <= l < l1:
                    continue
                where = f"{cfg.name} split s{s} l{l} h{h} N{ora['N']} B{budgets[l]}"
                if ora["scores"] is not None:
                    C = ora["N"] - cfg.window - cfg.sinks
                    PH.check_scores(sc[s, l - l0, h, :C], ora, where)
                    PH.check_agg(agg[s, l - l0, h, :C], ora, where)
                    PH.check_kept_same_precision(kp[s, l - l0, h], agg[s, l - l0, h, :C], ora["N"],
                                                 cfg, where, budget=budgets[l])
                PH.check_kept_vs_oracle(kp[s, l - l0, h], ora, cfg, where)
                sep[(s, l, h)] = kp[s, l - l0, h].copy()
        kept = torch.full((S, L, H, bmax), -7, dtype=torch.int32, device="cuda")
        freed = n_freed = None
        if cfg.layout == synth.LAYOUT_PAGED:
            freed = torch.full((S, w.max_blocks), -1, dtype=torch.int32, device="cuda")
            n_freed = torch.full((S,), -1, dtype=torch.int32, device="cuda")
        T.tria_compress_pass(st, cache, prm, kept, ws, freed, n_freed)
        torch.cuda.synchronize()
        assert T.tria_read_device_status(ws) == 0
        kh = kept.cpu().numpy()
        new_lens = O.pass_lengths(lens, np.asarray(budgets), interval)
        n_comp = 0
        for (s, l, h), ora in oras.items():
            where = f"{cfg.name} s{s} l{l} h{h} N{ora['N']} B{budgets[l]}"
            k = kh[s, l, h]
            PH.check_kept_vs_oracle(k, ora, cfg, where)
            if (s, l, h) in sep:
                assert np.array_equal(sep[(s, l, h)], k), f"{where}: fused vs separate kept"
            kb, vb, pos = saved[(s, l, h)]
            N, n_new = ora["N"], int(new_lens[s, l])
            n_comp += int(ora["compressed"])
            keep = k[:n_new] if ora["compressed"] else np.arange(N)
            got_k = w.unit_rows("k", s, l, h, N)
            got_v = w.unit_rows("v", s, l, h, N)
            assert np.array_equal(got_k[:n_new], kb[keep]), where
            assert np.array_equal(got_v[:n_new], vb[keep]), where
            assert np.array_equal(w.unit_positions(s, l, h, n_new), pos[keep]), where
        assert 0 < n_comp < len(oras) or interval == 0, "the case should mix compressed and left units"
        if d_ll is not None:
            assert np.array_equal(d_ll.cpu().numpy(), new_lens), "per-layer lengths"
            assert np.array_equal(w.seq_lens.cpu().numpy(), w.lens), "seq_lens must stay untouched"
        else:
            assert np.array_equal(w.seq_lens.cpu().numpy(), new_lens[:, 0]), "sequence lengths"
        if freed is not None:
            nf, fr = n_freed.cpu().numpy(), freed.cpu().numpy()
            for s in range(S):
                first, end = O.freed_block_range(lens[s], new_lens[s], cfg.block_size)
                assert nf[s] == end - first, (s, nf[s], first, end)
                assert np.array_equal(fr[s, :nf[s]], w.block_table_host[s, first:end]), s
        return budgets
    finally:
        st.free()
        del w
        torch.cuda.empty_cache()


def test_layer_scales_with_lengths_per_layer_gqa8():
    # four layers kept at 2048 x (1, 0.5, 1.25, 0.75) rows, lengths per layer
    # chosen so that layer 2 (2560 rows) stays short of its budget + interval
    cfg = synth.CONFIGS[2].scaled(n_layers=4, seq_len=5133)
    lens = np.array([[5133, 4000, 2600, 2300]])
    b = run_variant(cfg, layer_lens=lens, scales=[1.0, 0.5, 1.25, 0.75], interval=128,
                    split_layers=(1, 3))
    assert b == [2048, 1024, 2560, 1536]


def test_percent_budget_paged_interleaved_sinks_layer_lengths():
    # 40 % of the capacity as the base budget, the second layer at 0.6 of it;
    # lengths per (sequence, layer) differ, blocks are freed past the longest
    cfg = synth.CONFIGS[3].scaled(n_layers=2, n_seq=4, len_range=(1900, 5000))
    lens0 = synth.seq_lengths(cfg).astype(np.int64)
    lens = np.stack([lens0, np.maximum(lens0 - 700, 0)], axis=1)
    lens[1, 1] = lens0[1]          # a sequence whose second layer is its longest
    run_variant(cfg, layer_lens=lens, scales=[1.0, 0.6], pct=40.0, split_layers=(0, 2))


def test_interval_one_length_per_sequence_paged():
    # budget 2048, interval 128: sequences of 2040 .. 2300 rows; those with
    # N >= 2176 are compressed, the others keep every row (rows beyond the
    # kept row length 2048 included)
    cfg = synth.CONFIGS[3].scaled(n_layers=2, n_seq=6, len_range=(2040, 2300))
    run_variant(cfg, interval=128)


def test_interval_layer_lengths_contiguous_gqa4():
    cfg = synth.CONFIGS[1].scaled(n_layers=3, seq_len=3000)
    lens = np.array([[3000, 2100, 2180]])
    run_variant(cfg, layer_lens=lens, interval=128, split_layers=(0, 3))


def test_budget_variant_validation():
    cfg = synth.CONFIGS[0].scaled(n_layers=3, seq_len=1500)
    w = synth.Workload(cfg)
    st = _stats(w)
    try:
        L = cfg.n_layers
        ll = torch.from_numpy(np.full((cfg.n_seq, L), 1500, np.int32)).cuda()
        with_ll = T.Cache.from_workload(w, layer_seq_lens=ll)
        plain = T.Cache.from_workload(w)

        def status(cache, **kw):
            prm = T.params(cfg.budget, cfg.window, cfg.sinks, **kw)
            try:
                T.tria_layer_budgets(st, cache, prm)
                T.tria_workspace_size(st, cache, prm)
            except T.TriaError as e:
                return e.status
            return 0

        assert status(plain) == 0 and status(with_ll) == 0
        assert status(with_ll, layer_budget_scales=[1.0, 0.5, 2.0]) == 0
        # differing budgets need lengths per layer
        assert status(plain, layer_budget_scales=[1.0, 0.5, 2.0]) == 1
        assert status(plain, layer_budget_scales=[0.5, 0.5, 0.5]) == 0
        # a layer budget below window + sinks, non-finite or non-positive scales
        assert status(with_ll, layer_budget_scales=[1.0, 0.2, 1.0]) == 1
        assert status(with_ll, layer_budget_scales=[1.0, float("nan"), 1.0]) == 1
        assert status(with_ll, layer_budget_scales=[1.0, 0.0, 1.0]) == 1
        assert status(plain, budget_pct=101.0) == 1
        assert status(plain, budget_pct=-1.0) == 1
        assert status(plain, interval=-1) == 1
        # the percentage budget and the scales as the oracle computes them
        for pct, sc in ((50.0, None), (33.3, [1.0, 0.7, 1.3]), (25.0, [2.0, 1.0, 1.5])):
            prm = T.params(cfg.budget, cfg.window, cfg.sinks, budget_pct=pct, layer_budget_scales=sc)
            b, row = T.tria_layer_budgets(st, with_ll, prm)
            want = O.layer_budgets(L, cfg.budget, w.max_seq_len, pct, sc)
            assert b == [int(x) for x in want] and row == int(max(want)), (pct, sc, b, want)
        # lengths per layer: seq_lens may be absent
        nolens = T.Cache(0, w.k, w.v, None, w.query_pos, w.max_seq_len,
                         stride_seq=w.strides["seq"], stride_head=w.strides["head"],
                         stride_token=w.strides["token"], layer_seq_lens=ll)
        assert status(nolens) == 0
        nothing = T.Cache(0, w.k, w.v, None, w.query_pos, w.max_seq_len,
                          stride_seq=w.strides["seq"], stride_head=w.strides["head"],
                          stride_token=w.strides["token"], n_seq=1)
        assert status(nothing) == 1
    finally:
        st.free()


def test_layer_scales_max_over_offsets():
    # the max-over-offsets scorer with per-layer budgets and lengths
    cfg = synth.CONFIGS[2].scaled(n_layers=2, seq_len=4096)
    lens = np.array([[4096, 3000]])
    run_variant(cfg, layer_lens=lens, scales=[1.0, 0.5], split_layers=(0, 2),
                offset_reduce=T.OFFSET_MAX)
