"""Decode attention on the GPU (tria_decode_attention) against the fp64
oracle's decode_attention, through the C ABI (needs a B200); and the
retention check: after the compression pass the retained rows reproduce the
full-cache logits of the keys they hold, bit for bit."""
from __future__ import annotations

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import key_retention_scoring_b200 as T  # noqa: E402
from key_retention_scoring_b200 import build as tria_build  # noqa: E402
from oracle import tria_oracle as O  # noqa: E402

SCALE = 1.0 / np.sqrt(128.0)


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


def _decode(st, cache, w, layer, q_bits, want_logits=True):
    cfg = w.cfg
    S, Hq = cfg.n_seq, cfg.n_q_heads
    q = torch.from_numpy(q_bits.view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.full((S, Hq, 128), float("nan"), device="cuda")
    lse = torch.full((S, Hq), float("nan"), device="cuda")
    logits = (torch.full((S, Hq, w.max_seq_len), float("nan"), device="cuda")
              if want_logits else None)
    ws = T.alloc_workspace(T.tria_decode_workspace_size(st, cache))
    T.tria_read_device_status(ws)
    T.tria_decode_attention(st, cache, layer, q, SCALE, out, ws, lse=lse, logits=logits)
    torch.cuda.synchronize()
    status = T.tria_read_device_status(ws)
    return (out.cpu().numpy(), lse.cpu().numpy(),
            None if logits is None else logits.cpu().numpy(), status)


def _check_unit(out, lse, logits, q, k, v, where):
    """Tolerances from the arithmetic: a 128-term fp32 dot product is within
    2^-17 sum_d |q_d k_d| of the exact one (doubled here), so every logit is
    within E_j = scale 2^-16 sum_d |q_d k_jd|; softmax weights then move by
    at most ~2 E_max relative, exp2 and the fp32 sums add ~1e-5."""
    o_ref, l_ref, z_ref = O.decode_attention(q, k, v, SCALE)
    if k.shape[0] == 0:
        assert np.all(out == 0) and np.all(np.isneginf(lse)), where
        return
    e_j = SCALE * 2.0 ** -16 * (np.abs(q) @ np.abs(k).T)            # [G, N]
    e_max = e_j.max(axis=1)
    vmax = np.abs(v).max()
    tol_o = (4 * e_max + 1e-5)[:, None] * max(vmax, 1e-30)
    assert np.all(np.abs(out - o_ref) <= tol_o), (where, np.max(np.abs(out - o_ref) / tol_o))
    tol_l = 2 * e_max + 1e-5 * (1 + np.abs(l_ref))
    assert np.all(np.abs(lse - l_ref) <= tol_l), (where, lse, l_ref)
    if logits is not None:
        tol_z = e_j + 1e-6 * np.abs(z_ref)
        assert np.all(np.abs(logits - z_ref) <= tol_z), (where, np.max(np.abs(logits - z_ref) / tol_z))


def check_layer(w, st, cache, layer, lens, q_bits, units=None):
    """Every (sequence, KV head) of `layer` (or `units`) against the oracle."""
    cfg = w.cfg
    G = cfg.group
    out, lse, logits, status = _decode(st, cache, w, layer, q_bits)
    assert status == 0
    qf = O.bf16_bits_to_f64(q_bits)
    units = units or [(s, h) for s in range(cfg.n_seq) for h in range(cfg.n_kv_heads)]
    for s, h in units:
        n = int(lens[s])
        if n == 0:
            k = v = np.zeros((0, 128))
        else:
            k = O.bf16_bits_to_f64(w.unit_rows("k", s, layer, h, n))
            v = O.bf16_bits_to_f64(w.unit_rows("v", s, layer, h, n))
        sl = slice(h * G, (h + 1) * G)
        _check_unit(out[s, sl], lse[s, sl], logits[s, sl, :n], qf[s, sl], k, v,
                    f"{cfg.name} l{layer} s{s} h{h} N{n}")
    return out, lse, logits


def _queries(w, layer):
    return synth.decode_queries(w.cfg, layer, w.query_pos.cpu().numpy() + 1)


@pytest.mark.parametrize("case", ["gqa4_tiny", "gqa8_ragged", "gqa16", "gqa1", "gqa2_inter"])
def test_decode_matches_oracle_contiguous(case):
    cfg = {"gqa4_tiny": synth.CONFIGS[0],
           "gqa8_ragged": synth.CONFIGS[2].scaled(n_layers=1, seq_len=3001),
           "gqa16": synth.CONFIGS[0].scaled(n_q_heads=32, n_kv_heads=2, seq_len=1000),
           "gqa1": synth.CONFIGS[0].scaled(n_q_heads=2, n_kv_heads=2, seq_len=700),
           "gqa2_inter": synth.CONFIGS[0].scaled(n_q_heads=4, n_kv_heads=2, seq_len=513,
                                                 pairing=synth.PAIR_INTERLEAVED)}[case]
    w = synth.Workload(cfg)
    st = _stats(w)
    try:
        cache = T.Cache.from_workload(w)
        check_layer(w, st, cache, cfg.n_layers - 1, w.lens, _queries(w, cfg.n_layers - 1))
    finally:
        st.free()


def test_decode_paged_interleaved_lengths_per_layer_and_edges():
    # paged, G = 4, interleaved; lengths per (sequence, layer) including 0, 1
    # and a multiple of the 256-row split
    cfg = synth.CONFIGS[3].scaled(n_layers=2, n_seq=5, len_range=(1100, 3000))
    w = synth.Workload(cfg)
    st = _stats(w)
    try:
        lens0 = w.lens.astype(np.int64)
        ll = np.stack([lens0, lens0], axis=1)
        ll[0, 1], ll[1, 1], ll[2, 1] = 0, 1, 1024
        d_ll = torch.from_numpy(ll.astype(np.int32)).cuda()
        cache = T.Cache.from_workload(w, layer_seq_lens=d_ll)
        check_layer(w, st, cache, 1, ll[:, 1], _queries(w, 1))
        check_layer(w, st, cache, 0, ll[:, 0], _queries(w, 0),
                    units=[(s, h) for s in range(cfg.n_seq) for h in (0, 7)])
    finally:
        st.free()


def test_decode_bad_length_flagged():
    cfg = synth.CONFIGS[0]
    w = synth.Workload(cfg)
    st = _stats(w)
    try:
        cache = T.Cache.from_workload(w)
        w.seq_lens.fill_(w.max_seq_len + 3)
        out, lse, _, status = _decode(st, cache, w, 0, _queries(w, 0), want_logits=False)
        assert status == 1 and np.all(out == 0) and np.all(np.isneginf(lse))
        w.seq_lens.fill_(int(w.lens[0]))
        ws = T.alloc_workspace(T.tria_decode_workspace_size(st, cache))
        q = torch.zeros((1, cfg.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
        out_t = torch.empty((1, cfg.n_q_heads, 128), device="cuda")
        with pytest.raises(T.TriaError) as e:
            T.tria_decode_attention(st, cache, cfg.n_layers, q, SCALE, out_t, ws)
        assert e.value.status == 1
        with pytest.raises(T.TriaError) as e:
            T.tria_decode_attention(st, cache, 0, q, float("nan"), out_t, ws)
        assert e.value.status == 1
        with pytest.raises(T.TriaError) as e:
            T.tria_decode_attention(st, cache, 0, q, SCALE, out_t, ws[: ws.numel() - 1024])
        assert e.value.status == 3
    finally:
        st.free()


@pytest.mark.parametrize("budget_scales", [None, [1.0, 0.5]])
def test_retained_rows_reproduce_full_cache_logits(budget_scales):
    """Decode logits before the pass and after it: row j of a compressed unit
    has exactly the logit that row kept[j] had (the rows are byte copies and
    carry their rotation); the output over the retained rows matches the
    oracle over those rows."""
    cfg = synth.CONFIGS[2].scaled(n_layers=2, seq_len=5133)
    w = synth.Workload(cfg)
    st = _stats(w)
    try:
        S, L, H, G = cfg.n_seq, cfg.n_layers, cfg.n_kv_heads, cfg.group
        d_ll = None
        if budget_scales is not None:
            d_ll = torch.full((S, L), int(w.lens[0]), dtype=torch.int32, device="cuda")
        cache = T.Cache.from_workload(w, layer_seq_lens=d_ll)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks, layer_budget_scales=budget_scales)
        budgets, bmax = T.tria_layer_budgets(st, cache, prm)
        qb = [_queries(w, l) for l in range(L)]
        before = [_decode(st, cache, w, l, qb[l]) for l in range(L)]
        kept = torch.full((S, L, H, bmax), -7, dtype=torch.int32, device="cuda")
        ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
        T.tria_read_device_status(ws)
        T.tria_compress_pass(st, cache, prm, kept, ws)
        torch.cuda.synchronize()
        assert T.tria_read_device_status(ws) == 0
        kh = kept.cpu().numpy()
        lens_after = (d_ll.cpu().numpy() if d_ll is not None
                      else np.repeat(w.seq_lens.cpu().numpy()[:, None], L, axis=1))
        for l in range(L):
            B = budgets[l]
            assert np.all(lens_after[:, l] == B)
            out, lse, logits, status = _decode(st, cache, w, l, qb[l])
            assert status == 0
            z_full = before[l][2]
            qf = O.bf16_bits_to_f64(qb[l])
            for s in range(S):
                for h in range(H):
                    k_idx = kh[s, l, h, :B]
                    sl = slice(h * G, (h + 1) * G)
                    assert np.array_equal(logits[s, sl, :B], z_full[s, sl][:, k_idx]), (l, s, h)
                    k = O.bf16_bits_to_f64(w.unit_rows("k", s, l, h, B))
                    v = O.bf16_bits_to_f64(w.unit_rows("v", s, l, h, B))
                    _check_unit(out[s, sl], lse[s, sl], logits[s, sl, :B], qf[s, sl], k, v,
                                f"after l{l} s{s} h{h}")
    finally:
        st.free()
