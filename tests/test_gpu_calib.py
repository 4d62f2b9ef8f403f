"""Calibration reduction on the GPU (tria_calib_accumulate / _finalize) vs
the fp64 oracle's calibration_stats, through the C ABI (needs a B200)."""
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


@pytest.fixture(scope="module", autouse=True)
def _built():
    tria_build.build()
    yield
    torch.cuda.empty_cache()


def _desc(hq, pairing, head_dim=128):
    return T.model_desc(1, hq, 1, pairing, 1e4, head_dim=head_dim)


def _device_bf16(bits: np.ndarray):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def _run(desc, batches, hq):
    acc = torch.zeros((hq, 64, 3), dtype=torch.float64, device="cuda")
    n = 0
    for q in batches:
        T.tria_calib_accumulate(desc, q, acc)
        n += q.shape[0]
    outs = [torch.full((hq, 64), float("nan"), device="cuda") for _ in range(3)]
    T.tria_calib_finalize(desc, acc, n, *outs)
    torch.cuda.synchronize()
    return [o.cpu().numpy().astype(np.float64) for o in outs]


def _check(got, want, where):
    # fp32 |q_f| per token, fp64 sums, fp32 result: a few ulps of fp32
    for g, w, name in zip(got, want, ("E Re q", "E Im q", "E|q|")):
        scale = max(1.0, float(np.max(np.abs(w))))
        err = float(np.max(np.abs(g - w)))
        assert err <= 2e-6 * scale, f"{where} {name}: max error {err:.3g} (scale {scale:.3g})"


@pytest.mark.parametrize("pairing", [T.PAIR_NEOX, T.PAIR_INTERLEAVED], ids=["neox", "interleaved"])
def test_calibration_matches_oracle_two_batches(pairing):
    hq = 8
    bits = synth.calib_queries(3000, hq, seed=5, layer=2)
    q = _device_bf16(bits)
    got = _run(_desc(hq, pairing), [q[:1000], q[1000:]], hq)
    want = O.calibration_stats(O.bf16_bits_to_f64(bits), pairing)
    _check(got, want, f"pairing {pairing}")


def test_calibration_strided_heads_and_ragged_tokens():
    # heads taken from a wider buffer (head stride 128, token stride 11 x 128)
    # and token counts that leave ragged block ranges
    hq, wide = 8, 11
    bits = synth.calib_queries(777, wide, seed=6)
    qw = _device_bf16(bits)
    q = qw[:, 2:2 + hq, :]
    assert q.stride(1) == 128 and q.stride(0) == wide * 128
    got = _run(_desc(hq, T.PAIR_NEOX), [q[:1], q[1:130], q[130:]], hq)
    want = O.calibration_stats(O.bf16_bits_to_f64(bits[:, 2:2 + hq, :]), T.PAIR_NEOX)
    _check(got, want, "strided")


def test_calibration_single_token_is_exact_bands():
    hq = 3
    bits = synth.calib_queries(1, hq, seed=7)
    got = _run(_desc(hq, T.PAIR_INTERLEAVED), [_device_bf16(bits)], hq)
    z = O.to_bands(O.bf16_bits_to_f64(bits[0]), T.PAIR_INTERLEAVED)
    assert np.array_equal(got[0], z.real.astype(np.float32).astype(np.float64))
    assert np.array_equal(got[1], z.imag.astype(np.float32).astype(np.float64))
    _check(got, (z.real, z.imag, np.abs(z)), "one token")


def test_calibration_full_layer_sampled_heads():
    # one layer of the Qwen3-32B shape (64 query heads) over 8192 calibration
    # tokens (128 MB of bf16 queries); the oracle checks heads 0, 31 and 63
    hq, n = 64, 8192
    bits = synth.calib_queries(n, hq, seed=2, layer=17)
    q = _device_bf16(bits)
    got = _run(_desc(hq, T.PAIR_NEOX), [q], hq)
    for h in (0, 31, 63):
        want = O.calibration_stats(O.bf16_bits_to_f64(bits[:, h:h + 1, :]), T.PAIR_NEOX)
        _check([g[h:h + 1] for g in got], want, f"head {h}")


def test_calibration_argument_checks():
    hq = 4
    q = _device_bf16(synth.calib_queries(16, hq, seed=1))
    acc = torch.zeros((hq, 64, 3), dtype=torch.float64, device="cuda")
    with pytest.raises(T.TriaError) as ei:
        T.tria_calib_accumulate(_desc(hq, T.PAIR_NEOX, head_dim=64), q, acc)
    assert ei.value.status == 2  # UNSUPPORTED head_dim
    lib = T.lib()
    d = _desc(hq, T.PAIR_NEOX)
    # misaligned query pointer, negative token count
    assert lib.tria_calib_accumulate(d, q.data_ptr() + 2, 16, hq * 128, 128, acc.data_ptr(), None) == 1
    assert lib.tria_calib_accumulate(d, q.data_ptr(), -1, hq * 128, 128, acc.data_ptr(), None) == 1
    # no tokens: a no-op
    assert lib.tria_calib_accumulate(d, q.data_ptr(), 0, hq * 128, 128, acc.data_ptr(), None) == 0
    torch.cuda.synchronize()
    assert float(acc.abs().sum()) == 0.0
    with pytest.raises(T.TriaError):
        T.tria_calib_finalize(d, acc, 0, *[torch.empty((hq, 64), device="cuda") for _ in range(3)])


def test_calibrated_stats_through_a_stats_file(tmp_path):
    # calibrate on the device, save the statistics in the library's file
    # format, read them back and load them: the pass keeps the same rows as
    # with the statistics straight from the calibration
    cfg = synth.CONFIGS[0]
    hq = cfg.n_q_heads
    bits = synth.calib_queries(2048, hq, seed=9, layer=0)
    desc = T.model_desc(cfg.n_layers, hq, cfg.n_kv_heads, cfg.pairing, cfg.theta,
                        cfg.offset_log2_max)
    acc = torch.zeros((hq, 64, 3), dtype=torch.float64, device="cuda")
    T.tria_calib_accumulate(desc, _device_bf16(bits), acc)
    outs = [torch.empty((hq, 64), device="cuda") for _ in range(3)]
    T.tria_calib_finalize(desc, acc, 2048, *outs)
    torch.cuda.synchronize()
    re, im, am = (o.cpu().numpy().reshape(1, hq, 64) for o in outs)
    path = tmp_path / "calib.tria"
    T.tria_write_stats_file(path, desc, re, im, am)
    d2, re2, im2, am2, sc2, mk2 = T.tria_read_stats_file(path)
    assert sc2 is None and mk2 is None and d2.n_q_heads == hq

    kept = []
    for arrays, dd in (((re, im, am), desc), ((re2, im2, am2), d2)):
        w = synth.Workload(cfg)
        st = T.tria_load_stats(dd, *arrays)
        try:
            cache = T.Cache.from_workload(w)
            prm = T.params(cfg.budget, cfg.window, cfg.sinks)
            ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
            k = torch.full((cfg.n_seq, cfg.n_layers, cfg.n_kv_heads, cfg.budget), -7,
                           dtype=torch.int32, device="cuda")
            T.tria_compress_pass(st, cache, prm, k, ws)
            torch.cuda.synchronize()
            kept.append(k.cpu().numpy())
        finally:
            st.free()
            del w
    assert np.array_equal(kept[0], kept[1])
    assert np.all(kept[0][..., -cfg.window:] >= 0)
