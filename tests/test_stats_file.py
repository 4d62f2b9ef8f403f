"""The library's stats file format (tria_write_stats_file /
tria_read_stats_file): host-only, so these run without a GPU."""
import os
import struct

import numpy as np
import pytest

import key_retention_scoring_b200 as T
from key_retention_scoring_b200 import build as tria_build


@pytest.fixture(scope="module", autouse=True)
def _built():
    tria_build.build()


def _stats(L, H, F, seed):
    rng = np.random.default_rng(seed)
    re = rng.normal(size=(L, H, F)).astype(np.float32)
    im = rng.normal(size=(L, H, F)).astype(np.float32)
    am = (np.hypot(re, im) * (1 + 0.5 * rng.random((L, H, F)))).astype(np.float32)
    return re, im, am


@pytest.mark.parametrize("with_scales,with_mask", [(False, False), (True, False), (True, True)])
def test_round_trip_is_exact(tmp_path, with_scales, with_mask):
    L, H = 3, 8
    d = T.model_desc(L, H, 2, T.PAIR_INTERLEAVED, 5e5, offset_log2_max=12)
    re, im, am = _stats(L, H, 64, 3)
    sc = np.array([1.0, 0.5, 1.25], np.float32) if with_scales else None
    mk = np.linspace(0.1, 1.0, 64).astype(np.float32) if with_mask else None
    path = tmp_path / "stats.tria"
    T.tria_write_stats_file(path, d, re, im, am, sc, mk)
    # layout: 48-byte header, then the arrays
    raw = path.read_bytes()
    magic, version, nl, hq, hkv, hd, pair, m = struct.unpack_from("<IIiiiiii", raw, 0)
    assert (magic, version, nl, hq, hkv, hd, pair, m) == (0x54524941, 1, L, H, 2, 128, 1, 12)
    assert struct.unpack_from("<d", raw, 32)[0] == 5e5
    assert len(raw) == 48 + 4 * (3 * L * H * 64 + (L if with_scales else 0) + (64 if with_mask else 0))
    d2, re2, im2, am2, sc2, mk2 = T.tria_read_stats_file(path)
    assert (d2.n_layers, d2.n_q_heads, d2.n_kv_heads, d2.head_dim, d2.pairing,
            d2.rope_theta, d2.offset_log2_max) == (L, H, 2, 128, 1, 5e5, 12)
    for a, b in ((re, re2), (im, im2), (am, am2)):
        assert a.tobytes() == b.tobytes()
    assert (sc2 is None) == (sc is None) and (mk2 is None) == (mk is None)
    if sc is not None:
        assert sc.tobytes() == sc2.tobytes()
    if mk is not None:
        assert mk.tobytes() == mk2.tobytes()


def test_foreign_short_and_missing_files(tmp_path):
    d = T.model_desc(1, 4, 2, T.PAIR_NEOX, 1e4)
    re, im, am = _stats(1, 4, 64, 4)
    good = tmp_path / "good.tria"
    T.tria_write_stats_file(good, d, re, im, am)
    raw = good.read_bytes()
    cases = {"short": raw[:-4], "magic": b"XXXX" + raw[4:], "long": raw + b"\0\0\0\0"}
    for name, data in cases.items():
        p = tmp_path / f"{name}.tria"
        p.write_bytes(data)
        with pytest.raises(T.TriaError) as e:
            T.tria_read_stats_file(p)
        assert e.value.status == 6, name
    other = tmp_path / "v2.tria"
    other.write_bytes(raw[:4] + struct.pack("<I", 2) + raw[8:])
    with pytest.raises(T.TriaError) as e:
        T.tria_read_stats_file(other)
    assert e.value.status == 2
    with pytest.raises(T.TriaError) as e:
        T.tria_read_stats_file(tmp_path / "missing.tria")
    assert e.value.status == 6
    # asking for scales the file does not hold
    lib = T.lib()
    out = T.ModelDesc()
    buf = np.empty(1, np.float32)
    assert lib.tria_read_stats_file(os.fsencode(good), out, None, None, None, None, None,
                                    buf.ctypes.data, None) == 1
    assert lib.tria_write_stats_file(None, d, None, None, None, None, None) == 1
    assert T.tria_status_string(6).startswith("TRIA_ERR_IO")
