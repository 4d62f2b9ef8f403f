"""Pins of the fp64 oracle against things other than itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with a
hand-derived golden value (``tests/golden/``), a closed form, textbook RoPE
done by brute force with real rotation matrices, an invariant, or a brute-force
Python-loop computation on tiny inputs.  They are collected by
``test_oracle_pins.py`` and re-run against deliberately broken copies of the
oracle by ``test_oracle_mutations.py`` (every planted mistake must trip at
least one pin).
"""
from __future__ import annotations

import math
from pathlib import Path

import numpy as np

from oracle import tria_oracle as O

GOLDEN = Path(__file__).resolve().parent / "golden"


def _golden_kv(name: str) -> dict:
    out = {}
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.split("#", 1)[0].strip()
        if "=" in line:
            k, v = line.split("=", 1)
            out[k.strip()] = v.strip()
    return out


def _golden_rows(name: str) -> list[list[float]]:
    rows = []
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.split("#", 1)[0].strip()
        if line:
            rows.append([float(t) for t in line.split()])
    return rows


def _floats(s: str) -> np.ndarray:
    return np.array([float(t) for t in s.split()])


# ---------------------------------------------------------------------------
# textbook RoPE, written independently of the oracle: real 2x2 rotations
# ---------------------------------------------------------------------------
def _rope_pairs(d: int, pairing: int):
    """Index pairs (a, b) rotated together by RoPE."""
    if pairing == O.PAIR_NEOX:
        return [(i, i + d // 2) for i in range(d // 2)]
    return [(2 * i, 2 * i + 1) for i in range(d // 2)]


def _rope_inv_freq(d: int, base: float) -> np.ndarray:
    # RoFormer / HF convention: 1 / base^(arange(0, d, 2) / d)
    return 1.0 / (base ** (np.arange(0, d, 2, dtype=np.float64) / d))


def _rope_rotate(x: np.ndarray, pos: float, base: float, pairing: int) -> np.ndarray:
    d = x.shape[-1]
    inv = _rope_inv_freq(d, base)
    y = np.array(x, dtype=np.float64, copy=True)
    for i, (a, b) in enumerate(_rope_pairs(d, pairing)):
        ang = pos * inv[i]
        c, s = math.cos(ang), math.sin(ang)
        xa, xb = x[..., a], x[..., b]
        y[..., a] = c * xa - s * xb
        y[..., b] = s * xa + c * xb
    return y


def _vec_from_pairs(re: np.ndarray, im: np.ndarray, pairing: int) -> np.ndarray:
    d = 2 * len(re)
    v = np.zeros(d)
    for i, (a, b) in enumerate(_rope_pairs(d, pairing)):
        v[a], v[b] = re[i], im[i]
    return v


def _offsets_by_hand(m: int):
    out, x = [], 1
    for _ in range(m + 1):
        out.append(x)
        x *= 2
    return out


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------
def pin_pairing_golden():
    g = _golden_kv("pairing_d8.txt")
    x = _floats(g["x"])
    z = O.to_bands(x, O.PAIR_NEOX)
    assert np.array_equal(z.real, _floats(g["neox_re"])), z
    assert np.array_equal(z.imag, _floats(g["neox_im"])), z
    z = O.to_bands(x, O.PAIR_INTERLEAVED)
    assert np.array_equal(z.real, _floats(g["interleaved_re"])), z
    assert np.array_equal(z.imag, _floats(g["interleaved_im"])), z
    for p in (O.PAIR_NEOX, O.PAIR_INTERLEAVED):
        assert np.array_equal(O.from_bands(O.to_bands(x, p), p), x)


def pin_omega_golden():
    g = _golden_kv("omega_d128.txt")
    for key, theta in (("theta_1e4", 1e4), ("theta_1e6", 1e6), ("theta_5e5", 5e5)):
        om = O.band_frequencies(128, theta)
        assert om.shape == (64,)
        toks = g[key].split()
        for i in range(0, len(toks), 2):
            f = int(toks[i].split(":")[1])
            assert abs(om[f] - float(toks[i + 1])) <= 1e-15 * max(1.0, abs(float(toks[i + 1]))) * 10, (key, f, om[f])


def pin_offset_set_golden():
    g = _golden_kv("offset_set.txt")
    D = O.offset_set(int(g["log2_max"]))
    assert len(D) == int(g["size"])
    assert D[0] == float(g["first"]) and D[-1] == float(g["last"])
    assert list(D) == [float(v) for v in _offsets_by_hand(16)]
    assert len(O.offset_set()) == 17 and O.offset_set()[-1] == 65536.0


def pin_offset_weight_closed_forms():
    D = O.offset_set(16)
    for om, re, im in _golden_rows("offset_weight.txt"):
        W = O.offset_weight(np.array([om]), D)[0]
        # the largest angle, omega * 2^16, carries an fp64 rounding of ~5e-11 rad
        assert abs(W - complex(re, im)) < 1e-10, (om, W, re, im)
    om = np.array([0.3, 1.0, 2.5])
    W0 = O.offset_weight(om, O.offset_set(0))
    assert np.allclose(W0, np.exp(1j * om), atol=1e-15)


def _random_unit(rng, d, G, N, pairing, theta, pos_max=50000):
    F = d // 2
    q_center = rng.normal(size=(G, F)) + 1j * rng.normal(size=(G, F))
    q_abs = np.abs(q_center) * (1 + rng.uniform(0, 0.5, size=(G, F)))
    k_pre = rng.normal(0.5, 1.0, size=(N, d))
    pos = np.sort(rng.choice(pos_max, size=N, replace=False)).astype(np.int64)
    k_post = np.stack([_rope_rotate(k_pre[i], float(pos[i]), theta, pairing) for i in range(N)])
    p_q = int(pos[-1])
    return q_center, q_abs, k_pre, k_post, pos, p_q


def pin_brute_force_rope():
    """S~_trig equals the offset-averaged textbook RoPE logit of the query
    center (as a real vector rotated at p_q + delta) with the cached key."""
    rng = np.random.default_rng(11)
    for pairing in (O.PAIR_NEOX, O.PAIR_INTERLEAVED):
        for theta, m in ((1e4, 16), (5e5, 12), (1e6, 7)):
            d, G, N = 16, 2, 12
            qc, _, k_pre, k_post, pos, p_q = _random_unit(rng, d, G, N, pairing, theta)
            omega = O.band_frequencies(d, theta)
            offs = _offsets_by_hand(m)
            # S_norm vanishes when E|q| = |E q|
            got_f = O.unit_scores(k_post, pos, p_q, qc, np.abs(qc), omega, pairing, m, form="folded")
            got_d = O.unit_scores(k_post, pos, p_q, qc, np.abs(qc), omega, pairing, m, form="direct")
            for h in range(G):
                qv = _vec_from_pairs(qc[h].real, qc[h].imag, pairing)
                for i in range(N):
                    acc = 0.0
                    for dl in offs:
                        acc += float(np.dot(_rope_rotate(qv, p_q + dl, theta, pairing), k_post[i]))
                    ref = acc / len(offs)
                    scale = np.sum(np.abs(qv)) * np.sum(np.abs(k_post[i]))
                    assert abs(got_f[h, i] - ref) < 1e-9 * scale, (pairing, theta, h, i, got_f[h, i], ref)
                    assert abs(got_d[h, i] - ref) < 1e-9 * scale, (pairing, theta, h, i, got_d[h, i], ref)


def pin_offset_max_brute_force():
    """The max-over-offsets variant equals the largest textbook RoPE logit of
    the query center rotated at p_q + delta, delta in D, with the cached key;
    it bounds the offset average from above, and with D = {1} all forms agree
    with the single distance Delta + 1."""
    rng = np.random.default_rng(23)
    for pairing in (O.PAIR_NEOX, O.PAIR_INTERLEAVED):
        for theta, m in ((1e4, 16), (5e5, 5)):
            d, G, N = 16, 2, 10
            qc, _, k_pre, k_post, pos, p_q = _random_unit(rng, d, G, N, pairing, theta)
            omega = O.band_frequencies(d, theta)
            got = O.unit_scores(k_post, pos, p_q, qc, np.abs(qc), omega, pairing, m, form="max")
            avg = O.unit_scores(k_post, pos, p_q, qc, np.abs(qc), omega, pairing, m, form="direct")
            for h in range(G):
                qv = _vec_from_pairs(qc[h].real, qc[h].imag, pairing)
                for i in range(N):
                    vals = [float(np.dot(_rope_rotate(qv, p_q + dl, theta, pairing), k_post[i]))
                            for dl in _offsets_by_hand(m)]
                    scale = np.sum(np.abs(qv)) * np.sum(np.abs(k_post[i]))
                    assert abs(got[h, i] - max(vals)) < 1e-9 * scale, (pairing, theta, h, i)
                    assert got[h, i] >= avg[h, i] - 1e-9 * scale
            one_max = O.unit_scores(k_post, pos, p_q, qc, np.abs(qc), omega, pairing, 0, form="max")
            one_avg = O.unit_scores(k_post, pos, p_q, qc, np.abs(qc), omega, pairing, 0, form="folded")
            assert np.allclose(one_max, one_avg, atol=1e-9)


def pin_single_distance_brute_force():
    """Eq. 2 and Eq. 3 at one distance equal the plain RoPE dot product."""
    rng = np.random.default_rng(5)
    for pairing in (O.PAIR_NEOX, O.PAIR_INTERLEAVED):
        d, theta = 8, 1e4
        omega = O.band_frequencies(d, theta)
        q = rng.normal(size=d)
        k = rng.normal(size=d)
        for pq, pk in ((7, 3), (1000, 10), (40000, 39999), (5, 5)):
            ref = float(np.dot(_rope_rotate(q, pq, theta, pairing), _rope_rotate(k, pk, theta, pairing)))
            qb = O.to_bands(q, pairing)
            kb = O.to_bands(k, pairing)
            for fn in (O.s_trig_polar, O.s_trig_phasor):
                got = float(fn(qb, kb, omega, pq - pk))
                assert abs(got - ref) < 1e-10 * (1 + abs(ref)), (fn.__name__, pq, pk, got, ref)
            # de-rotating the post-RoPE key recovers the pre-RoPE bands
            kpost = O.to_bands(_rope_rotate(k, pk, theta, pairing), pairing)
            assert np.allclose(O.derotate(kpost, np.array(pk), omega), kb, atol=1e-10)


def pin_worked_example_golden():
    g = _golden_kv("worked_example_d4.txt")
    omega = np.array([math.pi / 2, math.pi / 4])
    qc = np.array([[1 + 0j, 2j]])
    qa = np.array([[1.0, 3.0]])
    r = math.sqrt(2) / 2
    k_post = np.array([[0.0, 2.0, 1.0, 0.0], [0.0, -r, 1.0, r]])
    pos = np.array([0, 1])
    for tag in ("a", "b"):
        m = int(g[f"log2_max_{tag}"])
        exp = _floats(g[f"expected_{tag}"])
        for form in ("folded", "direct"):
            got = O.unit_scores(k_post, pos, 2, qc, qa, omega, O.PAIR_NEOX, m, form=form)[0]
            # angles reach pi/2 * 2^16 with D up to 2^16: fp64 rounding ~1e-11
            assert np.allclose(got, exp, rtol=0, atol=1e-10), (tag, form, got, exp)


def pin_closed_form_phi_zero():
    """All phi_f = 0 (keys aligned with the center):
    S~_trig = sum_f |E q_f| r_f (1/|D|) sum_delta cos(omega_f (Delta + delta))."""
    rng = np.random.default_rng(3)
    d, G, theta = 32, 1, 1e4
    F = d // 2
    omega = O.band_frequencies(d, theta)
    qc = rng.normal(size=(G, F)) + 1j * rng.normal(size=(G, F))
    for m in (0, 7, 16):
        offs = _offsets_by_hand(m)
        N = 6
        pos = np.array([0, 3, 100, 2047, 30000, 65535])
        p_q = 70000
        radius = rng.uniform(0.5, 2.0, size=(N, F))
        k_pre_b = radius * (qc[0] / np.abs(qc[0]))
        # post-RoPE bands: multiply by e^{i omega p}, written with cos/sin
        ang = omega[None, :] * pos[:, None]
        kp = k_pre_b * (np.cos(ang) + 1j * np.sin(ang))
        k_post = np.stack([_vec_from_pairs(kp[i].real, kp[i].imag, O.PAIR_NEOX) for i in range(N)])
        got = O.unit_scores(k_post, pos, p_q, qc, np.abs(qc), omega, O.PAIR_NEOX, m)[0]
        for i in range(N):
            dl = p_q - pos[i]
            ref = 0.0
            for f in range(F):
                avg = sum(math.cos(omega[f] * (dl + o)) for o in offs) / len(offs)
                ref += abs(qc[0, f]) * radius[i, f] * avg
            assert abs(got[i] - ref) < 1e-10 * np.sum(np.abs(qc)) * 2, (m, i, got[i], ref)


def pin_folded_equals_direct():
    """Eq. 7 (and Eq. 8) reproduce the literal 17-fold loop of Eq. 4 to
    machine precision for delta_max in {2^7, 2^12, 2^16} (the numerical
    confirmation reported for the folded form)."""
    rng = np.random.default_rng(7)
    d, theta = 128, 1e4
    omega = O.band_frequencies(d, theta)
    F = d // 2
    for m in (7, 12, 16):
        D = O.offset_set(m)
        W = O.offset_weight(omega, D)
        qc = rng.normal(size=F) + 1j * rng.normal(size=F)
        k = rng.normal(size=(64, F)) + 1j * rng.normal(size=(64, F))
        delta = rng.integers(0, 40000, size=64)
        direct = O.s_trig_direct_average(qc, k, omega, delta, D)
        folded = O.s_trig_folded(O.folded_center(qc, W), k, omega, delta)
        realm = O.s_trig_real_map(qc, k, omega, delta, W)
        assert np.max(np.abs(direct - folded)) < 1e-10, (m, np.max(np.abs(direct - folded)))
        assert np.max(np.abs(direct - realm)) < 1e-10, (m, np.max(np.abs(direct - realm)))


def pin_rotation_equivariance():
    """Shifting every position and p_q by s (keys re-rotated) leaves every
    score unchanged."""
    rng = np.random.default_rng(9)
    for pairing in (O.PAIR_NEOX, O.PAIR_INTERLEAVED):
        d, G, N, theta = 16, 3, 10, 5e5
        qc, qa, k_pre, k_post, pos, p_q = _random_unit(rng, d, G, N, pairing, theta, 3000)
        omega = O.band_frequencies(d, theta)
        base = O.unit_scores(k_post, pos, p_q, qc, qa, omega, pairing)
        for s in (1, 777, 100000):
            k2 = np.stack([_rope_rotate(k_pre[i], float(pos[i] + s), theta, pairing) for i in range(N)])
            sh = O.unit_scores(k2, pos + s, p_q + s, qc, qa, omega, pairing)
            assert np.allclose(sh, base, rtol=0, atol=1e-8 * np.max(np.abs(base))), (pairing, s)


def pin_norm_term():
    rng = np.random.default_rng(13)
    d, G, N, theta = 16, 2, 8, 1e4
    F = d // 2
    qc, qa, k_pre, k_post, pos, p_q = _random_unit(rng, d, G, N, O.PAIR_NEOX, theta)
    omega = O.band_frequencies(d, theta)
    # E[q] = 0: the trigonometric term vanishes and the norm term is E|q|.|k|
    z = np.zeros_like(qc)
    got = O.unit_scores(k_post, pos, p_q, z, qa, omega, O.PAIR_NEOX)
    kb = O.to_bands(k_pre, O.PAIR_NEOX)
    for h in range(G):
        for i in range(N):
            ref = sum(qa[h, f] * abs(kb[i, f]) for f in range(F))
            assert abs(got[h, i] - ref) < 1e-10 * (1 + ref), (h, i)
    # hand value: one band, E|q| = 5, |E q| = 3 (R = 0.6), |k| = 2 -> (1-0.6)*5*2 = 4
    val = O.s_norm(np.array([3.0 + 0j]), np.array([5.0]), np.array([[0.0 + 2.0j]]))
    assert abs(val[0] - 4.0) < 1e-12, val
    assert abs(1 - O.concentration(np.array([3.0 + 0j]), np.array([5.0]))[0] - 0.4) < 1e-12
    # independent of distance: the difference of two p_q is the trig term alone
    a = O.unit_scores(k_post, pos, p_q, qc, qa, omega, O.PAIR_NEOX)
    b = O.unit_scores(k_post, pos, p_q, qc, np.abs(qc), omega, O.PAIR_NEOX)
    c = O.unit_scores(k_post, pos, p_q + 1234, qc, qa, omega, O.PAIR_NEOX)
    e = O.unit_scores(k_post, pos, p_q + 1234, qc, np.abs(qc), omega, O.PAIR_NEOX)
    assert np.allclose(a - b, c - e, atol=1e-9)
    assert np.all(a - b >= -1e-12)


def pin_gqa_normalize_then_max():
    rng = np.random.default_rng(17)
    G, C = 3, 9
    S = rng.normal(10, 4, size=(G, C))
    agg, m, sd = O.gqa_znorm_max(S)
    for i in range(C):
        best = -1e300
        for h in range(G):
            mean = sum(S[h]) / C
            var = sum((x - mean) ** 2 for x in S[h]) / C
            zz = (S[h, i] - mean) / (math.sqrt(var) + 1e-6)
            best = max(best, zz)
        assert abs(agg[i] - best) < 1e-12, (i, agg[i], best)
    # identical heads -> the single head's z; z has mean 0 and std ~1
    one = rng.normal(3, 2, size=C)
    agg1, _, _ = O.gqa_znorm_max(np.stack([one, one]))
    agg0, _, _ = O.gqa_znorm_max(one[None])
    assert np.allclose(agg1, agg0)
    assert abs(agg0.mean()) < 1e-12 and abs(agg0.std() - 1) < 1e-5


def pin_select_brute_force():
    rng = np.random.default_rng(19)
    for trial in range(60):
        N = int(rng.integers(5, 40))
        W = int(rng.integers(0, 5))
        S = int(rng.integers(0, 4))
        B = int(rng.integers(W + S, N + 3))
        C = N - W - S
        if C <= 0:
            continue
        agg = rng.integers(0, 6, size=C).astype(np.float64)  # many exact ties
        if trial % 3 == 0:
            agg = rng.normal(size=C)
        kept = O.select_kept(agg, N, B, W, S)
        if N <= B:
            assert list(kept) == list(range(N))
            continue
        K = B - W - S
        order = sorted(range(C), key=lambda i: (-agg[i], i))
        ref = sorted(list(range(S)) + [S + i for i in order[:K]] + list(range(N - W, N)))
        assert list(kept) == ref, (N, W, S, B, agg, kept, ref)
        assert len(kept) == B and all(kept[i] < kept[i + 1] for i in range(B - 1))
    # explicit tie: candidates (slot 0..3) scores 1, 3, 3, 2; keep 1 -> slot 1
    assert list(O.select_kept(np.array([1.0, 3.0, 3.0, 2.0]), 4, 1, 0, 0)) == [1]
    # -0.0 equals +0.0 (lower slot wins); NaN ranks last
    assert list(O.select_kept(np.array([-0.0, 0.0]), 2, 1, 0, 0)) == [0]
    assert list(O.select_kept(np.array([np.nan, -5.0]), 2, 1, 0, 0)) == [1]


def pin_p4_candidate_count():
    g = _golden_kv("p4_runtime_log.txt")
    n_kv, w, s = int(g["n_kv"]), int(g["window"]), int(g["sinks"])
    C = int(g["n_old"])
    agg = np.arange(C, dtype=np.float64)
    kept = O.select_kept(agg, n_kv, C // 2 + w, w, s)  # accepts exactly n_old candidates
    assert len(kept) == C // 2 + w
    assert list(kept[-w:]) == list(range(n_kv - w, n_kv))
    try:
        O.select_kept(agg[:-1], n_kv, C // 2 + w, w, s)
    except AssertionError:
        pass
    else:
        raise AssertionError("candidate count other than n_kv - window accepted")


def pin_calibration_golden():
    """Two hand-worked tokens, both pairings (tests/golden/calib_two_tokens_d4.txt)."""
    g = _golden_kv("calib_two_tokens_d4.txt")
    toks = np.array([[float(t) for t in row.split()] for row in g["tokens"].split(";")])
    q = toks[:, None, :]  # [2 tokens][1 head][4]
    for pairing, tag in ((O.PAIR_NEOX, "neox"), (O.PAIR_INTERLEAVED, "inter")):
        re, im, ab = O.calibration_stats(q, pairing)
        for got, key in ((re, "re"), (im, "im"), (ab, "abs")):
            want = np.array([float(t) for t in g[f"{tag}_{key}"].split()])
            assert np.allclose(got[0], want, rtol=0, atol=1e-12), (tag, key, got[0], want)


def pin_calibration_invariants():
    """E|q_f| >= |E q_f| (triangle inequality); token order does not matter;
    constant queries give their own bands; means scale with the queries."""
    rng = np.random.default_rng(11)
    q = rng.normal(size=(50, 3, 16)) + rng.normal(size=(1, 3, 16))
    for pairing in (O.PAIR_NEOX, O.PAIR_INTERLEAVED):
        re, im, ab = O.calibration_stats(q, pairing)
        assert np.all(ab + 1e-12 >= np.hypot(re, im))
        re2, im2, ab2 = O.calibration_stats(q[rng.permutation(50)], pairing)
        assert np.allclose(re, re2) and np.allclose(im, im2) and np.allclose(ab, ab2)
        re3, im3, ab3 = O.calibration_stats(-2.5 * q, pairing)
        assert np.allclose(re3, -2.5 * re) and np.allclose(im3, -2.5 * im)
        assert np.allclose(ab3, 2.5 * ab)
        one = np.repeat(q[:1], 7, axis=0)
        z = O.to_bands(q[0], pairing)
        re4, im4, ab4 = O.calibration_stats(one, pairing)
        assert np.allclose(re4, z.real) and np.allclose(im4, z.imag)
        assert np.allclose(ab4, np.abs(z))
        # strongly concentrated queries: E|q| and |E q| nearly agree (R -> 1)
        tight = q[:1] + 1e-6 * rng.normal(size=(50, 3, 16))
        re5, im5, ab5 = O.calibration_stats(tight, pairing)
        assert np.allclose(ab5, np.hypot(re5, im5), rtol=1e-5)


def pin_compaction():
    rng = np.random.default_rng(23)
    rows = rng.integers(0, 2 ** 16, size=(20, 4), dtype=np.uint16)
    kept = np.array([0, 3, 4, 9, 17, 18, 19])
    out = O.compact_rows(rows, kept)
    for j, src in enumerate(kept):
        assert np.array_equal(out[j], rows[src])


def pin_whole_unit_pipeline():
    """compress_unit: window and sinks kept, |kept| = B, ascending, and the
    candidate scores are the unit scores of slots sinks .. N-W-1."""
    rng = np.random.default_rng(29)
    d, G, N, theta = 16, 2, 40, 1e4
    qc, qa, _, k_post, pos, p_q = _random_unit(rng, d, G, N, O.PAIR_INTERLEAVED, theta)
    omega = O.band_frequencies(d, theta)
    res = O.compress_unit(k_post, pos, p_q, qc, qa, omega, O.PAIR_INTERLEAVED,
                          budget=20, window=6, sinks=2)
    kept = res["kept"]
    assert len(kept) == 20 and set(range(2)) <= set(kept) and set(range(34, 40)) <= set(kept)
    full = O.unit_scores(k_post, pos, p_q, qc, qa, omega, O.PAIR_INTERLEAVED)
    assert np.allclose(res["scores"], full[:, 2:34])
    res2 = O.compress_unit(k_post[:15], pos[:15], p_q, qc, qa, omega, O.PAIR_INTERLEAVED,
                           budget=20, window=6, sinks=2)
    assert list(res2["kept"]) == list(range(15))


def pin_budget_variants_golden():
    """Percentage budget, per-layer scales, the compression interval and the
    freed blocks, against tests/golden/budget_variants.txt (worked by hand from
    the runtime log of GitHub issue #10 and article 2607.13051 sec. 8)."""
    g = _golden_kv("budget_variants.txt")
    cap, n_kv, w = int(g["capacity"]), int(g["n_kv"]), int(g["window"])
    b50 = O.layer_budgets(1, 0, cap, budget_pct=50.0)
    assert list(b50) == [int(g["pct50_budget"])]
    assert list(O.layer_budgets(3, 0, cap, budget_pct=25.0)) == [int(g["pct25_budget"])] * 3
    # the logged pass evicts nothing: every one of the n_kv rows stays
    assert not O.is_compressed(n_kv, int(b50[0]), 128)
    agg = np.zeros(n_kv - w)
    assert len(O.select_kept(agg, n_kv, int(b50[0]), w, 0)) == n_kv
    sc = [float(x) for x in g["scales"].split()]
    want = [int(x) for x in g["budgets"].split()]
    assert list(O.layer_budgets(len(sc), int(g["base"]), cap, scales=sc)) == want
    assert list(O.layer_budgets(4, int(g["base"]), cap)) == [int(g["base"])] * 4
    assert list(O.layer_budgets(4, int(g["base"]), cap, scales=[1.0] * 4)) == [int(g["base"])] * 4
    assert list(O.layer_budgets(1, 7, cap, scales=[0.5])) == [int(g["half7"])]
    assert list(O.layer_budgets(1, 9, cap, scales=[0.5])) == [int(g["half9"])]
    B = int(g["base"])
    assert not O.is_compressed(B + 127, B, 128) and O.is_compressed(B + 128, B, 128)
    assert O.is_compressed(B + 1, B, 0) and not O.is_compressed(B, B, 0)
    assert O.is_compressed(B + 1, B, 1) and not O.is_compressed(B, B, 1)
    grow_in = [int(x) for x in g["growth_in"].split()]
    grow_out = [int(x) for x in g["growth_out"].split()]
    for n_in, n_out in zip(grow_in, grow_out):
        assert int(O.pass_lengths(np.array([[n_in]]), np.array([B]), 128)[0, 0]) == n_out
    old = np.array([2176, 2176])
    new_a = O.pass_lengths(old[None], np.array([2048, 1024]), 128)[0]
    assert list(new_a) == [2048, 1024]
    assert O.freed_block_range(old, new_a, 16) == tuple(int(x) for x in g["freed_a"].split())
    new_b = O.pass_lengths(old[None], np.array([1024, 1024]), 128)[0]
    assert O.freed_block_range(old, new_b, 16) == tuple(int(x) for x in g["freed_b"].split())
    # lengths that are not whole blocks, and a percentage that is not a whole row
    assert O.freed_block_range(np.array([2100, 2100]), np.array([1000, 1030]), 16) == \
        tuple(int(x) for x in g["freed_c"].split())
    assert list(O.layer_budgets(1, 0, int(g["pct_cap"]), budget_pct=float(g["pct_odd"]))) == \
        [int(g["pct_odd_budget"])]


def pin_interval_unit_pipeline():
    """compress_unit with an interval: a unit short of B + beta rows keeps all
    of them; at B + beta it is cut to exactly B with window and sinks kept."""
    rng = np.random.default_rng(31)
    d, G, theta = 16, 2, 1e4
    qc, qa, _, k_post, pos, p_q = _random_unit(rng, d, G, 40, O.PAIR_NEOX, theta)
    omega = O.band_frequencies(d, theta)
    kw = dict(budget=24, window=6, sinks=1, interval=16)
    short = O.compress_unit(k_post[:39], pos[:39], p_q, qc, qa, omega, O.PAIR_NEOX, **kw)
    assert list(short["kept"]) == list(range(39)) and short["agg"] is None
    full = O.compress_unit(k_post, pos, p_q, qc, qa, omega, O.PAIR_NEOX, **kw)
    kept = full["kept"]
    assert len(kept) == 24 and kept[0] == 0 and list(kept[-6:]) == list(range(34, 40))


def pin_decode_attention_closed_forms():
    """Softmax attention by closed forms: one row returns its value and its
    logit; equal logits average the values; two keys whose logits differ by
    ln 3 weigh 3/4 and 1/4; a constant added to every logit moves lse by that
    constant and leaves the output; the row order does not matter; no rows
    give zero and -inf."""
    rng = np.random.default_rng(37)
    d = 8
    q = rng.normal(size=(2, d))
    k1, v1 = rng.normal(size=(1, d)), rng.normal(size=(1, d))
    out, lse, z = O.decode_attention(q, k1, v1, 0.5)
    assert np.allclose(out, np.repeat(v1, 2, axis=0)) and np.allclose(lse, 0.5 * (q @ k1[0]))
    kk = np.repeat(k1, 4, axis=0)
    vv = rng.normal(size=(4, d))
    out, lse, _ = O.decode_attention(q, kk, vv, 1.0)
    assert np.allclose(out, np.repeat(vv.mean(axis=0)[None], 2, axis=0))
    assert np.allclose(lse, q @ k1[0] + np.log(4.0))
    # logits 0 and ln 3 with scale 1/2: keys 0 and e * 2 ln 3 / (q . e), one head
    e0 = np.zeros(d)
    e0[0] = 1.0
    qh = np.array([[2.0] + [0.0] * (d - 1)])
    k2 = np.stack([np.zeros(d), e0 * np.log(3.0)])     # q.k = 0, 2 ln 3; scaled 0, ln 3
    v2 = np.stack([np.full(d, 1.0), np.full(d, -1.0)])
    out, lse, z = O.decode_attention(qh, k2, v2, 0.5)
    assert np.allclose(z, [[0.0, np.log(3.0)]])
    assert np.allclose(out, 0.25 * v2[0] + 0.75 * v2[1]) and np.allclose(lse, np.log(4.0))
    # a key along q moves every logit of that head by the same amount
    k3 = rng.normal(size=(6, d))
    v3 = rng.normal(size=(6, d))
    o_a, l_a, _ = O.decode_attention(qh, k3, v3, 0.3)
    o_b, l_b, _ = O.decode_attention(qh, k3 + 1.5 * e0, v3, 0.3)
    assert np.allclose(o_a, o_b) and np.allclose(l_b - l_a, 0.3 * 2.0 * 1.5)
    perm = rng.permutation(6)
    o_c, l_c, _ = O.decode_attention(qh, k3[perm], v3[perm], 0.3)
    assert np.allclose(o_a, o_c) and np.allclose(l_a, l_c)
    out, lse, _ = O.decode_attention(q, np.zeros((0, d)), np.zeros((0, d)), 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def pin_attention_recall():
    """All rows kept: 1; none: 0; two rows with logits 0 and ln 3: keeping the
    second keeps 3/4 of the mass."""
    z = np.array([[0.0, np.log(3.0)], [1.0, 1.0]])
    assert np.allclose(O.attention_recall(z, [0, 1]), [1.0, 1.0])
    assert np.allclose(O.attention_recall(z, []), [0.0, 0.0])
    assert np.allclose(O.attention_recall(z, [1]), [0.75, 0.5])


def pin_select_signed_zeros():
    """-0.0 and +0.0 are equal numbers (IEEE 754), so they tie and the lower
    slot wins either way round; NaN ranks below -inf."""
    for agg, want in (([-0.0, 0.0, 1.0], [0, 2]), ([0.0, -0.0, 1.0], [0, 2]),
                      ([np.nan, -np.inf, -0.0], [1, 2])):
        kept = O.select_kept(np.array(agg), 3, 2, 0, 0)
        assert list(kept) == want, (agg, kept)


def pin_band_mask():
    """The high-frequency band mask rescales |mu'_f| in the trigonometric
    term only (article 2607.13051 sec. 7): the masked score equals the trig
    term of the query center multiplied by the mask (with the norm term
    zeroed by E|q| = |E q|) plus the unmasked norm term; an all-ones mask is
    no mask and an all-zero mask leaves the norm term alone."""
    rng = np.random.default_rng(41)
    d, G, N, theta = 16, 2, 12, 1e4
    qc, qa, k_pre, k_post, pos, p_q = _random_unit(rng, d, G, N, O.PAIR_NEOX, theta)
    omega = O.band_frequencies(d, theta)
    m = rng.random(d // 2)
    got = O.unit_scores(k_post, pos, p_q, qc, qa, omega, O.PAIR_NEOX, band_mask=m)
    trig = O.unit_scores(k_post, pos, p_q, qc * m, np.abs(qc * m), omega, O.PAIR_NEOX)
    kb = O.to_bands(k_pre, O.PAIR_NEOX)
    norm = np.stack([O.s_norm(qc[h], qa[h], kb) for h in range(G)])
    assert np.allclose(got, trig + norm, rtol=0, atol=1e-10 * (1 + np.abs(got).max()))
    plain = O.unit_scores(k_post, pos, p_q, qc, qa, omega, O.PAIR_NEOX)
    ones = O.unit_scores(k_post, pos, p_q, qc, qa, omega, O.PAIR_NEOX, band_mask=np.ones(d // 2))
    zero = O.unit_scores(k_post, pos, p_q, qc, qa, omega, O.PAIR_NEOX, band_mask=np.zeros(d // 2))
    assert np.allclose(ones, plain, rtol=0, atol=1e-12 * (1 + np.abs(plain).max()))
    assert np.allclose(zero, norm, rtol=0, atol=1e-12 * (1 + np.abs(norm).max()))


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
