"""Philox4x32-10 counter-based generator (Salmon, Moraes, Dror, Shaw, "Parallel
random numbers: as easy as 1, 2, 3", SC'11), vectorised in numpy.

The device generator in ``synth/csrc/synth.cu`` implements the same
definition; both feed the seeded synthetic workloads.  Nothing here belongs to
the compression method: it only draws random numbers.
"""
from __future__ import annotations

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = np.uint32(0x9E3779B9)
W1 = np.uint32(0xBB67AE85)
MASK32 = np.uint64(0xFFFFFFFF)
KEY_TAG = 0x74726961  # second key word of every stream ("tria")

# stream identifiers (fourth counter word)
STREAM_QMEAN = 1
STREAM_QRATIO = 2
STREAM_KCENTER = 3
STREAM_KNOISE = 4
STREAM_V = 5
STREAM_HEADPICK = 6
STREAM_LENGTHS = 7
STREAM_BLOCKS = 8
STREAM_QCAL_CENTER = 9
STREAM_QCAL_NOISE = 10
STREAM_DECODE_Q = 11


def philox4x32_10(c0, c1, c2, c3, k0, k1=KEY_TAG):
    """Ten rounds of Philox4x32 on broadcastable uint32 counter words.
    Returns four uint32 arrays."""
    x0, x1, x2, x3 = (np.asarray(v, dtype=np.uint64) & MASK32 for v in (c0, c1, c2, c3))
    x0, x1, x2, x3 = np.broadcast_arrays(x0, x1, x2, x3)
    x0, x1, x2, x3 = (np.array(v, dtype=np.uint64) for v in (x0, x1, x2, x3))
    ka = np.uint64(np.uint32(k0))
    kb = np.uint64(np.uint32(k1))
    for _ in range(10):
        p0 = M0 * x0
        p1 = M1 * x2
        hi0, lo0 = p0 >> np.uint64(32), p0 & MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & MASK32
        x0, x1, x2, x3 = (hi1 ^ x1 ^ ka) & MASK32, lo1, (hi0 ^ x3 ^ kb) & MASK32, lo0
        ka = (ka + np.uint64(W0)) & MASK32
        kb = (kb + np.uint64(W1)) & MASK32
    return tuple(v.astype(np.uint32) for v in (x0, x1, x2, x3))


def uniform01(x):
    """(x + 0.5) / 2^32: open interval (0, 1), fp64."""
    return (np.asarray(x, dtype=np.float64) + 0.5) * (1.0 / 4294967296.0)


def normals4(c0, c1, c2, c3, seed):
    """Four standard normals per counter (two Box-Muller pairs), fp64."""
    r = philox4x32_10(c0, c1, c2, c3, seed)
    u = [uniform01(v) for v in r]
    ra = np.sqrt(-2.0 * np.log(u[0]))
    rb = np.sqrt(-2.0 * np.log(u[2]))
    return (ra * np.cos(2.0 * np.pi * u[1]), ra * np.sin(2.0 * np.pi * u[1]),
            rb * np.cos(2.0 * np.pi * u[3]), rb * np.sin(2.0 * np.pi * u[3]))


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round fp32 values to bfloat16 (round to nearest even) as uint16 bits."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    out = ((u + bias) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(f)
    if np.any(nan):
        out[nan] = np.uint16(0x7FC0)
    return out
