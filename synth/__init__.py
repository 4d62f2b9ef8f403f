"""Seeded synthetic workloads shaped like the TriAttention pages' workloads.

Shared by the tests (both the oracle side and the CUDA side) and by
``bench.py``.  It holds none of the compression method's arithmetic: it draws
random numbers (Philox4x32-10, ``synth/philox.py`` on the host and
``synth/csrc/synth.cu`` on the device) and lays out KV caches.

Recipe (one seed per workload):
* calibrated statistics per (layer, query head, band f): Re and Im of E[q_f]
  ~ N(0, 1); E|q_f| = |E q_f| (1 + U(0, 0.5));
* pre-RoPE keys: per (layer, KV head) center ~ N(0, 2^2) per dimension plus
  per-token noise N(0, 0.5^2); rotated by RoPE at the token's position with
  the workload's pairing and base in fp64, then rounded to bf16;
* values: bf16 N(0, 1);
* the long-context chat workload gives 10% of its (layer, KV head) pairs
  near-zero centers (x0.01), i.e. non-concentrated heads.
"""
from __future__ import annotations

import ctypes
import math
import os
import shutil
import subprocess
from dataclasses import dataclass, replace

import numpy as np

from . import philox as P

PAIR_NEOX = 0
PAIR_INTERLEAVED = 1
LAYOUT_CONTIGUOUS = 0
LAYOUT_PAGED = 1

_DIR = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_DIR, "libtria_synth.so")
_lib = None


@dataclass(frozen=True)
class Config:
    name: str
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    pairing: int
    theta: float
    n_seq: int
    seq_len: int            # every sequence (0: drawn per sequence, see len_range)
    budget: int
    window: int
    sinks: int
    seed: int
    layout: int = LAYOUT_CONTIGUOUS
    block_size: int = 16
    len_range: tuple = (0, 0)
    near_zero_frac: float = 0.0
    head_dim: int = 128
    offset_log2_max: int = 16
    center_sigma: float = 2.0
    noise_sigma: float = 0.5

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def scaled(self, **kw) -> "Config":
        return replace(self, **kw)


CONFIGS = {
    0: Config("PR1 tiny (1 layer, 8q/2kv, 2304 tokens)", 1, 8, 2, PAIR_NEOX, 1e4, 1, 2304,
              1024, 256, 0, seed=0),
    1: Config("Qwen3-8B shape (36 layers, 32q/8kv, 8448 tokens)", 36, 32, 8, PAIR_NEOX, 1e4, 1,
              8448, 2048, 256, 0, seed=1),
    2: Config("Qwen3-32B shape, 32K decode (64 layers, 64q/8kv, 32768 tokens)", 64, 64, 8,
              PAIR_NEOX, 1e4, 1, 32768, 2048, 256, 0, seed=2),
    3: Config("Llama-3-8B shape, 64 paged sequences (32 layers, 32q/8kv, 4096-32768 tokens)",
              32, 32, 8, PAIR_INTERLEAVED, 5e5, 64, 0, 2048, 256, 4, seed=3,
              layout=LAYOUT_PAGED, block_size=16, len_range=(4096, 32768)),
    4: Config("Qwen3-32B shape, 131K chat budget (64 layers, 64q/8kv, 131072 tokens)", 64, 64, 8,
              PAIR_NEOX, 1e6, 1, 131072, 12000, 256, 0, seed=4, near_zero_frac=0.1),
}


# ---------------------------------------------------------------------------
# host-side draws
# ---------------------------------------------------------------------------
def seq_lengths(cfg: Config) -> np.ndarray:
    if cfg.seq_len > 0:
        return np.full(cfg.n_seq, cfg.seq_len, dtype=np.int64)
    lo, hi = cfg.len_range
    x = P.philox4x32_10(np.arange(cfg.n_seq), 0, 0, P.STREAM_LENGTHS, cfg.seed)[0]
    return (lo + np.floor(P.uniform01(x) * (hi - lo + 1))).astype(np.int64)


def make_stats(cfg: Config):
    """Calibrated statistics, fp32 [L][Hq][F] x 3: (E Re q, E Im q, E|q|)."""
    L, H, F = cfg.n_layers, cfg.n_q_heads, cfg.head_dim // 2
    l, h, f = np.meshgrid(np.arange(L), np.arange(H), np.arange(F), indexing="ij")
    n = P.normals4(f, h, l, P.STREAM_QMEAN, cfg.seed)
    re, im = n[0], n[1]
    ratio = P.uniform01(P.philox4x32_10(f, h, l, P.STREAM_QRATIO, cfg.seed)[0])
    am = np.hypot(re, im) * (1.0 + 0.5 * ratio)
    return re.astype(np.float32), im.astype(np.float32), am.astype(np.float32)


def calib_queries(n_tokens: int, n_q_heads: int, seed: int, layer: int = 0,
                  center_sigma: float = 1.0, noise_sigma: float = 0.7) -> np.ndarray:
    """Synthetic pre-RoPE calibration queries of one layer as bf16 bits
    [n_tokens][n_q_heads][128]: a per-(layer, head) center ~ N(0, sigma_c^2)
    per dimension plus per-token noise N(0, sigma_n^2) (concentrated bands,
    as calibrated queries are)."""
    h, j4 = np.meshgrid(np.arange(n_q_heads), np.arange(32), indexing="ij")
    c = np.stack(P.normals4(j4, h, layer, P.STREAM_QCAL_CENTER, seed), axis=-1)
    c = c.reshape(n_q_heads, 128) * center_sigma
    t, h2, j4b = np.meshgrid(np.arange(n_tokens), np.arange(n_q_heads), np.arange(32), indexing="ij")
    nz = np.stack(P.normals4(j4b, h2, t + (layer << 24), P.STREAM_QCAL_NOISE, seed), axis=-1)
    q = c[None] + nz.reshape(n_tokens, n_q_heads, 128) * noise_sigma
    return P.f32_to_bf16_bits(q.astype(np.float32))


def near_zero_heads(cfg: Config) -> np.ndarray:
    """Boolean [L][Hkv]: the (layer, KV head) pairs with near-zero centers."""
    L, Hk = cfg.n_layers, cfg.n_kv_heads
    mask = np.zeros((L, Hk), dtype=bool)
    n_pick = int(round(cfg.near_zero_frac * L * Hk))
    if n_pick:
        x = P.philox4x32_10(np.arange(L * Hk), 0, 0, P.STREAM_HEADPICK, cfg.seed)[0]
        mask.reshape(-1)[np.argsort(x, kind="stable")[:n_pick]] = True
    return mask


def make_centers(cfg: Config) -> np.ndarray:
    """Pre-RoPE key centers, fp32 [L][Hkv][128]."""
    L, Hk = cfg.n_layers, cfg.n_kv_heads
    l, h, j4 = np.meshgrid(np.arange(L), np.arange(Hk), np.arange(32), indexing="ij")
    n = P.normals4(j4, h, l, P.STREAM_KCENTER, cfg.seed)
    c = np.stack(n, axis=-1).reshape(L, Hk, 128) * cfg.center_sigma
    c[near_zero_heads(cfg)] *= 0.01
    return c.astype(np.float32)


def host_key_rows(cfg: Config, centers: np.ndarray, s: int, layer: int, h: int,
                  positions: np.ndarray) -> np.ndarray:
    """The generator's bf16 K rows (uint16 bits [n, 128]) computed on the host,
    used to check the device generator."""
    p = np.asarray(positions, dtype=np.int64)
    j4 = np.arange(32)
    n = P.normals4(p[:, None], j4[None, :] + 32 * h, layer + 256 * s, P.STREAM_KNOISE, cfg.seed)
    noise = np.stack(n, axis=-1).reshape(len(p), 128)
    pre = centers[layer, h].astype(np.float64)[None, :] + cfg.noise_sigma * noise
    post = np.empty_like(pre)
    for f in range(64):
        a, b = (f, f + 64) if cfg.pairing == PAIR_NEOX else (2 * f, 2 * f + 1)
        om = cfg.theta ** (-2.0 * f / 128.0)
        ang = om * p.astype(np.float64)
        cs, sn = np.cos(ang), np.sin(ang)
        post[:, a] = pre[:, a] * cs - pre[:, b] * sn
        post[:, b] = pre[:, a] * sn + pre[:, b] * cs
    return P.f32_to_bf16_bits(post.astype(np.float32))


def decode_queries(cfg: Config, layer: int, positions, noise: float = 0.5,
                   stream_seed: int = 0) -> np.ndarray:
    """Post-RoPE decode queries of one layer, bf16 bits [n_seq][Hq][128]: the
    pre-RoPE band f of query head qh is the calibrated center E[q_f] of
    make_stats plus complex normal noise (per part N(0, noise^2)), rotated to
    the sequence's query position with the config's pairing and theta."""
    re, im, _ = make_stats(cfg)
    pos = np.asarray(positions, dtype=np.int64)
    S, H = len(pos), cfg.n_q_heads
    s_i, h_i, f_i = np.meshgrid(np.arange(S), np.arange(H), np.arange(64), indexing="ij")
    n = P.normals4(f_i, h_i, layer + 256 * s_i, P.STREAM_DECODE_Q, cfg.seed + 977 * stream_seed)
    zr = re[layer][None].astype(np.float64) + noise * n[0]
    zi = im[layer][None].astype(np.float64) + noise * n[1]
    om = cfg.theta ** (-2.0 * np.arange(64) / 128.0)
    ang = om[None, None, :] * pos[:, None, None].astype(np.float64)
    cs, sn = np.cos(ang), np.sin(ang)
    pr, pi = zr * cs - zi * sn, zr * sn + zi * cs
    out = np.empty((S, H, 128))
    if cfg.pairing == PAIR_NEOX:
        out[..., :64], out[..., 64:] = pr, pi
    else:
        out[..., 0::2], out[..., 1::2] = pr, pi
    return P.f32_to_bf16_bits(out.astype(np.float32))


# ---------------------------------------------------------------------------
# device generator
# ---------------------------------------------------------------------------
def build(force: bool = False) -> str:
    src = os.path.join(_DIR, "csrc", "synth.cu")
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(src):
        return _LIB_PATH
    nvcc = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", "-o", _LIB_PATH + ".tmp", src]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is not built; run synth.build()")
        lib = ctypes.CDLL(_LIB_PATH)
        f = lib.synth_fill_layer
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                      ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                      ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                      ctypes.c_void_p, ctypes.c_int, ctypes.c_uint32, ctypes.c_int, ctypes.c_double,
                      ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                      ctypes.c_void_p]
        _lib = lib
    return _lib


class Workload:
    """A synthetic KV cache resident on one GPU (torch tensors), plus the
    calibrated statistics on the host."""

    def __init__(self, cfg: Config, device="cuda", capacity: int | None = None,
                 with_positions: bool = True, with_values: bool = True):
        import torch

        self.cfg = cfg
        self.device = torch.device(device)
        self.lens = seq_lengths(cfg)
        self.max_seq_len = int(capacity if capacity is not None else self.lens.max())
        assert self.max_seq_len >= int(self.lens.max())
        self.stats = make_stats(cfg)
        self.centers = make_centers(cfg)
        L, Hk, D = cfg.n_layers, cfg.n_kv_heads, cfg.head_dim
        dev = self.device
        self.block_table = None
        self.max_blocks = 0
        if cfg.layout == LAYOUT_CONTIGUOUS:
            cap = self.max_seq_len
            shape = (cfg.n_seq, Hk, cap, D)
            self.strides = dict(seq=Hk * cap * D, head=cap * D, token=D, block=0)
        else:
            bs = cfg.block_size
            nblk = (self.lens + bs - 1) // bs
            self.max_blocks = int((self.max_seq_len + bs - 1) // bs)
            total = int(nblk.sum())
            x = P.philox4x32_10(np.arange(total), 0, 0, P.STREAM_BLOCKS, cfg.seed)[0]
            perm = np.argsort(x, kind="stable").astype(np.int32)
            table = np.zeros((cfg.n_seq, self.max_blocks), dtype=np.int32)
            off = 0
            for s in range(cfg.n_seq):
                table[s, : nblk[s]] = perm[off: off + nblk[s]]
                off += nblk[s]
            self.block_table_host = table
            self.block_table = torch.from_numpy(table).to(dev)
            self.n_blocks = total
            shape = (total, bs, Hk, D)
            self.strides = dict(seq=0, head=D, token=Hk * D, block=bs * Hk * D)
        self.k = [torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(L)]
        self.v = ([torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(L)]
                  if with_values else None)
        self.seq_lens = torch.from_numpy(self.lens.astype(np.int32)).to(dev)
        self.query_pos = torch.from_numpy(self.lens.astype(np.int64) - 1).to(dev)
        self.positions = (torch.full((cfg.n_seq, L, Hk, self.max_seq_len), -1, dtype=torch.int32,
                                     device=dev) if with_positions else None)
        self._centers_dev = torch.from_numpy(self.centers).to(dev)
        self.next_pos = self.lens.astype(np.int64).copy()
        zero = np.zeros(cfg.n_seq, dtype=np.int64)
        self._fill(zero.astype(np.int32), self.lens.astype(np.int32), zero)
        torch.cuda.synchronize(dev)

    # -- generator calls -------------------------------------------------
    def _fill(self, slot0, count, pos0, stream=None):
        import torch

        lib = _load()
        cfg = self.cfg
        t_slot0 = torch.from_numpy(np.asarray(slot0, dtype=np.int32)).to(self.device)
        t_count = torch.from_numpy(np.asarray(count, dtype=np.int32)).to(self.device)
        t_pos0 = torch.from_numpy(np.asarray(pos0, dtype=np.int64)).to(self.device)
        if np.any(np.asarray(slot0) + np.asarray(count) > self.max_seq_len):
            raise ValueError("rows past the cache capacity")
        st = stream if stream is not None else torch.cuda.current_stream(self.device).cuda_stream
        mc = int(np.max(count)) if len(count) else 0
        for layer in range(cfg.n_layers):
            rc = lib.synth_fill_layer(
                self.k[layer].data_ptr(), self.v[layer].data_ptr() if self.v else None,
                cfg.layout, self.strides["seq"], self.strides["head"], self.strides["token"],
                self.strides["block"],
                self.block_table.data_ptr() if self.block_table is not None else None,
                self.max_blocks, cfg.block_size, cfg.n_seq, cfg.n_kv_heads,
                t_slot0.data_ptr(), t_count.data_ptr(), t_pos0.data_ptr(),
                self._centers_dev[layer].data_ptr(), layer, cfg.seed & 0xFFFFFFFF, cfg.pairing,
                cfg.theta, cfg.noise_sigma, mc,
                self.positions.data_ptr() if self.positions is not None else None,
                cfg.n_layers, self.max_seq_len, st)
            if rc != 0:
                raise RuntimeError(f"synth_fill_layer failed ({rc})")
        # keep the temporaries alive until the stream has consumed them
        torch.cuda.current_stream(self.device).synchronize()

    def append(self, n_new: int):
        """Decode n_new tokens per sequence: rows at the next slots and the
        next positions; seq_lens and query_pos advance (contiguous layout)."""
        import torch

        cur = self.seq_lens.cpu().numpy().astype(np.int64)
        self._fill(cur.astype(np.int32), np.full(self.cfg.n_seq, n_new, np.int32), self.next_pos)
        self.next_pos = self.next_pos + n_new
        self.seq_lens.copy_(torch.from_numpy((cur + n_new).astype(np.int32)))
        self.query_pos.copy_(torch.from_numpy(self.next_pos - 1))

    # -- host copies for the oracle ----------------------------------------
    def unit_rows(self, which: str, s: int, layer: int, h: int, n: int | None = None) -> np.ndarray:
        """uint16 bf16 bits [n, 128] of K or V rows 0..n-1 of one unit."""
        import torch

        n = int(self.seq_lens[s].item()) if n is None else n
        t = (self.k if which == "k" else self.v)[layer]
        if self.cfg.layout == LAYOUT_CONTIGUOUS:
            rows = t[s, h, :n]
        else:
            bs = self.cfg.block_size
            nb = (n + bs - 1) // bs
            blocks = self.block_table[s, :nb].long()
            rows = t[blocks, :, h].reshape(nb * bs, -1)[:n]
        return rows.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    def unit_positions(self, s: int, layer: int, h: int, n: int | None = None) -> np.ndarray:
        n = int(self.seq_lens[s].item()) if n is None else n
        return self.positions[s, layer, h, :n].cpu().numpy().astype(np.int64)

    def footprint_bytes(self) -> int:
        tot = sum(t.numel() * 2 for t in self.k)
        if self.v:
            tot += sum(t.numel() * 2 for t in self.v)
        return tot
