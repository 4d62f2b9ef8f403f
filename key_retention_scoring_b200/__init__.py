"""Python binding of libtria.so, the sm_100a TriAttention KV-cache
compression pass (C ABI in include/tria.h).

Argument marshalling only: every step of the pass runs in the CUDA library.
There is no CPU fallback; loading fails loudly when the library is missing.
The entry points keep the C names: tria_load_stats, tria_workspace_size,
tria_score, tria_select, tria_compact, tria_compress_pass, ...
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtria.so")

TRIA_OK = 0
STATUS_NAMES = {0: "TRIA_OK", 1: "TRIA_ERR_INVALID_ARG", 2: "TRIA_ERR_UNSUPPORTED",
                3: "TRIA_ERR_WORKSPACE", 4: "TRIA_ERR_CUDA", 5: "TRIA_ERR_OOM", 6: "TRIA_ERR_IO"}
PAIR_NEOX = 0
PAIR_INTERLEAVED = 1
LAYOUT_CONTIGUOUS = 0
LAYOUT_PAGED = 1
OFFSET_MEAN = 0
OFFSET_MAX = 1
MAX_LAYERS = 128

EXPORTS = ["tria_status_string", "tria_version", "tria_load_stats", "tria_free_stats",
           "tria_stats_desc", "tria_workspace_size", "tria_score", "tria_select", "tria_compact",
           "tria_compress_pass", "tria_read_device_status", "tria_set_pass_events",
           "tria_compress_pass_static", "tria_calib_accumulate", "tria_calib_finalize",
           "tria_layer_budgets", "tria_decode_workspace_size", "tria_decode_attention",
           "tria_write_stats_file", "tria_read_stats_file"]
STATIC_SCRATCH_BYTES = 32 * 1024 * 1024   # TRIA_STATIC_SCRATCH_BYTES


class TriaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class ModelDesc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("pairing", ctypes.c_int), ("rope_theta", ctypes.c_double),
                ("offset_log2_max", ctypes.c_int)]


class CacheView(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int), ("n_seq", ctypes.c_int), ("max_seq_len", ctypes.c_int),
                ("k_layers", ctypes.POINTER(ctypes.c_void_p)),
                ("v_layers", ctypes.POINTER(ctypes.c_void_p)),
                ("stride_seq", ctypes.c_int64), ("stride_head", ctypes.c_int64),
                ("stride_token", ctypes.c_int64), ("stride_block", ctypes.c_int64),
                ("block_table", ctypes.c_void_p), ("max_blocks_per_seq", ctypes.c_int),
                ("block_size", ctypes.c_int), ("num_blocks", ctypes.c_int64),
                ("seq_lens", ctypes.c_void_p),
                ("query_pos", ctypes.c_void_p), ("positions", ctypes.c_void_p),
                ("layer_seq_lens", ctypes.c_void_p)]


class Params(ctypes.Structure):
    _fields_ = [("budget", ctypes.c_int), ("window", ctypes.c_int), ("sinks", ctypes.c_int),
                ("offset_reduce", ctypes.c_int), ("budget_pct", ctypes.c_float),
                ("layer_budget_scales", ctypes.POINTER(ctypes.c_float)),
                ("interval", ctypes.c_int), ("wait_limit_ns", ctypes.c_int64)]


_lib = None
_VP = ctypes.c_void_p
_I = ctypes.c_int


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} missing: build it with key_retention_scoring_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    L.tria_status_string.restype = ctypes.c_char_p
    L.tria_status_string.argtypes = [_I]
    L.tria_version.restype = ctypes.c_char_p
    L.tria_version.argtypes = []
    L.tria_load_stats.argtypes = [ctypes.POINTER(ModelDesc), _VP, _VP, _VP, _VP, _VP,
                                  ctypes.POINTER(_VP)]
    L.tria_free_stats.argtypes = [_VP]
    L.tria_stats_desc.argtypes = [_VP, ctypes.POINTER(ModelDesc)]
    L.tria_workspace_size.argtypes = [_VP, ctypes.POINTER(CacheView), ctypes.POINTER(Params), _I,
                                      _I, ctypes.POINTER(ctypes.c_size_t)]
    L.tria_score.argtypes = [_VP, ctypes.POINTER(CacheView), ctypes.POINTER(Params), _I, _I, _VP,
                             _VP, _VP, ctypes.c_size_t, _VP]
    L.tria_select.argtypes = [_VP, ctypes.POINTER(CacheView), ctypes.POINTER(Params), _VP, _I, _I,
                              _VP, _VP, ctypes.c_size_t, _VP]
    L.tria_compact.argtypes = [_VP, ctypes.POINTER(CacheView), ctypes.POINTER(Params), _VP, _I, _I,
                               _VP, _VP, _VP]
    L.tria_compress_pass.argtypes = [_VP, ctypes.POINTER(CacheView), ctypes.POINTER(Params), _VP,
                                     _VP, _VP, _VP, ctypes.c_size_t, _VP]
    L.tria_read_device_status.argtypes = [_VP, _VP, ctypes.POINTER(ctypes.c_int32)]
    L.tria_set_pass_events.argtypes = [ctypes.POINTER(_VP)]
    L.tria_compress_pass_static.argtypes = [_VP, ctypes.POINTER(CacheView),
                                            ctypes.POINTER(Params), _VP, _VP, _VP, _VP, _VP]
    L.tria_calib_accumulate.argtypes = [ctypes.POINTER(ModelDesc), _VP, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_int64, _VP, _VP]
    L.tria_calib_finalize.argtypes = [ctypes.POINTER(ModelDesc), _VP, ctypes.c_int64, _VP, _VP,
                                      _VP, _VP]
    L.tria_layer_budgets.argtypes = [_VP, ctypes.POINTER(CacheView), ctypes.POINTER(Params),
                                     ctypes.POINTER(_I), ctypes.POINTER(_I)]
    L.tria_decode_workspace_size.argtypes = [_VP, ctypes.POINTER(CacheView),
                                             ctypes.POINTER(ctypes.c_size_t)]
    L.tria_decode_attention.argtypes = [_VP, ctypes.POINTER(CacheView), _I, _VP, ctypes.c_float,
                                        _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP]
    L.tria_write_stats_file.argtypes = [ctypes.c_char_p, ctypes.POINTER(ModelDesc), _VP, _VP, _VP,
                                        _VP, _VP]
    L.tria_read_stats_file.argtypes = [ctypes.c_char_p, ctypes.POINTER(ModelDesc),
                                       ctypes.POINTER(_I), ctypes.POINTER(_I), _VP, _VP, _VP, _VP,
                                       _VP]
    for name in EXPORTS:
        if name not in ("tria_status_string", "tria_version"):
            getattr(L, name).restype = _I
    _lib = L
    return L


def _check(status: int, where: str):
    if status != TRIA_OK:
        raise TriaError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    import torch

    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def tria_status_string(status: int) -> str:
    return lib().tria_status_string(status).decode()


def tria_version() -> str:
    return lib().tria_version().decode()


class Stats:
    """Owner of a tria_stats handle."""

    def __init__(self, handle: int, desc: ModelDesc):
        self.handle = handle
        self.desc = desc

    def free(self):
        if self.handle:
            _check(lib().tria_free_stats(self.handle), "tria_free_stats")
            self.handle = None


def model_desc(n_layers, n_q_heads, n_kv_heads, pairing, rope_theta, offset_log2_max=16,
               head_dim=128) -> ModelDesc:
    return ModelDesc(n_layers, n_q_heads, n_kv_heads, head_dim, pairing, float(rope_theta),
                     offset_log2_max)


def _f32(a):
    import numpy as np

    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def tria_write_stats_file(path, desc: ModelDesc, q_mean_re, q_mean_im, q_abs_mean,
                          layer_budget_scales=None, band_mask=None):
    """Save the calibrated statistics (host arrays [L][Hq][F]) in the
    library's stats file format."""
    arrs = [_f32(a) for a in (q_mean_re, q_mean_im, q_abs_mean, layer_budget_scales, band_mask)]
    n = desc.n_layers * desc.n_q_heads * (desc.head_dim // 2)
    if any(a.size != n for a in arrs[:3]):
        raise TriaError(1, "tria_write_stats_file: array sizes")
    _check(lib().tria_write_stats_file(os.fsencode(path), ctypes.byref(desc),
                                       *[None if a is None else a.ctypes.data for a in arrs]),
           "tria_write_stats_file")


def tria_read_stats_file(path):
    """(desc, q_mean_re, q_mean_im, q_abs_mean, layer_budget_scales or None,
    band_mask or None) from a stats file; arrays are numpy float32."""
    import numpy as np

    L = lib()
    desc = ModelDesc()
    sc, mk = _I(), _I()
    _check(L.tria_read_stats_file(os.fsencode(path), ctypes.byref(desc), ctypes.byref(sc),
                                  ctypes.byref(mk), None, None, None, None, None),
           "tria_read_stats_file")
    F = desc.head_dim // 2
    shape = (desc.n_layers, desc.n_q_heads, F)
    re, im, am = (np.empty(shape, np.float32) for _ in range(3))
    scales = np.empty(desc.n_layers, np.float32) if sc.value else None
    mask = np.empty(F, np.float32) if mk.value else None
    _check(L.tria_read_stats_file(os.fsencode(path), ctypes.byref(desc), None, None,
                                  re.ctypes.data, im.ctypes.data, am.ctypes.data,
                                  None if scales is None else scales.ctypes.data,
                                  None if mask is None else mask.ctypes.data),
           "tria_read_stats_file")
    return desc, re, im, am, scales, mask


def tria_load_stats(desc: ModelDesc, q_mean_re, q_mean_im, q_abs_mean, band_mask=None,
                    stream=None) -> Stats:
    """Host fp32 arrays [n_layers][n_q_heads][head_dim/2]."""
    arrs = [np.ascontiguousarray(a, dtype=np.float32) for a in (q_mean_re, q_mean_im, q_abs_mean)]
    n = desc.n_layers * desc.n_q_heads * (desc.head_dim // 2)
    for a in arrs:
        if a.size != n:
            raise ValueError("statistics must have n_layers * n_q_heads * head_dim/2 entries")
    mask = None if band_mask is None else np.ascontiguousarray(band_mask, dtype=np.float32)
    out = _VP()
    st = lib().tria_load_stats(ctypes.byref(desc), arrs[0].ctypes.data, arrs[1].ctypes.data,
                               arrs[2].ctypes.data,
                               None if mask is None else mask.ctypes.data,
                               _stream(stream), ctypes.byref(out))
    _check(st, "tria_load_stats")
    return Stats(out.value, desc)


def tria_free_stats(stats: Stats):
    stats.free()


class Cache:
    """A tria_cache_view over torch tensors (kept alive by this object)."""

    def __init__(self, layout, k_layers, v_layers, seq_lens, query_pos, max_seq_len, *,
                 stride_seq=0, stride_head=0, stride_token=128, stride_block=0,
                 block_table=None, max_blocks_per_seq=0, block_size=0, num_blocks=0,
                 positions=None, layer_seq_lens=None, n_seq=None):
        """layer_seq_lens: optional int32 [n_seq][n_layers] lengths per (sequence,
        layer); seq_lens may then be None (n_seq is taken from layer_seq_lens)."""
        self._keep = (k_layers, v_layers, seq_lens, query_pos, block_table, positions,
                      layer_seq_lens)
        n = len(k_layers)
        self._k = (_VP * n)(*[_ptr(t) for t in k_layers])
        self._v = (_VP * n)(*[_ptr(t) for t in v_layers]) if v_layers is not None else None
        if n_seq is None:
            n_seq = int(seq_lens.numel()) if seq_lens is not None else int(layer_seq_lens.shape[0])
        self.view = CacheView(
            layout, int(n_seq), int(max_seq_len),
            ctypes.cast(self._k, ctypes.POINTER(_VP)),
            ctypes.cast(self._v, ctypes.POINTER(_VP)) if self._v is not None else None,
            stride_seq, stride_head, stride_token, stride_block, _ptr(block_table),
            max_blocks_per_seq, block_size, num_blocks, _ptr(seq_lens), _ptr(query_pos),
            _ptr(positions), _ptr(layer_seq_lens))

    @classmethod
    def from_workload(cls, w, layer_seq_lens=None) -> "Cache":
        """View of a ``synth.Workload`` (optionally with lengths per (sequence,
        layer) instead of its per-sequence lengths)."""
        st = w.strides
        return cls(w.cfg.layout, w.k, w.v, None if layer_seq_lens is not None else w.seq_lens,
                   w.query_pos, w.max_seq_len,
                   stride_seq=st["seq"], stride_head=st["head"], stride_token=st["token"],
                   stride_block=st["block"], block_table=w.block_table,
                   max_blocks_per_seq=w.max_blocks, block_size=w.cfg.block_size,
                   num_blocks=getattr(w, "n_blocks", 0), positions=w.positions,
                   layer_seq_lens=layer_seq_lens, n_seq=int(w.seq_lens.numel()))


def params(budget, window, sinks, offset_reduce=0, budget_pct=0.0, layer_budget_scales=None,
           interval=0, wait_limit_ns=0) -> Params:
    """offset_reduce: OFFSET_MEAN (the published average over D) or OFFSET_MAX.
    budget_pct > 0: the budget is that percentage of the cache capacity;
    layer_budget_scales: per-layer multipliers of the budget (None: 1.0);
    interval: a unit is compressed only once it is that many rows past its budget;
    wait_limit_ns: bound of each wait of the scoring kernel (0: 2 s)."""
    prm = Params(budget, window, sinks, offset_reduce, float(budget_pct), None, int(interval),
                 int(wait_limit_ns))
    if layer_budget_scales is not None:
        arr = (ctypes.c_float * len(layer_budget_scales))(*[float(x) for x in layer_budget_scales])
        prm._scales = arr  # kept alive with the parameters
        prm.layer_budget_scales = ctypes.cast(arr, ctypes.POINTER(ctypes.c_float))
    return prm


def tria_layer_budgets(stats, cache, prm):
    """(per-layer budgets B_l as a list, kept_idx row length B_max)."""
    n = stats.desc.n_layers
    out = (_I * n)()
    row = _I()
    _check(lib().tria_layer_budgets(stats.handle, ctypes.byref(cache.view), ctypes.byref(prm),
                                    out, ctypes.byref(row)), "tria_layer_budgets")
    return list(out), row.value


def tria_workspace_size(stats: Stats, cache: Cache, prm: Params, layer0=0, layer1=None) -> int:
    layer1 = stats.desc.n_layers if layer1 is None else layer1
    out = ctypes.c_size_t()
    _check(lib().tria_workspace_size(stats.handle, ctypes.byref(cache.view), ctypes.byref(prm),
                                     layer0, layer1, ctypes.byref(out)), "tria_workspace_size")
    return out.value


def tria_score(stats, cache, prm, layer0, layer1, agg_out, scores_out, workspace, stream=None):
    _check(lib().tria_score(stats.handle, ctypes.byref(cache.view), ctypes.byref(prm), layer0,
                            layer1, _ptr(agg_out), _ptr(scores_out), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream(stream)),
           "tria_score")


def tria_select(stats, cache, prm, agg, layer0, layer1, kept_idx, workspace, stream=None):
    _check(lib().tria_select(stats.handle, ctypes.byref(cache.view), ctypes.byref(prm), _ptr(agg),
                             layer0, layer1, _ptr(kept_idx), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)),
           "tria_select")


def tria_compact(stats, cache, prm, kept_idx, layer0, layer1, freed_blocks=None, n_freed=None,
                 stream=None):
    _check(lib().tria_compact(stats.handle, ctypes.byref(cache.view), ctypes.byref(prm),
                              _ptr(kept_idx), layer0, layer1, _ptr(freed_blocks), _ptr(n_freed),
                              _stream(stream)), "tria_compact")


def tria_compress_pass(stats, cache, prm, kept_idx, workspace, freed_blocks=None, n_freed=None,
                       stream=None):
    _check(lib().tria_compress_pass(stats.handle, ctypes.byref(cache.view), ctypes.byref(prm),
                                    _ptr(kept_idx), _ptr(freed_blocks), _ptr(n_freed),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)), "tria_compress_pass")


def tria_compress_pass_static(stats, cache, prm, kept_idx=None, freed_blocks=None,
                              n_freed=None, device_status=None, stream=None):
    """tria_compress_pass with the library's fixed 32 MiB device scratch instead
    of a workspace: for callers that may not allocate device memory (an engine
    whose KV-cache pool holds all free memory, a loop that must not stall on
    cudaMalloc/cudaFree).  One scratch per device, shared by every call: calls
    that may overlap on the device race.  Make the first call on each device
    before any stream capture (it looks up the scratch address)."""
    rc = lib().tria_compress_pass_static(stats.handle, ctypes.byref(cache.view),
                                         ctypes.byref(prm), _ptr(kept_idx), _ptr(freed_blocks),
                                         _ptr(n_freed), _ptr(device_status), _stream(stream))
    if rc == 3:  # TRIA_ERR_WORKSPACE: say how much the pass needs
        need = tria_workspace_size(stats, cache, prm)
        raise TriaError(rc, f"tria_compress_pass_static: the pass needs {need} bytes of scratch, "
                            f"the static scratch holds {STATIC_SCRATCH_BYTES}; use "
                            f"tria_compress_pass with a workspace")
    _check(rc, "tria_compress_pass_static")


def tria_calib_accumulate(desc, q, acc, stream=None):
    """Add one batch of pre-RoPE queries q (bf16 tensor [tokens, n_q_heads,
    128], any token/head strides, unit stride inside a head) to the fp64 sums
    acc [n_q_heads, 64, 3] (zeroed by the caller before the first batch)."""
    import torch

    if q.dtype != torch.bfloat16 or q.dim() != 3 or q.stride(2) != 1:
        raise TriaError(1, "tria_calib_accumulate: q must be bf16 [tokens, heads, 128] "
                           "with unit stride inside a head")
    _check(lib().tria_calib_accumulate(ctypes.byref(desc), _ptr(q), q.shape[0], q.stride(0),
                                       q.stride(1), _ptr(acc), _stream(stream)),
           "tria_calib_accumulate")


def tria_calib_finalize(desc, acc, n_tokens, q_mean_re, q_mean_im, q_abs_mean, stream=None):
    """E[Re q_f], E[Im q_f], E|q_f| (fp32 [n_q_heads, 64] outputs) from the sums."""
    _check(lib().tria_calib_finalize(ctypes.byref(desc), _ptr(acc), int(n_tokens), _ptr(q_mean_re),
                                     _ptr(q_mean_im), _ptr(q_abs_mean), _stream(stream)),
           "tria_calib_finalize")


def tria_decode_workspace_size(stats, cache) -> int:
    out = ctypes.c_size_t()
    _check(lib().tria_decode_workspace_size(stats.handle, ctypes.byref(cache.view),
                                            ctypes.byref(out)), "tria_decode_workspace_size")
    return out.value


def tria_decode_attention(stats, cache, layer, q, scale, out, workspace, lse=None, logits=None,
                          stream=None):
    """Decode-step attention of layer `layer` over the cached rows:
    q bf16 [n_seq][n_q_heads][128] (post-RoPE), out fp32 [n_seq][n_q_heads][128];
    lse fp32 [n_seq][n_q_heads] and logits fp32 [n_seq][n_q_heads][max_seq_len]
    optional."""
    _check(lib().tria_decode_attention(stats.handle, ctypes.byref(cache.view), int(layer), _ptr(q),
                                       float(scale), _ptr(out), _ptr(lse), _ptr(logits),
                                       _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream)), "tria_decode_attention")


def tria_read_device_status(workspace, stream=None) -> int:
    out = ctypes.c_int32()
    _check(lib().tria_read_device_status(_ptr(workspace), _stream(stream), ctypes.byref(out)),
           "tria_read_device_status")
    return out.value


def alloc_workspace(nbytes: int, device="cuda"):
    """A zeroed, 256-byte aligned device buffer (torch allocations are)."""
    import torch

    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def tria_set_pass_events(events):
    """events: None or a list of 5 torch.cuda.Event (created with timing)."""
    if events is None:
        _check(lib().tria_set_pass_events(None), "tria_set_pass_events")
        return
    for e in events:
        if not e.cuda_event:   # torch creates the CUDA event on its first record
            e.record()
    arr = (_VP * 5)(*[e.cuda_event for e in events])
    _check(lib().tria_set_pass_events(arr), "tria_set_pass_events")
