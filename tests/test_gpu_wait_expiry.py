"""The scoring kernels' bounded waits running out (needs a B200).

Every wait of the tensor-core scoring kernels on their pipeline (tile loads,
MMA results, hand-offs between warps) is bounded by
tria_params.wait_limit_ns.  A limit of 1 ns makes the first wait that is not
already satisfied run out: the kernel must set status bit 1, let its own
loads and MMAs land, free its tensor memory and return.  No barrier is left
unsatisfied on purpose and nothing faults: the waits are cut short from
inside the kernel.  A normal pass on the same device and context afterwards
must be parity-green (a block that left tensor memory allocated, or a copy
or MMA in flight, would break the later launches).
"""
from __future__ import annotations

import time

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import key_retention_scoring_b200 as T  # noqa: E402
from key_retention_scoring_b200 import build as tria_build  # noqa: E402
from tests.test_gpu_parity import full_check, load_stats  # noqa: E402

STATUS_WAIT_EXPIRED = 2


@pytest.fixture(scope="module", autouse=True)
def _built():
    tria_build.build()
    synth.build()
    yield
    torch.cuda.empty_cache()


def _expire(cfg, offset_reduce, use_score):
    w = synth.Workload(cfg)
    st = load_stats(w)
    try:
        cache = T.Cache.from_workload(w)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks, offset_reduce, wait_limit_ns=1)
        ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
        T.tria_read_device_status(ws)
        kept = torch.full((cfg.n_seq, cfg.n_layers, cfg.n_kv_heads, cfg.budget), -7,
                          dtype=torch.int32, device="cuda")
        t0 = time.monotonic()
        if use_score:
            cmax = w.max_seq_len - cfg.window - cfg.sinks
            agg = torch.empty((cfg.n_seq, cfg.n_layers, cfg.n_kv_heads, cmax), device="cuda")
            T.tria_score(st, cache, prm, 0, cfg.n_layers, agg, None, ws)
        else:
            T.tria_compress_pass(st, cache, prm, kept, ws)
        flags = T.tria_read_device_status(ws)  # synchronises the stream
        elapsed = time.monotonic() - t0
        assert flags & STATUS_WAIT_EXPIRED, f"status {flags}: no wait ran out"
        # the drains are bounded by 2 s each; an expiry returns long before
        assert elapsed < 10.0, f"{elapsed:.1f} s"
        # the flags were cleared by the read
        assert T.tria_read_device_status(ws) == 0
    finally:
        st.free()
        del w
        torch.cuda.empty_cache()


@pytest.mark.parametrize("offset_reduce,use_score", [(0, False), (0, True), (1, False)],
                         ids=["fused_pass", "score_only", "offset_max_pass"])
def test_wait_expiry_sets_status_and_returns(offset_reduce, use_score):
    _expire(synth.CONFIGS[0], offset_reduce, use_score)
    # the same context then runs a normal pass of the same shape, parity-green
    full_check(synth.CONFIGS[0], offset_reduce=offset_reduce)


def test_wait_expiry_paged_whole_block_scoring():
    # a paged batch with 8 KV heads and 16-token blocks: the scoring kernel
    # that reads whole blocks (all heads per tile)
    cfg = synth.CONFIGS[3].scaled(n_layers=1, n_seq=2, len_range=(3000, 5000))
    _expire(cfg, 0, False)
    full_check(cfg)


def test_default_limit_is_not_hit():
    cfg = synth.CONFIGS[2].scaled(n_layers=2, seq_len=4096)
    w = synth.Workload(cfg)
    st = load_stats(w)
    try:
        cache = T.Cache.from_workload(w)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks)
        ws = T.alloc_workspace(T.tria_workspace_size(st, cache, prm))
        T.tria_read_device_status(ws)
        kept = torch.empty((1, cfg.n_layers, cfg.n_kv_heads, cfg.budget), dtype=torch.int32,
                           device="cuda")
        T.tria_compress_pass(st, cache, prm, kept, ws)
        assert T.tria_read_device_status(ws) == 0
        assert np.all(kept.cpu().numpy()[..., -cfg.window:] >= 0)
    finally:
        st.free()
        del w
        torch.cuda.empty_cache()


def test_negative_limit_rejected():
    cfg = synth.CONFIGS[0]
    w = synth.Workload(cfg, with_values=False, with_positions=False)
    st = load_stats(w)
    try:
        cache = T.Cache.from_workload(w)
        with pytest.raises(T.TriaError) as ei:
            T.tria_workspace_size(st, cache, T.params(cfg.budget, cfg.window, cfg.sinks,
                                                      wait_limit_ns=-1))
        assert ei.value.status == 1
    finally:
        st.free()
