"""tria_compress_pass_static (scratch in a fixed device array of the library,
no allocation) against tria_compress_pass (caller workspace), through the C
ABI on identical seeded caches.

Both calls run the same kernels on the same inputs and only the scratch
address differs, so the outputs are integers and bytes that must agree
exactly: kept slots, compacted K/V rows, positions, sequence lengths, freed
blocks.  Two calls in a row are compared (a second pass after decode appends,
and a paged batch after it), the second one also checked to leave the device's
free memory unchanged.  The file name sorts last so that the module also runs
after every other GPU test in the same process.
"""
from __future__ import annotations

import gc

import pytest

import synth

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


def _stats(w):
    cfg = w.cfg
    desc = T.model_desc(cfg.n_layers, cfg.n_q_heads, cfg.n_kv_heads, cfg.pairing, cfg.theta,
                        cfg.offset_log2_max)
    return T.tria_load_stats(desc, *w.stats)


def _outputs(w):
    return {"k": [t.clone() for t in w.k], "v": [t.clone() for t in w.v],
            "positions": w.positions.clone(), "seq_lens": w.seq_lens.clone()}


def _same(a, b, what):
    for key in ("k", "v"):
        for layer, (x, y) in enumerate(zip(a[key], b[key])):
            assert torch.equal(x.view(torch.int16), y.view(torch.int16)), f"{what}: {key}[{layer}]"
    assert torch.equal(a["positions"], b["positions"]), f"{what}: positions"
    assert torch.equal(a["seq_lens"], b["seq_lens"]), f"{what}: seq_lens"


class _Pair:
    """Two identical workloads: A for the workspace pass, B for the static one."""

    def __init__(self, cfg, **kw):
        self.a = synth.Workload(cfg, **kw)
        self.b = synth.Workload(cfg, **kw)
        self.cfg = cfg
        self.st = _stats(self.a)
        self.prm = T.params(cfg.budget, cfg.window, cfg.sinks)
        self.ca = T.Cache.from_workload(self.a)
        self.cb = T.Cache.from_workload(self.b)
        shape = (cfg.n_seq, cfg.n_layers, cfg.n_kv_heads, cfg.budget)
        self.kept_a = torch.full(shape, -7, dtype=torch.int32, device="cuda")
        self.kept_b = torch.full(shape, -9, dtype=torch.int32, device="cuda")
        self.ws = T.alloc_workspace(T.tria_workspace_size(self.st, self.ca, self.prm))
        T.tria_read_device_status(self.ws)  # clears the fresh workspace's flags
        self.status_b = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        self.freed_a = self.freed_b = self.nf_a = self.nf_b = None
        if cfg.layout == T.LAYOUT_PAGED:
            fshape = (cfg.n_seq, self.a.max_blocks)
            self.freed_a = torch.full(fshape, -1, dtype=torch.int32, device="cuda")
            self.freed_b = torch.full(fshape, -1, dtype=torch.int32, device="cuda")
            self.nf_a = torch.full((cfg.n_seq,), -1, dtype=torch.int32, device="cuda")
            self.nf_b = torch.full((cfg.n_seq,), -1, dtype=torch.int32, device="cuda")

    def run(self, what, check_no_alloc=False):
        assert T.tria_workspace_size(self.st, self.cb, self.prm) <= T.STATIC_SCRATCH_BYTES
        T.tria_compress_pass(self.st, self.ca, self.prm, self.kept_a, self.ws, self.freed_a,
                             self.nf_a)
        torch.cuda.synchronize()
        # no garbage collection inside the measured window: a collection could
        # free unrelated tensors and change the allocator's tally
        gc.collect()
        gc.disable()
        try:
            free0 = torch.cuda.mem_get_info()[0]
            alloc0 = torch.cuda.memory_allocated()
            T.tria_compress_pass_static(self.st, self.cb, self.prm, self.kept_b, self.freed_b,
                                        self.nf_b, self.status_b)
            torch.cuda.synchronize()
        finally:
            gc.enable()
        if check_no_alloc:
            assert torch.cuda.mem_get_info()[0] == free0, f"{what}: device memory changed"
            assert torch.cuda.memory_allocated() == alloc0
        assert T.tria_read_device_status(self.ws) == 0
        assert int(self.status_b.item()) == 0, f"{what}: device status"
        assert torch.equal(self.kept_a, self.kept_b), f"{what}: kept slots"
        _same(_outputs(self.a), _outputs(self.b), what)
        if self.nf_a is not None:
            assert torch.equal(self.nf_a, self.nf_b), f"{what}: freed block counts"
            assert torch.equal(self.freed_a, self.freed_b), f"{what}: freed blocks"
            assert int(self.nf_a.sum()) > 0

    def close(self):
        self.st.free()


def test_static_pass_matches_workspace_pass_two_calls():
    # contiguous Qwen3-32B-shaped heads: a pass, 640 decode steps, a second pass
    cfg = synth.CONFIGS[2].scaled(n_layers=2, seq_len=4096)
    p = _Pair(cfg, capacity=4096)
    try:
        p.run("first call")
        assert int(p.b.seq_lens[0]) == cfg.budget
        p.a.append(640)
        p.b.append(640)
        p.run("second call", check_no_alloc=True)
    finally:
        p.close()
    # then a paged batch of ragged sequences (sinks kept, blocks freed)
    cfg3 = synth.CONFIGS[3].scaled(n_layers=1, n_seq=4, len_range=(3000, 9000))
    q = _Pair(cfg3)
    try:
        q.run("paged call", check_no_alloc=True)
    finally:
        q.close()


def test_static_pass_rejects_passes_beyond_the_scratch():
    # 4 layers of one 32K-token sequence need more than 32 MiB of scratch
    cfg = synth.CONFIGS[2].scaled(n_layers=4)
    w = synth.Workload(cfg, with_positions=False)
    st = _stats(w)
    try:
        cache = T.Cache.from_workload(w)
        prm = T.params(cfg.budget, cfg.window, cfg.sinks)
        need = T.tria_workspace_size(st, cache, prm)
        assert need > T.STATIC_SCRATCH_BYTES
        lens0 = w.seq_lens.clone()
        with pytest.raises(T.TriaError, match="static scratch holds") as ei:
            T.tria_compress_pass_static(st, cache, prm)
        assert ei.value.status == 3
        torch.cuda.synchronize()
        assert torch.equal(w.seq_lens, lens0)  # nothing ran
    finally:
        st.free()
