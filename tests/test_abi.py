"""The C ABI: liblh.so loads, exports every symbol include/lh.h declares, and
its host-only logic (planning, argument checks, failure paths) behaves.
No GPU is needed: every call here returns before any CUDA work is queued."""

import ctypes
import os
import re
import subprocess

import pytest

from hierarchical_sparse_attention_pyramid_b200 import _lib, plan, Layer
from hierarchical_sparse_attention_pyramid_b200.api import kernels_per_step
from hierarchical_sparse_attention_pyramid_b200.synth import WORKLOADS, Workload
from oracle import lighthouse_oracle as lo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lh.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lh_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from hierarchical_sparse_attention_pyramid_b200.build import build
        build()
    return _lib.load()


def test_header_functions_are_exported(lib):
    names = declared_functions()
    assert len(names) >= 15
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (lh_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)
    assert set(names) == set(_lib.SIGNATURES)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_plan_matches_oracle_sizes(lib, name):
    w = WORKLOADS[name]
    info = plan(Layer.of(w))
    assert info.S == lo.gathered_length(w.N, w.p, w.L, w.k)
    assert info.pyr_entries == lo.pyramid_entry_count(w.N, w.p, w.L)
    assert list(info.kprime)[: w.L - 1] == lo.budgets(w.N, w.p, w.L, w.k)
    assert info.ctx_bytes > 0 and info.ws_bytes > 0
    for f in ("ctx_off_sel", "ctx_off_qs", "ctx_off_lse", "ws_off_pyr_q", "ws_off_dqs"):
        assert getattr(info, f) % 256 == 0
    # the lowest level lh_forward writes: the first level below the top whose
    # N/p^l rows cost no more than the p^(l+1) k' level-0 rows its kept
    # entries would read back, else the top level
    want = max(1, w.L - 1)
    for lvl, kp in enumerate(lo.budgets(w.N, w.p, w.L, w.k)):
        if 1 <= lvl and w.N // w.p ** lvl <= w.p ** (lvl + 1) * kp:
            want = lvl
            break
    assert info.first_level == want


@pytest.mark.parametrize("selection", ["direct", "nested"])
def test_plan_of_the_other_readings(lib, selection):
    for N, p, L, k in ((8192, 2, 4, 48), (8192, 2, 5, 40), (1 << 16, 4, 5, 300), (4096, 2, 3, 5000)):
        w = Workload("r", 1, 2, N, 64, L, p, k, "bf16", "qk_sum", "iid", 0, selection=selection)
        info = plan(Layer.of(w))
        kp = lo.budgets(N, p, L, k, selection)
        assert list(info.kprime)[: L - 1] == kp
        assert info.S == lo.gathered_length(N, p, L, k, selection)
        assert info.sel_per_head == sum(kp) * (p if selection == "direct" else 1)


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), 2),            # unsupported head dim
    (dict(p=3), 2),             # p not a power of two
    (dict(N=1000, L=5), 2),     # N not divisible by p^(L-1)
    (dict(L=9), 2),             # more levels than the kernels take
    (dict(k=0), 1),             # invalid budget
    (dict(chunk=-5), 1),        # negative chunk
    (dict(dtype=7), 1),         # bad enum
    (dict(selection=3), 1),     # bad enum
])
def test_plan_rejects(lib, kw, status):
    base = dict(B=1, H=2, N=4096, d=128, L=3, p=2, k=16, chunk=0, dtype=0, scorer=0, selection=0)
    base.update(kw)
    cfg = _lib.LhConfig(**base)
    info = _lib.LhPlanInfo()
    assert lib.lh_plan(ctypes.byref(cfg), ctypes.byref(info)) == status
    assert lib.lh_last_error_message().decode()


def test_failure_paths_return_before_any_gpu_work(lib):
    cfg = _lib.LhConfig(1, 1, 4096, 64, 3, 2, 256, 0, 1, 0)
    info = _lib.LhPlanInfo()
    assert lib.lh_plan(ctypes.byref(cfg), ctypes.byref(info)) == 0
    fake = ctypes.c_void_p(1 << 40)  # never dereferenced: every check below fails first
    mis = ctypes.c_void_p((1 << 40) + 8)
    # misaligned pointer
    assert lib.lh_pyramid_pool(ctypes.byref(cfg), mis, fake, fake, fake, fake, fake, fake, None) == 1
    # NULL pointer
    assert lib.lh_scatter_back(ctypes.byref(cfg), None, fake, fake, None) == 1
    # workspace too small
    assert lib.lh_forward(ctypes.byref(cfg), fake, fake, fake, fake, fake, info.ctx_bytes - 1, fake,
                          info.ws_bytes, None) == 3
    assert lib.lh_backward(ctypes.byref(cfg), fake, fake, info.ctx_bytes, fake, fake, fake, fake,
                           info.ws_bytes - 1, None) == 3
    # first_level outside [1, L-1]
    for first in (0, 3):
        assert lib.lh_pyramid_pool_from(ctypes.byref(cfg), first, fake, fake, fake, fake, fake, fake, fake,
                                        None) == 1
        assert lib.lh_gather_from(ctypes.byref(cfg), first, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                  fake, fake, fake, None) == 1
    # unsupported head dim in the attention stage
    bad = _lib.LhConfig(1, 1, 4096, 80, 3, 2, 256, 0, 0, 0)
    assert lib.lh_attn_fwd(ctypes.byref(bad), 100, fake, fake, fake, fake, fake, fake, None) == 2


def test_shard_and_window_calls_reject_bad_arguments_before_any_launch(lib):
    """The context-parallel entry points refuse, on the host, token windows
    that split a top-level block, row windows that are not tile-aligned,
    segment sizes out of range, unsupported layouts and missing pointers; an
    empty attention window is a successful no-op.  No case reaches a launch."""
    cfg = _lib.LhConfig(1, 2, 4096, 128, 3, 2, 16, 0, 0, 0, 0)  # bf16, p^(L-1) = 4
    info = _lib.LhPlanInfo()
    assert lib.lh_plan(ctypes.byref(cfg), ctypes.byref(info)) == 0
    S = info.S
    fake = ctypes.c_void_p(1 << 40)  # never dereferenced
    I64 = ctypes.c_int64

    def gather(t0, t1, seg_off, seg_rows):
        return lib.lh_gather_shard(ctypes.byref(cfg), I64(t0), I64(t1), seg_off, I64(seg_rows), *([fake] * 12), None)

    assert gather(2, 2050, fake, 10) == 1       # t0 inside a top-level block
    assert gather(0, 4100, fake, 10) == 1       # past N
    assert gather(2048, 2048, fake, 10) == 1    # empty shard
    assert gather(0, 2048, fake, 0) == 1        # no segment rows
    assert gather(0, 2048, fake, S + 1) == 1    # more rows than the whole sequence
    assert gather(0, 2048, None, 10) == 1       # no segment offsets
    assert "lh_gather_shard" in lib.lh_last_error_message().decode()

    def fwd(lo, hi):
        return lib.lh_attn_fwd_rows(ctypes.byref(cfg), I64(S), I64(lo), I64(hi), *([fake] * 6), None)

    assert fwd(64, 256) == 1       # lo not on a tile edge
    assert fwd(0, S + 128) == 1    # past S
    assert fwd(256, 128) == 1      # reversed
    assert fwd(0, 1000) == 1       # hi neither on a tile edge nor S
    assert fwd(256, 256) == 0      # empty: nothing to do

    def bwd(qlo, qhi, klo, khi):
        return lib.lh_attn_bwd_rows(ctypes.byref(cfg), I64(S), I64(qlo), I64(qhi), I64(klo), I64(khi),
                                    *([fake] * 10), None)

    assert bwd(64, 128, 0, 0) == 1
    assert bwd(0, 0, 0, 1000) == 1
    assert bwd(128, 128, 0, 0) == 0

    shard = _lib.LhConfig(1, 2, 2048, 128, 3, 2, 16, 0, 0, 0, 0)  # one shard's layer
    assert lib.lh_scatter_back_shard(ctypes.byref(shard), I64(0), fake, fake, fake, fake, None) == 1
    assert lib.lh_scatter_back_shard(ctypes.byref(shard), I64(10), fake, fake, None, fake, None) == 1  # no halo
    narrow = _lib.LhConfig(1, 2, 2048, 64, 3, 2, 16, 0, 0, 0, 0)
    assert lib.lh_scatter_back_shard(ctypes.byref(narrow), I64(10), fake, fake, fake, fake, None) == 2
    assert lib.lh_scatter_back_adjoint_shard(ctypes.byref(shard), I64(1 << 31), *([fake] * 6), None) == 1
    assert lib.lh_scatter_back_adjoint_shard(ctypes.byref(shard), I64(10), None, *([fake] * 5), None) == 1
    assert lib.lh_pool_adjoint_shard(ctypes.byref(shard), I64(-1), *([fake] * 7), None) == 1
    assert lib.lh_pool_adjoint_shard(ctypes.byref(shard), I64(10), fake, fake, fake, None, fake, fake, fake,
                                     None) == 1
    assert lib.lh_head_sums(ctypes.byref(shard), None, fake, None) == 1


def test_status_strings(lib):
    for s in range(7):
        assert lib.lh_status_string(s).decode()
    assert lib.lh_status_string(99).decode() == "unknown status"


# ---------------------------------------------------------------- PISA selection

def _pisa_cfg(**kw):
    base = dict(B=1, H=2, N=8192, d=128, p=4, L=3, block=64, group=128, topk=8)
    base.update(kw)
    return _lib.LhPisaConfig(**base)


@pytest.mark.parametrize("name", ["pisa_small_8k", "pisa_128k", "pisa_256k"])
def test_pisa_plan_matches_oracle_sizes(lib, name):
    from hierarchical_sparse_attention_pyramid_b200.synth import PISA_WORKLOADS
    from oracle import pisa_oracle as po
    w = PISA_WORKLOADS[name]
    info = _lib.LhPisaInfo()
    cfg = _pisa_cfg(B=w.B, H=w.H, N=w.N, d=w.d, p=w.p, L=w.L, block=w.block, group=w.group, topk=w.topk)
    assert lib.lh_pisa_plan(ctypes.byref(cfg), ctypes.byref(info)) == 0
    assert list(info.blocks)[: w.L] == po.level_blocks(w.N, w.p, w.L, w.block)
    assert info.n_groups == w.N // w.group
    assert info.upper_entries == sum(w.N // w.p ** l for l in range(1, w.L))
    assert info.pyr_bytes == w.B * w.H * info.upper_entries * w.d * 2
    assert info.kept_elems == w.B * w.H * info.n_groups * w.L * w.topk
    assert info.max_candidates == max(po.level_blocks(w.N, w.p, w.L, w.block)[-1], w.p * w.topk)
    off = 0
    for lv in range(1, w.L):
        assert info.level_off[lv] == off
        off += w.N // w.p ** lv


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), 2), (dict(block=32), 2), (dict(group=64), 2), (dict(p=3), 2), (dict(L=9), 2),
    (dict(N=8192 + 128), 2),            # not a whole number of coarsest blocks
    (dict(N=65536, L=1), 2),            # 1024 coarsest blocks > 512
    (dict(topk=200), 2),                # p * topk > 512
    (dict(topk=0), 1), (dict(N=0), 1), (dict(B=0), 1),
])
def test_pisa_plan_rejects(lib, kw, status):
    info = _lib.LhPisaInfo()
    assert lib.lh_pisa_plan(ctypes.byref(_pisa_cfg(**kw)), ctypes.byref(info)) == status
    assert lib.lh_last_error_message().decode().startswith("lh_pisa_plan")


def test_pisa_calls_reject_bad_pointers_before_any_launch(lib):
    cfg = _pisa_cfg()
    buf = ctypes.create_string_buffer(64)
    odd = ctypes.c_void_p(ctypes.addressof(buf) + 1)
    assert lib.lh_pisa_pool_keys(ctypes.byref(cfg), None, None, None) == 1
    assert lib.lh_pisa_pool_keys(ctypes.byref(cfg), odd, odd, None) == 1
    assert lib.lh_pisa_select(ctypes.byref(cfg), None, None, None, None, None, None, None) == 1
    assert lib.lh_pisa_plan(None, None) == 1


@pytest.mark.parametrize("L,p,want", [(5, 4, 10), (1, 2, 8), (3, 2, 10), (8, 2, 10), (7, 4, 11), (3, 8, 10)])
def test_kernels_per_step(L, p, want):
    """bench.py's gpu_launches claim: one pool, ceil((L-1) / (11 // log2 p))
    score-pyramid launches, one top-k, gather, attention forward and
    scatter-back; scatter adjoint, the two attention-backward kernels and the
    pool adjoint (no selection kernels at L = 1).  The 512K-token launch list
    under profiles/ shows the 10 of (L, p) = (5, 4) per step."""
    assert kernels_per_step(Layer(1, 1, 4096, 64, L, p, 1)) == want


def test_selftest_timeout_argument_checks(lib):
    # refused on the host before anything is queued
    fake = ctypes.c_void_p(1 << 40)
    assert lib.lh_selftest_wait_timeout(fake, ctypes.c_size_t(_lib.SELFTEST_WS_BYTES - 1), ctypes.c_int64(1000),
                                        None) == 3
    assert lib.lh_selftest_wait_timeout(fake, ctypes.c_size_t(_lib.SELFTEST_WS_BYTES), ctypes.c_int64(0), None) == 1
    assert lib.lh_selftest_wait_timeout(fake, ctypes.c_size_t(_lib.SELFTEST_WS_BYTES), ctypes.c_int64(5_000_000_000),
                                        None) == 1
    assert lib.lh_selftest_wait_timeout(None, ctypes.c_size_t(_lib.SELFTEST_WS_BYTES), ctypes.c_int64(1000),
                                        None) == 1


def test_no_pointer_from_a_temporary():
    """A pointer handed to the library must come from a tensor that outlives
    the call's launch: `_p(x.contiguous())` frees the copy as soon as the
    pointer is taken, and the allocator gives that memory to the next copy."""
    pkg = os.path.join(ROOT, "hierarchical_sparse_attention_pyramid_b200")
    bad = re.compile(r"\b_?p_?\([^()]*\.contiguous\(\)\)")
    hits = []
    for f in sorted(os.listdir(pkg)):
        if f.endswith(".py"):
            with open(os.path.join(pkg, f)) as fh:
                hits += [f"{f}:{i + 1}" for i, line in enumerate(fh) if bad.search(line)]
    assert not hits, hits


def test_binding_checks_tensor_sizes_and_dtypes_on_the_host():
    """The library sees only pointers, so the binding refuses tensors whose
    size or dtype does not match the layer before a pointer is passed (a
    wrong size would make a kernel read or write outside the tensor).  CPU
    tensors of the right size get past these checks and stop at the next one
    (the library takes CUDA tensors)."""
    import torch

    import hierarchical_sparse_attention_pyramid_b200 as lh

    layer = Layer(1, 2, 4096, 64, 3, 2, 16)
    info = plan(layer)
    S = info.S
    shp = (1, 2, 4096, 64)
    q, k, v, dy = (torch.zeros(shp, dtype=torch.bfloat16) for _ in range(4))
    short = torch.zeros((1, 2, 4095, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="^k: "):
        lh.forward(layer, q, short, v)
    with pytest.raises(ValueError, match="^q: dtype"):
        lh.forward(layer, q.float(), k, v)
    with pytest.raises(ValueError, match="liblh takes CUDA tensors"):
        lh.forward(layer, q, k, v)
    other = lh.Buffers(Layer(1, 2, 4096, 64, 3, 2, 8), "cpu")
    with pytest.raises(ValueError, match="another layer"):
        lh.backward(layer, dy, other)
    with pytest.raises(ValueError, match="^dy: "):
        lh.backward(layer, short, lh.Buffers(layer, "cpu"))
    with pytest.raises(ValueError, match="^norms: "):
        lh.score_topk(layer, torch.zeros((2, 2, 4095), dtype=torch.float32))
    with pytest.raises(ValueError, match="^sel: "):
        lh.gather(layer, q, k, v, *(torch.zeros((2, info.upper_entries, 64), dtype=torch.bfloat16)
                                    for _ in range(3)), torch.zeros(1, dtype=torch.int32))
    qs = torch.zeros((2, S, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="^qs: shape"):
        lh.attn_fwd(layer, torch.zeros((3, S, 64), dtype=torch.bfloat16), qs, qs)
    with pytest.raises(ValueError, match="^vs: shape"):
        lh.attn_fwd(layer, qs, qs, qs[:, :-1])
    lse = torch.zeros((2, S), dtype=torch.float32)
    with pytest.raises(ValueError, match="^dos: dtype"):
        lh.attn_bwd(layer, qs, qs, qs, lse, qs, lse)  # dOs must be fp16
    with pytest.raises(ValueError, match="^os_: shape"):
        lh.attn_fwd_rows(layer, qs, qs, qs, 0, 128, torch.zeros((2, S, 32), dtype=torch.float32))
    os_short = torch.zeros((2, S - 1, 64), dtype=torch.float32)
    seq_map = torch.zeros((2, S), dtype=torch.int32)
    with pytest.raises(ValueError, match="^os: shape"):
        lh.scatter_back_adjoint(layer, dy, seq_map, os_short)
    with pytest.raises(ValueError, match="^os: "):
        lh.scatter_back(layer, os_short, torch.zeros((2, info.pyr_entries), dtype=torch.int32))
    with pytest.raises(ValueError, match="^slot_of: "):
        lh.pool_adjoint(layer, *(torch.zeros((2, S, 64)) for _ in range(3)), torch.zeros(1, dtype=torch.int32))
    with pytest.raises(ValueError, match="^v: shape"):
        lh.lighthouse_attention(q, k, short, L=3, p=2, k_budget=16)


def test_pisa_binding_checks_sizes_and_dtypes_on_the_host():
    import torch

    from hierarchical_sparse_attention_pyramid_b200 import pisa

    s = pisa.Pisa(1, 2, 8192, 128, 4, 3)
    info = pisa.plan(s)
    k = torch.zeros((1, 2, 8192, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="^k: dtype"):
        pisa.pool_keys(s, k.float())
    with pytest.raises(ValueError, match="^k: "):
        pisa.pool_keys(s, k[:, :1])
    with pytest.raises(ValueError, match="liblh takes"):
        pisa.pool_keys(s, k)
    kp = torch.zeros((2, info.upper_entries, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="^kpyr: "):
        pisa.select(s, k, k, kp[:1])
    out = (torch.zeros((2, info.n_groups, 3, 8), dtype=torch.int32), torch.zeros((2, info.n_groups, 3, 7)))
    with pytest.raises(ValueError, match="^kept_score: "):
        pisa.select(s, k, k, kp, out)
    with pytest.raises(ValueError, match="^ws: "):
        pisa.select(s, k, k, kp, ws=torch.zeros(16, dtype=torch.uint8))
