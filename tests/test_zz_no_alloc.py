"""lh_score_topk_static: the selection for callers that cannot allocate device
memory (their allocator owns every buffer, or only inputs and outputs are
handed to them).  It must give the same selected indices as lh_score_topk with
a caller-provided workspace, call after call, and must refuse configurations
whose score pyramid does not fit its fixed 16 MiB array.

This file is named so that pytest collects it last."""

import ctypes

import pytest
import torch

import hierarchical_sparse_attention_pyramid_b200 as lh
from hierarchical_sparse_attention_pyramid_b200 import _lib, synth
from hierarchical_sparse_attention_pyramid_b200.synth import Workload

# the two large parents-selection workloads, and one small workload of each
# other reading: direct selection keeps its level-0 scores after the pyramid
# inside the array; nested selection walks the levels top down in one block
CASES = {
    "lognorm_32k": synth.WORKLOADS["lognorm_32k"],
    "sparse64_512k": synth.WORKLOADS["sparse64_512k"],
    "direct_sel": Workload("direct_sel", 1, 2, 8192, 128, 4, 2, 48, "bf16", "qk_sum", "iid", 18, chunk=512,
                           selection="direct"),
    "nested_sel": Workload("nested_sel", 1, 2, 8192, 64, 5, 2, 40, "bf16", "k", "lognormal_token", 19, chunk=32,
                           selection="nested"),
}


def _static_sel(layer, norms):
    info = lh.plan(layer)
    sel = torch.full((layer.BH, max(info.sel_per_head, 1)), -7, dtype=torch.int32, device=norms.device)
    _lib.call("lh_score_topk_static", ctypes.byref(layer.cfg()), ctypes.c_void_p(norms.data_ptr()),
              ctypes.c_void_p(sel.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return sel


def test_rejects_pyramid_larger_than_the_static_array():
    # 64 heads of 1M tokens need 89 MB of scores: refused on the host, nothing launched
    layer = lh.Layer(1, 64, 1 << 20, 128, 6, 4, 1536)
    cfg = layer.cfg()
    lib = _lib.load()
    fake = ctypes.c_void_p(1 << 40)
    assert lib.lh_score_topk_static(ctypes.byref(cfg), fake, fake, None) == 2
    assert b"static scratch" in lib.lh_last_error_message()


def test_limit_counts_the_level0_scores_of_direct_selection():
    # the 512K-token, 16-head layer fits with parents selection (11.1 MB of
    # pyramid scores) but not with direct selection (plus 33.5 MB of level-0
    # scores): the limit is topk_ws_bytes minus the error word
    lib = _lib.load()
    fake = ctypes.c_void_p(1 << 40)
    w = synth.WORKLOADS["sparse64_512k"]
    for sel, fits in (("parents", True), ("direct", False)):
        layer = lh.Layer.of(w.with_(selection=sel))
        need = lh.plan(layer).topk_ws_bytes - _lib.ERR_WORD_BYTES
        assert (need <= 16 << 20) == fits
        if not fits:
            assert lib.lh_score_topk_static(ctypes.byref(layer.cfg()), fake, fake, None) == 2


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(CASES))
def test_static_matches_workspace_entry_point(name):
    w = CASES[name]
    layer = lh.Layer.of(w)
    x = synth.cuda_inputs(w, "cuda")
    _, _, _, norms = lh.pyramid_pool(layer, x["q"], x["k"], x["v"])
    want = lh.score_topk(layer, norms)
    first = _static_sel(layer, norms)
    # a second call on different scores, then the original again: the shared
    # array keeps the previous call's contents, which must not leak through
    other = _static_sel(layer, norms.flip(-1).contiguous())
    second = _static_sel(layer, norms)
    torch.cuda.synchronize()
    assert torch.equal(first, want)
    assert torch.equal(second, want)
    assert torch.equal(other, lh.score_topk(layer, norms.flip(-1).contiguous()))
