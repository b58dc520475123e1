"""torch front end of the PISA block selection in liblh (include/lh.h,
lh_pisa_*): a coarse-to-fine top-K over a pooled key pyramid with LSE block
scores.  Only marshalling: outputs are allocated with torch and every step
runs in the library's kernels.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import LhPisaConfig, LhPisaInfo, call


@dataclass(frozen=True)
class Pisa:
    """Shape and selection parameters (names as in lh_pisa_config)."""
    B: int
    H: int
    N: int
    d: int
    p: int
    L: int
    block: int = 64
    group: int = 128
    topk: int = 8

    def cfg(self) -> LhPisaConfig:
        return LhPisaConfig(self.B, self.H, self.N, self.d, self.p, self.L, self.block, self.group, self.topk)

    @property
    def BH(self):
        return self.B * self.H


def plan(sel: Pisa) -> LhPisaInfo:
    info = LhPisaInfo()
    call("lh_pisa_plan", ctypes.byref(sel.cfg()), ctypes.byref(info))
    return info


def _p(t):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("liblh takes contiguous CUDA tensors")
    return ctypes.c_void_p(t.data_ptr())


def _need(name: str, t, dtype, numel: int | None = None, min_numel: int | None = None):
    """Host check before a pointer reaches the library, which cannot see sizes."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: {t.numel()} elements, expected {numel}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name}: {t.numel()} elements, expected at least {min_numel}")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def pool_keys(sel: Pisa, k, kpyr=None):
    """-> the key pyramid [BH, upper_entries, d] bf16 (levels >= 1)."""
    info = plan(sel)
    _need("k", k, torch.bfloat16, numel=sel.BH * sel.N * sel.d)
    if kpyr is not None:
        _need("kpyr", kpyr, torch.bfloat16, min_numel=sel.BH * info.upper_entries * sel.d)
    if kpyr is None:
        kpyr = torch.empty((sel.BH, max(info.upper_entries, 1), sel.d), dtype=torch.bfloat16, device=k.device)
    call("lh_pisa_pool_keys", ctypes.byref(sel.cfg()), _p(k), _p(kpyr), _stream())
    return kpyr


def select(sel: Pisa, q, k, kpyr, out=None, ws=None):
    """-> kept_idx [BH, n_groups, L, topk] int32, kept_score (same, fp32); level 0 is the selection."""
    info = plan(sel)
    for name, t in (("q", q), ("k", k)):
        _need(name, t, torch.bfloat16, numel=sel.BH * sel.N * sel.d)
    _need("kpyr", kpyr, torch.bfloat16, min_numel=sel.BH * info.upper_entries * sel.d)
    n_out = sel.BH * info.n_groups * sel.L * sel.topk
    if out is not None:
        _need("kept_idx", out[0], torch.int32, numel=n_out)
        _need("kept_score", out[1], torch.float32, numel=n_out)
    if ws is not None and ws.numel() * ws.element_size() < _lib.ERR_WORD_BYTES:
        raise ValueError(f"ws: {ws.numel() * ws.element_size()} bytes, expected at least {_lib.ERR_WORD_BYTES}")
    dev = q.device
    if out is None:
        shp = (sel.BH, info.n_groups, sel.L, sel.topk)
        out = (torch.empty(shp, dtype=torch.int32, device=dev), torch.empty(shp, dtype=torch.float32, device=dev))
    if ws is None:
        ws = torch.zeros(_lib.ERR_WORD_BYTES, dtype=torch.uint8, device=dev)
    call("lh_pisa_select", ctypes.byref(sel.cfg()), _p(q), _p(k), _p(kpyr), _p(out[0]), _p(out[1]), _p(ws),
         _stream())
    return out


def block_select(sel: Pisa, q, k):
    """Both steps: the pyramid, then the selection."""
    return select(sel, q, k, pool_keys(sel, k))
