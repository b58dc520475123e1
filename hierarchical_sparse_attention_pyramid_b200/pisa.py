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


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def pool_keys(sel: Pisa, k, kpyr=None):
    """-> the key pyramid [BH, upper_entries, d] bf16 (levels >= 1)."""
    info = plan(sel)
    if kpyr is None:
        kpyr = torch.empty((sel.BH, max(info.upper_entries, 1), sel.d), dtype=torch.bfloat16, device=k.device)
    call("lh_pisa_pool_keys", ctypes.byref(sel.cfg()), _p(k), _p(kpyr), _stream())
    return kpyr


def select(sel: Pisa, q, k, kpyr, out=None, ws=None):
    """-> kept_idx [BH, n_groups, L, topk] int32, kept_score (same, fp32); level 0 is the selection."""
    info = plan(sel)
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
