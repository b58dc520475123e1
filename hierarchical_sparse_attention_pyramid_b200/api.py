"""torch front end of liblh: marshals CUDA tensors into the C ABI calls.

Every function allocates its outputs with torch (device memory) and passes
raw pointers and the current CUDA stream to liblh; all arithmetic runs in the
library's kernels.  Shapes follow include/lh.h: Q, K, V, Y and their
gradients are [B, H, N, d]; the gathered sequence tensors are [B*H, S, d].
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import LhConfig, LhPlanInfo, call

_TORCH_DTYPE = {"bf16": torch.bfloat16, "fp32": torch.float32}


@dataclass(frozen=True)
class Layer:
    """Shape and method parameters of one Lighthouse attention layer."""
    B: int
    H: int
    N: int
    d: int
    L: int
    p: int
    k: int
    chunk: int = 2048
    dtype: str = "bf16"
    scorer: str = "qk_sum"
    selection: str = "parents"

    def cfg(self) -> LhConfig:
        return LhConfig(self.B, self.H, self.N, self.d, self.L, self.p, self.k, self.chunk,
                        _lib.DTYPES[self.dtype], _lib.SCORERS[self.scorer], _lib.SELECTIONS[self.selection])

    @property
    def torch_dtype(self):
        return _TORCH_DTYPE[self.dtype]

    @property
    def BH(self):
        return self.B * self.H

    @staticmethod
    def of(w) -> "Layer":
        """From a synth.Workload (or anything with the same fields)."""
        return Layer(w.B, w.H, w.N, w.d, w.L, w.p, w.k, w.chunk, w.dtype, w.scorer,
                     getattr(w, "selection", "parents"))


def plan(layer: Layer) -> LhPlanInfo:
    info = LhPlanInfo()
    call("lh_plan", ctypes.byref(layer.cfg()), ctypes.byref(info))
    return info


def _p(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("liblh takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("liblh takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _need(name: str, t, dtype=None, numel: int | None = None, min_numel: int | None = None, shape=None):
    """Host check of a tensor argument before its pointer reaches the library,
    which cannot see sizes: a wrong size would make a kernel read or write
    outside the tensor."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name}: {t.numel()} elements, expected {numel}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name}: {t.numel()} elements, expected at least {min_numel}")


def _need_qkv(layer: "Layer", **ts) -> None:
    """Token-major tensors of the layer: B*H*N*d elements ([B, H, N, d] or [B*H, N, d]) in the layer's dtype."""
    for name, t in ts.items():
        _need(name, t, layer.torch_dtype, numel=layer.BH * layer.N * layer.d)


def _need_seq(layer: "Layer", qs, **ts) -> int:
    """Sequence tensors: qs [B*H, S, d] bf16 (S from qs), the others of the same
    rows: name -> (tensor, dtype, trailing dims).  Returns S."""
    if not isinstance(qs, torch.Tensor) or qs.dim() != 3 or qs.shape[0] != layer.BH or qs.shape[2] != layer.d:
        raise ValueError(f"qs: shape {tuple(getattr(qs, 'shape', ()))}, expected ({layer.BH}, S, {layer.d})")
    _need("qs", qs, torch.bfloat16)
    S = qs.shape[1]
    for name, (t, dtype, tail) in ts.items():
        _need(name, t, dtype, shape=(layer.BH, S) + tail)
    return S


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.zeros(max(nbytes, _lib.ERR_WORD_BYTES), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ stages

def pyramid_pool(layer: Layer, q, k, v, first_level: int | None = None):
    """-> pyr_q, pyr_k, pyr_v [BH, upper_entries, d] (levels >= 1), norms [2, BH, N] fp32.
    With first_level (lh_pyramid_pool_from), levels below it are not written (rows left zero here)."""
    _need_qkv(layer, q=q, k=k, v=v)
    info = plan(layer)
    dev = q.device
    shp = (layer.BH, max(info.upper_entries, 1), layer.d)
    mk = torch.zeros if first_level is not None else _empty
    pq, pk, pv = (mk(shp, dtype=layer.torch_dtype, device=dev) for _ in range(3))
    norms = _empty((2, layer.BH, layer.N), torch.float32, dev)
    if first_level is None:
        call("lh_pyramid_pool", ctypes.byref(layer.cfg()), _p(q), _p(k), _p(v), _p(pq), _p(pk), _p(pv), _p(norms),
             _stream())
    else:
        call("lh_pyramid_pool_from", ctypes.byref(layer.cfg()), ctypes.c_int32(first_level), _p(q), _p(k), _p(v),
             _p(pq), _p(pk), _p(pv), _p(norms), _stream())
    return pq, pk, pv, norms


def score_topk(layer: Layer, norms, ws=None):
    """-> sel [BH, sel_per_head] int32 (per level l at sel_off[l], ascending parents at level l+1)."""
    _need("norms", norms, torch.float32, numel=2 * layer.BH * layer.N)
    info = plan(layer)
    if ws is not None and ws.numel() * ws.element_size() < max(info.topk_ws_bytes, _lib.ERR_WORD_BYTES):
        raise ValueError(f"ws: {ws.numel() * ws.element_size()} bytes, expected at least {info.topk_ws_bytes}")
    dev = norms.device
    sel = torch.zeros((layer.BH, max(info.sel_per_head, 1)), dtype=torch.int32, device=dev)
    ws = _ws(info.topk_ws_bytes, dev) if ws is None else ws
    call("lh_score_topk", ctypes.byref(layer.cfg()), _p(norms), _p(ws), _p(sel), _stream())
    return sel


def gather(layer: Layer, q, k, v, pq, pk, pv, sel, first_level: int | None = None):
    """-> qs, ks, vs [BH, S, d] bf16, seq_map [BH, S] int32, slot_of [BH, pyr_entries] int32.
    With first_level (lh_gather_from), kept entries of the levels below it are averaged from q, k, v."""
    _need_qkv(layer, q=q, k=k, v=v)
    info = plan(layer)
    for name, t in (("pq", pq), ("pk", pk), ("pv", pv)):
        _need(name, t, layer.torch_dtype, min_numel=layer.BH * info.upper_entries * layer.d)
    _need("sel", sel, torch.int32, min_numel=layer.BH * info.sel_per_head)
    dev = q.device
    S = info.S
    qs, ks, vs = (_empty((layer.BH, S, layer.d), torch.bfloat16, dev) for _ in range(3))
    seq_map = _empty((layer.BH, S), torch.int32, dev)
    slot_of = _empty((layer.BH, info.pyr_entries), torch.int32, dev)
    if first_level is None:
        call("lh_gather", ctypes.byref(layer.cfg()), _p(q), _p(k), _p(v), _p(pq), _p(pk), _p(pv), _p(sel),
             _p(qs), _p(ks), _p(vs), _p(seq_map), _p(slot_of), _stream())
    else:
        call("lh_gather_from", ctypes.byref(layer.cfg()), ctypes.c_int32(first_level), _p(q), _p(k), _p(v), _p(pq),
             _p(pk), _p(pv), _p(sel), _p(qs), _p(ks), _p(vs), _p(seq_map), _p(slot_of), _stream())
    return qs, ks, vs, seq_map, slot_of


def attn_fwd(layer: Layer, qs, ks, vs, ws=None):
    """Causal attention over the sequence -> os [BH, S, d] fp32, lse [BH, S] fp32."""
    _need_seq(layer, qs, ks=(ks, torch.bfloat16, (layer.d,)), vs=(vs, torch.bfloat16, (layer.d,)))
    BH, S, d = qs.shape
    os_ = _empty((BH, S, d), torch.float32, qs.device)
    lse = _empty((BH, S), torch.float32, qs.device)
    ws = _ws(0, qs.device) if ws is None else ws
    call("lh_attn_fwd", ctypes.byref(layer.cfg()), ctypes.c_int64(S), _p(qs), _p(ks), _p(vs), _p(os_), _p(lse),
         _p(ws), _stream())
    return os_, lse


def attn_bwd(layer: Layer, qs, ks, vs, lse, dos, delta, ws=None):
    """-> dqs, dks, dvs [BH, S, d] fp32.  dos: fp16 holding bf16 values."""
    _need_seq(layer, qs, ks=(ks, torch.bfloat16, (layer.d,)), vs=(vs, torch.bfloat16, (layer.d,)),
              lse=(lse, torch.float32, ()), dos=(dos, torch.float16, (layer.d,)), delta=(delta, torch.float32, ()))
    BH, S, d = qs.shape
    dqs, dks, dvs = (_empty((BH, S, d), torch.float32, qs.device) for _ in range(3))
    ws = _ws(0, qs.device) if ws is None else ws
    call("lh_attn_bwd", ctypes.byref(layer.cfg()), ctypes.c_int64(S), _p(qs), _p(ks), _p(vs), _p(lse), _p(dos),
         _p(delta), _p(dqs), _p(dks), _p(dvs), _p(ws), _stream())
    return dqs, dks, dvs


def attn_fwd_rows(layer: Layer, qs, ks, vs, row_lo: int, row_hi: int, os_=None, lse=None, ws=None):
    """Rows [row_lo, row_hi) of attn_fwd's os and lse, written into os_ [BH, S, d]
    and lse [BH, S] (allocated when None; other rows left as they are)."""
    out = {} if os_ is None else dict(os_=(os_, torch.float32, (layer.d,)))
    if lse is not None:
        out["lse"] = (lse, torch.float32, ())
    _need_seq(layer, qs, ks=(ks, torch.bfloat16, (layer.d,)), vs=(vs, torch.bfloat16, (layer.d,)), **out)
    BH, S, d = qs.shape
    os_ = _empty((BH, S, d), torch.float32, qs.device) if os_ is None else os_
    lse = _empty((BH, S), torch.float32, qs.device) if lse is None else lse
    ws = _ws(0, qs.device) if ws is None else ws
    call("lh_attn_fwd_rows", ctypes.byref(layer.cfg()), ctypes.c_int64(S), ctypes.c_int64(row_lo),
         ctypes.c_int64(row_hi), _p(qs), _p(ks), _p(vs), _p(os_), _p(lse), _p(ws), _stream())
    return os_, lse


def attn_bwd_rows(layer: Layer, qs, ks, vs, lse, dos, delta, q_rows, k_rows, dqs=None, dks=None, dvs=None, ws=None):
    """dqs rows q_rows = (lo, hi) and dks, dvs rows k_rows of attn_bwd, written into
    [BH, S, d] fp32 buffers (allocated when None; other rows left as they are)."""
    out = {n: (t, torch.float32, (layer.d,)) for n, t in (("dqs", dqs), ("dks", dks), ("dvs", dvs)) if t is not None}
    _need_seq(layer, qs, ks=(ks, torch.bfloat16, (layer.d,)), vs=(vs, torch.bfloat16, (layer.d,)),
              lse=(lse, torch.float32, ()), dos=(dos, torch.float16, (layer.d,)), delta=(delta, torch.float32, ()),
              **out)
    BH, S, d = qs.shape
    dqs, dks, dvs = (_empty((BH, S, d), torch.float32, qs.device) if t is None else t for t in (dqs, dks, dvs))
    ws = _ws(0, qs.device) if ws is None else ws
    call("lh_attn_bwd_rows", ctypes.byref(layer.cfg()), ctypes.c_int64(S), ctypes.c_int64(q_rows[0]),
         ctypes.c_int64(q_rows[1]), ctypes.c_int64(k_rows[0]), ctypes.c_int64(k_rows[1]), _p(qs), _p(ks), _p(vs),
         _p(lse), _p(dos), _p(delta), _p(dqs), _p(dks), _p(dvs), _p(ws), _stream())
    return dqs, dks, dvs


def scatter_back(layer: Layer, os_, slot_of):
    info = plan(layer)
    _need("os", os_, torch.float32, numel=layer.BH * info.S * layer.d)
    _need("slot_of", slot_of, torch.int32, min_numel=layer.BH * info.pyr_entries)
    y = _empty((layer.B, layer.H, layer.N, layer.d), layer.torch_dtype, os_.device)
    call("lh_scatter_back", ctypes.byref(layer.cfg()), _p(os_), _p(slot_of), _p(y), _stream())
    return y


def scatter_back_adjoint(layer: Layer, dy, seq_map, os_):
    info = plan(layer)
    _need_qkv(layer, dy=dy)
    _need("os", os_, torch.float32, shape=(layer.BH, info.S, layer.d))
    _need("seq_map", seq_map, torch.int32, min_numel=layer.BH * info.S)
    BH, S, d = os_.shape
    dos = _empty((BH, S, d), torch.float16, dy.device)  # bf16-rounded values, stored as fp16
    delta = _empty((BH, S), torch.float32, dy.device)
    call("lh_scatter_back_adjoint", ctypes.byref(layer.cfg()), _p(dy), _p(seq_map), _p(os_), _p(dos), _p(delta),
         _stream())
    return dos, delta


def pool_adjoint(layer: Layer, dqs, dks, dvs, slot_of):
    info = plan(layer)
    for name, t in (("dqs", dqs), ("dks", dks), ("dvs", dvs)):
        _need(name, t, torch.float32, numel=layer.BH * info.S * layer.d)
    _need("slot_of", slot_of, torch.int32, min_numel=layer.BH * info.pyr_entries)
    shp = (layer.B, layer.H, layer.N, layer.d)
    dq, dk, dv = (_empty(shp, layer.torch_dtype, dqs.device) for _ in range(3))
    call("lh_pool_adjoint", ctypes.byref(layer.cfg()), _p(dqs), _p(dks), _p(dvs), _p(slot_of), _p(dq), _p(dk),
         _p(dv), _stream())
    return dq, dk, dv


# ------------------------------------------------------------------ whole layer

def kernels_per_step(layer: Layer) -> int:
    """liblh kernel launches of one lh_forward + lh_backward (memsets excluded):
    pool, score pyramid (one launch per 11/log2(p) levels), top-k, gather,
    attention forward, scatter-back; scatter adjoint, attention backward (two
    kernels: dK/dV and dQ), pool adjoint.  With L = 1 there is no selection
    (no score pyramid or top-k)."""
    if layer.L == 1:
        return 8
    log2p = layer.p.bit_length() - 1
    per_launch = 11 // log2p
    return 9 + -(-(layer.L - 1) // per_launch)


class Buffers:
    """Saved context and scratch of one layer shape, reusable across steps."""

    def __init__(self, layer: Layer, device):
        self.layer = layer
        self.info = plan(layer)
        self.ctx = torch.empty(self.info.ctx_bytes, dtype=torch.uint8, device=device)
        self.ws = torch.zeros(self.info.ws_bytes, dtype=torch.uint8, device=device)

    def ctx_views(self) -> dict:
        """Typed views of what lh_forward saved (for inspection and tests)."""
        I, Lr = self.info, self.layer
        S, BH, d = I.S, Lr.BH, Lr.d

        def view(off, n, dtype, shape):
            esz = torch.empty((), dtype=dtype).element_size()
            return self.ctx[off:off + n * esz].view(dtype).view(shape)

        return dict(
            sel=view(I.ctx_off_sel, BH * I.sel_per_head, torch.int32, (BH, I.sel_per_head)),
            seq_map=view(I.ctx_off_seq_map, BH * S, torch.int32, (BH, S)),
            slot_of=view(I.ctx_off_slot_of, BH * I.pyr_entries, torch.int32, (BH, I.pyr_entries)),
            qs=view(I.ctx_off_qs, BH * S * d, torch.bfloat16, (BH, S, d)),
            ks=view(I.ctx_off_ks, BH * S * d, torch.bfloat16, (BH, S, d)),
            vs=view(I.ctx_off_vs, BH * S * d, torch.bfloat16, (BH, S, d)),
            os=view(I.ctx_off_os, BH * S * d, torch.float32, (BH, S, d)),
            lse=view(I.ctx_off_lse, BH * S, torch.float32, (BH, S)),
        )


def forward(layer: Layer, q, k, v, bufs: Buffers | None = None, y=None):
    """Whole forward -> (y, bufs).  bufs holds the saved context for backward."""
    _need_qkv(layer, q=q, k=k, v=v)
    if y is not None:
        _need_qkv(layer, y=y)
    if bufs is not None and bufs.layer != layer:
        raise ValueError("bufs were planned for another layer")
    bufs = Buffers(layer, q.device) if bufs is None else bufs
    y = _empty((layer.B, layer.H, layer.N, layer.d), layer.torch_dtype, q.device) if y is None else y
    call("lh_forward", ctypes.byref(layer.cfg()), _p(q), _p(k), _p(v), _p(y), _p(bufs.ctx),
         ctypes.c_size_t(bufs.info.ctx_bytes), _p(bufs.ws), ctypes.c_size_t(bufs.info.ws_bytes), _stream())
    return y, bufs


def backward(layer: Layer, dy, bufs: Buffers, grads=None):
    """Whole backward from the saved context -> (dq, dk, dv)."""
    _need_qkv(layer, dy=dy)
    if bufs.layer != layer:
        raise ValueError("bufs were saved by a forward of another layer")
    if grads is not None:
        _need_qkv(layer, dq=grads[0], dk=grads[1], dv=grads[2])
    shp = (layer.B, layer.H, layer.N, layer.d)
    if grads is None:
        grads = tuple(_empty(shp, layer.torch_dtype, dy.device) for _ in range(3))
    dq, dk, dv = grads
    call("lh_backward", ctypes.byref(layer.cfg()), _p(dy), _p(bufs.ctx), ctypes.c_size_t(bufs.info.ctx_bytes),
         _p(dq), _p(dk), _p(dv), _p(bufs.ws), ctypes.c_size_t(bufs.info.ws_bytes), _stream())
    return dq, dk, dv


def check_error(bufs_or_ws) -> None:
    """Synchronise and raise if a kernel reported a timeout, a bad index, or a
    value beyond the fp16 range where the backward keeps one (dOs, Vs)."""
    ws = bufs_or_ws.ws if isinstance(bufs_or_ws, Buffers) else bufs_or_ws
    call("lh_check_error", _p(ws), _stream())


class LighthouseAttentionFn(torch.autograd.Function):
    """Autograd wrapper: forward saves liblh's context, backward consumes it.
    The top-k selection is not differentiable; gradients reach Q, K, V only
    through the pooled values."""

    @staticmethod
    def forward(fn_ctx, q, k, v, layer: Layer):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        y, bufs = forward(layer, q, k, v)
        fn_ctx.layer = layer
        fn_ctx.bufs = bufs
        return y

    @staticmethod
    def backward(fn_ctx, dy):
        dq, dk, dv = backward(fn_ctx.layer, dy.contiguous(), fn_ctx.bufs)
        return dq, dk, dv, None


def lighthouse_attention(q, k, v, L: int, p: int, k_budget: int, chunk: int = 2048, scorer: str = "qk_sum",
                         selection: str = "parents"):
    """One Lighthouse attention layer over causal q, k, v of shape [B, H, N, d]."""
    if q.dim() != 4:
        raise ValueError(f"q: shape {tuple(q.shape)}, expected [B, H, N, d]")
    B, H, N, d = q.shape
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError(f"q: dtype {q.dtype}, expected bfloat16 or float32")
    for name, t in (("k", k), ("v", v)):
        _need(name, t, q.dtype, shape=q.shape)
    dtype = {torch.bfloat16: "bf16", torch.float32: "fp32"}[q.dtype]
    layer = Layer(B, H, N, d, L, p, k_budget, chunk, dtype, scorer, selection)
    return LighthouseAttentionFn.apply(q, k, v, layer)
