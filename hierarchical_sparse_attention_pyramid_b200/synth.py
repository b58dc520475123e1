"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no arithmetic of the attention method: it only draws
Q, K, V and the upstream gradient dY with the stated distribution and
structure.  It serves both the fp64 oracle (through the tests) and the CUDA
path (through the tests and ``bench.py``).

Two generators, both seeded:
  * ``head_inputs``  - CPU, one (batch, head) slice at a time, from a torch CPU
    generator per (seed, tensor, head).  Used where the oracle needs the data.
  * ``cuda_inputs``  - the full [B, H, N, d] tensors drawn on the GPU with a
    torch CUDA generator.  Used for throughput runs and for the heads of a
    full-size parity run that the oracle does not recompute.
The two do not produce the same numbers; a parity run overwrites the heads
it checks with ``head_inputs``.

Workloads (names give what they are):
  tiny_4k_fp32        B=1 H=1  N=4096    d=64  L=3 p=2 k=256  fp32 iid N(0,1)
  lognorm_32k         B=1 H=8  N=32768   d=128 L=3 p=4 k=1536 bf16, one LogNormal(0,0.5)
                      scalar per (head, token) multiplies that token's Q, K, V rows
  kscore_128k         B=1 H=16 N=131072  d=128 L=3 p=2 k=1536 bf16 iid, K-norm scorer
  sparse64_512k       B=1 H=16 N=524288  d=128 L=5 p=4 k=384  bf16 iid (about 1:64)
  outlier_1m          B=1 H=8  N=1048576 d=128 L=6 p=4 k=1536 bf16 iid, 1% of the
                      positions (uniform, shared by all heads) have Q, K, V rows x4
dY is iid N(0,1) in the input dtype for every workload.

PISA block selection workloads (PISA_WORKLOADS) take Q and K from the same
generators: pisa_small_8k (H=2, N=8192), pisa_128k and pisa_256k (H=16),
all d=128, p=4, blocks of 64, groups of 128, K=8, L = 3, 4, 5, LogNormal(0,0.5)
per token.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

import torch

_TENSORS = {"q": 0, "k": 1, "v": 2, "dy": 3, "scale": 4, "positions": 5}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    L: int
    p: int
    k: int
    dtype: str          # "fp32" or "bf16"
    scorer: str         # "qk_sum", "k" or "q"
    structure: str      # "iid", "lognormal_token" or "outlier_tokens"
    seed: int
    chunk: int = 2048
    selection: str = "parents"  # "parents", "direct" or "nested"

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny_4k_fp32", 1, 1, 4096, 64, 3, 2, 256, "fp32", "qk_sum", "iid", 0),
        Workload("lognorm_32k", 1, 8, 32768, 128, 3, 4, 1536, "bf16", "qk_sum", "lognormal_token", 1),
        Workload("kscore_128k", 1, 16, 131072, 128, 3, 2, 1536, "bf16", "k", "iid", 2),
        Workload("sparse64_512k", 1, 16, 524288, 128, 5, 4, 384, "bf16", "qk_sum", "iid", 3),
        Workload("outlier_1m", 1, 8, 1048576, 128, 6, 4, 1536, "bf16", "qk_sum", "outlier_tokens", 4),
    )
}


@dataclass(frozen=True)
class PisaWorkload:
    """PISA block selection inputs: q, k [B, H, N, d] bf16 drawn by the same
    generators as the Lighthouse workloads (head_inputs / cuda_inputs)."""
    name: str
    B: int
    H: int
    N: int
    d: int
    p: int
    L: int
    block: int
    group: int
    topk: int
    structure: str
    seed: int
    dtype: str = "bf16"

    @property
    def torch_dtype(self):
        return torch.bfloat16

    def with_(self, **kw) -> "PisaWorkload":
        return replace(self, **kw)


# The review of PISA times block selection at 64K, 128K and 256K tokens
# (section 3, Figure 3) without model sizes; these take d = 128, blocks of 64,
# groups of 128 queries, K = 8 kept blocks per level and p = 4, with L chosen
# so the coarsest level has no more blocks than a finer level scores (p K = 32).
# Per-token LogNormal(0, 0.5) scales on the rows give the block scores spread.
PISA_WORKLOADS = {
    w.name: w
    for w in (
        PisaWorkload("pisa_small_8k", 1, 2, 8192, 128, 4, 3, 64, 128, 8, "lognormal_token", 20),
        PisaWorkload("pisa_128k", 1, 16, 131072, 128, 4, 4, 64, 128, 8, "lognormal_token", 21),
        PisaWorkload("pisa_256k", 1, 16, 262144, 128, 4, 5, 64, 128, 8, "lognormal_token", 22),
    )
}


def _stream_seed(seed: int, tensor: str, bh: int) -> int:
    # the torch CPU generator keeps only 32 seed bits: 12 for the seed, 4 for
    # the tensor, 16 for the (batch, head) index
    if not (0 <= seed < 4096 and 0 <= bh < 65536):
        raise ValueError("seed must be < 4096 and B*H <= 65536")
    return (seed << 20) | (_TENSORS[tensor] << 16) | bh


def _cpu_gen(seed: int, tensor: str, bh: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(_stream_seed(seed, tensor, bh))
    return g


def outlier_positions(w: Workload, seed: int | None = None) -> torch.Tensor:
    """Positions whose rows are scaled x4 (shared across heads), sorted."""
    seed = w.seed if seed is None else seed
    n = int(0.01 * w.N)
    perm = torch.randperm(w.N, generator=_cpu_gen(seed, "positions", 0))
    return torch.sort(perm[:n]).values


def head_inputs(w: Workload, bh: int, seed: int | None = None) -> dict:
    """CPU tensors q, k, v, dy of shape [N, d] in the workload dtype for the
    flattened (batch, head) index ``bh``."""
    seed = w.seed if seed is None else seed
    out = {}
    for name in ("q", "k", "v", "dy"):
        out[name] = torch.randn(w.N, w.d, generator=_cpu_gen(seed, name, bh), dtype=torch.float32)
    if w.structure == "lognormal_token":
        z = torch.randn(w.N, generator=_cpu_gen(seed, "scale", bh), dtype=torch.float64)
        c = torch.exp(0.5 * z).to(torch.float32)[:, None]
        for name in ("q", "k", "v"):
            out[name] = out[name] * c
    elif w.structure == "outlier_tokens":
        pos = outlier_positions(w, seed)
        for name in ("q", "k", "v"):
            out[name][pos] *= 4.0
    elif w.structure != "iid":
        raise ValueError(w.structure)
    return {n: t.to(w.torch_dtype).contiguous() for n, t in out.items()}


def cpu_inputs(w: Workload, seed: int | None = None) -> dict:
    """All heads on the CPU, [B, H, N, d] (small workloads only)."""
    heads = [head_inputs(w, bh, seed) for bh in range(w.B * w.H)]
    return {n: torch.stack([h[n] for h in heads]).reshape(w.B, w.H, w.N, w.d) for n in ("q", "k", "v", "dy")}


def cuda_inputs(w: Workload, device="cuda", seed: int | None = None) -> dict:
    """All heads drawn on the GPU, [B, H, N, d] in the workload dtype."""
    seed = w.seed if seed is None else seed
    g = torch.Generator(device=device)
    out = {}
    for name in ("q", "k", "v", "dy"):
        g.manual_seed(_stream_seed(seed, name, 0xFFFF))
        t = torch.empty(w.B, w.H, w.N, w.d, dtype=w.torch_dtype, device=device)
        # draw in fp32 slices of one head to bound the temporary
        for b in range(w.B):
            for h in range(w.H):
                t[b, h] = torch.randn(w.N, w.d, generator=g, device=device, dtype=torch.float32).to(w.torch_dtype)
        out[name] = t
    if w.structure == "lognormal_token":
        g.manual_seed(_stream_seed(seed, "scale", 0xFFFF))
        for b in range(w.B):
            for h in range(w.H):
                z = torch.randn(w.N, generator=g, device=device, dtype=torch.float32)
                c = torch.exp(0.5 * z)[:, None]
                for name in ("q", "k", "v"):
                    out[name][b, h] = (out[name][b, h].float() * c).to(w.torch_dtype)
    elif w.structure == "outlier_tokens":
        pos = outlier_positions(w, seed).to(device)
        for name in ("q", "k", "v"):
            out[name][:, :, pos] = (out[name][:, :, pos].float() * 4.0).to(w.torch_dtype)
    return out
