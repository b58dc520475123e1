"""Throughput of one Lighthouse attention layer, forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = lh_forward + lh_backward of one layer (all heads) over one batch of
seeded synthetic inputs already resident in HBM.  The default workload is the
512K-token layer (B=1, H=16, d=128, L=5, p=4, k=384, S=8192).  Each rank runs
its own layer (weak scaling, no collective on the data path); the step time is
the max over ranks of CUDA-event time on the launching stream.  Rank 0 prints
one JSON line.

--impl reference times the fp64 CPU oracle (the only other implementation of
the layer) on the host cores, one head per step, on rank 0 only.

--workload pisa_128k (or pisa_small_8k, pisa_256k) times the second workload
instead: one step = lh_pisa_pool_keys + lh_pisa_select over all heads (PISA
block selection), same timing rules, its own metric.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from hierarchical_sparse_attention_pyramid_b200 import _lib, pisa, synth  # noqa: E402
from hierarchical_sparse_attention_pyramid_b200 import api as lh  # noqa: E402

METRIC = "Lighthouse attn fwd+bwd tokens/s/layer at N=512K on 1 B200; % of roofline"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
# the kernels each stage entry point launches (names as the ncu launch list shows them)
STAGE_KERNELS = {"pool": ["pool_kernel", "pool_pairs_kernel"], "score_topk": ["score_pyramid_kernel", "topk_kernel"],
                 "gather": ["gather_kernel"], "attn_fwd": ["attn_fwd_kernel"],
                 "scatter_back": ["scatter_back_kernel", "scatter_back_stream_kernel"],
                 "scatter_adjoint": ["scatter_adjoint_kernel"], "attn_bwd": ["attn_bwd_kv_kernel", "attn_bwd_q_kernel"],
                 "pool_adjoint": ["pool_adjoint_kernel"]}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ distributed

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while running: NVML
    every 5 ms when pynvml can open the device, else nvidia-smi every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, gpu_index: int, period_s: float = 0.005):
        self.gpu = gpu_index
        self.period = period_s
        self.proc = None
        self.lines = []
        self.samples = []  # (sm_mhz, reasons bitmask) from NVML
        self.thread = None
        self.stop_evt = threading.Event()
        self.nvml = None
        self.max_mhz = None
        self.recording = False

    def window(self, on: bool):
        """NVML samples are kept only inside the window (the timed region)."""
        self.recording = on

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
        except Exception:  # noqa: BLE001
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self.stop_evt.is_set():
                    if self.recording:
                        try:
                            self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                                 int(get_reasons(h))))
                        except Exception:  # noqa: BLE001
                            pass
                    time.sleep(self.period)

            self.nvml = nv
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:  # noqa: BLE001
            self.nvml = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:  # noqa: BLE001
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nvml is not None:
            self.stop_evt.set()
            self.thread.join(timeout=2)
            sm = [c for c, _ in self.samples]
            reasons = sorted(n for n, bit in self.REASON_BITS.items() if any(r & bit for _, r in self.samples))
            return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "samples": len(sm), "source": f"NVML every {self.period * 1e3:.0f} ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:  # noqa: BLE001
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi every 200 ms"}


# ------------------------------------------------------------------ stage-by-stage timing

def _vp(base: int, off: int = 0):
    return ctypes.c_void_p(base + off)


def stage_calls(layer: lh.Layer, bufs: lh.Buffers, x: dict, y, grads):
    """The eight stage entry points in lh_forward/lh_backward order, with the
    arguments lh_forward uses (the pool and gather at the plan's first_level),
    on the same buffers, so each kernel of the step can be timed alone."""
    I = bufs.info
    cfg = layer.cfg()
    c = bufs.ctx.data_ptr()
    w = bufs.ws.data_ptr()
    q, k, v, dy = (x[n].data_ptr() for n in ("q", "k", "v", "dy"))
    dq, dk, dv = (g.data_ptr() for g in grads)
    st = lambda: ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)  # noqa: E731
    S = ctypes.c_int64(I.S)
    first = ctypes.c_int32(I.first_level)  # the levels lh_forward materialises
    call = _lib.call
    return [
        ("pool", lambda: call("lh_pyramid_pool_from", ctypes.byref(cfg), first, _vp(q), _vp(k), _vp(v),
                              _vp(w, I.ws_off_pyr_q), _vp(w, I.ws_off_pyr_k), _vp(w, I.ws_off_pyr_v),
                              _vp(w, I.ws_off_norms), st())),
        ("score_topk", lambda: call("lh_score_topk", ctypes.byref(cfg), _vp(w, I.ws_off_norms), _vp(w, I.ws_off_topk),
                                    _vp(c, I.ctx_off_sel), st())),
        ("gather", lambda: call("lh_gather_from", ctypes.byref(cfg), first, _vp(q), _vp(k), _vp(v),
                                _vp(w, I.ws_off_pyr_q),
                                _vp(w, I.ws_off_pyr_k), _vp(w, I.ws_off_pyr_v), _vp(c, I.ctx_off_sel),
                                _vp(c, I.ctx_off_qs), _vp(c, I.ctx_off_ks), _vp(c, I.ctx_off_vs),
                                _vp(c, I.ctx_off_seq_map), _vp(c, I.ctx_off_slot_of), st())),
        ("attn_fwd", lambda: call("lh_attn_fwd", ctypes.byref(cfg), S, _vp(c, I.ctx_off_qs), _vp(c, I.ctx_off_ks),
                                  _vp(c, I.ctx_off_vs), _vp(c, I.ctx_off_os), _vp(c, I.ctx_off_lse), _vp(w), st())),
        ("scatter_back", lambda: call("lh_scatter_back", ctypes.byref(cfg), _vp(c, I.ctx_off_os),
                                      _vp(c, I.ctx_off_slot_of), _vp(y.data_ptr()), st())),
        ("scatter_adjoint", lambda: call("lh_scatter_back_adjoint", ctypes.byref(cfg), _vp(dy), _vp(c, I.ctx_off_seq_map),
                                         _vp(c, I.ctx_off_os), _vp(w, I.ws_off_dos), _vp(w, I.ws_off_delta), st())),
        ("attn_bwd", lambda: call("lh_attn_bwd", ctypes.byref(cfg), S, _vp(c, I.ctx_off_qs), _vp(c, I.ctx_off_ks),
                                  _vp(c, I.ctx_off_vs), _vp(c, I.ctx_off_lse), _vp(w, I.ws_off_dos),
                                  _vp(w, I.ws_off_delta), _vp(w, I.ws_off_dqs), _vp(w, I.ws_off_dks),
                                  _vp(w, I.ws_off_dvs), _vp(w), st())),
        ("pool_adjoint", lambda: call("lh_pool_adjoint", ctypes.byref(cfg), _vp(w, I.ws_off_dqs), _vp(w, I.ws_off_dks),
                                      _vp(w, I.ws_off_dvs), _vp(c, I.ctx_off_slot_of), _vp(dq), _vp(dk), _vp(dv),
                                      st())),
    ]


def stage_work(layer: lh.Layer, info) -> dict:
    """Algorithmic bytes (HBM stages) or flops (attention) of one launch over the whole layer."""
    e = 2 if layer.dtype == "bf16" else 4
    BH, N, d, S = layer.BH, layer.N, layer.d, info.S
    U, E = info.upper_entries, info.pyr_entries
    L, p, first = layer.L, layer.p, info.first_level
    # pyramid rows the pool writes (levels >= first) and rows the gather reads:
    # a kept entry of a level below first is the mean of its p^l level-0 rows
    U_first = sum(info.level_len[lvl] for lvl in range(first, L)) if L > 1 else 0
    kept = [p * info.kprime[lvl] for lvl in range(L - 1)] + [info.level_len[L - 1]] if L > 1 else [N]
    read_rows = sum(n * (p ** lvl if 1 <= lvl < first else 1) for lvl, n in enumerate(kept))
    return {
        "pool": ("hbm", 3 * BH * N * d * e),
        "score_topk": ("hbm", 2 * BH * N * 4 + 2 * BH * U * 4 + BH * info.sel_per_head * 4),
        "gather": ("hbm", 3 * BH * read_rows * d * e + 3 * BH * S * d * 2 + BH * S * 4 + BH * E * 4),
        "attn_fwd": ("tensor", 2 * S * S * d * BH),
        "scatter_back": ("hbm", BH * N * d * e + BH * S * d * 2 + BH * E * 4),
        "scatter_adjoint": ("hbm", BH * N * d * e + 2 * BH * S * d * 2 + BH * S * 8),
        "attn_bwd": ("tensor", 5 * S * S * d * BH),
        "pool_adjoint": ("hbm", 3 * BH * N * d * e + 3 * BH * S * d * 4 + BH * E * 4),
    }


def stage_extra_bytes(layer: lh.Layer, info) -> dict:
    """Bytes a stage moves beyond its algorithmic figure: the pool's writes of
    the pyramid levels >= first_level and of the level-0 norms."""
    e = 2 if layer.dtype == "bf16" else 4
    L, first = layer.L, info.first_level
    U_first = sum(info.level_len[lvl] for lvl in range(first, L)) if L > 1 else 0
    return {"pool": 3 * layer.BH * U_first * layer.d * e + 2 * layer.BH * layer.N * 4}


def stage_clocks(calls, gpu: int, seconds: float = 0.25) -> dict:
    """Median SM clock while each stage call runs back to back for about
    `seconds` (NVML samples every 5 ms): the clock a kernel settles at under
    its own power draw, which a whole-step sample averages away."""
    out = {}
    st = torch.cuda.current_stream()
    for n, f in calls:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        f()
        b.record(st)
        torch.cuda.synchronize()
        reps = max(1, int(seconds * 1e3 / max(a.elapsed_time(b), 1e-3)))
        smp = ClockSampler(gpu)
        smp.start()
        if smp.nvml is None:
            smp.stop()
            return {}
        smp.window(True)
        for _ in range(reps):
            f()
        torch.cuda.synchronize()
        smp.window(False)
        c = smp.stop()
        out[n] = {"sm_mhz": c["sm_mhz"], "reasons": c["reasons"], "samples": c["samples"]}
    return out


def time_stages(calls, iters: int) -> dict:
    """Average CUDA-event duration of each stage call on the current stream."""
    st = torch.cuda.current_stream()
    evs = {n: [] for n, _ in calls}
    for _ in range(iters):
        for n, f in calls:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            f()
            b.record(st)
            evs[n].append((a, b))
    torch.cuda.synchronize()
    return {n: float(np.mean([a.elapsed_time(b) for a, b in v])) for n, v in evs.items()}


def source_sha(kernel: str) -> str:
    files = {"pool": "lh_pool.cu", "pool_adjoint": "lh_pool.cu", "score_topk": "lh_select.cu",
             "gather": "lh_gather.cu", "scatter_back": "lh_gather.cu", "scatter_adjoint": "lh_gather.cu",
             "attn_fwd": "lh_attn_fwd.cu", "attn_bwd": "lh_attn_bwd.cu", "select": "lh_pisa.cu",
             "pool_keys": "lh_pisa.cu"}
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hierarchical_sparse_attention_pyramid_b200", "csrc")
    for f in (files[kernel], "lh_common.cuh", "sm100.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        ent = t.get(workload, {}).get(kernel)
        if ent and ent.get("source_sha") == source_sha(kernel):
            return ent["dram_bytes_per_launch"]
    except Exception:  # noqa: BLE001
        pass
    return None


# ------------------------------------------------------------------ CPU oracle

def oracle_sample(w: synth.Workload, heads: int = 1, max_seconds: float = 60.0) -> dict:
    """fp64 oracle forward + backward on `heads` head(s) of the workload; returns seconds per head."""
    from oracle import lighthouse_oracle as lo
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    times = []
    for h in range(heads):
        x = synth.head_inputs(w, h)
        arr = {n: t.double().numpy() for n, t in x.items()}
        t0 = time.perf_counter()
        Y, sv = lo.forward_head(arr["q"], arr["k"], arr["v"], w.p, w.L, w.k, w.chunk, w.scorer,
                                selection=w.selection)
        lo.backward_head(arr["dy"], sv)
        times.append(time.perf_counter() - t0)
        if sum(times) > max_seconds:
            break
    return {"sec_per_head": float(np.mean(times)), "heads": len(times), "cores": cores}


def run_reference(args, world, rank):
    """The fp64 oracle on the host cores: each step is one head's forward +
    backward of the timed workload (a bounded sample of the layer), timed by
    wall clock.  ms_per_step is that measured step; value extrapolates it to
    the layer (all heads).  Nothing here loads the CUDA library: S comes from
    the oracle's own size formula."""
    if rank != 0:
        return
    from oracle import lighthouse_oracle as lo
    w = synth.WORKLOADS[args.workload]
    if args.selection != "parents":
        w = w.with_(selection=args.selection)
    # warm-up steps run the same one-head sample (at most 2: the oracle keeps
    # no state between steps, so they only load code paths and caches)
    for _ in range(min(args.warmup, 2)):
        oracle_sample(w, 1)
    r_times = []
    cores = None
    for s in range(args.steps):
        r = oracle_sample(w, 1)
        r_times.append(r["sec_per_head"])
        cores = r["cores"]
    sec_step = float(np.mean(r_times))
    sec_layer = sec_step * w.B * w.H
    value = w.B * w.N / sec_layer
    sample = f"one of {w.B * w.H} heads per step (fp64 forward + backward), extrapolated to the layer"
    S = lo.gathered_length(w.N, w.p, w.L, w.k, w.selection)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, S),
        "layer_extrapolation": {"heads_per_step": 1, "heads_per_layer": w.B * w.H, "ms_per_layer": sec_layer * 1e3,
                                "warmup_steps_run": min(args.warmup, 2)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w: synth.Workload, S: int) -> dict:
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "L": w.L, "p": w.p, "k": w.k,
            "chunk": w.chunk, "scorer": w.scorer, "selection": w.selection, "S": int(S),
            "parallelism": "replicas (one layer per GPU)",
            "l2": "inputs larger than L2 (Q,K,V,dY %.1f GB per GPU)" % (4 * w.B * w.H * w.N * w.d * 2 / 1e9)}


# ------------------------------------------------------------------ PISA block selection

PISA_METRIC = "PISA block selection tokens/s (key pyramid + coarse-to-fine LSE top-K, all heads) on 1 B200"
# ex2 results per clock per SM: 4 per SM sub-partition (the special-function
# unit rate of sm_100), 4 sub-partitions
MUFU_EX2_PER_CLK_SM = 16
SMS = 148


def pisa_of(w) -> pisa.Pisa:
    return pisa.Pisa(w.B, w.H, w.N, w.d, w.p, w.L, w.block, w.group, w.topk)


def pisa_config(w) -> dict:
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "p": w.p, "L": w.L, "block": w.block,
            "group": w.group, "topk": w.topk, "structure": w.structure,
            "parallelism": "replicas (one selection per GPU)",
            "l2": ("inputs larger than L2" if 2 * w.B * w.H * w.N * w.d * 2 > 126e6 else "inputs smaller than L2")
                  + " (Q, K %.2f GB per GPU); key blocks are re-read from L2 by design" % (2 * w.B * w.H * w.N * w.d * 2 / 1e9)}


def pisa_scored_candidates(w, idx) -> int:
    """Candidate blocks the selection kernel scores (loads and multiplies):
    every visible block of the coarsest level, then every visible sub-block of
    the blocks kept one level up, summed over groups, levels and heads."""
    G, C, p, L = w.group, w.block, w.p, w.L
    n_groups = w.N // G
    last = (torch.arange(n_groups, device=idx.device, dtype=torch.int64) + 1) * G - 1   # [n_groups]
    n_top = w.N // (C * p ** (L - 1))
    b = torch.arange(n_top, device=idx.device, dtype=torch.int64)
    total = int((((b[None, :] * C + 1) * p ** (L - 1) - 1) <= last[:, None]).sum()) * w.B * w.H
    for lv in range(L - 2, -1, -1):
        kept = idx[:, :, lv + 1, :].long()                                   # [BH, n_groups, K]
        sub = kept[..., None] * p + torch.arange(p, device=idx.device)      # [BH, n_groups, K, p]
        vis = (kept[..., None] >= 0) & (((sub * C + 1) * p ** lv - 1) <= last[None, :, None, None])
        total += int(vis.sum())
    return total


def pisa_oracle_sample(w, max_seconds: float = 20.0) -> dict:
    """fp64 oracle on a bounded sample: head 0's key pyramid plus as many of
    its groups (spread over the sequence) as fit in max_seconds; returns
    seconds per group (the pyramid's time spread over the head's groups)."""
    from oracle import pisa_oracle as po
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    h = synth.head_inputs(w, 0)
    Q, K = h["q"].double().numpy(), h["k"].double().numpy()
    n_groups = w.N // w.group
    t0 = time.perf_counter()
    levels = po.key_pyramid(K, w.p, w.L)
    t_pyr = time.perf_counter() - t0
    order = np.random.default_rng(0).permutation(n_groups)
    t_sel, done = 0.0, 0
    for g in order:
        t0 = time.perf_counter()
        po.select_group(Q, levels, int(g), w.group, w.block, w.p, w.L, w.topk)
        t_sel += time.perf_counter() - t0
        done += 1
        if t_pyr + t_sel > max_seconds:
            break
    per_group = t_sel / done + t_pyr / n_groups
    return {"sec_per_group": per_group, "groups": done, "cores": cores,
            "sample": f"head 0: key pyramid + {done} of {n_groups} groups (random order), fp64, scaled to "
                      f"{w.B * w.H} heads x {n_groups} groups"}


def run_pisa_reference(args, world, rank):
    if rank != 0:
        return
    w = synth.PISA_WORKLOADS[args.workload]
    total_groups = w.B * w.H * (w.N // w.group)
    budget = max(5.0, 150.0 / max(1, args.steps + min(args.warmup, 1)))
    secs, cores, sample = [], None, ""
    for _ in range(min(args.warmup, 1)):
        pisa_oracle_sample(w, 2.0)
    for _ in range(args.steps):
        r = pisa_oracle_sample(w, budget)
        secs.append(r["sec_per_group"] * total_groups)
        cores, sample = r["cores"], r["sample"]
    sec = float(np.mean(secs))
    value = w.B * w.N / sec
    print(json.dumps({
        "impl": "reference", "metric": PISA_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": pisa_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)


def run_pisa(args, world, rank, local):
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.PISA_WORKLOADS[args.workload]
    if args.heads:
        w = w.with_(H=args.heads)
    sel = pisa_of(w)
    info = pisa.plan(sel)
    x = synth.cuda_inputs(w, dev, seed=w.seed + 16 * rank)
    q, k = x["q"], x["k"]
    del x
    kpyr = torch.empty((sel.BH, max(info.upper_entries, 1), w.d), dtype=torch.bfloat16, device=dev)
    shp = (sel.BH, info.n_groups, w.L, w.topk)
    out = (torch.empty(shp, dtype=torch.int32, device=dev), torch.empty(shp, dtype=torch.float32, device=dev))
    ws = torch.zeros(_lib.ERR_WORD_BYTES, dtype=torch.uint8, device=dev)

    def step():
        pisa.pool_keys(sel, k, kpyr)
        pisa.select(sel, q, k, kpyr, out, ws)

    for _ in range(max(args.warmup, 0)):
        step()
    _lib.call("lh_check_error", ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    barrier(world)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    sampler.window(True)
    e0.record(st)
    for _ in range(args.steps):
        step()
    e1.record(st)
    torch.cuda.synchronize()
    sampler.window(False)
    barrier(world)
    clocks = sampler.stop()
    _lib.call("lh_check_error", ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    value = world * w.B * w.N / (ms / 1e3)

    # each kernel alone (same buffers), CUDA events on the launching stream
    stage_ms = time_stages([("pool_keys", lambda: pisa.pool_keys(sel, k, kpyr)),
                            ("select", lambda: pisa.select(sel, q, k, kpyr, out, ws))], max(3, min(args.steps, 10)))
    pk, pk_src = peaks()
    scored = pisa_scored_candidates(w, out[0])
    exps = scored * w.group * w.block
    sm_mhz = pk.get("sm_max_mhz", 1965.0)
    mufu_peak = SMS * MUFU_EX2_PER_CLK_SM * sm_mhz * 1e6 / 1e12   # T ex2 / s
    t_sel = stage_ms["select"] / 1e3
    mma_flops = 2.0 * exps * w.d
    roofline = {"bound": "alu", "kernel": "select", "kernels": ["pisa_select_kernel"],
                "achieved": exps / t_sel / 1e12, "peak": mufu_peak, "unit": "T ex2/s",
                "frac": exps / t_sel / 1e12 / mufu_peak, "traffic": measured_traffic("select", w.name), "peak_source":
                f"derived: {SMS} SMs x {MUFU_EX2_PER_CLK_SM} ex2/clk x {sm_mhz:.0f} MHz",
                "scored_blocks": scored, "exp_per_block": w.group * w.block,
                "tensor": {"achieved_tflops": mma_flops / t_sel / 1e12, "peak": pk["bf16_tflops"],
                           "frac": mma_flops / t_sel / 1e12 / pk["bf16_tflops"]},
                "share_of_step": stage_ms["select"] / sum(stage_ms.values())}
    pool_bytes = sel.BH * w.N * w.d * 2 + sel.BH * info.upper_entries * w.d * 2
    stages = {"pool_keys": {"ms": stage_ms["pool_keys"], "bound": "hbm",
                            "achieved": pool_bytes / (stage_ms["pool_keys"] / 1e3) / 1e9, "unit": "GB/s",
                            "frac": pool_bytes / (stage_ms["pool_keys"] / 1e3) / 1e9 / pk["hbm_gbs"]},
              "select": {"ms": stage_ms["select"], "bound": "alu", "frac": roofline["frac"]}}

    e2e = None
    if not args.no_e2e:
        hq, hk = q.cpu().pin_memory(), k.cpu().pin_memory()
        hi = torch.empty(shp, dtype=torch.int32).pin_memory()
        hs = torch.empty(shp, dtype=torch.float32).pin_memory()
        dq, dk = torch.empty_like(q), torch.empty_like(k)
        h2d = 2 * q.numel() * 2
        d2h = hi.numel() * 4 + hs.numel() * 4

        def e2e_step():
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            pisa.pool_keys(sel, dk, kpyr)
            pisa.select(sel, dq, dk, kpyr, out, ws)
            hi.copy_(out[0], non_blocking=True)
            hs.copy_(out[1], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        k_e = max(2, min(args.steps, 5))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for _ in range(k_e):
            e2e_step()
        b.record(st)
        torch.cuda.synchronize()
        barrier(world)
        _lib.call("lh_check_error", ctypes.c_void_p(ws.data_ptr()),
                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        ms_e = max_over_ranks(a.elapsed_time(b) / k_e, world, dev)
        e2e = {"value": world * w.B * w.N / (ms_e / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ms_e, "steps": k_e}

    cpu = None
    if not args.no_cpu and rank == 0 and world == 1:
        r = pisa_oracle_sample(w, 20.0)
        sec = r["sec_per_group"] * sel.BH * info.n_groups
        cpu = {"value": w.B * w.N / sec, "unit": UNIT, "cores": r["cores"], "kind": "oracle", "sample": r["sample"]}

    if rank == 0:
        print(json.dumps({
            "metric": PISA_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": pisa_config(w), "clocks": clocks,
            "e2e": e2e, "gpu_launches": 2 * args.steps, "roofline": roofline, "stages": stages,
            "cpu_baseline": cpu}), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ one attention stage alone

def run_stage(args, world, rank, local):
    """The S-token attention of the workload alone (its B*H and S), on seeded
    N(0,1) bf16 sequences: a small-memory run of the tensor-core kernels at
    their full launch shape, for timing and for ncu captures.  Prints one
    JSON line with the stage's time and its fraction of the bf16 peak."""
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        w = w.with_(H=args.heads)
    layer = lh.Layer.of(w)
    S = lh.plan(layer).S
    BH, d = layer.BH, w.d
    g = torch.Generator(device=dev).manual_seed(1234 + rank)
    qs, ks, vs, dos = (torch.randn(BH, S, d, generator=g, device=dev).to(torch.bfloat16) for _ in range(4))
    ws = torch.zeros(_lib.ERR_WORD_BYTES, dtype=torch.uint8, device=dev)
    os_, lse = lh.attn_fwd(layer, qs, ks, vs, ws)
    dos = dos.to(torch.float16)  # the backward takes dOs as fp16 holding bf16 values (exact)
    delta = (dos.float() * os_).sum(-1)
    calls = {"attn_fwd": lambda: lh.attn_fwd(layer, qs, ks, vs, ws),
             "attn_bwd": lambda: lh.attn_bwd(layer, qs, ks, vs, lse, dos, delta, ws)}
    f = calls[args.stage]
    for _ in range(max(args.warmup, 1)):
        f()
    _lib.call("lh_check_error", ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    sampler = ClockSampler(local)
    sampler.start()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    sampler.window(True)
    e0.record(st)
    for _ in range(args.steps):
        f()
    e1.record(st)
    torch.cuda.synchronize()
    sampler.window(False)
    barrier(world)
    clocks = sampler.stop()
    _lib.call("lh_check_error", ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    flops = (2 if args.stage == "attn_fwd" else 5) * S * S * d * BH
    pk, pk_src = peaks()
    tf = flops / (ms / 1e3) / 1e12
    if rank == 0:
        print(json.dumps({"stage": args.stage, "workload": w.name, "BH": BH, "S": S, "d": d, "ms": ms,
                          "tflops": tf, "frac_burst": tf / pk["bf16_tflops"],
                          "frac_sustained": tf / pk["bf16_tflops_sustained"], "peak_source": pk_src,
                          "clocks": clocks, "steps": args.steps, "n_gpus": world}), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 200 for the GPU arms, about 1 s at 512K; 20 for --impl reference, "
                         "one oracle head per step)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="sparse64_512k", choices=sorted(synth.WORKLOADS) + sorted(synth.PISA_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-stage-clocks", action="store_true")
    ap.add_argument("--stage", choices=["attn_fwd", "attn_bwd"], default=None,
                    help="time only this attention stage of the workload (its B*H and S, random sequences)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with this many heads instead (a smaller cut for profiling)")
    ap.add_argument("--selection", default="parents", choices=["parents", "direct", "nested"],
                    help="what a level keeps (the default reading, or one of the two others)")
    args = ap.parse_args()

    if args.steps is None:
        args.steps = 20 if args.impl == "reference" else 200
    world, rank, local = dist_setup()
    if args.workload in synth.PISA_WORKLOADS:
        if args.impl == "reference":
            run_pisa_reference(args, world, rank)
        else:
            run_pisa(args, world, rank, local)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    if args.stage:
        run_stage(args, world, rank, local)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        w = w.with_(H=args.heads)
    if args.selection != "parents":
        w = w.with_(selection=args.selection)
    layer = lh.Layer.of(w)
    x = synth.cuda_inputs(w, dev, seed=w.seed + 16 * rank)
    bufs = lh.Buffers(layer, dev)
    shp = (w.B, w.H, w.N, w.d)
    y = torch.empty(shp, dtype=layer.torch_dtype, device=dev)
    grads = tuple(torch.empty(shp, dtype=layer.torch_dtype, device=dev) for _ in range(3))

    def step():
        lh.forward(layer, x["q"], x["k"], x["v"], bufs, y)
        lh.backward(layer, x["dy"], bufs, grads)

    for _ in range(max(args.warmup, 0)):
        step()
    lh.check_error(bufs)
    torch.cuda.synchronize()
    barrier(world)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    sampler.window(True)
    e0.record(st)
    for _ in range(args.steps):
        step()
    e1.record(st)
    torch.cuda.synchronize()
    sampler.window(False)
    barrier(world)
    clocks = sampler.stop()
    lh.check_error(bufs)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    value = world * w.B * w.N / (ms / 1e3)

    # per-stage durations (same buffers, stage entry points one at a time)
    calls = stage_calls(layer, bufs, x, y, grads)
    stage_ms = time_stages(calls, max(3, min(args.steps, 10)))
    lh.check_error(bufs)
    st_clk = stage_clocks(calls, local) if not args.no_stage_clocks else {}
    lh.check_error(bufs)
    pk, pk_src = peaks()
    work = stage_work(layer, bufs.info)
    stages = {}
    for n, t in stage_ms.items():
        kind, amount = work[n]
        if kind == "hbm":
            ach = amount / (t / 1e3) / 1e9
            stages[n] = {"ms": t, "bound": "hbm", "achieved": ach, "unit": "GB/s", "frac": ach / pk["hbm_gbs"]}
        else:
            ach = amount / (t / 1e3) / 1e12
            stages[n] = {"ms": t, "bound": "tensor", "achieved": ach, "unit": "TFLOP/s",
                         "frac": ach / pk["bf16_tflops"]}
        if n in st_clk:
            stages[n]["clock"] = st_clk[n]
    top = max(stage_ms, key=stage_ms.get)
    ts = stages[top]
    roofline = {"bound": ts["bound"], "kernel": top, "kernels": STAGE_KERNELS[top], "achieved": ts["achieved"],
                "peak": pk["hbm_gbs"] if ts["bound"] == "hbm" else pk["bf16_tflops"], "unit": ts["unit"],
                "frac": ts["frac"], "traffic": measured_traffic(top, w.name), "peak_source": pk_src,
                "share_of_step": stage_ms[top] / sum(stage_ms.values()),
                "alg_bytes": work[top][1] if ts["bound"] == "hbm" else None,
                "extra_bytes": stage_extra_bytes(layer, bufs.info).get(top, 0) if ts["bound"] == "hbm" else None}
    # whole-layer roofline: algorithmic bytes (Q,K,V,dY in; Y,dQ,dK,dV out) at the HBM
    # peak plus the attention flops at the tensor peak
    e = 2 if layer.dtype == "bf16" else 4
    alg_bytes = 8 * layer.BH * w.N * w.d * e
    t_roof = alg_bytes / (pk["hbm_gbs"] * 1e9) + (work["attn_fwd"][1] + work["attn_bwd"][1]) / (pk["bf16_tflops"] * 1e12)
    layer_roof = {"t_roof_ms": t_roof * 1e3, "t_meas_ms": ms, "frac": t_roof * 1e3 / ms,
                  "alg_bytes": alg_bytes, "attn_flops": work["attn_fwd"][1] + work["attn_bwd"][1]}

    launches = lh.kernels_per_step(layer)

    # end to end through the C ABI with host buffers: H2D of q,k,v,dy from pinned
    # memory, forward + backward, D2H of y,dq,dk,dv, every step.  Steps are
    # pipelined over two device slots: step i's H2D (copy stream) and step
    # i-1's D2H (another copy stream) run while the GPU computes, so PCIe
    # carries both directions at once; each slot's inputs are overwritten only
    # after the compute that read them, its outputs only after their D2H.
    e2e = None
    if not args.no_e2e:
        hx = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "dy")}
        hout = [torch.empty(shp, dtype=layer.torch_dtype).pin_memory() for _ in range(4)]
        dxs = [{n: torch.empty_like(x[n]) for n in hx} for _ in range(2)]
        outs = [(y, *grads), tuple(torch.empty(shp, dtype=layer.torch_dtype, device=dev) for _ in range(4))]
        h2d = sum(t.numel() * t.element_size() for t in hx.values())
        d2h = sum(t.numel() * t.element_size() for t in hout)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_cmp, ev_out = [None, None], [None, None]

        def e2e_step(i):
            b = i & 1
            dx, o = dxs[b], outs[b]
            with torch.cuda.stream(s_in):
                if ev_cmp[b] is not None:
                    s_in.wait_event(ev_cmp[b])  # the compute of step i-2 has read these inputs
                for n in hx:
                    dx[n].copy_(hx[n], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            st.wait_event(ev_in)
            if ev_out[b] is not None:
                st.wait_event(ev_out[b])  # step i-2's outputs have reached the host
            lh.forward(layer, dx["q"], dx["k"], dx["v"], bufs, o[0])
            lh.backward(layer, dx["dy"], bufs, o[1:])
            ev_cmp[b] = torch.cuda.Event()
            ev_cmp[b].record(st)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[b])
                for t, src in zip(hout, o):
                    t.copy_(src, non_blocking=True)
                ev_out[b] = torch.cuda.Event()
                ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier(world)
        k_e = max(2, min(args.steps, 8))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        s_in.wait_event(a)  # the first H2D starts inside the timed region
        for i in range(k_e):
            e2e_step(i)
        for ev in ev_out:
            st.wait_event(ev)  # the last D2H ends inside it
        b.record(st)
        torch.cuda.synchronize()
        barrier(world)
        lh.check_error(bufs)
        ms_e = max_over_ranks(a.elapsed_time(b) / k_e, world, dev)
        e2e = {"value": world * w.B * w.N / (ms_e / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ms_e, "steps": k_e,
               "pipelined": "H2D of step i and D2H of step i-1 overlap the compute (two device slots)"}
        del hx, hout, dxs, outs

    dense = None
    if not args.no_dense and rank == 0 and world == 1:
        dense = dense_sdpa(x, ms, stage_ms)

    cpu = None
    if not args.no_cpu and rank == 0 and world == 1:
        r = oracle_sample(w, 1)
        sec_layer = r["sec_per_head"] * w.B * w.H
        cpu = {"value": w.B * w.N / sec_layer, "unit": UNIT, "cores": r["cores"], "kind": "oracle",
               "sample": f"one of {w.B * w.H} heads, fp64 forward + backward ({r['sec_per_head']:.1f} s), scaled to the layer"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp32", "data": "synthetic",
            "config": workload_config(w, bufs.info.S), "clocks": clocks, "e2e": e2e, "gpu_launches": launches * args.steps,
            "roofline": roofline, "layer_roofline": layer_roof, "stages": stages, "cpu_baseline": cpu,
            "dense_sdpa": dense,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def dense_sdpa(x, lh_ms, stage_ms):
    """Dense causal attention over all N tokens (cuDNN SDPA) for the speedup figure."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    q, k, v, dy = (x[n] for n in ("q", "k", "v", "dy"))
    try:
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION]):
            def fwd():
                return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
            fwd()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fwd()
            b.record()
            torch.cuda.synchronize()
            t_fwd = a.elapsed_time(b)
            qq, kk, vv = (t.detach().requires_grad_(True) for t in (q, k, v))
            o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True)
            o.backward(dy)
            torch.cuda.synchronize()
            a.record()
            o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, is_causal=True)
            o.backward(dy)
            b.record()
            torch.cuda.synchronize()
            t_fb = a.elapsed_time(b)
        lh_fwd = sum(stage_ms[n] for n in ("pool", "score_topk", "gather", "attn_fwd", "scatter_back"))
        return {"backend": "cudnn", "fwd_ms": t_fwd, "fwdbwd_ms": t_fb, "speedup_fwd": t_fwd / lh_fwd,
                "speedup_fwdbwd": t_fb / lh_ms}
    except Exception as ex:  # noqa: BLE001
        return {"error": str(ex)[:200]}


if __name__ == "__main__":
    main()
